// fa_fwd_ws.cuh — forward for d <= 128 with a split softmax and two alternating
// output accumulators (bf16 and FP8 e4m3 inputs).
//
// Same mathematics as fa_fwd.cuh: S = Q K^T, exp2 online softmax that rescales the
// output only when a row max rises, O += P V, causal tiles above the diagonal
// skipped, persistent heaviest-first schedule.  What differs is how the work is laid
// out on the SM so that the tensor core never waits for a round trip:
//
//  * Two S buffers: S(j+1) is computed while the softmax works on S(j).
//  * Two O accumulators, O_0 for even and O_1 for odd key steps.  The MMA warp issues
//    ... S(j), P(j-1)V, S(j+1), P(j)V ..., and tcgen05 operations complete in order,
//    so "S(j) is ready" implies "P(j-2)V, the last product into O_{j%2}, is done": the
//    softmax rescales O_{j%2} (when its reference max is stale) without waiting for
//    any P V.  The epilogue adds the two: O = O_0 2^(r_0 - m) + O_1 2^(r_1 - m).
//  * Eight softmax warps: two per TMEM lane quadrant, each owning 64 of the 128
//    score columns (and half of O's columns) of its 32 rows; the two halves of a row
//    exchange their partial maxima through shared memory and a two-warp mbarrier.
//
// Roles: warps 0-7 softmax (warp w: lanes 32*(w%4).., column half w/4), warp 8 TMA
// producer, warp 9 MMA issuer + TMEM owner, warps 10-11 idle (warpgroup alignment).
// Tensor memory: S_0 [0,128), S_1 [128,256), O_0 [256,256+D), O_1 [256+D,256+2D).
#pragma once

#include <type_traits>

#include "fa_fwd.cuh"

namespace fa {

template <int D_, int KST_, int VST_, bool FP8_, int EMU_ = 1, int EMU_MQ_ = EMU_, bool SPLIT_ = false,
          bool INDEP_ = false, int TAU_ = 0>
struct WSCfg {
  static constexpr int D = D_;
  static constexpr int BN = 128;
  static constexpr int BM = 128;
  static constexpr int KST = KST_, VST = VST_;
  static constexpr bool FP8 = FP8_;
  static constexpr int EMU = EMU_;
  static constexpr int EMU_MQ = EMU_MQ_;             // same, for the MMA warp's quadrant
  // Issue S = Q K^T and O += P V from two warps on different SM sub-partitions: a
  // sub-partition's instruction queue holds each tcgen05.mma until the tensor core
  // takes it, so one issuing warp delays the softmax warps beside it.
  static constexpr bool SPLIT = SPLIT_;
  // Independent row halves: each half-warp keeps its own running max and sum and its
  // own output accumulator O_h (h = column half of the scores), so the two halves of a
  // row never wait for each other inside the key loop; they are combined once per tile.
  static constexpr bool INDEP = INDEP_;
  // bf16, independent halves only: a row's reference max moves (and O_h is rescaled)
  // only when the row max exceeds it by more than TAU (log2 units), so P <= 2^TAU.  O is
  // then normalised by the sum of the bf16-ROUNDED probabilities, the very values the
  // P V product uses, so the largest probability (no longer exactly 1) carries no
  // rounding bias into O; the logsumexp uses the unrounded sum.
  static constexpr float TAU = FP8 ? 0.f : static_cast<float>(TAU_);
  static constexpr int HALF = BN / 2;                 // score columns per softmax warp
  static constexpr int DH = D / 2;                    // output columns per softmax warp
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int ROW_BYTES = D * ELEM;
  static constexpr int NBOX = ROW_BYTES / 128;
  static constexpr int BOX_ELEMS = 128 / ELEM;
  static constexpr int Q_BYTES = BM * ROW_BYTES;
  static constexpr int KV_BYTES = BN * ROW_BYTES;
  static constexpr int MMA_K = FP8 ? 32 : 16;
  static constexpr int KSTEP_BYTES = MMA_K * ELEM;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = Q_BYTES;
  static constexpr int SMEM_V = SMEM_K + KST * KV_BYTES;
  // exchange slots between the two half-warps of a row: [3][2 half][128 rows] fp32 --
  // slots 0/1 for the row maxima of even/odd steps, slot 2 for the final row sums
  static constexpr int SMEM_X = SMEM_V + VST * KV_BYTES;
  static constexpr int SMEM_BAR = SMEM_X + 3 * 2 * 128 * 4;
  // B_XCHG + quad: barrier of the two half-warps sharing a lane quadrant (one arrival each)
  static constexpr int B_QFULL = 0, B_QEMPTY = 1, B_SFULL = 2, B_PFULL = 4, B_ODONE = 6,
                       B_DRAIN = 7, B_XCHG = 8, B_KFULL = 12, B_KEMPTY = 12 + KST,
                       B_VFULL = 12 + 2 * KST, B_VEMPTY = 12 + 2 * KST + VST,
                       B_PVDONE = 12 + 2 * KST + 2 * VST, B_DRAIN2 = B_PVDONE + 2,
                       B_PFULLH = B_DRAIN2 + 1,          // + 2 * half + buffer, 4 warps each
                       B_PVDONEH = B_PFULLH + 4,         // + half
                       NBARS = B_PVDONEH + 2;
  static constexpr int SMEM_MISC = SMEM_BAR + NBARS * 8;
  static constexpr int SMEM_ALLOC = SMEM_MISC + 64 + 1024;
  static constexpr int TM_S = 0;                      // + b * BN
  static constexpr int TM_O = 2 * BN;                 // + a * D
  static constexpr int TM_COLS = 512;
  static constexpr int THREADS = 384;
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9, PV_WARP = 10;
  static_assert(2 * BN + 2 * D <= TM_COLS, "tensor memory budget");
  static_assert(!(SPLIT && INDEP), "one issuer layout at a time");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(DH % 32 == 0, "32-column output chunks per warp");
};

// ---------------------------------------------------------------- MMA helpers
// Issued by a whole warp; one elected lane executes each tcgen05.mma.
template <class C>
__device__ __forceinline__ void ws_issue_s(uint32_t s_tmem, uint64_t qdesc, uint64_t kdesc) {
  constexpr uint32_t IDESC_S = C::FP8 ? idesc_e4m3(128, C::BN, false) : idesc_bf16(128, C::BN, false);
#pragma unroll
  for (int kb = 0; kb < C::D / C::MMA_K; ++kb) {
    const int box = (kb * C::KSTEP_BYTES) / 128, off = (kb * C::KSTEP_BYTES) % 128;
    umma_ss_elect(C::FP8, s_tmem, qdesc + static_cast<uint64_t>((box * C::BM * 128 + off) >> 4),
                  kdesc + static_cast<uint64_t>((box * C::BN * 128 + off) >> 4), IDESC_S,
                  kb > 0 ? 1u : 0u);
  }
}
template <class C>
__device__ __forceinline__ void ws_issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint64_t vdesc,
                                            bool first) {
  constexpr uint32_t IDESC_O = C::FP8 ? idesc_e4m3(128, C::D, true) : idesc_bf16(128, C::D, true);
#pragma unroll
  for (int kb = 0; kb < C::BN / C::MMA_K; ++kb)
    umma_ts_elect(C::FP8, o_tmem, p_tmem + kb * (C::MMA_K * C::ELEM / 4),
                  vdesc + static_cast<uint64_t>((kb * C::MMA_K * 128) >> 4), IDESC_O,
                  (first && kb == 0) ? 0u : 1u);
}

// ---------------------------------------------------------------- producer (whole warp)
// The warp runs the loop together; one elected lane posts each expected byte count and
// issues the copies.
template <class C>
__device__ void ws_producer(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                            const FwdParams& p, uint32_t sbase, uint32_t bars, const WaitCtl& wc) {
  const uint32_t b_qfull = bars + 8u * C::B_QFULL, b_qempty = bars + 8u * C::B_QEMPTY;
  const uint32_t b_kfull = bars + 8u * C::B_KFULL, b_kempty = bars + 8u * C::B_KEMPTY;
  const uint32_t b_vfull = bars + 8u * C::B_VFULL, b_vempty = bars + 8u * C::B_VEMPTY;
  uint32_t gk = 0, gv = 0, t = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int w = fwd_item_index(k);
    if (w >= p.total_items) break;
    int bh, qt;
    fwd_decode_item(p, w, bh, qt);
    const int n = fwd_num_kv_tiles<C>(p, qt);
    if (t > 0 && !mbar_wait_warp(b_qempty, (t - 1) & 1, wc, kSiteQEmpty)) { ok = false; break; }
    if (elect_one()) {
      mbar_arrive_expect_tx(b_qfull, C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < C::NBOX; ++c)
        tma_load_3d(sbase + C::SMEM_Q + c * C::BM * 128, tq, b_qfull, c * C::BOX_ELEMS, qt * C::BM, bh);
    }
    __syncwarp();
    ++t;
    // MMA consumption order: K_0, then (K_j, V_{j-1}) for j >= 1, then V_{n-1}
    for (int j = 0; j <= n; ++j) {
      if (j < n) {
        const uint32_t s = gk % C::KST;
        if (gk >= C::KST &&
            !mbar_wait_warp(b_kempty + 8u * s, ((gk / C::KST) - 1) & 1, wc, kSiteKVEmpty)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(b_kfull + 8u * s, C::KV_BYTES);
#pragma unroll
          for (int c = 0; c < C::NBOX; ++c)
            tma_load_3d(sbase + C::SMEM_K + s * C::KV_BYTES + c * C::BN * 128, tk, b_kfull + 8u * s,
                        c * C::BOX_ELEMS, j * C::BN, fwd_kv_head(p, bh));
        }
        __syncwarp();
        ++gk;
      }
      if (j > 0) {
        const uint32_t s = gv % C::VST;
        if (gv >= C::VST &&
            !mbar_wait_warp(b_vempty + 8u * s, ((gv / C::VST) - 1) & 1, wc, kSiteKVEmpty)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(b_vfull + 8u * s, C::KV_BYTES);
#pragma unroll
          for (int c = 0; c < C::NBOX; ++c)
            tma_load_3d(sbase + C::SMEM_V + s * C::KV_BYTES + c * C::BN * 128, tv, b_vfull + 8u * s,
                        c * C::BOX_ELEMS, (j - 1) * C::BN, fwd_kv_head(p, bh));
        }
        __syncwarp();
        ++gv;
      }
    }
  }
  if (!ok) {
    if (t > 0) mbar_wait_drain(b_qfull, (t - 1) & 1, 100000000ull);
    for (uint32_t i = (gk > C::KST ? gk - C::KST : 0); i < gk; ++i)
      mbar_wait_drain(b_kfull + 8u * (i % C::KST), (i / C::KST) & 1, 100000000ull);
    for (uint32_t i = (gv > C::VST ? gv - C::VST : 0); i < gv; ++i)
      mbar_wait_drain(b_vfull + 8u * (i % C::VST), (i / C::VST) & 1, 100000000ull);
    return;
  }
  if (t > 0) ok = mbar_wait_warp(b_qempty, (t - 1) & 1, wc, kSiteQEmpty);
  for (uint32_t i = (gk > C::KST ? gk - C::KST : 0); ok && i < gk; ++i)
    ok = mbar_wait_warp(b_kempty + 8u * (i % C::KST), (i / C::KST) & 1, wc, kSiteKVEmpty);
  for (uint32_t i = (gv > C::VST ? gv - C::VST : 0); ok && i < gv; ++i)
    ok = mbar_wait_warp(b_vempty + 8u * (i % C::VST), (i / C::VST) & 1, wc, kSiteKVEmpty);
}

// ---------------------------------------------------------------- MMA issuer (whole warp)
template <class C>
__device__ void ws_mma(const FwdParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                       const WaitCtl& wc) {
  const uint32_t b_qfull = bars + 8u * C::B_QFULL, b_qempty = bars + 8u * C::B_QEMPTY;
  const uint32_t b_sfull = bars + 8u * C::B_SFULL, b_pfull = bars + 8u * C::B_PFULL;
  const uint32_t b_odone = bars + 8u * C::B_ODONE;
  const uint32_t b_kfull = bars + 8u * C::B_KFULL, b_kempty = bars + 8u * C::B_KEMPTY;
  const uint32_t b_vfull = bars + 8u * C::B_VFULL, b_vempty = bars + 8u * C::B_VEMPTY;
  const uint64_t qdesc = sdesc_sw128(sbase + C::SMEM_Q, 16, 1024);
  const uint64_t kdesc_base = sdesc_sw128(sbase + C::SMEM_K, 16, 1024);
  const uint64_t vdesc_base = sdesc_sw128(sbase + C::SMEM_V, C::BN * 128, 1024);
  uint32_t g = 0, t = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int w = fwd_item_index(k);
    if (w >= p.total_items) break;
    int bh, qt;
    fwd_decode_item(p, w, bh, qt);
    const int n = fwd_num_kv_tiles<C>(p, qt);
    if (!mbar_wait_warp(b_qfull, t & 1, wc, kSiteQFull)) { ok = false; break; }
    tc_fence_after();
    for (int j = 0; j <= n; ++j) {
      const uint32_t gj = g + j;
      if (j < n) {
        // S(j) into S_{gj%2}: the buffer's previous P was read by a P V issued earlier
        const uint32_t ks = gj % C::KST;
        if (!mbar_wait_warp(b_kfull + 8u * ks, (gj / C::KST) & 1, wc, kSiteKFull)) { ok = false; break; }
        tc_fence_after();
        ws_issue_s<C>(tmem + C::TM_S + (gj & 1) * C::BN, qdesc,
                      kdesc_base + static_cast<uint64_t>(ks * (C::KV_BYTES >> 4)));
        tc_commit_elect(b_kempty + 8u * ks);
        tc_commit_elect(b_sfull + 8u * (gj & 1));
        if (j == n - 1) tc_commit_elect(b_qempty);
      }
      if (j > 0) {
        // P(j-1) V into O_{(j-1)%2}; each accumulator is overwritten on its first use
        const uint32_t gp = gj - 1;
        const uint32_t vs = gp % C::VST;
        if (!mbar_wait_warp(b_pfull + 8u * (gp & 1), (gp >> 1) & 1, wc, kSitePFull)) { ok = false; break; }
        if (!mbar_wait_warp(b_vfull + 8u * vs, (gp / C::VST) & 1, wc, kSiteVFull)) { ok = false; break; }
        tc_fence_after();
        ws_issue_pv<C>(tmem + C::TM_O + ((j - 1) & 1) * C::D, tmem + C::TM_S + (gp & 1) * C::BN,
                       vdesc_base + static_cast<uint64_t>(vs * (C::KV_BYTES >> 4)), j - 1 < 2);
        tc_commit_elect(b_vempty + 8u * vs);
        if (j == n) tc_commit_elect(b_odone);
      }
    }
    if (!ok) break;
    g += n;
    ++t;
  }
  tc_commit_elect(bars + 8u * C::B_DRAIN);
  if (!mbar_wait_drain(bars + 8u * C::B_DRAIN, 0, wc.timeout_ns) && (threadIdx.x & 31) == 0)
    atomicCAS(wc.status, 0u, kStatusTimeout | kSiteDrain);
}

// ---------------------------------------------------------------- split issuers
// S issuer (the TMEM owner's warp).  S(j) reuses the buffer of S(j-2), whose P the
// product P(j-2) V reads: S(j) is issued only once that product is complete, which
// also keeps "S(j) complete => P(j-2) V complete" true for the softmax warps.
template <class C>
__device__ void ws_mma_s(const FwdParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                         const WaitCtl& wc) {
  const uint32_t b_qfull = bars + 8u * C::B_QFULL, b_qempty = bars + 8u * C::B_QEMPTY;
  const uint32_t b_sfull = bars + 8u * C::B_SFULL, b_pvdone = bars + 8u * C::B_PVDONE;
  const uint32_t b_kfull = bars + 8u * C::B_KFULL, b_kempty = bars + 8u * C::B_KEMPTY;
  const uint64_t qdesc = sdesc_sw128(sbase + C::SMEM_Q, 16, 1024);
  const uint64_t kdesc_base = sdesc_sw128(sbase + C::SMEM_K, 16, 1024);
  uint32_t g = 0, t = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int w = fwd_item_index(k);
    if (w >= p.total_items) break;
    int bh, qt;
    fwd_decode_item(p, w, bh, qt);
    const int n = fwd_num_kv_tiles<C>(p, qt);
    if (!mbar_wait_warp(b_qfull, t & 1, wc, kSiteQFull)) { ok = false; break; }
    for (int j = 0; j < n; ++j) {
      const uint32_t gj = g + j;
      const uint32_t ks = gj % C::KST;
      if (!mbar_wait_warp(b_kfull + 8u * ks, (gj / C::KST) & 1, wc, kSiteKFull)) { ok = false; break; }
      if (gj >= 2 && !mbar_wait_warp(b_pvdone + 8u * (gj & 1), ((gj - 2) >> 1) & 1, wc, kSitePFull)) {
        ok = false;
        break;
      }
      tc_fence_after();
      ws_issue_s<C>(tmem + C::TM_S + (gj & 1) * C::BN, qdesc,
                    kdesc_base + static_cast<uint64_t>(ks * (C::KV_BYTES >> 4)));
      tc_commit_elect(b_kempty + 8u * ks);
      tc_commit_elect(b_sfull + 8u * (gj & 1));
      if (j == n - 1) tc_commit_elect(b_qempty);
    }
    if (!ok) break;
    g += n;
    ++t;
  }
  tc_commit_elect(bars + 8u * C::B_DRAIN);
  if (!mbar_wait_drain(bars + 8u * C::B_DRAIN, 0, wc.timeout_ns) && (threadIdx.x & 31) == 0)
    atomicCAS(wc.status, 0u, kStatusTimeout | kSiteDrain);
}

// P V issuer: P(j) V into O_{j%2}; each accumulator is overwritten on its first use.
template <class C>
__device__ void ws_mma_pv(const FwdParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                          const WaitCtl& wc) {
  const uint32_t b_pfull = bars + 8u * C::B_PFULL, b_pvdone = bars + 8u * C::B_PVDONE;
  const uint32_t b_odone = bars + 8u * C::B_ODONE;
  const uint32_t b_vfull = bars + 8u * C::B_VFULL, b_vempty = bars + 8u * C::B_VEMPTY;
  const uint64_t vdesc_base = sdesc_sw128(sbase + C::SMEM_V, C::BN * 128, 1024);
  uint32_t g = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int w = fwd_item_index(k);
    if (w >= p.total_items) break;
    int bh, qt;
    fwd_decode_item(p, w, bh, qt);
    const int n = fwd_num_kv_tiles<C>(p, qt);
    for (int j = 0; j < n; ++j) {
      const uint32_t gp = g + j;
      const uint32_t vs = gp % C::VST;
      if (!mbar_wait_warp(b_pfull + 8u * (gp & 1), (gp >> 1) & 1, wc, kSitePFull)) { ok = false; break; }
      if (!mbar_wait_warp(b_vfull + 8u * vs, (gp / C::VST) & 1, wc, kSiteVFull)) { ok = false; break; }
      tc_fence_after();
      ws_issue_pv<C>(tmem + C::TM_O + (j & 1) * C::D, tmem + C::TM_S + (gp & 1) * C::BN,
                     vdesc_base + static_cast<uint64_t>(vs * (C::KV_BYTES >> 4)), j < 2);
      tc_commit_elect(b_vempty + 8u * vs);
      tc_commit_elect(b_pvdone + 8u * (gp & 1));
      if (j == n - 1) tc_commit_elect(b_odone);
    }
    if (!ok) break;
    g += n;
  }
  tc_commit_elect(bars + 8u * C::B_DRAIN2);
  if (!mbar_wait_drain(bars + 8u * C::B_DRAIN2, 0, wc.timeout_ns) && (threadIdx.x & 31) == 0)
    atomicCAS(wc.status, 0u, kStatusTimeout | kSiteDrain);
}

// Scale this warp's half of an output accumulator row by `a` (one TMEM round trip).
template <class C>
__device__ __forceinline__ void ws_scale_o(uint32_t taddr, float a) {
  uint32_t r[C::DH];
  if constexpr (C::DH == 64) {
    tmem_ld64(taddr, r);
    tmem_ld_wait64(r);
  } else {
    tmem_ld32(taddr, r);
    tmem_ld_wait(r);
  }
  const uint64_t a2 = f2_pack(a, a);
#pragma unroll
  for (int i = 0; i < C::DH; i += 2) {
    float x, y;
    f2_unpack(f2_mul(f2_pack(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), a2), x, y);
    r[i] = __float_as_uint(x);
    r[i + 1] = __float_as_uint(y);
  }
  if constexpr (C::DH == 64)
    tmem_st64(taddr, r);
  else
    tmem_st32(taddr, r);
}

// ---------------------------------------------------------------- softmax warps
template <class C>
__device__ void ws_softmax(const FwdParams& p, uint32_t bars, uint32_t tmem, float* xbuf,
                           const WaitCtl& wc) {
  const int warp = threadIdx.x / 32;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + (threadIdx.x & 31);
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const uint32_t b_sfull = bars + 8u * C::B_SFULL, b_pfull = bars + 8u * C::B_PFULL;
  const uint32_t b_odone = bars + 8u * C::B_ODONE;
  // The two half-warps of a row trade a value through shared memory and this pair's
  // barrier: arrive (release) after the store, bounded wait (acquire), then load.  A
  // warp cannot run a phase ahead: each wait needs the partner's arrival.
  const uint32_t b_x = bars + 8u * (C::B_XCHG + quad);
  uint32_t xc = 0;                                    // exchanges done by this warp
  const float LOG2E = 1.4426950408889634f;
  const float LN2 = 0.6931471805599453f;
  const float sl2 = p.scale * LOG2E;
  __nv_bfloat16* o_out = reinterpret_cast<__nv_bfloat16*>(p.o);
  uint32_t g = 0, t = 0;
  bool ok = true;

  for (int k = 0; ok; ++k) {
    const int w = fwd_item_index(k);
    if (w >= p.total_items) break;
    int bh, qt;
    fwd_decode_item(p, w, bh, qt);
    const int n = fwd_num_kv_tiles<C>(p, qt);
    const int q_idx = qt * C::BM + row;
    float m = -INFINITY, l = 0.f;
    float r0 = -INFINITY, r1 = -INFINITY;             // reference max of O_0 / O_1
    float qsc = 1.f, vmax = 1.f;
    if constexpr (C::FP8) {
      qsc = p.q_scale[bh * p.n_st + qt];
      vmax = 0.f;
      for (int j = 0; j < n; ++j) vmax = fmaxf(vmax, p.v_scale[fwd_kv_head(p, bh) * p.n_st + j]);
    }
    for (int j = 0; j < n; ++j) {
      const uint32_t gj = g + j;
      const uint32_t b = gj & 1;
      if (!mbar_wait(b_sfull + 8u * b, (gj >> 1) & 1, wc, kSiteSFull)) { ok = false; break; }
      tc_fence_after();
      float s[C::HALF];
      {
        uint32_t r[C::HALF];
        tmem_ld64(lane_base + C::TM_S + b * C::BN + half * C::HALF, r);
        tmem_ld_wait64(r);
#pragma unroll
        for (int i = 0; i < C::HALF; ++i) s[i] = __uint_as_float(r[i]);
      }
      const int kv0 = j * C::BN + half * C::HALF;
      const bool need_mask = (p.causal && j * C::BN + C::BN - 1 > qt * C::BM) || (j * C::BN + C::BN > p.N);
      if (need_mask) {
        const int lim = p.causal ? min(q_idx, p.N - 1) : p.N - 1;
#pragma unroll
        for (int c = 0; c < C::HALF; ++c)
          if (kv0 + c > lim) s[c] = -INFINITY;
      }
      float c_j = sl2, fold = 1.f;
      if constexpr (C::FP8) {
        c_j = sl2 * qsc * p.k_scale[fwd_kv_head(p, bh) * p.n_st + j];
        fold = 256.f * p.v_scale[fwd_kv_head(p, bh) * p.n_st + j] / vmax;
      }
      float mx[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) mx[i] = fmaxf(s[2 * i], s[2 * i + 1]);
#pragma unroll
      for (int c = 8; c < C::HALF; c += 8)
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = max3f(mx[i], s[c + 2 * i], s[c + 2 * i + 1]);
      float mine = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      // exchange with the other half of the row (slot by step parity, so a fast warp
      // never overwrites a value its partner has not read yet)
      xbuf[(b * 2 + half) * 128 + row] = mine;
      mbar_arrive_warp(b_x);
      if (!mbar_wait(b_x, xc & 1, wc, kSiteXchg)) { ok = false; break; }
      ++xc;
      const float other = xbuf[(b * 2 + (half ^ 1)) * 128 + row];
      const float m_cand = fmaxf(mine, other) * c_j;
      const bool raise = m_cand > m;
      const float m_new = raise ? m_cand : m;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = raise ? ex2(m - m_use) : 1.f;
      const uint64_t c2 = f2_pack(c_j, c_j);
      const uint64_t nm2 = f2_pack(-m_use, -m_use);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      auto exps = [&](auto emu_tag) {
        constexpr int kEmu = decltype(emu_tag)::value;
#pragma unroll
        for (int c = 0; c < C::HALF; c += 2) {
          const uint64_t x2 = f2_fma(f2_pack(s[c], s[c + 1]), c2, nm2);
          uint64_t p2;
          if ((c / 2) % 4 < kEmu) {
            p2 = ex2_poly_pair(x2);
          } else {
            float xa, xb;
            f2_unpack(x2, xa, xb);
            p2 = f2_pack(ex2(xa), ex2(xb));
          }
          acc[(c / 2) % 4] = f2_add(acc[(c / 2) % 4], p2);
          f2_unpack(p2, s[c], s[c + 1]);
        }
      };
      if (need_mask)
        exps(std::integral_constant<int, 0>{});
      else if (quad == (C::MMA_WARP & 3))
        exps(std::integral_constant<int, C::EMU_MQ>{});
      else
        exps(std::integral_constant<int, C::EMU>{});
      float sa, sb;
      f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), sa, sb);
      l = l * alpha + (sa + sb);           // this half's share of the row sum
      if constexpr (C::FP8) {
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          r[i] = pack_e4m3x4(s[4 * i] * fold, s[4 * i + 1] * fold, s[4 * i + 2] * fold,
                             s[4 * i + 3] * fold);
        tmem_st16(lane_base + C::TM_S + b * C::BN + half * 16, r);
      } else {
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = pack_bf16x2(s[2 * i], s[2 * i + 1]);
        tmem_st32(lane_base + C::TM_S + b * C::BN + half * 32, r);
      }
      // Rescale the accumulator this step adds to: its last product, P(j-2) V, is
      // complete because S(j) is.  Done after P is stored, when the score row no longer
      // occupies registers.  Warp-uniform decision (TMEM access is per warp).
      {
        float& ra = (j & 1) ? r1 : r0;
        const bool stale = j >= 2 && ra != m_use;
        if (__any_sync(0xffffffffu, stale))
          ws_scale_o<C>(lane_base + C::TM_O + (j & 1) * C::D + half * C::DH,
                        stale ? ex2(ra - m_use) : 1.f);
        ra = m_use;
      }
      m = m_new;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(b_pfull + 8u * b);
    }
    if (!ok) break;
    // epilogue: both accumulators complete (the last commit tracks every earlier MMA)
    if (!mbar_wait(b_odone, t & 1, wc, kSiteODone)) { ok = false; break; }
    ++t;
    tc_fence_after();
    // total row sum = both halves' shares (each already relative to the final m)
    xbuf[(4 + half) * 128 + row] = l;
    mbar_arrive_warp(b_x);
    if (!mbar_wait(b_x, xc & 1, wc, kSiteXchg)) { ok = false; break; }
    ++xc;
    const float l_row = l + xbuf[(4 + (half ^ 1)) * 128 + row];
    const float m_fin = (m == -INFINITY) ? 0.f : m;
    const float inv_l = (C::FP8 ? vmax * (1.f / 256.f) : 1.f) / l_row;
    const float w0 = ex2(r0 - m_fin) * inv_l;
    const float w1 = n >= 2 ? ex2(r1 - m_fin) * inv_l : 0.f;
    const bool row_ok = q_idx < p.N;
    __nv_bfloat16* orow = o_out + (static_cast<size_t>(bh) * p.N + q_idx) * p.ld + half * C::DH;
#pragma unroll 1
    for (int c = 0; c < C::DH; c += 32) {
      uint32_t a0[32], a1[32];
      tmem_ld32(lane_base + C::TM_O + half * C::DH + c, a0);
      tmem_ld_wait(a0);
      if (n >= 2) {
        tmem_ld32(lane_base + C::TM_O + C::D + half * C::DH + c, a1);
        tmem_ld_wait(a1);
      }
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float x0 = __uint_as_float(a0[2 * i]) * w0, y0 = __uint_as_float(a0[2 * i + 1]) * w0;
        if (n >= 2) {
          x0 = fmaf(__uint_as_float(a1[2 * i]), w1, x0);
          y0 = fmaf(__uint_as_float(a1[2 * i + 1]), w1, y0);
        }
        pk[i] = pack_bf16x2(x0, y0);
      }
      if (row_ok && half * C::DH + c < p.ld) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
    if (half == 0 && row_ok && p.lse != nullptr)
      p.lse[static_cast<size_t>(bh) * p.N + q_idx] = (m_fin + __log2f(l_row)) * LN2;
    tc_fence_before();
    g += n;
  }
}

// ---------------------------------------------------------------- independent halves
// P_h(j) V_h into O_h, h = 0, 1: the key block of half h is keys [64h, 64h + 64) of the
// tile; its probabilities sit at columns [64h, 64h + P_COLS_H) of the S buffer, inside
// the columns that half's own scores occupied.
template <class C>
__device__ __forceinline__ void ws_issue_pv_half(uint32_t o_tmem, uint32_t s_tmem, uint64_t vdesc,
                                                 int h, bool first) {
  constexpr uint32_t IDESC_O = C::FP8 ? idesc_e4m3(128, C::D, true) : idesc_bf16(128, C::D, true);
  constexpr int KB_H = C::HALF / C::MMA_K;                  // MMAs per half
#pragma unroll
  for (int i = 0; i < KB_H; ++i) {
    const int kb = h * KB_H + i;
    umma_ts_elect(C::FP8, o_tmem, s_tmem + h * C::HALF + i * (C::MMA_K * C::ELEM / 4),
                  vdesc + static_cast<uint64_t>((kb * C::MMA_K * 128) >> 4), IDESC_O,
                  (first && i == 0) ? 0u : 1u);
  }
}

template <class C>
__device__ void ws_mma_indep(const FwdParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                             const WaitCtl& wc) {
  const uint32_t b_qfull = bars + 8u * C::B_QFULL, b_qempty = bars + 8u * C::B_QEMPTY;
  const uint32_t b_sfull = bars + 8u * C::B_SFULL, b_pfullh = bars + 8u * C::B_PFULLH;
  const uint32_t b_pvdoneh = bars + 8u * C::B_PVDONEH, b_odone = bars + 8u * C::B_ODONE;
  const uint32_t b_kfull = bars + 8u * C::B_KFULL, b_kempty = bars + 8u * C::B_KEMPTY;
  const uint32_t b_vfull = bars + 8u * C::B_VFULL, b_vempty = bars + 8u * C::B_VEMPTY;
  const uint64_t qdesc = sdesc_sw128(sbase + C::SMEM_Q, 16, 1024);
  const uint64_t kdesc_base = sdesc_sw128(sbase + C::SMEM_K, 16, 1024);
  const uint64_t vdesc_base = sdesc_sw128(sbase + C::SMEM_V, C::BN * 128, 1024);
  uint32_t g = 0, t = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int w = fwd_item_index(k);
    if (w >= p.total_items) break;
    int bh, qt;
    fwd_decode_item(p, w, bh, qt);
    const int n = fwd_num_kv_tiles<C>(p, qt);
    if (!mbar_wait_warp(b_qfull, t & 1, wc, kSiteQFull)) { ok = false; break; }
    tc_fence_after();
    for (int j = 0; j <= n; ++j) {
      const uint32_t gj = g + j;
      if (j < n) {
        // S(j) into S_{gj%2}: the P V products that read the buffer's last P were
        // issued earlier by this thread and complete first
        const uint32_t ks = gj % C::KST;
        if (!mbar_wait_warp(b_kfull + 8u * ks, (gj / C::KST) & 1, wc, kSiteKFull)) { ok = false; break; }
        tc_fence_after();
        ws_issue_s<C>(tmem + C::TM_S + (gj & 1) * C::BN, qdesc,
                      kdesc_base + static_cast<uint64_t>(ks * (C::KV_BYTES >> 4)));
        tc_commit_elect(b_kempty + 8u * ks);
        tc_commit_elect(b_sfull + 8u * (gj & 1));
        if (j == n - 1) tc_commit_elect(b_qempty);
      }
      if (j > 0) {
        const uint32_t gp = gj - 1;
        const uint32_t vs = gp % C::VST;
        const uint32_t pb = gp & 1, pph = (gp >> 1) & 1;
        if (!mbar_wait_warp(b_vfull + 8u * vs, (gp / C::VST) & 1, wc, kSiteVFull)) { ok = false; break; }
        const uint64_t vdesc = vdesc_base + static_cast<uint64_t>(vs * (C::KV_BYTES >> 4));
        const uint32_t s_tmem = tmem + C::TM_S + pb * C::BN;
        if (j == 1) {
          // first products of a tile overwrite both accumulators: wait until both
          // halves are past the previous tile's epilogue, which reads both
          if (!mbar_wait_warp(b_pfullh + 8u * pb, pph, wc, kSitePFull) ||
              !mbar_wait_warp(b_pfullh + 8u * (2 + pb), pph, wc, kSitePFull)) {
            ok = false;
            break;
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (j > 1 && !mbar_wait_warp(b_pfullh + 8u * (2 * h + pb), pph, wc, kSitePFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          ws_issue_pv_half<C>(tmem + C::TM_O + h * C::D, s_tmem, vdesc, h, j == 1);
          tc_commit_elect(b_pvdoneh + 8u * h);
        }
        if (!ok) break;
        tc_commit_elect(b_vempty + 8u * vs);
        if (j == n) tc_commit_elect(b_odone);
      }
    }
    if (!ok) break;
    g += n;
    ++t;
  }
  tc_commit_elect(bars + 8u * C::B_DRAIN);
  if (!mbar_wait_drain(bars + 8u * C::B_DRAIN, 0, wc.timeout_ns) && (threadIdx.x & 31) == 0)
    atomicCAS(wc.status, 0u, kStatusTimeout | kSiteDrain);
}

// Scale a full output accumulator row (D columns) of this warp's lanes by `a`, in
// 32-column pieces.
template <class C>
__device__ __forceinline__ void ws_scale_o_full(uint32_t taddr, float a) {
  const uint64_t a2 = f2_pack(a, a);
#pragma unroll 1
  for (int c = 0; c < C::D; c += 64) {
    uint32_t r[64];
    tmem_ld64(taddr + c, r);
    tmem_ld_wait64(r);
#pragma unroll
    for (int i = 0; i < 64; i += 2) {
      float x, y;
      f2_unpack(f2_mul(f2_pack(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), a2), x, y);
      r[i] = __float_as_uint(x);
      r[i + 1] = __float_as_uint(y);
    }
    tmem_st64(taddr + c, r);
  }
}

template <class C>
__device__ void ws_softmax_indep(const FwdParams& p, uint32_t bars, uint32_t tmem, float* xbuf,
                                 const WaitCtl& wc) {
  const int warp = threadIdx.x / 32;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + (threadIdx.x & 31);
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const uint32_t b_sfull = bars + 8u * C::B_SFULL;
  const uint32_t b_pfull = bars + 8u * (C::B_PFULLH + 2 * half);
  const uint32_t b_pvdone = bars + 8u * (C::B_PVDONEH + half);
  const uint32_t b_odone = bars + 8u * C::B_ODONE;
  const uint32_t b_x = bars + 8u * (C::B_XCHG + quad);
  const uint32_t o_mine = lane_base + C::TM_O + half * C::D;
  uint32_t xc = 0;
  const float LOG2E = 1.4426950408889634f;
  const float LN2 = 0.6931471805599453f;
  const float sl2 = p.scale * LOG2E;
  __nv_bfloat16* o_out = reinterpret_cast<__nv_bfloat16*>(p.o);
  uint32_t g = 0, t = 0;
  bool ok = true;

  for (int k = 0; ok; ++k) {
    const int w = fwd_item_index(k);
    if (w >= p.total_items) break;
    int bh, qt;
    fwd_decode_item(p, w, bh, qt);
    const int n = fwd_num_kv_tiles<C>(p, qt);
    const int q_idx = qt * C::BM + row;
    float m = -INFINITY, l = 0.f, lx = 0.f;   // lx: unrounded row sum (TAU > 0)
    float qsc = 1.f, vmax = 1.f;
    if constexpr (C::FP8) {
      qsc = p.q_scale[bh * p.n_st + qt];
      vmax = 0.f;
      for (int j = 0; j < n; ++j) vmax = fmaxf(vmax, p.v_scale[fwd_kv_head(p, bh) * p.n_st + j]);
    }
    for (int j = 0; j < n; ++j) {
      const uint32_t gj = g + j;
      const uint32_t b = gj & 1;
      if (!mbar_wait(b_sfull + 8u * b, (gj >> 1) & 1, wc, kSiteSFull)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_cols = lane_base + C::TM_S + b * C::BN + half * C::HALF;
      float s[C::HALF];
      {
        uint32_t r[C::HALF];
        tmem_ld64(s_cols, r);
        tmem_ld_wait64(r);
#pragma unroll
        for (int i = 0; i < C::HALF; ++i) s[i] = __uint_as_float(r[i]);
      }
      const int kv0 = j * C::BN + half * C::HALF;
      // warp-uniform: some row of this warp has a key of this half beyond its limit
      const bool need_mask = (p.causal && kv0 + C::HALF - 1 > qt * C::BM + quad * 32) ||
                             (kv0 + C::HALF > p.N);
      if (need_mask) {
        const int lim = p.causal ? min(q_idx, p.N - 1) : p.N - 1;
#pragma unroll
        for (int c = 0; c < C::HALF; ++c)
          if (kv0 + c > lim) s[c] = -INFINITY;
      }
      float c_j = sl2, fold = 1.f;
      if constexpr (C::FP8) {
        c_j = sl2 * qsc * p.k_scale[fwd_kv_head(p, bh) * p.n_st + j];
        fold = 256.f * p.v_scale[fwd_kv_head(p, bh) * p.n_st + j] / vmax;
      }
      float mx[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) mx[i] = fmaxf(s[2 * i], s[2 * i + 1]);
#pragma unroll
      for (int c = 8; c < C::HALF; c += 8)
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = max3f(mx[i], s[c + 2 * i], s[c + 2 * i + 1]);
      const float m_cand = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c_j;
      const bool raise = m_cand > m + C::TAU;
      const float m_new = raise ? m_cand : m;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = raise ? ex2(m - m_use) : 1.f;
      const uint64_t c2 = f2_pack(c_j, c_j);
      const uint64_t nm2 = f2_pack(-m_use, -m_use);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      uint64_t accr[4] = {0ull, 0ull, 0ull, 0ull};    // sums of the rounded P (TAU > 0)
      constexpr bool kRounded = C::TAU > 0.f;
      uint32_t pk[kRounded ? C::HALF / 2 : 1];
      auto exps = [&](auto emu_tag) {
        constexpr int kEmu = decltype(emu_tag)::value;
#pragma unroll
        for (int c = 0; c < C::HALF; c += 2) {
          const uint64_t x2 = f2_fma(f2_pack(s[c], s[c + 1]), c2, nm2);
          uint64_t p2;
          if ((c / 2) % 4 < kEmu) {
            p2 = ex2_poly_pair(x2);
          } else {
            float xa, xb;
            f2_unpack(x2, xa, xb);
            p2 = f2_pack(ex2(xa), ex2(xb));
          }
          acc[(c / 2) % 4] = f2_add(acc[(c / 2) % 4], p2);
          if constexpr (kRounded) {
            float pa, pb;
            f2_unpack(p2, pa, pb);
            const uint32_t u = pack_bf16x2(pa, pb);
            pk[c / 2] = u;
            accr[(c / 2) % 4] = f2_add(accr[(c / 2) % 4], f2_pack(__uint_as_float(u << 16),
                                                                   __uint_as_float(u & 0xFFFF0000u)));
          } else {
            f2_unpack(p2, s[c], s[c + 1]);
          }
        }
      };
      if (need_mask)
        exps(std::integral_constant<int, 0>{});
      else if (quad == (C::MMA_WARP & 3))
        exps(std::integral_constant<int, C::EMU_MQ>{});
      else
        exps(std::integral_constant<int, C::EMU>{});
      float sa, sb;
      f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), sa, sb);
      if constexpr (kRounded) {
        float ra, rb;
        f2_unpack(f2_add(f2_add(accr[0], accr[1]), f2_add(accr[2], accr[3])), ra, rb);
        l = l * alpha + (ra + rb);
        lx = lx * alpha + (sa + sb);
      } else {
        l = l * alpha + (sa + sb);
      }
      // P_h(j) over this half's own score columns
      if constexpr (kRounded) {
        tmem_st32(s_cols, *reinterpret_cast<uint32_t(*)[32]>(pk));
      } else if constexpr (C::FP8) {
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          r[i] = pack_e4m3x4(s[4 * i] * fold, s[4 * i + 1] * fold, s[4 * i + 2] * fold,
                             s[4 * i + 3] * fold);
        tmem_st16(s_cols, r);
      } else {
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = pack_bf16x2(s[2 * i], s[2 * i + 1]);
        tmem_st32(s_cols, r);
      }
      // O_h was last updated by P_h(j-1) V_h: once it is complete, scale it to the
      // new reference max (warp-uniform decision; alpha = 1 on rows that kept theirs)
      if (j > 0 && __any_sync(0xffffffffu, raise)) {
        if (!mbar_wait(b_pvdone, (gj - 1) & 1, wc, kSitePvDone)) { ok = false; break; }
        tc_fence_after();
        ws_scale_o_full<C>(o_mine, alpha);
      }
      m = m_new;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(b_pfull + 8u * b);
    }
    if (!ok) break;
    if (!mbar_wait(b_odone, t & 1, wc, kSiteODone)) { ok = false; break; }
    ++t;
    tc_fence_after();
    // combine the halves: O = sum_h O_h 2^(m_h - m), l = sum_h l_h 2^(m_h - m)
    xbuf[half * 128 + row] = m;
    xbuf[(2 + half) * 128 + row] = l;
    if constexpr (C::TAU > 0.f) xbuf[(4 + half) * 128 + row] = lx;
    mbar_arrive_warp(b_x);
    if (!mbar_wait(b_x, xc & 1, wc, kSiteXchg)) { ok = false; break; }
    ++xc;
    const float m_o = xbuf[(half ^ 1) * 128 + row];
    const float l_o = xbuf[(2 + (half ^ 1)) * 128 + row];
    const float m_fin = fmaxf(m, m_o);
    const float m_ref = (m_fin == -INFINITY) ? 0.f : m_fin;
    const float e_me = ex2(((m == -INFINITY) ? m_ref : m) - m_ref) * (m == -INFINITY ? 0.f : 1.f);
    const float e_ot = ex2(((m_o == -INFINITY) ? m_ref : m_o) - m_ref) * (m_o == -INFINITY ? 0.f : 1.f);
    const float l_row = l * e_me + l_o * e_ot;
    // the logsumexp from the unrounded sums (TAU > 0) or the one sum kept
    float lx_row = l_row;
    if constexpr (C::TAU > 0.f) lx_row = lx * e_me + xbuf[(4 + (half ^ 1)) * 128 + row] * e_ot;
    const float inv_l = (C::FP8 ? vmax * (1.f / 256.f) : 1.f) / l_row;
    const float w_self = e_me * inv_l, w_other = e_ot * inv_l;
    const float w0 = half == 0 ? w_self : w_other;
    const float w1 = half == 0 ? w_other : w_self;
    const bool row_ok = q_idx < p.N;
    __nv_bfloat16* orow = o_out + (static_cast<size_t>(bh) * p.N + q_idx) * p.ld + half * C::DH;
#pragma unroll 1
    for (int c = 0; c < C::DH; c += 32) {
      uint32_t a0[32], a1[32];
      tmem_ld32(lane_base + C::TM_O + half * C::DH + c, a0);
      tmem_ld32(lane_base + C::TM_O + C::D + half * C::DH + c, a1);
      tmem_ld_wait(a0);
      tmem_ld_wait(a1);
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float x0 = fmaf(__uint_as_float(a1[2 * i]), w1, __uint_as_float(a0[2 * i]) * w0);
        const float y0 = fmaf(__uint_as_float(a1[2 * i + 1]), w1, __uint_as_float(a0[2 * i + 1]) * w0);
        pk[i] = pack_bf16x2(x0, y0);
      }
      if (row_ok && half * C::DH + c < p.ld) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
    if (half == 0 && row_ok && p.lse != nullptr)
      p.lse[static_cast<size_t>(bh) * p.N + q_idx] = (m_ref + __log2f(lx_row)) * LN2;
    tc_fence_before();
    g += n;
  }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    fa_fwd_ws_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::SMEM_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
  float* xbuf = reinterpret_cast<float*>(smem + C::SMEM_X);
  const int warp = threadIdx.x / 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBARS; ++i) {
      uint32_t cnt = 1;
      if (i == C::B_PFULL || i == C::B_PFULL + 1) cnt = 8;           // the 8 softmax warps
      if (i >= C::B_PFULLH && i < C::B_PFULLH + 4) cnt = 4;           // one column half
      if (i >= C::B_XCHG && i < C::B_XCHG + 4) cnt = 2;               // one half-warp pair
      mbar_init(bars + 8u * i, cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.status, p.timeout_ns};

  if (warp == C::PRODUCER_WARP) {
    ws_producer<C>(&tq, &tk, &tv, p, sbase, bars, wc);
  } else if (warp == C::MMA_WARP) {
    if constexpr (C::SPLIT)
      ws_mma_s<C>(p, sbase, bars, tmem, wc);
    else if constexpr (C::INDEP)
      ws_mma_indep<C>(p, sbase, bars, tmem, wc);
    else
      ws_mma<C>(p, sbase, bars, tmem, wc);
  } else if (C::SPLIT && warp == C::PV_WARP) {
    ws_mma_pv<C>(p, sbase, bars, tmem, wc);
  } else if (warp < 8) {
    if constexpr (C::INDEP)
      ws_softmax_indep<C>(p, bars, tmem, xbuf, wc);
    else
      ws_softmax<C>(p, bars, tmem, xbuf, wc);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

}  // namespace fa
