// fa_fwd_pp.cuh — forward with two query tiles per CTA ("ping-pong"), for d <= 128.
//
// Same mathematics as fa_fwd.cuh (tiled S = Q K^T, exp2 online softmax with the
// output rescaled only when a row max rises, O += P V, causal tile skip), but a
// work item is a PAIR of 128-row query tiles of one head that share every K/V tile
// load, and each tile has its own softmax warps.  The tensor core alternates
// between the tiles:
//
//      ... PV_0(j-1)  S_0(j)  PV_1(j-1)  S_1(j)  PV_0(j)  S_0(j+1) ...
//
// so while one tile's warps turn S_t(j) into P_t(j), the tensor core works on the
// other tile.  Because PV_t(j-1) is issued before S_t(j) and tcgen05 operations
// complete in order, "S_t(j) is ready" also means "PV_t(j-1) has finished": the
// softmax warps may rescale O_t right away, with no separate wait.
//
// Roles: warps 0-3 softmax for tile 0, warps 4-7 softmax for tile 1 (TMEM lane
// quadrant = warp % 4; a thread owns one 128-key score row), warp 8 TMA producer,
// warp 9 MMA issuer + TMEM owner.
// Tensor memory: S_0 [0,128), S_1 [128,256), O_0 [256, 256+D), O_1 [256+D, 256+2D);
// P_t overwrites the first columns of S_t after they are read.
#pragma once

#include "fa_fwd.cuh"

namespace fa {

template <int D_, int KST_, int VST_, bool FP8_, int EMU_ = 0, int TAU_ = 0, int NORM_ = 0>
struct PPCfg {
  static constexpr int D = D_;
  static constexpr int BN = 128;
  static constexpr int BM = 128;                     // rows of one query tile
  static constexpr int KST = KST_, VST = VST_;
  static constexpr bool FP8 = FP8_;
  // Of every 16 pairs of exponentials in a score row, EMU are evaluated by the software
  // exp2 on the FMA/ALU pipes (ex2_poly_pair) instead of the special-function unit, on
  // tiles without masked scores.
  static constexpr int EMU = EMU_;
  // bf16 only: the reference max used for the exponentials moves (and O is rescaled)
  // only when a row max exceeds it by more than TAU (log2 units), so P <= 2^TAU.
  static constexpr float TAU = FP8 ? 0.f : static_cast<float>(TAU_);
  // The row sum that normalises O (bf16 with TAU > 0, where a probability can reach
  // 2^TAU and its bf16 rounding no longer averages out):
  //   NORM 1: the unrounded probabilities plus, per key tile, the bf16 rounding error of
  //           the tile's largest probability;
  //   NORM 2: the bf16-rounded probabilities themselves, the very weights of the P V
  //           product, so O is their convex combination of V rows.
  // The logsumexp always uses the plain unrounded sum.
  static constexpr int NORM = (FP8 || TAU == 0.f) ? 0 : NORM_;
  static constexpr bool COMP = NORM == 1;
  static constexpr bool RSUM = NORM == 2;
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int ROW_BYTES = D * ELEM;
  static constexpr int NBOX = ROW_BYTES / 128;
  static constexpr int BOX_ELEMS = 128 / ELEM;
  static constexpr int QT_BYTES = BM * ROW_BYTES;
  static constexpr int KV_BYTES = BN * ROW_BYTES;
  static constexpr int MMA_K = FP8 ? 32 : 16;
  static constexpr int KSTEP_BYTES = MMA_K * ELEM;
  static constexpr int SMEM_Q = 0;                   // Q_0 then Q_1
  static constexpr int SMEM_K = 2 * QT_BYTES;
  static constexpr int SMEM_V = SMEM_K + KST * KV_BYTES;
  static constexpr int SMEM_BAR = SMEM_V + VST * KV_BYTES;
  // per-tile barriers come in pairs (tile 0, tile 1)
  static constexpr int B_QFULL = 0, B_QEMPTY = 2, B_SFULL = 4, B_PFULL = 6, B_ODONE = 8,
                       B_DRAIN = 10, B_KFULL = 11, B_KEMPTY = 11 + KST, B_VFULL = 11 + 2 * KST,
                       B_VEMPTY = 11 + 2 * KST + VST, NBARS = 11 + 2 * KST + 2 * VST;
  static constexpr int SMEM_MISC = SMEM_BAR + NBARS * 8;
  static constexpr int SMEM_ITEM = SMEM_MISC + 64;    // work-item ring
  static constexpr int SMEM_ALLOC = SMEM_ITEM + kItemBytes + 1024;
  static constexpr int SOFTMAX_WARPS = 8;
  static constexpr uint32_t ITEM_READERS = 1 + SOFTMAX_WARPS;   // the MMA thread and the softmax warps
  static constexpr int TM_S = 0;                     // + t * BN
  static constexpr int TM_O = 2 * BN;                // + t * D
  static constexpr int TM_COLS = 512;
  // 3 warpgroups: two softmax groups and one group holding the producer warp, the
  // MMA warp and two idle warps.  Launch budget 384 x 168 registers = 64,512; the
  // softmax groups take 208 each and the third group 88: 2*128*208 + 128*88 = 64,512
  // (a split with no spills in either role).
  static constexpr int THREADS = 384;
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9;
  static constexpr int REGS_SOFTMAX = 208, REGS_OTHER = 88;
  static constexpr int REGS_TOTAL = 2 * 128 * REGS_SOFTMAX + 128 * REGS_OTHER;
  static_assert(REGS_TOTAL <= THREADS * 168, "register split");
  static_assert(2 * BN + 2 * D <= TM_COLS, "tensor memory budget");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(EMU >= 0 && EMU <= 16, "software exponentials per 16 pairs");
};

// Work item = (head, pair of query tiles).  Same orders as the one-tile kernel:
// non-causal head-major, causal heaviest pair first in L2-sized head groups.
// `n_qt` of FwdParams holds the number of PAIRS per head here.
__device__ __forceinline__ void pp_decode_item(const FwdParams& p, int w, int& bh, int& pr) {
  fwd_decode_item(p, w, bh, pr);
}

template <class C>
__device__ __forceinline__ int pp_kv_tiles(const FwdParams& p, int qt) {
  const int n_qt = (p.N + C::BM - 1) / C::BM;
  if (qt >= n_qt) return 0;
  if (!p.causal) return p.n_kt;
  return min(p.n_kt - 1, ((qt + 1) * C::BM - 1) / C::BN) + 1;
}

// ---------------------------------------------------------------- MMA helpers
// S_t = Q_t K^T (D / MMA_K instructions into S_t) then commit to `sfull`.  The
// descriptors are built once; a K step is a constant start-address offset.
template <class C>
__device__ __forceinline__ void pp_issue_s(uint32_t s_tmem, uint64_t qdesc, uint64_t kdesc,
                                           uint32_t sfull) {
  constexpr uint32_t IDESC_S = C::FP8 ? idesc_e4m3(128, C::BN, false) : idesc_bf16(128, C::BN, false);
#pragma unroll
  for (int kb = 0; kb < C::D / C::MMA_K; ++kb) {
    const int box = (kb * C::KSTEP_BYTES) / 128, off = (kb * C::KSTEP_BYTES) % 128;
    const uint64_t qo = static_cast<uint64_t>((box * C::BM * 128 + off) >> 4);
    const uint64_t ko = static_cast<uint64_t>((box * C::BN * 128 + off) >> 4);
    umma_ss<C::FP8>(s_tmem, qdesc + qo, kdesc + ko, IDESC_S, kb > 0 ? 1u : 0u);
  }
  tc_commit(sfull);
}
// O_t (+)= P_t V: A = P_t from tensor memory, B = V (MN-major) from shared memory.
template <class C>
__device__ __forceinline__ void pp_issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint64_t vdesc,
                                            bool first) {
  constexpr uint32_t IDESC_O = C::FP8 ? idesc_e4m3(128, C::D, true) : idesc_bf16(128, C::D, true);
#pragma unroll
  for (int kb = 0; kb < C::BN / C::MMA_K; ++kb) {
    umma_ts<C::FP8>(o_tmem, p_tmem + kb * (C::MMA_K * C::ELEM / 4), vdesc + static_cast<uint64_t>((kb * C::MMA_K * 128) >> 4),
                    IDESC_O, (first && kb == 0) ? 0u : 1u);
  }
}

// ---------------------------------------------------------------- producer (one thread)
// Straight-line code with scalar state: small per-tile arrays indexed by a loop
// variable end up in local memory, and every barrier wait (a memory clobber) would
// reload them.
template <class C>
__device__ void pp_producer(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                            const FwdParams& p, uint32_t sbase, uint32_t bars, const ItemRing& ring,
                            const WaitCtl& wc) {
  const uint32_t b_qfull0 = bars + 8u * C::B_QFULL, b_qfull1 = b_qfull0 + 8u;
  const uint32_t b_qempty0 = bars + 8u * C::B_QEMPTY, b_qempty1 = b_qempty0 + 8u;
  const uint32_t b_kfull = bars + 8u * C::B_KFULL, b_kempty = bars + 8u * C::B_KEMPTY;
  const uint32_t b_vfull = bars + 8u * C::B_VFULL, b_vempty = bars + 8u * C::B_VEMPTY;
  uint32_t gk = 0, gv = 0, tq0 = 0, tq1 = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    int w;
    if (!(ok = ring.put(p, k, w, wc))) break;
    if (w >= p.total_items) break;
    int bh, pr;
    pp_decode_item(p, w, bh, pr);
    const int n0 = pp_kv_tiles<C>(p, 2 * pr), n1 = pp_kv_tiles<C>(p, 2 * pr + 1);
    const int ns = max(n0, n1);
    if (n0 > 0) {
      if (tq0 > 0 && !mbar_wait(b_qempty0, (tq0 - 1) & 1, wc, kSiteQEmpty)) { ok = false; break; }
      mbar_arrive_expect_tx(b_qfull0, C::QT_BYTES);
#pragma unroll
      for (int c = 0; c < C::NBOX; ++c)
        tma_load_3d(sbase + C::SMEM_Q + c * C::BM * 128, tq, b_qfull0, c * C::BOX_ELEMS,
                    (2 * pr) * C::BM, bh);
      ++tq0;
    }
    if (n1 > 0) {
      if (tq1 > 0 && !mbar_wait(b_qempty1, (tq1 - 1) & 1, wc, kSiteQEmpty)) { ok = false; break; }
      mbar_arrive_expect_tx(b_qfull1, C::QT_BYTES);
#pragma unroll
      for (int c = 0; c < C::NBOX; ++c)
        tma_load_3d(sbase + C::SMEM_Q + C::QT_BYTES + c * C::BM * 128, tq, b_qfull1,
                    c * C::BOX_ELEMS, (2 * pr + 1) * C::BM, bh);
      ++tq1;
    }
    // consumption order of the MMA warp: K_0, then (V_{j-1}, K_j) ..., then V_{ns-1}
    for (int j = 0; j <= ns; ++j) {
      if (j > 0) {
        const uint32_t s = gv % C::VST;
        if (gv >= C::VST && !mbar_wait(b_vempty + 8u * s, ((gv / C::VST) - 1) & 1, wc, kSiteKVEmpty)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(b_vfull + 8u * s, C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < C::NBOX; ++c)
          tma_load_3d(sbase + C::SMEM_V + s * C::KV_BYTES + c * C::BN * 128, tv, b_vfull + 8u * s,
                      c * C::BOX_ELEMS, (j - 1) * C::BN, fwd_kv_head(p, bh));
        ++gv;
      }
      if (j < ns) {
        const uint32_t s = gk % C::KST;
        if (gk >= C::KST && !mbar_wait(b_kempty + 8u * s, ((gk / C::KST) - 1) & 1, wc, kSiteKVEmpty)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(b_kfull + 8u * s, C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < C::NBOX; ++c)
          tma_load_3d(sbase + C::SMEM_K + s * C::KV_BYTES + c * C::BN * 128, tk, b_kfull + 8u * s,
                      c * C::BOX_ELEMS, j * C::BN, fwd_kv_head(p, bh));
        ++gk;
      }
    }
  }
  if (!ok) {
    // Aborted: let the tile copies already issued land before the CTA exits.
    if (tq0 > 0) mbar_wait_drain(b_qfull0, (tq0 - 1) & 1, 100000000ull);
    if (tq1 > 0) mbar_wait_drain(b_qfull1, (tq1 - 1) & 1, 100000000ull);
    for (uint32_t i = (gk > C::KST ? gk - C::KST : 0); i < gk; ++i)
      mbar_wait_drain(b_kfull + 8u * (i % C::KST), (i / C::KST) & 1, 100000000ull);
    for (uint32_t i = (gv > C::VST ? gv - C::VST : 0); i < gv; ++i)
      mbar_wait_drain(b_vfull + 8u * (i % C::VST), (i / C::VST) & 1, 100000000ull);
    return;
  }
  // Drain: every buffer released, so no tensor-core commit is still due when the CTA exits.
  if (tq0 > 0) ok = mbar_wait(b_qempty0, (tq0 - 1) & 1, wc, kSiteQEmpty);
  if (ok && tq1 > 0) ok = mbar_wait(b_qempty1, (tq1 - 1) & 1, wc, kSiteQEmpty);
  for (uint32_t i = (gk > C::KST ? gk - C::KST : 0); ok && i < gk; ++i)
    ok = mbar_wait(b_kempty + 8u * (i % C::KST), (i / C::KST) & 1, wc, kSiteKVEmpty);
  for (uint32_t i = (gv > C::VST ? gv - C::VST : 0); ok && i < gv; ++i)
    ok = mbar_wait(b_vempty + 8u * (i % C::VST), (i / C::VST) & 1, wc, kSiteKVEmpty);
}

// ---------------------------------------------------------------- MMA issuer (one thread)
template <class C>
__device__ void pp_mma(const FwdParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                       const ItemRing& ring, const WaitCtl& wc) {
  const uint32_t b_qfull0 = bars + 8u * C::B_QFULL, b_qfull1 = b_qfull0 + 8u;
  const uint32_t b_qempty0 = bars + 8u * C::B_QEMPTY, b_qempty1 = b_qempty0 + 8u;
  const uint32_t b_sfull0 = bars + 8u * C::B_SFULL, b_sfull1 = b_sfull0 + 8u;
  const uint32_t b_pfull0 = bars + 8u * C::B_PFULL, b_pfull1 = b_pfull0 + 8u;
  const uint32_t b_odone0 = bars + 8u * C::B_ODONE, b_odone1 = b_odone0 + 8u;
  const uint32_t b_kfull = bars + 8u * C::B_KFULL, b_kempty = bars + 8u * C::B_KEMPTY;
  const uint32_t b_vfull = bars + 8u * C::B_VFULL, b_vempty = bars + 8u * C::B_VEMPTY;
  // K-major Q / K tiles: 128-byte swizzled rows, 8-row groups 1024 B apart.  V is the
  // MN-major B operand of P V: LBO = distance between 128-byte column boxes.
  const uint64_t qdesc0 = sdesc_sw128(sbase + C::SMEM_Q, 16, 1024);
  const uint64_t qdesc1 = sdesc_sw128(sbase + C::SMEM_Q + C::QT_BYTES, 16, 1024);
  const uint64_t kdesc_base = sdesc_sw128(sbase + C::SMEM_K, 16, 1024);
  const uint64_t vdesc_base = sdesc_sw128(sbase + C::SMEM_V, C::BN * 128, 1024);
  const uint32_t s0 = tmem + C::TM_S, s1 = tmem + C::TM_S + C::BN;
  const uint32_t o0 = tmem + C::TM_O, o1 = tmem + C::TM_O + C::D;
  uint32_t g = 0, gs0 = 0, gs1 = 0, tq0 = 0, tq1 = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    int w;
    if (!(ok = ring.get(k, w, wc))) break;
    if (w >= p.total_items) break;
    int bh, pr;
    pp_decode_item(p, w, bh, pr);
    const int n0 = pp_kv_tiles<C>(p, 2 * pr), n1 = pp_kv_tiles<C>(p, 2 * pr + 1);
    const int ns = max(n0, n1);
    if (n0 > 0 && !mbar_wait(b_qfull0, tq0 & 1, wc, kSiteQFull)) { ok = false; break; }
    if (n1 > 0 && !mbar_wait(b_qfull1, tq1 & 1, wc, kSiteQFull)) { ok = false; break; }
    tc_fence_after();
    // per step: P_0 V, S_0, P_1 V, S_1 -- each tile's P V before its next S, so the
    // completion of S_t also tells its softmax warps that O_t is up to date
    for (int j = 0; j <= ns; ++j) {
      const uint32_t gk = g + j;
      const uint32_t ks = gk % C::KST;
      const uint32_t vs = (gk + C::VST - 1) % C::VST;   // stage of V_{j-1}
      const uint64_t kdesc = kdesc_base + static_cast<uint64_t>(ks * (C::KV_BYTES >> 4));
      const uint64_t vdesc = vdesc_base + static_cast<uint64_t>(vs * (C::KV_BYTES >> 4));
      if (j > 0 && !mbar_wait(b_vfull + 8u * vs, ((gk - 1) / C::VST) & 1, wc, kSiteVFull)) {
        ok = false;
        break;
      }
      bool k_ready = false;
      // tile 0
      if (j > 0 && j <= n0) {
        if (!mbar_wait(b_pfull0, gs0 & 1, wc, kSitePFull)) { ok = false; break; }
        tc_fence_after();
        pp_issue_pv<C>(o0, s0, vdesc, j == 1);
        ++gs0;
        if (j == n0) tc_commit(b_odone0);
      }
      if (j < n0) {
        if (!mbar_wait(b_kfull + 8u * ks, (gk / C::KST) & 1, wc, kSiteKFull)) { ok = false; break; }
        tc_fence_after();
        k_ready = true;
        pp_issue_s<C>(s0, qdesc0, kdesc, b_sfull0);
        if (j == n0 - 1) tc_commit(b_qempty0);
      }
      // tile 1
      if (j > 0 && j <= n1) {
        if (!mbar_wait(b_pfull1, gs1 & 1, wc, kSitePFull)) { ok = false; break; }
        tc_fence_after();
        pp_issue_pv<C>(o1, s1, vdesc, j == 1);
        ++gs1;
        if (j == n1) tc_commit(b_odone1);
      }
      if (j < n1) {
        if (!k_ready) {
          if (!mbar_wait(b_kfull + 8u * ks, (gk / C::KST) & 1, wc, kSiteKFull)) { ok = false; break; }
          tc_fence_after();
        }
        pp_issue_s<C>(s1, qdesc1, kdesc, b_sfull1);
        if (j == n1 - 1) tc_commit(b_qempty1);
      }
      if (j < ns) tc_commit(b_kempty + 8u * ks);
      if (j > 0) tc_commit(b_vempty + 8u * vs);
    }
    if (!ok) break;
    g += ns;
    tq0 += n0 > 0 ? 1u : 0u;
    tq1 += n1 > 0 ? 1u : 0u;
  }
  // nothing may be in flight when the CTA frees tensor memory
  tc_commit(bars + 8u * C::B_DRAIN);
  if (!mbar_wait_drain(bars + 8u * C::B_DRAIN, 0, wc.timeout_ns))
    atomicCAS(wc.status, 0u, kStatusTimeout | kSiteDrain);
}

// ---------------------------------------------------------------- softmax (one tile)
template <class C>
__device__ void pp_softmax(const FwdParams& p, uint32_t bars, uint32_t tmem, int t, const ItemRing& ring,
                           const WaitCtl& wc) {
  auto bar = [&](int i) { return bars + 8u * i; };
  const int warp = threadIdx.x / 32;
  const int quad = warp & 3;
  const int row = quad * 32 + (threadIdx.x & 31);
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const uint32_t tm_s = C::TM_S + t * C::BN, tm_o = C::TM_O + t * C::D;
  const float LOG2E = 1.4426950408889634f;
  const float LN2 = 0.6931471805599453f;
  const float sl2 = p.scale * LOG2E;
  __nv_bfloat16* o_out = reinterpret_cast<__nv_bfloat16*>(p.o);
  uint32_t gs = 0, ti = 0;   // this tile's steps and items so far
  bool ok = true;

  for (int k = 0; ok; ++k) {
    int w;
    if (!(ok = ring.get_warp(k, w, wc))) break;
    if (w >= p.total_items) break;
    int bh, pr;
    pp_decode_item(p, w, bh, pr);
    const int qt = 2 * pr + t;
    const int n = pp_kv_tiles<C>(p, qt);
    if (n == 0) continue;
    const int q_idx = qt * C::BM + row;
    float m = -INFINITY, l = 0.f;
    float lc = 0.f;                           // row sum that normalises O (COMP, RSUM)
    float qsc = 1.f, vmax = 1.f;
    // FP8: the V tile scales' max, one load per lane per 32 tiles and a warp reduction;
    // the per-step K and V scales are fetched a step ahead, so their load latency
    // overlaps the wait for the scores
    float ksc_n = 1.f, vsc_n = 1.f;
    if constexpr (C::FP8) {
      const float* vs = p.v_scale + fwd_kv_head(p, bh) * p.n_st;
      qsc = p.q_scale[bh * p.n_st + qt];
      vmax = 0.f;
      for (int j = threadIdx.x & 31; j < n; j += 32) vmax = fmaxf(vmax, vs[j]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
      ksc_n = p.k_scale[fwd_kv_head(p, bh) * p.n_st];
      vsc_n = vs[0];
    }
    for (int j = 0; j < n; ++j) {
      const float ksc = ksc_n, vsc = vsc_n;
      if constexpr (C::FP8) {
        if (j + 1 < n) {
          ksc_n = p.k_scale[fwd_kv_head(p, bh) * p.n_st + j + 1];
          vsc_n = p.v_scale[fwd_kv_head(p, bh) * p.n_st + j + 1];
        }
      }
      if (!(ok = mbar_wait(bar(C::B_SFULL + t), gs & 1, wc, kSiteSFull))) break;
      tc_fence_after();
      float s[C::BN];
      {
        uint32_t r[C::BN];
        tmem_ld128(lane_base + tm_s, r);
        tmem_ld_wait128(r);
#pragma unroll
        for (int i = 0; i < C::BN; ++i) s[i] = __uint_as_float(r[i]);
      }
      const int kv0 = j * C::BN;
      const bool need_mask = (p.causal && kv0 + C::BN - 1 > qt * C::BM) || (kv0 + C::BN > p.N);
      if (need_mask) {
        const int lim = p.causal ? min(q_idx, p.N - 1) : p.N - 1;
#pragma unroll
        for (int c = 0; c < C::BN; ++c)
          if (kv0 + c > lim) s[c] = -INFINITY;
      }
      float c_j = sl2, lfold = 0.f, inv_fold = 1.f;
      if constexpr (C::FP8) {
        c_j = sl2 * qsc * ksc;
        // P is stored as P~ * fold, fold = 256 * vsc / vmax (reading of the V-scale
        // folding): the factor enters the exponent, 2^(x + log2 fold), and the row sum
        // takes it out again once per step
        lfold = 8.f + __log2f(vsc / vmax);
        inv_fold = ex2(-lfold);
      }
      // row max: eight independent three-input chains, then a short tree
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = fmaxf(s[2 * i], s[2 * i + 1]);
#pragma unroll
      for (int c = 16; c < C::BN; c += 16)
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = max3f(mx[i], s[c + 2 * i], s[c + 2 * i + 1]);
      const float m_cand = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]),
                                 fmaxf(mx[6], mx[7])) * c_j;
      const bool raise = m_cand > m + C::TAU;
      const float m_new = raise ? m_cand : m;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = raise ? ex2(m - m_use) : 1.f;
      float l_comp = 0.f;
      if constexpr (C::COMP) {
        // the tile's largest probability and its bf16 rounding error
        const float pt = ex2(m_cand - m_use);
        l_comp = __bfloat162float(__float2bfloat16_rn(pt)) - pt;
      }
      const uint64_t c2 = f2_pack(c_j, c_j);
      const uint64_t nm2 = f2_pack(lfold - m_use, lfold - m_use);
      // Exponentials, their row sum, P packing and the P store per 32-key chunk, so
      // that packing and the tensor-memory stores overlap the special-function unit.
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      uint64_t accr[4] = {0ull, 0ull, 0ull, 0ull};   // RSUM: the rounded probabilities
      auto chunks = [&](auto emu_tag) {
        constexpr int kEmu = decltype(emu_tag)::value;
#pragma unroll
        for (int c0 = 0; c0 < C::BN; c0 += 32) {
          float pv[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c = c0 + 2 * i;
            const uint64_t x2 = f2_fma(f2_pack(s[c], s[c + 1]), c2, nm2);
            uint64_t p2;
            if ((((i + 1) * kEmu) / 16) != ((i * kEmu) / 16)) {
              p2 = ex2_poly_pair(x2);
            } else {
              float xa, xb;
              f2_unpack(x2, xa, xb);
              p2 = f2_pack(ex2(xa), ex2(xb));
            }
            acc[i % 4] = f2_add(acc[i % 4], p2);
            f2_unpack(p2, pv[2 * i], pv[2 * i + 1]);
          }
          if constexpr (C::FP8) {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              pk[i] = pack_e4m3x4(pv[4 * i], pv[4 * i + 1], pv[4 * i + 2], pv[4 * i + 3]);
            tmem_st8(lane_base + tm_s + c0 / 4, pk);
          } else {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              pk[i] = pack_bf16x2(pv[2 * i], pv[2 * i + 1]);
              if constexpr (C::RSUM)
                accr[i % 4] = f2_add(accr[i % 4], f2_pack(__uint_as_float(pk[i] << 16),
                                                          __uint_as_float(pk[i] & 0xFFFF0000u)));
            }
            tmem_st16(lane_base + tm_s + c0 / 2, pk);
          }
        }
      };
      if (need_mask)
        chunks(std::integral_constant<int, 0>{});
      else
        chunks(std::integral_constant<int, C::EMU>{});
      float sa, sb;
      f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), sa, sb);
      if constexpr (C::FP8) {
        sa *= inv_fold;
        sb *= inv_fold;
      }
      l = l * alpha + (sa + sb);
      if constexpr (C::COMP) lc = lc * alpha + (sa + sb) + l_comp;
      if constexpr (C::RSUM) {
        float ra, rb;
        f2_unpack(f2_add(f2_add(accr[0], accr[1]), f2_add(accr[2], accr[3])), ra, rb);
        lc = lc * alpha + (ra + rb);
      }
      // S_t(j) ready => P_t(j-1) V has completed, so O_t may be rescaled now (after P
      // is stored, when the score row no longer occupies registers).
      if (j > 0 && __any_sync(0xffffffffu, raise)) {
        // the whole O row in one tensor-memory round trip, scaled in packed pairs
        uint32_t r[C::D];
        if constexpr (C::D == 128) {
          tmem_ld128(lane_base + tm_o, r);
          tmem_ld_wait128(r);
        } else {
          tmem_ld64(lane_base + tm_o, r);
          tmem_ld_wait64(r);
        }
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int i = 0; i < C::D; i += 2) {
          float x, y;
          f2_unpack(f2_mul(f2_pack(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), a2), x, y);
          r[i] = __float_as_uint(x);
          r[i + 1] = __float_as_uint(y);
        }
        if constexpr (C::D == 128)
          tmem_st128(lane_base + tm_o, r);
        else
          tmem_st64(lane_base + tm_o, r);
      }
      m = m_new;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(bar(C::B_PFULL + t));
      ++gs;
    }
    if (!ok) break;
    const float inv_l = (C::FP8 ? vmax * (1.f / 256.f) : 1.f) / ((C::COMP || C::RSUM) ? lc : l);
    const bool row_ok = q_idx < p.N;
    if (!(ok = mbar_wait(bar(C::B_ODONE + t), ti & 1, wc, kSiteODone))) break;
    ++ti;
    tc_fence_after();
    __nv_bfloat16* orow = o_out + (static_cast<size_t>(bh) * p.N + q_idx) * p.ld;
#pragma unroll 1
    for (int c = 0; c < C::D; c += 32) {
      uint32_t r[32];
      tmem_ld32(lane_base + tm_o + c, r);
      tmem_ld_wait(r);
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
      if (row_ok && c < p.ld) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
    if (row_ok && p.lse != nullptr)
      p.lse[static_cast<size_t>(bh) * p.N + q_idx] = (m + __log2f(l)) * LN2;
    tc_fence_before();
  }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    fa_fwd_pp_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::SMEM_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
  const ItemRing ring{sbase + C::SMEM_ITEM,
                      reinterpret_cast<volatile int*>(smem + C::SMEM_ITEM + 2 * kItemSlots * 8)};
  const int warp = threadIdx.x / 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBARS; ++i) {
      mbar_init(bars + 8u * i, (i == C::B_PFULL || i == C::B_PFULL + 1) ? 4u : 1u);  // warps
    }
    ring.init(C::ITEM_READERS);
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

  if (warp >= C::SOFTMAX_WARPS) {
    regs_decrease<C::REGS_OTHER>();
    if (warp == C::PRODUCER_WARP && (threadIdx.x & 31) == 0)
      pp_producer<C>(&tq, &tk, &tv, p, sbase, bars, ring, wc);
    else if (warp == C::MMA_WARP && (threadIdx.x & 31) == 0)
      pp_mma<C>(p, sbase, bars, tmem, ring, wc);
  } else {
    regs_increase<C::REGS_SOFTMAX>();
    pp_softmax<C>(p, bars, tmem, warp / 4, ring, wc);
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) sched_release(p);
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

}  // namespace fa
