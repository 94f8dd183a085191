// fa_fwd_sp.cuh — forward for d <= 128 with the probabilities in their own tensor-memory
// buffers (bf16 and FP8 e4m3 inputs).
//
// Same mathematics as fa_fwd.cuh (S = Q K^T, exp2 online softmax with a rescale only
// when a row max rises, O += P V, causal tiles above the diagonal skipped, persistent
// heaviest-first schedule).  The layout on the SM is chosen so that the tensor core's
// next score tile never waits for the softmax to finish the current one:
//
//  * P(j) is written to a buffer of its own (two of them, alternating), not over S(j).
//    The single S buffer is free again as soon as the softmax warps have loaded S(j)
//    into registers, so S(j+1) is computed while they work on S(j).
//  * Each row is split into two column halves handled by two warps on the same TMEM
//    lane quadrant.  Each half keeps its own running max m_h and sum l_h and its own
//    output accumulator O_h += P_h V_h (P_h: that half's 64 probabilities, V_h: the
//    matching 64 value rows), so the halves never wait for each other inside the key
//    loop.  At the end of a tile they combine:
//        O = (O_0 2^(m_0 - m) + O_1 2^(m_1 - m)) / (l_0 2^(m_0 - m) + l_1 2^(m_1 - m)),
//    m = max(m_0, m_1) -- the merge rule of partial softmax results.
//  * O_h is rescaled by the half itself once P_h(j-1) V_h is complete; that product was
//    issued a whole softmax step earlier, so the wait is normally already satisfied.
//
// Roles: warps 0-7 softmax (warp w: lanes 32*(w%4).., column half w/4), warp 8 TMA
// producer, warp 9 S issuer + TMEM owner, warp 10 P V issuer (warp 9 issues both when
// SPLIT is off), warp 11 idle (warpgroup alignment).
// Tensor memory: S [0,128), P_0 [128,192), P_1 [192,256), O_0 [256,256+D), O_1 [256+D,256+2D).
#pragma once

#include <type_traits>

#include "fa_fwd_ws.cuh"

namespace fa {

template <int D_, int KST_, int VST_, bool FP8_, int EMU_ = 1, bool SPLIT_ = true>
struct SPCfg {
  static constexpr int D = D_;
  static constexpr int BN = 128;
  static constexpr int BM = 128;
  static constexpr int KST = KST_, VST = VST_;
  static constexpr bool FP8 = FP8_;
  static constexpr int EMU = EMU_;                    // software exp2 share, in quarters
  static constexpr bool SEPARATE_P = true;
  // Two issuing warps: S = Q K^T from one, the P V products from another.  The two
  // streams share no tensor-memory buffer, so neither waits for the other, and each
  // warp's barrier waits overlap the other's MMAs.
  static constexpr bool SPLIT = SPLIT_;
  static constexpr int HALF = BN / 2;                 // score columns per softmax warp
  static constexpr int DH = D / 2;                    // output columns written per warp
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int ROW_BYTES = D * ELEM;
  static constexpr int NBOX = ROW_BYTES / 128;
  static constexpr int BOX_ELEMS = 128 / ELEM;
  static constexpr int Q_BYTES = BM * ROW_BYTES;
  static constexpr int KV_BYTES = BN * ROW_BYTES;
  static constexpr int MMA_K = FP8 ? 32 : 16;
  static constexpr int KSTEP_BYTES = MMA_K * ELEM;
  static constexpr int KB_H = HALF / MMA_K;           // P V MMAs per half
  static constexpr int PCOL_H = HALF * ELEM / 4;      // 32-bit TMEM columns of P_h
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = Q_BYTES;
  static constexpr int SMEM_V = SMEM_K + KST * KV_BYTES;
  // epilogue exchange between the two halves of a row: [m, l][half][128 rows] fp32
  static constexpr int SMEM_X = SMEM_V + VST * KV_BYTES;
  static constexpr int SMEM_BAR = SMEM_X + 4 * 128 * 4;
  static constexpr int B_QFULL = 0, B_QEMPTY = 1, B_SFULL = 2, B_SEMPTY = 3, B_ODONE = 4,
                       B_DRAIN = 5,
                       B_DRAIN2 = 6,                  // drain of the P V issuer
                       B_XCHG = 7,                    // + quad, one arrival per half-warp
                       B_PFULLH = 11,                 // + 2 * half + buffer, 4 warps each
                       B_PVDONEH = 15,                // + half
                       B_KFULL = 17, B_KEMPTY = 17 + KST, B_VFULL = 17 + 2 * KST,
                       B_VEMPTY = 17 + 2 * KST + VST, NBARS = 17 + 2 * KST + 2 * VST;
  static constexpr int SMEM_MISC = SMEM_BAR + NBARS * 8;
  static constexpr int SMEM_ALLOC = SMEM_MISC + 64 + 1024;
  static constexpr int TM_S = 0;
  static constexpr int TM_P = BN;                     // + b * 64 + half * PCOL_H
  static constexpr int TM_O = 2 * BN;                 // + half * D
  static constexpr int TM_COLS = 512;
  static constexpr int THREADS = 384;
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9, PV_WARP = 10;
  static_assert(TM_O + 2 * D <= TM_COLS, "tensor memory budget");
  static_assert(2 * PCOL_H <= 64, "P buffer width");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(DH % 32 == 0, "32-column output chunks per warp");
};

// P_h(j) V_h into O_h: the MMAs of key blocks [h*KB_H, (h+1)*KB_H) of the tile.
template <class C>
__device__ __forceinline__ void sp_issue_pv_half(uint32_t o_tmem, uint32_t p_tmem, uint64_t vdesc,
                                                 int h, bool first) {
  constexpr uint32_t IDESC_O = C::FP8 ? idesc_e4m3(128, C::D, true) : idesc_bf16(128, C::D, true);
#pragma unroll
  for (int i = 0; i < C::KB_H; ++i) {
    const int kb = h * C::KB_H + i;
    umma_ts_elect(C::FP8, o_tmem, p_tmem + i * (C::MMA_K * C::ELEM / 4),
                  vdesc + static_cast<uint64_t>((kb * C::MMA_K * 128) >> 4), IDESC_O,
                  (first && i == 0) ? 0u : 1u);
  }
}

// ---------------------------------------------------------------- MMA issuer (whole warp)
// Iteration j of a tile: S(j) as soon as every softmax warp has loaded S(j-1), then the
// two halves' P(j-1) V products as their probabilities arrive.
template <class C>
__device__ void sp_mma(const FwdParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                       const WaitCtl& wc) {
  const uint32_t b_qfull = bars + 8u * C::B_QFULL, b_qempty = bars + 8u * C::B_QEMPTY;
  const uint32_t b_sfull = bars + 8u * C::B_SFULL, b_sempty = bars + 8u * C::B_SEMPTY;
  const uint32_t b_pfullh = bars + 8u * C::B_PFULLH, b_pvdoneh = bars + 8u * C::B_PVDONEH;
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
    for (int j = 0; j <= n; ++j) {
      const uint32_t gj = g + j;
      if (j < n) {
        const uint32_t ks = gj % C::KST;
        if (!mbar_wait_warp(b_kfull + 8u * ks, (gj / C::KST) & 1, wc, kSiteKFull)) { ok = false; break; }
        if (gj > 0 && !mbar_wait_warp(b_sempty, (gj - 1) & 1, wc, kSiteSFull)) { ok = false; break; }
        tc_fence_after();
        ws_issue_s<C>(tmem + C::TM_S, qdesc, kdesc_base + static_cast<uint64_t>(ks * (C::KV_BYTES >> 4)));
        tc_commit_elect(b_kempty + 8u * ks);
        tc_commit_elect(b_sfull);
        if (j == n - 1) tc_commit_elect(b_qempty);
      }
      if (j > 0) {
        const uint32_t gp = gj - 1;
        const uint32_t vs = gp % C::VST;
        const uint32_t pb = gp & 1, pph = (gp >> 1) & 1;
        if (!mbar_wait_warp(b_vfull + 8u * vs, (gp / C::VST) & 1, wc, kSiteVFull)) { ok = false; break; }
        const uint64_t vdesc = vdesc_base + static_cast<uint64_t>(vs * (C::KV_BYTES >> 4));
        if (j == 1) {
          // the first products of a tile overwrite both accumulators: both halves must
          // be past the previous tile's epilogue, which reads both
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
          sp_issue_pv_half<C>(tmem + C::TM_O + h * C::D, tmem + C::TM_P + pb * 64 + h * C::PCOL_H,
                              vdesc, h, j == 1);
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

// ---------------------------------------------------------------- split issuers
// S issuer (warp MMA_WARP, also the TMEM owner).
template <class C>
__device__ void sp_mma_s(const FwdParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                         const WaitCtl& wc) {
  const uint32_t b_qfull = bars + 8u * C::B_QFULL, b_qempty = bars + 8u * C::B_QEMPTY;
  const uint32_t b_sfull = bars + 8u * C::B_SFULL, b_sempty = bars + 8u * C::B_SEMPTY;
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
      if (gj > 0 && !mbar_wait_warp(b_sempty, (gj - 1) & 1, wc, kSiteSFull)) { ok = false; break; }
      tc_fence_after();
      ws_issue_s<C>(tmem + C::TM_S, qdesc, kdesc_base + static_cast<uint64_t>(ks * (C::KV_BYTES >> 4)));
      tc_commit_elect(b_kempty + 8u * ks);
      tc_commit_elect(b_sfull);
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

// P V issuer (warp PV_WARP): P_h(j) V_h into O_h as each half's probabilities arrive.
template <class C>
__device__ void sp_mma_pv(const FwdParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                          const WaitCtl& wc) {
  const uint32_t b_pfullh = bars + 8u * C::B_PFULLH, b_pvdoneh = bars + 8u * C::B_PVDONEH;
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
      const uint32_t pb = gp & 1, pph = (gp >> 1) & 1;
      if (!mbar_wait_warp(b_vfull + 8u * vs, (gp / C::VST) & 1, wc, kSiteVFull)) { ok = false; break; }
      const uint64_t vdesc = vdesc_base + static_cast<uint64_t>(vs * (C::KV_BYTES >> 4));
      if (j == 0) {
        // the first products of a tile overwrite both accumulators: both halves must
        // be past the previous tile's epilogue, which reads both
        if (!mbar_wait_warp(b_pfullh + 8u * pb, pph, wc, kSitePFull) ||
            !mbar_wait_warp(b_pfullh + 8u * (2 + pb), pph, wc, kSitePFull)) {
          ok = false;
          break;
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (j > 0 && !mbar_wait_warp(b_pfullh + 8u * (2 * h + pb), pph, wc, kSitePFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        sp_issue_pv_half<C>(tmem + C::TM_O + h * C::D, tmem + C::TM_P + pb * 64 + h * C::PCOL_H,
                            vdesc, h, j == 0);
        tc_commit_elect(b_pvdoneh + 8u * h);
      }
      if (!ok) break;
      tc_commit_elect(b_vempty + 8u * vs);
      if (j == n - 1) tc_commit_elect(b_odone);
    }
    if (!ok) break;
    g += n;
  }
  tc_commit_elect(bars + 8u * C::B_DRAIN2);
  if (!mbar_wait_drain(bars + 8u * C::B_DRAIN2, 0, wc.timeout_ns) && (threadIdx.x & 31) == 0)
    atomicCAS(wc.status, 0u, kStatusTimeout | kSiteDrain);
}

// Scale a full accumulator row (D columns) of this warp's lanes by `a`.
template <class C>
__device__ __forceinline__ void sp_scale_o(uint32_t taddr, float a) {
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

// ---------------------------------------------------------------- softmax warps
template <class C>
__device__ void sp_softmax(const FwdParams& p, uint32_t bars, uint32_t tmem, float* xbuf,
                           const WaitCtl& wc) {
  const int warp = threadIdx.x / 32;
  const int quad = warp & 3, half = warp >> 2;
  const int row = quad * 32 + (threadIdx.x & 31);
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const uint32_t b_sfull = bars + 8u * C::B_SFULL, b_sempty = bars + 8u * C::B_SEMPTY;
  const uint32_t b_pfull = bars + 8u * (C::B_PFULLH + 2 * half);
  const uint32_t b_pvdone = bars + 8u * (C::B_PVDONEH + half);
  const uint32_t b_odone = bars + 8u * C::B_ODONE;
  const uint32_t b_x = bars + 8u * (C::B_XCHG + quad);
  const uint32_t s_cols = lane_base + C::TM_S + half * C::HALF;
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
    float m = -INFINITY, l = 0.f;
    float qsc = 1.f, vmax = 1.f;
    if constexpr (C::FP8) {
      qsc = p.q_scale[bh * p.n_st + qt];
      vmax = 0.f;
      for (int j = 0; j < n; ++j) vmax = fmaxf(vmax, p.v_scale[fwd_kv_head(p, bh) * p.n_st + j]);
    }
    for (int j = 0; j < n; ++j) {
      const uint32_t gj = g + j;
      if (!mbar_wait(b_sfull, gj & 1, wc, kSiteSFull)) { ok = false; break; }
      tc_fence_after();
      float s[C::HALF];
      {
        uint32_t r[C::HALF];
        tmem_ld64(s_cols, r);
        tmem_ld_wait64(r);
#pragma unroll
        for (int i = 0; i < C::HALF; ++i) s[i] = __uint_as_float(r[i]);
      }
      // the scores are in registers: the MMA warp may compute S(j+1) now
      tc_fence_before();
      mbar_arrive_warp(b_sempty);
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
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = fmaxf(s[2 * i], s[2 * i + 1]);
#pragma unroll
      for (int c = 16; c < C::HALF; c += 16)
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = max3f(mx[i], s[c + 2 * i], s[c + 2 * i + 1]);
      const float m_cand =
          fmaxf(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], max3f(mx[5], mx[6], mx[7]))) * c_j;
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
      else
        exps(std::integral_constant<int, C::EMU>{});
      float sa, sb;
      f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), sa, sb);
      l = l * alpha + (sa + sb);
      // P_h(j-1) V_h complete: P buffer j%2 is no longer read (its last reader,
      // P_h(j-2) V_h, completed before) and O_h holds every earlier product
      if (gj > 0) {
        if (!mbar_wait(b_pvdone, (gj - 1) & 1, wc, kSitePvDone)) { ok = false; break; }
        tc_fence_after();
      }
      const uint32_t p_cols = lane_base + C::TM_P + (gj & 1) * 64 + half * C::PCOL_H;
      if constexpr (C::FP8) {
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          r[i] = pack_e4m3x4(s[4 * i] * fold, s[4 * i + 1] * fold, s[4 * i + 2] * fold,
                             s[4 * i + 3] * fold);
        tmem_st16(p_cols, r);
      } else {
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = pack_bf16x2(s[2 * i], s[2 * i + 1]);
        tmem_st32(p_cols, r);
      }
      // bring O_h to the new reference max (warp-uniform; alpha = 1 on rows that kept it)
      if (j > 0 && __any_sync(0xffffffffu, raise)) sp_scale_o<C>(o_mine, alpha);
      m = m_new;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(b_pfull + 8u * (gj & 1));
    }
    if (!ok) break;
    if (!mbar_wait(b_odone, t & 1, wc, kSiteODone)) { ok = false; break; }
    ++t;
    tc_fence_after();
    // merge the two halves of each row
    xbuf[half * 128 + row] = m;
    xbuf[(2 + half) * 128 + row] = l;
    mbar_arrive_warp(b_x);
    if (!mbar_wait(b_x, xc & 1, wc, kSiteXchg)) { ok = false; break; }
    ++xc;
    const float m_o = xbuf[(half ^ 1) * 128 + row];
    const float l_o = xbuf[(2 + (half ^ 1)) * 128 + row];
    const float m_fin = fmaxf(m, m_o);
    const float m_ref = (m_fin == -INFINITY) ? 0.f : m_fin;
    // a half that saw only masked keys has m = -inf, l = 0 and O_h = 0: weight 0
    const float e_me = (m == -INFINITY) ? 0.f : ex2(m - m_ref);
    const float e_ot = (m_o == -INFINITY) ? 0.f : ex2(m_o - m_ref);
    const float l_row = l * e_me + l_o * e_ot;
    const float inv_l = (C::FP8 ? vmax * (1.f / 256.f) : 1.f) / l_row;
    const float w0 = (half == 0 ? e_me : e_ot) * inv_l;
    const float w1 = (half == 0 ? e_ot : e_me) * inv_l;
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
      p.lse[static_cast<size_t>(bh) * p.N + q_idx] = (m_ref + __log2f(l_row)) * LN2;
    tc_fence_before();
    g += n;
  }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    fa_fwd_sp_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
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
      if (i == C::B_SEMPTY) cnt = 8;                                   // the 8 softmax warps
      if (i >= C::B_XCHG && i < C::B_XCHG + 4) cnt = 2;               // one half-warp pair
      if (i >= C::B_PFULLH && i < C::B_PFULLH + 4) cnt = 4;           // one column half
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
      sp_mma_s<C>(p, sbase, bars, tmem, wc);
    else
      sp_mma<C>(p, sbase, bars, tmem, wc);
  } else if (C::SPLIT && warp == C::PV_WARP) {
    sp_mma_pv<C>(p, sbase, bars, tmem, wc);
  } else if (warp < 8) {
    sp_softmax<C>(p, bars, tmem, xbuf, wc);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

}  // namespace fa
