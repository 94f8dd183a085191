// fa_decode.cuh — attention for few queries against a long key/value sequence
// (decoding with a KV cache), split along the keys, with grouped query heads.
//
// The same exact attention as the forward, O = softmax(scale Q K^T) V, with
//   * Nq query rows per head (Nq <= Nk) and Nk keys;
//   * Hq query heads sharing Hkv key/value heads (Hq = g Hkv: query head h reads
//     key/value head h / g);
//   * causal masking aligned to the end of the keys: query i sees keys
//     j <= Nk - Nq + i (the queries are the last Nq positions of the sequence).
// Decoding reads Q of length 1 against the whole KV cache, so reading K and V bounds
// it ("FlashAttentionとは？…" (issoh.co.jp), section 短い系列の効果とデコード向け最適化の違い);
// grouped K/V heads: "FlashAttention — フラッシュアテンション" (systems-analysis.info),
// section FlashAttention-2（2023年）.
// Work is split along the keys: a work item is one key/value head
// and one key range; it produces, for the R = g * Nq query rows that read that head,
// the partial result over its keys — the row-normalised O_s and the logsumexp
// lse_s.  A second kernel merges the splits exactly:
//   lse = log sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s,
// the same rule the online softmax applies key tile by key tile.
//
// The R rows of one group are consecutive in memory ([B, Hq, Nq, d] viewed as
// [B, Hkv, R, d]), so they form one query tile (R <= 128, padded with zero rows by
// the tensor-map load).  Each work item is then the one-tile forward pipeline over
// its key range: TMA producer warp, one MMA warp (S = Q K^T, O += P V on the tensor
// core; at R << 128 most of the tensor work is padding, but the item is bound by
// reading K and V from memory), four softmax warps.  The work is memory-bound:
// 4 R d FLOPs per key against 4 d bytes of K and V.
#pragma once

#include <type_traits>

#include "fa_fwd.cuh"

namespace fa {

struct DecParams {
  int BHkv;            // B * Hkv
  int R;               // query rows per key/value head: (Hq / Hkv) * Nq, <= 128
  int Nq, Nk;
  int ld;              // head dim as stored (row length of q, k, v, o); D may be larger
  int causal;
  int n_kt;            // ceil(Nk / BN)
  int split_tiles;     // key tiles per split
  int n_split;         // splits per key/value head
  int total_items;     // BHkv * n_split
  float scale;
  float* part_o;       // fp32 [BHkv, n_split, R, D], row-normalised partial O
  float* part_lse;     // fp32 [BHkv, n_split, R], natural log; -inf: no visible key
  unsigned* status;
  unsigned long long timeout_ns;
};

template <int D_, int KST_, int VST_>
struct DecCfg {
  static constexpr int D = D_;
  static constexpr int BN = D <= 128 ? 128 : 64;
  static constexpr int BM = 128;
  static constexpr int KST = KST_, VST = VST_;
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int NBOX = ROW_BYTES / 128;
  static constexpr int BOX_ELEMS = 64;
  static constexpr int Q_BYTES = BM * ROW_BYTES;
  static constexpr int KV_BYTES = BN * ROW_BYTES;
  static constexpr int MMA_K = 16;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = Q_BYTES;
  static constexpr int SMEM_V = SMEM_K + KST * KV_BYTES;
  static constexpr int SMEM_BAR = SMEM_V + VST * KV_BYTES;
  static constexpr int B_QFULL = 0, B_QEMPTY = 1, B_SFULL = 2, B_PFULL = 4, B_ODONE = 6,
                       B_DRAIN = 7, B_KFULL = 8, B_KEMPTY = 8 + KST, B_VFULL = 8 + 2 * KST,
                       B_VEMPTY = 8 + 2 * KST + VST, NBARS = 8 + 2 * KST + 2 * VST;
  static constexpr int SMEM_MISC = SMEM_BAR + NBARS * 8;
  static constexpr int SMEM_ALLOC = SMEM_MISC + 64 + 1024;
  static constexpr int TM_S = 0;          // + b * BN, two S buffers
  static constexpr int TM_O = 2 * BN;
  static constexpr int TM_COLS = 512;
  static constexpr int THREADS = 192;     // warp 0 TMA, warp 1 MMA, warps 2-5 softmax
  static_assert(2 * BN + D <= TM_COLS, "tensor memory budget");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// Work item w -> (key/value head, key tiles [j0, j1)).
__device__ __forceinline__ void dec_item(const DecParams& p, int w, int& bh, int& j0, int& j1) {
  bh = w / p.n_split;
  const int s = w - bh * p.n_split;
  j0 = s * p.split_tiles;
  j1 = min(p.n_kt, j0 + p.split_tiles);
}

// ---------------------------------------------------------------- producer (one thread)
template <class C>
__device__ void dec_producer(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                             const DecParams& p, uint32_t sbase, uint32_t bars, const WaitCtl& wc) {
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t gk = 0, gv = 0, t = 0;
  bool ok = true;
  auto load_k = [&](int j, int bh) -> bool {
    const int s = gk % C::KST;
    if (gk >= C::KST && !mbar_wait(bar(C::B_KEMPTY + s), ((gk / C::KST) - 1) & 1, wc, kSiteKVEmpty))
      return false;
    mbar_arrive_expect_tx(bar(C::B_KFULL + s), C::KV_BYTES);
#pragma unroll
    for (int c = 0; c < C::NBOX; ++c)
      tma_load_3d(sbase + C::SMEM_K + s * C::KV_BYTES + c * C::BN * 128, tk, bar(C::B_KFULL + s),
                  c * C::BOX_ELEMS, j * C::BN, bh);
    ++gk;
    return true;
  };
  auto load_v = [&](int j, int bh) -> bool {
    const int s = gv % C::VST;
    if (gv >= C::VST && !mbar_wait(bar(C::B_VEMPTY + s), ((gv / C::VST) - 1) & 1, wc, kSiteKVEmpty))
      return false;
    mbar_arrive_expect_tx(bar(C::B_VFULL + s), C::KV_BYTES);
#pragma unroll
    for (int c = 0; c < C::NBOX; ++c)
      tma_load_3d(sbase + C::SMEM_V + s * C::KV_BYTES + c * C::BN * 128, tv, bar(C::B_VFULL + s),
                  c * C::BOX_ELEMS, j * C::BN, bh);
    ++gv;
    return true;
  };
  for (int k = 0; ok; ++k) {
    const int w = fwd_item_index(k);
    if (w >= p.total_items) break;
    int bh, j0, j1;
    dec_item(p, w, bh, j0, j1);
    if (t > 0 && !(ok = mbar_wait(bar(C::B_QEMPTY), (t - 1) & 1, wc, kSiteQEmpty))) break;
    mbar_arrive_expect_tx(bar(C::B_QFULL), C::Q_BYTES);
#pragma unroll
    for (int c = 0; c < C::NBOX; ++c)
      tma_load_3d(sbase + C::SMEM_Q + c * C::BM * 128, tq, bar(C::B_QFULL), c * C::BOX_ELEMS, 0, bh);
    ++t;
    if (!(ok = load_k(j0, bh))) break;
    for (int j = j0 + 1; j < j1 && ok; ++j) ok = load_k(j, bh) && load_v(j - 1, bh);
    if (ok) ok = load_v(j1 - 1, bh);
  }
  if (!ok) {
    if (t > 0) mbar_wait_drain(bar(C::B_QFULL), (t - 1) & 1, 100000000ull);
    for (uint32_t i = (gk > C::KST ? gk - C::KST : 0); i < gk; ++i)
      mbar_wait_drain(bar(C::B_KFULL + i % C::KST), (i / C::KST) & 1, 100000000ull);
    for (uint32_t i = (gv > C::VST ? gv - C::VST : 0); i < gv; ++i)
      mbar_wait_drain(bar(C::B_VFULL + i % C::VST), (i / C::VST) & 1, 100000000ull);
    return;
  }
  if (t > 0) {
    ok = mbar_wait(bar(C::B_QEMPTY), (t - 1) & 1, wc, kSiteQEmpty);
    for (uint32_t i = (gk > C::KST ? gk - C::KST : 0); ok && i < gk; ++i)
      ok = mbar_wait(bar(C::B_KEMPTY + i % C::KST), (i / C::KST) & 1, wc, kSiteKVEmpty);
    for (uint32_t i = (gv > C::VST ? gv - C::VST : 0); ok && i < gv; ++i)
      ok = mbar_wait(bar(C::B_VEMPTY + i % C::VST), (i / C::VST) & 1, wc, kSiteKVEmpty);
  }
}

// ---------------------------------------------------------------- MMA issuer (one thread)
template <class C>
__device__ void dec_mma(const DecParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                        const WaitCtl& wc) {
  auto bar = [&](int i) { return bars + 8u * i; };
  constexpr uint32_t IDESC_S = idesc_bf16(128, C::BN, false);
  constexpr uint32_t IDESC_O = idesc_bf16(128, C::D, true);
  uint32_t g = 0, t = 0;
  bool ok = true;
  auto issue_pv = [&](uint32_t gk, bool first) -> bool {
    const int b = gk & 1;
    if (!mbar_wait(bar(C::B_PFULL + b), (gk >> 1) & 1, wc, kSitePFull)) return false;
    const int s = gk % C::VST;
    if (!mbar_wait(bar(C::B_VFULL + s), (gk / C::VST) & 1, wc, kSiteVFull)) return false;
    tc_fence_after();
    const uint32_t vbase = sbase + C::SMEM_V + s * C::KV_BYTES;
#pragma unroll
    for (int kb = 0; kb < C::BN / C::MMA_K; ++kb)
      umma_ts<false>(tmem + C::TM_O, tmem + C::TM_S + b * C::BN + kb * (C::MMA_K / 2),
                     sdesc_sw128(vbase + kb * C::MMA_K * 128, C::BN * 128, 1024), IDESC_O,
                     (first && kb == 0) ? 0u : 1u);
    tc_commit(bar(C::B_VEMPTY + s));
    tc_commit(bar(C::B_ODONE));
    return true;
  };
  for (int k = 0; ok; ++k) {
    const int w = fwd_item_index(k);
    if (w >= p.total_items) break;
    int bh, j0, j1;
    dec_item(p, w, bh, j0, j1);
    const int n = j1 - j0;
    if (!(ok = mbar_wait(bar(C::B_QFULL), t & 1, wc, kSiteQFull))) break;
    tc_fence_after();
    for (int j = 0; j < n && ok; ++j) {
      const uint32_t gj = g + j;
      const int s = gj % C::KST;
      if (!(ok = mbar_wait(bar(C::B_KFULL + s), (gj / C::KST) & 1, wc, kSiteKFull))) break;
      tc_fence_after();
      const int b = gj & 1;
      const uint32_t kbase = sbase + C::SMEM_K + s * C::KV_BYTES;
#pragma unroll
      for (int kb = 0; kb < C::D / C::MMA_K; ++kb) {
        const int box = (kb * 32) / 128, off = (kb * 32) % 128;
        umma_ss<false>(tmem + C::TM_S + b * C::BN,
                       sdesc_sw128(sbase + C::SMEM_Q + box * C::BM * 128 + off, 16, 1024),
                       sdesc_sw128(kbase + box * C::BN * 128 + off, 16, 1024), IDESC_S,
                       kb > 0 ? 1u : 0u);
      }
      tc_commit(bar(C::B_KEMPTY + s));
      tc_commit(bar(C::B_SFULL + b));
      if (j == n - 1) tc_commit(bar(C::B_QEMPTY));
      if (j > 0) ok = issue_pv(gj - 1, j == 1);
    }
    if (ok) ok = issue_pv(g + n - 1, n == 1);
    g += n;
    ++t;
  }
  tc_commit(bar(C::B_DRAIN));
  if (!mbar_wait_drain(bar(C::B_DRAIN), 0, wc.timeout_ns))
    atomicCAS(wc.status, 0u, kStatusTimeout | kSiteDrain);
}

// ---------------------------------------------------------------- softmax warps
// Thread = one query row rho of the group (rho < R; rows >= R are zero padding whose
// results are discarded).  Row rho is query i = rho % Nq of its head.
template <class C>
__device__ void dec_softmax(const DecParams& p, uint32_t bars, uint32_t tmem, const WaitCtl& wc) {
  auto bar = [&](int i) { return bars + 8u * i; };
  const int warp = threadIdx.x / 32;
  const int quad = warp & 3;
  const int row = quad * 32 + (threadIdx.x & 31);
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const float LOG2E = 1.4426950408889634f;
  const float LN2 = 0.6931471805599453f;
  const float sl2 = p.scale * LOG2E;
  const bool row_ok = row < p.R;
  // last key this row may see
  const int lim = p.causal ? p.Nk - p.Nq + (row % p.Nq) : p.Nk - 1;
  uint32_t g = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int w = fwd_item_index(k);
    if (w >= p.total_items) break;
    int bh, j0, j1;
    dec_item(p, w, bh, j0, j1);
    const int n = j1 - j0;
    float m = -INFINITY, l = 0.f;
    for (int j = 0; j < n; ++j) {
      const uint32_t gj = g + j;
      const int b = gj & 1;
      if (!(ok = mbar_wait(bar(C::B_SFULL + b), (gj >> 1) & 1, wc, kSiteSFull))) break;
      tc_fence_after();
      float s[C::BN];
      {
        uint32_t r[C::BN];
        if constexpr (C::BN == 128) {
          tmem_ld128(lane_base + C::TM_S + b * C::BN, r);
          tmem_ld_wait128(r);
        } else {
          tmem_ld64(lane_base + C::TM_S + b * C::BN, r);
          tmem_ld_wait64(r);
        }
#pragma unroll
        for (int i = 0; i < C::BN; ++i) s[i] = __uint_as_float(r[i]);
      }
      const int kv0 = (j0 + j) * C::BN;
      if (__any_sync(0xffffffffu, kv0 + C::BN - 1 > lim)) {
#pragma unroll
        for (int c = 0; c < C::BN; ++c)
          if (kv0 + c > lim) s[c] = -INFINITY;
      }
      float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < C::BN; c += 8) {
        a0 = max3f(a0, s[c], s[c + 1]);
        a1 = max3f(a1, s[c + 2], s[c + 3]);
        a2 = max3f(a2, s[c + 4], s[c + 5]);
        a3 = max3f(a3, s[c + 6], s[c + 7]);
      }
      const float m_cand = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) * sl2;
      const bool raise = m_cand > m;
      const float m_new = raise ? m_cand : m;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = raise ? ex2(m - m_use) : 1.f;
      const uint64_t c2 = f2_pack(sl2, sl2);
      const uint64_t nm2 = f2_pack(-m_use, -m_use);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < C::BN; c += 2) {
        const uint64_t x2 = f2_fma(f2_pack(s[c], s[c + 1]), c2, nm2);
        float xa, xb;
        f2_unpack(x2, xa, xb);
        const uint64_t p2 = f2_pack(ex2(xa), ex2(xb));
        acc[(c / 2) % 4] = f2_add(acc[(c / 2) % 4], p2);
        f2_unpack(p2, s[c], s[c + 1]);
      }
      float sa, sb;
      f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), sa, sb);
      l = l * alpha + (sa + sb);
#pragma unroll
      for (int c = 0; c < C::BN; c += 64) {
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = pack_bf16x2(s[c + 2 * i], s[c + 2 * i + 1]);
        tmem_st32(lane_base + C::TM_S + b * C::BN + c / 2, r);
      }
      // the previous P V product must be complete before O is rescaled
      if (j > 0) {
        if (!(ok = mbar_wait(bar(C::B_ODONE), (gj - 1) & 1, wc, kSiteODone))) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, raise)) {
#pragma unroll 1
          for (int c = 0; c < C::D; c += 32) {
            uint32_t r[32];
            tmem_ld32(lane_base + C::TM_O + c, r);
            tmem_ld_wait(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(lane_base + C::TM_O + c, r);
          }
        }
      }
      m = m_new;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(bar(C::B_PFULL + b));
    }
    if (!ok) break;
    // epilogue: this split's row-normalised O and logsumexp (fp32) to the workspace
    const uint32_t glast = g + n - 1;
    if (!(ok = mbar_wait(bar(C::B_ODONE), glast & 1, wc, kSiteODone))) break;
    tc_fence_after();
    const bool any = l > 0.f;                     // some key of this split is visible
    const float inv_l = any ? 1.f / l : 0.f;
    float* orow = p.part_o + (static_cast<size_t>(w) * p.R + row) * C::D;
#pragma unroll 1
    for (int c = 0; c < C::D; c += 32) {
      uint32_t r[32];
      tmem_ld32(lane_base + C::TM_O + c, r);
      tmem_ld_wait(r);
      if (row_ok) {
        float4* d4 = reinterpret_cast<float4*>(orow + c);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          d4[i] = make_float4(__uint_as_float(r[4 * i]) * inv_l, __uint_as_float(r[4 * i + 1]) * inv_l,
                              __uint_as_float(r[4 * i + 2]) * inv_l, __uint_as_float(r[4 * i + 3]) * inv_l);
      }
    }
    if (row_ok) p.part_lse[static_cast<size_t>(w) * p.R + row] = any ? (m + __log2f(l)) * LN2 : -INFINITY;
    tc_fence_before();
    g += n;
  }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    fa_decode_split_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                           const __grid_constant__ CUtensorMap tv, const DecParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::SMEM_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
  const int warp = threadIdx.x / 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBARS; ++i)
      mbar_init(bars + 8u * i, (i == C::B_PFULL || i == C::B_PFULL + 1) ? 4u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.status, p.timeout_ns};
  if (warp == 0) {
    if ((threadIdx.x & 31) == 0) dec_producer<C>(&tq, &tk, &tv, p, sbase, bars, wc);
  } else if (warp == 1) {
    if ((threadIdx.x & 31) == 0) dec_mma<C>(p, sbase, bars, tmem, wc);
  } else {
    dec_softmax<C>(p, bars, tmem, wc);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

// ---------------------------------------------------------------- combine
// lse = log sum_s exp(lse_s) and O = sum_s exp(lse_s - lse) O_s per query row, written as
// bf16 (and lse as fp32).  One thread per (row, four output columns): every thread reads
// its row's split logsumexps (cached after the first thread) and then the partial values
// of its columns from all splits, several loads in flight, so the merge costs a few
// memory round trips rather than one per split.
// Launched as a programmatic dependent of the split kernel: its blocks start while the
// split kernel's last CTAs run, and wait here until that grid has completed and its
// partial results are visible.
template <int D>
__global__ void __launch_bounds__(256) fa_decode_combine_kernel(const DecParams p, void* o, float* lse) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int C4 = D / 4;                       // float4 groups per row
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<long long>(p.BHkv) * p.R * C4) return;
  const int c4 = static_cast<int>(t % C4);
  const long long rr = t / C4;
  const int row = static_cast<int>(rr % p.R);
  const int bh = static_cast<int>(rr / p.R);
  const float* pl = p.part_lse + static_cast<size_t>(bh) * p.n_split * p.R + row;
  float mx = -INFINITY;
#pragma unroll 8
  for (int s = 0; s < p.n_split; ++s) mx = fmaxf(mx, __ldg(pl + static_cast<size_t>(s) * p.R));
  // every row sees at least one key, so mx is finite
  float sum = 0.f;
#pragma unroll 8
  for (int s = 0; s < p.n_split; ++s) sum += __expf(__ldg(pl + static_cast<size_t>(s) * p.R) - mx);
  const float lse_row = mx + __logf(sum);
  const float4* src = reinterpret_cast<const float4*>(
      p.part_o + (static_cast<size_t>(bh) * p.n_split * p.R + row) * D) + c4;
  const size_t split_stride = static_cast<size_t>(p.R) * C4;   // float4s between splits
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
  for (int s = 0; s < p.n_split; ++s) {
    const float ls = __ldg(pl + static_cast<size_t>(s) * p.R);
    const float w = ls == -INFINITY ? 0.f : __expf(ls - lse_row);   // a split with no key
    const float4 v = __ldg(src + s * split_stride);
    acc.x = fmaf(w, v.x, acc.x);
    acc.y = fmaf(w, v.y, acc.y);
    acc.z = fmaf(w, v.z, acc.z);
    acc.w = fmaf(w, v.w, acc.w);
  }
  const int col = 4 * c4;
  if (col < p.ld) {
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(o) + (static_cast<size_t>(bh) * p.R + row) * p.ld + col;
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(dst) = pk;   // ld is a multiple of 16, so 8-byte aligned
  }
  if (lse != nullptr && c4 == 0) lse[static_cast<size_t>(bh) * p.R + row] = lse_row;
}

}  // namespace fa
