// fa_bwd.cuh — attention backward for sm_100a by recomputation.
//
// The score tiles are recomputed from Q and K and the probabilities rebuilt
// from the forward's saved row logsumexp, so no N x N matrix is ever stored
// ("FlashAttentionとは？…" (issoh.co.jp), section 逆伝播でL×L行列を保存せず
// 再計算する設計).  Gradients of L = sum(O * dO):
//
//   P  = exp(scale S - lse)  = 2^(S * scale*log2e - lse*log2e)
//   dV = P^T dO              dP = dO V^T
//   D_i = sum_c dO_ic O_ic   (= sum_j P_ij dP_ij)
//   dS = P * (dP - D)        dK = scale dS^T Q        dQ = scale dS K
//
// Three kernels, in stream order:
//   1. fa_bwd_rowdot   D_i = dO_i . O_i into the caller's workspace (HBM-bound).
//   2. fa_bwd_dkdv     one CTA per (head, 128-row key tile[, half of d]); it keeps
//                      K, V in shared memory and dK, dV accumulators in tensor
//                      memory, and streams the query tiles.  Thread t of the
//                      compute warps owns key row t (transposed tiles S^T, dP^T).
//   3. fa_bwd_dq       one CTA per (head, 128-row query tile); it keeps Q, dO in
//                      shared memory and dQ in tensor memory, and streams K/V.
// Splitting dQ into its own pass costs a second recompute of S and dP but needs
// no fp32 atomics and is deterministic.
//
// Roles in kernels 2 and 3: warp 0 = TMA producer, warp 1 = MMA issuer (one
// thread, owns tensor memory), warps 2..5 = elementwise work on TMEM lanes.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

struct BwdParams {
  int BH, N;
  int n_qt;              // query tiles of BMQ rows (dK/dV pass) / 128 rows (dQ pass)
  int n_kt;              // key tiles
  int causal;
  float scale;
  const float* lse;      // [BH, N]
  const float* drow;     // D_i workspace [BH, N]
  void* dq;              // bf16 [BH, N, D]
  void* dk;
  void* dv;
  unsigned* status;
  unsigned long long timeout_ns;
};

// --------------------------------------------------------------------------- 1. D_i
// D_i = sum_c dO_ic * O_ic, fp32 accumulation of the bf16 products.  Each group of
// D/8 threads reads one row with 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_rowdot(const __nv_bfloat16* __restrict__ o,
                                                     const __nv_bfloat16* __restrict__ dout,
                                                     float* __restrict__ drow, long long rows) {
  constexpr int TPR = D / 8;                 // threads per row
  constexpr int RPB = 256 / TPR;             // rows per block pass
  const int sub = threadIdx.x % TPR;
  for (long long r = static_cast<long long>(blockIdx.x) * RPB + threadIdx.x / TPR; r < rows;
       r += static_cast<long long>(gridDim.x) * RPB) {
    const uint4 a = reinterpret_cast<const uint4*>(o + r * D)[sub];
    const uint4 b = reinterpret_cast<const uint4*>(dout + r * D)[sub];
    const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&b);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 fa2 = __bfloat1622float2(ha[i]);
      const float2 fb2 = __bfloat1622float2(hb[i]);
      acc = fmaf(fa2.x, fb2.x, acc);
      acc = fmaf(fa2.y, fb2.y, acc);
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (sub == 0) drow[r] = acc;
  }
}

// --------------------------------------------------------------------------- 2. dK, dV
template <int D_, int DH_, int BMQ_, int STAGES_>
struct DkdvCfg {
  static constexpr int D = D_;          // head dim (contraction of S^T and dP^T)
  static constexpr int DH = DH_;        // columns of dK/dV this CTA produces
  static constexpr int NSPLIT = D / DH;
  static constexpr int BMQ = BMQ_;      // query rows per streamed tile
  static constexpr int BN = 128;        // key rows of the CTA = TMEM lanes
  static constexpr int STAGES = STAGES_;
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int NBOX = ROW_BYTES / 128;
  static constexpr int KT_BYTES = BN * ROW_BYTES;       // K or V tile
  static constexpr int QT_BYTES = BMQ * ROW_BYTES;      // Q_i or dO_i tile
  static constexpr int SMEM_K = 0;
  static constexpr int SMEM_V = KT_BYTES;
  static constexpr int SMEM_Q = 2 * KT_BYTES;
  static constexpr int SMEM_DO = SMEM_Q + STAGES * QT_BYTES;
  static constexpr int SMEM_LSE = SMEM_DO + STAGES * QT_BYTES;    // [STAGES][BMQ] fp32
  static constexpr int SMEM_DD = SMEM_LSE + STAGES * BMQ * 4;     // [STAGES][BMQ] fp32
  static constexpr int SMEM_BAR = SMEM_DD + STAGES * BMQ * 4;
  static constexpr int B_KV = 0, B_SDP = 1, B_P = 2, B_DS = 3, B_ACC = 4, B_DRAIN = 5,
                       B_FULL = 6, B_EMPTY = 6 + STAGES, NBARS = 6 + 2 * STAGES;
  static constexpr int SMEM_MISC = SMEM_BAR + NBARS * 8;
  static constexpr int SMEM_ALLOC = SMEM_MISC + 64 + 1024;
  static constexpr int TM_ST = 0, TM_DPT = BMQ, TM_DV = 2 * BMQ, TM_DK = 2 * BMQ + DH;
  static constexpr int TM_COLS = 512;
  static constexpr int THREADS = 192;
  static_assert(2 * BMQ + 2 * DH <= TM_COLS, "tensor memory budget");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(BMQ % 64 == 0 && DH % 64 == 0, "64-column boxes and 32-column TMEM chunks");
};

template <class C>
__device__ __forceinline__ void dkdv_q_range(const BwdParams& p, int kt, int& i0, int& i1) {
  i1 = p.n_qt;
  i0 = p.causal ? (kt * C::BN) / C::BMQ : 0;   // first query tile that reaches key kt*128
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    fa_bwd_dkdv(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::SMEM_BAR;
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
  float* lse_s = reinterpret_cast<float*>(smem + C::SMEM_LSE);
  float* dd_s = reinterpret_cast<float*>(smem + C::SMEM_DD);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;

  // block -> (bh, key tile, d half); heaviest causal tiles (small kt) first
  const int split = blockIdx.x % C::NSPLIT;
  const int rest = blockIdx.x / C::NSPLIT;
  const int kt = rest % p.n_kt;
  const int bh = rest / p.n_kt;
  int i0, i1;
  dkdv_q_range<C>(p, kt, i0, i1);
  const int nsteps = i1 - i0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBARS; ++i)
      mbar_init(bar(i), (i == C::B_P || i == C::B_DS) ? 4u : 1u);   // 4 compute warps
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
    // ---------------- producer (whole warp: lanes stage lse/D, lane 0 issues TMA)
    bool ok = true;
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(C::B_KV), 2 * C::KT_BYTES);
      for (int c = 0; c < C::NBOX; ++c) {
        tma_load_3d(sbase + C::SMEM_K + c * C::BN * 128, &tk, bar(C::B_KV), c * 64, kt * C::BN, bh);
        tma_load_3d(sbase + C::SMEM_V + c * C::BN * 128, &tv, bar(C::B_KV), c * 64, kt * C::BN, bh);
      }
    }
    for (int st = 0; st < nsteps && ok; ++st) {
      const int s = st % C::STAGES;
      const int qi = i0 + st;
      if (st >= C::STAGES) {
        // every lane waits; the warp then agrees on the outcome so it stays converged
        ok = mbar_wait(bar(C::B_EMPTY + s), ((st / C::STAGES) - 1) & 1, wc, kSiteKVEmpty);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      for (int c = lane; c < C::BMQ; c += 32) {
        const int q = qi * C::BMQ + c;
        const bool in = q < p.N;
        lse_s[s * C::BMQ + c] = in ? p.lse[static_cast<size_t>(bh) * p.N + q] : 0.f;
        dd_s[s * C::BMQ + c] = in ? p.drow[static_cast<size_t>(bh) * p.N + q] : 0.f;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(C::B_FULL + s), 2 * C::QT_BYTES);
        for (int c = 0; c < C::NBOX; ++c) {
          tma_load_3d(sbase + C::SMEM_Q + s * C::QT_BYTES + c * C::BMQ * 128, &tq,
                      bar(C::B_FULL + s), c * 64, qi * C::BMQ, bh);
          tma_load_3d(sbase + C::SMEM_DO + s * C::QT_BYTES + c * C::BMQ * 128, &tdo,
                      bar(C::B_FULL + s), c * 64, qi * C::BMQ, bh);
        }
      }
    }
    if (lane == 0) {
      if (ok) {
        for (int st = (nsteps > C::STAGES ? nsteps - C::STAGES : 0); ok && st < nsteps; ++st)
          ok = mbar_wait(bar(C::B_EMPTY + st % C::STAGES), (st / C::STAGES) & 1, wc, kSiteKVEmpty);
      } else {
        mbar_wait_drain(bar(C::B_KV), 0, 100000000ull);
        for (int st = (nsteps > C::STAGES ? nsteps - C::STAGES : 0); st < nsteps; ++st)
          mbar_wait_drain(bar(C::B_FULL + st % C::STAGES), (st / C::STAGES) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_T = idesc_bf16(128, C::BMQ, false);    // S^T, dP^T: 128 x BMQ
      constexpr uint32_t ID_G = idesc_bf16(128, C::DH, true);      // dV, dK: 128 x DH, B MN-major
      bool ok = mbar_wait(bar(C::B_KV), 0, wc, kSiteKFull);
      for (int st = 0; st < nsteps && ok; ++st) {
        const int s = st % C::STAGES;
        if (!(ok = mbar_wait(bar(C::B_FULL + s), (st / C::STAGES) & 1, wc, kSiteQFull))) break;
        tc_fence_after();
        const uint32_t qb = sbase + C::SMEM_Q + s * C::QT_BYTES;
        const uint32_t dob = sbase + C::SMEM_DO + s * C::QT_BYTES;
#pragma unroll
        for (int kb = 0; kb < C::D / 16; ++kb) {
          const int box = kb / 4, off = (kb % 4) * 32;
          umma_ss<false>(tmem + C::TM_ST,
                         sdesc_sw128(sbase + C::SMEM_K + box * C::BN * 128 + off, 16, 1024),
                         sdesc_sw128(qb + box * C::BMQ * 128 + off, 16, 1024), ID_T, kb > 0);
        }
#pragma unroll
        for (int kb = 0; kb < C::D / 16; ++kb) {
          const int box = kb / 4, off = (kb % 4) * 32;
          umma_ss<false>(tmem + C::TM_DPT,
                         sdesc_sw128(sbase + C::SMEM_V + box * C::BN * 128 + off, 16, 1024),
                         sdesc_sw128(dob + box * C::BMQ * 128 + off, 16, 1024), ID_T, kb > 0);
        }
        tc_commit(bar(C::B_SDP));
        // dV += P^T dO[:, half]   (A = P^T bf16 in TMEM over the S^T columns)
        if (!(ok = mbar_wait(bar(C::B_P), st & 1, wc, kSitePFull))) break;
        tc_fence_after();
        const int hbox = split * (C::DH / 64);
#pragma unroll
        for (int kb = 0; kb < C::BMQ / 16; ++kb)
          umma_ts<false>(tmem + C::TM_DV, tmem + C::TM_ST + kb * 8,
                         sdesc_sw128(dob + hbox * C::BMQ * 128 + kb * 16 * 128, C::BMQ * 128, 1024),
                         ID_G, (st > 0 || kb > 0) ? 1u : 0u);
        // dK += dS^T Q[:, half]   (A = dS^T bf16 in TMEM over the dP^T columns)
        if (!(ok = mbar_wait(bar(C::B_DS), st & 1, wc, kSiteDsFull))) break;
        tc_fence_after();
#pragma unroll
        for (int kb = 0; kb < C::BMQ / 16; ++kb)
          umma_ts<false>(tmem + C::TM_DK, tmem + C::TM_DPT + kb * 8,
                         sdesc_sw128(qb + hbox * C::BMQ * 128 + kb * 16 * 128, C::BMQ * 128, 1024),
                         ID_G, (st > 0 || kb > 0) ? 1u : 0u);
        tc_commit(bar(C::B_EMPTY + s));
      }
      tc_commit(bar(C::B_ACC));
      tc_commit(bar(C::B_DRAIN));
      if (!mbar_wait_drain(bar(C::B_DRAIN), 0, wc.timeout_ns))
        atomicCAS(wc.status, 0u, kStatusTimeout | kSiteDrain);
    }
  } else {
    // ---------------- compute warps: thread owns key row `row`
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int kv = kt * C::BN + row;
    const uint32_t lb = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float LOG2E = 1.4426950408889634f;
    const float sl2 = p.scale * LOG2E;
    bool ok = true;
    for (int st = 0; st < nsteps && ok; ++st) {
      const int s = st % C::STAGES;
      const int qi = i0 + st;
      if (!(ok = mbar_wait(bar(C::B_FULL + s), (st / C::STAGES) & 1, wc, kSiteQFull))) break;
      if (!(ok = mbar_wait(bar(C::B_SDP), st & 1, wc, kSiteSFull))) break;
      tc_fence_after();
      const float* ls = lse_s + s * C::BMQ;
      const float* ds_ = dd_s + s * C::BMQ;
      // P^T row: p_c = 2^(s_c*sl2 - lse_c*log2e), zero where the query may not see this key
      float pr[C::BMQ];
#pragma unroll
      for (int c0 = 0; c0 < C::BMQ; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lb + C::TM_ST + c0, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int q = qi * C::BMQ + c0 + i;
          const bool vis = (q < p.N) && (kv < p.N) && (!p.causal || kv <= q);
          pr[c0 + i] = vis ? ex2(fmaf(__uint_as_float(r[i]), sl2, -ls[c0 + i] * LOG2E)) : 0.f;
        }
      }
#pragma unroll
      for (int c0 = 0; c0 < C::BMQ; c0 += 64) {
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = pack_bf16x2(pr[c0 + 2 * i], pr[c0 + 2 * i + 1]);
        tmem_st32(lb + C::TM_ST + c0 / 2, r);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(bar(C::B_P));
      // dS^T row = P^T * (dP^T - D_q), written as bf16 over the consumed dP^T columns
#pragma unroll
      for (int c0 = 0; c0 < C::BMQ; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lb + C::TM_DPT + c0, r);
        tmem_ld_wait(r);
        uint32_t w16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float a = pr[c0 + 2 * i] * (__uint_as_float(r[2 * i]) - ds_[c0 + 2 * i]);
          const float b = pr[c0 + 2 * i + 1] * (__uint_as_float(r[2 * i + 1]) - ds_[c0 + 2 * i + 1]);
          w16[i] = pack_bf16x2(a, b);
        }
        tmem_st16(lb + C::TM_DPT + c0 / 2, w16);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(bar(C::B_DS));
    }
    // epilogue: dV and scale*dK -> bf16 global
    if (ok && mbar_wait(bar(C::B_ACC), 0, wc, kSiteDqDone)) {
      tc_fence_after();
      const bool row_ok = kv < p.N;
      const size_t base = (static_cast<size_t>(bh) * p.N + kv) * C::D + split * C::DH;
      __nv_bfloat16* dvp = reinterpret_cast<__nv_bfloat16*>(p.dv) + base;
      __nv_bfloat16* dkp = reinterpret_cast<__nv_bfloat16*>(p.dk) + base;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t col0 = which == 0 ? C::TM_DV : C::TM_DK;
        const float mul = which == 0 ? 1.f : p.scale;
        __nv_bfloat16* dst = which == 0 ? dvp : dkp;
#pragma unroll 1
        for (int c = 0; c < C::DH; c += 32) {
          uint32_t r[32];
          tmem_ld32(lb + col0 + c, r);
          tmem_ld_wait(r);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
          if (row_ok) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

// --------------------------------------------------------------------------- 3. dQ
template <int D_, int BN_, int STAGES_>
struct DqCfg {
  static constexpr int D = D_;
  static constexpr int BN = BN_;        // streamed key rows
  static constexpr int BM = 128;        // query rows of the CTA = TMEM lanes
  static constexpr int STAGES = STAGES_;
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int NBOX = ROW_BYTES / 128;
  static constexpr int QT_BYTES = BM * ROW_BYTES;
  static constexpr int KT_BYTES = BN * ROW_BYTES;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_DO = QT_BYTES;
  static constexpr int SMEM_K = 2 * QT_BYTES;
  static constexpr int SMEM_V = SMEM_K + STAGES * KT_BYTES;
  static constexpr int SMEM_BAR = SMEM_V + STAGES * KT_BYTES;
  static constexpr int B_QDO = 0, B_SDP = 1, B_DS = 2, B_ACC = 3, B_DRAIN = 4, B_FULL = 5,
                       B_EMPTY = 5 + STAGES, NBARS = 5 + 2 * STAGES;
  static constexpr int SMEM_MISC = SMEM_BAR + NBARS * 8;
  static constexpr int SMEM_ALLOC = SMEM_MISC + 64 + 1024;
  static constexpr int TM_S = 0, TM_DP = BN, TM_DQ = 2 * BN;
  static constexpr int TM_COLS = 512;
  static constexpr int THREADS = 192;
  static_assert(2 * BN + D <= TM_COLS, "tensor memory budget");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    fa_bwd_dq(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
              const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::SMEM_BAR;
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;

  // block -> (bh, q tile); highest causal q tile (most key tiles) first
  const int bh = blockIdx.x / p.n_qt;
  const int qt = p.n_qt - 1 - (blockIdx.x - bh * p.n_qt);
  const int nsteps = p.causal ? min(p.n_kt, ((qt + 1) * C::BM - 1) / C::BN + 1) : p.n_kt;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBARS; ++i) mbar_init(bar(i), i == C::B_DS ? 4u : 1u);   // 4 warps
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
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(bar(C::B_QDO), 2 * C::QT_BYTES);
      for (int c = 0; c < C::NBOX; ++c) {
        tma_load_3d(sbase + C::SMEM_Q + c * C::BM * 128, &tq, bar(C::B_QDO), c * 64, qt * C::BM, bh);
        tma_load_3d(sbase + C::SMEM_DO + c * C::BM * 128, &tdo, bar(C::B_QDO), c * 64, qt * C::BM, bh);
      }
      for (int j = 0; j < nsteps && ok; ++j) {
        const int s = j % C::STAGES;
        if (j >= C::STAGES &&
            !(ok = mbar_wait(bar(C::B_EMPTY + s), ((j / C::STAGES) - 1) & 1, wc, kSiteKVEmpty)))
          break;
        mbar_arrive_expect_tx(bar(C::B_FULL + s), 2 * C::KT_BYTES);
        for (int c = 0; c < C::NBOX; ++c) {
          tma_load_3d(sbase + C::SMEM_K + s * C::KT_BYTES + c * C::BN * 128, &tk, bar(C::B_FULL + s),
                      c * 64, j * C::BN, bh);
          tma_load_3d(sbase + C::SMEM_V + s * C::KT_BYTES + c * C::BN * 128, &tv, bar(C::B_FULL + s),
                      c * 64, j * C::BN, bh);
        }
      }
      if (ok) {
        for (int j = (nsteps > C::STAGES ? nsteps - C::STAGES : 0); ok && j < nsteps; ++j)
          ok = mbar_wait(bar(C::B_EMPTY + j % C::STAGES), (j / C::STAGES) & 1, wc, kSiteKVEmpty);
      } else {
        mbar_wait_drain(bar(C::B_QDO), 0, 100000000ull);
        for (int j = (nsteps > C::STAGES ? nsteps - C::STAGES : 0); j < nsteps; ++j)
          mbar_wait_drain(bar(C::B_FULL + j % C::STAGES), (j / C::STAGES) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16(128, C::BN, false);
      constexpr uint32_t ID_Q = idesc_bf16(128, C::D, true);
      bool ok = mbar_wait(bar(C::B_QDO), 0, wc, kSiteQFull);
      for (int j = 0; j < nsteps && ok; ++j) {
        const int s = j % C::STAGES;
        if (!(ok = mbar_wait(bar(C::B_FULL + s), (j / C::STAGES) & 1, wc, kSiteKFull))) break;
        tc_fence_after();
        const uint32_t kb_ = sbase + C::SMEM_K + s * C::KT_BYTES;
        const uint32_t vb_ = sbase + C::SMEM_V + s * C::KT_BYTES;
#pragma unroll
        for (int kb = 0; kb < C::D / 16; ++kb) {
          const int box = kb / 4, off = (kb % 4) * 32;
          umma_ss<false>(tmem + C::TM_S, sdesc_sw128(sbase + C::SMEM_Q + box * C::BM * 128 + off, 16, 1024),
                         sdesc_sw128(kb_ + box * C::BN * 128 + off, 16, 1024), ID_S, kb > 0);
        }
#pragma unroll
        for (int kb = 0; kb < C::D / 16; ++kb) {
          const int box = kb / 4, off = (kb % 4) * 32;
          umma_ss<false>(tmem + C::TM_DP, sdesc_sw128(sbase + C::SMEM_DO + box * C::BM * 128 + off, 16, 1024),
                         sdesc_sw128(vb_ + box * C::BN * 128 + off, 16, 1024), ID_S, kb > 0);
        }
        tc_commit(bar(C::B_SDP));
        if (!(ok = mbar_wait(bar(C::B_DS), j & 1, wc, kSiteDsFull))) break;
        tc_fence_after();
        // dQ += dS K_j: A = dS (query rows x key cols) bf16 in TMEM, B = K_j MN-major
#pragma unroll
        for (int kb = 0; kb < C::BN / 16; ++kb)
          umma_ts<false>(tmem + C::TM_DQ, tmem + C::TM_DP + kb * 8,
                         sdesc_sw128(kb_ + kb * 16 * 128, C::BN * 128, 1024), ID_Q,
                         (j > 0 || kb > 0) ? 1u : 0u);
        tc_commit(bar(C::B_EMPTY + s));
      }
      tc_commit(bar(C::B_ACC));
      tc_commit(bar(C::B_DRAIN));
      if (!mbar_wait_drain(bar(C::B_DRAIN), 0, wc.timeout_ns))
        atomicCAS(wc.status, 0u, kStatusTimeout | kSiteDrain);
    }
  } else {
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int q = qt * C::BM + row;
    const uint32_t lb = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float LOG2E = 1.4426950408889634f;
    const float sl2 = p.scale * LOG2E;
    const bool row_ok = q < p.N;
    const float lse2 = row_ok ? p.lse[static_cast<size_t>(bh) * p.N + q] * LOG2E : 0.f;
    const float dq_i = row_ok ? p.drow[static_cast<size_t>(bh) * p.N + q] : 0.f;
    bool ok = true;
    for (int j = 0; j < nsteps && ok; ++j) {
      if (!(ok = mbar_wait(bar(C::B_SDP), j & 1, wc, kSiteSFull))) break;
      tc_fence_after();
      float pr[C::BN];
#pragma unroll
      for (int c0 = 0; c0 < C::BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lb + C::TM_S + c0, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int kv = j * C::BN + c0 + i;
          const bool vis = row_ok && (kv < p.N) && (!p.causal || kv <= q);
          pr[c0 + i] = vis ? ex2(fmaf(__uint_as_float(r[i]), sl2, -lse2)) : 0.f;
        }
      }
#pragma unroll
      for (int c0 = 0; c0 < C::BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lb + C::TM_DP + c0, r);
        tmem_ld_wait(r);
        uint32_t w16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w16[i] = pack_bf16x2(pr[c0 + 2 * i] * (__uint_as_float(r[2 * i]) - dq_i),
                               pr[c0 + 2 * i + 1] * (__uint_as_float(r[2 * i + 1]) - dq_i));
        tmem_st16(lb + C::TM_DP + c0 / 2, w16);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(bar(C::B_DS));
    }
    if (ok && mbar_wait(bar(C::B_ACC), 0, wc, kSiteDqDone)) {
      tc_fence_after();
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.dq) + (static_cast<size_t>(bh) * p.N + q) * C::D;
#pragma unroll 1
      for (int c = 0; c < C::D; c += 32) {
        uint32_t r[32];
        tmem_ld32(lb + C::TM_DQ + c, r);
        tmem_ld_wait(r);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * p.scale, __uint_as_float(r[2 * i + 1]) * p.scale);
        if (row_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

}  // namespace fa
