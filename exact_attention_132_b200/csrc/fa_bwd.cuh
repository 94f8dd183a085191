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
//                      memory, and streams the query tiles.  Lane t of the compute
//                      warps owns key row t (transposed tiles S^T, dP^T).
//   3. fa_bwd_dq       one CTA per (head, 128-row query tile); it keeps Q, dO in
//                      shared memory and dQ in tensor memory, and streams K/V.
// Splitting dQ into its own pass costs a second recompute of S and dP but needs
// no fp32 atomics and is deterministic.
//
// At d = 64 (tensor memory has room there) the dK/dV pass also produces dQ:
//   dQ_i += dS_i K                                      (tensor core, A = dS from smem)
// accumulated in fp32 in the caller's workspace by TMA reduce-adds (each compute warp
// stages its 32 x 32 block in shared memory, warp 10 issues the adds), the sums zeroed
// by pass 1;
// a fourth kernel, fa_bwd_dq_convert, writes dQ = scale dQ_acc in bf16, and pass 3 is
// not run (a build choice: the pages give only the recompute).  The fp32 sums' order,
// and so dQ's last bits, vary from run to run.
//
// Roles in kernels 2 and 3: warps 0..7 elementwise work (two warps per TMEM lane
// quadrant, each on half of the streamed tile's columns), warp 8 TMA producer, warp 9
// MMA issuer (one elected lane issues; owns tensor memory); at d = 64, warp 10 issues
// the dQ reduce-adds.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

struct BwdParams {
  int BH, N;             // BH = B * H query heads
  int H;                 // query heads per batch entry
  int g;                 // query heads per key/value head (1 = one K/V head per query head)
  int ld;                // head dim as stored (row length of every bf16 tensor); the kernel's
                         // D may be larger: columns past ld load as zeros, are not stored
  int n_qt;              // query tiles of BMQ rows (dK/dV pass) / 128 rows (dQ pass)
  int n_kt;              // key tiles
  int causal;
  int group_heads;       // heads per level-major sweep of the CTA order (bwd_block_item)
  float scale;
  const float* lse;      // [BH, N]
  const float* drow;     // D_i workspace [BH, N]
  float* dq_acc;         // fused d = 64 dK/dV pass: fp32 [BH, N, 64] dQ sums, zeroed by pass 1
  void* dq;              // bf16 [BH, N, D]
  void* dk;
  void* dv;
  unsigned* status;
  unsigned long long timeout_ns;
};

// CTA -> (head, level, part).  Heads go in groups of p.group_heads; inside a group the
// order is level-major: level 0 (the heaviest causal tile) of every head of the group,
// then level 1, ...  The hardware hands out CTAs in index order, so the long tiles
// start first and the short ones fill the end (a head-major order leaves the last
// heads' long tiles running alone), while the CTAs in flight together stream only one
// group's operands through L2.
__device__ __forceinline__ void bwd_block_item(int block, int heads, int levels, int parts,
                                               int group, int& head, int& lvl, int& part) {
  part = block % parts;
  int r = block / parts;
  const int per_group = group * levels;
  const int gi = r / per_group;
  r -= gi * per_group;
  const int gsize = min(group, heads - gi * group);
  lvl = r / gsize;
  head = gi * group + (r - lvl * gsize);
}

// --------------------------------------------------------------------------- 1. D_i
// D_i = sum_c dO_ic * O_ic, fp32 accumulation of the bf16 products.  A row of D
// elements is D/8 16-byte pieces; TPR threads (a power of two) share a row, PER pieces
// each: D = 64 -> 8 x 1, 128 -> 16 x 1, 256 -> 32 x 1, 96 -> 4 x 3, 192 -> 8 x 3.
// With dq_acc (rows of D fp32 values, D = 64 only) the pass also zeroes each row's dQ
// accumulator.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_rowdot(const __nv_bfloat16* __restrict__ o,
                                                     const __nv_bfloat16* __restrict__ dout,
                                                     float* __restrict__ drow, long long rows,
                                                     float* __restrict__ dq_acc) {
  constexpr int PIECES = D / 8;
  constexpr int PER = (PIECES % 3 == 0) ? 3 : 1;   // pieces per thread
  constexpr int TPR = PIECES / PER;                  // threads per row
  static_assert((TPR & (TPR - 1)) == 0 && TPR <= 32, "power-of-two threads per row");
  constexpr int RPB = 256 / TPR;                     // rows per block pass
  const int sub = threadIdx.x % TPR;
  for (long long r = static_cast<long long>(blockIdx.x) * RPB + threadIdx.x / TPR; r < rows;
       r += static_cast<long long>(gridDim.x) * RPB) {
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const uint4 a = reinterpret_cast<const uint4*>(o + r * D)[sub * PER + u];
      const uint4 b = reinterpret_cast<const uint4*>(dout + r * D)[sub * PER + u];
      const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 fa2 = __bfloat1622float2(ha[i]);
        const float2 fb2 = __bfloat1622float2(hb[i]);
        acc = fmaf(fa2.x, fb2.x, acc);
        acc = fmaf(fa2.y, fb2.y, acc);
      }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (sub == 0) drow[r] = acc;
    if (dq_acc != nullptr) {
      float4* z = reinterpret_cast<float4*>(dq_acc + r * D);
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        z[2 * (sub * PER + u)] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[2 * (sub * PER + u) + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
}

// --------------------------------------------------------------------------- 4. dQ (fused)
// dQ = scale * dQ_acc -> bf16, eight values per thread step (rows of 64, stored = kernel
// head dim).  A programmatic dependent of the dK/dV pass: waits for all its sums.
__global__ void __launch_bounds__(256) fa_bwd_dq_convert(const float* __restrict__ acc,
                                                         __nv_bfloat16* __restrict__ dq,
                                                         long long n8, float scale) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * 256) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    reinterpret_cast<uint4*>(dq)[i] =
        make_uint4(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale),
                   pack_bf16x2(b.x * scale, b.y * scale), pack_bf16x2(b.z * scale, b.w * scale));
  }
}

// --------------------------------------------------------------------------- 2. dK, dV
// One CTA per (head, 128-row key tile[, part of d]).  K and V stay in shared memory,
// dV and dK accumulate in tensor memory, and the query tiles stream through a ring.
// Per query tile i (BMQ rows):
//   S^T = K Q_i^T, dP^T = V dO_i^T                      (tensor core, into TMEM)
//   P^T = 2^(S^T scale log2e - lse_i log2e)           (compute warps, bf16 over S^T)
//   dV += P^T dO_i                                      (tensor core, A = P^T from TMEM)
//   dS^T = P^T (dP^T - D_i)                             (compute warps, bf16 over dP^T)
//   dK += dS^T Q_i                                      (tensor core, A = dS^T from TMEM)
// S^T and dP^T have SB / DB buffers, so the products of tile i+1 run on the tensor
// core while the compute warps work on tile i.  Q_i (with lse_i) and dO_i (with D_i)
// stream through rings of their own, QST and OST deep: dO_i is free once dV has read
// it, Q_i only after dK, so at d = 256, where shared memory holds three query-tile
// slots, Q gets two and dO one.  Eight compute warps: two per TMEM lane
// quadrant, each owning half of the BMQ query columns (P needs no row reduction, so
// the halves never talk to each other).  Each half writes its bf16 P^T / dS^T into
// the first half of its own column range.
template <int D_, int DH_, int BMQ_, int QST_, int OST_, int SB_, int DB_, int EMU_ = 1,
          bool FUSEDQ_ = false>
struct DkdvCfg {
  static constexpr int D = D_;          // head dim (contraction of S^T and dP^T)
  static constexpr int DH = DH_;        // columns of dK/dV this CTA produces
  static constexpr int NSPLIT = D / DH;
  static constexpr int BMQ = BMQ_;      // query rows per streamed tile
  static constexpr int BN = 128;        // key rows of the CTA = TMEM lanes
  static constexpr int QST = QST_, OST = OST_;
  static constexpr int SB = SB_, DB = DB_;
  static constexpr int EMU = EMU_;      // software exp2 share, in quarters
  static constexpr int CH = BMQ / 2;    // query columns per compute warp
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int NBOX = ROW_BYTES / 128;
  static constexpr int KT_BYTES = BN * ROW_BYTES;       // K or V tile
  static constexpr int QT_BYTES = BMQ * ROW_BYTES;      // Q_i or dO_i tile
  static constexpr int SMEM_K = 0;
  static constexpr int SMEM_V = KT_BYTES;
  static constexpr int SMEM_Q = 2 * KT_BYTES;
  static constexpr int SMEM_DO = SMEM_Q + QST * QT_BYTES;
  static constexpr int SMEM_LSE = SMEM_DO + OST * QT_BYTES;       // [QST][BMQ] fp32
  // D_i has one slot more than dO: the producer refills a slot once dV has read the dO
  // tile OST steps back, which can precede the compute warps' last use of that step's
  // D_i by one step
  static constexpr int DDR = OST + 1;
  static constexpr int SMEM_DD = SMEM_LSE + QST * BMQ * 4;        // [DDR][BMQ] fp32
  // Fused dQ (d = 64): dS^T also goes to shared memory in bf16, as two 128-byte
  // swizzled boxes of 64 query columns x BN key rows.  Read column-wise, that is the
  // A operand (MN-major) of dQ_i = dS_i K; K's resident tile is its B operand
  // (MN-major, like V in the forward's P V).  dQ_i lands in the middle BMQ/2 columns
  // of the step's S^T buffer: the halves' packed P^T sit at its two ends (PACK_HI).
  static constexpr bool FUSEDQ = FUSEDQ_;
  static constexpr int SMEM_DS =
      FUSEDQ ? (SMEM_DD + DDR * BMQ * 4 + 1023) / 1024 * 1024 : SMEM_DD + DDR * BMQ * 4;
  static constexpr int DS_BOX = BN * 128;                 // one box of 64 query columns
  // and one 4 KB staging block per compute warp for its dQ reduce-add (32 rows x 32
  // fp32, 128-byte swizzled)
  static constexpr int SMEM_DQ = SMEM_DS + (FUSEDQ ? BN * BMQ * 2 : 0);
  static constexpr int SMEM_BAR = SMEM_DQ + (FUSEDQ ? 8 * 4096 : 0);
  static constexpr int PACK_HI = FUSEDQ ? BMQ - BMQ / 4 : BMQ / 2;
  static constexpr int TM_DQ_OFF = BMQ / 4;
  static constexpr int B_KV = 0, B_ACC = 1, B_DRAIN = 2,
                       B_SFULL = 3, B_P = 3 + SB,                   // + buffer
                       B_DPFULL = 3 + 2 * SB, B_DS = 3 + 2 * SB + DB,
                       B_QFULL = 3 + 2 * SB + 2 * DB, B_QEMPTY = B_QFULL + QST,
                       B_OFULL = B_QEMPTY + QST, B_OEMPTY = B_OFULL + OST,
                       B_DQFULL = B_OEMPTY + OST, B_DQFREE = B_DQFULL + 1,
                       B_DQSTG = B_DQFULL + 2,    // fused dQ: the 8 blocks of a step are staged
                       B_DQSFR = B_DQFULL + 3,    // fused dQ: their reduce-adds have read them
                       NBARS = B_OEMPTY + OST + (FUSEDQ ? 4 : 0);
  static constexpr int SMEM_MISC = SMEM_BAR + NBARS * 8;
  static constexpr int SMEM_ALLOC = SMEM_MISC + 64 + 1024;
  static constexpr int TM_ST = 0;                        // + b * BMQ
  static constexpr int TM_DPT = SB * BMQ;                // + b * BMQ
  static constexpr int TM_DV = (SB + DB) * BMQ, TM_DK = TM_DV + DH;
  static constexpr int TM_COLS = 512;
  // 8 compute warps, producer, MMA; fused dQ: one more warp issues the dQ reduce-adds
  static constexpr int THREADS = FUSEDQ ? 352 : 320;
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9, REDUCE_WARP = FUSEDQ ? 10 : -1;
  static_assert((SB + DB) * BMQ + 2 * DH <= TM_COLS, "tensor memory budget");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(BMQ % 64 == 0 && DH % 64 == 0 && CH % 32 == 0, "box and TMEM chunk sizes");
  static_assert(SB >= 1 && SB <= 2 && DB >= 1 && DB <= 2, "one or two buffers");
  static_assert(!FUSEDQ || (D == 64 && DH == 64 && BMQ == 128 && SB == 2 && DB == 1),
                "fused dQ: d = 64, 128-row query tiles, two S^T buffers, one dP^T buffer");
};

template <class C>
__device__ __forceinline__ void dkdv_q_range(const BwdParams& p, int kt, int& i0, int& i1) {
  i1 = p.n_qt;
  i0 = p.causal ? (kt * C::BN) / C::BMQ : 0;   // first query tile that reaches key kt*128
}

// A = (BMQ x 128)^T operand kb (16 query columns) of the bf16 tile written over a
// BMQ-column fp32 buffer: half h of the columns keeps its values in its own range.
// The second half's values start at column HI (BMQ / 2: each half at the start of
// its own range).
template <int BMQ, int HI = BMQ / 2>
__device__ __forceinline__ uint32_t half_packed_col(int kb) {
  constexpr int KB_H = BMQ / 2 / 16;      // 16-column blocks per half
  return (kb / KB_H) * HI + (kb % KB_H) * 8;
}

// 2^x of an even-length row segment into `pr`: EMU of every 4 pairs on the FMA pipe,
// the rest on the special-function unit.  x = s * c - b, with b per element (a query
// column's lse) or one value for the whole segment (the row's lse).
__device__ __forceinline__ void exp2_pair_into(uint64_t x2, bool soft, float& a, float& b) {
  if (soft) {
    f2_unpack(ex2_poly_pair(x2), a, b);
  } else {
    float xa, xb;
    f2_unpack(x2, xa, xb);
    a = ex2(xa);
    b = ex2(xb);
  }
}
template <int N, int EMU>
__device__ __forceinline__ void exp2_row(const uint32_t (&r)[N], float c, const float* b, float (&pr)[N]) {
  const uint64_t c2 = f2_pack(c, c);
#pragma unroll
  for (int i = 0; i < N; i += 2) {
    const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), c2,
                               f2_pack(-b[i], -b[i + 1]));
    exp2_pair_into(x2, (i / 2) % 4 < EMU, pr[i], pr[i + 1]);
  }
}
template <int N, int EMU>
__device__ __forceinline__ void exp2_row(const uint32_t (&r)[N], float c, float b, float (&pr)[N]) {
  const uint64_t c2 = f2_pack(c, c), nb2 = f2_pack(-b, -b);
#pragma unroll
  for (int i = 0; i < N; i += 2) {
    const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), c2, nb2);
    exp2_pair_into(x2, (i / 2) % 4 < EMU, pr[i], pr[i + 1]);
  }
}

// Launched as a programmatic dependent of the row-dot pass: it waits for that grid (its
// D_i rows) before anything else, then lets the dQ pass be scheduled, so the dQ CTAs
// fill the SMs this pass's last wave leaves idle (the two passes are independent).
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    fa_bwd_dkdv(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                const __grid_constant__ CUtensorMap tdq, const BwdParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + C::SMEM_BAR;
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_MISC + 4);
  float* lse_s = reinterpret_cast<float*>(smem + C::SMEM_LSE);   // lse * log2(e)
  float* dd_s = reinterpret_cast<float*>(smem + C::SMEM_DD);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const float LOG2E = 1.4426950408889634f;

  // block -> (key/value head, key tile, d part); heaviest causal tiles (small kt) first.
  // With grouped heads the g query heads reading this K/V head all contribute to its
  // dK, dV: the steps run over (query head of the group, query tile).
  int split, kt, bh;                                  // bh: key/value head (b * H / g + h / g)
  bwd_block_item(blockIdx.x, p.BH / p.g, p.n_kt, C::NSPLIT, p.group_heads, bh, kt, split);
  int i0, i1;
  dkdv_q_range<C>(p, kt, i0, i1);
  const int nqt = i1 - i0;                            // query tiles per query head
  const int nsteps = nqt * p.g;
  const int hkv_per_b = p.H / p.g;
  const int bq0 = (bh / hkv_per_b) * p.H + (bh % hkv_per_b) * p.g;   // first query head
  // step -> (query head, query tile index)
  auto q_head = [&](int st) { return bq0 + st / nqt; };
  auto q_tile = [&](int st) { return i0 + st % nqt; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBARS; ++i) {
      const bool warps8 = (i >= C::B_P && i < C::B_P + C::SB) || (i >= C::B_DS && i < C::B_DS + C::DB) ||
                          (C::FUSEDQ && (i == C::B_DQFREE || i == C::B_DQSTG));
      mbar_init(bar(i), warps8 ? 8u : 1u);                  // 8 compute warps arrive
    }
    *abort_flag = 0;
    fence_mbar_init();
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
    // ---------------- producer (whole warp: lanes stage lse/D, one lane issues TMA)
    bool ok = true;
    if (elect_one()) {
      mbar_arrive_expect_tx(bar(C::B_KV), 2 * C::KT_BYTES);
      for (int c = 0; c < C::NBOX; ++c) {
        tma_load_3d(sbase + C::SMEM_K + c * C::BN * 128, &tk, bar(C::B_KV), c * 64, kt * C::BN, bh);
        tma_load_3d(sbase + C::SMEM_V + c * C::BN * 128, &tv, bar(C::B_KV), c * 64, kt * C::BN, bh);
      }
    }
    __syncwarp();
    // Q_i (and lse_i) into its ring, then dO_i (and D_i) into its own.  Q_i first: the
    // MMA warp may ask for Q_i (an early S^T) before it has issued the dV product that
    // frees the dO slot.  lse and D of the next tile are fetched into registers one
    // step ahead, so their global-load latency overlaps this step's waits.
    constexpr int PL = C::BMQ / 32;          // values per lane
    float lse_n[PL], dd_n[PL];
    auto fetch = [&](int st) {
#pragma unroll
      for (int i = 0; i < PL; ++i) {
        const int q = q_tile(st) * C::BMQ + lane + 32 * i;
        const bool in = q < p.N;
        const size_t hq = static_cast<size_t>(q_head(st));
        lse_n[i] = in ? p.lse[hq * p.N + q] * LOG2E : 0.f;
        dd_n[i] = in ? p.drow[hq * p.N + q] : 0.f;
      }
    };
    if (nsteps > 0) fetch(0);
    int nq = 0, no = 0;                      // tiles issued per ring
    for (int st = 0; st < nsteps && ok; ++st) {
      const int qi = q_tile(st), hq = q_head(st);
      const int so = st % C::OST, sq = st % C::QST;
      float lse_c[PL], dd_c[PL];
#pragma unroll
      for (int i = 0; i < PL; ++i) {
        lse_c[i] = lse_n[i];
        dd_c[i] = dd_n[i];
      }
      if (st + 1 < nsteps) fetch(st + 1);
      if (st >= C::QST &&
          !(ok = mbar_wait_warp(bar(C::B_QEMPTY + sq), ((st / C::QST) - 1) & 1, wc, kSiteKVEmpty)))
        break;
#pragma unroll
      for (int i = 0; i < PL; ++i) lse_s[sq * C::BMQ + lane + 32 * i] = lse_c[i];
      __syncwarp();
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(C::B_QFULL + sq), C::QT_BYTES);
        for (int c = 0; c < C::NBOX; ++c)
          tma_load_3d(sbase + C::SMEM_Q + sq * C::QT_BYTES + c * C::BMQ * 128, &tq,
                      bar(C::B_QFULL + sq), c * 64, qi * C::BMQ, hq);
      }
      __syncwarp();
      ++nq;
      if (st >= C::OST &&
          !(ok = mbar_wait_warp(bar(C::B_OEMPTY + so), ((st / C::OST) - 1) & 1, wc, kSiteKVEmpty)))
        break;
#pragma unroll
      for (int i = 0; i < PL; ++i) dd_s[(st % C::DDR) * C::BMQ + lane + 32 * i] = dd_c[i];
      __syncwarp();
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(C::B_OFULL + so), C::QT_BYTES);
        for (int c = 0; c < C::NBOX; ++c)
          tma_load_3d(sbase + C::SMEM_DO + so * C::QT_BYTES + c * C::BMQ * 128, &tdo,
                      bar(C::B_OFULL + so), c * 64, qi * C::BMQ, hq);
      }
      __syncwarp();
      ++no;
    }
    if (ok) {
      for (int st = (nsteps > C::OST ? nsteps - C::OST : 0); ok && st < nsteps; ++st)
        ok = mbar_wait_warp(bar(C::B_OEMPTY + st % C::OST), (st / C::OST) & 1, wc, kSiteKVEmpty);
      for (int st = (nsteps > C::QST ? nsteps - C::QST : 0); ok && st < nsteps; ++st)
        ok = mbar_wait_warp(bar(C::B_QEMPTY + st % C::QST), (st / C::QST) & 1, wc, kSiteKVEmpty);
    } else {
      mbar_wait_drain(bar(C::B_KV), 0, 100000000ull);
      for (int st = (no > C::OST ? no - C::OST : 0); st < no; ++st)
        mbar_wait_drain(bar(C::B_OFULL + st % C::OST), (st / C::OST) & 1, 100000000ull);
      for (int st = (nq > C::QST ? nq - C::QST : 0); st < nq; ++st)
        mbar_wait_drain(bar(C::B_QFULL + st % C::QST), (st / C::QST) & 1, 100000000ull);
    }
  } else if (warp == C::MMA_WARP) {
    // ---------------- MMA issuer (whole warp, one elected lane issues)
    constexpr uint32_t ID_T = idesc_bf16(128, C::BMQ, false);    // S^T, dP^T: 128 x BMQ
    constexpr uint32_t ID_G = idesc_bf16(128, C::DH, true);      // dV, dK: 128 x DH, B MN-major
    const int hbox = split * (C::DH / 64);
    auto qbuf = [&](int st) { return sbase + C::SMEM_Q + (st % C::QST) * C::QT_BYTES; };
    auto dobuf = [&](int st) { return sbase + C::SMEM_DO + (st % C::OST) * C::QT_BYTES; };
    // S^T(st) = K Q^T and, with it or later, dP^T(st) = V dO^T
    auto issue_st = [&](int st) -> bool {
      if (!mbar_wait_warp(bar(C::B_QFULL + st % C::QST), (st / C::QST) & 1, wc, kSiteQFull))
        return false;
      tc_fence_after();
#pragma unroll
      for (int kb = 0; kb < C::D / 16; ++kb) {
        const int box = kb / 4, off = (kb % 4) * 32;
        umma_ss_elect(false, tmem + C::TM_ST + (st % C::SB) * C::BMQ,
                      sdesc_sw128(sbase + C::SMEM_K + box * C::BN * 128 + off, 16, 1024),
                      sdesc_sw128(qbuf(st) + box * C::BMQ * 128 + off, 16, 1024), ID_T, kb > 0);
      }
      tc_commit_elect(bar(C::B_SFULL + st % C::SB));
      return true;
    };
    auto issue_dpt = [&](int st) -> bool {
      if (!mbar_wait_warp(bar(C::B_OFULL + st % C::OST), (st / C::OST) & 1, wc, kSiteQFull))
        return false;
      tc_fence_after();
#pragma unroll
      for (int kb = 0; kb < C::D / 16; ++kb) {
        const int box = kb / 4, off = (kb % 4) * 32;
        umma_ss_elect(false, tmem + C::TM_DPT + (st % C::DB) * C::BMQ,
                      sdesc_sw128(sbase + C::SMEM_V + box * C::BN * 128 + off, 16, 1024),
                      sdesc_sw128(dobuf(st) + box * C::BMQ * 128 + off, 16, 1024), ID_T, kb > 0);
      }
      tc_commit_elect(bar(C::B_DPFULL + st % C::DB));
      return true;
    };
    bool ok = mbar_wait_warp(bar(C::B_KV), 0, wc, kSiteKFull);
    // prologue: tile 0's products, then tile 1's where the buffers allow
    if (ok && nsteps > 0) {
      ok = issue_st(0) && issue_dpt(0);
    }
    // Tile st+1's products go ahead of tile st's gradient products when they have a
    // buffer of their own and their operand tile can already be resident (a second
    // ring slot); otherwise they follow them.
    // fused dQ: S^T(st+1) goes into the buffer that holds dQ(st-1), once the compute
    // warps have drained it (after dV(st), below)
    constexpr bool EARLY_S = C::SB == 2 && C::QST >= 2 && !C::FUSEDQ;
    constexpr bool EARLY_DP = EARLY_S && C::DB == 2 && C::OST >= 2;
    // one S^T buffer: S^T(st+1) goes right behind dV(st), the last reader of P^T(st), so
    // the tensor core computes it while the compute warps form dS^T(st)
    constexpr bool S_AFTER_DV = C::SB == 1 && !C::FUSEDQ;
    for (int st = 0; st < nsteps && ok; ++st) {
      const int nx = st + 1;
      // S^T(st+1) into the other buffer (its last reader, dV(st+1-SB), is issued)
      if (EARLY_S && nx < nsteps && !(ok = issue_st(nx))) break;
      if (EARLY_DP && nx < nsteps && !(ok = issue_dpt(nx))) break;
      // dV += P^T dO[:, part]   (A = P^T bf16 in TMEM over the S^T columns)
      if (!(ok = mbar_wait_warp(bar(C::B_P + st % C::SB), (st / C::SB) & 1, wc, kSitePFull))) break;
      tc_fence_after();
      const uint32_t stb = tmem + C::TM_ST + (st % C::SB) * C::BMQ;
#pragma unroll
      for (int kb = 0; kb < C::BMQ / 16; ++kb)
        umma_ts_elect(false, tmem + C::TM_DV, stb + half_packed_col<C::BMQ, C::PACK_HI>(kb),
                      sdesc_sw128(dobuf(st) + hbox * C::BMQ * 128 + kb * 16 * 128, C::BMQ * 128, 1024),
                      ID_G, (st > 0 || kb > 0) ? 1u : 0u);
      tc_commit_elect(bar(C::B_OEMPTY + st % C::OST));     // dP^T(st) and dV(st) read dO(st)
      if (S_AFTER_DV && nx < nsteps && !(ok = issue_st(nx))) break;
      if constexpr (C::FUSEDQ) {
        if (nx < nsteps) {
          if (st >= 1 &&
              !(ok = mbar_wait_warp(bar(C::B_DQFREE), (st - 1) & 1, wc, kSiteDqDone)))
            break;
          if (!(ok = issue_st(nx))) break;
        }
      }
      // dK += dS^T Q[:, part]   (A = dS^T bf16 in TMEM over the dP^T columns)
      if (!(ok = mbar_wait_warp(bar(C::B_DS + st % C::DB), (st / C::DB) & 1, wc, kSiteDsFull))) break;
      tc_fence_after();
      const uint32_t dpb = tmem + C::TM_DPT + (st % C::DB) * C::BMQ;
#pragma unroll
      for (int kb = 0; kb < C::BMQ / 16; ++kb)
        umma_ts_elect(false, tmem + C::TM_DK, dpb + half_packed_col<C::BMQ>(kb),
                      sdesc_sw128(qbuf(st) + hbox * C::BMQ * 128 + kb * 16 * 128, C::BMQ * 128, 1024),
                      ID_G, (st > 0 || kb > 0) ? 1u : 0u);
      tc_commit_elect(bar(C::B_QEMPTY + st % C::QST));     // S^T(st) and dK(st) read Q(st)
      if constexpr (C::FUSEDQ) {
        // dQ(st) = dS(st) K: A = dS from shared memory (MN-major), B = K (MN-major)
        constexpr uint32_t ID_Q = idesc_bf16_amn(128, C::D, true);
        const uint32_t dqt = tmem + C::TM_ST + (st % C::SB) * C::BMQ + C::TM_DQ_OFF;
#pragma unroll
        for (int kb = 0; kb < C::BN / 16; ++kb)
          umma_ss_elect(false, dqt, sdesc_sw128(sbase + C::SMEM_DS + kb * 16 * 128, C::DS_BOX, 1024),
                        sdesc_sw128(sbase + C::SMEM_K + kb * 16 * 128, C::BN * 128, 1024), ID_Q,
                        kb > 0 ? 1u : 0u);
        tc_commit_elect(bar(C::B_DQFULL));
      }
      // the next tile's remaining products go after this tile's readers
      if (nx < nsteps) {
        if (!EARLY_S && !C::FUSEDQ && !S_AFTER_DV && !(ok = issue_st(nx))) break;
        if (!EARLY_DP && !(ok = issue_dpt(nx))) break;
      }
    }
    tc_commit_elect(bar(C::B_ACC));
    tc_commit_elect(bar(C::B_DRAIN));
    if (!mbar_wait_drain(bar(C::B_DRAIN), 0, wc.timeout_ns) && lane == 0)
      atomicCAS(wc.status, 0u, kStatusTimeout | kSiteDrain);
  } else if (warp == C::REDUCE_WARP) {
    // ---------------- fused dQ: per step, the eight staged 32 x 32 blocks of dQ_i go to
    // the fp32 sums as TMA reduce-adds (issued here, off the compute warps' path); the
    // compute warps reuse the staging blocks once these have read them
    bool ok = true;
    for (int sp = 0; sp < nsteps && ok; ++sp) {
      if (!(ok = mbar_wait_warp(bar(C::B_DQSTG), sp & 1, wc, kSiteDqDone))) break;
      if (lane == 0) {
        const int y0 = q_tile(sp) * C::BMQ;
        for (int w = 0; w < 8; ++w) {
          const int y = y0 + (w & 3) * 32;              // rows past N are clipped
          if (y < p.N)
            tma_reduce_add_3d(&tdq, sbase + C::SMEM_DQ + w * 4096, (w >> 2) * 32, y, q_head(sp));
        }
        bulk_commit();
        bulk_wait_read_all();
      }
      mbar_arrive_warp(bar(C::B_DQSFR));
    }
    // the reduce-adds complete before the shared memory goes away and the kernel ends
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else {
    // ---------------- compute warps: thread owns key row `row`, query columns of `half`
    const int quad = warp & 3, half = warp >> 2;
    const int row = quad * 32 + lane;
    const int kv = kt * C::BN + row;
    const uint32_t lb = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float sl2 = p.scale * LOG2E;
    bool ok = true;
    // fused dQ: add dQ(sp) (this warp's lane quadrant of query rows, its half of the
    // columns) into the fp32 accumulator, then free its tensor-memory columns
    auto drain_dq = [&](int sp) -> bool {
      if (!mbar_wait(bar(C::B_DQFULL), sp & 1, wc, kSiteDqDone)) return false;
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(lb + C::TM_ST + (sp % C::SB) * C::BMQ + C::TM_DQ_OFF + half * 32, r);
      tmem_ld_wait(r);
      tc_fence_before();
      mbar_arrive_warp(bar(C::B_DQFREE));          // the columns are free once loaded
      // staging block: row `lane`, 16-byte chunk c at position c ^ (lane & 7), once the
      // reduce-add of step sp-1 has read it; the reduce warp adds it to the sums
      const uint32_t stg = sbase + C::SMEM_DQ + warp * 4096;
      if (sp > 0 && !mbar_wait(bar(C::B_DQSFR), (sp - 1) & 1, wc, kSiteDqDone)) return false;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(stg + lane * 128 + ((c ^ (lane & 7)) << 4), r[4 * c], r[4 * c + 1], r[4 * c + 2],
                     r[4 * c + 3]);
      fence_proxy_async_smem();
      mbar_arrive_warp(bar(C::B_DQSTG));
      return true;
    };
    for (int st = 0; st < nsteps && ok; ++st) {
      const int qi = q_tile(st);
      const int c_first = qi * C::BMQ + half * C::CH;      // first query of this half
      // lse_i and D_i come with their rings' tiles (and are in place once they are)
      if (!(ok = mbar_wait(bar(C::B_QFULL + st % C::QST), (st / C::QST) & 1, wc, kSiteQFull))) break;
      if (!(ok = mbar_wait(bar(C::B_OFULL + st % C::OST), (st / C::OST) & 1, wc, kSiteQFull))) break;
      const float* dd = dd_s + (st % C::DDR) * C::BMQ + half * C::CH;
      if (!(ok = mbar_wait(bar(C::B_SFULL + st % C::SB), (st / C::SB) & 1, wc, kSiteSFull))) break;
      tc_fence_after();
      const float* ls = lse_s + (st % C::QST) * C::BMQ + half * C::CH;
      const uint32_t stc = lb + C::TM_ST + (st % C::SB) * C::BMQ + half * C::CH;
      const uint32_t stp = lb + C::TM_ST + (st % C::SB) * C::BMQ + half * C::PACK_HI;
      // P^T row segment, zero where the query may not see this key
      float pr[C::CH];
      {
        uint32_t r[C::CH];
        if constexpr (C::CH == 64) {
          tmem_ld64(stc, r);
          tmem_ld_wait64(r);
        } else {
          tmem_ld32(stc, r);
          tmem_ld_wait(r);
        }
        exp2_row<C::CH, C::EMU>(r, sl2, ls, pr);
      }
      const bool full_vis = (kv < p.N) && (c_first + C::CH <= p.N) &&
                            (!p.causal || kt * C::BN + C::BN - 1 <= c_first);
      if (!__all_sync(0xffffffffu, full_vis)) {
#pragma unroll
        for (int i = 0; i < C::CH; ++i) {
          const int q = c_first + i;
          if (!((q < p.N) && (kv < p.N) && (!p.causal || kv <= q))) pr[i] = 0.f;
        }
      }
      {
        uint32_t w[C::CH / 2];
#pragma unroll
        for (int i = 0; i < C::CH / 2; ++i) w[i] = pack_bf16x2(pr[2 * i], pr[2 * i + 1]);
        if constexpr (C::CH == 64)
          tmem_st32(stp, w);
        else
          tmem_st16(stp, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(bar(C::B_P + st % C::SB));
      if constexpr (C::FUSEDQ) {
        // dQ(st-1) is done by now; its drain also frees the shared dS tile for this step
        if (st > 0 && !(ok = drain_dq(st - 1))) break;
      }
      // dS^T row segment = P^T (dP^T - D_q), bf16 over this half's dP^T columns
      if (!(ok = mbar_wait(bar(C::B_DPFULL + st % C::DB), (st / C::DB) & 1, wc, kSiteSFull))) break;
      tc_fence_after();
      const uint32_t dpc = lb + C::TM_DPT + (st % C::DB) * C::BMQ + half * C::CH;
      {
        uint32_t r[C::CH];
        if constexpr (C::CH == 64) {
          tmem_ld64(dpc, r);
          tmem_ld_wait64(r);
        } else {
          tmem_ld32(dpc, r);
          tmem_ld_wait(r);
        }
        uint32_t w[C::CH / 2];
#pragma unroll
        for (int i = 0; i < C::CH / 2; ++i) {
          float a, b;
          f2_unpack(f2_mul(f2_pack(pr[2 * i], pr[2 * i + 1]),
                           f2_add(f2_pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])),
                                  f2_pack(-dd[2 * i], -dd[2 * i + 1]))),
                    a, b);
          w[i] = pack_bf16x2(a, b);
        }
        if constexpr (C::CH == 64)
          tmem_st32(dpc, w);
        else
          tmem_st16(dpc, w);
        if constexpr (C::FUSEDQ) {
          // the same row of dS^T into shared memory: box `half`, row `row`, 16-byte
          // chunk c of 8 queries at chunk position c ^ (row & 7) (128-byte swizzle)
          const uint32_t ds_row = sbase + C::SMEM_DS + half * C::DS_BOX + row * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(ds_row + ((c ^ (row & 7)) << 4), w[4 * c], w[4 * c + 1], w[4 * c + 2],
                         w[4 * c + 3]);
          fence_proxy_async_smem();
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(bar(C::B_DS + st % C::DB));
    }
    if constexpr (C::FUSEDQ) {
      if (ok && nsteps > 0) ok = drain_dq(nsteps - 1);
    }
    // epilogue: dV and scale*dK -> bf16 global, this half's DH/2 columns of the row
    if (ok && mbar_wait(bar(C::B_ACC), 0, wc, kSiteDqDone)) {
      tc_fence_after();
      const bool row_ok = kv < p.N;
      const size_t base =
          (static_cast<size_t>(bh) * p.N + kv) * p.ld + split * C::DH + half * (C::DH / 2);
      const int cbase = split * C::DH + half * (C::DH / 2);   // first column written here
      __nv_bfloat16* dvp = reinterpret_cast<__nv_bfloat16*>(p.dv) + base;
      __nv_bfloat16* dkp = reinterpret_cast<__nv_bfloat16*>(p.dk) + base;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t col0 = (which == 0 ? C::TM_DV : C::TM_DK) + half * (C::DH / 2);
        const float mul = which == 0 ? 1.f : p.scale;
        __nv_bfloat16* dst = which == 0 ? dvp : dkp;
#pragma unroll 1
        for (int c = 0; c < C::DH / 2; c += 32) {
          uint32_t r[32];
          tmem_ld32(lb + col0 + c, r);
          tmem_ld_wait(r);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
          if (row_ok && cbase + c < p.ld) {
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
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

// --------------------------------------------------------------------------- 3. dQ
// One CTA per (head, 128-row query tile).  Q and dO stay in shared memory, dQ
// accumulates in tensor memory, and the key tiles stream through a ring.  Per key
// tile j (BN keys): S = Q K_j^T and dP = dO V_j^T on the tensor core; the compute
// warps form P from the saved logsumexp and dS = P (dP - D) (bf16 over the dP
// columns); then dQ += dS K_j.  S has SB buffers and dP DB buffers so tile j+1's
// products overlap the elementwise work on tile j; eight compute warps split the key
// columns in halves as in the dK/dV pass.  K_j and V_j have rings of their own (KST,
// VST deep): V_j is free as soon as dP has read it, K_j only after dQ.
template <int D_, int BN_, int KST_, int VST_, int SB_, int DB_, int EMU_ = 1>
struct DqCfg {
  static constexpr int D = D_;
  static constexpr int BN = BN_;        // streamed key rows
  static constexpr int BM = 128;        // query rows of the CTA = TMEM lanes
  static constexpr int KST = KST_, VST = VST_;
  static constexpr int SB = SB_, DB = DB_;
  static constexpr int EMU = EMU_;
  static constexpr int CH = BN / 2;     // key columns per compute warp
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int NBOX = ROW_BYTES / 128;
  static constexpr int QT_BYTES = BM * ROW_BYTES;
  static constexpr int KT_BYTES = BN * ROW_BYTES;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_DO = QT_BYTES;
  static constexpr int SMEM_K = 2 * QT_BYTES;
  static constexpr int SMEM_V = SMEM_K + KST * KT_BYTES;
  static constexpr int SMEM_BAR = SMEM_V + VST * KT_BYTES;
  static constexpr int B_QDO = 0, B_ACC = 1, B_DRAIN = 2,
                       B_SFULL = 3, B_DPFULL = 3 + SB, B_DS = 3 + SB + DB,
                       B_KFULL = 3 + SB + 2 * DB, B_KEMPTY = B_KFULL + KST,
                       B_VFULL = B_KEMPTY + KST, B_VEMPTY = B_VFULL + VST,
                       B_SFREE = B_VEMPTY + VST,   // one S buffer: the compute warps loaded S(j)
                       NBARS = B_SFREE + 1;
  static constexpr int SMEM_MISC = SMEM_BAR + NBARS * 8;
  static constexpr int SMEM_ALLOC = SMEM_MISC + 64 + 1024;
  static constexpr int TM_S = 0;                 // + b * BN
  static constexpr int TM_DP = SB * BN;          // + b * BN
  static constexpr int TM_DQ = (SB + DB) * BN;
  static constexpr int TM_COLS = 512;
  static constexpr int THREADS = 320;
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9;
  static_assert((SB + DB) * BN + D <= TM_COLS, "tensor memory budget");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(BN % 64 == 0 && CH % 32 == 0, "box and TMEM chunk sizes");
  static_assert(SB >= 1 && SB <= 2 && DB >= 1 && DB <= 2, "one or two buffers");
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
  int bh, lvl, part;
  bwd_block_item(blockIdx.x, p.BH, p.n_qt, 1, p.group_heads, bh, lvl, part);
  const int bkv = p.g == 1 ? bh : (bh / p.H) * (p.H / p.g) + (bh % p.H) / p.g;   // K/V head
  const int qt = p.n_qt - 1 - lvl;
  const int nsteps = p.causal ? min(p.n_kt, ((qt + 1) * C::BM - 1) / C::BN + 1) : p.n_kt;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBARS; ++i)
      mbar_init(bar(i), ((i >= C::B_DS && i < C::B_DS + C::DB) || i == C::B_SFREE)
                            ? 8u : 1u);                     // the 8 compute warps arrive
    *abort_flag = 0;
    fence_mbar_init();
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
    bool ok = true;
    if (elect_one()) {
      mbar_arrive_expect_tx(bar(C::B_QDO), 2 * C::QT_BYTES);
      for (int c = 0; c < C::NBOX; ++c) {
        tma_load_3d(sbase + C::SMEM_Q + c * C::BM * 128, &tq, bar(C::B_QDO), c * 64, qt * C::BM, bh);
        tma_load_3d(sbase + C::SMEM_DO + c * C::BM * 128, &tdo, bar(C::B_QDO), c * 64, qt * C::BM, bh);
      }
    }
    __syncwarp();
    // K_j then V_j, each into its own ring (an early S(j) needs K_j before the dP
    // product that frees V's slot is issued)
    int nk = 0, nv = 0;
    for (int j = 0; j < nsteps && ok; ++j) {
      const int sk = j % C::KST, sv = j % C::VST;
      if (j >= C::KST &&
          !(ok = mbar_wait_warp(bar(C::B_KEMPTY + sk), ((j / C::KST) - 1) & 1, wc, kSiteKVEmpty)))
        break;
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(C::B_KFULL + sk), C::KT_BYTES);
        for (int c = 0; c < C::NBOX; ++c)
          tma_load_3d(sbase + C::SMEM_K + sk * C::KT_BYTES + c * C::BN * 128, &tk,
                      bar(C::B_KFULL + sk), c * 64, j * C::BN, bkv);
      }
      __syncwarp();
      ++nk;
      if (j >= C::VST &&
          !(ok = mbar_wait_warp(bar(C::B_VEMPTY + sv), ((j / C::VST) - 1) & 1, wc, kSiteKVEmpty)))
        break;
      if (elect_one()) {
        mbar_arrive_expect_tx(bar(C::B_VFULL + sv), C::KT_BYTES);
        for (int c = 0; c < C::NBOX; ++c)
          tma_load_3d(sbase + C::SMEM_V + sv * C::KT_BYTES + c * C::BN * 128, &tv,
                      bar(C::B_VFULL + sv), c * 64, j * C::BN, bkv);
      }
      __syncwarp();
      ++nv;
    }
    if (ok) {
      for (int j = (nsteps > C::KST ? nsteps - C::KST : 0); ok && j < nsteps; ++j)
        ok = mbar_wait_warp(bar(C::B_KEMPTY + j % C::KST), (j / C::KST) & 1, wc, kSiteKVEmpty);
      for (int j = (nsteps > C::VST ? nsteps - C::VST : 0); ok && j < nsteps; ++j)
        ok = mbar_wait_warp(bar(C::B_VEMPTY + j % C::VST), (j / C::VST) & 1, wc, kSiteKVEmpty);
    } else {
      mbar_wait_drain(bar(C::B_QDO), 0, 100000000ull);
      for (int j = (nk > C::KST ? nk - C::KST : 0); j < nk; ++j)
        mbar_wait_drain(bar(C::B_KFULL + j % C::KST), (j / C::KST) & 1, 100000000ull);
      for (int j = (nv > C::VST ? nv - C::VST : 0); j < nv; ++j)
        mbar_wait_drain(bar(C::B_VFULL + j % C::VST), (j / C::VST) & 1, 100000000ull);
    }
  } else if (warp == C::MMA_WARP) {
    constexpr uint32_t ID_S = idesc_bf16(128, C::BN, false);
    constexpr uint32_t ID_Q = idesc_bf16(128, C::D, true);
    auto kbuf = [&](int j) { return sbase + C::SMEM_K + (j % C::KST) * C::KT_BYTES; };
    auto vbuf = [&](int j) { return sbase + C::SMEM_V + (j % C::VST) * C::KT_BYTES; };
    auto issue_s = [&](int j) -> bool {
      if (!mbar_wait_warp(bar(C::B_KFULL + j % C::KST), (j / C::KST) & 1, wc, kSiteKFull))
        return false;
      tc_fence_after();
#pragma unroll
      for (int kb = 0; kb < C::D / 16; ++kb) {
        const int box = kb / 4, off = (kb % 4) * 32;
        umma_ss_elect(false, tmem + C::TM_S + (j % C::SB) * C::BN,
                      sdesc_sw128(sbase + C::SMEM_Q + box * C::BM * 128 + off, 16, 1024),
                      sdesc_sw128(kbuf(j) + box * C::BN * 128 + off, 16, 1024), ID_S, kb > 0);
      }
      tc_commit_elect(bar(C::B_SFULL + j % C::SB));
      return true;
    };
    auto issue_dp = [&](int j) -> bool {
      if (!mbar_wait_warp(bar(C::B_VFULL + j % C::VST), (j / C::VST) & 1, wc, kSiteVFull))
        return false;
      tc_fence_after();
#pragma unroll
      for (int kb = 0; kb < C::D / 16; ++kb) {
        const int box = kb / 4, off = (kb % 4) * 32;
        umma_ss_elect(false, tmem + C::TM_DP + (j % C::DB) * C::BN,
                      sdesc_sw128(sbase + C::SMEM_DO + box * C::BM * 128 + off, 16, 1024),
                      sdesc_sw128(vbuf(j) + box * C::BN * 128 + off, 16, 1024), ID_S, kb > 0);
      }
      tc_commit_elect(bar(C::B_DPFULL + j % C::DB));
      tc_commit_elect(bar(C::B_VEMPTY + j % C::VST));         // dP(j) is V(j)'s only reader
      return true;
    };
    // S(j+1) may run ahead of dQ(j): its buffer's last reader, the compute warps'
    // load of S(j+1-SB), happened before they released dS(j+1-SB).  With one S buffer
    // S(j+1) waits only for that load (the compute warps signal it at once), so it and
    // the next dP run under the exponentials of tile j.  dP(j+1) has to follow dQ(j)
    // unless it has a second buffer.
    constexpr bool EARLY_S = C::SB == 2 && C::KST >= 2;
    constexpr bool S_ON_FREE = C::SB == 1 && C::KST >= 2;
    constexpr bool EARLY_DP = (EARLY_S || S_ON_FREE) && C::DB == 2 && C::VST >= 2;
    bool ok = mbar_wait_warp(bar(C::B_QDO), 0, wc, kSiteQFull);
    if (ok && nsteps > 0) ok = issue_s(0) && issue_dp(0);
    for (int j = 0; j < nsteps && ok; ++j) {
      const int nx = j + 1;
      if (EARLY_S && nx < nsteps) {
        // S(nx) overwrites the buffer S(nx - 2) was loaded from: that load preceded
        // dS(nx - 2), which this warp waited for one iteration ago
        if (!(ok = issue_s(nx))) break;
        if (EARLY_DP && !(ok = issue_dp(nx))) break;
      }
      if (S_ON_FREE && nx < nsteps) {
        // S(nx) overwrites S(j) once every compute warp has loaded it; dP(nx) goes to
        // the buffer dQ(j-1), issued one iteration ago, read dS(j-1) from
        if (!(ok = mbar_wait_warp(bar(C::B_SFREE), j & 1, wc, kSiteSFull))) break;
        tc_fence_after();
        if (!(ok = issue_s(nx))) break;
        if (EARLY_DP && !(ok = issue_dp(nx))) break;
      }
      if (!(ok = mbar_wait_warp(bar(C::B_DS + j % C::DB), (j / C::DB) & 1, wc, kSiteDsFull))) break;
      tc_fence_after();
      // dQ += dS K_j: A = dS (query rows x key cols) bf16 in TMEM, B = K_j MN-major
      const uint32_t dpb = tmem + C::TM_DP + (j % C::DB) * C::BN;
#pragma unroll
      for (int kb = 0; kb < C::BN / 16; ++kb)
        umma_ts_elect(false, tmem + C::TM_DQ, dpb + half_packed_col<C::BN>(kb),
                      sdesc_sw128(kbuf(j) + kb * 16 * 128, C::BN * 128, 1024), ID_Q,
                      (j > 0 || kb > 0) ? 1u : 0u);
      tc_commit_elect(bar(C::B_KEMPTY + j % C::KST));         // S(j) and dQ(j) read K(j)
      if (nx < nsteps) {
        if (!EARLY_S && !S_ON_FREE && !(ok = issue_s(nx))) break;
        if (!EARLY_DP && !(ok = issue_dp(nx))) break;
      }
    }
    tc_commit_elect(bar(C::B_ACC));
    tc_commit_elect(bar(C::B_DRAIN));
    if (!mbar_wait_drain(bar(C::B_DRAIN), 0, wc.timeout_ns) && lane == 0)
      atomicCAS(wc.status, 0u, kStatusTimeout | kSiteDrain);
  } else {
    const int quad = warp & 3, half = warp >> 2;
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
      const int k_first = j * C::BN + half * C::CH;          // first key of this half
      if (!(ok = mbar_wait(bar(C::B_SFULL + j % C::SB), (j / C::SB) & 1, wc, kSiteSFull))) break;
      tc_fence_after();
      float pr[C::CH];
      {
        const uint32_t sc = lb + C::TM_S + (j % C::SB) * C::BN + half * C::CH;
        uint32_t r[C::CH];
        if constexpr (C::CH == 64) {
          tmem_ld64(sc, r);
          tmem_ld_wait64(r);
        } else {
          tmem_ld32(sc, r);
          tmem_ld_wait(r);
        }
        if constexpr (C::SB == 1) {            // the MMA warp may now overwrite S(j)
          tc_fence_before();
          mbar_arrive_warp(bar(C::B_SFREE));
        }
        exp2_row<C::CH, C::EMU>(r, sl2, lse2, pr);
      }
      const bool full_vis = row_ok && (k_first + C::CH <= p.N) &&
                            (!p.causal || k_first + C::CH - 1 <= qt * C::BM);
      if (!__all_sync(0xffffffffu, full_vis)) {
#pragma unroll
        for (int i = 0; i < C::CH; ++i) {
          const int kv = k_first + i;
          if (!(row_ok && (kv < p.N) && (!p.causal || kv <= q))) pr[i] = 0.f;
        }
      }
      if (!(ok = mbar_wait(bar(C::B_DPFULL + j % C::DB), (j / C::DB) & 1, wc, kSiteSFull))) break;
      tc_fence_after();
      {
        const uint32_t dc = lb + C::TM_DP + (j % C::DB) * C::BN + half * C::CH;
        uint32_t r[C::CH];
        if constexpr (C::CH == 64) {
          tmem_ld64(dc, r);
          tmem_ld_wait64(r);
        } else {
          tmem_ld32(dc, r);
          tmem_ld_wait(r);
        }
        const uint64_t nd2 = f2_pack(-dq_i, -dq_i);
        uint32_t w[C::CH / 2];
#pragma unroll
        for (int i = 0; i < C::CH / 2; ++i) {
          float a, b;
          f2_unpack(f2_mul(f2_pack(pr[2 * i], pr[2 * i + 1]),
                           f2_add(f2_pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), nd2)),
                    a, b);
          w[i] = pack_bf16x2(a, b);
        }
        if constexpr (C::CH == 64)
          tmem_st32(dc, w);
        else
          tmem_st16(dc, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_warp(bar(C::B_DS + j % C::DB));
    }
    if (ok && mbar_wait(bar(C::B_ACC), 0, wc, kSiteDqDone)) {
      tc_fence_after();
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.dq) +
                           (static_cast<size_t>(bh) * p.N + q) * p.ld + half * (C::D / 2);
#pragma unroll 1
      for (int c = 0; c < C::D / 2; c += 32) {
        uint32_t r[32];
        tmem_ld32(lb + C::TM_DQ + half * (C::D / 2) + c, r);
        tmem_ld_wait(r);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * p.scale, __uint_as_float(r[2 * i + 1]) * p.scale);
        if (row_ok && half * (C::D / 2) + c < p.ld) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
  // This pass may start before the dK/dV pass ends (it reads nothing that pass writes);
  // it ends only after it, so work queued behind the backward sees dK and dV complete.
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace fa
