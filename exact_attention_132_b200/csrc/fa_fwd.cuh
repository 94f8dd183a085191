// fa_fwd.cuh — fused attention forward for sm_100a (bf16 and FP8 e4m3 inputs).
//
// One persistent CTA per SM walks a static list of work items (b, h, 128-row
// query tile).  For each item it streams the key/value tiles of that head:
//
//   S_j = Q K_j^T                      tcgen05.mma, fp32 accumulator in TMEM
//   m'  = max(m, rowmax(S_j) * c)      c = scale * log2(e) (times the FP8 tile scales)
//   P_j = 2^(S_j * c - m')             on the special-function unit, P written to TMEM
//   l   = l * 2^(m - m') + rowsum(P_j)
//   O   = O * 2^(m - m')               only for warps where some row max changed
//   O  += P_j V_j                      tcgen05.mma with A = P from TMEM
//
// and finally O / l -> bf16 and lse = (m + log2 l) * ln 2.  This is the tiling +
// online softmax + fusion of "FlashAttention — フラッシュアテンション" (wiki,
// sections タイリングとブロック処理, オンラインSoftmax計算, CUDAカーネルの融合) and of
// the issoh.co.jp page (sections QKVをブロック分割してSRAMへ載せるタイリングの手順 and
// 最大値と正規化項を持ち回るオンラインsoftmaxの再スケール).  Rescaling only when the
// max moves follows the same page's section on FA4 (FA4のB200で1613TFLOPs…:
// "rescale only when needed").  Causal tiles wholly above the diagonal are
// never visited (mypcrig.com post, section "FA2 の改善").
//
// Roles (warp specialisation, mypcrig.com post, section "FA3 の飛躍"):
//   warp 0       TMA producer: Q tile per item, K and V tiles into separate rings
//   warp 1       MMA issuer (one thread) + tensor-memory owner
//   warps 2..5   softmax/correction/epilogue: thread t owns query row 32*(w%4)+lane,
//                which is TMEM lane 32*(w%4)+lane (the lane quadrant a warp may use)
//
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   [0, BN)      S buffer 0 (fp32); P of that step overwrites its first columns
//   [BN, 2BN)    S buffer 1
//   [2BN, 2BN+D) O accumulator (fp32)
#pragma once

#include <type_traits>

#include "sm100_ptx.cuh"

namespace fa {

struct FwdParams {
  int BH;             // B * H (query heads)
  int H;              // query heads per batch entry
  int g;              // query heads per key/value head (1 = one K/V head per query head)
  int ld;             // head dim as stored (row length of q, k, v, o); the kernel's D may
                      // be larger: columns past ld load as zeros and are not stored
  int N;              // sequence length (queries = keys)
  int n_qt;           // ceil(N / 128)
  int n_kt;           // ceil(N / BN)
  int n_st;           // ceil(N / 128): FP8 scale tiles per head
  int causal;
  int group_heads;    // causal ordering: heads that share one heaviest-first sweep
  int total_items;    // BH * n_qt
  float scale;        // multiplier of Q K^T
  void* o;            // bf16 [BH, N, D]
  float* lse;         // fp32 [BH, N] or null
  const float* q_scale;   // FP8 only: [BH, n_st]
  const float* k_scale;
  const float* v_scale;
  unsigned* status;
  unsigned long long timeout_ns;
  int* sched;         // {next item, CTAs finished}: zero at launch, zero again at exit
};

// Shared-memory ring of work items (ItemRing below): slots and bytes
constexpr int kItemSlots = 4;
constexpr int kItemBytes = 2 * kItemSlots * 8 + kItemSlots * 4;   // barriers, then slots

// Key/value head of query head `bh` (flattened b * H + h): K/V hold H / g heads per
// batch entry and query head h reads K/V head h / g.
__device__ __forceinline__ int fwd_kv_head(const FwdParams& p, int bh) {
  if (p.g == 1) return bh;
  const int b = bh / p.H;
  return b * (p.H / p.g) + (bh - b * p.H) / p.g;
}

template <int D_, int BN_, int KST_, int VST_, bool FP8_, int EMU_ = 1, int TAU_ = 0>
struct FwdCfg {
  static constexpr int D = D_;
  static constexpr int BN = BN_;
  // Separate K and V rings: a K stage is released as soon as its S = Q K^T product
  // completes, a V stage when its P V product completes.
  static constexpr int KST = KST_;
  static constexpr int VST = VST_;
  static constexpr bool FP8 = FP8_;
  // Of every 4 column pairs of a score row, EMU take their exponentials on the FMA
  // pipe (ex2_poly_pair), the rest on the special-function unit.
  static constexpr int EMU = EMU_;
  // Reference-max slack in log2 units (bf16 only): the running max used for the
  // exponentials moves (and O is rescaled) only when a row max exceeds it by more than
  // TAU.  With TAU > 0 the largest probability of a row is no longer exactly 1.0, so
  // the row sum that normalises O takes on, per key tile, the bf16 rounding error of
  // the tile's largest probability, as the P V product does (the logsumexp keeps the
  // plain unrounded sum).
  static constexpr float TAU = FP8_ ? 0.f : static_cast<float>(TAU_);
  static constexpr int BM = 128;
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int ROW_BYTES = D * ELEM;        // bytes of one tile row
  static constexpr int NBOX = ROW_BYTES / 128;      // 128-byte swizzle boxes per row
  static constexpr int BOX_ELEMS = 128 / ELEM;
  static constexpr int Q_BYTES = BM * ROW_BYTES;
  static constexpr int KV_BYTES = BN * ROW_BYTES;
  static constexpr int MMA_K = FP8 ? 32 : 16;       // K of one tcgen05.mma
  static constexpr int KSTEP_BYTES = MMA_K * ELEM;  // always 32
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = Q_BYTES;
  static constexpr int SMEM_V = SMEM_K + KST * KV_BYTES;
  static constexpr int SMEM_BAR = SMEM_V + VST * KV_BYTES;
  // barriers
  static constexpr int B_QFULL = 0, B_QEMPTY = 1, B_SFULL = 2, B_PFULL = 4, B_ODONE = 6,
                       B_DRAIN = 7, B_KFULL = 8, B_KEMPTY = 8 + KST, B_VFULL = 8 + 2 * KST,
                       B_VEMPTY = 8 + 2 * KST + VST, NBARS = 8 + 2 * KST + 2 * VST;
  static constexpr int SMEM_MISC = SMEM_BAR + NBARS * 8;   // tmem slot, abort flag, reductions
  static constexpr int SMEM_ITEM = SMEM_MISC + 64;         // work-item ring
  static constexpr int SMEM_TOTAL = SMEM_ITEM + kItemBytes;
  static constexpr uint32_t ITEM_READERS = 1 + 4;          // the MMA thread, 4 softmax warps
  static constexpr int SMEM_ALLOC = SMEM_TOTAL + 1024;     // slack to align the base to 1024
  static constexpr int TM_S = 0;
  static constexpr int TM_O = 2 * BN;
  static constexpr int TM_COLS = 512;
  static constexpr int P_COLS = BN * (FP8 ? 1 : 2) / 4;    // 32-bit columns holding P
  static constexpr int THREADS = 192;
  static_assert(2 * BN + D <= TM_COLS, "tensor memory budget");
  static_assert(ROW_BYTES % 128 == 0, "rows must be whole 128-byte swizzle rows");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(BN % 32 == 0 && D % 32 == 0, "32-column TMEM chunks");
};

// Work item k of this CTA: rounds of gridDim.x items, alternate rounds walked in
// reverse CTA order so the heaviest-first list evens out across CTAs.
__device__ __forceinline__ int fwd_item_index(int k) {
  const int pos = (k & 1) ? (gridDim.x - 1 - blockIdx.x) : blockIdx.x;
  return k * gridDim.x + pos;
}

// ---------------------------------------------------------------- dynamic work distribution
// A CTA's first item is blockIdx.x; each further one is drawn by the producer thread
// from a global counter, so a CTA that finishes early takes the next item and the
// heaviest-first causal order balances itself (a static round-robin of the same order
// leaves the CTAs that drew the longest rows working alone at the end).  The producer
// publishes every item in a small shared-memory ring that the other roles read; a value
// >= total_items ends every role's loop.  The last CTA to leave sets the counter back to
// zero for the next launch on the same stream.
struct ItemRing {
  uint32_t bars;        // kItemSlots "full" barriers, then kItemSlots "empty" barriers
  volatile int* slot;   // kItemSlots item values
  // one-time setup by a single thread: `readers` arrivals release a slot
  __device__ __forceinline__ void init(uint32_t readers) const {
    for (int s = 0; s < kItemSlots; ++s) {
      mbar_init(bars + 8u * s, 1u);
      mbar_init(bars + 8u * (kItemSlots + s), readers);
    }
  }
  // producer thread: draw item k and publish it; false when a wait gave up
  __device__ __forceinline__ bool put(const FwdParams& p, int k, int& w, const WaitCtl& wc) const {
    w = k == 0 ? static_cast<int>(blockIdx.x) : static_cast<int>(gridDim.x) + atomicAdd(p.sched, 1);
    const int s = k % kItemSlots;
    if (k >= kItemSlots &&
        !mbar_wait(bars + 8u * (kItemSlots + s), ((k / kItemSlots) - 1) & 1, wc, kSiteItem))
      return false;
    slot[s] = w;
    mbar_arrive(bars + 8u * s);   // release: the slot value is visible to every waiter
    return true;
  }
  // one reader thread: read item k and release its slot
  __device__ __forceinline__ bool get(int k, int& w, const WaitCtl& wc) const {
    const int s = k % kItemSlots;
    if (!mbar_wait(bars + 8u * s, (k / kItemSlots) & 1, wc, kSiteItem)) return false;
    w = slot[s];
    mbar_arrive(bars + 8u * (kItemSlots + s));
    return true;
  }
  // every lane of a warp reads item k; the warp releases the slot once
  __device__ __forceinline__ bool get_warp(int k, int& w, const WaitCtl& wc) const {
    const int s = k % kItemSlots;
    if (!mbar_wait_warp(bars + 8u * s, (k / kItemSlots) & 1, wc, kSiteItem)) return false;
    w = slot[s];
    mbar_arrive_warp(bars + 8u * (kItemSlots + s));
    return true;
  }
};

// Thread 0 of each CTA after every role has left its item loop: the last CTA out
// resets the counter.  Every draw of a CTA completes (its value is used) before that
// CTA's arrival here, so the reset follows the final draw of the launch.
__device__ __forceinline__ void sched_release(const FwdParams& p) {
  __threadfence();
  if (atomicAdd(p.sched + 1, 1) == static_cast<int>(gridDim.x) - 1) {
    p.sched[0] = 0;
    p.sched[1] = 0;
    __threadfence();
  }
}

// Map a linear item to (bh, q tile).  Non-causal: head-major, so CTAs running at
// the same time share a head's K/V in L2.  Causal: heads are swept in groups;
// inside a group the longest rows (highest q tile) come first.
__device__ __forceinline__ void fwd_decode_item(const FwdParams& p, int w, int& bh, int& qt) {
  if (!p.causal) {
    bh = w / p.n_qt;
    qt = w - bh * p.n_qt;
    return;
  }
  const int per_group = p.group_heads * p.n_qt;
  const int g = w / per_group;
  const int r = w - g * per_group;
  const int gsize = min(p.group_heads, p.BH - g * p.group_heads);
  const int lvl = r / gsize;
  qt = p.n_qt - 1 - lvl;
  bh = g * p.group_heads + (r - lvl * gsize);
}

template <class C>
__device__ __forceinline__ int fwd_num_kv_tiles(const FwdParams& p, int qt) {
  if (!p.causal) return p.n_kt;
  const int last = min(p.n_kt - 1, ((qt + 1) * C::BM - 1) / C::BN);
  return last + 1;
}

// ---------------------------------------------------------------- producer (one thread)
template <class C>
__device__ void fwd_producer(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                             const FwdParams& p, uint32_t sbase, uint32_t bars, const ItemRing& ring,
                             const WaitCtl& wc) {
  auto bar = [&](int i) { return bars + 8u * i; };
  // Loads follow the order the MMA warp consumes them: per item Q, K_0, then
  // (K_j, V_{j-1}) for j >= 1, then V_{n-1}; K therefore runs one step ahead of V.
  uint32_t gk = 0, gv = 0, t = 0;   // K loads, V loads, items issued so far
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
    int w;
    if (!(ok = ring.put(p, k, w, wc))) break;
    if (w >= p.total_items) break;
    int bh, qt;
    fwd_decode_item(p, w, bh, qt);
    const int n = fwd_num_kv_tiles<C>(p, qt);
    if (t > 0 && !(ok = mbar_wait(bar(C::B_QEMPTY), (t - 1) & 1, wc, kSiteQEmpty))) break;
    mbar_arrive_expect_tx(bar(C::B_QFULL), C::Q_BYTES);
#pragma unroll
    for (int c = 0; c < C::NBOX; ++c)
      tma_load_3d(sbase + C::SMEM_Q + c * C::BM * 128, tq, bar(C::B_QFULL), c * C::BOX_ELEMS,
                  qt * C::BM, bh);
    ++t;
    const int kvh = fwd_kv_head(p, bh);
    if (!(ok = load_k(0, kvh))) break;
    for (int j = 1; j < n && ok; ++j) ok = load_k(j, kvh) && load_v(j - 1, kvh);
    if (ok) ok = load_v(n - 1, kvh);
  }
  if (!ok) {
    // Aborted: let the tile copies already issued land before the CTA exits.
    if (t > 0) mbar_wait_drain(bar(C::B_QFULL), (t - 1) & 1, 100000000ull);
    for (uint32_t i = (gk > C::KST ? gk - C::KST : 0); i < gk; ++i)
      mbar_wait_drain(bar(C::B_KFULL + i % C::KST), (i / C::KST) & 1, 100000000ull);
    for (uint32_t i = (gv > C::VST ? gv - C::VST : 0); i < gv; ++i)
      mbar_wait_drain(bar(C::B_VFULL + i % C::VST), (i / C::VST) & 1, 100000000ull);
    return;
  }
  // Drain: wait until the MMA side has released every buffer, so no tensor-core
  // commit is still due to arrive on this CTA's barriers when it exits.
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
__device__ void fwd_mma(const FwdParams& p, uint32_t sbase, uint32_t bars, uint32_t tmem,
                        const ItemRing& ring, const WaitCtl& wc) {
  auto bar = [&](int i) { return bars + 8u * i; };
  constexpr uint32_t IDESC_S = C::FP8 ? idesc_e4m3(128, C::BN, false) : idesc_bf16(128, C::BN, false);
  constexpr uint32_t IDESC_O = C::FP8 ? idesc_e4m3(128, C::D, true) : idesc_bf16(128, C::D, true);
  constexpr int KSTEPS_S = C::D / C::MMA_K;     // over the head dimension
  constexpr int KSTEPS_O = C::BN / C::MMA_K;    // over the key tile
  uint32_t g = 0, t = 0;
  bool ok = true;

  // O += P V for global step gk; `first` = first step of its item (overwrite O).
  auto issue_pv = [&](uint32_t gk, bool first) -> bool {
    const int b = gk & 1;
    if (!mbar_wait(bar(C::B_PFULL + b), (gk >> 1) & 1, wc, kSitePFull)) return false;
    const int s = gk % C::VST;
    if (!mbar_wait(bar(C::B_VFULL + s), (gk / C::VST) & 1, wc, kSiteVFull)) return false;
    tc_fence_after();
    const uint32_t vbase = sbase + C::SMEM_V + s * C::KV_BYTES;
#pragma unroll
    for (int kb = 0; kb < KSTEPS_O; ++kb) {
      // V tile is K(=key)-rows x N(=d) with d contiguous: MN-major operand.
      // LBO = distance between 128-byte column boxes, SBO = 8 rows * 128 B.
      const uint64_t bdesc = sdesc_sw128(vbase + kb * C::MMA_K * 128, C::BN * 128, 1024);
      const uint32_t a_tmem = tmem + C::TM_S + b * C::BN + kb * (C::MMA_K * C::ELEM / 4);
      umma_ts<C::FP8>(tmem + C::TM_O, a_tmem, bdesc, IDESC_O, (first && kb == 0) ? 0u : 1u);
    }
    tc_commit(bar(C::B_VEMPTY + s));
    tc_commit(bar(C::B_ODONE));
    return true;
  };

  for (int k = 0; ok; ++k) {
    int w;
    if (!(ok = ring.get(k, w, wc))) break;
    if (w >= p.total_items) break;
    int bh, qt;
    fwd_decode_item(p, w, bh, qt);
    const int n = fwd_num_kv_tiles<C>(p, qt);
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
      for (int kb = 0; kb < KSTEPS_S; ++kb) {
        // K-major operands: 128-byte swizzled rows, 8-row groups 1024 B apart;
        // a K step inside a 128-byte row is a 32-byte start-address offset.
        const int box = (kb * C::KSTEP_BYTES) / 128;
        const int off = (kb * C::KSTEP_BYTES) % 128;
        const uint64_t adesc = sdesc_sw128(sbase + C::SMEM_Q + box * C::BM * 128 + off, 16, 1024);
        const uint64_t bdesc = sdesc_sw128(kbase + box * C::BN * 128 + off, 16, 1024);
        umma_ss<C::FP8>(tmem + C::TM_S + b * C::BN, adesc, bdesc, IDESC_S, kb > 0 ? 1u : 0u);
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
  // Make sure nothing is in flight before the CTA frees tensor memory.
  tc_commit(bar(C::B_DRAIN));
  if (!mbar_wait_drain(bar(C::B_DRAIN), 0, wc.timeout_ns))
    atomicCAS(wc.status, 0u, kStatusTimeout | kSiteDrain);
}

// ---------------------------------------------------------------- exp2 variants
// ex2_poly_pair (software 2^x on the FMA pipe) lives in sm100_ptx.cuh.

// 2^x for a pair of fp32 values on the special-function unit in half precision:
// one ex2.approx.f16x2 for both.  The argument is rounded to f16 (relative 2^-11,
// so an absolute error below 0.004 for |x| <= 8); results below the f16 range
// become 0.  Returned as fp32.
__device__ __forceinline__ uint64_t ex2_f16_pair(uint64_t x2) {
  float xa, xb;
  f2_unpack(x2, xa, xb);
  uint32_t h, e;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(xb), "f"(xa));
  asm("ex2.approx.f16x2 %0, %1;" : "=r"(e) : "r"(h));
  float ra, rb;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "cvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
      : "=f"(ra), "=f"(rb)
      : "r"(e));
  return f2_pack(ra, rb);
}

// ---------------------------------------------------------------- softmax warps
template <class C>
__device__ void fwd_softmax(const FwdParams& p, uint32_t bars, uint32_t tmem, const ItemRing& ring,
                            const WaitCtl& wc) {
  auto bar = [&](int i) { return bars + 8u * i; };
  const int warp = threadIdx.x / 32;
  const int quad = warp & 3;
  const int row = quad * 32 + (threadIdx.x & 31);         // query row inside the tile
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const float LOG2E = 1.4426950408889634f;
  const float LN2 = 0.6931471805599453f;
  const float sl2 = p.scale * LOG2E;
  __nv_bfloat16* o_out = reinterpret_cast<__nv_bfloat16*>(p.o);
  uint32_t g = 0;
  bool ok = true;

  for (int k = 0; ok; ++k) {
    int w;
    if (!(ok = ring.get_warp(k, w, wc))) break;
    if (w >= p.total_items) break;
    int bh, qt;
    fwd_decode_item(p, w, bh, qt);
    const int n = fwd_num_kv_tiles<C>(p, qt);
    const int q_idx = qt * C::BM + row;
    float m = -INFINITY, l = 0.f;
    float lc = 0.f;                               // compensated row sum (TAU > 0)
    float qsc = 1.f, vmax = 1.f;
    if constexpr (C::FP8) {
      static_assert(!C::FP8 || C::BN == 128, "FP8 key tile = one 128-row scale tile");
      qsc = p.q_scale[bh * p.n_st + qt];
      // vmax = largest V tile scale among the visited key tiles; every thread reads
      // the same few values (L1 broadcast), so no cross-warp barrier is needed.
      vmax = 0.f;
      for (int j = 0; j < n; ++j) vmax = fmaxf(vmax, p.v_scale[fwd_kv_head(p, bh) * p.n_st + j]);
    }

    for (int j = 0; j < n; ++j) {
      const uint32_t gj = g + j;
      const int b = gj & 1;
      if (!(ok = mbar_wait(bar(C::B_SFULL + b), (gj >> 1) & 1, wc, kSiteSFull))) break;
      tc_fence_after();
      // the whole score row of this thread in one TMEM load
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
      const int kv0 = j * C::BN;
      const bool need_mask = (p.causal && kv0 + C::BN - 1 > qt * C::BM) || (kv0 + C::BN > p.N);
      if (need_mask) {
        const int lim = p.causal ? min(q_idx, p.N - 1) : p.N - 1;   // last visible key
#pragma unroll
        for (int c = 0; c < C::BN; ++c)
          if (kv0 + c > lim) s[c] = -INFINITY;
      }
      float c_j = sl2;
      float fold = 1.f;
      if constexpr (C::FP8) {
        c_j = sl2 * qsc * p.k_scale[fwd_kv_head(p, bh) * p.n_st + j];
        fold = 256.f * p.v_scale[fwd_kv_head(p, bh) * p.n_st + j] / vmax;
      }
      // row max: four independent three-input chains
      float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < C::BN; c += 8) {
        a0 = max3f(a0, s[c], s[c + 1]);
        a1 = max3f(a1, s[c + 2], s[c + 3]);
        a2 = max3f(a2, s[c + 4], s[c + 5]);
        a3 = max3f(a3, s[c + 6], s[c + 7]);
      }
      const float m_cand = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) * c_j;
      // Reference max: moved only when the row max rises by more than TAU (log2
      // units); P then stays <= 2^TAU and the final O / l is unchanged.
      const bool raise = m_cand > m + C::TAU;
      const float m_new = raise ? m_cand : m;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = raise ? ex2(m - m_use) : 1.f;   // 0 on the first tile (m = -inf)
      float l_comp = 0.f;
      if constexpr (C::TAU > 0.f) {
        // the tile's largest probability and its bf16 rounding error
        const float pt = ex2(m_cand - m_use);
        l_comp = __bfloat162float(__float2bfloat16_rn(pt)) - pt;
      }
      // P = 2^(S c - m): pairs through the f32x2 FMA; most exponentials on the
      // special-function unit, EMU of every 4 pairs on the FMA pipe.
      const uint64_t c2 = f2_pack(c_j, c_j);
      const uint64_t nm2 = f2_pack(-m_use, -m_use);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      // masked tiles (diagonal / ragged) use the special-function unit throughout, so a
      // masked score gives exactly 0
      auto exps = [&](auto emu_tag) {
        constexpr int kEmu = decltype(emu_tag)::value;
#pragma unroll
        for (int c = 0; c < C::BN; c += 2) {
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
      if constexpr (C::TAU > 0.f) lc = lc * alpha + (sa + sb) + l_comp;
      // P -> tensor memory over the consumed S columns
      if constexpr (C::FP8) {
#pragma unroll
        for (int c = 0; c < C::BN; c += 128) {
          uint32_t r[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            r[i] = pack_e4m3x4(s[c + 4 * i] * fold, s[c + 4 * i + 1] * fold,
                               s[c + 4 * i + 2] * fold, s[c + 4 * i + 3] * fold);
          tmem_st32(lane_base + C::TM_S + b * C::BN + c / 4, r);
        }
      } else {
#pragma unroll
        for (int c = 0; c < C::BN; c += 64) {
          uint32_t r[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = pack_bf16x2(s[c + 2 * i], s[c + 2 * i + 1]);
          tmem_st32(lane_base + C::TM_S + b * C::BN + c / 2, r);
        }
      }
      // The previous P V product must be complete before O is touched; waiting on
      // every step also keeps this warp's view of the O barrier phase exact.
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
    // epilogue: O / l -> bf16 -> global; row logsumexp
    const uint32_t glast = g + n - 1;
    if (!(ok = mbar_wait(bar(C::B_ODONE), glast & 1, wc, kSiteODone))) break;
    tc_fence_after();
    const float inv_l = (C::FP8 ? vmax * (1.f / 256.f) : 1.f) / (C::TAU > 0.f ? lc : l);
    const bool row_ok = q_idx < p.N;
    __nv_bfloat16* orow = o_out + (static_cast<size_t>(bh) * p.N + q_idx) * p.ld;
#pragma unroll 1
    for (int c = 0; c < C::D; c += 32) {
      uint32_t r[32];
      tmem_ld32(lane_base + C::TM_O + c, r);
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
    g += n;
  }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
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
      uint32_t cnt = 1;
      if (i == C::B_PFULL || i == C::B_PFULL + 1) cnt = 4;   // one arrival per softmax warp
      mbar_init(bars + 8u * i, cnt);
    }
    ring.init(C::ITEM_READERS);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
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
    if ((threadIdx.x & 31) == 0) fwd_producer<C>(&tq, &tk, &tv, p, sbase, bars, ring, wc);
  } else if (warp == 1) {
    if ((threadIdx.x & 31) == 0) fwd_mma<C>(p, sbase, bars, tmem, ring, wc);
  } else {
    fwd_softmax<C>(p, bars, tmem, ring, wc);
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) sched_release(p);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

}  // namespace fa
