// fa_api.cu — the C ABI of libfa.so (declared in include/fa.h): argument
// checks, TMA tensor-map construction, kernel selection by head dimension and
// launches.  The library allocates no device memory on any call path.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <type_traits>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_fwd.cuh"
#include "fa_fwd_pp.cuh"
#include "fa_decode.cuh"
#include "fa_dequant.cuh"
#include "sm100_ptx.cuh"

namespace fa {

// Device status word written by kernels whose bounded waits expired.
__device__ unsigned g_fa_status = 0;
// Work counters of the forward kernels' dynamic scheduler, one pair per stream that
// launched a forward on this device.  A launch leaves its pair at zero when it ends, so
// launches in one stream (which run one after the other) can share it.
constexpr int kSchedSlots = 256;
__device__ int g_fa_sched[kSchedSlots][2];

constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;   // 2 s per wait
constexpr int kMaxDevices = 64;

thread_local std::string t_last_error;

fa_status fail(fa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return st;
}

fa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// ------------------------------------------------------------------ per-device cache
struct DeviceInfo {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  int sms = 0;
  unsigned* status = nullptr;
  int* sched = nullptr;                 // g_fa_sched of this device
  std::mutex sched_mu;
  // host-buffer forward (fa_fwd_host): two copy streams and an event pool, made on first
  // use; the mutex also keeps concurrent calls from reusing each other's events
  std::mutex host_mu;
  bool host_ready = false;
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
  cudaEvent_t host_ev[128] = {};   // >= 1 + 3 * kHostChunks
  cudaStream_t sched_stream[kSchedSlots] = {};
  int sched_used = 0;
};
DeviceInfo g_dev[kMaxDevices];

fa_status device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FA_ERR_CUDA, "device index %d out of range", dev);
  DeviceInfo& d = g_dev[dev];
  std::call_once(d.once, [&] {
    d.err = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (d.err == cudaSuccess) {
      int major = 0, minor = 0;
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
      if (major != 10 || minor != 0) d.err = cudaErrorNoKernelImageForDevice;
    }
    if (d.err == cudaSuccess)
      d.err = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.status), g_fa_status);
    if (d.err == cudaSuccess)
      d.err = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.sched), g_fa_sched);
  });
  if (d.err != cudaSuccess) return cuda_fail(d.err, "device setup (needs an sm_100 GPU)");
  *out = &d;
  return FA_OK;
}

// The scheduler counter pair of `stream`.  Streams get slots in order of first use;
// beyond kSchedSlots distinct streams the slots are reused round-robin, so at most
// kSchedSlots streams may run forwards on one device at the same time.  Slots are
// keyed by the stream handle: a stream destroyed while its forwards are still queued
// and a new stream that receives the same handle would share one counter pair, so a
// stream's forwards must finish before the stream is destroyed (stated in fa.h).
int* sched_counter(DeviceInfo* d, cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(d->sched_mu);
  const int n = d->sched_used < kSchedSlots ? d->sched_used : kSchedSlots;
  for (int i = 0; i < n; ++i)
    if (d->sched_stream[i] == stream) return d->sched + 2 * i;
  const int i = d->sched_used % kSchedSlots;
  d->sched_stream[i] = stream;
  ++d->sched_used;
  return d->sched + 2 * i;
}

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// [BH, N, d] row-major tensor seen as 3-D (d, N, BH); box = (inner, rows, 1) with
// 128-byte swizzle.  Rows past N read as zero.
fa_status make_map(CUtensorMap* m, const void* ptr, bool fp8, int d, int N, int BH, int rows) {
  auto fn = encode_fn();
  if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  const int eb = fp8 ? 1 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * eb, static_cast<cuuint64_t>(N) * d * eb};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / eb), static_cast<cuuint32_t>(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return FA_OK;
}

// fp32 [BH, N, d] tensor (the fused backward's dQ sums) in 32 x 32 boxes, 128-byte
// swizzle: the target of the compute warps' reduce-adds.
fa_status make_map_f32(CUtensorMap* m, void* ptr, int d, int N, int BH) {
  auto fn = encode_fn();
  if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4, static_cast<cuuint64_t>(N) * d * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return FA_OK;
}

// Set the dynamic shared-memory limit of a kernel once per device.  `Tag` makes the
// cache per kernel: every kernel here has the same signature, so K alone does not.
template <class Tag, class K>
fa_status prepare_kernel(K kernel, int smem_bytes) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return FA_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  done.fetch_or(bit, std::memory_order_acq_rel);
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_common(int B, int H, int N, float scale, bool* empty) {
  if (B < 0 || H < 0 || N < 0) return fail(FA_ERR_INVALID_ARG, "negative size B=%d H=%d N=%d", B, H, N);
  if (!std::isfinite(scale) || !(scale > 0.f))
    return fail(FA_ERR_INVALID_ARG, "scale must be finite and > 0 (got %g)", static_cast<double>(scale));
  const long long bh = static_cast<long long>(B) * H;
  if (bh > (1ll << 30)) return fail(FA_ERR_INVALID_ARG, "B*H too large");
  *empty = (bh == 0 || N == 0);
  return FA_OK;
}

fa_status check_ptrs(const void* const* ptrs, const char* const* names, int n) {
  for (int i = 0; i < n; ++i) {
    if (ptrs[i] == nullptr) return fail(FA_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned16(ptrs[i])) return fail(FA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  return FA_OK;
}

int causal_group_heads(int BH, long long kv_bytes_per_head) {
  // heads whose K/V together fill about 32 MB of L2
  long long g = (32ll << 20) / (kv_bytes_per_head > 0 ? kv_bytes_per_head : 1);
  if (g < 1) g = 1;
  if (g > BH) g = BH;
  return static_cast<int>(g);
}

template <class C>
fa_status launch_fwd(const void* q, const void* k, const void* v, FwdParams p, cudaStream_t stream) {
  DeviceInfo* di = nullptr;
  if (fa_status s = device_info(&di)) return s;
  CUtensorMap mq, mk, mv;
  if (fa_status s = make_map(&mq, q, C::FP8, p.ld, p.N, p.BH, C::BM)) return s;
  if (fa_status s = make_map(&mk, k, C::FP8, p.ld, p.N, p.BH / p.g, C::BN)) return s;
  if (fa_status s = make_map(&mv, v, C::FP8, p.ld, p.N, p.BH / p.g, C::BN)) return s;
  auto kern = fa_fwd_kernel<C>;
  if (fa_status s = prepare_kernel<C>(kern, C::SMEM_ALLOC)) return s;
  p.n_qt = (p.N + C::BM - 1) / C::BM;
  p.n_kt = (p.N + C::BN - 1) / C::BN;
  p.n_st = (p.N + 127) / 128;
  p.total_items = p.BH * p.n_qt;
  p.group_heads = causal_group_heads(p.BH, 2ll * p.N * C::D * C::ELEM);
  p.status = di->status;
  p.timeout_ns = kWaitTimeoutNs;
  p.sched = sched_counter(di, stream);
  const int grid = p.total_items < di->sms ? p.total_items : di->sms;
  kern<<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(mq, mk, mv, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "forward kernel launch");
  return FA_OK;
}

// Two query tiles per CTA (fa_fwd_pp.cuh) for d <= 128.
template <class C>
fa_status launch_fwd_pp(const void* q, const void* k, const void* v, FwdParams p,
                        cudaStream_t stream) {
  DeviceInfo* di = nullptr;
  if (fa_status s = device_info(&di)) return s;
  CUtensorMap mq, mk, mv;
  if (fa_status s = make_map(&mq, q, C::FP8, p.ld, p.N, p.BH, C::BM)) return s;
  if (fa_status s = make_map(&mk, k, C::FP8, p.ld, p.N, p.BH / p.g, C::BN)) return s;
  if (fa_status s = make_map(&mv, v, C::FP8, p.ld, p.N, p.BH / p.g, C::BN)) return s;
  auto kern = fa_fwd_pp_kernel<C>;
  if (fa_status s = prepare_kernel<C>(kern, C::SMEM_ALLOC)) return s;
  {
    // The kernel re-splits its registers between warpgroups (setmaxnreg); the split
    // must fit the launch allocation or the growing warpgroups would wait forever.
    cudaFuncAttributes fa_attr;
    cudaError_t e = cudaFuncGetAttributes(&fa_attr, kern);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
    if (fa_attr.numRegs * C::THREADS < C::REGS_TOTAL)
      return fail(FA_ERR_CUDA, "forward kernel built with %d registers/thread: too few for its "
                  "register split", fa_attr.numRegs);
  }
  const int tiles = (p.N + C::BM - 1) / C::BM;
  p.n_qt = (tiles + 1) / 2;                       // query-tile PAIRS per head
  p.n_kt = (p.N + C::BN - 1) / C::BN;
  p.n_st = (p.N + 127) / 128;
  p.total_items = p.BH * p.n_qt;
  p.group_heads = causal_group_heads(p.BH, 2ll * p.N * C::D * C::ELEM);
  p.status = di->status;
  p.timeout_ns = kWaitTimeoutNs;
  p.sched = sched_counter(di, stream);
  const int grid = p.total_items < di->sms ? p.total_items : di->sms;
  kern<<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(mq, mk, mv, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "forward kernel launch");
  return FA_OK;
}

// Tuning knobs (compile-time): software-exp2 share, pipeline depth, softmax layout.
// Software-exp2 share of the two-tile kernel, in pairs of every 16 exponential pairs,
// per problem class; the one-tile d = 256 kernel counts quarters.
#ifndef FA_FWD_EMU
#define FA_FWD_EMU 0
#endif
#ifndef FA_FWD_D64_EMU
#define FA_FWD_D64_EMU 4
#endif
#ifndef FA_FWD_F8_EMU
#define FA_FWD_F8_EMU 0
#endif
#ifndef FA_FWD_D256_EMU
#define FA_FWD_D256_EMU 0
#endif
// d = 256 (one-tile kernel): rescale threshold with the compensated row sum
#ifndef FA_FWD_D256_TAU
#define FA_FWD_D256_TAU 8
#endif
// ring depth of the two-tile kernel at d = 64 and FP8 (K and V each)
#ifndef FA_FWD_NARROW_ST
#define FA_FWD_NARROW_ST 4
#endif
#ifndef FA_FWD_D128_KST
#define FA_FWD_D128_KST 2
#endif
#ifndef FA_FWD_D128_VST
#define FA_FWD_D128_VST 2
#endif
// two-tile kernel, bf16: rescale threshold (log2 units) with the compensated row sum.
// Measured against no threshold: +6 % on N(0,1) inputs at B1 H16 N32768, +4 % at d = 64,
// neutral on the outlier-key B4 H16 N4096 workload.  4 rather than 8: equally fast,
// and with 8 the uncompensated rounding of the other large probabilities (up to 2^8)
// took one row of that workload 0.0109 beyond the output's own rounding (4: 0.0058).
#ifndef FA_FWD_TAU
#define FA_FWD_TAU 4
#endif
#ifndef FA_FWD_PP_NORM
#define FA_FWD_PP_NORM 1
#endif
template <int D, bool FP8, int EMU>
struct FwdPick {
  // stage depths: deep rings where shared memory allows, 2 + 2 for bf16 d = 128
  static constexpr bool kWide = (D == 128 && !FP8);
  static constexpr int KST = kWide ? FA_FWD_D128_KST : FA_FWD_NARROW_ST;
  static constexpr int VST = kWide ? FA_FWD_D128_VST : FA_FWD_NARROW_ST;
  using Cfg = PPCfg<D, KST, VST, FP8, EMU, FA_FWD_TAU, FA_FWD_PP_NORM>;
  static const char* name() {
    static const std::string n = [] {
      char buf[128];
      std::snprintf(buf, sizeof buf, "fa_fwd_pp_kernel<PPCfg<%d,KST%d,VST%d,%s>>", D, Cfg::KST,
                    Cfg::VST, FP8 ? "e4m3" : "bf16");
      return std::string(buf);
    }();
    return n.c_str();
  }
  static fa_status launch(const void* q, const void* k, const void* v, FwdParams p,
                          cudaStream_t st) {
    return launch_fwd_pp<Cfg>(q, k, v, p, st);
  }
};
using FwdD64 = FwdPick<64, false, FA_FWD_D64_EMU>;
using FwdD128 = FwdPick<128, false, FA_FWD_EMU>;
using FwdF8D128 = FwdPick<128, true, FA_FWD_F8_EMU>;
using FwdD256 = FwdCfg<256, 64, 3, 2, false, FA_FWD_D256_EMU, FA_FWD_D256_TAU>;
using FwdF8D256 = FwdCfg<256, 128, 3, 2, true, FA_FWD_F8_EMU>;

// backward software-exp2 share: none (measured: at d = 64 with dQ formed in the dK/dV pass
// 671 against 658 TFLOP/s with a quarter, a half 649; at d = 128 750 either way)
#ifndef FA_BWD_EMU
#define FA_BWD_EMU 0
#endif
#ifndef FA_BWD_D256_EMU
#define FA_BWD_D256_EMU 0
#endif
#ifndef FA_BWD_D64_STAGES
#define FA_BWD_D64_STAGES 3
#endif
// d = 64: dQ accumulated by the dK/dV pass (fp32 atomics into the workspace) instead of
// a dQ pass of its own
#ifndef FA_BWD_D64_FUSED
#define FA_BWD_D64_FUSED 1
#endif
using DkdvD64 = DkdvCfg<64, 64, 128, FA_BWD_D64_STAGES, FA_BWD_D64_STAGES, 2, 1, FA_BWD_EMU>;
using DkdvD64F =
    DkdvCfg<64, 64, 128, FA_BWD_D64_STAGES, FA_BWD_D64_STAGES, 2, 1, FA_BWD_EMU, true>;
// d = 128: 128-row query tiles with one S^T and one dP^T buffer (TMEM: 128 + 128 + 2 x 128
// columns) run ahead of 64-row tiles with two of each: full-width (N = 128) products, half
// the hand-offs per query row, and S^T(i+1) still overlaps the dS^T(i) work
#ifndef FA_BWD_D128_EMU
#define FA_BWD_D128_EMU 1
#endif
using DkdvD128 = DkdvCfg<128, 128, 128, 2, 2, 1, 1, FA_BWD_D128_EMU>;
using DkdvD256 = DkdvCfg<256, 128, 64, 2, 1, 2, 2, FA_BWD_D256_EMU>;
using DqD64 = DqCfg<64, 128, FA_BWD_D64_STAGES, FA_BWD_D64_STAGES, 2, 1, FA_BWD_EMU>;
#ifndef FA_BWD_DQ128_EMU
#define FA_BWD_DQ128_EMU FA_BWD_EMU
#endif
// d = 128 dQ pass: one S buffer and two dP buffers (TMEM 128 + 2 x 128 + 128); S(j+1) and
// dP(j+1) are issued as soon as the compute warps have loaded S(j)
#ifndef FA_BWD_DQ128_SB
#define FA_BWD_DQ128_SB 1
#endif
using DqD128 = DqCfg<128, 128, 3, 2, FA_BWD_DQ128_SB, 3 - FA_BWD_DQ128_SB, FA_BWD_DQ128_EMU>;
using DqD256 = DqCfg<256, 64, 2, 1, 2, 2, FA_BWD_D256_EMU>;

// Launch `kern` as a programmatic dependent of the previous kernel in `stream`: it may
// be scheduled before that kernel ends; the kernel itself waits (griddepcontrol.wait)
// where it needs the previous one's results.
template <class K, class... Args>
cudaError_t launch_dependent(K kern, unsigned grid, unsigned threads, int smem, cudaStream_t stream,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <class CK, class CQ>
fa_status launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                     BwdParams p, cudaStream_t stream) {
  DeviceInfo* di = nullptr;
  if (fa_status s = device_info(&di)) return s;
  constexpr int D = CK::D;
  p.status = di->status;
  p.timeout_ns = kWaitTimeoutNs;
  // 1. D_i = dO_i . O_i over the stored head dim
  {
    const long long rows = static_cast<long long>(p.BH) * p.N;
    auto rowdot = [&](auto kern, int rpb) {
      long long blocks = (rows + rpb - 1) / rpb;
      const long long cap = static_cast<long long>(di->sms) * 8;
      if (blocks > cap) blocks = cap;
      kern<<<static_cast<int>(blocks), 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO),
          const_cast<float*>(p.drow), rows, CK::FUSEDQ ? p.dq_acc : nullptr);
    };
    static_assert(D == 64 || D == 128 || D == 256, "kernel head dims");
    if (p.ld == D)
      rowdot(fa_bwd_rowdot<D>, 256 / (D / 8));
    else if (p.ld == 96)
      rowdot(fa_bwd_rowdot<96>, 64);
    else
      rowdot(fa_bwd_rowdot<192>, 32);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "row-dot kernel launch");
  }
  // 2. dK, dV
  {
    CUtensorMap mq, mk, mv, mdo;
    if (fa_status s = make_map(&mq, q, false, p.ld, p.N, p.BH, CK::BMQ)) return s;
    if (fa_status s = make_map(&mdo, dO, false, p.ld, p.N, p.BH, CK::BMQ)) return s;
    if (fa_status s = make_map(&mk, k, false, p.ld, p.N, p.BH / p.g, CK::BN)) return s;
    if (fa_status s = make_map(&mv, v, false, p.ld, p.N, p.BH / p.g, CK::BN)) return s;
    CUtensorMap mdq = mq;                 // the dQ sums' map (fused path; unused otherwise)
    if constexpr (CK::FUSEDQ) {
      if (fa_status s = make_map_f32(&mdq, p.dq_acc, D, p.N, p.BH)) return s;
    }
    auto kern = fa_bwd_dkdv<CK>;
    if (fa_status s = prepare_kernel<CK>(kern, CK::SMEM_ALLOC)) return s;
    BwdParams pk = p;
    pk.n_qt = (p.N + CK::BMQ - 1) / CK::BMQ;
    pk.n_kt = (p.N + CK::BN - 1) / CK::BN;
    // a K/V head streams its g query heads' Q and dO
    pk.group_heads = causal_group_heads(p.BH / p.g, 4ll * p.g * p.N * p.ld);
    // one CTA per key/value head, key tile and d part
    const long long grid = static_cast<long long>(p.BH / p.g) * pk.n_kt * CK::NSPLIT;
    cudaError_t e = launch_dependent(kern, static_cast<unsigned>(grid), CK::THREADS, CK::SMEM_ALLOC,
                                     stream, mq, mk, mv, mdo, mdq, pk);
    if (e != cudaSuccess) return cuda_fail(e, "dK/dV kernel launch");
  }
  if constexpr (CK::FUSEDQ) {
    // 4. dQ = scale dQ_acc (the dK/dV pass summed it)
    const long long n8 = static_cast<long long>(p.BH) * p.N * D / 8;
    long long blocks = (n8 + 255) / 256;
    const long long cap = static_cast<long long>(di->sms) * 8;
    if (blocks > cap) blocks = cap;
    cudaError_t e = launch_dependent(fa_bwd_dq_convert, static_cast<unsigned>(blocks), 256, 0, stream,
                                     static_cast<const float*>(p.dq_acc),
                                     static_cast<__nv_bfloat16*>(p.dq), n8, p.scale);
    if (e != cudaSuccess) return cuda_fail(e, "dQ convert kernel launch");
    return FA_OK;
  }
  // 3. dQ
  {
    CUtensorMap mq, mk, mv, mdo;
    if (fa_status s = make_map(&mq, q, false, p.ld, p.N, p.BH, CQ::BM)) return s;
    if (fa_status s = make_map(&mdo, dO, false, p.ld, p.N, p.BH, CQ::BM)) return s;
    if (fa_status s = make_map(&mk, k, false, p.ld, p.N, p.BH / p.g, CQ::BN)) return s;
    if (fa_status s = make_map(&mv, v, false, p.ld, p.N, p.BH / p.g, CQ::BN)) return s;
    auto kern = fa_bwd_dq<CQ>;
    if (fa_status s = prepare_kernel<CQ>(kern, CQ::SMEM_ALLOC)) return s;
    BwdParams pq = p;
    pq.n_qt = (p.N + CQ::BM - 1) / CQ::BM;
    pq.n_kt = (p.N + CQ::BN - 1) / CQ::BN;
    pq.group_heads = causal_group_heads(p.BH, 4ll * p.N * p.ld);   // K and V of the head
    const long long grid = static_cast<long long>(p.BH) * pq.n_qt;
    cudaError_t e0 = launch_dependent(kern, static_cast<unsigned>(grid), CQ::THREADS,
                                      CQ::SMEM_ALLOC, stream, mq, mk, mv, mdo, pq);
    if (e0 != cudaSuccess) return cuda_fail(e0, "dQ kernel launch");
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "dQ kernel launch");
  }
  return FA_OK;
}

__global__ void wait_selftest_kernel(unsigned* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtl wc{&abort_flag, status, timeout_ns};
  // Nothing ever arrives on `bar`: the wait has to run out and report.
  mbar_wait(smem_u32(&bar), 0, wc, kSiteSelfTest);
  __syncthreads();
}

// Evaluates the kernels' exponential helpers on n values: the software exp2 of the
// FMA pipe (ex2_poly_pair, two values per call), the special-function-unit ex2 and
// CUDA's exp2f, for the accuracy test of the software exp2.
__global__ void exp2_probe_kernel(const float* x, float* y_poly, float* y_sfu, float* y_exp2f,
                                  int n) {
  const long long i = 2ll * (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const bool two = i + 1 < n;
  const float a = x[i], b = two ? x[i + 1] : 0.f;
  float pa, pb;
  f2_unpack(ex2_poly_pair(f2_pack(a, b)), pa, pb);
  y_poly[i] = pa;
  y_sfu[i] = ex2(a);
  y_exp2f[i] = exp2f(a);
  if (two) {
    y_poly[i + 1] = pb;
    y_sfu[i + 1] = ex2(b);
    y_exp2f[i + 1] = exp2f(b);
  }
}

size_t workspace_bytes(int B, int H, int N) {
  const size_t rows = static_cast<size_t>(B) * H * N;
  return (rows * sizeof(float) + 255) & ~static_cast<size_t>(255);
}

// The backward's workspace: D_i rows, then (fused d = 64 path) the fp32 dQ sums.
bool bwd_fused_dq(int d) { return FA_BWD_D64_FUSED != 0 && d == 64; }
size_t bwd_workspace_need(int B, int H, int N, int d) {
  size_t n = workspace_bytes(B, H, N);
  if (bwd_fused_dq(d))
    n += (static_cast<size_t>(B) * H * N * d * sizeof(float) + 255) & ~static_cast<size_t>(255);
  return n;
}

// FP8 backward: one bf16 [B,H,N,d] copy of a dequantised input, 256-byte aligned
size_t fp8_bwd_tensor_bytes(int B, int H, int N, int d) {
  return (static_cast<size_t>(B) * H * N * d * 2 + 255) & ~static_cast<size_t>(255);
}

// Host-buffer forward: the heads go through in kHostChunks chunks (fewer for small B*H;
// more chunks shorten the copy-in before the first kernel and the copy-out after the last),
// each staged in one of two device slots.  A slot holds Q, K, V, O (bf16) and LSE (fp32)
// of `hc` heads, each part 256-byte aligned.
#ifndef FA_HOST_CHUNKS
#define FA_HOST_CHUNKS 16
#endif
constexpr int kHostChunks = FA_HOST_CHUNKS;
static_assert(1 + 3 * kHostChunks <= 128, "host pipeline event pool");
int host_chunk_heads(int BH) {
  const int nc = BH < kHostChunks ? BH : kHostChunks;
  return (BH + nc - 1) / nc;
}
size_t host_slot_bytes(int hc, int N, int d) {
  const size_t t = (static_cast<size_t>(hc) * N * d * 2 + 255) & ~static_cast<size_t>(255);
  const size_t l = (static_cast<size_t>(hc) * N * 4 + 255) & ~static_cast<size_t>(255);
  return 4 * t + l;
}

// ------------------------------------------------------------------ no-allocation backward
// Fixed scratch for fa_bwd_noalloc: one fp32 D_i per row (B*H*N rows at most
// FA_BWD_NOALLOC_MAX_ROWS).  It lives in the module image, so every GPU that loads
// this library holds these 8 MiB until the process exits.  In host code the name
// is only a host-side stand-in; kernels get the device address looked up below.
static __device__ __align__(256) float g_bwd_noalloc_scratch[FA_BWD_NOALLOC_MAX_ROWS];

struct NoallocScratch {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  float* ptr = nullptr;
};
NoallocScratch g_noalloc[kMaxDevices];

// Device address of the scratch array on the current device, looked up once per
// device with that device current.
fa_status noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FA_ERR_CUDA, "device index %d out of range", dev);
  NoallocScratch& s = g_noalloc[dev];
  std::call_once(s.once, [&] {
    s.err = cudaGetSymbolAddress(reinterpret_cast<void**>(&s.ptr), g_bwd_noalloc_scratch);
  });
  if (s.err != cudaSuccess) return cuda_fail(s.err, "cudaGetSymbolAddress(no-alloc scratch)");
  *out = s.ptr;
  return FA_OK;
}

// ---------------------------------------------------------------- decoding
using DecD64 = DecCfg<64, 6, 6>;
using DecD128 = DecCfg<128, 3, 3>;
using DecD256 = DecCfg<256, 2, 2>;

struct DecPlan {
  int BHkv, R, bn, n_kt, split_tiles, n_split;
  size_t part_o_bytes, part_lse_bytes, total;
};

fa_status dec_check(int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                    bool* empty) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Nq < 0 || Nk < 0)
    return fail(FA_ERR_INVALID_ARG, "negative size B=%d Hq=%d Hkv=%d Nq=%d Nk=%d", B, Hq, Hkv, Nq, Nk);
  if (!std::isfinite(scale) || !(scale > 0.f))
    return fail(FA_ERR_INVALID_ARG, "scale must be finite and > 0 (got %g)", static_cast<double>(scale));
  if (d != 64 && d != 96 && d != 128 && d != 192 && d != 256)
    return fail(FA_ERR_UNSUPPORTED, "head dim %d not supported (64, 96, 128, 192, 256)", d);
  *empty = (B == 0 || Hq == 0 || Nq == 0);
  if (*empty) return FA_OK;
  if (Hkv == 0 || Hq % Hkv != 0)
    return fail(FA_ERR_INVALID_ARG, "Hq=%d must be a multiple of Hkv=%d", Hq, Hkv);
  if (static_cast<long long>(Hq / Hkv) * Nq > 128)
    return fail(FA_ERR_INVALID_ARG, "(Hq/Hkv)*Nq = %lld query rows per key/value head exceed 128",
                static_cast<long long>(Hq / Hkv) * Nq);
  if (Nk < 1) return fail(FA_ERR_INVALID_ARG, "Nk must be >= 1");
  if (causal && Nq > Nk) return fail(FA_ERR_INVALID_ARG, "causal decoding needs Nq <= Nk");
  if (static_cast<long long>(B) * Hkv > (1ll << 30)) return fail(FA_ERR_INVALID_ARG, "B*Hkv too large");
  return FA_OK;
}

// Split count: about two work items per SM, at least one key tile per split.
fa_status dec_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, DecPlan* pl) {
  DeviceInfo* di = nullptr;
  if (fa_status s = device_info(&di)) return s;
  pl->BHkv = B * Hkv;
  pl->R = (Hq / Hkv) * Nq;
  pl->bn = d <= 128 ? 128 : 64;
  const int dk = d <= 64 ? 64 : (d <= 128 ? 128 : 256);   // kernel head dim
  pl->n_kt = (Nk + pl->bn - 1) / pl->bn;
  // Splits per head: equal key ranges, CTAs taking items round-robin, so the kernel
  // lasts (rounds of items) x (longest item).  Pick the split count whose useful share
  // of that, all key tiles / (rounds x SMs x tiles per item), is within 1 % of the best,
  // with the fewest items (each item adds a partial result to write and merge).
  const long long tiles = static_cast<long long>(pl->BHkv) * pl->n_kt;
  const int max_ns = pl->n_kt < 1024 ? pl->n_kt : 1024;
  double eff[1025] = {};
  double best = 0.0;
  for (int ns = 1; ns <= max_ns; ++ns) {
    const long long st = (pl->n_kt + ns - 1) / ns;
    const long long items = static_cast<long long>(pl->BHkv) * ((pl->n_kt + st - 1) / st);
    const long long rounds = (items + di->sms - 1) / di->sms;
    eff[ns] = static_cast<double>(tiles) / static_cast<double>(rounds * di->sms * st);
    if (eff[ns] > best) best = eff[ns];
  }
  int pick = 1;
  long long pick_items = -1;
  for (int ns = 1; ns <= max_ns; ++ns) {
    if (eff[ns] < best - 0.01) continue;
    const long long st = (pl->n_kt + ns - 1) / ns;
    const long long items = static_cast<long long>(pl->BHkv) * ((pl->n_kt + st - 1) / st);
    if (pick_items < 0 || items < pick_items) {
      pick = ns;
      pick_items = items;
    }
  }
  pl->split_tiles = (pl->n_kt + pick - 1) / pick;
  pl->n_split = (pl->n_kt + pl->split_tiles - 1) / pl->split_tiles;
  const size_t rows = static_cast<size_t>(pl->BHkv) * pl->n_split * pl->R;
  pl->part_o_bytes = (rows * dk * sizeof(float) + 255) & ~static_cast<size_t>(255);
  pl->part_lse_bytes = (rows * sizeof(float) + 255) & ~static_cast<size_t>(255);
  pl->total = pl->part_o_bytes + pl->part_lse_bytes;
  return FA_OK;
}

template <class C>
fa_status launch_decode(const void* q, const void* k, const void* v, void* o, float* lse, DecParams p,
                        cudaStream_t stream) {
  DeviceInfo* di = nullptr;
  if (fa_status s = device_info(&di)) return s;
  CUtensorMap mq, mk, mv;
  if (fa_status s = make_map(&mq, q, false, p.ld, p.R, p.BHkv, C::BM)) return s;
  if (fa_status s = make_map(&mk, k, false, p.ld, p.Nk, p.BHkv, C::BN)) return s;
  if (fa_status s = make_map(&mv, v, false, p.ld, p.Nk, p.BHkv, C::BN)) return s;
  auto kern = fa_decode_split_kernel<C>;
  if (fa_status s = prepare_kernel<C>(kern, C::SMEM_ALLOC)) return s;
  p.status = di->status;
  p.timeout_ns = kWaitTimeoutNs;
  const int grid = p.total_items < di->sms ? p.total_items : di->sms;
  kern<<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(mq, mk, mv, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode split kernel launch");
  const long long threads = static_cast<long long>(p.BHkv) * p.R * (C::D / 4);
  const long long blocks = (threads + 255) / 256;
  // programmatic dependent launch: the merge kernel is scheduled while the split kernel
  // finishes and waits for it on the device (griddepcontrol.wait), which hides its launch
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, fa_decode_combine_kernel<C::D>, p, o, lse);
  if (e != cudaSuccess) return cuda_fail(e, "decode combine kernel launch");
  return FA_OK;
}

}  // namespace fa

using namespace fa;

extern "C" {

fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                     int Hkv, int N, int d, float scale, int causal, void* stream) {
  bool empty = false;
  if (fa_status s = check_common(B, Hq, N, scale, &empty)) return s;
  if (d != 64 && d != 96 && d != 128 && d != 192 && d != 256)
    return fail(FA_ERR_UNSUPPORTED, "head dim %d not supported (64, 96, 128, 192, 256)", d);
  if (empty) return FA_OK;
  if (Hkv <= 0 || Hq % Hkv != 0)
    return fail(FA_ERR_INVALID_ARG, "Hq=%d must be a positive multiple of Hkv=%d", Hq, Hkv);
  const void* ptrs[] = {q, k, v, o};
  const char* names[] = {"q", "k", "v", "o"};
  if (fa_status s = check_ptrs(ptrs, names, 4)) return s;
  if (lse && !aligned16(lse)) return fail(FA_ERR_INVALID_ARG, "lse is not 16-byte aligned");
  FwdParams p{};
  p.BH = B * Hq;
  p.H = Hq;
  p.g = Hq / Hkv;
  p.ld = d;
  p.N = N;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.o = o;
  p.lse = lse;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // d = 96 and 192 run on the 128 and 256 kernels: the tensor maps know the true row
  // length, so the extra columns load as zeros (adding nothing to Q K^T or P V) and the
  // epilogue stores only the first d
  switch (d) {
    case 64: return FwdD64::launch(q, k, v, p, st);
    case 96:
    case 128: return FwdD128::launch(q, k, v, p, st);
    default: return launch_fwd<FwdD256>(q, k, v, p, st);
  }
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                 int d, float scale, int causal, void* stream) {
  return fa_fwd_gqa(q, k, v, o, lse, B, H, H > 0 ? H : 1, N, d, scale, causal, stream);
}

fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale,
                     const float* k_scale, const float* v_scale, void* o, float* lse, int B, int H,
                     int N, int d, float scale, int causal, void* stream) {
  bool empty = false;
  if (fa_status s = check_common(B, H, N, scale, &empty)) return s;
  if (d != 64 && d != 96 && d != 128 && d != 192 && d != 256)
    return fail(FA_ERR_UNSUPPORTED, "FP8 head dim %d not supported (64, 96, 128, 192, 256)", d);
  if (empty) return FA_OK;
  const void* ptrs[] = {q8, k8, v8, o};
  const char* names[] = {"q8", "k8", "v8", "o"};
  if (fa_status s = check_ptrs(ptrs, names, 4)) return s;
  if (!q_scale || !k_scale || !v_scale) return fail(FA_ERR_INVALID_ARG, "FP8 scale pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(q_scale) | reinterpret_cast<uintptr_t>(k_scale) |
       reinterpret_cast<uintptr_t>(v_scale)) & 3u)
    return fail(FA_ERR_INVALID_ARG, "FP8 scales must be 4-byte aligned");
  if (lse && !aligned16(lse)) return fail(FA_ERR_INVALID_ARG, "lse is not 16-byte aligned");
  FwdParams p{};
  p.BH = B * H;
  p.H = H;
  p.g = 1;
  p.ld = d;
  p.N = N;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.o = o;
  p.lse = lse;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  // d <= 128 on the d = 128 kernel, larger on the one-tile d = 256 kernel (128-key tiles, as
  // the per-128-row scales need); narrower rows load zero columns past d
  if (d <= 128) return FwdF8D128::launch(q8, k8, v8, p, static_cast<cudaStream_t>(stream));
  return launch_fwd<FwdF8D256>(q8, k8, v8, p, static_cast<cudaStream_t>(stream));
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0) return 0;
  return bwd_workspace_need(B, H, N, d);
}

fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dO,
                     const float* lse, void* dq, void* dk, void* dv, void* workspace,
                     size_t workspace_bytes_, int B, int Hq, int Hkv, int N, int d, float scale,
                     int causal, void* stream) {
  bool empty = false;
  if (fa_status s = check_common(B, Hq, N, scale, &empty)) return s;
  if (d != 64 && d != 96 && d != 128 && d != 192 && d != 256)
    return fail(FA_ERR_UNSUPPORTED, "head dim %d not supported (64, 96, 128, 192, 256)", d);
  if (empty) return FA_OK;
  if (Hkv <= 0 || Hq % Hkv != 0)
    return fail(FA_ERR_INVALID_ARG, "Hq=%d must be a positive multiple of Hkv=%d", Hq, Hkv);
  const void* ptrs[] = {q, k, v, o, dO, lse, dq, dk, dv, workspace};
  const char* names[] = {"q", "k", "v", "o", "dO", "lse", "dq", "dk", "dv", "workspace"};
  if (fa_status s = check_ptrs(ptrs, names, 10)) return s;
  if (workspace_bytes_ < bwd_workspace_need(B, Hq, N, d))
    return fail(FA_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes_,
                bwd_workspace_need(B, Hq, N, d));
  BwdParams p{};
  p.BH = B * Hq;
  p.H = Hq;
  p.g = Hq / Hkv;
  p.ld = d;
  p.N = N;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.lse = lse;
  p.drow = static_cast<const float*>(workspace);
  p.dq_acc = bwd_fused_dq(d) ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                                        workspace_bytes(B, Hq, N))
                             : nullptr;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 64:
      if (bwd_fused_dq(d)) return launch_bwd<DkdvD64F, DqD64>(q, k, v, o, dO, p, st);
      return launch_bwd<DkdvD64, DqD64>(q, k, v, o, dO, p, st);
    case 96:
    case 128: return launch_bwd<DkdvD128, DqD128>(q, k, v, o, dO, p, st);
    default: return launch_bwd<DkdvD256, DqD256>(q, k, v, o, dO, p, st);
  }
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, void* dq, void* dk, void* dv, void* workspace,
                 size_t workspace_bytes_, int B, int H, int N, int d, float scale, int causal,
                 void* stream) {
  return fa_bwd_gqa(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes_, B, H,
                    H > 0 ? H : 1, N, d, scale, causal, stream);
}

// ------------------------------------------------------------------ host-buffer forward
size_t fa_fwd_host_workspace_size(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 0;
  return 2 * host_slot_bytes(host_chunk_heads(B * H), N, d);
}

fa_status fa_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                      float* lse_host, void* workspace, size_t workspace_bytes_, int B, int H,
                      int N, int d, float scale, int causal, void* stream) {
  bool empty = false;
  if (fa_status s = check_common(B, H, N, scale, &empty)) return s;
  if (d != 64 && d != 96 && d != 128 && d != 192 && d != 256)
    return fail(FA_ERR_UNSUPPORTED, "head dim %d not supported (64, 96, 128, 192, 256)", d);
  if (empty) return FA_OK;
  if (!q_host || !k_host || !v_host || !o_host)
    return fail(FA_ERR_INVALID_ARG, "host tensor pointer is NULL");
  const void* ptrs[] = {workspace};
  const char* names[] = {"workspace"};
  if (fa_status s = check_ptrs(ptrs, names, 1)) return s;
  const size_t need = fa_fwd_host_workspace_size(B, H, N, d);
  if (workspace_bytes_ < need)
    return fail(FA_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes_, need);
  DeviceInfo* di = nullptr;
  if (fa_status s = device_info(&di)) return s;
  std::lock_guard<std::mutex> lock(di->host_mu);
  if (!di->host_ready) {
    cudaError_t e = cudaStreamCreateWithFlags(&di->copy_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&di->copy_out, cudaStreamNonBlocking);
    for (int i = 0; e == cudaSuccess && i < 1 + 3 * kHostChunks; ++i)
      e = cudaEventCreateWithFlags(&di->host_ev[i], cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "host pipeline setup");
    di->host_ready = true;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H, hc = host_chunk_heads(BH), nc = (BH + hc - 1) / hc;
  const size_t slot = host_slot_bytes(hc, N, d);
  const size_t tb = (static_cast<size_t>(hc) * N * d * 2 + 255) & ~static_cast<size_t>(255);
  const size_t head_bytes = static_cast<size_t>(N) * d * 2, head_rows = static_cast<size_t>(N);
  // events: 0 = entry, then per chunk c: 1 + 3c inputs copied, 2 + 3c forward done,
  // 3 + 3c outputs copied
  cudaEvent_t* ev = di->host_ev;
  auto ck = [&](cudaError_t e, const char* what) -> fa_status {
    return e == cudaSuccess ? FA_OK : cuda_fail(e, what);
  };
  // the copies start after the work already queued on the caller's stream
  if (fa_status s = ck(cudaEventRecord(ev[0], st), "event record")) return s;
  if (fa_status s = ck(cudaStreamWaitEvent(di->copy_in, ev[0], 0), "stream wait")) return s;
  if (fa_status s = ck(cudaStreamWaitEvent(di->copy_out, ev[0], 0), "stream wait")) return s;
  for (int c = 0; c < nc; ++c) {
    const int h0 = c * hc, hn = (h0 + hc <= BH) ? hc : BH - h0;
    uint8_t* base = static_cast<uint8_t*>(workspace) + (c % 2) * slot;
    void* qd = base;
    void* kd = base + tb;
    void* vd = base + 2 * tb;
    void* od = base + 3 * tb;
    float* ld = reinterpret_cast<float*>(base + 4 * tb);
    const size_t off = static_cast<size_t>(h0) * head_bytes, nb = static_cast<size_t>(hn) * head_bytes;
    // inputs of this slot's previous chunk consumed by its forward
    if (c >= 2)
      if (fa_status s = ck(cudaStreamWaitEvent(di->copy_in, ev[2 + 3 * (c - 2)], 0), "stream wait"))
        return s;
    const void* src[3] = {q_host, k_host, v_host};
    void* dst[3] = {qd, kd, vd};
    for (int t = 0; t < 3; ++t)
      if (fa_status s = ck(cudaMemcpyAsync(dst[t], static_cast<const uint8_t*>(src[t]) + off, nb,
                                           cudaMemcpyHostToDevice, di->copy_in), "host-to-device copy"))
        return s;
    if (fa_status s = ck(cudaEventRecord(ev[1 + 3 * c], di->copy_in), "event record")) return s;
    // forward of the chunk, once its inputs are in and the slot's previous outputs are out
    if (fa_status s = ck(cudaStreamWaitEvent(st, ev[1 + 3 * c], 0), "stream wait")) return s;
    if (c >= 2)
      if (fa_status s = ck(cudaStreamWaitEvent(st, ev[3 + 3 * (c - 2)], 0), "stream wait")) return s;
    if (fa_status s = fa_fwd(qd, kd, vd, od, lse_host ? ld : nullptr, 1, hn, N, d, scale, causal, st))
      return s;
    if (fa_status s = ck(cudaEventRecord(ev[2 + 3 * c], st), "event record")) return s;
    // outputs back to the host
    if (fa_status s = ck(cudaStreamWaitEvent(di->copy_out, ev[2 + 3 * c], 0), "stream wait")) return s;
    if (fa_status s = ck(cudaMemcpyAsync(static_cast<uint8_t*>(o_host) + off, od, nb,
                                         cudaMemcpyDeviceToHost, di->copy_out), "device-to-host copy"))
      return s;
    if (lse_host)
      if (fa_status s = ck(cudaMemcpyAsync(lse_host + static_cast<size_t>(h0) * head_rows, ld,
                                           static_cast<size_t>(hn) * head_rows * 4,
                                           cudaMemcpyDeviceToHost, di->copy_out), "device-to-host copy"))
        return s;
    if (fa_status s = ck(cudaEventRecord(ev[3 + 3 * c], di->copy_out), "event record")) return s;
  }
  // the caller's stream completes only after the last copy out (the copy stream runs
  // its copies in order)
  return ck(cudaStreamWaitEvent(st, ev[3 + 3 * (nc - 1)], 0), "stream wait");
}

// ------------------------------------------------------------------ FP8 backward
size_t fa_bwd_fp8_workspace_size(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 0;
  return 3 * fp8_bwd_tensor_bytes(B, H, N, d) + bwd_workspace_need(B, H, N, d);
}

fa_status fa_bwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale,
                     const float* k_scale, const float* v_scale, const void* o, const void* dO,
                     const float* lse, void* dq, void* dk, void* dv, void* workspace,
                     size_t workspace_bytes_, int B, int H, int N, int d, float scale, int causal,
                     void* stream) {
  bool empty = false;
  if (fa_status s = check_common(B, H, N, scale, &empty)) return s;
  if (d != 64 && d != 96 && d != 128 && d != 192 && d != 256)
    return fail(FA_ERR_UNSUPPORTED, "FP8 head dim %d not supported (64, 96, 128, 192, 256)", d);
  if (empty) return FA_OK;
  const void* ptrs[] = {q8, k8, v8, o, dO, lse, dq, dk, dv, workspace};
  const char* names[] = {"q8", "k8", "v8", "o", "dO", "lse", "dq", "dk", "dv", "workspace"};
  if (fa_status s = check_ptrs(ptrs, names, 10)) return s;
  if (!q_scale || !k_scale || !v_scale) return fail(FA_ERR_INVALID_ARG, "FP8 scale pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(q_scale) | reinterpret_cast<uintptr_t>(k_scale) |
       reinterpret_cast<uintptr_t>(v_scale)) & 3u)
    return fail(FA_ERR_INVALID_ARG, "FP8 scales must be 4-byte aligned");
  const size_t need = fa_bwd_fp8_workspace_size(B, H, N, d);
  if (workspace_bytes_ < need)
    return fail(FA_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes_, need);
  DeviceInfo* di = nullptr;
  if (fa_status s = device_info(&di)) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // 1. the dequantised inputs, bf16, at the front of the workspace
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t tb = fp8_bwd_tensor_bytes(B, H, N, d);
  void* qd = ws;
  void* kd = ws + tb;
  void* vd = ws + 2 * tb;
  const long long groups = static_cast<long long>(B) * H * N * d / 16;
  const int n_st = (N + 127) / 128;
  long long blocks = (groups + 255) / 256;
  const long long cap = static_cast<long long>(di->sms) * 8;
  if (blocks > cap) blocks = cap;
  const void* src[3] = {q8, k8, v8};
  const float* scl[3] = {q_scale, k_scale, v_scale};
  void* dst[3] = {qd, kd, vd};
  for (int t = 0; t < 3; ++t) {
    fa_dequant_e4m3<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint8_t*>(src[t]), scl[t], static_cast<__nv_bfloat16*>(dst[t]), groups, d,
        N, n_st);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "dequantisation kernel launch");
  }
  // 2. the bf16 backward on them, with the rest of the workspace for D_i
  return fa_bwd(qd, kd, vd, o, dO, lse, dq, dk, dv, ws + 3 * tb, need - 3 * tb, B, H, N, d, scale,
                causal, stream);
}

// Same kernels and results as fa_bwd, but the per-row D_i scratch comes from the
// library's own fixed device array instead of a caller workspace, so this call
// never allocates.  The first call on a device looks up the array's address
// (cudaGetSymbolAddress) with that device current.  D_i is fully rewritten before
// it is read, so nothing needs clearing between calls; calls that overlap on the
// GPU (other streams, other threads) share the array and race.
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                         float scale, int causal, void* stream) {
  bool empty = false;
  if (fa_status s = check_common(B, H, N, scale, &empty)) return s;
  if (d != 64 && d != 96 && d != 128 && d != 192 && d != 256)
    return fail(FA_ERR_UNSUPPORTED, "head dim %d not supported (64, 96, 128, 192, 256)", d);
  if (empty) return FA_OK;
  const long long rows = static_cast<long long>(B) * H * N;
  if (rows > FA_BWD_NOALLOC_MAX_ROWS)
    return fail(FA_ERR_INVALID_ARG,
                "fa_bwd_noalloc: B*H*N = %lld rows exceeds the fixed scratch of %d rows; "
                "use fa_bwd with a caller workspace", rows, FA_BWD_NOALLOC_MAX_ROWS);
  const void* ptrs[] = {q, k, v, o, dO, lse, dq, dk, dv};
  const char* names[] = {"q", "k", "v", "o", "dO", "lse", "dq", "dk", "dv"};
  if (fa_status s = check_ptrs(ptrs, names, 9)) return s;
  float* scratch = nullptr;
  if (fa_status s = noalloc_scratch(&scratch)) return s;
  BwdParams p{};
  p.BH = B * H;
  p.H = H;
  p.g = 1;
  p.ld = d;
  p.N = N;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.lse = lse;
  p.drow = scratch;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 64: return launch_bwd<DkdvD64, DqD64>(q, k, v, o, dO, p, st);
    case 96:
    case 128: return launch_bwd<DkdvD128, DqD128>(q, k, v, o, dO, p, st);
    default: return launch_bwd<DkdvD256, DqD256>(q, k, v, o, dO, p, st);
  }
}

const char* fa_last_error_string(void) { return t_last_error.c_str(); }

fa_status fa_get_device_status(void* stream, int* code) {
  if (!code) return fail(FA_ERR_INVALID_ARG, "code is NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned v = 0;
  e = cudaMemcpyFromSymbol(&v, g_fa_status, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "read status word");
  const unsigned zero = 0;
  e = cudaMemcpyToSymbol(g_fa_status, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "clear status word");
  *code = static_cast<int>(v);
  return FA_OK;
}

fa_status fa_debug_wait_timeout_selftest(int timeout_us, void* stream) {
  if (timeout_us < 1 || timeout_us > 2000000)
    return fail(FA_ERR_INVALID_ARG, "timeout_us must be in [1, 2000000]");
  DeviceInfo* di = nullptr;
  if (fa_status s = device_info(&di)) return s;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      di->status, static_cast<unsigned long long>(timeout_us) * 1000ull);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return FA_OK;
}

fa_status fa_debug_exp2(const float* x, float* y_poly, float* y_sfu, float* y_exp2f, int n,
                        void* stream) {
  if (n < 0) return fail(FA_ERR_INVALID_ARG, "n = %d is negative", n);
  if (n == 0) return FA_OK;
  if (!x || !y_poly || !y_sfu || !y_exp2f) return fail(FA_ERR_INVALID_ARG, "null pointer");
  const int threads = 256;
  const long long pairs = (static_cast<long long>(n) + 1) / 2;
  const unsigned blocks = static_cast<unsigned>((pairs + threads - 1) / threads);
  exp2_probe_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly, y_sfu,
                                                                                 y_exp2f, n);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "exp2 probe launch");
  return FA_OK;
}

size_t fa_decode_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
  bool empty = false;
  if (dec_check(B, Hq, Hkv, Nq, Nk, d, 1.f, 0, &empty) != FA_OK || empty) return 0;
  DecPlan pl;
  if (dec_plan(B, Hq, Hkv, Nq, Nk, d, &pl) != FA_OK) return 0;
  return pl.total;
}

fa_status fa_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                    void* workspace, size_t workspace_bytes, void* stream) {
  bool empty = false;
  if (fa_status s = dec_check(B, Hq, Hkv, Nq, Nk, d, scale, causal, &empty)) return s;
  if (empty) return FA_OK;
  const void* ptrs[] = {q, k, v, o, workspace};
  const char* names[] = {"q", "k", "v", "o", "workspace"};
  if (fa_status s = check_ptrs(ptrs, names, 5)) return s;
  if (lse && !aligned16(lse)) return fail(FA_ERR_INVALID_ARG, "lse is not 16-byte aligned");
  DecPlan pl;
  if (fa_status s = dec_plan(B, Hq, Hkv, Nq, Nk, d, &pl)) return s;
  if (workspace_bytes < pl.total)
    return fail(FA_ERR_INVALID_ARG, "workspace of %zu bytes, %zu needed", workspace_bytes, pl.total);
  DecParams p{};
  p.BHkv = pl.BHkv;
  p.R = pl.R;
  p.Nq = Nq;
  p.Nk = Nk;
  p.ld = d;
  p.causal = causal ? 1 : 0;
  p.n_kt = pl.n_kt;
  p.split_tiles = pl.split_tiles;
  p.n_split = pl.n_split;
  p.total_items = pl.BHkv * pl.n_split;
  p.scale = scale;
  p.part_o = static_cast<float*>(workspace);
  p.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.part_o_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 64: return launch_decode<DecD64>(q, k, v, o, lse, p, st);
    case 96:
    case 128: return launch_decode<DecD128>(q, k, v, o, lse, p, st);
    default: return launch_decode<DecD256>(q, k, v, o, lse, p, st);
  }
}

int fa_version(void) { return 100; }

const char* fa_fwd_kernel_name(int head_dim, int fp8) {
  using namespace fa;
  if (fp8) {
    if (head_dim == 64 || head_dim == 96 || head_dim == 128) return FwdF8D128::name();
    if (head_dim == 192 || head_dim == 256) {
      static const std::string n = "fa_fwd_kernel<FwdCfg<256,KST3,VST2,e4m3>>";
      return n.c_str();
    }
    return nullptr;
  }
  switch (head_dim) {
    case 64: return FwdD64::name();
    case 96:
    case 128: return FwdD128::name();
    case 192:
    case 256: {
      static const std::string n = "fa_fwd_kernel<FwdCfg<256,KST" + std::to_string(FwdD256::KST) +
                                   ",VST" + std::to_string(FwdD256::VST) + ",bf16>>";
      return n.c_str();
    }
    default: return nullptr;
  }
}

}  // extern "C"
