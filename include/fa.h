/*
 * fa.h — C ABI of libfa.so: exact scaled-dot-product attention on B200 (sm_100a).
 *
 * What is computed (every entry point): for every batch b and head h,
 *
 *     O = softmax(Q K^T * scale) V
 *
 * "FlashAttention — フラッシュアテンション" (systems-analysis.info wiki), section
 * 標準的なアテンションの問題点, displayed formula.  The work is done by fused,
 * tiled kernels that never write the N x N score matrix to global memory
 * (same page, sections タイリングとブロック処理 and CUDAカーネルの融合), with an
 * online softmax that carries a running row max and row sum
 * ("FlashAttentionとは？…" (issoh.co.jp), section 最大値と正規化項を持ち回る
 * オンラインsoftmaxの再スケール).  Results equal the definition up to
 * floating-point rounding, not bit for bit.
 *
 * Conventions shared by all entry points
 * --------------------------------------
 *  Layout    Q, K, V, O, dO, dQ, dK, dV are dense row-major [B, H, N, d]
 *            (d contiguous, then N, then H, then B); LSE and the FP8 scales
 *            are dense [B, H, N] and [B, H, ceil(N/128)].
 *  Pointers  device pointers (cudaMalloc / torch CUDA memory) on the current
 *            device, 16-byte aligned.  The caller owns every buffer; the
 *            library allocates and frees no device memory on any call.
 *  Sizes     B, H, N >= 0; d in {64, 96, 128, 192, 256} (bf16 and FP8).  N need
 *            not be a multiple of 128.  A call with B*H*N == 0 returns FA_OK
 *            and launches nothing (pointers may then be NULL).
 *  causal    0 = every key visible; 1 = key j visible to query i iff j <= i
 *            (lower triangular, top-left aligned; N_q == N_k).
 *  scale     multiplier of Q K^T, finite and > 0 (SDPA's default is 1/sqrt(d)).
 *  Streams   every call is asynchronous on `stream` (a cudaStream_t, 0 = the
 *            legacy default stream) and never synchronises the host.  The
 *            forwards keep a small work counter per stream handle: let a
 *            stream's forwards finish before destroying the stream, since a
 *            stream created afterwards may receive the same handle.
 *  Errors    argument errors return at once, before any CUDA call, and launch
 *            nothing.  There is no fallback path: an unsupported request fails
 *            (issoh.co.jp page, section CPUのPyTorch SDPA…: a forced fused path
 *            raises rather than silently running a slower one).
 *            fa_last_error_string() describes the most recent failure of the
 *            calling host thread.
 *  Device    every spin-wait inside the kernels is bounded in time; on expiry
 *            the kernel records a code in a device status word, drains its own
 *            in-flight work, frees its tensor memory and exits.  Read it with
 *            fa_get_device_status().
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,     /* NULL pointer, negative size, misalignment, bad scale */
  FA_ERR_UNSUPPORTED = 2,     /* valid request outside what the kernels implement (d) */
  FA_ERR_CUDA = 3,            /* a CUDA runtime call or kernel launch failed */
  FA_ERR_DEVICE_TIMEOUT = 4   /* reported by fa_get_device_status: a bounded wait expired */
} fa_status;

/*
 * fa_fwd — bf16 forward.  Tiled fused kernel: TMA tile loads, tcgen05 MMAs for
 * S = Q K^T and O += P V with fp32 accumulators in tensor memory, exp2-based
 * online softmax that rescales O only when a row max changes, causal tiles
 * above the diagonal skipped, persistent heaviest-first tile scheduler.
 *   q, k, v  in   bf16 [B,H,N,d]
 *   o        out  bf16 [B,H,N,d]  = softmax(scale Q K^T) V, rounded to nearest even
 *   lse      out  fp32 [B,H,N]    row logsumexp, natural log:
 *                                  lse_i = ln sum_{j visible} exp(scale q_i . k_j)
 *                                  (the normalisation statistic the backward reuses;
 *                                  issoh.co.jp page, section 逆伝播でL×L行列を保存せず
 *                                  再計算する設計).  May be NULL if not wanted.
 * Work distribution: the CTAs draw work items from a counter the library keeps per
 * stream (and per device); each launch leaves it at zero when it ends.  Launches in one
 * stream run one after the other and share it, launches in different streams have
 * their own.  A CUDA graph captured from this call keeps the counter of the capturing
 * stream, so two replays of it must not run at the same time.
 * Returns FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED (d not 64/96/128/192/256) or
 * FA_ERR_CUDA.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * fa_fwd_host_workspace_size — device workspace fa_fwd_host needs: two staging slots,
 * each with Q, K, V, O (bf16) and LSE (fp32) of one chunk of heads.  0 when empty.
 */
size_t fa_fwd_host_workspace_size(int B, int H, int N, int d);

/*
 * fa_fwd_host — fa_fwd on HOST buffers.  The heads go through in up to 16 chunks: while
 * one chunk's forward runs on `stream`, the next chunk's Q, K, V are copied in and the
 * previous chunk's O and LSE copied out, on two copy streams of the library's own, so
 * the host-to-device copies, the kernels and the device-to-host copies overlap.
 *   q_host, k_host, v_host   in   bf16 [B,H,N,d] in host memory (page-locked memory
 *                                 lets the copies overlap; pageable memory works too)
 *   o_host                   out  bf16 [B,H,N,d] in host memory
 *   lse_host                 out  fp32 [B,H,N] in host memory, or NULL
 *   workspace                device scratch of >= fa_fwd_host_workspace_size() bytes,
 *                            owned by the caller; contents on entry are ignored
 * Asynchronous like cudaMemcpyAsync: the work is queued in the order of `stream`, and
 * the results are in o_host / lse_host once `stream` has completed (the stream waits
 * for the last copy out).  Results equal fa_fwd's.  Errors as fa_fwd, plus
 * FA_ERR_INVALID_ARG for a NULL host pointer or a small workspace.
 */
fa_status fa_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                      float* lse_host, void* workspace, size_t workspace_bytes,
                      int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * fa_fwd_fp8 — FP8 (e4m3, OCP "fn" variant) forward with per-tile scales
 * (mypcrig.com post, section "FA3 の飛躍": per-tile rescaling and block-wise
 * quantisation keep FP8 attention accurate).
 *   q8, k8, v8        in  e4m3 [B,H,N,d]; real value = code * scale of its tile
 *   q_scale, k_scale,
 *   v_scale           in  fp32 [B,H,ceil(N/128)]: one scale per 128 consecutive rows
 *   o                 out bf16 [B,H,N,d]; lse out fp32 [B,H,N] (may be NULL)
 * The probabilities are rounded to e4m3 before the P V product (the product runs
 * on the FP8 tensor cores); everything else accumulates in fp32.
 * d is 64, 96, 128, 192 or 256.  Errors as fa_fwd.
 */
fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8,
                     const float* q_scale, const float* k_scale, const float* v_scale,
                     void* o, float* lse,
                     int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * fa_bwd_workspace_size — bytes of device workspace fa_bwd needs for these sizes:
 * fp32 D_i = sum_c dO_ic O_ic for every row, 256-byte aligned, and at d = 64 also
 * the fp32 dQ sums [B,H,N,64] (256-byte aligned).  0 when B*H*N == 0.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * fa_bwd — bf16 backward by recomputation: the score tile is recomputed from
 * Q and K, P is rebuilt from the saved lse, and no N x N matrix is stored
 * (issoh.co.jp page, section 逆伝播でL×L行列を保存せず再計算する設計).
 * Gradients of L = sum(O * dO):
 *   dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,  dS = P * (dP - D),
 *   dQ = scale dS K,  dK = scale dS^T Q.
 *   q, k, v, o, dO   in  bf16 [B,H,N,d] (o = fa_fwd's output for the same inputs)
 *   lse              in  fp32 [B,H,N]   (fa_fwd's lse for the same inputs)
 *   dq, dk, dv       out bf16 [B,H,N,d]
 *   workspace        scratch device memory of >= fa_bwd_workspace_size() bytes,
 *                    owned by the caller; contents on entry are ignored.
 * Launches, in stream order: the D_i row-sum pass, the dK/dV pass (one CTA per
 * key tile) and the dQ pass (one CTA per query tile); deterministic.  At d = 64
 * the dK/dV pass also forms dQ (a build choice): the row-sum pass zeroes
 * fp32 dQ sums in the workspace, the dK/dV CTAs add their key tile's share with
 * TMA reduce-adds, and a last pass writes dQ = scale * sums in bf16.  There dK
 * and dV repeat bit for bit, dQ to within its last bits (the order of the fp32
 * additions varies).  Errors as fa_fwd, plus FA_ERR_INVALID_ARG when the
 * workspace is too small.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, void* dq, void* dk, void* dv,
                 void* workspace, size_t workspace_bytes,
                 int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * fa_bwd_fp8_workspace_size — bytes of device workspace fa_bwd_fp8 needs: bf16 copies of
 * the three dequantised inputs followed by fa_bwd's workspace, each part 256-byte
 * aligned.  0 when B*H*N*d == 0.
 */
size_t fa_bwd_fp8_workspace_size(int B, int H, int N, int d);

/*
 * fa_bwd_fp8 — backward of the FP8 forward.  The pages define no FP8 backward; they
 * note only that FA3 still lacks one (issoh.co.jp page, sections
 * FA3のhopper配下からの導入とFA4のパッケージ導入 and FlashAttention-3と4のどちらを入れれば
 * よいですか？).  Reading taken: the gradients of L = sum(O * dO) with respect to the
 * dequantised inputs Q = q8 * q_scale, K = k8 * k_scale, V = v8 * v_scale (the
 * quantisation passes gradients straight through), computed by the bf16 backward after
 * one streaming pass that writes those inputs, rounded to bf16, into the workspace.
 *   q8, k8, v8, q_scale, k_scale, v_scale   in  as fa_fwd_fp8
 *   o, lse           in   fa_fwd_fp8's outputs for the same inputs
 *   dO               in   bf16 [B,H,N,d]
 *   dq, dk, dv       out  bf16 [B,H,N,d]: gradients for the dequantised Q, K, V
 *   workspace        scratch device memory of >= fa_bwd_fp8_workspace_size() bytes,
 *                    owned by the caller; contents on entry are ignored.
 * Launches, in stream order: three dequantisation passes, then fa_bwd's three passes.
 * Errors as fa_bwd.
 */
fa_status fa_bwd_fp8(const void* q8, const void* k8, const void* v8,
                     const float* q_scale, const float* k_scale, const float* v_scale,
                     const void* o, const void* dO, const float* lse,
                     void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                     int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * fa_bwd_noalloc — fa_bwd for callers that cannot allocate device memory.
 * (The pages describe nothing like it; it exists for integration only.)
 * Some callers have no way to hand the library a workspace: a plugin inside a
 * host program that owns every byte of device memory through its own pool, or a
 * latency-critical path where cudaMalloc's implicit device-wide synchronisation
 * is not acceptable.  This entry point takes the same inputs and outputs as
 * fa_bwd and gives the same results (at d = 64 through the separate dQ pass, which
 * needs no dQ sums), but keeps the per-row D_i scratch in a fixed
 * array inside the library (FA_BWD_NOALLOC_MAX_ROWS fp32 values = 8 MiB, held on
 * every GPU that loads the library until the process exits).  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *   Sizes: B*H*N must be <= FA_BWD_NOALLOC_MAX_ROWS, else FA_ERR_INVALID_ARG
 *          (use fa_bwd with a caller workspace for larger problems).
 *   Set-up: the first call on each device looks up the array's device address
 *          with that device current; make that first call before any stream
 *          capture.
 *   Sharing: all calls on a device share the one array.  D_i is fully rewritten
 *          by each call before it is read, so no clearing is needed, but calls
 *          that overlap on the GPU (other streams or host threads) race and give
 *          wrong gradients: serialise them.
 * Other arguments and errors as fa_bwd.
 */
#define FA_BWD_NOALLOC_MAX_ROWS (1 << 21)
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                         const void* dO, const float* lse, void* dq, void* dk, void* dv,
                         int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * Grouped query heads (GQA / MQA, "FlashAttention — フラッシュアテンション"
 * (systems-analysis.info), section FlashAttention-2（2023年）) for the full-length
 * forward and backward: Hq query heads share Hkv key/value heads, query head h reads
 * key/value head h / (Hq / Hkv).
 *   q, o, dO, dq     bf16 [B, Hq, N, d];  k, v, dk, dv  bf16 [B, Hkv, N, d];
 *   lse              fp32 [B, Hq, N];     workspace     >= fa_bwd_workspace_size(B, Hq, N, d)
 * dk, dv sum the contributions of every query head of the group.  Hq % Hkv must be
 * 0 (FA_ERR_INVALID_ARG otherwise).  Everything else as fa_fwd / fa_bwd, which are
 * these calls with Hkv = Hq.
 */
fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int Hq, int Hkv, int N, int d, float scale, int causal, void* stream);
fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dO,
                     const float* lse, void* dq, void* dk, void* dv, void* workspace,
                     size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d, float scale,
                     int causal, void* stream);

/*
 * Decoding: few query rows against a long key/value sequence, with grouped query
 * heads (GQA / MQA).  Same exact attention as fa_fwd.  Decoding reads Q of length 1
 * against the whole KV cache, so reading K and V bounds it ("FlashAttentionとは？…"
 * (issoh.co.jp), section 短い系列の効果とデコード向け最適化の違い); shared K/V heads
 * are the GQA/MQA of "FlashAttention — フラッシュアテンション" (systems-analysis.info),
 * section FlashAttention-2（2023年）.  The key split and its merge are the
 * online-softmax rescale applied across key ranges:
 *   O[b,h,i,:] = softmax_j(scale * q[b,h,i,:] . k[b,h/g,j,:]) v[b,h/g,j,:],
 *   g = Hq / Hkv, causal: query i sees keys j <= Nk - Nq + i (the queries are the
 *   last Nq positions of the sequence).
 *
 * fa_decode_workspace_size — bytes of device workspace fa_decode needs (partial
 * results of the key splits; the split count follows the current device's SM
 * count).  0 for arguments fa_decode would reject.
 */
size_t fa_decode_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d);

/*
 * fa_decode — O and row logsumexp for the layout above.
 *   q          bf16 [B, Hq, Nq, d], d contiguous       (device, read)
 *   k, v       bf16 [B, Hkv, Nk, d]                    (device, read)
 *   o          bf16 [B, Hq, Nq, d]                     (device, written)
 *   lse        fp32 [B, Hq, Nq] natural-log logsumexp  (device, written; may be NULL)
 *   d in {64, 96, 128, 192, 256}; Hq % Hkv == 0; (Hq / Hkv) * Nq <= 128; 1 <= Nq; 1 <= Nk;
 *   causal requires Nq <= Nk.
 *   workspace  >= fa_decode_workspace_size() bytes of device memory, 16-byte aligned,
 *              owned by the caller, contents ignored and overwritten.
 * Asynchronous on `stream`; allocates nothing.  Errors: FA_ERR_INVALID_ARG for a
 * null or misaligned pointer, out-of-range sizes or a too-small workspace (nothing
 * launched); FA_ERR_UNSUPPORTED for another d; FA_ERR_CUDA if a launch fails.
 */
fa_status fa_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                    void* workspace, size_t workspace_bytes, void* stream);

/* fa_last_error_string — text of the calling thread's last failure ("" if none). */
const char* fa_last_error_string(void);

/*
 * fa_get_device_status — synchronises `stream`, then reads and clears the
 * device status word of the current device.  *code = 0 when no kernel has
 * reported a problem; otherwise (FA_ERR_DEVICE_TIMEOUT << 24) | site, where
 * site names the wait that expired.  Returns FA_ERR_CUDA if the copy fails.
 */
fa_status fa_get_device_status(void* stream, int* code);

/*
 * fa_debug_wait_timeout_selftest — launches one CTA that waits on a barrier
 * nothing will ever complete, with the given bound in microseconds (1..2000000).
 * The wait must expire, record FA_ERR_DEVICE_TIMEOUT in the status word and
 * return; the context stays usable.  Used by the tests of the fault path.
 */
fa_status fa_debug_wait_timeout_selftest(int timeout_us, void* stream);

/*
 * fa_debug_exp2 — evaluates, for the n fp32 values x[0..n-1], the exponential
 * helpers the kernels use: y_poly = the software 2^x on the FMA pipe (Cody-Waite
 * reduction and a degree-3 minimax polynomial; FA4's partial software exponential,
 * "FlashAttentionとは？…" (issoh.co.jp), section FA4のB200で1613TFLOPs…), y_sfu =
 * the special-function unit's ex2.approx.ftz, y_exp2f = CUDA's exp2f.  All four
 * are fp32 device arrays of n elements owned by the caller.  The software form is
 * specified for x <= 127 with relative error <= 7.5e-5 on (-125.99, 127] and
 * <= 1.5e-4 on [-126, -125.99] (a subnormal encoding there); inputs at or below
 * -126 give a value in [0, 2^-126].  n < 0 or a null pointer with n > 0:
 * FA_ERR_INVALID_ARG.  Used by the accuracy test of the software exponential.
 */
fa_status fa_debug_exp2(const float* x, float* y_poly, float* y_sfu, float* y_exp2f, int n,
                        void* stream);

/* fa_version — library version, major*10000 + minor*100 + patch. */
int fa_version(void);

/*
 * fa_fwd_kernel_name — name of the forward kernel that fa_fwd (fp8 = 0) or
 * fa_fwd_fp8 (fp8 != 0) launches for head dimension `head_dim`, with its
 * tile configuration, e.g. "fa_fwd_pp_kernel<PPCfg<128,KST2,VST2,bf16>>".  The
 * string is static and owned by the library.  Returns NULL for an unsupported
 * head dimension.  Host only; launches nothing.
 */
const char* fa_fwd_kernel_name(int head_dim, int fp8);

#ifdef __cplusplus
}
#endif
#endif /* FA_H_ */
