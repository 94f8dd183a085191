// fa_dequant.cuh — FP8 e4m3 codes with per-128-row tile scales back to bf16.
//
// The FP8 forward's inputs are stored as code * scale, one fp32 scale per 128
// consecutive rows of a head (mypcrig.com post, section "FA3 の飛躍": block-wise
// quantisation).  The FP8 backward recomputes in bf16 from these values, so this
// pass expands them once: value = bf16_rne(float(code) * scale[tile]).  Every e4m3
// code is exact in fp16, so the only rounding is the final one to bf16.
//
// HBM-bound streaming pass: each thread step reads 16 codes (16 bytes) and writes 16
// bf16 values (32 bytes); the grid is a multiple of the SM count and strides over the
// whole tensor.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace fa {

// x8: e4m3 [BH, N, d]; scale: fp32 [BH, n_st]; out: bf16 [BH, N, d].  d % 16 == 0, so a
// group of 16 codes never crosses a row.
__global__ void __launch_bounds__(256) fa_dequant_e4m3(const uint8_t* __restrict__ x8,
                                                       const float* __restrict__ scale,
                                                       __nv_bfloat16* __restrict__ out,
                                                       long long groups, int d, int N, int n_st) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < groups;
       i += stride) {
    const long long row = (i * 16) / d;           // flattened (bh, n)
    const long long bh = row / N;
    const int tile = static_cast<int>(row - bh * N) / 128;
    const float s = __ldg(scale + bh * n_st + tile);
    const uint4 codes = __ldg(reinterpret_cast<const uint4*>(x8) + i);
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
    uint32_t res[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {   // two codes per step
        const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>(w[k] >> (16 * h));
        const __half2 v = static_cast<__half2>(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3));
        const float2 f = __half22float2(v);
        const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * s, f.y * s);
        res[2 * k + h] = *reinterpret_cast<const uint32_t*>(&b);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(out) + 2 * i;
    dst[0] = make_uint4(res[0], res[1], res[2], res[3]);
    dst[1] = make_uint4(res[4], res[5], res[6], res[7]);
  }
}

}  // namespace fa
