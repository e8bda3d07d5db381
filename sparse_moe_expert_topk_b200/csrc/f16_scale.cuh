// The f16 copy of one token's bf16 activations that the NVFP4 experts' f16
// MMAs read, as a device function for a CTA of NT threads: used by the
// standalone conversion kernel and by the fused decode routing kernel, so
// both produce the same bytes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace ft {

// y = f16(x * 2^-s) and *xscale = 2^s, where the power of two s brings
// max_i |x_i| into [1, 2) (bf16 carries 8 significant bits, so every element
// down to 2^-14 of the largest is exact in f16; the smaller ones, below
// 2^-14 of the largest, keep an absolute error under 2^-25 of it). A row of
// zeros keeps s = 0; s is held to [-60, 60], so that xscale^2 is an fp32
// power of two; non-finite values pass through. The maximum is exact in any
// order, so the CTA size does not change the result. s_max: NT / 32 floats
// of shared memory; every thread of the CTA calls this.
template <int NT>
__device__ __forceinline__ void to_f16_scaled_row(const __nv_bfloat16* __restrict__ xr, int d,
                                                  __half* __restrict__ yr, float* __restrict__ xscale,
                                                  float* s_max) {
  float m = 0.f;
  for (int i = threadIdx.x; i < d; i += NT) m = fmaxf(m, fabsf(__bfloat162float(xr[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = m;
  __syncthreads();
  m = s_max[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) m = fmaxf(m, s_max[w]);
  int sh = 0;
  if (m > 0.f && m <= 3.0e38f) {
    int e;
    frexpf(m, &e);  // m = f * 2^e, f in [0.5, 1)
    sh = min(60, max(-60, e - 1));
  }
  const float down = ldexpf(1.f, -sh);
  for (int i = threadIdx.x; i < d; i += NT) yr[i] = __float2half_rn(__bfloat162float(xr[i]) * down);
  if (threadIdx.x == 0) *xscale = ldexpf(1.f, sh);
  __syncthreads();  // s_max may be reused by the caller
}

}  // namespace ft
