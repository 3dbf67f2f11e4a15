// Ternary product on the CUDA cores: Z = alpha * X . W_base^T with the
// weights read straight from the 2-bit codes.  Multiplying by -1, 0 or +1 is
// exact, so each term is an exact add, subtract or skip in float32 (the
// "additions only" form of the ternary multiply, technical summary 2.3).
// Used for the float32 path (a tensor-core tf32 product would round the
// activations) and for d < 64.
#pragma once
#include "common.cuh"

namespace bfmoe {

// 64 rows x 64 outputs per 256-thread block, 4x4 per thread, 32-wide slices.
template <typename Tin>
__global__ __launch_bounds__(256) void ternary_gemm_simt_kernel(const Tin* __restrict__ X,
                                                                const uint32_t* __restrict__ Wp, int wpr, long long R,
                                                                int d, float alpha, float* __restrict__ Z) {
  __shared__ float xs[32][64 + 4];
  __shared__ float ws[32][64 + 4];
  const long long r0 = static_cast<long long>(blockIdx.x) * 64;
  const int o0 = blockIdx.y * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < d; k0 += 32) {
    for (int q = threadIdx.x; q < 64 * 32; q += 256) {
      const int rr = q >> 5, kk = q & 31;
      const long long r = r0 + rr;
      const int o = o0 + rr, i = k0 + kk;
      xs[kk][rr] = (r < R && i < d) ? to_f32(X[static_cast<size_t>(r) * d + i]) : 0.f;
      float w = 0.f;
      if (o < d && i < d) w = ternary_code_value((Wp[static_cast<size_t>(o) * wpr + (i >> 4)] >> (2 * (i & 15))) & 3u);
      ws[kk][rr] = w;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long r = r0 + ty * 4 + i;
    if (r >= R) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = o0 + tx * 4 + j;
      if (o < d) Z[static_cast<size_t>(r) * d + o] = alpha * acc[i][j];
    }
  }
}

}  // namespace bfmoe
