// Dense expert alpha * B(phi_e) . W_base . B(theta_e)^T (technical summary,
// 2.1), for checking the non-materialising forward.  One block per input
// column i: the column is the expert applied to the unit vector e_i, computed
// in shared memory stage by stage; no scratch memory beyond shared memory.
#pragma once
#include "common.cuh"

namespace bfmoe {

// In stage s the q-th pair (in ascending order of its lower element) has
// lower element ((q >> s) << (s+1)) | (q & (2^s - 1)) and rotation index q.
__device__ __forceinline__ void smem_stage(float* u, int d, int s, const float* __restrict__ ang_s, bool transpose) {
  const int h = 1 << s;
  for (int q = threadIdx.x; q < d / 2; q += blockDim.x) {
    const int lo = ((q >> s) << (s + 1)) | (q & (h - 1));
    const int hi = lo + h;
    float sn, c;
    sincosf(ang_s[q], &sn, &c);
    if (transpose) sn = -sn;
    const float a = u[lo], b = u[hi];
    u[lo] = c * a - sn * b;
    u[hi] = sn * a + c * b;
  }
  __syncthreads();
}

__global__ __launch_bounds__(256) void materialize_kernel(const uint32_t* __restrict__ Wp, int wpr, int d, int L,
                                                          float alpha, const float* __restrict__ theta_e,
                                                          const float* __restrict__ phi_e, float* __restrict__ out) {
  extern __shared__ float sm[];
  float* u = sm;
  float* z = sm + d;
  const int col = blockIdx.x;
  for (int a = threadIdx.x; a < d; a += blockDim.x) u[a] = (a == col) ? 1.f : 0.f;
  __syncthreads();
  const int half = d / 2;
  for (int s = L - 1; s >= 0; --s) smem_stage(u, d, s, theta_e + static_cast<size_t>(s) * half, true);
  for (int o = threadIdx.x; o < d; o += blockDim.x) {
    float acc = 0.f;
    for (int i = 0; i < d; ++i)
      acc = fmaf(ternary_code_value((Wp[static_cast<size_t>(o) * wpr + (i >> 4)] >> (2 * (i & 15))) & 3u), u[i], acc);
    z[o] = alpha * acc;
  }
  __syncthreads();
  for (int s = 0; s < L; ++s) smem_stage(z, d, s, phi_e + static_cast<size_t>(s) * half, false);
  for (int a = threadIdx.x; a < d; a += blockDim.x) out[static_cast<size_t>(a) * d + col] = z[a];
}

}  // namespace bfmoe
