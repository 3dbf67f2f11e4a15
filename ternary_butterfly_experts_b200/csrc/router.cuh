// Router: float32 logits x W_g^T (+ b), top-k with the lower expert index
// first on equal logits, gates renormalised over the selected k.
//
// Mixture-of-experts selection is only defined in general on the pages
// (signalfieldnotes ButterflyMoE article, glossary "Mixtures of Experts");
// the logit, tie-break and gate conventions are this library's reading.
#pragma once
#include "common.cuh"

namespace bfmoe {

// Tiled float32 SIMT product: a 64-token x 64-expert tile per 256-thread
// block, 4x4 outputs per thread, 32-wide slices of d staged in shared memory.
template <typename Tx>
__global__ __launch_bounds__(256) void router_logits_simt_kernel(const Tx* __restrict__ x,
                                                                 const float* __restrict__ wg,
                                                                 const float* __restrict__ bias, int T, int d, int N,
                                                                 float* __restrict__ logits) {
  __shared__ float xs[32][64 + 4];
  __shared__ float gs[32][64 + 4];
  const int t0 = blockIdx.x * 64, e0 = blockIdx.y * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < d; k0 += 32) {
    for (int q = threadIdx.x; q < 64 * 32; q += 256) {
      const int rr = q >> 5, kk = q & 31;
      const int t = t0 + rr, e = e0 + rr, kx = k0 + kk;
      xs[kk][rr] = (t < T && kx < d) ? to_f32(x[static_cast<size_t>(t) * d + kx]) : 0.f;
      gs[kk][rr] = (e < N && kx < d) ? wg[static_cast<size_t>(e) * d + kx] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = gs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < N) logits[static_cast<size_t>(t) * N + e] = acc[i][j] + (bias ? bias[e] : 0.f);
    }
  }
}

// (va, ia) ranks before (vb, ib): larger logit, then lower index.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// One warp per token: each lane keeps its own sorted top-k over a strided
// subset of experts, then k rounds of a warp-wide arg-max merge.
__global__ __launch_bounds__(256) void router_topk_kernel(const float* __restrict__ logits, int T, int N, int k,
                                                          int32_t* __restrict__ idx, float* __restrict__ gates) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    float v[BFMOE_MAX_K];
    int id[BFMOE_MAX_K];
#pragma unroll
    for (int j = 0; j < BFMOE_MAX_K; ++j) {
      v[j] = -INFINITY;
      id[j] = 0x7fffffff;
    }
    const float* lrow = logits + static_cast<size_t>(t) * N;
    float th_v = -INFINITY;  // the lane's current k-th entry
    int th_i = 0x7fffffff;
    for (int e = lane; e < N; e += 32) {
      float l = lrow[e];
      if (isnan(l)) l = -INFINITY;
      if (!ranks_before(l, e, th_v, th_i)) continue;
      // insert, keeping v[0..k) sorted
      float cv = l;
      int ci = e;
#pragma unroll
      for (int j = 0; j < BFMOE_MAX_K; ++j) {
        if (j < k && ranks_before(cv, ci, v[j], id[j])) {
          const float tv = v[j];
          const int ti = id[j];
          v[j] = cv;
          id[j] = ci;
          cv = tv;
          ci = ti;
        }
        if (j == k - 1) {
          th_v = v[j];
          th_i = id[j];
        }
      }
    }
    float sel_v[BFMOE_MAX_K];
    int sel_i[BFMOE_MAX_K];
#pragma unroll
    for (int j = 0; j < BFMOE_MAX_K; ++j) {
      if (j >= k) break;
      float bv = v[0];
      int bi = id[0];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(FULL_MASK, bv, off);
        const int oi = __shfl_xor_sync(FULL_MASK, bi, off);
        if (ranks_before(ov, oi, bv, bi)) {
          bv = ov;
          bi = oi;
        }
      }
      sel_v[j] = bv;
      sel_i[j] = bi;
      if (id[0] == bi) {  // the owner pops its head
#pragma unroll
        for (int q = 0; q + 1 < BFMOE_MAX_K; ++q) {
          v[q] = v[q + 1];
          id[q] = id[q + 1];
        }
        v[BFMOE_MAX_K - 1] = -INFINITY;
        id[BFMOE_MAX_K - 1] = 0x7fffffff;
      }
    }
    if (lane == 0) {
      float z[BFMOE_MAX_K];
      float sum = 0.f;
      const bool finite_top = sel_v[0] > -INFINITY;
#pragma unroll
      for (int j = 0; j < BFMOE_MAX_K; ++j) {
        if (j >= k) break;
        z[j] = finite_top ? expf(sel_v[j] - sel_v[0]) : 1.f;
        sum += z[j];
      }
#pragma unroll
      for (int j = 0; j < BFMOE_MAX_K; ++j) {
        if (j >= k) break;
        idx[static_cast<size_t>(t) * k + j] = sel_i[j];
        gates[static_cast<size_t>(t) * k + j] = z[j] / sum;
      }
    }
  }
}

}  // namespace bfmoe
