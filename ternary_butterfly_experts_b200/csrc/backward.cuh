// Backward pass of the ButterflyMoE layer (the pages train the angles with
// the quantised base: technical summary, 2.4).  For dL/dy = gy:
//   per routed row r = t*k + j of expert e, with u = B(theta)^T x_t,
//   z = alpha W u, v = B(phi) z:
//     dg_r  = <v, gy_t>,          dv = g_r gy_t,
//     dz    = B(phi)^T dv,        dphi_e += d<dv, B(phi) z>/dphi,
//     du    = alpha W^T dz,       dW += alpha dz u^T (straight-through),
//     dx_t += B(theta) du,        dtheta_e += d<du, B(theta)^T x>/dtheta;
//   router: dl = g (dg - sum_j g dg), dW_g[e] += dl x_t, db[e] += dl,
//   dx_t += sum_j dl_j W_g[e_j].
//
// Rotations are invertible, so no stage's activations are stored: the
// backward walk starts from the butterfly's output and recovers each stage's
// input by the inverse rotation while it carries the gradient back.  For a
// Givens block [[c, -sg s], [sg s, c]] (sg = +1 for B, -1 for the blocks of
// B^T) with outputs (p', q') and their gradients (gp', gq'):
//     da += sg (gq' p' - gp' q'),
//     p = c p' + sg s q',   q = -sg s p' + c q'   (the same for the gradients).
//
// Layout: one warp per routed row; lane l holds the E = max(1, d/32)
// consecutive elements [l E, l E + E) of the row's value and gradient.
// gridDim.y CTAs per expert share that expert's bucket (warp w of CTA y takes
// the rows y*8 + w, y*8 + w + 8*gridDim.y, ...); a CTA sums the angle
// gradients of its rows in shared memory ([L][d/2] float32, shared atomics)
// and adds them to the expert's (zeroed) gradient with global atomics.  The
// order of the additions, and so the last bits, varies between runs.
#pragma once
#include "common.cuh"
#include "rotate.cuh"
#include "rotate_fast.cuh"

namespace bfmoe {

// Stage S (compile time, stride below E: both elements in this lane) of the
// forward walk, block sign sg.
template <int E, int S>
__device__ __forceinline__ void bw_fwd_in(float (&v)[E], const float2* __restrict__ tab_s, float sg, int lane,
                                          bool active) {
  constexpr int h = 1 << S;
#pragma unroll
  for (int q = 0; q < E; ++q) {
    if (q & h) continue;
    const float2 cs = active ? __ldg(tab_s + rot_index(lane * E + q, S)) : make_float2(1.f, 0.f);
    const float sn = sg * cs.y;
    const float a = v[q], b = v[q + h];
    v[q] = cs.x * a - sn * b;
    v[q + h] = sn * a + cs.x * b;
  }
}

// Stage s (stride h >= E: partner element in lane ^ (h/E)) of the forward walk.
template <int E>
__device__ __forceinline__ void bw_fwd_cross(float (&v)[E], int s, const float2* __restrict__ tab_s, float sg,
                                             int lane, bool active) {
  const int m = (1 << s) / E;
  const bool upper = (lane & m) != 0;
  const int i_lo = (lane & ~m) * E;
#pragma unroll
  for (int q = 0; q < E; ++q) {
    const float pv = __shfl_xor_sync(FULL_MASK, v[q], m);
    const float2 cs = active ? __ldg(tab_s + rot_index(i_lo + q, s)) : make_float2(1.f, 0.f);
    const float sn = sg * cs.y;
    const float a = upper ? pv : v[q];
    const float b = upper ? v[q] : pv;
    v[q] = upper ? (sn * a + cs.x * b) : (cs.x * a - sn * b);
  }
}

// One stage of the backward walk: v holds the stage's outputs, gv their
// gradients; on return they hold its inputs and their gradients, and the
// stage's angle gradients have been added to acc_s[d/2] (shared memory).
template <int E, int S>
__device__ __forceinline__ void bw_back_in(float (&v)[E], float (&gv)[E], const float2* __restrict__ tab_s, float sg,
                                           float* acc_s, int lane, bool active) {
  constexpr int h = 1 << S;
#pragma unroll
  for (int q = 0; q < E; ++q) {
    if (q & h) continue;
    const int r = rot_index(lane * E + q, S);
    const float2 cs = active ? __ldg(tab_s + r) : make_float2(1.f, 0.f);
    const float sn = sg * cs.y;
    const float p1 = v[q], q1 = v[q + h], gp = gv[q], gq = gv[q + h];
    if (active) atomicAdd(acc_s + r, sg * (gq * p1 - gp * q1));
    v[q] = cs.x * p1 + sn * q1;
    v[q + h] = -sn * p1 + cs.x * q1;
    gv[q] = cs.x * gp + sn * gq;
    gv[q + h] = -sn * gp + cs.x * gq;
  }
}

template <int E>
__device__ __forceinline__ void bw_back_cross(float (&v)[E], float (&gv)[E], int s, const float2* __restrict__ tab_s,
                                              float sg, float* acc_s, int lane, bool active) {
  const int m = (1 << s) / E;
  const bool upper = (lane & m) != 0;
  const int i_lo = (lane & ~m) * E;
#pragma unroll
  for (int q = 0; q < E; ++q) {
    const float pv = __shfl_xor_sync(FULL_MASK, v[q], m);
    const float pg = __shfl_xor_sync(FULL_MASK, gv[q], m);
    const int r = rot_index(i_lo + q, s);
    const float2 cs = active ? __ldg(tab_s + r) : make_float2(1.f, 0.f);
    const float sn = sg * cs.y;
    const float p1 = upper ? pv : v[q], q1 = upper ? v[q] : pv;
    const float gp = upper ? pg : gv[q], gq = upper ? gv[q] : pg;
    if (active && !upper) atomicAdd(acc_s + r, sg * (gq * p1 - gp * q1));
    v[q] = upper ? (-sn * p1 + cs.x * q1) : (cs.x * p1 + sn * q1);
    gv[q] = upper ? (-sn * gp + cs.x * gq) : (cs.x * gp + sn * gq);
  }
}

// Walks over all L stages: forward (0 .. L-1), backward descending
// (L-1 .. 0) and backward ascending (0 .. L-1); the in-lane stages are
// s < log2 E, unrolled at compile time.
template <int E, int S>
__device__ __forceinline__ void bw_fwd_in_all(float (&v)[E], const float2* tab, int half, float sg, int lane,
                                              bool active) {
  if constexpr (S < Log2<E>::value) {
    bw_fwd_in<E, S>(v, tab + static_cast<size_t>(S) * half, sg, lane, active);
    bw_fwd_in_all<E, S + 1>(v, tab, half, sg, lane, active);
  }
}
template <int E>
__device__ __forceinline__ void bw_walk_fwd(float (&v)[E], const float2* tab, int half, int L, float sg, int lane,
                                            bool active) {
  bw_fwd_in_all<E, 0>(v, tab, half, sg, lane, active);
  for (int s = Log2<E>::value; s < L; ++s) bw_fwd_cross<E>(v, s, tab + static_cast<size_t>(s) * half, sg, lane, active);
}
template <int E, int S>
__device__ __forceinline__ void bw_back_in_desc(float (&v)[E], float (&gv)[E], const float2* tab, int half, float sg,
                                                float* acc, int lane, bool active) {
  if constexpr (S >= 0) {
    bw_back_in<E, S>(v, gv, tab + static_cast<size_t>(S) * half, sg, acc + S * half, lane, active);
    bw_back_in_desc<E, S - 1>(v, gv, tab, half, sg, acc, lane, active);
  }
}
template <int E, int S>
__device__ __forceinline__ void bw_back_in_asc(float (&v)[E], float (&gv)[E], const float2* tab, int half, float sg,
                                               float* acc, int lane, bool active) {
  if constexpr (S < Log2<E>::value) {
    bw_back_in<E, S>(v, gv, tab + static_cast<size_t>(S) * half, sg, acc + S * half, lane, active);
    bw_back_in_asc<E, S + 1>(v, gv, tab, half, sg, acc, lane, active);
  }
}
template <int E>
__device__ __forceinline__ void bw_walk_back_desc(float (&v)[E], float (&gv)[E], const float2* tab, int half, int L,
                                                  float sg, float* acc, int lane, bool active) {
  for (int s = L - 1; s >= Log2<E>::value; --s)
    bw_back_cross<E>(v, gv, s, tab + static_cast<size_t>(s) * half, sg, acc + s * half, lane, active);
  bw_back_in_desc<E, Log2<E>::value - 1>(v, gv, tab, half, sg, acc, lane, active);
}
template <int E>
__device__ __forceinline__ void bw_walk_back_asc(float (&v)[E], float (&gv)[E], const float2* tab, int half, int L,
                                                 float sg, float* acc, int lane, bool active) {
  bw_back_in_asc<E, 0>(v, gv, tab, half, sg, acc, lane, active);
  for (int s = Log2<E>::value; s < L; ++s)
    bw_back_cross<E>(v, gv, s, tab + static_cast<size_t>(s) * half, sg, acc + s * half, lane, active);
}

template <int E>
__device__ __forceinline__ void bw_load(const float* __restrict__ src, float (&v)[E], int lane, bool active) {
#pragma unroll
  for (int q = 0; q < E; ++q) v[q] = active ? src[lane * E + q] : 0.f;
}
template <int E>
__device__ __forceinline__ void bw_store(float* __restrict__ dst, const float (&v)[E], int lane, bool active) {
  if (!active) return;
#pragma unroll
  for (int q = 0; q < E; ++q) dst[lane * E + q] = v[q];
}

// Output side, gridDim.y CTAs per expert e: for its rows (bucket position p, row
// r = rows[p], token t = r / k), from z = Z[p]: v = B(phi) z, dg[r] = <v, gy_t>,
// dv = gates[r] gy_t, then back through B(phi): dZ[p] = B(phi)^T dv and
// dphi[e] (added to the zeroed gradient).
template <int E>
__global__ __launch_bounds__(256) void bw_post_kernel(const float* __restrict__ Z, const float* __restrict__ gy,
                                                      const int32_t* __restrict__ rows,
                                                      const int32_t* __restrict__ offsets,
                                                      const float* __restrict__ gates,
                                                      const float2* __restrict__ cs_phi, int d, int L, int k, int N,
                                                      long long R, float* __restrict__ dZ, float* __restrict__ dg,
                                                      float* __restrict__ dphi) {
  extern __shared__ float acc[];  // [L][d/2]
  const int e = blockIdx.x;
  const int half = d / 2;
  for (int i = threadIdx.x; i < L * half; i += blockDim.x) acc[i] = 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const bool active = lane * E < d;
  const float2* tab = cs_phi + static_cast<size_t>(e) * L * half;
  const int p0 = offsets[e], p1 = offsets[e + 1];
  if (p0 < 0 || p1 < p0 || p1 > R) {
    if (threadIdx.x == 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(e));
  } else {
    for (int p = p0 + blockIdx.y * nw + w; p < p1; p += nw * gridDim.y) {
      const int r = rows[p];
      if (r < 0 || r >= R) {
        if (lane == 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(p));
        continue;
      }
      const int t = r / k;
      float v[E], gv[E];
      bw_load<E>(Z + static_cast<size_t>(p) * d, v, lane, active);
      bw_walk_fwd<E>(v, tab, half, L, 1.f, lane, active);
      bw_load<E>(gy + static_cast<size_t>(t) * d, gv, lane, active);
      float dot = 0.f;
#pragma unroll
      for (int q = 0; q < E; ++q) dot += v[q] * gv[q];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(FULL_MASK, dot, o);
      if (lane == 0) dg[r] = dot;
      const float g = gates[r];
#pragma unroll
      for (int q = 0; q < E; ++q) gv[q] *= g;
      bw_walk_back_desc<E>(v, gv, tab, half, L, 1.f, acc, lane, active);
      bw_store<E>(dZ + static_cast<size_t>(p) * d, gv, lane, active);
    }
  }
  __syncthreads();
  float* out = dphi + static_cast<size_t>(e) * L * half;
  for (int i = threadIdx.x; i < L * half; i += blockDim.x)
    if (acc[i] != 0.f) atomicAdd(out + i, acc[i]);
}

// Input side, gridDim.y CTAs per expert e: for its rows, from u = U[p] and
// du = dU[p], back through B(theta)^T (stages 0 .. L-1, blocks transposed):
// dXr[r] = B(theta) du and dtheta[e].
template <int E>
__global__ __launch_bounds__(256) void bw_pre_kernel(const float* __restrict__ U, const float* __restrict__ dU,
                                                     const int32_t* __restrict__ rows,
                                                     const int32_t* __restrict__ offsets,
                                                     const float2* __restrict__ cs_theta, int d, int L, long long R,
                                                     float* __restrict__ dXr, float* __restrict__ dtheta) {
  extern __shared__ float acc[];  // [L][d/2]
  const int e = blockIdx.x;
  const int half = d / 2;
  for (int i = threadIdx.x; i < L * half; i += blockDim.x) acc[i] = 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const bool active = lane * E < d;
  const float2* tab = cs_theta + static_cast<size_t>(e) * L * half;
  const int p0 = offsets[e], p1 = offsets[e + 1];
  if (p0 < 0 || p1 < p0 || p1 > R) {
    if (threadIdx.x == 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(e));
  } else {
    for (int p = p0 + blockIdx.y * nw + w; p < p1; p += nw * gridDim.y) {
      const int r = rows[p];
      if (r < 0 || r >= R) {
        if (lane == 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(p));
        continue;
      }
      float v[E], gv[E];
      bw_load<E>(U + static_cast<size_t>(p) * d, v, lane, active);
      bw_load<E>(dU + static_cast<size_t>(p) * d, gv, lane, active);
      bw_walk_back_asc<E>(v, gv, tab, half, L, -1.f, acc, lane, active);
      bw_store<E>(dXr + static_cast<size_t>(r) * d, gv, lane, active);
    }
  }
  __syncthreads();
  float* out = dtheta + static_cast<size_t>(e) * L * half;
  for (int i = threadIdx.x; i < L * half; i += blockDim.x)
    if (acc[i] != 0.f) atomicAdd(out + i, acc[i]);
}

// 2-bit codes of W^T: wt[i][o] = w[o][i] (the base read by columns, for
// du = alpha W^T dz with the row-reading ternary product).
__global__ void transpose_packed_kernel(const uint32_t* __restrict__ w, int d, int wpr, uint32_t* __restrict__ wt) {
  const long long n = static_cast<long long>(d) * wpr;
  for (long long q = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; q < n;
       q += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(q / wpr);       // row of W^T = column of W
    const int o0 = static_cast<int>(q % wpr) * 16;  // first column of W^T in this word
    uint32_t word = 0;
    for (int c = 0; c < 16 && o0 + c < d; ++c) {
      const uint32_t code = (w[static_cast<size_t>(o0 + c) * wpr + i / 16] >> (2 * (i % 16))) & 3u;
      word |= code << (2 * c);
    }
    wt[q] = word;
  }
}

// M partials: part[sl][o][i] = sum over bucket positions p of slice sl of
// dZ[p][o] U[p][i] (64 x 64 output tiles, 256 threads, 4 x 4 per thread;
// the positions are cut into gridDim.z slices).
constexpr int kOuterTile = 64;
constexpr int kOuterK = 16;
__global__ __launch_bounds__(256) void outer_tn_kernel(const float* __restrict__ dZ, const float* __restrict__ U,
                                                       long long R, int d, float* __restrict__ part) {
  __shared__ float sa[kOuterK][kOuterTile];
  __shared__ float sb[kOuterK][kOuterTile];
  const int o0 = blockIdx.y * kOuterTile, i0 = blockIdx.x * kOuterTile;
  const long long per = (R + gridDim.z - 1) / gridDim.z;
  const long long pa = blockIdx.z * per, pb = pa + per < R ? pa + per : R;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (long long p = pa; p < pb; p += kOuterK) {
    for (int l = threadIdx.x; l < kOuterK * kOuterTile; l += blockDim.x) {
      const int kk = l / kOuterTile, c = l % kOuterTile;
      const long long pp = p + kk;
      const bool in = pp < pb;
      sa[kk][c] = in && o0 + c < d ? dZ[pp * d + o0 + c] : 0.f;
      sb[kk][c] = in && i0 + c < d ? U[pp * d + i0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kOuterK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = sa[kk][ty * 4 + u];
        b[u] = sb[kk][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] += a[u] * b[v];
    }
    __syncthreads();
  }
  float* out = part + static_cast<size_t>(blockIdx.z) * d * d;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int o = o0 + ty * 4 + u, i = i0 + tx * 4 + v;
      if (o < d && i < d) out[static_cast<size_t>(o) * d + i] = acc[u][v];
    }
}

// dW = alpha * sum of the partials (fixed order); dalpha partial sums of
// W .* M per block (reduced by the next kernel in a fixed order).
__global__ __launch_bounds__(256) void outer_reduce_kernel(const float* __restrict__ part, int slices, int d,
                                                           float alpha, const uint32_t* __restrict__ w, int wpr,
                                                           float* __restrict__ dW, float* __restrict__ dalpha_part) {
  __shared__ float red[256];
  const long long n = static_cast<long long>(d) * d;
  float a = 0.f;
  for (long long q = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; q < n;
       q += static_cast<long long>(gridDim.x) * blockDim.x) {
    float m = 0.f;
    for (int sl = 0; sl < slices; ++sl) m += part[static_cast<size_t>(sl) * n + q];
    dW[q] = alpha * m;
    const int o = static_cast<int>(q / d), i = static_cast<int>(q % d);
    a += ternary_code_value((w[static_cast<size_t>(o) * wpr + i / 16] >> (2 * (i % 16))) & 3u) * m;
  }
  red[threadIdx.x] = a;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) dalpha_part[blockIdx.x] = red[0];
}

__global__ void sum_kernel(const float* __restrict__ part, int n, float* __restrict__ out) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    float s = 0.f;
    for (int i = 0; i < n; ++i) s += part[i];
    *out = s;
  }
}

// Per token: dl_j = g_j (dg_j - sum_j' g_j' dg_j'), then
// dx_t = sum_j (dXr[t k + j] + dl_j W_g[e_j]) in slot order.  One warp per
// token.
template <typename Tx>
__global__ __launch_bounds__(256) void bw_token_kernel(const float* __restrict__ dXr, const float* __restrict__ dg,
                                                       const float* __restrict__ gates,
                                                       const int32_t* __restrict__ idx,
                                                       const float* __restrict__ w_gate, long long T, int k, int d,
                                                       int N, float* __restrict__ dl, float* __restrict__ dx) {
  const int lane = threadIdx.x & 31;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long t = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5; t < T; t += nwarps) {
    float gd = 0.f;
    for (int j = 0; j < k; ++j) gd += gates[t * k + j] * dg[t * k + j];
    float dlj[BFMOE_MAX_K];
    int ej[BFMOE_MAX_K];
    for (int j = 0; j < k; ++j) {
      dlj[j] = gates[t * k + j] * (dg[t * k + j] - gd);
      ej[j] = idx[t * k + j];
      if (ej[j] < 0 || ej[j] >= N) {
        if (lane == 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(t));
        ej[j] = -1;
      }
      if (lane == 0) dl[t * k + j] = dlj[j];
    }
    for (int c = lane; c < d; c += 32) {
      float s = 0.f;
      for (int j = 0; j < k; ++j) {
        s += dXr[(t * k + j) * d + c];
        if (ej[j] >= 0) s += dlj[j] * w_gate[static_cast<size_t>(ej[j]) * d + c];
      }
      dx[t * d + c] = s;
    }
  }
}

// Router weights, one CTA per expert: dW_g[e] = sum over the expert's bucket
// (ascending tokens) of dl_r x_t, db[e] = sum of dl_r.  The bucket's tokens
// and dl are staged in shared memory 256 rows at a time; thread c sums the
// columns c, c + 256, ... in bucket order (the x loads of successive rows
// are independent, so many are in flight).
constexpr int kRouterGradCols = BFMOE_MAX_D / 256;
template <typename Tx>
__global__ __launch_bounds__(256) void bw_router_kernel(const Tx* __restrict__ x, const float* __restrict__ dl,
                                                        const int32_t* __restrict__ rows,
                                                        const int32_t* __restrict__ offsets, int k, int d,
                                                        long long R, float* __restrict__ dw_gate,
                                                        float* __restrict__ dbias) {
  __shared__ int s_tok[256];
  __shared__ float s_dl[256];
  const int e = blockIdx.x;
  const int p0 = offsets[e], p1 = offsets[e + 1];
  const bool ok = p0 >= 0 && p1 >= p0 && p1 <= R;
  float acc[kRouterGradCols];
#pragma unroll
  for (int m = 0; m < kRouterGradCols; ++m) acc[m] = 0.f;
  float db = 0.f;
  for (int base = ok ? p0 : p1; base < p1; base += 256) {
    const int n = p1 - base < 256 ? p1 - base : 256;
    if (static_cast<int>(threadIdx.x) < n) {
      const int r = rows[base + threadIdx.x];
      const bool valid = r >= 0 && r < R;
      s_tok[threadIdx.x] = valid ? r / k : -1;
      s_dl[threadIdx.x] = valid ? dl[r] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < n; ++j) {
      const int t = s_tok[j];
      if (t < 0) continue;
      const float g = s_dl[j];
      const Tx* xr = x + static_cast<size_t>(t) * d;
#pragma unroll
      for (int m = 0; m < kRouterGradCols; ++m) {
        const int c = threadIdx.x + 256 * m;
        if (c < d) acc[m] += g * to_f32(xr[c]);
      }
    }
    if (threadIdx.x == 0)
      for (int j = 0; j < n; ++j) db += s_dl[j];
    __syncthreads();
  }
#pragma unroll
  for (int m = 0; m < kRouterGradCols; ++m) {
    const int c = threadIdx.x + 256 * m;
    if (c < d) dw_gate[static_cast<size_t>(e) * d + c] = acc[m];
  }
  if (dbias && threadIdx.x == 0) dbias[e] = db;
}

}  // namespace bfmoe
