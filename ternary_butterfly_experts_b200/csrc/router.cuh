// Router: float32 logits x W_g^T (+ b), top-k with the lower expert index
// first on equal logits, gates renormalised over the selected k.  A token
// whose k-th and (k+1)-th float32 logits are too close for float32 to rank
// them is settled again from exact logits (router_fixup_kernel).
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

// ---------------------------------------------------------------------------
// Undecided tokens.
//
// Float32 logits carry rounding errors that grow with |l| and d: simulated
// for the tensor-core router's order of accumulation, at most
// 4.3e-6 (1 + |l|) at d = 2048 and 1.1e-6 (1 + |l|) at d = 512.  That is the
// width of the near-tie band (1e-5) within which a float64 reference may rank
// differently, so a float32 top-k is only trusted when each selected logit
// clears the next one (and the k-th the best logit left out) by more than
// 2 eps, with
//     eps(l) = eps_c (1 + |l|),   eps_c = 2e-5 sqrt(d / 2048)
// (about 5 to 10 times the simulated worst case).  Other tokens (a few per
// thousand; every near tie) are listed for router_fixup_kernel, which settles
// them with logits that are exact to ~1e-13 (double-float32 sums).
// ---------------------------------------------------------------------------
// Every gap of the sorted list v[0] >= ... >= v[k-1] >= rej (the order of
// the slots as well as the set) must clear the band.
__device__ __forceinline__ bool gap_is_clear(float a, float b, float eps_c) {
  if (!(b > -INFINITY)) return true;
  const float e = eps_c * (1.f + fmaxf(fabsf(a), fabsf(b)));
  return a - b > 2.f * e;
}
__device__ __forceinline__ bool topk_is_clear(const float* v, int k, float rej, float eps_c) {
  bool clear = true;
#pragma unroll
  for (int j = 0; j < BFMOE_MAX_K; ++j)
    if (j < k) clear = clear && gap_is_clear(v[j], j + 1 < k ? v[j + 1] : rej, eps_c);
  return clear;
}

// Gates from float32 logits in descending order: softmax over the k.
__device__ __forceinline__ void gates_f32(const float* v, int k, float* g) {
  float z[BFMOE_MAX_K];
  float sum = 0.f;
  const bool finite_top = v[0] > -INFINITY;
  for (int j = 0; j < k; ++j) {
    z[j] = finite_top ? expf(v[j] - v[0]) : 1.f;
    sum += z[j];
  }
  for (int j = 0; j < k; ++j) g[j] = z[j] / sum;
}

// Double-float32 arithmetic (error-free transformations; the _rn intrinsics
// keep the compiler from fusing the products into the sums).
__device__ __forceinline__ void two_sum(float a, float b, float& s, float& e) {
  s = __fadd_rn(a, b);
  const float bb = __fsub_rn(s, a);
  e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
}
// (s, c) += x * w, the product's rounding error carried exactly
__device__ __forceinline__ void df_mac(float x, float w, float& s, float& c) {
  const float p = __fmul_rn(x, w);
  const float pe = fmaf(x, w, -p);
  float t;
  two_sum(s, p, s, t);
  c = __fadd_rn(c, __fadd_rn(t, pe));
}
// (s, c) += (s2, c2)
__device__ __forceinline__ void df_add(float& s, float& c, float s2, float c2) {
  float t;
  two_sum(s, s2, s, t);
  c = __fadd_rn(c, __fadd_rn(c2, t));
}
// (hi, lo) with |lo| <= ulp(hi) / 2, so pairs compare lexicographically
__device__ __forceinline__ void df_normalize(float s, float c, float& hi, float& lo) {
  hi = __fadd_rn(s, c);
  lo = __fsub_rn(c, __fsub_rn(hi, s));
}
__device__ __forceinline__ bool df_ranks_before(float ah, float al, int ai, float bh, float bl, int bi) {
  return ah > bh || (ah == bh && (al > bl || (al == bl && ai < bi)));
}

// Four consecutive elements of a row as float32 (16-byte aligned for
// float32, 8-byte for bfloat16).
__device__ __forceinline__ void load4_f32(const float* p, float (&v)[4]) {
  const float4 q = *reinterpret_cast<const float4*>(p);
  v[0] = q.x;
  v[1] = q.y;
  v[2] = q.z;
  v[3] = q.w;
}
__device__ __forceinline__ void load4_f32(const __nv_bfloat16* p, float (&v)[4]) {
  const uint2 q = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&q.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&q.y);
  v[0] = __low2float(a);
  v[1] = __high2float(a);
  v[2] = __low2float(b);
  v[3] = __high2float(b);
}

// Double-float logits of four experts at once (e[j] < 0: none; its result is
// not used), so that the loads and sums of the four overlap.
template <typename Tx>
__device__ __forceinline__ void df_logits4(const Tx* __restrict__ xr, const float* __restrict__ wg,
                                           const float* __restrict__ bias, int d, const int (&e)[4], int lane,
                                           float (&h)[4], float (&l)[4]) {
  const float* wr[4];
  float sa[4], ca[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    wr[j] = wg + static_cast<size_t>(e[j] >= 0 ? e[j] : 0) * d;
    sa[j] = 0.f;
    ca[j] = 0.f;
  }
  const bool aligned = ((reinterpret_cast<uintptr_t>(xr) & (4 * sizeof(Tx) - 1)) |
                        (reinterpret_cast<uintptr_t>(wg) & 15)) == 0;
  if ((d & 127) == 0 && aligned) {
    // four consecutive elements per lane and step: 16-byte weight loads
    for (int i0 = 4 * lane; i0 < d; i0 += 128) {
      float xv[4];
      load4_f32(xr + i0, xv);
      float4 w4[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) w4[j] = *reinterpret_cast<const float4*>(wr[j] + i0);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        df_mac(xv[0], w4[j].x, sa[j], ca[j]);
        df_mac(xv[1], w4[j].y, sa[j], ca[j]);
        df_mac(xv[2], w4[j].z, sa[j], ca[j]);
        df_mac(xv[3], w4[j].w, sa[j], ca[j]);
      }
    }
  } else {
#pragma unroll 4
    for (int i = lane; i < d; i += 32) {
      const float xv = to_f32(xr[i]);
#pragma unroll
      for (int j = 0; j < 4; ++j) df_mac(xv, wr[j][i], sa[j], ca[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float s2 = __shfl_xor_sync(FULL_MASK, sa[j], o);
      const float c2 = __shfl_xor_sync(FULL_MASK, ca[j], o);
      df_add(sa[j], ca[j], s2, c2);
    }
    if (bias && e[j] >= 0) df_add(sa[j], ca[j], bias[e[j]], 0.f);
    df_normalize(sa[j], ca[j], h[j], l[j]);
    if (isnan(h[j]) || isnan(l[j])) {
      h[j] = -INFINITY;
      l[j] = 0.f;
    }
  }
}

// One warp per token: each lane keeps its own sorted list of the k + 1 best
// logits of a strided subset of experts, then k + 1 rounds of a warp-wide
// arg-max merge give the k candidates and the best of the rest.
template <typename Tx>
__global__ __launch_bounds__(256) void router_topk_kernel(const float* __restrict__ logits, const Tx* __restrict__ x,
                                                          const float* __restrict__ wg, const float* __restrict__ bias,
                                                          int T, int d, int N, int k, float eps_c,
                                                          int32_t* __restrict__ idx, float* __restrict__ gates,
                                                          int* __restrict__ unsure_list) {
  constexpr int M = BFMOE_MAX_K + 1;
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int kk = k + 1;  // list length
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    float v[M];
    int id[M];
#pragma unroll
    for (int j = 0; j < M; ++j) {
      v[j] = -INFINITY;
      id[j] = 0x7fffffff;
    }
    const float* lrow = logits + static_cast<size_t>(t) * N;
    float th_v = -INFINITY;  // the lane's current last entry
    int th_i = 0x7fffffff;
    for (int e = lane; e < N; e += 32) {
      float l = lrow[e];
      if (isnan(l)) l = -INFINITY;
      if (!ranks_before(l, e, th_v, th_i)) continue;
      // insert, keeping v[0..kk) sorted
      float cv = l;
      int ci = e;
#pragma unroll
      for (int j = 0; j < M; ++j) {
        if (j < kk && ranks_before(cv, ci, v[j], id[j])) {
          const float tv = v[j];
          const int ti = id[j];
          v[j] = cv;
          id[j] = ci;
          cv = tv;
          ci = ti;
        }
        if (j == kk - 1) {
          th_v = v[j];
          th_i = id[j];
        }
      }
    }
    // k + 1 rounds: the last one finds the best float32 logit left out
    float sel_v[BFMOE_MAX_K];
    int sel_i[BFMOE_MAX_K];
    float rej = -INFINITY;
#pragma unroll
    for (int j = 0; j < M; ++j) {
      if (j > k) break;
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
      if (j == k) {
        rej = bv;
        break;
      }
      sel_v[j] = bv;
      sel_i[j] = bi;
      if (id[0] == bi) {  // the owner pops its head
#pragma unroll
        for (int q = 0; q + 1 < M; ++q) {
          v[q] = v[q + 1];
          id[q] = id[q + 1];
        }
        v[M - 1] = -INFINITY;
        id[M - 1] = 0x7fffffff;
      }
    }
    float g[BFMOE_MAX_K];
    gates_f32(sel_v, k, g);
    if (lane == 0) {
      for (int j = 0; j < k; ++j) {
        idx[static_cast<size_t>(t) * k + j] = sel_i[j];
        gates[static_cast<size_t>(t) * k + j] = g[j];
      }
      if (!topk_is_clear(sel_v, k, rej, eps_c)) unsure_list[2 + atomicAdd(unsure_list, 1)] = t;
    }
  }
}

// The undecided tokens (unsure_list: [0] count, [2 ..] token ids), a warp
// per token, from the float32 logits the router stored ([T][N]) and its
// provisional float32 top-k (idx):
//   1. the float32 k-th logit V; the true top-k lies among the experts whose
//      float32 logit is at least V - 2 eps (each of the k first has a true
//      logit >= V - eps); the window keeps those at V - 4 eps or above (all N
//      experts if more than kFixWindow qualify);
//   2. the window's logits as double-float32 sums (exact products,
//      compensated sums: error ~1e-13 relative), lanes across d;
//   3. the exact top-k (lower index first on equal logits), gates from the
//      exact differences, and the bucket-chunk histograms moved from the
//      provisional experts to the final ones (when the router wrote them
//      already: chunk_counts, else NULL).
constexpr int kFixWindow = 64;
constexpr int kFixWarps = 8;

// Settle token t from exact logits (steps 1-3 above), one warp: lr is its
// row of float32 logits, idx[t][k-1] its provisional k-th pick, win a
// per-warp buffer of kFixWindow ints.  Lane 0 writes idx and gates and, when
// cc is given, moves the token's rows in that bucket-chunk histogram from
// the provisional experts to the final ones.
template <typename Tx>
__device__ void settle_token(int t, const Tx* __restrict__ xr, const float* __restrict__ wg,
                             const float* __restrict__ bias, const float* lr, int d, int N, int k, float eps_c,
                             int* win, int lane, int32_t* idx, float* gates, int32_t* cc) {
  // 1. the float32 k-th logit V: the router's provisional k-th pick is the
  // float32 top-k's last entry; then the window
  const int ik = idx[static_cast<size_t>(t) * k + (k - 1)];
  float vk = ik >= 0 && ik < N ? lr[ik] : -INFINITY;
  if (isnan(vk)) vk = -INFINITY;
  const float thr = vk > -INFINITY ? vk - 4.f * eps_c * (1.f + fabsf(vk)) : -INFINITY;
  int nwin = 0;
#pragma unroll 4
  for (int e0 = 0; e0 < N; e0 += 32) {
    const int e = e0 + lane;
    float l = e < N ? lr[e] : -INFINITY;
    if (isnan(l)) l = -INFINITY;
    const bool in = e < N && l >= thr;
    const unsigned m = __ballot_sync(FULL_MASK, in);
    const int pos = nwin + __popc(m & ((1u << lane) - 1u));
    if (in && pos < kFixWindow) win[pos] = e;
    nwin += __popc(m);
  }
  __syncwarp();
  // 2. exact logits of the window (all experts when it overflows) and
  // 3. the exact top-k
  const bool all = nwin > kFixWindow;
  const int cnt = all ? N : nwin;
  float vh[BFMOE_MAX_K], vl[BFMOE_MAX_K];
  int id[BFMOE_MAX_K];
#pragma unroll
  for (int j = 0; j < BFMOE_MAX_K; ++j) {
    vh[j] = -INFINITY;
    vl[j] = 0.f;
    id[j] = 0x7fffffff;
  }
  for (int q0 = 0; q0 < cnt; q0 += 4) {
    int es[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) es[j] = q0 + j < cnt ? (all ? q0 + j : win[q0 + j]) : -1;
    float h4[4], l4[4];
    df_logits4(xr, wg, bias, d, es, lane, h4, l4);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (es[j] < 0) break;
      // every lane holds the same value: a uniform insertion
      float ch = h4[j], cl = l4[j];
      int ci = es[j];
#pragma unroll
      for (int r = 0; r < BFMOE_MAX_K; ++r) {
        if (r < k && df_ranks_before(ch, cl, ci, vh[r], vl[r], id[r])) {
          const float th = vh[r], tl = vl[r];
          const int ti = id[r];
          vh[r] = ch;
          vl[r] = cl;
          id[r] = ci;
          ch = th;
          cl = tl;
          ci = ti;
        }
      }
    }
  }
  if (lane == 0) {
    // gates from the exact differences l_j - l_0
    float z[BFMOE_MAX_K];
    float sum = 0.f;
    const bool finite_top = vh[0] > -INFINITY;
    for (int j = 0; j < k; ++j) {
      z[j] = finite_top ? expf(__fadd_rn(__fsub_rn(vh[j], vh[0]), __fsub_rn(vl[j], vl[0]))) : 1.f;
      sum += z[j];
    }
    for (int j = 0; j < k; ++j) {
      const size_t o = static_cast<size_t>(t) * k + j;
      if (cc) {
        const int old = idx[o];
        if (old >= 0 && old < N) atomicSub(cc + old, 1);
        if (id[j] >= 0 && id[j] < N) atomicAdd(cc + id[j], 1);
      }
      idx[o] = id[j];
      gates[o] = z[j] / sum;
    }
  }
  __syncwarp();
}

template <typename Tx>
__global__ __launch_bounds__(kFixWarps * 32) void router_fixup_kernel(
    const Tx* __restrict__ x, const float* __restrict__ wg, const float* __restrict__ bias,
    const float* __restrict__ logits, int T, int d, int N, int k, float eps_c, const int* __restrict__ unsure_list,
    int32_t* __restrict__ idx, float* __restrict__ gates, int32_t* __restrict__ chunk_counts) {
  pdl_wait();
  pdl_trigger();
  __shared__ int win_s[kFixWarps][kFixWindow];
  const int n = unsure_list[0];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int gw = blockIdx.x * kFixWarps + w, nwarps = gridDim.x * kFixWarps;
  for (int u = gw; u < n; u += nwarps) {
    const int t = unsure_list[2 + u];
    if (t < 0 || t >= T) {
      if (lane == 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(u));
      continue;
    }
    settle_token(t, x + static_cast<size_t>(t) * d, wg, bias, logits + static_cast<size_t>(t) * N, d, N, k, eps_c,
                 win_s[w], lane, idx, gates, chunk_counts ? chunk_counts + static_cast<size_t>(t / 128) * N : nullptr);
  }
}

}  // namespace bfmoe
