// Token-to-expert buckets: a stable counting sort of the routed rows
// r = t*k + j by expert.  Within an expert, rows come in ascending r, which is
// ascending token order because a token's k experts are distinct.
//
// Rows are cut into chunks of 128*k rows, the routed rows of 128 tokens (one
// block of 128*k threads each):
//   count    per-chunk expert histogram (the tensor-core router writes it from
//            its epilogue; this kernel serves the float32 router)
//   scan     per expert, exclusive prefix over chunks (+ totals)
//   scatter  offsets = exclusive prefix over experts (each block); position =
//            offsets[e] + chunk prefix + earlier warps of the chunk + rank
//            among equal experts inside the warp
#pragma once
#include "common.cuh"

namespace bfmoe {

// Routed rows per bucket chunk: those of 128 tokens (k <= 8, so <= 1024).
__host__ __device__ constexpr int bucket_chunk(int k) { return 128 * k; }

__global__ __launch_bounds__(1024) void bucket_count_kernel(const int32_t* __restrict__ idx, long long R, int N,
                                                            int32_t* __restrict__ chunk_counts) {
  extern __shared__ int cnt[];
  for (int e = threadIdx.x; e < N; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const long long r = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r < R) {
    const int e = idx[r];
    if (e >= 0 && e < N) {
      atomicAdd(&cnt[e], 1);
    } else {
      report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(r));
    }
  }
  __syncthreads();
  int32_t* dst = chunk_counts + static_cast<size_t>(blockIdx.x) * N;
  for (int e = threadIdx.x; e < N; e += blockDim.x) dst[e] = cnt[e];
}

// Block of 32 experts (x) by 32 chunk slices (y).  Rewrites chunk_counts
// into exclusive prefixes over chunks; totals[e] = rows of expert e.
__global__ __launch_bounds__(1024) void bucket_scan_kernel(int32_t* __restrict__ chunk_counts, int nchunks, int N,
                                                           int32_t* __restrict__ totals) {
  __shared__ int part[32][33];
  pdl_wait();
  pdl_trigger();
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + tx;
  const int per = (nchunks + 31) / 32;
  const int c0 = min(ty * per, nchunks), c1 = min(c0 + per, nchunks);
  int s = 0;
  if (e < N)
    for (int c = c0; c < c1; ++c) s += chunk_counts[static_cast<size_t>(c) * N + e];
  part[ty][tx] = s;
  __syncthreads();
  if (ty == 0) {
    int run = 0;
    for (int q = 0; q < 32; ++q) {
      const int tmp = part[q][tx];
      part[q][tx] = run;
      run += tmp;
    }
    if (e < N) totals[e] = run;
  }
  __syncthreads();
  int run = part[ty][tx];
  if (e < N)
    for (int c = c0; c < c1; ++c) {
      const size_t a = static_cast<size_t>(c) * N + e;
      const int tmp = chunk_counts[a];
      chunk_counts[a] = run;
      run += tmp;
    }
}

// Exclusive prefix sum of val(0..N) into off[0..N] (shared memory), by a
// block of any multiple of 32 threads up to 1024; thread i sums experts
// i*per .. i*per + per - 1.
template <class F>
__device__ __forceinline__ void block_exclusive_scan(F val, int N, int* off) {
  __shared__ int warp_sum[32];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nw = blockDim.x >> 5;
  const int per = (N + blockDim.x - 1) / blockDim.x;
  int local = 0;
  for (int q = 0; q < per; ++q) {
    const int e = tid * per + q;
    local += e < N ? val(e) : 0;
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(FULL_MASK, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_sum[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int ws = lane < nw ? warp_sum[lane] : 0;
    int inc = ws;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(FULL_MASK, inc, o);
      if (lane >= o) inc += t;
    }
    warp_sum[lane] = inc - ws;
  }
  __syncthreads();
  int run = warp_sum[w] + incl - local;
  for (int q = 0; q < per; ++q) {
    const int e = tid * per + q;
    if (e < N) {
      off[e] = run;
      run += val(e);
    }
  }
  if (tid == static_cast<int>(blockDim.x) - 1) off[N] = run;
  __syncthreads();
}

// Every block scans the per-expert totals itself (N <= 4096 ints), so the
// offsets need no launch of their own; block 0 also writes counts and
// offsets out; block b reads its chunk's prefixes from chunk_prefix
// (bucket_scan_kernel).  With pad given ([N+1] padded offsets, then [p_cap]
// row map, then [p_cap / 32] quadrant experts), the blocks also write the
// padded bucket order that bucket_pad_kernel would build from the buckets.
__global__ __launch_bounds__(1024) void bucket_scatter_kernel(const int32_t* __restrict__ idx, long long R, int N,
                                                              const int32_t* __restrict__ chunk_prefix,
                                                              const int32_t* __restrict__ totals,
                                                              int32_t* __restrict__ counts_out,
                                                              int32_t* __restrict__ offsets_out,
                                                              int32_t* __restrict__ rows, int32_t* __restrict__ pad,
                                                              long long p_cap) {
  extern __shared__ uint8_t scatter_smem[];
  int* off = reinterpret_cast<int*>(scatter_smem);                   // [N+1]
  uint8_t* wcnt = scatter_smem + ((N + 1) * 4 + 15) / 16 * 16;       // [N][32]: rows of expert e in warp w
  int* poff = reinterpret_cast<int*>(wcnt + static_cast<size_t>(N) * 32);  // [N+1] (padded order only)
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int q = tid; q < N * 8; q += blockDim.x) reinterpret_cast<uint32_t*>(wcnt)[q] = 0u;
  pdl_wait();
  pdl_trigger();
  block_exclusive_scan([&](int e) { return totals[e]; }, N, off);
  int32_t* pmap = nullptr;
  if (pad) {
    // the padded order: every bucket rounded up to 32 rows; this block fills
    // the padding and quadrant experts of experts b, b + gridDim.x, ... and
    // its share of the tail up to p_cap
    block_exclusive_scan([&](int e) { return (off[e + 1] - off[e] + 31) & ~31; }, N, poff);
    pmap = pad + (N + 1);
    int32_t* qex = pmap + p_cap;
    if (blockIdx.x == 0)
      for (int e = tid; e <= N; e += blockDim.x) pad[e] = poff[e];
    for (int e = blockIdx.x; e < N; e += gridDim.x) {
      const int p0 = poff[e], c = off[e + 1] - off[e], p1 = poff[e + 1];
      for (int q = tid; q < p1 - p0 - c; q += blockDim.x) pmap[p0 + c + q] = -1;
      for (int q = tid; q < (p1 - p0) / 32; q += blockDim.x) qex[p0 / 32 + q] = e;
    }
    for (long long P = poff[N] + static_cast<long long>(blockIdx.x) * blockDim.x + tid; P < p_cap;
         P += static_cast<long long>(gridDim.x) * blockDim.x) {
      pmap[P] = -1;
      if ((P & 31) == 0) qex[P >> 5] = -1;
    }
  }
  if (blockIdx.x == 0) {
    for (int e = tid; e <= N; e += blockDim.x) {
      offsets_out[e] = off[e];
      if (e < N) counts_out[e] = off[e + 1] - off[e];
    }
  }
  const long long r = static_cast<long long>(blockIdx.x) * blockDim.x + tid;
  int e = -1 - lane;
  bool valid = false;
  if (r < R) {
    const int v = idx[r];
    if (v >= 0 && v < N) {
      e = v;
      valid = true;
    }
  }
  const unsigned peers = __match_any_sync(FULL_MASK, e);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (valid && rank == 0) wcnt[e * 32 + w] = static_cast<uint8_t>(__popc(peers));
  __syncthreads();
  int before = 0;
  if (valid && rank == 0)
    for (int q = 0; q < w; ++q) before += wcnt[e * 32 + q];
  const int leader = __ffs(peers) - 1;
  before = __shfl_sync(FULL_MASK, before, leader);
  if (valid) {
    const int pos = off[e] + chunk_prefix[static_cast<size_t>(blockIdx.x) * N + e] + before + rank;
    rows[pos] = static_cast<int32_t>(r);
    if (pmap) pmap[poff[e] + (pos - off[e])] = static_cast<int32_t>(r);
  }
}

// The buckets padded to whole multiples of 32 rows, as a map from padded
// position to routed row.  pad_off[e] = sum over e' < e of
// ceil32(offsets[e'+1] - offsets[e']); pad_off[N] is the padded row count.
// Padded position P in expert e's segment [pad_off[e], pad_off[e+1]) holds
// bucket position offsets[e] + P - pad_off[e] when that is below the
// bucket's end: pmap[P] is then its routed row (checked against idx), else
// -1; qex[P / 32] is the expert of the 32 rows from P (-1 past the last
// segment).  Every block scans the padded sizes itself (N <= 4096); the map
// covers [0, p_cap), p_cap a multiple of 32 at least pad_off[N].  The fused
// expert kernel walks this order, so that no warp's 32 rows mix experts.
__global__ __launch_bounds__(256) void bucket_pad_kernel(const int32_t* __restrict__ offsets,
                                                         const int32_t* __restrict__ rows,
                                                         const int32_t* __restrict__ idx, long long R, int N,
                                                         long long p_cap, int32_t* __restrict__ pad_off,
                                                         int32_t* __restrict__ pmap, int32_t* __restrict__ qex) {
  extern __shared__ int poff[];  // [N+1] padded offsets, then [N+1] offsets
  int* off = poff + (N + 1);
  pdl_wait();
  pdl_trigger();
  for (int e = threadIdx.x; e <= N; e += blockDim.x) off[e] = offsets[e];
  __syncthreads();
  block_exclusive_scan([&](int e) { return (off[e + 1] - off[e] + 31) & ~31; }, N, poff);
  if (blockIdx.x == 0)
    for (int e = threadIdx.x; e <= N; e += blockDim.x) pad_off[e] = poff[e];
  const long long total = poff[N];
  for (long long P = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; P < p_cap;
       P += static_cast<long long>(gridDim.x) * blockDim.x) {
    int e = -1, row = -1;
    if (P < total) {
      int lo = 0, hi = N - 1;  // the last e with poff[e] <= P
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (poff[mid] <= P) lo = mid;
        else hi = mid - 1;
      }
      e = lo;
      const long long b = off[e] + (P - poff[e]);
      if (b < off[e + 1]) {
        const int r = b >= 0 && b < R ? rows[b] : -1;
        if (r >= 0 && r < R && idx[r] == e) row = r;
        else report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(b));
      }
    }
    pmap[P] = row;
    if ((P & 31) == 0) qex[P >> 5] = e;
  }
}

}  // namespace bfmoe
