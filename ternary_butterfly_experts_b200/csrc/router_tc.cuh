// Router on the tensor cores, with top-k and gates fused into the epilogue.
//
// logits = x W_g^T + b with x in bfloat16 and W_g in float32.  W_g is split
// exactly into three bfloat16 parts, w = hi + mid + lo (each part holds the
// next 8 significant bits; the remainders are exact in float32), so the
// logits are three bf16 x bf16 products with exact terms, accumulated in
// float32 in tensor memory: the same sum as a float32 dot product, in another
// order.
//
// One CTA owns 128 tokens and walks the experts in chunks of BN columns.
// Warp 0 (one lane) loads with TMA the 128x64 token tile and the three BNx64
// weight tiles per 64-wide slice of d; warp 1 (one lane) issues the MMAs into
// one of two TMEM accumulators; warps 2..9 read the logits from TMEM (warp w
// owns TMEM lanes 32*(w%4) .., warps w and w+4 take the two halves of each
// chunk's columns), each keeping a running top-k of its half (larger logit
// first, lower expert index on ties, NaN below every number), and the largest
// logit it left out, while the next chunk is being multiplied; the two partial
// lists of a row are merged through shared memory, and the row's idx and
// renormalised gates are written.  A row whose selected logits are not
// separated from each other and from the best one left out by more than the
// float32 error band (topk_is_clear, router.cuh) is listed for
// router_fixup_kernel.  The CTA's 128*k routed rows form one bucket
// chunk: the epilogue also writes their expert histogram
// (chunk_counts[blockIdx.x][e]).
#pragma once
#include "common.cuh"
#include "gemm_tc.cuh"
#include "router.cuh"

namespace bfmoe {

// w [N][d] float32 -> parts [3][N][d] bfloat16 with hi + mid + lo == w.
__global__ void router_split_kernel(const float* __restrict__ w, long long n, __nv_bfloat16* __restrict__ parts) {
  pdl_wait();
  pdl_trigger();
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float v = w[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    parts[i] = hi;
    parts[n + i] = mid;
    parts[2 * n + i] = __float2bfloat16_rn(r2);
  }
}

template <int BN, int STAGES>
struct RouterTcCfg {
  static constexpr uint32_t A_BYTES = kGemmBM * kGemmBK * 2;
  static constexpr uint32_t B_BYTES = BN * kGemmBK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + 3 * B_BYTES;
  static constexpr uint32_t BAR_BYTES = (2 * STAGES + 4) * 8 + 8;
  static constexpr uint32_t BIAS_BYTES = BFMOE_MAX_EXPERTS * 4;             // bias staged once
  static constexpr uint32_t MERGE_BYTES = kGemmBM * BFMOE_MAX_K * 8 + kGemmBM * 4;  // top-k lists, rejected maxima
  static constexpr uint32_t WIN_BYTES = 4 * kFixWindow * 4;  // the settling warps' expert windows
  static constexpr uint32_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + BIAS_BYTES + MERGE_BYTES + WIN_BYTES;
  static constexpr uint32_t TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64 ? 64 : (2 * BN <= 128 ? 128 : 256));
};

constexpr int kRouterThreads = 320;
constexpr int kRouterEpiWarps = 8;

// Running top-K of one row in registers (K compile-time): larger logit first,
// lower expert index first on equal logits; `rej` is the largest logit that
// is not (or no longer) in the list.
template <int K>
struct TopK {
  float v[K];
  int id[K];
  float rej;
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j < K; ++j) {
      v[j] = -INFINITY;
      id[j] = 0x7fffffff;
    }
    rej = -INFINITY;
  }
  // Small K: the K compare-and-select steps run for every column, with no
  // branch (the lanes of a warp hold different rows, so an early exit would
  // diverge on most columns); larger K exits first when l cannot enter.
  __device__ __forceinline__ void push(float l, int e) {
    if (K > 4 && !ranks_before(l, e, v[K - 1], id[K - 1])) {
      rej = fmaxf(rej, l);
      return;
    }
    float cv = l;
    int ci = e;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      const bool sw = ranks_before(cv, ci, v[j], id[j]);
      const float tv = v[j];
      const int ti = id[j];
      v[j] = sw ? cv : tv;
      id[j] = sw ? ci : ti;
      cv = sw ? tv : cv;
      ci = sw ? ti : ci;
    }
    rej = fmaxf(rej, cv);  // what fell out of the list
  }
};

template <int BN, int STAGES, int K>
__global__ __launch_bounds__(kRouterThreads, 1) void router_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                                                           const __grid_constant__ CUtensorMap tmW,
                                                           const float* __restrict__ bias, int T, int d, int N,
                                                           float eps_c, float* __restrict__ logits,
                                                           const __nv_bfloat16* __restrict__ x,
                                                           const float* __restrict__ w_gate,
                                                           int32_t* __restrict__ idx,
                                                           float* __restrict__ gates,
                                                           int32_t* __restrict__ chunk_counts) {
  using Cfg = RouterTcCfg<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  float* bias_s = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + Cfg::BAR_BYTES);
  float* merge_v = bias_s + BFMOE_MAX_EXPERTS;                       // [128][K]
  int* merge_i = reinterpret_cast<int*>(merge_v + kGemmBM * BFMOE_MAX_K);  // [128][K]
  float* merge_r = reinterpret_cast<float*>(merge_i + kGemmBM * BFMOE_MAX_K);  // [128]
  int* win_s = reinterpret_cast<int*>(merge_r + kGemmBM);                      // [4][kFixWindow]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kGemmBM;
  const int nk = d / kGemmBK;
  const int nchunks = (N + BN - 1) / BN;
  // CTAs start at different k-blocks and expert chunks, so that they do not
  // all read the same weight tile from L2 at the same moment.  Each logit is
  // still one float32 sum of exact products, in an order fixed per CTA.
  const int k_rot = blockIdx.x % nk;
  const int c_rot = (blockIdx.x / nk) % nchunks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, kRouterEpiWarps);  // one arrival per epilogue warp
    }
    mbar_fence_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 0) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
  for (int e = threadIdx.x; e < N; e += blockDim.x) bias_s[e] = bias ? bias[e] : 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // the split weights come from the previous kernel
  pdl_trigger();

  if (warp == 0 && lane == 0) {
    int it = 0;
    bool alive = true;
    for (int ci = 0; ci < nchunks && alive; ++ci) {
      const int c = (ci + c_rot) % nchunks;
      for (int ki = 0; ki < nk; ++ki, ++it) {
        const int kb = (ki + k_rot) % nk;
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        if (it >= STAGES && !mbar_wait(empty + s, ph ^ 1u, 0x1100u | s)) {
          alive = false;
          break;
        }
        mbar_expect_tx(full + s, Cfg::STAGE_BYTES);
        uint8_t* a = smem + s * Cfg::STAGE_BYTES;
        tma_load_2d(a, &tmX, full + s, kb * kGemmBK, m0);
#pragma unroll
        for (int p = 0; p < 3; ++p)
          tma_load_2d(a + Cfg::A_BYTES + p * Cfg::B_BYTES, &tmW, full + s, kb * kGemmBK, p * N + c * BN);
      }
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(kGemmBM, BN);
    int it = 0;
    bool alive = true;
    for (int c = 0; c < nchunks && alive; ++c) {
      const int buf = c & 1;
      if (c >= 2 && !mbar_wait(acc_empty + buf, ((c >> 1) - 1) & 1u, 0x1300u | buf)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + static_cast<uint32_t>(buf * BN);
      for (int kb = 0; kb < nk; ++kb, ++it) {  // kb counts k-blocks in arrival order
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        if (!mbar_wait(full + s, ph, 0x1200u | s)) {
          alive = false;
          break;
        }
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * Cfg::STAGE_BYTES);
        const uint64_t ad = desc_kmajor_sw128(a);
#pragma unroll
        for (int p = 0; p < 3; ++p) {
          const uint64_t bd = desc_kmajor_sw128(a + Cfg::A_BYTES + p * Cfg::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk)
            mma_bf16_ss(d_tmem, ad + 2u * kk, bd + 2u * kk, idesc, (kb | kk | p) != 0 ? 1u : 0u);
        }
        mma_commit(empty + s);
      }
      mma_commit(acc_full + buf);
    }
  }
  if (warp < 2) {
    // producer and MMA warps take no part in the epilogue
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, Cfg::TMEM_COLS);
    return;
  }

  // Epilogue (warps 2..9): one token row per thread, half of each chunk.
  const int sp = warp & 3;
  const int hf = (warp - 2) >> 2;  // which half of the chunk's columns
  const int lr = sp * 32 + lane;   // row within the tile
  const int row = m0 + lr;
  constexpr int HALF = BN >= 64 ? BN / 2 : BN;  // columns per warp and chunk
  TopK<K> top;
  top.init();
  bool ok = true;
  for (int ci = 0; ci < nchunks; ++ci) {
    const int c = (ci + c_rot) % nchunks;
    const int buf = ci & 1;
    if (!mbar_wait(acc_full + buf, (ci >> 1) & 1u, 0x1400u | buf)) {
      ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t base = tmem + (static_cast<uint32_t>(sp * 32) << 16) + static_cast<uint32_t>(buf * BN);
    if (BN >= 64 || hf == 0) {
#pragma unroll 1
      for (int col = hf * HALF; col < hf * HALF + HALF; col += 32) {
        const int e0 = c * BN + col;
        uint32_t r[32];
        tmem_ld_32x32b_x32(base + static_cast<uint32_t>(col), r);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const int e = e0 + q;
          float l = e < N ? __uint_as_float(r[q]) + bias_s[e] : -INFINITY;
          if (isnan(l)) l = -INFINITY;
          r[q] = __float_as_uint(l);
          top.push(l, e < N ? e : 0x7fffffff);
        }
        // the float32 logits are kept for the fix-up of undecided tokens
        if (row < T) {
          float* dst = logits + static_cast<size_t>(row) * N + e0;
          if ((N & 7) == 0 && e0 + 32 <= N) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + 8 * u),
                           "r"(r[8 * u]), "r"(r[8 * u + 1]), "r"(r[8 * u + 2]), "r"(r[8 * u + 3]), "r"(r[8 * u + 4]),
                           "r"(r[8 * u + 5]), "r"(r[8 * u + 6]), "r"(r[8 * u + 7])
                           : "memory");
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q)
              if (e0 + q < N) dst[q] = __uint_as_float(r[q]);
          }
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acc_empty + buf);
  }
  // merge the two halves of each row
  if (hf == 1) {
#pragma unroll
    for (int j = 0; j < K; ++j) {
      merge_v[lr * BFMOE_MAX_K + j] = top.v[j];
      merge_i[lr * BFMOE_MAX_K + j] = top.id[j];
    }
    merge_r[lr] = top.rej;
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kRouterEpiWarps * 32) : "memory");
  // the bias is no longer read from shared memory: it becomes the histogram
  int* hist = reinterpret_cast<int*>(bias_s);
  const int et = threadIdx.x - 64;  // 0 .. 255
  for (int e = et; e < N; e += kRouterEpiWarps * 32) hist[e] = 0;
  asm volatile("bar.sync 1, %0;" ::"r"(kRouterEpiWarps * 32) : "memory");
  bool unsure = false;
  if (hf == 0 && ok && row < T) {
#pragma unroll
    for (int j = 0; j < K; ++j) top.push(merge_v[lr * BFMOE_MAX_K + j], merge_i[lr * BFMOE_MAX_K + j]);
    top.rej = fmaxf(top.rej, merge_r[lr]);
    float g[BFMOE_MAX_K];
    gates_f32(top.v, K, g);
#pragma unroll
    for (int j = 0; j < K; ++j) {
      idx[static_cast<size_t>(row) * K + j] = top.id[j];
      gates[static_cast<size_t>(row) * K + j] = g[j];
      if (top.id[j] < N) atomicAdd(&hist[top.id[j]], 1);
    }
    unsure = !topk_is_clear(top.v, K, top.rej, eps_c);
  }
  if (hf == 0) {
    // rows whose float32 top-k is undecided (a few per thousand) are settled
    // here from exact logits, the warp working on one row at a time; the
    // row's float32 logits were stored above and are visible to the warp
    __syncwarp();
    unsigned um = __ballot_sync(FULL_MASK, unsure);
    while (um) {
      const int src = __ffs(um) - 1;
      um &= um - 1;
      const int t = m0 + sp * 32 + src;
      settle_token(t, x + static_cast<size_t>(t) * d, w_gate, bias, logits + static_cast<size_t>(t) * N, d, N, K,
                   eps_c, win_s + sp * kFixWindow, lane, idx, gates, hist);
    }
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kRouterEpiWarps * 32) : "memory");
  for (int e = et; e < N; e += kRouterEpiWarps * 32)
    chunk_counts[static_cast<size_t>(blockIdx.x) * N + e] = hist[e];
  tc_fence_before();
  __syncthreads();
}

}  // namespace bfmoe
