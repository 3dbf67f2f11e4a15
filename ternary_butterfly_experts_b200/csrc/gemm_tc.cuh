// Ternary GEMM on the 5th-generation tensor cores:
//   Z = alpha * X_rot . W_base^T        (X_rot [R][d] bf16, W_base [d][d])
// the step "ternary multiply with the shared base" of the ButterflyMoE
// inference (technical summary, 2.3).  Because W_base is shared by every
// expert, all R routed rows form one dense GEMM; no grouped GEMM is needed.
// The ternary weights are exact in bf16; the product accumulates in fp32.
//
// Persistent kernel, one CTA per SM, 128 x BN output tiles.  The tiles that
// would form a last, partial wave are cut into 128 x BN/2 halves, so that no
// CTA runs a whole tile more than the others; each tile walks its k-blocks
// from a different start, so that the CTAs do not read the same B tile from
// L2 at the same moment (each output is still one float32 sum of exact
// products, in an order fixed per tile).
//   warp 0 (one lane)  TMA producer: 128x64 A and BNx64 B tiles (128-byte
//                      swizzle) into a STAGES-deep shared-memory ring;
//   warp 1 (one lane)  MMA issuer: tcgen05.mma M=128 N=BN K=16 into one of two
//                      TMEM accumulators (2*BN columns);
//   warps 2..5         epilogue: TMEM -> registers -> alpha * acc rounded to
//                      bf16 -> a per-warp shared-memory transpose -> coalesced
//                      stores of Z; the accumulator is released as soon as it
//                      is read, so the next tile's MMAs overlap these stores.
#pragma once
#include "common.cuh"

namespace bfmoe {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;
constexpr int kGemmThreads = 192;

template <int BN, int STAGES>
struct GemmTcCfg {
  static constexpr uint32_t A_BYTES = kGemmBM * kGemmBK * 2;
  static constexpr uint32_t B_BYTES = BN * kGemmBK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t EPI_BYTES = 4 * 32 * 32 * 2;  // 4 warps x 32x32 bf16
  static constexpr uint32_t BAR_BYTES = (2 * STAGES + 4) * 8 + 8;
  static constexpr uint32_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
};

// Work item i of the kernel: a whole tile, or a half of one of the last
// tiles.
struct GemmItem {
  int m0, n0, n;  // rows m0.., columns n0 .. n0+n-1
  int rot;        // first k-block
};
template <int BN>
__device__ __forceinline__ GemmItem gemm_item(int i, int n_full, int n_tiles_n, int nk) {
  int t, half = -1;
  if (i < n_full) {
    t = i;
  } else {
    t = n_full + (i - n_full) / 2;
    half = (i - n_full) & 1;
  }
  GemmItem it;
  it.m0 = (t / n_tiles_n) * kGemmBM;
  it.n0 = (t % n_tiles_n) * BN + (half > 0 ? BN / 2 : 0);
  it.n = half >= 0 ? BN / 2 : BN;
  it.rot = t % nk;
  return it;
}

// Items: whole tiles up to the last full wave of the grid, then the rest in
// halves (when BN/2 is a valid MMA width).
__host__ __device__ inline void gemm_items(int n_tiles, int grid, int bn, int* n_full, int* n_items) {
  const int full = (bn >= 128) ? (n_tiles / grid) * grid : n_tiles;
  *n_full = full;
  *n_items = full + 2 * (n_tiles - full);
}

template <int BN, int STAGES>
__global__ __launch_bounds__(kGemmThreads, 1) void ternary_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                                                                          const __grid_constant__ CUtensorMap tmB,
                                                                          const __grid_constant__ CUtensorMap tmBh,
                                                                          __nv_bfloat16* __restrict__ Z, int R, int d,
                                                                          float alpha) {
  using Cfg = GemmTcCfg<BN, STAGES>;
  static_assert(2 * BN == 64 || 2 * BN == 128 || 2 * BN == 256 || 2 * BN == 512, "TMEM columns");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint32_t* epi = reinterpret_cast<uint32_t*>(smem + STAGES * Cfg::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE_BYTES + Cfg::EPI_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;  // [2]
  uint64_t* tempty = tfull + 2;      // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = d / kGemmBK;
  const int n_tiles_n = d / BN;
  const int n_tiles = ((R + kGemmBM - 1) / kGemmBM) * n_tiles_n;
  int n_full, n_items;
  gemm_items(n_tiles, gridDim.x, BN, &n_full, &n_items);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, 4);
    }
    mbar_fence_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmBh);
  }
  if (warp == 0) tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // X_rot comes from the previous kernel
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int i = blockIdx.x; i < n_items; i += gridDim.x) {
        const GemmItem w = gemm_item<BN>(i, n_full, n_tiles_n, nk);
        bool alive = true;
        for (int ki = 0; ki < nk; ++ki, ++it) {
          const int kb = (ki + w.rot) % nk;
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (it >= STAGES && !mbar_wait(empty + s, ph ^ 1u, 0x100u | s)) {
            alive = false;
            break;
          }
          const bool half = w.n < BN;
          mbar_expect_tx(full + s, Cfg::A_BYTES + (half ? Cfg::B_BYTES / 2 : Cfg::B_BYTES));
          uint8_t* a = smem + s * Cfg::STAGE_BYTES;
          tma_load_2d(a, &tmA, full + s, kb * kGemmBK, w.m0);
          tma_load_2d(a + Cfg::A_BYTES, half ? &tmBh : &tmB, full + s, kb * kGemmBK, w.n0);
        }
        if (!alive) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_full = idesc_bf16_f32(kGemmBM, BN);
      constexpr uint32_t idesc_half = idesc_bf16_f32(kGemmBM, BN >= 128 ? BN / 2 : BN);
      int it = 0, i = 0;
      bool alive = true;
      for (int wi = blockIdx.x; wi < n_items && alive; wi += gridDim.x, ++i) {
        const uint32_t idesc = wi < n_full ? idesc_full : idesc_half;
        const int buf = i & 1;
        if (i >= 2 && !mbar_wait(tempty + buf, ((i >> 1) - 1) & 1u, 0x300u | buf)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(buf * BN);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(full + s, ph, 0x200u | s)) {
            alive = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint64_t ad = desc_kmajor_sw128(a);
          const uint64_t bd = desc_kmajor_sw128(a + Cfg::A_BYTES);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk)
            mma_bf16_ss(d_tmem, ad + 2u * kk, bd + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          mma_commit(empty + s);
        }
        mma_commit(tfull + buf);
      }
    }
  } else {
    // epilogue warps 2..5: TMEM sub-partition (warp % 4) holds rows 32*(warp%4) ..
    const int sp = warp & 3;
    uint32_t* buf_w = epi + (warp - 2) * 32 * 16;  // 32 rows x 16 bf16 pairs
    int i = 0;
    for (int wi = blockIdx.x; wi < n_items; wi += gridDim.x, ++i) {
      const GemmItem w = gemm_item<BN>(wi, n_full, n_tiles_n, nk);
      const int m0 = w.m0, n0 = w.n0;
      const int buf = i & 1;
      if (!mbar_wait(tfull + buf, (i >> 1) & 1u, 0x400u | buf)) break;
      tc_fence_after();
      const uint32_t base = tmem + (static_cast<uint32_t>(sp * 32) << 16) + static_cast<uint32_t>(buf * BN);
      const int row0 = m0 + sp * 32;
#pragma unroll 1
      for (int c = 0; c < w.n; c += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(base + static_cast<uint32_t>(c), v);
        tmem_wait_ld();
        if (c + 32 >= w.n) {
          // whole accumulator read: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty + buf);
        }
        // lane = row: 16 bf16 pairs as 4 x 16 bytes, swizzled by row ...
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          __nv_bfloat162 h = __floats2bfloat162_rn(alpha * __uint_as_float(v[2 * j]), alpha * __uint_as_float(v[2 * j + 1]));
          pk[j] = *reinterpret_cast<uint32_t*>(&h);
        }
        const int sw = (lane >> 1) & 3;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<uint4*>(buf_w + lane * 16 + ((u ^ sw) << 2)) =
              make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        __syncwarp();
        // ... then 8 rows x 64 bytes per store instruction
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int rr = q * 8 + (lane >> 2), u = lane & 3;
          const uint4 val = *reinterpret_cast<const uint4*>(buf_w + rr * 16 + ((u ^ ((rr >> 1) & 3)) << 2));
          const int row = row0 + rr;
          if (row < R) *reinterpret_cast<uint4*>(Z + static_cast<size_t>(row) * d + n0 + c + 8 * u) = val;
        }
        __syncwarp();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

}  // namespace bfmoe
