// Ternary GEMM on the 5th-generation tensor cores:
//   Z = alpha * X_rot . W_base^T        (X_rot [R][d] bf16, W_base [d][d])
// the step "ternary multiply with the shared base" of the ButterflyMoE
// inference (technical summary, 2.3).  Because W_base is shared by every
// expert, all R routed rows form one dense GEMM; no grouped GEMM is needed.
// The ternary weights are exact in bf16, the product accumulates in fp32.
//
// Per CTA: one 128 x BN output tile.  Warp 0 (one lane) streams 128x64 A and
// BNx64 B tiles with TMA (128-byte swizzle) into a STAGES-deep ring; warp 1
// (one lane) issues tcgen05.mma (M=128, N=BN, K=16) into a TMEM accumulator;
// all four warps then drain TMEM (warp w owns lanes 32w..32w+31 = rows) and
// store alpha * acc.
#pragma once
#include "common.cuh"

namespace bfmoe {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;

template <int BN, int STAGES>
struct GemmTcCfg {
  static constexpr uint32_t A_BYTES = kGemmBM * kGemmBK * 2;
  static constexpr uint32_t B_BYTES = BN * kGemmBK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t BAR_BYTES = (2 * STAGES + 1) * 8 + 8;
  static constexpr uint32_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
};

template <int BN, int STAGES>
__global__ __launch_bounds__(128, 1) void ternary_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                                                                 const __grid_constant__ CUtensorMap tmB,
                                                                 float* __restrict__ Z, int R, int d, float alpha) {
  using Cfg = GemmTcCfg<BN, STAGES>;
  static_assert(BN == 32 || BN == 64 || BN == 128 || BN == 256, "TMEM columns must be a power of two >= 32");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accb = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accb + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kGemmBM, n0 = blockIdx.y * BN;
  const int nk = d / kGemmBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(accb, 1);
    mbar_fence_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 0) tmem_alloc(tmem_slot, BN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // TMA producer
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1u;
      if (kb >= STAGES && !mbar_wait(empty + s, ph ^ 1u, 0x100u | s)) break;
      mbar_expect_tx(full + s, Cfg::STAGE_BYTES);
      uint8_t* a = smem + s * Cfg::STAGE_BYTES;
      tma_load_2d(a, &tmA, full + s, kb * kGemmBK, m0);
      tma_load_2d(a + Cfg::A_BYTES, &tmB, full + s, kb * kGemmBK, n0);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(kGemmBM, BN);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1u;
      if (!mbar_wait(full + s, ph, 0x200u | s)) break;
      tc_fence_after();
      const uint32_t a = smem_u32(smem + s * Cfg::STAGE_BYTES);
      const uint64_t ad = desc_kmajor_sw128(a);
      const uint64_t bd = desc_kmajor_sw128(a + Cfg::A_BYTES);
#pragma unroll
      for (int kk = 0; kk < kGemmBK / 16; ++kk) {
        // +32 bytes along K inside the 128-byte swizzle atom = +2 in the
        // descriptor's 16-byte address units.
        mma_bf16_ss(tmem, ad + 2u * kk, bd + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
      }
      mma_commit(empty + s);
    }
    mma_commit(accb);
  }
  __syncwarp();

  // Epilogue: TMEM -> registers -> global.
  const bool ok = mbar_wait(accb, 0, 0x300u);
  tc_fence_after();
  const int row = m0 + warp * 32 + lane;
  if (ok) {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c), v);
      tmem_wait_ld();
      if (row < R) {
        float4* dst = reinterpret_cast<float4*>(Z + static_cast<size_t>(row) * d + n0 + c);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = make_float4(alpha * __uint_as_float(v[4 * q]), alpha * __uint_as_float(v[4 * q + 1]),
                               alpha * __uint_as_float(v[4 * q + 2]), alpha * __uint_as_float(v[4 * q + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, BN);
}

}  // namespace bfmoe
