// 2-bit storage of the shared ternary base, and its exact bf16 expansion.
//
// The shared base W_base in {-1, 0, +1}^{d x d} is stored at 2 bits per weight
// (the ButterflyMoE technical summary, section 2.1, quotes log2 3 = 1.58
// bits): 0 -> 00, +1 -> 01, -1 -> 11, sixteen codes per uint32, row-major,
// column i of a word at bits 2*(i mod 16).
#pragma once
#include "common.cuh"

namespace bfmoe {

// One thread per output word.
__global__ void pack_base_kernel(const int8_t* __restrict__ w, int d, int wpr, uint32_t* __restrict__ out) {
  const long long n = static_cast<long long>(d) * wpr;
  for (long long q = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; q < n;
       q += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int o = static_cast<int>(q / wpr);
    const int wi = static_cast<int>(q % wpr);
    uint32_t word = 0;
    bool bad = false;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const int i = wi * 16 + m;
      if (i < d) {
        const int v = w[static_cast<size_t>(o) * d + i];
        uint32_t code = 0;
        if (v == 1) {
          code = 1u;
        } else if (v == -1) {
          code = 3u;
        } else if (v != 0) {
          bad = true;
        }
        word |= code << (2 * m);
      }
    }
    if (bad) atomicOr(&g_not_ternary, 1u);
    out[q] = word;
  }
}

// One thread per packed word: writes its (up to) 16 bf16 weights.
__global__ void expand_base_bf16_kernel(const uint32_t* __restrict__ packed, int d, int wpr,
                                        uint16_t* __restrict__ out) {
  const long long n = static_cast<long long>(d) * wpr;
  for (long long q = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; q < n;
       q += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int o = static_cast<int>(q / wpr);
    const int wi = static_cast<int>(q % wpr);
    const uint32_t word = packed[q];
    uint16_t* dst = out + static_cast<size_t>(o) * d + wi * 16;
    if (d >= 16) {
      uint32_t pr[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const uint32_t lo = ternary_code_bf16((word >> (4 * m)) & 3u);
        const uint32_t hi = ternary_code_bf16((word >> (4 * m + 2)) & 3u);
        pr[m] = lo | (hi << 16);
      }
      uint4* d4 = reinterpret_cast<uint4*>(dst);
      d4[0] = make_uint4(pr[0], pr[1], pr[2], pr[3]);
      d4[1] = make_uint4(pr[4], pr[5], pr[6], pr[7]);
    } else {
      for (int m = 0; m < d; ++m) dst[m] = ternary_code_bf16((word >> (2 * m)) & 3u);
    }
  }
}

}  // namespace bfmoe
