// Add-only expert forward for small batches (decode).
//
// The ternary product of each expert needs no multiplications: with the base
// stored as 2-bit codes (0, +1, -1), z_o = alpha * sum_i W_base[o][i] u_i is a
// signed sum of the rotated inputs u (ButterflyMoE technical summary on
// gist.science, 2.3 step 2 and 3: the base multiply reduces to additions and
// subtractions).  One CTA takes one token; its k slot rows (up to 8 at a
// time) go through each step together, in float32 throughout:
//   u = B(theta_e)^T x_t           stages L-1 .. 0, transposed blocks
//   z = alpha * (W_base u)         2-bit codes decoded in registers; each
//                                  code adds u_i, subtracts it or skips it
//                                  (one load of a code word serves every row)
//   v = B(phi_e) z                 stages 0 .. L-1
//   y_t += g_j v                   float32, j ascending; one rounding of y
// The rows live in shared memory; a stage's rotations of all rows are spread
// over the threads, one barrier per stage; cos and sin come from the float32
// angles through sincosf.  Nothing here depends on T being small, but a token
// costs one CTA and k d^2 code decodes, which suits decode batches (T up to
// a few hundred); larger batches belong to the tensor-core forward.
#pragma once
#include "common.cuh"

namespace bfmoe {

constexpr int kDecodeThreads = 512;
constexpr int kDecodeRows = 8;                                  // slots of a token handled together
constexpr int kDecodeOut = BFMOE_MAX_D / kDecodeThreads;        // outputs per thread, at most

// Slots of a token processed together: 2 kc d floats of shared memory.
__host__ __device__ inline int decode_rows(int d, int k) {
  int kc = 16384 / d;
  if (kc < 1) kc = 1;
  if (kc > kDecodeRows) kc = kDecodeRows;
  return kc < k ? kc : k;
}

// One stage of rotations on nj shared-memory rows v[jj * d ..] with angles
// ang[jj] (stage s of row jj's expert; NULL: the row is skipped).  Stage s
// pairs (i, i + 2^s) for every i with bit s clear, rotation index r = i with
// bit s removed; forward block [[c, -s], [s, c]], transposed [[c, s], [-s, c]].
template <bool TR>
__device__ __forceinline__ void decode_stage(float* v, const float* const* ang, int nj, int d, int s) {
  const int h = 1 << s, half = d / 2;
  for (int q = threadIdx.x; q < nj * half; q += blockDim.x) {
    const int jj = q / half, r = q - jj * half;
    if (!ang[jj]) continue;
    const int i = ((r >> s) << (s + 1)) | (r & (h - 1));
    const int j = i + h;
    float sn, cs;
    sincosf(ang[jj][static_cast<size_t>(s) * half + r], &sn, &cs);
    float* w = v + static_cast<size_t>(jj) * d;
    const float a = w[i], b = w[j];
    if (TR) {
      w[i] = cs * a + sn * b;
      w[j] = cs * b - sn * a;
    } else {
      w[i] = cs * a - sn * b;
      w[j] = sn * a + cs * b;
    }
  }
  __syncthreads();
}

// z[j][o] = alpha * sum_i W_base[o][i] u[j][i] for the NJ rows of u, one
// output o per thread at a time: the 16 codes of a word are decoded from a
// register and each adds u_i to the row's positive or negative sum, or
// nothing.  Rows are d floats apart in shared memory.
template <int NJ>
__device__ __forceinline__ void decode_product(const float* u, float* z, const uint32_t* __restrict__ w_packed, int d,
                                               int words, float alpha) {
  for (int o = threadIdx.x; o < d; o += blockDim.x) {
    const uint32_t* wr = w_packed + static_cast<size_t>(o) * words;
    float pos[NJ], neg[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) pos[j] = neg[j] = 0.f;
    if (d >= 16) {
#pragma unroll 2
      for (int w = 0; w < words; ++w) {
        const uint32_t word = __ldg(wr + w);
#pragma unroll
        for (int b = 0; b < 16; ++b) {
          const uint32_t c = (word >> (2 * b)) & 3u;
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            const float ui = u[static_cast<size_t>(j) * d + 16 * w + b];
            pos[j] += c == 1u ? ui : 0.f;
            neg[j] += c == 3u ? ui : 0.f;
          }
        }
      }
    } else {
      const uint32_t word = __ldg(wr);  // one word holds the whole row
      for (int b = 0; b < d; ++b) {
        const uint32_t c = (word >> (2 * b)) & 3u;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const float ui = u[static_cast<size_t>(j) * d + b];
          pos[j] += c == 1u ? ui : 0.f;
          neg[j] += c == 3u ? ui : 0.f;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < NJ; ++j) z[static_cast<size_t>(j) * d + o] = alpha * (pos[j] - neg[j]);
  }
}

template <typename Tx>
__global__ __launch_bounds__(kDecodeThreads) void decode_kernel(const Tx* __restrict__ x, int T, int d, int L, int k,
                                                                const int32_t* __restrict__ idx,
                                                                const float* __restrict__ gates,
                                                                const uint32_t* __restrict__ w_packed, float alpha,
                                                                const float* __restrict__ theta,
                                                                const float* __restrict__ phi, int N,
                                                                Tx* __restrict__ y) {
  extern __shared__ float dec_smem[];
  const int kc = decode_rows(d, k);
  float* u = dec_smem;                          // [kc][d] rotated inputs
  float* z = u + static_cast<size_t>(kc) * d;   // [kc][d] products, then rotated outputs
  __shared__ const float* th_s[kDecodeRows];
  __shared__ const float* ph_s[kDecodeRows];
  __shared__ float g_s[kDecodeRows];
  const int words = d >= 16 ? d / 16 : 1;
  const size_t per_expert = static_cast<size_t>(L) * (d / 2);
  pdl_wait();
  pdl_trigger();
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    float acc[kDecodeOut];
#pragma unroll
    for (int m = 0; m < kDecodeOut; ++m) acc[m] = 0.f;
    for (int j0 = 0; j0 < k; j0 += kc) {
      const int nj = k - j0 < kc ? k - j0 : kc;
      if (threadIdx.x < nj) {
        const int jj = threadIdx.x;
        const int e = idx[static_cast<size_t>(t) * k + j0 + jj];
        const bool good = e >= 0 && e < N;
        if (!good) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(t));
        th_s[jj] = good ? theta + e * per_expert : nullptr;
        ph_s[jj] = good ? phi + e * per_expert : nullptr;
        g_s[jj] = gates[static_cast<size_t>(t) * k + j0 + jj];
      }
      for (int q = threadIdx.x; q < nj * d; q += blockDim.x)
        u[q] = to_f32(x[static_cast<size_t>(t) * d + (q % d)]);
      __syncthreads();
      for (int s = L - 1; s >= 0; --s) decode_stage<true>(u, th_s, nj, d, s);
      // the ternary product of every slot row at once: each 2-bit code adds
      // u_i, subtracts it or skips it; a row's code words are loaded once
      switch (nj) {
        case 1: decode_product<1>(u, z, w_packed, d, words, alpha); break;
        case 2: decode_product<2>(u, z, w_packed, d, words, alpha); break;
        case 3: decode_product<3>(u, z, w_packed, d, words, alpha); break;
        case 4: decode_product<4>(u, z, w_packed, d, words, alpha); break;
        case 5: decode_product<5>(u, z, w_packed, d, words, alpha); break;
        case 6: decode_product<6>(u, z, w_packed, d, words, alpha); break;
        case 7: decode_product<7>(u, z, w_packed, d, words, alpha); break;
        default: decode_product<8>(u, z, w_packed, d, words, alpha); break;
      }
      __syncthreads();
      for (int s = 0; s < L; ++s) decode_stage<false>(z, ph_s, nj, d, s);
      // gated sum in slot order
#pragma unroll
      for (int m = 0; m < kDecodeOut; ++m) {
        const int i = threadIdx.x + m * kDecodeThreads;
        if (i < d)
          for (int jj = 0; jj < nj; ++jj)
            if (ph_s[jj]) acc[m] += g_s[jj] * z[static_cast<size_t>(jj) * d + i];
      }
      __syncthreads();
    }
#pragma unroll
    for (int m = 0; m < kDecodeOut; ++m) {
      const int i = threadIdx.x + m * kDecodeThreads;
      if (i < d) y[static_cast<size_t>(t) * d + i] = from_f32<Tx>(acc[m]);
    }
  }
}

}  // namespace bfmoe
