// The whole expert of the ButterflyMoE inference in one persistent kernel, for
// bf16 tokens and 64 <= d <= 512 (technical summary, 2.3: B(theta)^T, the
// ternary product with the shared base, B(phi), without forming any expert
// and without writing the rotated rows or the product to memory):
//
//   slot[r] = g_r * B(phi_e) (alpha * W_base (B(theta_e)^T x_t))
//
// for the 128 bucket positions p of a tile (row r = rows[p], t = r / k,
// e = idx[r]).  One CTA per SM walks tiles; per tile
//   warps 2..9    (producers)  gather the tile's token rows, apply
//                 B(theta_e)^T in registers (the two warp layouts of
//                 rotate_fast.cuh), round to bf16 and write them straight into
//                 the MMA's A operand: 128 x d bf16 in shared memory, K-major
//                 with the 128-byte swizzle that TMA would produce;
//   warp 0 (lane 0) streams the bf16 base with TMA, 256 x 64 tiles, through
//                 a two-stage ring;
//   warp 1 (lane 0) issues tcgen05.mma (M = 128, N = min(d, 256), K = 16)
//                 into one fp32 accumulator of d TMEM columns: the tile's full
//                 output rows;
//   warps 10..17  (epilogue, two per TMEM lane quadrant, one thread per row)
//                 apply alpha and B(phi_e) with tensor memory as the row's
//                 fp32 backing store: stages 0..4 act inside each 32-column
//                 chunk (tcgen05.ld, rotate, tcgen05.st); stages 5..L-1 act
//                 on column slices c, c+32, c+64, ... loaded two slices at a
//                 time; finally the gated row is rounded to bf16 and stored
//                 with 32-byte stores.
// A (128 x d bf16) and the accumulator (128 x d fp32) fill most of shared and
// tensor memory at d = 512, so a tile's MMAs wait for the previous tile's
// epilogue, and the producers refill A once the previous tile's MMAs have
// read it; the producers' and the epilogue's CUDA-core work of consecutive
// tiles runs at the same time.
//
// cos/sin tables: the producers read the quad tables of rotate_fast.cuh; the
// epilogue reads pair quads (cos a_2u, cos a_2u+1, sin a_2u, sin a_2u+1) of
// each stage in natural rotation order, [N][L][d/4] float4: rotations
// 16j .. 16j+15 of a stage s < 5 are the chunk j ones, and rotations
// 32m + c, 32m + c + 1 of a stage s >= 5 those of slices c and c + 1.
#pragma once
#include "common.cuh"
#include "gemm_tc.cuh"
#include "rotate_fast.cuh"

namespace bfmoe {

constexpr int kFusedProdWarps = 8;
constexpr int kFusedEpiWarps = 8;
constexpr int kFusedThreads = (2 + kFusedProdWarps + kFusedEpiWarps) * 32;
constexpr int kFusedBStages = 2;

template <int D>
struct FusedCfg {
  static_assert(D >= 64 && D <= 512, "fused path: 64 <= d <= 512");
  static constexpr int E = D / 32;
  using Gm = Geo<E>;
  static constexpr int L = Gm::L;
  static constexpr int BN = D < 256 ? D : 256;  // MMA N
  static constexpr int NH = D / BN;             // MMAs per k-step (N halves)
  static constexpr int NK = D / kGemmBK;        // k-blocks
  static constexpr int NCH = D / 32;            // 32-column chunks of a row
  static constexpr int PG = E >= 16 ? 2 : 4;    // rows per producer group
  static constexpr int ROWS_PER_PROD = kGemmBM / kFusedProdWarps;
  static constexpr uint32_t A_KB_BYTES = kGemmBM * kGemmBK * 2;
  static constexpr uint32_t A_BYTES = NK * A_KB_BYTES;
  static constexpr uint32_t B_BYTES = BN * kGemmBK * 2;
  static constexpr uint32_t PROD_BUF = D * 4;  // one float32 row: the layout switch
  static constexpr uint32_t BAR_BYTES = (2 * kFusedBStages + 3 + 4) * 8 + 8;
  static constexpr uint32_t SMEM_BYTES =
      1024 + A_BYTES + kFusedBStages * B_BYTES + kFusedProdWarps * PROD_BUF + BAR_BYTES;
  static constexpr uint32_t TMEM_COLS = D;
  static_assert(ROWS_PER_PROD % PG == 0, "producer groups");
};

// Byte offset, inside the A tile, of the 16-byte unit that holds elements
// [8u, 8u+8) of tile row m: k-block u/8, 8-row atoms of 1024 bytes, the unit
// index XOR (m mod 8) (the 128-byte swizzle).
template <int D>
__device__ __forceinline__ uint32_t a_unit_offset(int m, int u) {
  return static_cast<uint32_t>((u >> 3) * FusedCfg<D>::A_KB_BYTES + (m >> 3) * 1024 + (m & 7) * 128 +
                               (((u & 7) ^ (m & 7)) << 4));
}

// Lane `lane`'s elements [lane*E, lane*E + E) of a row in layout 1, rounded to
// bf16, into tile row m of A.
template <int D>
__device__ __forceinline__ void store_a_row(uint8_t* A, int m, const float (&v)[D / 32], int lane) {
  constexpr int E = D / 32;
  if constexpr (E >= 8) {
#pragma unroll
    for (int w = 0; w < E / 8; ++w) {
      uint32_t pk[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * w + 2 * j], v[8 * w + 2 * j + 1]);
        pk[j] = *reinterpret_cast<uint32_t*>(&h);
      }
      *reinterpret_cast<uint4*>(A + a_unit_offset<D>(m, lane * (E / 8) + w)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  } else {
    // E = 2 or 4: a lane holds half or a quarter of a 16-byte unit
    constexpr int PER = 8 / E;  // lanes per unit
    uint32_t pk[E / 2];
#pragma unroll
    for (int j = 0; j < E / 2; ++j) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
      pk[j] = *reinterpret_cast<uint32_t*>(&h);
    }
    uint8_t* dst = A + a_unit_offset<D>(m, lane / PER) + (lane % PER) * (2 * E);
    if constexpr (E == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
    else *reinterpret_cast<uint32_t*>(dst) = pk[0];
  }
}

template <int D>
__device__ __forceinline__ void zero_a_row(uint8_t* A, int m, int lane) {
  float z[D / 32];
#pragma unroll
  for (int q = 0; q < D / 32; ++q) z[q] = 0.f;
  store_a_row<D>(A, m, z, lane);
}

// Rows of a group in layout 2 straight from global memory (lane l reads
// element q*32 + l of each row: 64 contiguous bytes per warp load).
template <int E, int G>
__device__ __forceinline__ void load_x_rows_l2(const __nv_bfloat16* __restrict__ x, const int (&tok)[G],
                                               float (&v)[G][E], int lane) {
  constexpr int D = 32 * E;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const __nv_bfloat16* src = x + static_cast<size_t>(tok[g]) * D + lane;
#pragma unroll
    for (int q = 0; q < E; ++q) v[g][q] = __bfloat162float(src[q * 32]);
  }
}

// B(theta)^T of G rows held in layout 2; leaves them in layout 1.
template <class Gm, int G>
__device__ __forceinline__ void pre_rotate_core(float (&v)[G][Gm::E], const float4* tq, float* buf, int lane) {
  l2_tr<Gm, G, Gm::L - 1>(v, tq, lane);
#pragma unroll
  for (int g = 0; g < G; ++g) to_layout1<Gm::E>(v[g], buf, lane);
  l1_tr<Gm, G, Gm::P - 1>(v, tq, lane);
}

// One Givens rotation, forward block [[c, -s], [s, c]].
__device__ __forceinline__ void rot_fwd(float& a, float& b, float c, float s) {
  const float na = c * a - s * b;
  b = s * a + c * b;
  a = na;
}

// Stages 0..4 of B(phi) on one 32-column chunk j of a row (thread = row).
// tp: the row's expert table, [L][D/4] pair quads.
template <int D>
__device__ __forceinline__ void epi_chunk_stages(float (&v)[32], const float4* __restrict__ tp, int j) {
  constexpr int L = FusedCfg<D>::L;
  constexpr int S5 = L < 5 ? L : 5;
#pragma unroll
  for (int s = 0; s < S5; ++s) {
    const int h = 1 << s;
    const float4* t = tp + s * (D / 4) + 8 * j;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float4 q = __ldg(t + u);
      // local rotations 2u and 2u+1 of this chunk: lower elements i0, i1
      const int r0 = 2 * u, r1 = 2 * u + 1;
      const int i0 = ((r0 >> s) << (s + 1)) | (r0 & (h - 1));
      const int i1 = ((r1 >> s) << (s + 1)) | (r1 & (h - 1));
      if (s >= 1) {
        // i1 = i0 + 1: two rotations in one packed op
        float2 x = make_float2(v[i0], v[i1]);
        float2 y = make_float2(v[i0 + h], v[i1 + h]);
        const float2 c2 = make_float2(q.x, q.y), s2 = make_float2(q.z, q.w);
        const float2 nx = __ffma2_rn(c2, x, __fmul2_rn(make_float2(-q.z, -q.w), y));
        const float2 ny = __ffma2_rn(c2, y, __fmul2_rn(s2, x));
        v[i0] = nx.x;
        v[i1] = nx.y;
        v[i0 + h] = ny.x;
        v[i1 + h] = ny.y;
      } else {
        rot_fwd(v[i0], v[i0 + 1], q.x, q.z);
        rot_fwd(v[i1], v[i1 + 1], q.y, q.w);
      }
    }
  }
}

template <int D>
__global__ __launch_bounds__(kFusedThreads, 1) void fused_expert_kernel(
    const __grid_constant__ CUtensorMap tmB, const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ idx,
    const float* __restrict__ gates, const int32_t* __restrict__ rows, const float4* __restrict__ tq_theta,
    const float4* __restrict__ pq_phi, long long R, int k, int N, float alpha, __nv_bfloat16* __restrict__ slot) {
  using C = FusedCfg<D>;
  using Gm = typename C::Gm;
  constexpr int E = C::E;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* A = smem;
  uint8_t* Bs = smem + C::A_BYTES;
  float* prod_buf = reinterpret_cast<float*>(Bs + kFusedBStages * C::B_BYTES);
  uint64_t* bfull = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(prod_buf) + kFusedProdWarps * C::PROD_BUF);
  uint64_t* bempty = bfull + kFusedBStages;
  uint64_t* a_full = bempty + kFusedBStages;  // producers -> MMA (one arrival per producer warp)
  uint64_t* mma_done = a_full + 1;            // MMA -> producers (A free) and epilogue (accumulator ready)
  uint64_t* acc_empty = mma_done + 1;         // epilogue -> MMA (one arrival per epilogue warp)
  uint64_t* qbar = acc_empty + 1;             // [4]: the two epilogue warps of a lane quadrant
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qbar + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long n_tiles = (R + kGemmBM - 1) / kGemmBM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFusedBStages; ++s) {
      mbar_init(bfull + s, 1);
      mbar_init(bempty + s, 1);
    }
    mbar_init(a_full, kFusedProdWarps);
    mbar_init(mma_done, 1);
    mbar_init(acc_empty, kFusedEpiWarps);
    for (int q = 0; q < 4; ++q) mbar_init(qbar + q, 2);
    mbar_fence_init();
    tma_prefetch_desc(&tmB);
  }
  if (warp == 0) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // routing and buckets come from the previous kernel
  pdl_trigger();

  if (warp == 0) {
    // ---- TMA: the bf16 base, k-block by k-block, for every tile -----------
    if (lane == 0) {
      int it = 0;
      bool alive = true;
      for (long long t = blockIdx.x; t < n_tiles && alive; t += gridDim.x) {
        for (int h = 0; h < C::NH && alive; ++h) {
          for (int kb = 0; kb < C::NK; ++kb, ++it) {
            const int s = it % kFusedBStages;
            const uint32_t ph = (it / kFusedBStages) & 1u;
            if (it >= kFusedBStages && !mbar_wait(bempty + s, ph ^ 1u, 0x2100u | s)) {
              alive = false;
              break;
            }
            mbar_expect_tx(bfull + s, C::B_BYTES);
            tma_load_2d(Bs + s * C::B_BYTES, &tmB, bfull + s, kb * kGemmBK, h * C::BN);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer ---------------------------------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kGemmBM, C::BN);
      int it = 0, i = 0;
      bool alive = true;
      for (long long t = blockIdx.x; t < n_tiles && alive; t += gridDim.x, ++i) {
        if (!mbar_wait(a_full, i & 1u, 0x2200u)) break;
        if (i >= 1 && !mbar_wait(acc_empty, (i - 1) & 1u, 0x2300u)) break;
        tc_fence_after();
        for (int h = 0; h < C::NH && alive; ++h) {
          for (int kb = 0; kb < C::NK; ++kb, ++it) {
            const int s = it % kFusedBStages;
            const uint32_t ph = (it / kFusedBStages) & 1u;
            if (!mbar_wait(bfull + s, ph, 0x2400u | s)) {
              alive = false;
              break;
            }
            tc_fence_after();
            const uint64_t ad = desc_kmajor_sw128(smem_u32(A + kb * C::A_KB_BYTES));
            const uint64_t bd = desc_kmajor_sw128(smem_u32(Bs + s * C::B_BYTES));
#pragma unroll
            for (int kk = 0; kk < kGemmBK / 16; ++kk)
              mma_bf16_ss(tmem + static_cast<uint32_t>(h * C::BN), ad + 2u * kk, bd + 2u * kk, idesc,
                          (kb | kk) != 0 ? 1u : 0u);
            mma_commit(bempty + s);
          }
        }
        if (alive) mma_commit(mma_done);
      }
    }
  } else if (warp < 2 + kFusedProdWarps) {
    // ---- producers: gather, B(theta)^T, bf16 into A -------------------------
    const int pw = warp - 2;
    float* buf = prod_buf + pw * (C::PROD_BUF / 4);
    constexpr int PG = C::PG;
    int i = 0;
    for (long long t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const long long pb = t * kGemmBM + pw * C::ROWS_PER_PROD;
      const RowMeta mine = lane < C::ROWS_PER_PROD ? fetch_row_meta(rows, idx, nullptr, pb + lane, R, N)
                                                   : RowMeta{-1, -1, 0.f};
      const int my_tok = mine.row >= 0 ? mine.row / k : 0;
      bool ok = true;
#pragma unroll 1
      for (int g0 = 0; g0 < C::ROWS_PER_PROD; g0 += PG) {
        int tok[PG];
#pragma unroll
        for (int g = 0; g < PG; ++g) tok[g] = __shfl_sync(FULL_MASK, my_tok, g0 + g);
        const int e0 = __shfl_sync(FULL_MASK, mine.ex, g0);
        const unsigned gm = ((1u << PG) - 1u) << g0;
        const unsigned same = __ballot_sync(FULL_MASK, mine.ex >= 0 && mine.ex == e0) & gm;
        float v[PG][E];
        load_x_rows_l2<E, PG>(x, tok, v, lane);
        if (same == gm) {
          pre_rotate_core<Gm, PG>(v, tq_theta + static_cast<size_t>(e0) * tab_quads(E), buf, lane);
        } else {
          // rows of different experts (or past the end): one at a time
#pragma unroll
          for (int g = 0; g < PG; ++g) {
            const int e = __shfl_sync(FULL_MASK, mine.ex, g0 + g);
            float v1[1][E];
#pragma unroll
            for (int q = 0; q < E; ++q) v1[0][q] = v[g][q];
            if (e >= 0) pre_rotate_core<Gm, 1>(v1, tq_theta + static_cast<size_t>(e) * tab_quads(E), buf, lane);
#pragma unroll
            for (int q = 0; q < E; ++q) v[g][q] = e >= 0 ? v1[0][q] : 0.f;
          }
        }
        // A is free once the previous tile's MMAs have completed
        if (g0 == 0 && i >= 1 && !mbar_wait(mma_done, (i - 1) & 1u, 0x2500u)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int g = 0; g < PG; ++g) store_a_row<D>(A, pw * C::ROWS_PER_PROD + g0 + g, v[g], lane);
      }
      if (!ok) break;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(a_full);
    }
  } else {
    // ---- epilogue: alpha, B(phi), gate; one thread per row ---------------
    const int qd = warp & 3;                                  // TMEM lane quadrant
    const int wq = (warp - 2 - kFusedProdWarps) >> 2;         // which half of the work
    const int m = qd * 32 + lane;                             // row within the tile
    const uint32_t trow = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    int i = 0;
    for (long long t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const long long p = t * kGemmBM + m;
      const RowMeta mt = p < R ? fetch_row_meta(rows, idx, gates, p, R, N) : RowMeta{-1, -1, 0.f};
      const float4* tp = pq_phi + static_cast<size_t>(mt.ex >= 0 ? mt.ex : 0) * C::L * (D / 4);
      if (!mbar_wait(mma_done, i & 1u, 0x2600u)) break;
      tc_fence_after();
      // stages 0..4 inside each 32-column chunk (the two warps take alternate chunks)
#pragma unroll 1
      for (int j = wq; j < C::NCH; j += 2) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(trow + 32 * j, r);
        tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = alpha * __uint_as_float(r[q]);
        epi_chunk_stages<D>(v, tp, j);
#pragma unroll
        for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(v[q]);
        tmem_st_32x32b_x32(trow + 32 * j, r);
      }
      tmem_wait_st();
      // both warps of the quadrant have finished the chunk stages
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(qbar + qd);
      if (!mbar_wait(qbar + qd, i & 1u, 0x2700u | qd)) break;
      tc_fence_after();
      // stages 5..L-1 on column slices c, c+32, ...; this warp takes the
      // slices c in [16 wq, 16 wq + 16), two at a time
#pragma unroll 1
      for (int c = 16 * wq; c < 16 * wq + 16; c += 2) {
        float2 w[C::NCH];
#pragma unroll
        for (int jj = 0; jj < C::NCH; ++jj) {
          uint32_t a0, a1;
          tmem_ld_32x32b_x2(trow + 32 * jj + c, a0, a1);
          w[jj] = make_float2(__uint_as_float(a0), __uint_as_float(a1));
        }
        tmem_wait_ld();
#pragma unroll
        for (int s = 5; s < C::L; ++s) {
          const int hh = 1 << (s - 5);
          const float4* ts = tp + s * (D / 4) + (c >> 1);
#pragma unroll
          for (int mr = 0; mr < C::NCH / 2; ++mr) {
            // mr-th pair (jj, jj + hh) of the slice with bit (s-5) of jj clear
            const int jj = ((mr >> (s - 5)) << (s - 4)) | (mr & (hh - 1));
            const float4 q = __ldg(ts + 16 * mr);  // rotations 32 mr + c, 32 mr + c + 1
            const float2 c2 = make_float2(q.x, q.y), s2 = make_float2(q.z, q.w);
            const float2 a = w[jj], b = w[jj + hh];
            w[jj] = __ffma2_rn(c2, a, __fmul2_rn(make_float2(-q.z, -q.w), b));
            w[jj + hh] = __ffma2_rn(c2, b, __fmul2_rn(s2, a));
          }
        }
#pragma unroll
        for (int jj = 0; jj < C::NCH; ++jj)
          tmem_st_32x32b_x2(trow + 32 * jj + c, __float_as_uint(w[jj].x), __float_as_uint(w[jj].y));
      }
      tmem_wait_st();
      // gated rows out: columns [16 wq, 16 wq + 16) of each chunk (the ones
      // this warp finished), 32 bytes per store
#pragma unroll 1
      for (int j = 0; j < C::NCH; ++j) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(trow + 32 * j + 16 * wq, r);
        tmem_wait_ld();
        if (mt.ex >= 0) {
          uint32_t pk[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            __nv_bfloat162 h2 =
                __floats2bfloat162_rn(mt.gate * __uint_as_float(r[2 * u]), mt.gate * __uint_as_float(r[2 * u + 1]));
            pk[u] = *reinterpret_cast<uint32_t*>(&h2);
          }
          __nv_bfloat16* dst = slot + static_cast<size_t>(mt.row) * D + 32 * j + 16 * wq;
          asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(pk[0]),
                       "r"(pk[1]), "r"(pk[2]), "r"(pk[3]), "r"(pk[4]), "r"(pk[5]), "r"(pk[6]), "r"(pk[7])
                       : "memory");
        }
      }
      // the accumulator may be overwritten by the next tile's MMAs
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, C::TMEM_COLS);
}

// Pair quads of one butterfly's angles: out[(e*L + s)*(d/4) + u] =
// (cos a_2u, cos a_2u+1, sin a_2u, sin a_2u+1) with a = ang[e][s][.].
__global__ void rot_pairq_kernel(const float* __restrict__ ang, long long n_pairs, float4* __restrict__ out) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n_pairs;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float2 a = reinterpret_cast<const float2*>(ang)[i];
    float s0, c0, s1, c1;
    sincosf(a.x, &s0, &c0);
    sincosf(a.y, &s1, &c1);
    out[i] = make_float4(c0, c1, s0, s1);
  }
}

}  // namespace bfmoe
