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
//                 with the 128-byte swizzle that TMA would produce.  The rows
//                 are claimed in units of 8 from a shared counter, and the
//                 epilogue warps join in whenever they have no epilogue work
//                 (the first tile, and the next tile once theirs is done);
//   warp 0 (lane 0) streams the bf16 base with TMA, 128 x 64 tiles, through
//                 a ring of 2 (d = 512) or 4 stages;
//   warp 1 (lane 0) issues tcgen05.mma (M = 128, N = min(d, 128), K = 16)
//                 into one fp32 accumulator of d TMEM columns: the tile's full
//                 output rows;
//   warps 10..17  (epilogue, two per TMEM lane quadrant, one thread per row)
//                 apply B(phi_e) with tensor memory as the row's fp32
//                 backing store: stages 0..4 act inside each 32-column chunk
//                 (tcgen05.ld, rotate, tcgen05.st); stages 5..L-1 act on
//                 column slices c, c+32, c+64, ... loaded two slices at a
//                 time; finally the row times gate * alpha (the butterfly is
//                 linear: g B(phi)(alpha z) = (g alpha) B(phi) z) is rounded
//                 to bf16 and stored with 32-byte stores.
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
constexpr int kFusedSimtWarps = kFusedProdWarps + kFusedEpiWarps;  // all of them produce A
constexpr int kFusedThreads = (2 + kFusedSimtWarps) * 32;

template <int D>
struct FusedCfg {
  static_assert(D >= 64 && D <= 512, "fused path: 64 <= d <= 512");
  static constexpr int E = D / 32;
  using Gm = Geo<E>;
  static constexpr int L = Gm::L;
  static constexpr int BN = D < 128 ? D : 128;  // MMA N (a 128-row W_base tile per stage)
  static constexpr int NH = D / BN;             // MMAs per k-step (N halves)
  static constexpr int NK = D / kGemmBK;        // k-blocks
  static constexpr int NCH = D / 32;            // 32-column chunks of a row
  static constexpr int PG = E >= 16 ? 2 : 4;    // rows per producer group
  static constexpr uint32_t A_KB_BYTES = kGemmBM * kGemmBK * 2;
  static constexpr uint32_t A_BYTES = NK * A_KB_BYTES;
  static constexpr uint32_t B_BYTES = BN * kGemmBK * 2;
  static constexpr int BSTAGES = D >= 512 ? 2 : 4;  // W_base ring
  // the theta quads of one expert, staged per tile for the producers
  static constexpr int TABQ = tab_quads(E);
  static constexpr uint32_t TAB_FULL = TABQ * 16;
  static constexpr uint32_t PROD_BUF = D * 4;  // one float32 row: the layout switch
  // per epilogue warp, two buffers of cos/sin quads staged from global memory:
  // a chunk's stages 0..4 (5 x 8 quads) or a slice pair's stages 5.. (<= 32)
  static constexpr int EPI_QUADS = 40;
  // (also the layout-switch buffer when an epilogue warp helps produce A)
  static constexpr uint32_t EPI_BUF = 2 * EPI_QUADS * 16 > D * 4 ? 2 * EPI_QUADS * 16 : D * 4;
  // production of a tile's A is claimed in units of UNIT rows
  static constexpr int UNIT = 8;
  static constexpr int NUNITS = kGemmBM / UNIT;
  static constexpr uint32_t BAR_BYTES = (2 * BSTAGES + 4 + 4 + NH) * 8 + 8 + 32;
  static constexpr uint32_t SMEM_NO_TAB =
      1024 + A_BYTES + BSTAGES * B_BYTES + kFusedProdWarps * PROD_BUF + kFusedEpiWarps * EPI_BUF + BAR_BYTES;
  // the staged theta table where it fits (not at d = 512)
  static constexpr bool USE_TAB = SMEM_NO_TAB + TAB_FULL <= 232448;
  static constexpr uint32_t TAB_BYTES = USE_TAB ? TAB_FULL : 0;
  static constexpr uint32_t SMEM_BYTES = SMEM_NO_TAB + TAB_BYTES;
  static_assert(SMEM_BYTES <= 232448, "shared memory of one CTA");
  static_assert((L - 5) * (NCH / 2) <= EPI_QUADS, "slice-pair quads fit the staging buffer");
  static constexpr uint32_t TMEM_COLS = D;
  static_assert(UNIT % PG == 0, "producer groups");
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
// element q*32 + l of each row: 64 contiguous bytes per warp load); a
// negative token gives a row of zeros.
template <int E, int G>
__device__ __forceinline__ void load_x_rows_l2(const __nv_bfloat16* __restrict__ x, const int (&tok)[G],
                                               float (&v)[G][E], int lane) {
  constexpr int D = 32 * E;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const bool valid = tok[g] >= 0;
    const __nv_bfloat16* src = x + static_cast<size_t>(valid ? tok[g] : 0) * D + lane;
#pragma unroll
    for (int q = 0; q < E; ++q) v[g][q] = valid ? __bfloat162float(src[q * 32]) : 0.f;
  }
}

// The kernel walks the buckets padded to whole multiples of 32 rows
// (bucket_pad_kernel): position P holds routed row pmap[P] (-1: padding) of
// expert qex[P / 32] (-1 past the last segment).  So the 32 rows of a TMEM
// lane quadrant, and the 8 rows of a production unit, never mix experts.
struct PadRow {
  int e, row;  // expert; routed row r = t*k + j (or -1)
};
__device__ __forceinline__ PadRow pad_row(long long P, const int32_t* __restrict__ pmap,
                                          const int32_t* __restrict__ qex) {
  return PadRow{qex[P >> 5], pmap[P]};
}

// Untiled bulk copy global -> shared (no multicast); completes on bar.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
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

// Stages 0..4 of B(phi) on one 32-column chunk of a row (thread = row).
// t[s * stride + u] holds the pair quad of the chunk's local rotations 2u and
// 2u+1 in stage s: the row's expert table in global memory (stride d/4, t at
// the chunk's first quad) or the warp's staged copy in shared memory
// (stride 8).
template <int D, bool SHARED>
__device__ __forceinline__ void epi_chunk_stages(float (&v)[32], const float4* __restrict__ t, int stride) {
  constexpr int L = FusedCfg<D>::L;
  constexpr int S5 = L < 5 ? L : 5;
#pragma unroll
  for (int s = 0; s < S5; ++s) {
    const int h = 1 << s;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float4 q = SHARED ? t[s * stride + u] : __ldg(t + s * stride + u);
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

// Stages 5..L-1 of B(phi) on the column slices c and c+1 of a row:
// w[jj] = (column 32 jj + c, column 32 jj + c + 1).  The pair quad of stage s
// and slice rotation mr is t[(s - 5) * st_s + mr * st_m].
template <int D, bool SHARED>
__device__ __forceinline__ void epi_slice_stages(float2 (&w)[D / 32], const float4* __restrict__ t, int st_s,
                                                 int st_m) {
  constexpr int L = FusedCfg<D>::L;
  constexpr int NCH = D / 32;
#pragma unroll
  for (int s = 5; s < L; ++s) {
    const int hh = 1 << (s - 5);
#pragma unroll
    for (int mr = 0; mr < NCH / 2; ++mr) {
      // mr-th pair (jj, jj + hh) of the slice with bit (s-5) of jj clear
      const int jj = ((mr >> (s - 5)) << (s - 4)) | (mr & (hh - 1));
      const float4 q = SHARED ? t[(s - 5) * st_s + mr * st_m] : __ldg(t + (s - 5) * st_s + mr * st_m);
      const float2 c2 = make_float2(q.x, q.y), s2 = make_float2(q.z, q.w);
      const float2 a = w[jj], b = w[jj + hh];
      w[jj] = __ffma2_rn(c2, a, __fmul2_rn(make_float2(-q.z, -q.w), b));
      w[jj + hh] = __ffma2_rn(c2, b, __fmul2_rn(s2, a));
    }
  }
}

// What the producers of a CTA share.
struct ProdCtx {
  uint8_t* A;
  int* claim;           // [2] unit counters (tile parity), [2] finished warps
  uint64_t* a_full;     // producers -> MMA
  uint64_t* mma_done;   // MMA -> producers (A free)
  uint64_t* tab_full;   // the staged theta table has landed
  const float4* tab_s;  // staged theta quads of expert *tab_ex
  int* tab_ex;
  int* tab_n;  // stagings issued (tab_full phases)
  const __nv_bfloat16* x;
  const int32_t* pmap;
  const int32_t* qex;
  const float4* tq_theta;
  long long n_tiles;
  int k, grid;
};

// Stage the theta quads of the expert that leads tile t (or none) and signal
// tab_full.
template <int D>
__device__ __forceinline__ void stage_theta(const ProdCtx& c, long long t) {
  using C = FusedCfg<D>;
  const int e = C::USE_TAB && t < c.n_tiles ? c.qex[t * (kGemmBM / 32)] : -1;
  *c.tab_ex = e;
  *c.tab_n += 1;
  if (e >= 0) {
    mbar_expect_tx(c.tab_full, C::TAB_BYTES);
    bulk_load(const_cast<float4*>(c.tab_s), c.tq_theta + static_cast<size_t>(e) * C::TABQ, C::TAB_BYTES, c.tab_full);
  } else {
    mbar_arrive(c.tab_full);
  }
}

// Produce tile t's A operand (the tile's i-th in this CTA): every CUDA-core
// warp of the CTA calls this once per tile and claims units of UNIT rows from
// a shared counter until none are left; a unit's rows are gathered, rotated
// by B(theta_e)^T in groups of PG rows of one expert, rounded to bf16 and
// stored in A.  The quads of the tile's leading expert come from shared
// memory (staged by stage_theta), others from global memory.  With
// wait_free, the stores, and in any case the arrival, first wait for the
// previous tile's MMAs (A still holds their operand).  The last warp to
// finish resets the counters for tile i + 2 and stages the next tile's
// table, then every warp arrives on a_full.
template <int D>
__device__ __forceinline__ bool produce_tile(const ProdCtx& c, long long t, int i, bool wait_free, float* buf,
                                             int lane) {
  using C = FusedCfg<D>;
  using Gm = typename C::Gm;
  constexpr int E = C::E, PG = C::PG;
  int* ctr = c.claim + (i & 1);
  int* done = c.claim + 2 + (i & 1);
  bool ok = true, free_ = !wait_free, have_tab = false;
  int tab_e = -1;
  while (ok) {
    int u = 0;
    if (lane == 0) u = atomicAdd(ctr, 1);
    u = __shfl_sync(FULL_MASK, u, 0);
    if (u >= C::NUNITS) break;
    if (!have_tab) {
      if (!mbar_wait(c.tab_full, i & 1u, 0x2800u)) {
        ok = false;
        break;
      }
      tab_e = *c.tab_ex;
      have_tab = true;
    }
    const int r0 = u * C::UNIT;
    const PadRow mine = lane < C::UNIT ? pad_row(t * kGemmBM + r0 + lane, c.pmap, c.qex) : PadRow{-1, -1};
    const int my_tok = mine.row >= 0 ? mine.row / c.k : -1;
#pragma unroll 1
    for (int g0 = 0; g0 < C::UNIT; g0 += PG) {
      int tok[PG];
#pragma unroll
      for (int g = 0; g < PG; ++g) tok[g] = __shfl_sync(FULL_MASK, my_tok, g0 + g);
      const int e0 = __shfl_sync(FULL_MASK, mine.e, g0);
      const unsigned gm = ((1u << PG) - 1u) << g0;
      const unsigned same = __ballot_sync(FULL_MASK, mine.e >= 0 && mine.e == e0) & gm;
      float v[PG][E];
      load_x_rows_l2<E, PG>(c.x, tok, v, lane);
      if (same == gm) {
        // one expert (padding rows are zeros and stay zeros)
        const float4* tq = e0 == tab_e ? c.tab_s : c.tq_theta + static_cast<size_t>(e0) * C::TABQ;
        pre_rotate_core<Gm, PG>(v, tq, buf, lane);
      } else {
        // rows past the last segment (zeros), or inconsistent routing: one at a time
#pragma unroll
        for (int g = 0; g < PG; ++g) {
          const int e = __shfl_sync(FULL_MASK, mine.e, g0 + g);
          float v1[1][E];
#pragma unroll
          for (int q = 0; q < E; ++q) v1[0][q] = v[g][q];
          if (e >= 0) pre_rotate_core<Gm, 1>(v1, c.tq_theta + static_cast<size_t>(e) * C::TABQ, buf, lane);
#pragma unroll
          for (int q = 0; q < E; ++q) v[g][q] = e >= 0 ? v1[0][q] : 0.f;
        }
      }
      if (!free_) {
        if (!mbar_wait(c.mma_done, (i - 1) & 1u, 0x2500u)) {
          ok = false;
          break;
        }
        free_ = true;
      }
#pragma unroll
      for (int g = 0; g < PG; ++g) store_a_row<D>(c.A, r0 + g0 + g, v[g], lane);
    }
  }
  // a warp left without rows still waits for the previous tile's MMAs before
  // it arrives: an arrival for tile i must not land in tile i-1's phase, and
  // tile i+1's counters are only reset once every warp is past tile i-1
  if (ok && !free_ && !mbar_wait(c.mma_done, (i - 1) & 1u, 0x2500u)) ok = false;
  // every warp has seen this tile's table before the next one replaces it
  if (ok && !have_tab && !mbar_wait(c.tab_full, i & 1u, 0x2800u)) ok = false;
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    if (atomicAdd(done, 1) == kFusedSimtWarps - 1) {
      *ctr = 0;
      *done = 0;
      stage_theta<D>(c, t + c.grid);
    }
    mbar_arrive(c.a_full);
  }
  return ok;
}

template <int D>
__global__ __launch_bounds__(kFusedThreads, 1) void fused_expert_kernel(
    const __grid_constant__ CUtensorMap tmB, const __nv_bfloat16* __restrict__ x, const float* __restrict__ gates,
    const int32_t* __restrict__ pmap, const int32_t* __restrict__ qex, const int32_t* __restrict__ pad_total,
    const float4* __restrict__ tq_theta, const float4* __restrict__ pq_phi, int k, float alpha,
    __nv_bfloat16* __restrict__ slot) {
  using C = FusedCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint8_t* A = smem;
  uint8_t* Bs = smem + C::A_BYTES;
  float* prod_buf = reinterpret_cast<float*>(Bs + C::BSTAGES * C::B_BYTES);
  float4* epi_buf = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(prod_buf) + kFusedProdWarps * C::PROD_BUF);
  float4* tab_s = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(epi_buf) + kFusedEpiWarps * C::EPI_BUF);
  uint64_t* bfull = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(tab_s) + C::TAB_BYTES);
  uint64_t* bempty = bfull + C::BSTAGES;
  uint64_t* a_full = bempty + C::BSTAGES;  // producers -> MMA (one arrival per producer warp)
  uint64_t* mma_done = a_full + 1;            // MMA -> producers (A free)
  uint64_t* acc_empty = mma_done + 1;         // epilogue -> MMA (one arrival per epilogue warp)
  uint64_t* qbar = acc_empty + 1;             // [4]: the two epilogue warps of a lane quadrant
  uint64_t* tab_full = qbar + 4;              // staged theta table
  uint64_t* acc_blk = tab_full + 1;           // [NH]: MMA -> epilogue, one N block of the accumulator ready
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_blk + C::NH);
  int* claim = reinterpret_cast<int*>(tmem_slot + 2);  // [2] unit counters (tile parity), [2] finished warps
  int* tab_ex = claim + 4;
  int* tab_n = claim + 5;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::BSTAGES; ++s) {
      mbar_init(bfull + s, 1);
      mbar_init(bempty + s, 1);
    }
    mbar_init(a_full, kFusedSimtWarps);
    for (int q = 0; q < 6; ++q) claim[q] = 0;
    mbar_init(mma_done, 1);
    mbar_init(acc_empty, kFusedEpiWarps);
    for (int q = 0; q < 4; ++q) mbar_init(qbar + q, 2);
    mbar_init(tab_full, 1);
    for (int q = 0; q < C::NH; ++q) mbar_init(acc_blk + q, 1);
    mbar_fence_init();
    tma_prefetch_desc(&tmB);
  }
  if (warp == 0) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // routing and buckets come from the previous kernels
  pdl_trigger();
  const long long n_tiles = (static_cast<long long>(*pad_total) + kGemmBM - 1) / kGemmBM;
  const ProdCtx pc{A,    claim, a_full,    mma_done, tab_full, tab_s, tab_ex, tab_n, x, pmap, qex, tq_theta,
                   n_tiles, k,     static_cast<int>(gridDim.x)};
  if (threadIdx.x == 0) stage_theta<D>(pc, blockIdx.x);
  // every CTA walks the base's (N block, k block) tiles from its own starting
  // point, so that the CTAs do not all read the same L2 lines at once
  const int b_h0 = static_cast<int>(blockIdx.x % C::NH);
  const int b_kb0 = static_cast<int>((blockIdx.x / C::NH) % C::NK);

  if (warp == 0) {
    // ---- TMA: the bf16 base, k-block by k-block, for every tile -----------
    if (lane == 0) {
      int it = 0;
      bool alive = true;
      for (long long t = blockIdx.x; t < n_tiles && alive; t += gridDim.x) {
        for (int h0 = 0; h0 < C::NH && alive; ++h0) {
          const int h = (h0 + b_h0) % C::NH;
          for (int kb0 = 0; kb0 < C::NK; ++kb0, ++it) {
            const int kb = (kb0 + b_kb0) % C::NK;
            const int s = it % C::BSTAGES;
            const uint32_t ph = (it / C::BSTAGES) & 1u;
            if (it >= C::BSTAGES && !mbar_wait(bempty + s, ph ^ 1u, 0x2100u | s)) {
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
        for (int h0 = 0; h0 < C::NH && alive; ++h0) {
          const int h = (h0 + b_h0) % C::NH;
          for (int kb0 = 0; kb0 < C::NK; ++kb0, ++it) {
            const int kb = (kb0 + b_kb0) % C::NK;
            const int s = it % C::BSTAGES;
            const uint32_t ph = (it / C::BSTAGES) & 1u;
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
                          (kb0 | kk) != 0 ? 1u : 0u);
            mma_commit(bempty + s);
          }
          // the epilogue may start on this N block's columns
          if (alive) mma_commit(acc_blk + h0);
        }
        if (alive) mma_commit(mma_done);
      }
    }
  } else if (warp < 2 + kFusedProdWarps) {
    // ---- producers: gather, B(theta)^T, bf16 into A -------------------------
    const int pw = warp - 2;
    float* buf = prod_buf + pw * (C::PROD_BUF / 4);
    int i = 0;
    for (long long t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i)
      if (!produce_tile<D>(pc, t, i, i >= 1, buf, lane))
        break;
  } else {
    // ---- epilogue: B(phi), then gate * alpha; one thread per row ----------
    const int qd = warp & 3;                                  // TMEM lane quadrant
    const int ew = warp - 2 - kFusedProdWarps;                // epilogue warp 0..7
    const int wq = ew >> 2;                                   // which half of the work
    const int m = qd * 32 + lane;                             // row within the tile
    const uint32_t trow = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    float4* ebuf = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(epi_buf) + ew * C::EPI_BUF);
    constexpr int S5 = C::L < 5 ? C::L : 5;
    constexpr int NB = (C::L - 5) * (C::NCH / 2);  // quads of a slice pair
    float* pbuf = reinterpret_cast<float*>(ebuf);  // layout-switch buffer while producing
    int i = 0;
    if (blockIdx.x < n_tiles &&
        !produce_tile<D>(pc, blockIdx.x, 0, false, pbuf, lane))
      i = -1;
    for (long long t = blockIdx.x; t < n_tiles && i >= 0; t += gridDim.x, ++i) {
      const PadRow pr = pad_row(t * kGemmBM + m, pmap, qex);
      const RowMeta mt{pr.row, pr.e, pr.row >= 0 ? gates[pr.row] * alpha : 0.f};
      const float4* tp = pq_phi + static_cast<size_t>(mt.ex >= 0 ? mt.ex : 0) * C::L * (D / 4);
      // the quadrant's rows share one expert (padded buckets): its quads are
      // staged into shared memory ahead of use, bypassing L1; else (past the
      // last segment) each row reads its own
      const int ex0 = __shfl_sync(FULL_MASK, mt.ex, 0);
      const bool uni = __all_sync(FULL_MASK, mt.ex == ex0) && ex0 >= 0;
      const float4* tpu = pq_phi + static_cast<size_t>(ex0 >= 0 ? ex0 : 0) * C::L * (D / 4);
      auto stage_chunk = [&](int j, int b) {
        for (int l = lane; l < S5 * 8; l += 32)
          cp_async16(ebuf + b * C::EPI_QUADS + l, tpu + (l >> 3) * (D / 4) + 8 * j + (l & 7));
        cp_async_commit();
      };
      auto stage_slice = [&](int c, int b) {
        for (int l = lane; l < NB; l += 32)
          cp_async16(ebuf + b * C::EPI_QUADS + l,
                     tpu + (5 + l / (C::NCH / 2)) * (D / 4) + (c >> 1) + 16 * (l % (C::NCH / 2)));
        cp_async_commit();
      };
      // stages 0..4 inside each 32-column chunk, N block by N block in the
      // order the MMAs finish them (the two warps take alternate chunks)
      constexpr int CPW = C::BN / 64 > 0 ? C::BN / 64 : 1;  // chunks of an N block per warp
      auto chunk_of = [&](int n) {
        const int h = (n / CPW + b_h0) % C::NH;
        return h * (C::BN / 32) + 2 * (n % CPW) + wq;
      };
      if (uni) stage_chunk(chunk_of(0), 0);
      int b = 0;
      bool alive = true;
#pragma unroll 1
      for (int n = 0; n < C::NCH / 2; ++n, b ^= 1) {
        const int j = chunk_of(n);
        if (n % CPW == 0) {
          if (!mbar_wait(acc_blk + n / CPW, i & 1u, 0x2600u | (n / CPW))) {
            alive = false;
            break;
          }
          tc_fence_after();
        }
        uint32_t r[32];
        tmem_ld_32x32b_x32(trow + 32 * j, r);
        if (uni) {
          if (n + 1 < C::NCH / 2) {
            stage_chunk(chunk_of(n + 1), b ^ 1);
            cp_async_wait<1>();
          } else {
            cp_async_wait<0>();
          }
          __syncwarp();
        }
        tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = __uint_as_float(r[q]);
        if (uni) epi_chunk_stages<D, true>(v, ebuf + b * C::EPI_QUADS, 8);
        else epi_chunk_stages<D, false>(v, tp + 8 * j, D / 4);
#pragma unroll
        for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(v[q]);
        tmem_st_32x32b_x32(trow + 32 * j, r);
        __syncwarp();  // buffer b is refilled two chunks later
      }
      if (!alive) {
        cp_async_wait<0>();
        break;
      }
      if (uni) stage_slice(16 * wq, 0);
      tmem_wait_st();
      // both warps of the quadrant have finished the chunk stages
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(qbar + qd);
      if (!mbar_wait(qbar + qd, i & 1u, 0x2700u | qd)) break;
      tc_fence_after();
      // stages 5..L-1 on column slices c, c+32, ...; this warp takes the
      // slices c in [16 wq, 16 wq + 16), two at a time
      b = 0;
#pragma unroll 1
      for (int c = 16 * wq; c < 16 * wq + 16; c += 2, b ^= 1) {
        float2 w[C::NCH];
#pragma unroll
        for (int jj = 0; jj < C::NCH; ++jj) {
          uint32_t a0, a1;
          tmem_ld_32x32b_x2(trow + 32 * jj + c, a0, a1);
          w[jj] = make_float2(__uint_as_float(a0), __uint_as_float(a1));
        }
        if (uni) {
          if (c + 2 < 16 * wq + 16) {
            stage_slice(c + 2, b ^ 1);
            cp_async_wait<1>();
          } else {
            cp_async_wait<0>();
          }
          __syncwarp();
        }
        tmem_wait_ld();
        if (uni) epi_slice_stages<D, true>(w, ebuf + b * C::EPI_QUADS, C::NCH / 2, 1);
        else epi_slice_stages<D, false>(w, tp + 5 * (D / 4) + (c >> 1), D / 4, 16);
#pragma unroll
        for (int jj = 0; jj < C::NCH; ++jj)
          tmem_st_32x32b_x2(trow + 32 * jj + c, __float_as_uint(w[jj].x), __float_as_uint(w[jj].y));
        __syncwarp();  // buffer b is refilled two slice pairs later
      }
      tmem_wait_st();
      // gated rows out: columns [16 wq, 16 wq + 16) of each chunk (the ones
      // this warp finished), 32 bytes per store
#pragma unroll 1
      for (int j = 0; j < C::NCH; ++j) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(trow + 32 * j + 16 * wq, r);
        tmem_wait_ld();
        if (mt.row >= 0) {  // (padding rows have an expert but no row)
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
      // then help produce the next tile's A (free: its MMAs have completed)
      const long long tn = t + gridDim.x;
      if (tn < n_tiles &&
          !produce_tile<D>(pc, tn, i + 1, false, pbuf, lane))
        break;
    }
  }
  tc_fence_before();
  __syncthreads();
  // only the last staging can still be in flight (after an error exit)
  if (threadIdx.x == 0 && *tab_n > 0) mbar_wait(tab_full, (*tab_n - 1) & 1u, 0x2a00u);
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
