// Butterfly rotations of routed rows for d = 32*E >= 64, several rows of one
// expert per warp.
//
// Two register layouts of a row across the 32 lanes of a warp:
//   layout 1: lane l holds elements l*E + q        (q < E): index bits 0..e-1 in registers
//   layout 2: lane l holds elements q*32 + l       (q < E): index bits 5..L-1 in registers
// with e = log2 E and L = e + 5.  Stage s is done in layout 1 for s < P and in
// layout 2 for s >= P, P = max(5, e); in layout 1 the stages e..4 (only when
// e < 5) pair lanes l and l ^ 2^(s-e) through shuffles.  One transpose through
// a per-warp shared-memory buffer switches layouts.  A warp applies each
// loaded (cos, sin) to G rows of the same expert.
//
// Most stages process two rotations per packed float32 instruction
// (__ffma2_rn / __fmul2_rn).  The cos/sin table stores, per stage, quads
// (c_a, c_b, s_a, s_b) in the order the warp reads them: quad u*32 + l holds
// the u-th pair of rotations that lane l applies, so each warp-wide table read
// is 32 consecutive quads (no shared-memory bank conflicts).  A cross-lane
// stage stores its slice for every lane (partner lanes hold the same
// rotations), so it is twice the size of the others; layout-2 stage 5 keeps
// the natural order (a, b) = (2j, 2j+1).
#pragma once
#include "common.cuh"
#include "rotate.cuh"

namespace bfmoe {

template <int E_>
struct Geo {
  static constexpr int E = E_;
  static constexpr int e = Log2<E_>::value;
  static constexpr int L = e + 5;
  static constexpr int P = e > 5 ? e : 5;
  static constexpr int D = 32 * E_;
  // rows per warp: each cos/sin table load serves G rows of one expert
  static constexpr int G = E_ <= 16 ? 4 : (E_ <= 32 ? 2 : 1);
  static constexpr int WARPS = E_ <= 64 ? 8 : 4;
};

// Rotation index of element i in stage s (lower element of its pair).
__host__ __device__ __forceinline__ int rot_index(int i, int s) {
  return ((i >> (s + 1)) << s) + (i & ((1 << s) - 1));
}

// Quads of stage s in the table of one expert, for E elements per lane.
__host__ __device__ constexpr int tab_stage_quads(int E, int s) {
  int e = 0;
  while ((1 << e) < E) ++e;
  const int P = e > 5 ? e : 5;
  if (s < P && s >= e) return 32 * (E / 2);            // cross-lane (layout 1)
  if (s < P) return 32 * (E / 4 > 0 ? E / 4 : 1);      // in registers (layout 1)
  return 8 * E;                                         // layout 2 (d/4)
}
__host__ __device__ constexpr int tab_stage_offset(int E, int s) {
  int o = 0;
  for (int i = 0; i < s; ++i) o += tab_stage_quads(E, i);
  return o;
}
__host__ __device__ constexpr int tab_quads(int E) {
  int e = 0;
  while ((1 << e) < E) ++e;
  return tab_stage_offset(E, e + 5);
}

// Offsets of each stage's quads inside one expert's table (host-computed).
struct TabLayout {
  int off[13];   // quad offset of stage s
  int nq[13];    // quads of stage s
  int total;     // quads per expert
};

inline TabLayout make_tab_layout(int E, int L) {
  TabLayout t{};
  for (int s = 0; s < L; ++s) {
    t.off[s] = tab_stage_offset(E, s);
    t.nq[s] = tab_stage_quads(E, s);
  }
  t.total = tab_quads(E);
  return t;
}

// Quad tables: [2][N][total] float4 (theta then phi).  Blocks [0, 2N): one
// (table, expert) each.  The expert's L*d/2 angles are read once (coalesced,
// many loads in flight), their cos and sin kept in shared memory, then every
// stage's quads are gathered from there.  Blocks from 2N on expand the packed
// ternary base to bf16 (when expand_out is set), so both weight-derived
// inputs of the forward come from one launch.
__global__ __launch_bounds__(256) void rot_quads_kernel(const float* __restrict__ theta,
                                                        const float* __restrict__ phi, int N, int d, int L,
                                                        const TabLayout tl, float4* __restrict__ quads,
                                                        const uint32_t* __restrict__ w_packed,
                                                        uint16_t* __restrict__ expand_out) {
  extern __shared__ float cs_smem[];  // [L*d/2] cos, then [L*d/2] sin
  const int n_tab_blocks = 2 * N;
  if (static_cast<int>(blockIdx.x) >= n_tab_blocks) {
    // expand the 2-bit base: one thread per packed word (16 weights)
    const int wpr = d / 16;
    const long long nw = static_cast<long long>(d) * wpr;
    for (long long q = (blockIdx.x - n_tab_blocks) * static_cast<long long>(blockDim.x) + threadIdx.x; q < nw;
         q += static_cast<long long>(gridDim.x - n_tab_blocks) * blockDim.x) {
      const uint32_t word = w_packed[q];
      uint32_t pr[8];
#pragma unroll
      for (int m = 0; m < 8; ++m)
        pr[m] = ternary_code_bf16((word >> (4 * m)) & 3u) |
                (static_cast<uint32_t>(ternary_code_bf16((word >> (4 * m + 2)) & 3u)) << 16);
      uint4* d4 = reinterpret_cast<uint4*>(expand_out + q * 16);
      d4[0] = make_uint4(pr[0], pr[1], pr[2], pr[3]);
      d4[1] = make_uint4(pr[4], pr[5], pr[6], pr[7]);
    }
    return;
  }
  const int E = d / 32;
  const int e = L - 5;
  const int P = e > 5 ? e : 5;
  const int ex = blockIdx.x % N;
  const int which = blockIdx.x / N;
  const int half = d / 2;
  const int nang = L * half;
  const float* base = (which ? phi : theta) + static_cast<size_t>(ex) * nang;
  float* cs = cs_smem;
  float* sn = cs_smem + nang;
  for (int i = threadIdx.x; i < nang; i += blockDim.x) sincosf(base[i], &sn[i], &cs[i]);
  __syncthreads();
  float4* out0 = quads + (static_cast<size_t>(which) * N + ex) * tl.total;
  for (int s = 0; s < L; ++s) {
    const float* cst = cs + s * half;
    const float* snt = sn + s * half;
    float4* out = out0 + tl.off[s];
    const int nq = tl.nq[s];
    for (int Q = threadIdx.x; Q < nq; Q += blockDim.x) {
      const int lane = Q & 31, u = Q >> 5;
      int a, b;
      if (s < P && s >= e) {  // cross-lane: rotations base + 2u, base + 2u + 1
        const int m = 1 << (s - e);
        const int i_lo = (lane & ~m) * E;
        a = rot_index(i_lo, s) + 2 * u;
        b = a + 1;
      } else if (s == 0) {  // layout 1, pairs (q, q+1): rotations l*E/2 + 2u, +1
        a = lane * (E / 2) + 2 * u;
        b = E >= 4 ? a + 1 : a;
      } else if (s < P) {  // layout 1 in registers: the u-th even q with bit s clear
        const int q = ((u >> (s - 1)) << (s + 1)) | ((u & ((1 << (s - 1)) - 1)) << 1);
        a = lane * (E / 2) + ((q >> (s + 1)) << s) + (q & ((1 << s) - 1));
        b = a + 1;
      } else if (s == 5) {  // layout 2, stage 5: natural order
        a = 2 * Q;
        b = a + 1;
      } else {  // layout 2, s >= 6: lane l's registers q and q+1 (b = a + 32)
        const int qq = ((u >> (s - 6)) << (s - 4)) | ((u & ((1 << (s - 6)) - 1)) << 1);
        a = ((qq >> (s - 4)) << s) | ((qq & ((1 << (s - 5)) - 1)) << 5) | lane;
        b = a + 32;
      }
      out[Q] = make_float4(cst[a], cst[b], snt[a], snt[b]);
    }
  }
}

__device__ __forceinline__ float2 f2neg(float2 v) { return make_float2(-v.x, -v.y); }

// ---- layout-1 stages --------------------------------------------------------

// Stage 0: pairs (q, q+1); one rotation per pair (scalar arithmetic).
template <int E, int G, bool TR>
__device__ __forceinline__ void l1_stage0(float (&v)[G][E], const float4* __restrict__ tq, int lane) {
#pragma unroll
  for (int q = 0; q < E; q += 2) {
    const float4 qd = tq[(q >> 2) * 32 + lane];
    const bool hi = (q >> 1) & 1;
    const float c = hi ? qd.y : qd.x;
    const float s = hi ? qd.w : qd.z;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float a = v[g][q], b = v[g][q + 1];
      if (TR) {
        v[g][q] = c * a + s * b;
        v[g][q + 1] = c * b - s * a;
      } else {
        v[g][q] = c * a - s * b;
        v[g][q + 1] = s * a + c * b;
      }
    }
  }
}

// In-register stage S >= 1: pairs (q, q+2^S); q and q+1 share a packed op.
template <int E, int G, int S, bool TR>
__device__ __forceinline__ void l1_stage_reg(float (&v)[G][E], const float4* __restrict__ tq, int lane) {
  constexpr int h = 1 << S;
  int u = 0;
#pragma unroll
  for (int q = 0; q < E; q += 2) {
    if (q & h) continue;
    const float4 qd = tq[u * 32 + lane];
    ++u;
    const float2 c = make_float2(qd.x, qd.y);
    const float2 s = make_float2(qd.z, qd.w);
    const float2 ns = f2neg(s);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float2 x = make_float2(v[g][q], v[g][q + 1]);
      float2 y = make_float2(v[g][q + h], v[g][q + h + 1]);
      float2 nx, ny;
      if (TR) {
        nx = __ffma2_rn(c, x, __fmul2_rn(s, y));
        ny = __ffma2_rn(c, y, __fmul2_rn(ns, x));
      } else {
        nx = __ffma2_rn(c, x, __fmul2_rn(ns, y));
        ny = __ffma2_rn(c, y, __fmul2_rn(s, x));
      }
      v[g][q] = nx.x;
      v[g][q + 1] = nx.y;
      v[g][q + h] = ny.x;
      v[g][q + h + 1] = ny.y;
    }
  }
}

// Cross-lane stage s (e <= s <= 4): partner lane l ^ 2^(s-e), same register.
template <int E, int G, int s, bool TR>
__device__ __forceinline__ void l1_stage_cross(float (&v)[G][E], const float4* __restrict__ tq, int lane) {
  constexpr int e = Log2<E>::value;
  constexpr int m = 1 << (s - e);
  const bool upper = (lane & m) != 0;
  // own' = c*own + sg*partner with sg = (upper ? s : -s) forward, (upper ? -s : s) transposed
  const bool neg = TR ? upper : !upper;
#pragma unroll
  for (int q = 0; q < E; q += 2) {
    const float4 qd = tq[(q >> 1) * 32 + lane];
    const float2 c = make_float2(qd.x, qd.y);
    const float2 sg = neg ? make_float2(-qd.z, -qd.w) : make_float2(qd.z, qd.w);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float p0 = __shfl_xor_sync(FULL_MASK, v[g][q], m);
      const float p1 = __shfl_xor_sync(FULL_MASK, v[g][q + 1], m);
      const float2 o = __ffma2_rn(c, make_float2(v[g][q], v[g][q + 1]), __fmul2_rn(sg, make_float2(p0, p1)));
      v[g][q] = o.x;
      v[g][q + 1] = o.y;
    }
  }
}

// ---- layout-2 stages ----------------------------------------------------------

// Stage 5 in layout 2 (only when P == 5): pairs (q, q+1), rotation 32*(q/2) + l.
template <int E, int G, bool TR>
__device__ __forceinline__ void l2_stage5(float (&v)[G][E], const float4* __restrict__ tq, int lane) {
#pragma unroll
  for (int q = 0; q < E; q += 2) {
    const int r = 32 * (q >> 1) + lane;
    const float4 qd = tq[r >> 1];
    const float c = (r & 1) ? qd.y : qd.x;
    const float s = (r & 1) ? qd.w : qd.z;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float a = v[g][q], b = v[g][q + 1];
      if (TR) {
        v[g][q] = c * a + s * b;
        v[g][q + 1] = c * b - s * a;
      } else {
        v[g][q] = c * a - s * b;
        v[g][q + 1] = s * a + c * b;
      }
    }
  }
}

// Stage s >= 6 in layout 2: pairs (q, q + 2^(s-5)); q and q+1 share a packed op.
template <int E, int G, int s, bool TR>
__device__ __forceinline__ void l2_stage_reg(float (&v)[G][E], const float4* __restrict__ tq, int lane) {
  constexpr int h = 1 << (s - 5);
  int qp = 0;
#pragma unroll
  for (int q = 0; q < E; q += 2) {
    if (q & h) continue;
    const float4 qd = tq[qp * 32 + lane];
    ++qp;
    const float2 c = make_float2(qd.x, qd.y);
    const float2 sn = make_float2(qd.z, qd.w);
    const float2 ns = f2neg(sn);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float2 x = make_float2(v[g][q], v[g][q + 1]);
      float2 y = make_float2(v[g][q + h], v[g][q + h + 1]);
      float2 nx, ny;
      if (TR) {
        nx = __ffma2_rn(c, x, __fmul2_rn(sn, y));
        ny = __ffma2_rn(c, y, __fmul2_rn(ns, x));
      } else {
        nx = __ffma2_rn(c, x, __fmul2_rn(ns, y));
        ny = __ffma2_rn(c, y, __fmul2_rn(sn, x));
      }
      v[g][q] = nx.x;
      v[g][q + 1] = nx.y;
      v[g][q + h] = ny.x;
      v[g][q + h + 1] = ny.y;
    }
  }
}

// ---- stage sequences (compile-time recursion) ------------------------------------

template <class Gm, int G, int s, bool TR>
__device__ __forceinline__ void l1_stage(float (&v)[G][Gm::E], const float4* __restrict__ tq, int lane) {
  const float4* t = tq + tab_stage_offset(Gm::E, s);
  if constexpr (s == 0) {
    l1_stage0<Gm::E, G, TR>(v, t, lane);
  } else if constexpr (s < Gm::e) {
    l1_stage_reg<Gm::E, G, s, TR>(v, t, lane);
  } else {
    l1_stage_cross<Gm::E, G, s, TR>(v, t, lane);
  }
}
template <class Gm, int G, int s, bool TR>
__device__ __forceinline__ void l2_stage(float (&v)[G][Gm::E], const float4* __restrict__ tq, int lane) {
  const float4* t = tq + tab_stage_offset(Gm::E, s);
  if constexpr (s == 5) {
    l2_stage5<Gm::E, G, TR>(v, t, lane);
  } else {
    l2_stage_reg<Gm::E, G, s, TR>(v, t, lane);
  }
}

// forward: layout-1 stages 0..P-1 ascending
template <class Gm, int G, int s>
__device__ __forceinline__ void l1_fwd(float (&v)[G][Gm::E], const float4* tq, int lane) {
  if constexpr (s < Gm::P) {
    l1_stage<Gm, G, s, false>(v, tq, lane);
    l1_fwd<Gm, G, s + 1>(v, tq, lane);
  }
}
// forward: layout-2 stages P..L-1 ascending
template <class Gm, int G, int s>
__device__ __forceinline__ void l2_fwd(float (&v)[G][Gm::E], const float4* tq, int lane) {
  if constexpr (s < Gm::L) {
    l2_stage<Gm, G, s, false>(v, tq, lane);
    l2_fwd<Gm, G, s + 1>(v, tq, lane);
  }
}
// transposed: layout-2 stages L-1..P descending
template <class Gm, int G, int s>
__device__ __forceinline__ void l2_tr(float (&v)[G][Gm::E], const float4* tq, int lane) {
  if constexpr (s >= Gm::P) {
    l2_stage<Gm, G, s, true>(v, tq, lane);
    l2_tr<Gm, G, s - 1>(v, tq, lane);
  }
}
// transposed: layout-1 stages P-1..0 descending
template <class Gm, int G, int s>
__device__ __forceinline__ void l1_tr(float (&v)[G][Gm::E], const float4* tq, int lane) {
  if constexpr (s >= 0) {
    l1_stage<Gm, G, s, true>(v, tq, lane);
    l1_tr<Gm, G, s - 1>(v, tq, lane);
  }
}

// ---- layout switch through shared memory -------------------------------------------
__device__ __forceinline__ int swz(int i) { return i ^ (((i >> 5) & 7) << 2); }

template <int E>
__device__ __forceinline__ void to_layout2(float (&r)[E], float* buf, int lane) {
  if constexpr (E >= 4) {
#pragma unroll
    for (int u = 0; u < E / 4; ++u) {
      const int i = lane * E + 4 * u;
      *reinterpret_cast<float4*>(buf + swz(i)) = make_float4(r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3]);
    }
  } else {
#pragma unroll
    for (int q = 0; q < E; ++q) buf[swz(lane * E + q)] = r[q];
  }
  __syncwarp();
#pragma unroll
  for (int q = 0; q < E; ++q) r[q] = buf[swz(q * 32 + lane)];
  __syncwarp();
}

template <int E>
__device__ __forceinline__ void to_layout1(float (&r)[E], float* buf, int lane) {
#pragma unroll
  for (int q = 0; q < E; ++q) buf[swz(q * 32 + lane)] = r[q];
  __syncwarp();
  if constexpr (E >= 4) {
#pragma unroll
    for (int u = 0; u < E / 4; ++u) {
      const float4 t = *reinterpret_cast<const float4*>(buf + swz(lane * E + 4 * u));
      r[4 * u] = t.x;
      r[4 * u + 1] = t.y;
      r[4 * u + 2] = t.z;
      r[4 * u + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int q = 0; q < E; ++q) r[q] = buf[swz(lane * E + q)];
  }
  __syncwarp();
}

// The same switches through a buffer of only D/2 floats, one half of the row
// at a time.  Half h of the elements (indices [h*16E, (h+1)*16E)) is held by
// lanes 16h..16h+15 in layout 1 and by registers [h*E/2, (h+1)*E/2) of every
// lane in layout 2; t keeps the values that the first pass moved until the
// second pass no longer needs the registers they land in.
template <int E>
__device__ __forceinline__ void to_layout2_halves(float (&r)[E], float* buf, int lane) {
  static_assert(E >= 8, "vector stores of four");
  constexpr int H = E / 2;
  float t[H];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if ((lane >> 4) == h) {
#pragma unroll
      for (int u = 0; u < E / 4; ++u) {
        const int i = (lane & 15) * E + 4 * u;
        *reinterpret_cast<float4*>(buf + swz(i)) = make_float4(r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3]);
      }
    }
    __syncwarp();
#pragma unroll
    for (int q = 0; q < H; ++q) {
      const float val = buf[swz(q * 32 + lane)];
      if (h == 0) t[q] = val; else r[H + q] = val;
    }
    __syncwarp();
  }
#pragma unroll
  for (int q = 0; q < H; ++q) r[q] = t[q];
}

template <int E>
__device__ __forceinline__ void to_layout1_halves(float (&r)[E], float* buf, int lane) {
  static_assert(E >= 8, "vector loads of four");
  constexpr int H = E / 2;
  float t[H];
#pragma unroll
  for (int q = 0; q < H; ++q) t[q] = r[H + q];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int q = 0; q < H; ++q) buf[swz(q * 32 + lane)] = h == 0 ? r[q] : t[q];
    __syncwarp();
    if ((lane >> 4) == h) {
#pragma unroll
      for (int u = 0; u < E / 4; ++u) {
        const float4 v4 = *reinterpret_cast<const float4*>(buf + swz((lane & 15) * E + 4 * u));
        r[4 * u] = v4.x;
        r[4 * u + 1] = v4.y;
        r[4 * u + 2] = v4.z;
        r[4 * u + 3] = v4.w;
      }
    }
    __syncwarp();
  }
}

// ---- kernels: persistent warps, rows double-buffered in shared memory ----------
//
// The bucket positions are cut into groups of G consecutive positions.  The
// grid is sized to what stays resident; CTA b takes an even, contiguous range
// of groups and its warp w takes groups w, w + WARPS, w + 2*WARPS, ... of that
// range, so the warps of a CTA work on neighbouring positions (mostly one
// expert, whose cos/sin table they share through L1).  A warp first reads the
// ids, experts and gates of all its rows (lane l holds row l % G of its group
// l / G), then walks its groups with two shared-memory row buffers: while it
// rotates group j, cp.async brings in group j + 1.  A group whose rows share
// one expert is rotated together (G rows per cos/sin load); a mixed or partial
// group row by row.  No CTA-wide barrier is used.

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 16-byte chunk c of a staged row sits at chunk c ^ ((c >> 3) & 7): layout-1
// reads of 8 lanes then hit 8 different bank groups.
__device__ __forceinline__ int chunk_swz(int c) { return c ^ ((c >> 3) & 7); }

// HALVES: whether a staging buffer of half a float32 row may hold the
// transpose buffer (layout switches in two halves); the pre-rotation gains
// from it at d = 2048 (2775 -> 2512 us), the post-rotation does not.
template <int E, typename Tin, bool HALVES = true>
struct StagedCfg {
  using Gm = Geo<E>;
  static constexpr int G = Gm::G;
  static constexpr int THREADS = Gm::WARPS * 32;
  static constexpr size_t TAB_QUADS = tab_quads(E);
  static constexpr int MIN_BLOCKS = E <= 32 ? 2 : 1;
  static constexpr int MAXJ = 32 / G;  // groups per warp (one row's metadata per lane)
  // per warp: two buffers of G staged rows, and a float32 transpose buffer.
  // Once a group's rows are in registers its staging buffer is free until
  // the group after next is fetched, so the transpose buffer lives there when
  // it fits; the shared memory saved is left to L1, which holds the cos/sin
  // tables.
  static constexpr size_t BUF_BYTES = G * Gm::D * sizeof(Tin);
  // (at d = 512 the tables fit in L1 anyway, and the register-resident group
  // walk below costs spills there: 33 -> 36 us pre, 37 -> 47 us post)
  static constexpr bool TBUF_IN_STAGE = E >= 32 && E <= 64 && BUF_BYTES >= Gm::D * (HALVES ? 2 : 4);
  // a staging buffer of half a float32 row (one bf16 row) switches layouts in halves
  static constexpr bool TBUF_HALVES = TBUF_IN_STAGE && BUF_BYTES < Gm::D * 4;
  static constexpr size_t WARP_BYTES = 2 * BUF_BYTES + (TBUF_IN_STAGE ? 0 : Gm::D * 4);
  static constexpr size_t SMEM = Gm::WARPS * WARP_BYTES;
};

// Grid for `groups` groups when `resident` CTAs fit on the device at once.
// A warp takes at most MAXJ groups, so `need` CTAs at least; the grid is a
// whole number of full waves of `resident` CTAs (no partly filled last wave),
// and no larger than one group per warp.
template <int E, typename Tin, bool HALVES = true>
__host__ inline int staged_grid(long long groups, int resident) {
  using C = StagedCfg<E, Tin, HALVES>;
  const long long per = static_cast<long long>(C::Gm::WARPS);
  const long long res = resident > 0 ? resident : 1;
  long long g = (groups + per - 1) / per;                               // one group per warp at most
  const long long need = (groups + per * C::MAXJ - 1) / (per * C::MAXJ);  // MAXJ groups per warp at least
  const long long want = (need + res - 1) / res * res;
  if (g > want) g = want;
  return static_cast<int>(g < 1 ? 1 : g);
}

// The groups of warp w of this CTA: gb0 + w + WARPS*j for j < nj.
struct WarpGroups {
  long long gb0;
  int nj;
};
template <int WARPS>
__device__ __forceinline__ WarpGroups warp_groups(long long groups, int w) {
  const long long gb0 = blockIdx.x * groups / gridDim.x, gb1 = (blockIdx.x + 1) * groups / gridDim.x;
  const long long n = gb1 - gb0 - w;
  return WarpGroups{gb0, n > 0 ? static_cast<int>((n + WARPS - 1) / WARPS) : 0};
}

struct RowMeta {
  int row;    // routed row r = t*k + j (or -1)
  int ex;     // expert (or -1)
  float gate;
};

// Row metadata of bucket position p: its row, expert and gate.
__device__ __forceinline__ RowMeta fetch_row_meta(const int32_t* __restrict__ rows, const int32_t* __restrict__ idx,
                                                  const float* __restrict__ gates, long long p, long long R, int N) {
  RowMeta m{-1, -1, 0.f};
  if (p < R) {
    const int r = rows[p];
    if (r >= 0 && r < R) {
      const int e = idx[r];
      if (e >= 0 && e < N) m = RowMeta{r, e, gates ? gates[r] : 0.f};
    }
    if (m.ex < 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(p));
  }
  return m;
}

__device__ __forceinline__ RowMeta shfl_meta(const RowMeta& m, int src) {
  return RowMeta{__shfl_sync(FULL_MASK, m.row, src), __shfl_sync(FULL_MASK, m.ex, src),
                 __shfl_sync(FULL_MASK, m.gate, src)};
}

// G staged rows (natural order) into registers, layout 2.
template <class Gm, int G, typename Tin>
__device__ __forceinline__ void load_rows_l2(const Tin* xs0, float (&v)[G][Gm::E], int lane) {
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int q = 0; q < Gm::E; ++q) v[g][q] = to_f32(xs0[g * Gm::D + q * 32 + lane]);
}

template <class Gm, int G, typename Tout, bool HALVES = false>
__device__ __forceinline__ void pre_rotate_regs(float (&v)[G][Gm::E], const float4* tq, Tout* __restrict__ dst0,
                                                float* buf, int lane) {
  constexpr int E = Gm::E;
  l2_tr<Gm, G, Gm::L - 1>(v, tq, lane);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if constexpr (HALVES) to_layout1_halves<E>(v[g], buf, lane);
    else to_layout1<E>(v[g], buf, lane);
  }
  l1_tr<Gm, G, Gm::P - 1>(v, tq, lane);
#pragma unroll
  for (int g = 0; g < G; ++g) store_row<E, Tout>(dst0 + static_cast<size_t>(g) * Gm::D + lane * E, v[g], true);
}

template <class Gm, int G, typename Tin, typename Tout>
__device__ __forceinline__ void pre_rotate_rows_smem(const Tin* xs0, const float4* tq, Tout* __restrict__ dst0,
                                                     float* buf, int lane) {
  float v[G][Gm::E];
  load_rows_l2<Gm, G, Tin>(xs0, v, lane);
  pre_rotate_regs<Gm, G, Tout>(v, tq, dst0, buf, lane);
}

// Row 0 of v <- row 1 <- ... (static register moves), for walking a group
// row by row without indexing the register array.
template <int G, int E>
__device__ __forceinline__ void shift_rows(float (&v)[G][E]) {
#pragma unroll
  for (int h = 0; h + 1 < G; ++h)
#pragma unroll
    for (int q = 0; q < E; ++q) v[h][q] = v[h + 1][q];
}

// xrot[p] = B(theta_e)^T x_t for bucket positions p (row r = rows[p],
// t = r / k, e = idx[r]).
template <int E, typename Tin, typename Tout>
__global__ __launch_bounds__(StagedCfg<E, Tin>::THREADS, StagedCfg<E, Tin>::MIN_BLOCKS) void pre_rotate_fast_kernel(
    const Tin* __restrict__ x, const int32_t* __restrict__ idx, const int32_t* __restrict__ rows,
    const float4* __restrict__ quads, long long R, int k, int N, Tout* __restrict__ xrot) {
  pdl_wait();
  pdl_trigger();
  using C = StagedCfg<E, Tin>;
  using Gm = typename C::Gm;
  constexpr int G = C::G, D = Gm::D;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const long long groups = (R + G - 1) / G;
  const WarpGroups wg = warp_groups<Gm::WARPS>(groups, w);
  if (wg.nj == 0) return;
  if (wg.nj > C::MAXJ) {  // the host sizes the grid so that this cannot happen
    if (lane == 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(wg.nj));
    return;
  }
  uint8_t* wbase = smem_raw + w * C::WARP_BYTES;
  Tin* xs = reinterpret_cast<Tin*>(wbase);
  float* tbuf = reinterpret_cast<float*>(wbase + 2 * C::BUF_BYTES);
  auto pos0 = [&](int j) { return (wg.gb0 + w + static_cast<long long>(Gm::WARPS) * j) * G; };

  const int jl = lane / G;
  const RowMeta mine = jl < wg.nj ? fetch_row_meta(rows, idx, nullptr, pos0(jl) + lane % G, R, N)
                                  : RowMeta{-1, -1, 0.f};
  const int my_tok = mine.row >= 0 ? mine.row / k : 0;  // invalid rows read token 0; output zeroed

  constexpr int CH = D * sizeof(Tin) / 16;  // 16-byte chunks per row; G*CH is a multiple of 32
  auto issue = [&](int j) {
    uint8_t* dst = reinterpret_cast<uint8_t*>(xs) + (j & 1) * C::BUF_BYTES;
#pragma unroll 4
    for (int i = lane; i < G * CH; i += 32) {
      const int g = i / CH, c = i % CH;
      const int t = __shfl_sync(FULL_MASK, my_tok, j * G + g);
      cp_async16(dst + static_cast<size_t>(g) * D * sizeof(Tin) + c * 16,
                 reinterpret_cast<const uint8_t*>(x + static_cast<size_t>(t) * D) + c * 16);
    }
    cp_async_commit();
  };

  issue(0);
#pragma unroll 1
  for (int j = 0; j < wg.nj; ++j) {
    if (j + 1 < wg.nj) {
      issue(j + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    Tin* cur = xs + (j & 1) * G * D;
    const long long p0 = pos0(j);
    const int e0 = __shfl_sync(FULL_MASK, mine.ex, j * G);
    const unsigned gm = ((1u << G) - 1u) << (j * G);
    const unsigned same = __ballot_sync(FULL_MASK, mine.ex >= 0 && mine.ex == e0) & gm;
    if constexpr (C::TBUF_IN_STAGE) {
      // the whole group goes to registers first; its staging buffer then
      // serves as the transpose buffer, and a mixed group is walked row by
      // row in registers
      float* buf = reinterpret_cast<float*>(cur);
      float v[G][E];
      load_rows_l2<Gm, G, Tin>(cur, v, lane);
      __syncwarp();  // all lanes have read the staged rows before buf (which aliases them) is written
      if (same == gm && p0 + G <= R) {
        pre_rotate_regs<Gm, G, Tout, C::TBUF_HALVES>(v, quads + static_cast<size_t>(e0) * C::TAB_QUADS, xrot + p0 * D, buf, lane);
      } else {
#pragma unroll 1
        for (int g = 0; g < G; ++g) {
          const long long p = p0 + g;
          if (p >= R) break;
          const int e = __shfl_sync(FULL_MASK, mine.ex, j * G + g);
          float v1[1][E];
#pragma unroll
          for (int q = 0; q < E; ++q) v1[0][q] = e < 0 ? 0.f : v[0][q];
          if (e < 0) {
            store_row<E, Tout>(xrot + p * D + lane * E, v1[0], true);
          } else {
            pre_rotate_regs<Gm, 1, Tout, C::TBUF_HALVES>(v1, quads + static_cast<size_t>(e) * C::TAB_QUADS, xrot + p * D, buf, lane);
          }
          shift_rows<G, E>(v);
        }
      }
    } else {
      if (same == gm && p0 + G <= R) {
        pre_rotate_rows_smem<Gm, G, Tin, Tout>(cur, quads + static_cast<size_t>(e0) * C::TAB_QUADS, xrot + p0 * D,
                                               tbuf, lane);
      } else {
#pragma unroll 1
        for (int g = 0; g < G; ++g) {
          const long long p = p0 + g;
          if (p >= R) break;
          const int e = __shfl_sync(FULL_MASK, mine.ex, j * G + g);
          if (e < 0) {
            float z[E];
#pragma unroll
            for (int q = 0; q < E; ++q) z[q] = 0.f;
            store_row<E, Tout>(xrot + p * D + lane * E, z, true);
            continue;
          }
          pre_rotate_rows_smem<Gm, 1, Tin, Tout>(cur + g * D, quads + static_cast<size_t>(e) * C::TAB_QUADS,
                                                 xrot + p * D, tbuf, lane);
        }
      }
    }
    __syncwarp();  // buffer j & 1 is refilled by issue(j + 2)
  }
}

// G staged rows (16-byte chunks swizzled by chunk_swz) into registers, layout 1.
template <class Gm, int G, typename Tz>
__device__ __forceinline__ void load_rows_l1(const Tz* zs0, float (&v)[G][Gm::E], int lane) {
  constexpr int E = Gm::E;
  constexpr int PER = 16 / sizeof(Tz);  // elements per 16-byte chunk
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint8_t* zr = reinterpret_cast<const uint8_t*>(zs0 + g * Gm::D);
    if constexpr (E % PER == 0) {
#pragma unroll
      for (int u = 0; u < E / PER; ++u) {
        const uint4 raw = *reinterpret_cast<const uint4*>(zr + 16 * chunk_swz(lane * (E / PER) + u));
        const Tz* t = reinterpret_cast<const Tz*>(&raw);
#pragma unroll
        for (int j = 0; j < PER; ++j) v[g][u * PER + j] = to_f32(t[j]);
      }
    } else {
#pragma unroll
      for (int q = 0; q < E; ++q) {
        const int i = lane * E + q;
        v[g][q] = to_f32(*reinterpret_cast<const Tz*>(zr + 16 * chunk_swz(i / PER) + (i % PER) * sizeof(Tz)));
      }
    }
  }
}

// meta_of(g): row and gate of row g of the group.  At d <= 512 each row
// leaves straight from layout 2 (a warp store covers 32 consecutive
// elements: two whole sectors in bf16); from d = 1024 on it goes through the
// transpose buffer in natural order and leaves as 16-byte stores, which
// measured faster there.
template <class Gm, int G, typename Ts, bool HALVES = false, class MetaOf>
__device__ __forceinline__ void post_rotate_regs(float (&v)[G][Gm::E], const float4* tq, MetaOf meta_of,
                                                 Ts* __restrict__ slot, float* buf, int lane) {
  constexpr int E = Gm::E;
  l1_fwd<Gm, G, 0>(v, tq, lane);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if constexpr (HALVES) to_layout2_halves<E>(v[g], buf, lane);
    else to_layout2<E>(v[g], buf, lane);
  }
  l2_fwd<Gm, G, Gm::P>(v, tq, lane);
  if constexpr (E <= 16) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const RowMeta mg = meta_of(g);
      Ts* dst = slot + static_cast<size_t>(mg.row) * Gm::D + lane;
#pragma unroll
      for (int q = 0; q < E; ++q) dst[q * 32] = from_f32<Ts>(mg.gate * v[g][q]);
    }
  } else {
    constexpr int NCH = Gm::D * static_cast<int>(sizeof(Ts)) / 16;  // 16-byte chunks per row
    Ts* row_buf = reinterpret_cast<Ts*>(buf);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const RowMeta mg = meta_of(g);
#pragma unroll
      for (int q = 0; q < E; ++q) row_buf[q * 32 + lane] = from_f32<Ts>(mg.gate * v[g][q]);
      __syncwarp();
      uint4* dst = reinterpret_cast<uint4*>(slot + static_cast<size_t>(mg.row) * Gm::D);
      const uint4* src = reinterpret_cast<const uint4*>(row_buf);
#pragma unroll
      for (int c = lane; c < NCH; c += 32) dst[c] = src[c];
      __syncwarp();
    }
  }
}

template <class Gm, int G, typename Tz, typename Ts, class MetaOf>
__device__ __forceinline__ void post_rotate_rows_smem(const Tz* zs0, const float4* tq, MetaOf meta_of,
                                                      Ts* __restrict__ slot, float* buf, int lane) {
  float v[G][Gm::E];
  load_rows_l1<Gm, G, Tz>(zs0, v, lane);
  post_rotate_regs<Gm, G, Ts>(v, tq, meta_of, slot, buf, lane);
}

// slot[r] = g_r * B(phi_e) z_p for bucket positions p (z already scaled by
// alpha), r = rows[p], e = idx[r].
template <int E, typename Tz, typename Ts>
__global__ __launch_bounds__(StagedCfg<E, Tz, false>::THREADS, StagedCfg<E, Tz, false>::MIN_BLOCKS) void post_rotate_fast_kernel(
    const Tz* __restrict__ z, const int32_t* __restrict__ idx, const float* __restrict__ gates,
    const int32_t* __restrict__ rows, const float4* __restrict__ quads, long long R, int N, Ts* __restrict__ slot) {
  pdl_wait();
  pdl_trigger();
  using C = StagedCfg<E, Tz, false>;
  using Gm = typename C::Gm;
  constexpr int G = C::G, D = Gm::D;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const long long groups = (R + G - 1) / G;
  const WarpGroups wg = warp_groups<Gm::WARPS>(groups, w);
  if (wg.nj == 0) return;
  if (wg.nj > C::MAXJ) {  // the host sizes the grid so that this cannot happen
    if (lane == 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(wg.nj));
    return;
  }
  uint8_t* wbase = smem_raw + w * C::WARP_BYTES;
  Tz* zs = reinterpret_cast<Tz*>(wbase);
  float* tbuf = reinterpret_cast<float*>(wbase + 2 * C::BUF_BYTES);
  auto pos0 = [&](int j) { return (wg.gb0 + w + static_cast<long long>(Gm::WARPS) * j) * G; };

  const int jl = lane / G;
  const RowMeta mine = jl < wg.nj ? fetch_row_meta(rows, idx, gates, pos0(jl) + lane % G, R, N)
                                  : RowMeta{-1, -1, 0.f};

  constexpr int CH = D * sizeof(Tz) / 16;  // 16-byte chunks per row; G*CH is a multiple of 32
  auto issue = [&](int j) {
    uint8_t* dst = reinterpret_cast<uint8_t*>(zs) + (j & 1) * C::BUF_BYTES;
    const long long p0 = pos0(j);
#pragma unroll 4
    for (int i = lane; i < G * CH; i += 32) {
      const int g = i / CH, c = i % CH;
      const long long p = p0 + g < R ? p0 + g : R - 1;
      cp_async16(dst + static_cast<size_t>(g) * D * sizeof(Tz) + 16 * chunk_swz(c),
                 reinterpret_cast<const uint8_t*>(z + p * D) + 16 * c);
    }
    cp_async_commit();
  };

  issue(0);
#pragma unroll 1
  for (int j = 0; j < wg.nj; ++j) {
    if (j + 1 < wg.nj) {
      issue(j + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    Tz* cur = zs + (j & 1) * G * D;
    const long long p0 = pos0(j);
    const int e0 = __shfl_sync(FULL_MASK, mine.ex, j * G);
    const unsigned gm = ((1u << G) - 1u) << (j * G);
    const unsigned same = __ballot_sync(FULL_MASK, mine.ex >= 0 && mine.ex == e0) & gm;
    if constexpr (C::TBUF_IN_STAGE) {
      // as in the pre-rotation: group in registers, staging buffer reused
      float* buf = reinterpret_cast<float*>(cur);
      float v[G][E];
      load_rows_l1<Gm, G, Tz>(cur, v, lane);
      __syncwarp();  // all lanes have read the staged rows before buf (which aliases them) is written
      if (same == gm && p0 + G <= R) {
        const float4* tq = quads + static_cast<size_t>(e0) * C::TAB_QUADS;
        if constexpr (E <= 32) {  // metadata fetched at the store: fewer live registers
          post_rotate_regs<Gm, G, Ts, C::TBUF_HALVES>(
              v, tq, [&](int g) { return shfl_meta(mine, j * G + g); }, slot, buf, lane);
        } else {
          RowMeta m[G];
#pragma unroll
          for (int g = 0; g < G; ++g) m[g] = shfl_meta(mine, j * G + g);
          post_rotate_regs<Gm, G, Ts, C::TBUF_HALVES>(v, tq, [&](int g) { return m[g]; }, slot, buf, lane);
        }
      } else {
#pragma unroll 1
        for (int g = 0; g < G; ++g) {
          if (p0 + g >= R) break;
          const RowMeta m1[1] = {shfl_meta(mine, j * G + g)};
          if (m1[0].ex >= 0) {
            float v1[1][E];
#pragma unroll
            for (int q = 0; q < E; ++q) v1[0][q] = v[0][q];
            post_rotate_regs<Gm, 1, Ts, C::TBUF_HALVES>(v1, quads + static_cast<size_t>(m1[0].ex) * C::TAB_QUADS,
                                                        [&](int) { return m1[0]; }, slot, buf, lane);
          }
          shift_rows<G, E>(v);
        }
      }
    } else {
      if (same == gm && p0 + G <= R) {
        const float4* tq = quads + static_cast<size_t>(e0) * C::TAB_QUADS;
        if constexpr (E <= 32) {  // metadata fetched at the store: fewer live registers
          post_rotate_rows_smem<Gm, G, Tz, Ts>(cur, tq, [&](int g) { return shfl_meta(mine, j * G + g); }, slot, tbuf,
                                               lane);
        } else {
          RowMeta m[G];
#pragma unroll
          for (int g = 0; g < G; ++g) m[g] = shfl_meta(mine, j * G + g);
          post_rotate_rows_smem<Gm, G, Tz, Ts>(cur, tq, [&](int g) { return m[g]; }, slot, tbuf, lane);
        }
      } else {
#pragma unroll 1
        for (int g = 0; g < G; ++g) {
          if (p0 + g >= R) break;
          const RowMeta m1[1] = {shfl_meta(mine, j * G + g)};
          if (m1[0].ex < 0) continue;
          post_rotate_rows_smem<Gm, 1, Tz, Ts>(cur + g * D, quads + static_cast<size_t>(m1[0].ex) * C::TAB_QUADS,
                                               [&](int) { return m1[0]; }, slot, tbuf, lane);
        }
      }
    }
    __syncwarp();  // buffer j & 1 is refilled by issue(j + 2)
  }
}

}  // namespace bfmoe
