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
// (__ffma2_rn / __fmul2_rn): the table stores, per stage, quads
// (c_a, c_b, s_a, s_b) of the two rotations a lane pairs up.  Natural order
// (a, b) = (2j, 2j+1) for layout-1 stages and stage 5; for layout-2 stages
// s >= 6, quad qp*32 + l holds the rotations of lane l at registers q and q+1
// (b = a + 32).
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
  static constexpr int G = E_ <= 16 ? 4 : (E_ <= 32 ? 2 : 1);  // rows per warp
  static constexpr int WARPS = 8;
};

// Rotation index of element i in stage s (lower element of its pair).
__host__ __device__ __forceinline__ int rot_index(int i, int s) {
  return ((i >> (s + 1)) << s) + (i & ((1 << s) - 1));
}

// Quad table: [N][L][D/4] float4, layout described above.
__global__ void rot_quads_kernel(const float* __restrict__ ang, int N, int d, int L, float4* __restrict__ quads) {
  const int e = L - 5;
  const int P = e > 5 ? e : 5;
  const long long per_stage = d / 4;
  const long long n = static_cast<long long>(N) * L * per_stage;
  for (long long q = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; q < n;
       q += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int Q = static_cast<int>(q % per_stage);
    const int s = static_cast<int>((q / per_stage) % L);
    const long long ex = q / (per_stage * L);
    int a, b;
    if (s < P || s == 5) {
      a = 2 * Q;
      b = a + 1;
    } else {
      const int lane = Q & 31, qp = Q >> 5;
      const int qq = ((qp >> (s - 6)) << (s - 4)) | ((qp & ((1 << (s - 6)) - 1)) << 1);
      a = ((qq >> (s - 4)) << s) | ((qq & ((1 << (s - 5)) - 1)) << 5) | lane;
      b = a + 32;
    }
    const float* base = ang + (ex * L + s) * static_cast<long long>(d / 2);
    float sa, ca, sb, cb;
    sincosf(base[a], &sa, &ca);
    sincosf(base[b], &sb, &cb);
    quads[q] = make_float4(ca, cb, sa, sb);
  }
}

__device__ __forceinline__ float2 f2neg(float2 v) { return make_float2(-v.x, -v.y); }

// ---- layout-1 stages --------------------------------------------------------

// Stage 0: pairs (q, q+1); one rotation per pair (scalar arithmetic).
template <int E, int G, bool TR>
__device__ __forceinline__ void l1_stage0(float (&v)[G][E], const float4* __restrict__ tq, int lane) {
#pragma unroll
  for (int q = 0; q < E; q += 2) {
    const int r = lane * (E / 2) + (q >> 1);
    const float4 qd = __ldg(tq + (r >> 1));
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

// In-register stage S >= 1: pairs (q, q+2^S); q and q+1 share a packed op.
template <int E, int G, int S, bool TR>
__device__ __forceinline__ void l1_stage_reg(float (&v)[G][E], const float4* __restrict__ tq, int lane) {
  constexpr int h = 1 << S;
#pragma unroll
  for (int q = 0; q < E; q += 2) {
    if (q & h) continue;
    const int r = lane * (E / 2) + ((q >> (S + 1)) << S) + (q & (h - 1));
    const float4 qd = __ldg(tq + (r >> 1));
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
  const int i_lo = (lane & ~m) * E;
  const int base = rot_index(i_lo, s);
  // own' = c*own + sg*partner with sg = (upper ? s : -s) forward, (upper ? -s : s) transposed
  const bool neg = TR ? upper : !upper;
#pragma unroll
  for (int q = 0; q < E; q += 2) {
    const float4 qd = __ldg(tq + ((base + q) >> 1));
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
    const float4 qd = __ldg(tq + (r >> 1));
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
    const float4 qd = __ldg(tq + qp * 32 + lane);
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
  const float4* t = tq + static_cast<size_t>(s) * (Gm::D / 4);
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
  const float4* t = tq + static_cast<size_t>(s) * (Gm::D / 4);
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

// ---- kernels ------------------------------------------------------------------------

template <class Gm, int G, typename Tin, typename Tout>
__device__ __forceinline__ void pre_rotate_rows(const Tin* __restrict__ x, const int (&tok)[G],
                                                const float4* __restrict__ tq, Tout* __restrict__ dst0,
                                                float* buf, int lane) {
  constexpr int E = Gm::E;
  float v[G][E];
  // load in layout 2: element q*32 + lane (each warp load covers 32 consecutive elements)
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const Tin* src = x + static_cast<size_t>(tok[g]) * Gm::D + lane;
#pragma unroll
    for (int q = 0; q < E; ++q) v[g][q] = to_f32(src[q * 32]);
  }
  l2_tr<Gm, G, Gm::L - 1>(v, tq, lane);
#pragma unroll
  for (int g = 0; g < G; ++g) to_layout1<E>(v[g], buf, lane);
  l1_tr<Gm, G, Gm::P - 1>(v, tq, lane);
#pragma unroll
  for (int g = 0; g < G; ++g) store_row<E, Tout>(dst0 + static_cast<size_t>(g) * Gm::D + lane * E, v[g], true);
}

// xrot[p] = B(theta_e)^T x_t for bucket positions p (row r = rows[p],
// t = r / k, e = idx[r]); each warp takes G consecutive positions.
template <int E, typename Tin, typename Tout>
__global__ __launch_bounds__(256) void pre_rotate_fast_kernel(const Tin* __restrict__ x,
                                                              const int32_t* __restrict__ idx,
                                                              const int32_t* __restrict__ rows,
                                                              const float4* __restrict__ quads, long long R, int k,
                                                              int N, Tout* __restrict__ xrot) {
  using Gm = Geo<E>;
  constexpr int G = Gm::G;
  extern __shared__ __align__(16) float sbuf[];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float* buf = sbuf + w * Gm::D;
  const long long p0 = (static_cast<long long>(blockIdx.x) * Gm::WARPS + w) * G;
  if (p0 >= R) return;
  const size_t stage_quads = static_cast<size_t>(Gm::L) * (Gm::D / 4);
  int tok[G], ex[G];
  bool ok = true;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const long long p = p0 + g;
    tok[g] = 0;
    ex[g] = -1;
    if (p < R) {
      const int r = rows[p];
      if (r >= 0 && r < R) {
        const int e = idx[r];
        if (e >= 0 && e < N) {
          ex[g] = e;
          tok[g] = r / k;
        }
      }
      if (ex[g] < 0) ok = false;
    }
  }
  bool same = ok;
#pragma unroll
  for (int g = 1; g < G; ++g)
    if (p0 + g < R && ex[g] != ex[0]) same = false;
  if (same && p0 + G <= R) {
    pre_rotate_rows<Gm, G, Tin, Tout>(x, tok, quads + ex[0] * stage_quads, xrot + p0 * Gm::D, buf, lane);
    return;
  }
#pragma unroll 1
  for (int g = 0; g < G; ++g) {
    const long long p = p0 + g;
    if (p >= R) break;
    if (ex[g] < 0) {
      if (lane == 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(p));
      float z[E];
#pragma unroll
      for (int q = 0; q < E; ++q) z[q] = 0.f;
      store_row<E, Tout>(xrot + p * Gm::D + lane * E, z, true);
      continue;
    }
    const int t1[1] = {tok[g]};
    pre_rotate_rows<Gm, 1, Tin, Tout>(x, t1, quads + ex[g] * stage_quads, xrot + p * Gm::D, buf, lane);
  }
}

template <class Gm, int G>
__device__ __forceinline__ void post_rotate_rows(const float* __restrict__ z0, const float4* __restrict__ tq,
                                                 const int (&row)[G], const float (&gate)[G],
                                                 float* __restrict__ slot, float* buf, int lane) {
  constexpr int E = Gm::E;
  float v[G][E];
#pragma unroll
  for (int g = 0; g < G; ++g) load_row<E, float>(z0 + static_cast<size_t>(g) * Gm::D + lane * E, v[g], true);
  l1_fwd<Gm, G, 0>(v, tq, lane);
#pragma unroll
  for (int g = 0; g < G; ++g) to_layout2<E>(v[g], buf, lane);
  l2_fwd<Gm, G, Gm::P>(v, tq, lane);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float* dst = slot + static_cast<size_t>(row[g]) * Gm::D + lane;
#pragma unroll
    for (int q = 0; q < E; ++q) dst[q * 32] = gate[g] * v[g][q];
  }
}

// slot[r] = g_r * B(phi_e) z_p for bucket positions p; G positions per warp.
template <int E>
__global__ __launch_bounds__(256) void post_rotate_fast_kernel(const float* __restrict__ z,
                                                               const int32_t* __restrict__ idx,
                                                               const float* __restrict__ gates,
                                                               const int32_t* __restrict__ rows,
                                                               const float4* __restrict__ quads, long long R, int N,
                                                               float* __restrict__ slot) {
  using Gm = Geo<E>;
  constexpr int G = Gm::G;
  extern __shared__ __align__(16) float sbuf[];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float* buf = sbuf + w * Gm::D;
  const long long p0 = (static_cast<long long>(blockIdx.x) * Gm::WARPS + w) * G;
  if (p0 >= R) return;
  const size_t stage_quads = static_cast<size_t>(Gm::L) * (Gm::D / 4);
  int row[G], ex[G];
  float gate[G];
  bool ok = true;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const long long p = p0 + g;
    row[g] = 0;
    ex[g] = -1;
    gate[g] = 0.f;
    if (p < R) {
      const int r = rows[p];
      if (r >= 0 && r < R) {
        const int e = idx[r];
        if (e >= 0 && e < N) {
          ex[g] = e;
          row[g] = r;
          gate[g] = gates[r];
        }
      }
      if (ex[g] < 0) ok = false;
    }
  }
  bool same = ok;
#pragma unroll
  for (int g = 1; g < G; ++g)
    if (p0 + g < R && ex[g] != ex[0]) same = false;
  if (same && p0 + G <= R) {
    post_rotate_rows<Gm, G>(z + p0 * Gm::D, quads + ex[0] * stage_quads, row, gate, slot, buf, lane);
    return;
  }
#pragma unroll 1
  for (int g = 0; g < G; ++g) {
    const long long p = p0 + g;
    if (p >= R) break;
    if (ex[g] < 0) {
      if (lane == 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(p));
      continue;
    }
    const int r1[1] = {row[g]};
    const float g1[1] = {gate[g]};
    post_rotate_rows<Gm, 1>(z + p * Gm::D, quads + ex[g] * stage_quads, r1, g1, slot, buf, lane);
  }
}

}  // namespace bfmoe
