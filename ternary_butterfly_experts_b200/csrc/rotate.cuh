// Butterfly rotations of routed rows (ButterflyMoE technical summary, 2.3:
// B(theta)^T on the input side, B(phi) on the output side).
//
// Layout: one warp per routed row; lane l holds the E = max(1, d/32)
// consecutive elements [l*E, l*E + E) in registers.  A stage with stride
// h < E pairs two registers of one lane; a stage with h >= E pairs the same
// register of lanes l and l ^ (h/E) (one shuffle per element).
//
// Stage s rotates (i, i + 2^s) for i with bit s clear by the angle of
// rotation r(i) = (i >> (s+1)) * 2^s + (i & (2^s - 1)), with the block
// [[c, -s], [s, c]]; B applies stages 0 .. L-1, B^T applies L-1 .. 0 with the
// block transposed.  cos and sin come from a table built once per call.
#pragma once
#include "common.cuh"

namespace bfmoe {

__global__ void rot_table_kernel(const float* __restrict__ ang, long long n, float2* __restrict__ cs) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float s, c;
    sincosf(ang[i], &s, &c);
    cs[i] = make_float2(c, s);
  }
}

// Stage S with stride below E: both elements of a pair live in this lane.
template <int E, int S, bool TR>
__device__ __forceinline__ void stage_in_lane(float (&v)[E], const float2* __restrict__ tab_s, int lane) {
  constexpr int h = 1 << S;
  const float2* t = tab_s + lane * (E / 2);
#pragma unroll
  for (int q = 0; q < E; ++q) {
    if (q & h) continue;
    const int r_off = ((q >> (S + 1)) << S) + (q & (h - 1));
    const float2 cs = __ldg(t + r_off);
    const float a = v[q], b = v[q + h];
    if (TR) {
      v[q] = cs.x * a + cs.y * b;
      v[q + h] = cs.x * b - cs.y * a;
    } else {
      v[q] = cs.x * a - cs.y * b;
      v[q + h] = cs.y * a + cs.x * b;
    }
  }
}

// Stage s with stride h >= E: partner element in lane ^ (h/E), same register.
// Lanes holding no element (d < 32) take part in the shuffles only.
template <int E, bool TR>
__device__ __forceinline__ void stage_cross_lane(float (&v)[E], int s, const float2* __restrict__ tab_s, int lane,
                                                 bool active) {
  const int h = 1 << s;
  const int m = h / E;
  const bool upper = (lane & m) != 0;
  const int i_lo = (lane & ~m) * E;
  const int base = ((i_lo >> (s + 1)) << s) + (i_lo & (h - 1));
#pragma unroll
  for (int q = 0; q < E; ++q) {
    const float p = __shfl_xor_sync(FULL_MASK, v[q], m);
    const float2 cs = active ? __ldg(tab_s + base + q) : make_float2(1.f, 0.f);
    const float a = upper ? p : v[q];  // lower element of the pair
    const float b = upper ? v[q] : p;  // upper element
    if (TR) {
      v[q] = upper ? (cs.x * b - cs.y * a) : (cs.x * a + cs.y * b);
    } else {
      v[q] = upper ? (cs.y * a + cs.x * b) : (cs.x * a - cs.y * b);
    }
  }
}

template <int E>
struct Log2 {
  static constexpr int value = 1 + Log2<E / 2>::value;
};
template <>
struct Log2<1> {
  static constexpr int value = 0;
};

// In-lane stages S = SMAX-1 .. 0 (transposed order).
template <int E, int S>
__device__ __forceinline__ void in_lane_desc_T(float (&v)[E], const float2* __restrict__ tab, int half, int lane) {
  if constexpr (S >= 0) {
    stage_in_lane<E, S, true>(v, tab + static_cast<size_t>(S) * half, lane);
    in_lane_desc_T<E, S - 1>(v, tab, half, lane);
  }
}
// In-lane stages S = 0 .. SMAX-1 (forward order).
template <int E, int S, int SMAX>
__device__ __forceinline__ void in_lane_asc(float (&v)[E], const float2* __restrict__ tab, int half, int lane) {
  if constexpr (S < SMAX) {
    stage_in_lane<E, S, false>(v, tab + static_cast<size_t>(S) * half, lane);
    in_lane_asc<E, S + 1, SMAX>(v, tab, half, lane);
  }
}

template <int E, typename T>
__device__ __forceinline__ void load_row(const T* __restrict__ src, float (&v)[E], bool active) {
  if (!active) {
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = 0.f;
    return;
  }
  if constexpr ((E * sizeof(T)) % 16 == 0) {
    constexpr int NV = E * sizeof(T) / 16;
    constexpr int PER = 16 / sizeof(T);
#pragma unroll
    for (int u = 0; u < NV; ++u) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src) + u);
      const T* p = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int q = 0; q < PER; ++q) v[u * PER + q] = to_f32(p[q]);
    }
  } else {
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = to_f32(src[q]);
  }
}

template <int E, typename T>
__device__ __forceinline__ void store_row(T* __restrict__ dst, const float (&v)[E], bool active) {
  if (!active) return;
  if constexpr ((E * sizeof(T)) % 32 == 0) {
    // 32 bytes per store: one whole L2 sector per lane (dst is 32-byte aligned:
    // rows of 32*E elements in a 256-byte aligned workspace)
    constexpr int NV = E * sizeof(T) / 32;
    constexpr int PER = 32 / sizeof(T);
#pragma unroll
    for (int u = 0; u < NV; ++u) {
      uint32_t w[8];
      T* p = reinterpret_cast<T*>(w);
#pragma unroll
      for (int q = 0; q < PER; ++q) p[q] = from_f32<T>(v[u * PER + q]);
      asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + u * PER), "r"(w[0]),
                   "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                   : "memory");
    }
  } else if constexpr ((E * sizeof(T)) % 16 == 0) {
    constexpr int NV = E * sizeof(T) / 16;
    constexpr int PER = 16 / sizeof(T);
#pragma unroll
    for (int u = 0; u < NV; ++u) {
      uint4 raw;
      T* p = reinterpret_cast<T*>(&raw);
#pragma unroll
      for (int q = 0; q < PER; ++q) p[q] = from_f32<T>(v[u * PER + q]);
      reinterpret_cast<uint4*>(dst)[u] = raw;
    }
  } else {
#pragma unroll
    for (int q = 0; q < E; ++q) dst[q] = from_f32<T>(v[q]);
  }
}

// xrot[p] = B(theta_e)^T x_t for bucket position p, row r = rows[p],
// t = r / k, e = idx[r].
template <int E, typename Tin, typename Tout>
__global__ __launch_bounds__(256) void pre_rotate_kernel(const Tin* __restrict__ x, const int32_t* __restrict__ idx,
                                                         const int32_t* __restrict__ rows,
                                                         const float2* __restrict__ cs_theta, long long R, int k,
                                                         int d, int L, int N, Tout* __restrict__ xrot) {
  constexpr int LOG2E = Log2<E>::value;
  const int lane = threadIdx.x & 31;
  const bool active = lane * E < d;
  const int half = d / 2;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long p = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5; p < R; p += nwarps) {
    const int r = rows[p];
    int e = -1;
    bool ok = r >= 0 && r < R;
    if (ok) {
      e = idx[r];
      ok = e >= 0 && e < N;
    }
    float v[E];
    Tout* dst = xrot + static_cast<size_t>(p) * d + lane * E;
    if (!ok) {
      if (lane == 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(p));
#pragma unroll
      for (int q = 0; q < E; ++q) v[q] = 0.f;
      store_row<E, Tout>(dst, v, active);
      continue;
    }
    const int t = r / k;
    load_row<E, Tin>(x + static_cast<size_t>(t) * d + lane * E, v, active);
    const float2* tab = cs_theta + static_cast<size_t>(e) * L * half;
    for (int s = L - 1; s >= LOG2E; --s) stage_cross_lane<E, true>(v, s, tab + static_cast<size_t>(s) * half, lane, active);
    in_lane_desc_T<E, LOG2E - 1>(v, tab, half, lane);
    store_row<E, Tout>(dst, v, active);
  }
}

// slot[r] = g_r * B(phi_e) z_p for bucket position p (z already scaled by
// alpha), r = rows[p], e = idx[r].
template <int E>
__global__ __launch_bounds__(256) void post_rotate_kernel(const float* __restrict__ z, const int32_t* __restrict__ idx,
                                                          const float* __restrict__ gates,
                                                          const int32_t* __restrict__ rows,
                                                          const float2* __restrict__ cs_phi, long long R, int d,
                                                          int L, int N, float* __restrict__ slot) {
  constexpr int LOG2E = Log2<E>::value;
  const int lane = threadIdx.x & 31;
  const bool active = lane * E < d;
  const int half = d / 2;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long p = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5; p < R; p += nwarps) {
    const int r = rows[p];
    int e = -1;
    bool ok = r >= 0 && r < R;
    if (ok) {
      e = idx[r];
      ok = e >= 0 && e < N;
    }
    if (!ok) {
      if (lane == 0) report_error(BFMOE_EDEVICE_BOUNDS, static_cast<unsigned>(p));
      continue;
    }
    float v[E];
    load_row<E, float>(z + static_cast<size_t>(p) * d + lane * E, v, active);
    const float2* tab = cs_phi + static_cast<size_t>(e) * L * half;
    in_lane_asc<E, 0, LOG2E>(v, tab, half, lane);
    for (int s = LOG2E; s < L; ++s) stage_cross_lane<E, false>(v, s, tab + static_cast<size_t>(s) * half, lane, active);
    const float g = gates[r];
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] *= g;
    store_row<E, float>(slot + static_cast<size_t>(r) * d + lane * E, v, active);
  }
}

// y_t = sum_{j<k} slot[t*k + j] in slot order, in float32, rounded once.
// Each thread takes 16 bytes of every slot (VEC = 16 / sizeof(Ts) columns).
template <typename Ts, typename Tout>
__global__ __launch_bounds__(256) void combine_kernel(const Ts* __restrict__ slot, long long T, int k, int d,
                                                      Tout* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  constexpr int VEC = 16 / sizeof(Ts);
  const int dv = d / VEC;
  const long long n = T * dv;
  for (long long q = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; q < n;
       q += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = q / dv;
    const int c = static_cast<int>(q % dv) * VEC;
    const Ts* src = slot + static_cast<size_t>(t) * k * d + c;
    float acc[VEC];
#pragma unroll
    for (int u = 0; u < VEC; ++u) acc[u] = 0.f;
    for (int j = 0; j < k; ++j) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(j) * d));
      const Ts* h = reinterpret_cast<const Ts*>(&raw);
#pragma unroll
      for (int u = 0; u < VEC; ++u) acc[u] += to_f32(h[u]);
    }
    Tout* dst = y + static_cast<size_t>(t) * d + c;
    if constexpr (sizeof(Tout) == 4) {
#pragma unroll
      for (int u = 0; u < VEC; u += 4)
        *reinterpret_cast<float4*>(dst + u) = make_float4(acc[u], acc[u + 1], acc[u + 2], acc[u + 3]);
    } else {
      uint32_t pk[VEC / 2];
#pragma unroll
      for (int u = 0; u < VEC / 2; ++u) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * u], acc[2 * u + 1]);
        pk[u] = *reinterpret_cast<uint32_t*>(&b2);
      }
      if constexpr (VEC == 8) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      } else {
        *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
      }
    }
  }
}

}  // namespace bfmoe
