// Host side of the ButterflyMoE C ABI (include/bfmoe.h): argument checks,
// workspace layout, tensor maps, launch tracing and the order of the kernels.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "backward.cuh"
#include "bucket.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "fused_tc.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "materialize.cuh"
#include "pack.cuh"
#include "rotate.cuh"
#include "rotate_fast.cuh"
#include "router.cuh"
#include "router_tc.cuh"

using namespace bfmoe;

namespace {

thread_local char g_last_error[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}
int ok() {
  g_last_error[0] = '\0';
  return BFMOE_OK;
}
int cuda_fail(cudaError_t e, const char* what) {
  return fail(BFMOE_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool is_pow2(long long v) { return v > 0 && (v & (v - 1)) == 0; }
int ilog2(int v) {
  int l = 0;
  while ((1 << l) < v) ++l;
  return l;
}
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int words_per_row(int d) { return std::max(1, (d + 15) / 16); }

// ---------------------------------------------------------------------------
// Launch accounting and optional per-launch CUDA events.
// ---------------------------------------------------------------------------
std::atomic<unsigned long long> g_launches{0};
std::mutex g_prof_mu;
bool g_prof_on = false;
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

template <typename F>
cudaError_t launch(const char* name, cudaStream_t s, F&& f) {
  ProfRec rec{name, nullptr, nullptr};
  bool prof;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    prof = g_prof_on;
    if (prof) {
      rec.a = pool_event();
      rec.b = pool_event();
    }
  }
  if (prof) cudaEventRecord(rec.a, s);
  f();
  const cudaError_t e = cudaGetLastError();
  if (prof) {
    cudaEventRecord(rec.b, s);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof.push_back(rec);
  }
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return e;
}

// Launch with programmatic stream serialisation: the kernel may start while
// the previous kernel of the stream finishes; it waits for that kernel's
// results with pdl_wait() before touching global memory.
template <typename... KP, typename... A>
void pdl_launch(void (*kern)(KP...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

// Kernel attributes (dynamic shared-memory limits) are set per device: the
// first launch of a kernel on each device sets them.  `done` holds one bit
// per device and is set only after the attribute, so concurrent first calls
// both set it (the call is idempotent).
int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev & 63;
}
bool needs_attr(const std::atomic<uint64_t>& done) {
  return (done.load(std::memory_order_acquire) >> current_device() & 1u) == 0;
}
void attr_set(std::atomic<uint64_t>& done) {
  done.fetch_or(uint64_t(1) << current_device(), std::memory_order_release);
}

int grid_for(long long work, int per_block, int cap) {
  long long g = (work + per_block - 1) / per_block;
  if (g < 1) g = 1;
  if (g > cap) g = cap;
  return static_cast<int>(g);
}

// SMs of the current device (cached per device).
int sm_count() {
  static std::atomic<int> n[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  dev &= 63;
  int v = n[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (v <= 0) v = 148;
    n[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

// ---------------------------------------------------------------------------
// Workspace: router and forward share one buffer (stream-ordered).
// ---------------------------------------------------------------------------
// The weight-only tables of a layer: the cos/sin of theta and phi in the
// layouts the rotation kernels read, and the bf16 copy of the base that the
// tensor cores multiply by.  Built per call into the workspace, or once by
// bfmoe_prepare_layer into caller memory.
struct TabPlan {
  size_t theta, phi, phi_pq, w_bf16, total;
};

TabPlan make_tab_plan(int d, int N) {
  TabPlan t{};
  const int L = ilog2(d);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  // quad layout for d >= 64, (c, s) pairs below; theta's table is followed
  // directly by phi's (one launch writes both)
  const size_t tab = d >= 64 ? static_cast<size_t>(N) * tab_quads(d / 32) * sizeof(float4)
                             : static_cast<size_t>(N) * L * (d / 2) * sizeof(float2);
  t.theta = take(2 * tab);
  t.phi = t.theta + tab;
  // pair quads of phi for the fused epilogue, [N][L][d/4]
  t.phi_pq = take(d >= 64 ? static_cast<size_t>(N) * L * (d / 4) * sizeof(float4) : 0);
  t.w_bf16 = take(d >= 64 ? static_cast<size_t>(d) * d * 2 : 0);
  t.total = off;
  return t;
}

// bf16 tokens with 64 <= d <= 512: the whole expert runs in one kernel
// (fused_tc.cuh) and only the gated slots reach memory.
bool fused_path(int xdt, int d) { return xdt == BFMOE_BF16 && d >= 64 && d <= 512; }

// ---------------------------------------------------------------------------
// Workspace: router and forward share one buffer (stream-ordered).
// ---------------------------------------------------------------------------
// Positions of the padded bucket order that the fused expert kernel may
// read: every bucket rounded up to 32 rows, the whole rounded up to tiles.
long long pad_cap(long long R, int N) { return (R + 31LL * N + kGemmBM - 1) / kGemmBM * kGemmBM; }

struct Plan {
  // forward
  size_t tabs, xrot, z, slot, pad, fwd_end;
  // router
  size_t logits, chunk_counts, totals, wg_parts, unsure, rt_end;
  size_t total;
};

// The router runs on the tensor cores for bf16 tokens whose width is a whole
// number of 64-column k-blocks, else on the CUDA cores.
bool tc_router_path(int x_dtype, int d) { return x_dtype == BFMOE_BF16 && d % kGemmBK == 0; }

Plan make_plan(int d, int N, long long T, int k, int xdt) {
  Plan p{};
  const long long R = T * k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  p.tabs = take(make_tab_plan(d, N).total);
  // the bf16 tensor-core path keeps Z and the per-slot outputs in bf16; the
  // fused path writes only the slots
  const size_t inter = (xdt == BFMOE_BF16 && d >= 64) ? 2 : 4;
  if (!fused_path(xdt, d)) {
    p.xrot = take(static_cast<size_t>(R) * d * (xdt == BFMOE_BF16 ? 2 : 4));
    p.z = take(static_cast<size_t>(R) * d * inter);
  }
  p.slot = take(static_cast<size_t>(R) * d * inter);
  // padded bucket offsets, padded row map and quadrant experts (fused path)
  p.pad = take(static_cast<size_t>(N + 1) * 4 + static_cast<size_t>(pad_cap(R, N)) * 4 +
               static_cast<size_t>(pad_cap(R, N) / 32) * 4);
  p.fwd_end = off;
  off = 0;
  const long long nchunks = (R + bucket_chunk(k) - 1) / bucket_chunk(k);
  // float32 logits [T][N] (both routers keep them for the fix-up)
  p.logits = take(static_cast<size_t>(T) * N * 4);
  p.chunk_counts = take(static_cast<size_t>(std::max(1LL, nchunks)) * N * 4);
  p.totals = take(static_cast<size_t>(N) * 4);
  p.wg_parts = take(static_cast<size_t>(3) * N * d * 2);
  // tokens whose float32 shortlist needs the float64 scan: count, spare, ids
  p.unsure = take((2 + static_cast<size_t>(T)) * 4);
  p.rt_end = off;
  p.total = std::max(p.fwd_end, p.rt_end);
  return p;
}

int check_sizes(int d, int N, long long T, int k) {
  if (d < 4 || d > BFMOE_MAX_D || !is_pow2(d)) return fail(BFMOE_EINVAL, "d=%d must be a power of two in [4, %d]", d, BFMOE_MAX_D);
  if (N < 1 || N > BFMOE_MAX_EXPERTS) return fail(BFMOE_EINVAL, "n_experts=%d must be in [1, %d]", N, BFMOE_MAX_EXPERTS);
  if (k < 1 || k > BFMOE_MAX_K || k > N) return fail(BFMOE_EINVAL, "k=%d must be in [1, min(%d, N=%d)]", k, BFMOE_MAX_K, N);
  if (T < 0) return fail(BFMOE_EINVAL, "T=%lld must be >= 0", T);
  if (T * k > 0x7fffffffLL) return fail(BFMOE_EUNSUPPORTED, "T*k=%lld exceeds int32 row ids", T * k);
  return BFMOE_OK;
}
int check_dtype(int xdt) {
  if (xdt != BFMOE_F32 && xdt != BFMOE_BF16) return fail(BFMOE_EINVAL, "x_dtype=%d is not BFMOE_F32 or BFMOE_BF16", xdt);
  return BFMOE_OK;
}
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_ws(const Plan& p, void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return BFMOE_OK;
  if (!ws) return fail(BFMOE_EWORKSPACE, "workspace is NULL (%zu bytes needed)", need);
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(BFMOE_EWORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < need) return fail(BFMOE_EWORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes, need);
  (void)p;
  return BFMOE_OK;
}

// ---------------------------------------------------------------------------
// Tensor maps (driver entry point looked up through the runtime).
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Row-major bf16 [outer][inner], box [box_outer][64] with 128-byte swizzle.
bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  auto enc = tmap_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kGemmBK), box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// Dispatch helpers
// ---------------------------------------------------------------------------
template <template <int> class F, typename... A>
cudaError_t dispatch_e(int d, A&&... a) {
  switch (d) {
    case 4: case 8: case 16: case 32: return F<1>::run(std::forward<A>(a)...);
    case 64: return F<2>::run(std::forward<A>(a)...);
    case 128: return F<4>::run(std::forward<A>(a)...);
    case 256: return F<8>::run(std::forward<A>(a)...);
    case 512: return F<16>::run(std::forward<A>(a)...);
    case 1024: return F<32>::run(std::forward<A>(a)...);
    case 2048: return F<64>::run(std::forward<A>(a)...);
    case 4096: return F<128>::run(std::forward<A>(a)...);
    default: return cudaErrorInvalidValue;
  }
}

struct RotArgs {
  const void* x;
  bool bf16;
  const int32_t* idx;
  const float* gates;
  const int32_t* rows;
  const float2* cs;
  long long R;
  int k, d, L, N;
  void* out;
  const void* z;
  cudaStream_t s;
};

template <int E>
struct PreRotate {
  static cudaError_t run(const RotArgs& a) {
    const int grid = grid_for(a.R, 8, sm_count() * 16);
    return launch("pre_rotate", a.s, [&] {
      if (a.bf16)
        pre_rotate_kernel<E, __nv_bfloat16, __nv_bfloat16><<<grid, 256, 0, a.s>>>(
            static_cast<const __nv_bfloat16*>(a.x), a.idx, a.rows, a.cs, a.R, a.k, a.d, a.L, a.N,
            static_cast<__nv_bfloat16*>(a.out));
      else
        pre_rotate_kernel<E, float, float><<<grid, 256, 0, a.s>>>(static_cast<const float*>(a.x), a.idx, a.rows,
                                                                   a.cs, a.R, a.k, a.d, a.L, a.N,
                                                                   static_cast<float*>(a.out));
    });
  }
};

template <int E>
struct PostRotate {
  static cudaError_t run(const RotArgs& a) {
    const int grid = grid_for(a.R, 8, sm_count() * 16);
    return launch("post_rotate", a.s, [&] {
      post_rotate_kernel<E><<<grid, 256, 0, a.s>>>(static_cast<const float*>(a.z), a.idx, a.gates, a.rows, a.cs,
                                                   a.R, a.d, a.L, a.N, static_cast<float*>(a.out));
    });
  }
};

// CTAs of `kernel` that stay resident on the whole device (at least one per SM).
template <typename K>
int resident_ctas(K kernel, int threads, size_t smem) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  return per_sm * sm_count();
}

template <int E>
struct PreRotateFast {
  template <typename T>
  static cudaError_t go(const RotArgs& a) {
    using C = StagedCfg<E, T>;
    auto kern = pre_rotate_fast_kernel<E, T, T>;
    static std::atomic<uint64_t> done{0};
    static int resident[64] = {};
    const int dev = current_device();
    if (needs_attr(done)) {
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM));
      resident[dev] = resident_ctas(kern, C::THREADS, C::SMEM);
      attr_set(done);
    }
    const int grid = staged_grid<E, T>((a.R + C::G - 1) / C::G, resident[dev]);
    return launch("pre_rotate", a.s, [&] {
      pdl_launch(kern, grid, C::THREADS, C::SMEM, a.s, static_cast<const T*>(a.x), a.idx, a.rows,
                 reinterpret_cast<const float4*>(a.cs), a.R, a.k, a.N, static_cast<T*>(a.out));
    });
  }
  // bf16 path: x and X_rot in bf16; float32 path: float32
  static cudaError_t run(const RotArgs& a) { return a.bf16 ? go<__nv_bfloat16>(a) : go<float>(a); }
};

template <int E>
struct PostRotateFast {
  template <typename T>
  static cudaError_t go(const RotArgs& a) {
    using C = StagedCfg<E, T, false>;
    auto kern = post_rotate_fast_kernel<E, T, T>;
    static std::atomic<uint64_t> done{0};
    static int resident[64] = {};
    const int dev = current_device();
    if (needs_attr(done)) {
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM));
      resident[dev] = resident_ctas(kern, C::THREADS, C::SMEM);
      attr_set(done);
    }
    const int grid = staged_grid<E, T, false>((a.R + C::G - 1) / C::G, resident[dev]);
    return launch("post_rotate", a.s, [&] {
      pdl_launch(kern, grid, C::THREADS, C::SMEM, a.s, static_cast<const T*>(a.z), a.idx, a.gates, a.rows,
                 reinterpret_cast<const float4*>(a.cs), a.R, a.N, static_cast<T*>(a.out));
    });
  }
  // bf16 path: Z and slots in bf16; float32 path: float32
  static cudaError_t run(const RotArgs& a) { return a.bf16 ? go<__nv_bfloat16>(a) : go<float>(a); }
};

template <template <int> class F, typename... A>
cudaError_t dispatch_fast(int d, A&&... a) {
  switch (d) {
    case 64: return F<2>::run(std::forward<A>(a)...);
    case 128: return F<4>::run(std::forward<A>(a)...);
    case 256: return F<8>::run(std::forward<A>(a)...);
    case 512: return F<16>::run(std::forward<A>(a)...);
    case 1024: return F<32>::run(std::forward<A>(a)...);
    case 2048: return F<64>::run(std::forward<A>(a)...);
    case 4096: return F<128>::run(std::forward<A>(a)...);
    default: return cudaErrorInvalidValue;
  }
}

template <int BN, int STAGES>
cudaError_t launch_gemm_tc(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tbh, __nv_bfloat16* z,
                           int R, int d, float alpha, cudaStream_t s) {
  using Cfg = GemmTcCfg<BN, STAGES>;
  static std::atomic<uint64_t> done{0};
  if (needs_attr(done)) {
    cudaError_t e = cudaFuncSetAttribute(ternary_gemm_tc_kernel<BN, STAGES>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set(done);
  }
  const long long tiles = static_cast<long long>((R + kGemmBM - 1) / kGemmBM) * (d / BN);
  const int grid = static_cast<int>(std::min<long long>(tiles, sm_count()));
  return launch("ternary_gemm_tc", s, [&] {
    pdl_launch(ternary_gemm_tc_kernel<BN, STAGES>, grid, kGemmThreads, Cfg::SMEM_BYTES, s, ta, tb, tbh, z, R, d, alpha);
  });
}

template <int BN, int STAGES, int K>
cudaError_t launch_router_tc_k(const CUtensorMap& tx, const CUtensorMap& tw, const float* bias, int T, int d, int N,
                               float eps_c, float* logits, const __nv_bfloat16* x, const float* w_gate,
                               int32_t* idx, float* gates, int32_t* cc, cudaStream_t s) {
  using Cfg = RouterTcCfg<BN, STAGES>;
  static std::atomic<uint64_t> done{0};
  if (needs_attr(done)) {
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel<BN, STAGES, K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set(done);
  }
  const int grid = (T + kGemmBM - 1) / kGemmBM;
  return launch("router_tc", s, [&] {
    pdl_launch(router_tc_kernel<BN, STAGES, K>, grid, kRouterThreads, Cfg::SMEM_BYTES, s, tx, tw, bias, T, d, N,
               eps_c, logits, x, w_gate, idx, gates, cc);
  });
}

template <int BN, int STAGES>
cudaError_t launch_router_tc(const CUtensorMap& tx, const CUtensorMap& tw, const float* bias, int T, int d, int N,
                             int k, float eps_c, float* logits, const __nv_bfloat16* x, const float* w_gate,
                             int32_t* idx, float* gates, int32_t* cc, cudaStream_t s) {
  switch (k) {
    case 1: return launch_router_tc_k<BN, STAGES, 1>(tx, tw, bias, T, d, N, eps_c, logits, x, w_gate, idx, gates, cc, s);
    case 2: return launch_router_tc_k<BN, STAGES, 2>(tx, tw, bias, T, d, N, eps_c, logits, x, w_gate, idx, gates, cc, s);
    case 3: return launch_router_tc_k<BN, STAGES, 3>(tx, tw, bias, T, d, N, eps_c, logits, x, w_gate, idx, gates, cc, s);
    case 4: return launch_router_tc_k<BN, STAGES, 4>(tx, tw, bias, T, d, N, eps_c, logits, x, w_gate, idx, gates, cc, s);
    case 5: return launch_router_tc_k<BN, STAGES, 5>(tx, tw, bias, T, d, N, eps_c, logits, x, w_gate, idx, gates, cc, s);
    case 6: return launch_router_tc_k<BN, STAGES, 6>(tx, tw, bias, T, d, N, eps_c, logits, x, w_gate, idx, gates, cc, s);
    case 7: return launch_router_tc_k<BN, STAGES, 7>(tx, tw, bias, T, d, N, eps_c, logits, x, w_gate, idx, gates, cc, s);
    default: return launch_router_tc_k<BN, STAGES, 8>(tx, tw, bias, T, d, N, eps_c, logits, x, w_gate, idx, gates, cc, s);
  }
}

}  // namespace

namespace {

int check_forward_args(const bfmoe_layer* layer, const void* x, int x_dtype, int T, int k, const int32_t* idx,
                       const float* gates, const int32_t* offsets, const int32_t* rows, const void* y) {
  if (!layer) return fail(BFMOE_EINVAL, "forward: NULL layer");
  int rc = check_sizes(layer->d, layer->n_experts, T, k);
  if (rc) return rc;
  if ((rc = check_dtype(x_dtype))) return rc;
  if (T == 0) return BFMOE_OK;
  if (!layer->w_packed || !layer->theta || !layer->phi) return fail(BFMOE_EINVAL, "forward: NULL layer weights");
  if (!x || !idx || !gates || !offsets || !rows || !y) return fail(BFMOE_EINVAL, "forward: NULL pointer");
  if (!aligned16(x) || !aligned16(y)) return fail(BFMOE_EINVAL, "forward: x and y must be 16-byte aligned");
  return BFMOE_OK;
}

// The inputs of the forward that depend on the weights only (TabPlan), into
// `tabs`: the cos/sin tables of theta and phi and, from d = 64 on, phi's pair
// quads and the bf16 copy of the base for the tensor cores.
int build_weight_tables(const bfmoe_layer* layer, uint8_t* tabs, cudaStream_t s) {
  const int d = layer->d, N = layer->n_experts, L = ilog2(d);
  const TabPlan tp = make_tab_plan(d, N);
  float2* tab_t = reinterpret_cast<float2*>(tabs + tp.theta);
  float2* tab_p = reinterpret_cast<float2*>(tabs + tp.phi);
  uint16_t* wbf = reinterpret_cast<uint16_t*>(tabs + tp.w_bf16);
  const long long nang = static_cast<long long>(N) * L * (d / 2);
  cudaError_t e;
  if (d >= 64) {
    // one launch builds both quad tables (the phi table follows the theta
    // table) and the bf16 copy of the base
    const TabLayout tl = make_tab_layout(d / 32, L);
    const int tab_blocks = 2 * N;
    const int exp_blocks = grid_for(static_cast<long long>(d) * (d / 16), 256, 1024);
    const size_t tab_smem = static_cast<size_t>(L) * d * sizeof(float);  // cos and sin of one expert
    static std::atomic<uint64_t> done{0};
    if (needs_attr(done)) {
      cudaFuncSetAttribute(rot_quads_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(12 * BFMOE_MAX_D * sizeof(float)));
      attr_set(done);
    }
    e = launch("rot_table", s, [&] {
      rot_quads_kernel<<<tab_blocks + exp_blocks, 256, tab_smem, s>>>(
          layer->theta, layer->phi, N, d, L, tl, reinterpret_cast<float4*>(tab_t), layer->w_packed, wbf);
    });
    if (e == cudaSuccess)
      e = launch("rot_table", s, [&] {
        rot_pairq_kernel<<<grid_for(nang / 2, 256, 4096), 256, 0, s>>>(
            layer->phi, nang / 2, reinterpret_cast<float4*>(tabs + tp.phi_pq));
      });
  } else {
    e = launch("rot_table", s, [&] { rot_table_kernel<<<grid_for(nang, 256, 8192), 256, 0, s>>>(layer->theta, nang, tab_t); });
    if (e == cudaSuccess)
      e = launch("rot_table", s, [&] { rot_table_kernel<<<grid_for(nang, 256, 8192), 256, 0, s>>>(layer->phi, nang, tab_p); });
  }
  if (e != cudaSuccess) return cuda_fail(e, "forward: rotation tables");
  return BFMOE_OK;
}

template <int D>
cudaError_t launch_fused(const CUtensorMap& tb, const __nv_bfloat16* x, const int32_t* idx, const float* gates,
                         const int32_t* rows, const int32_t* offsets, int32_t* pad, const float4* tq,
                         const float4* pq, long long R, int k, int N, float alpha, __nv_bfloat16* slot,
                         bool pad_ready, cudaStream_t s) {
  using C = FusedCfg<D>;
  static std::atomic<uint64_t> done{0};
  if (needs_attr(done)) {
    cudaError_t e = cudaFuncSetAttribute(fused_expert_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set(done);
  }
  // the buckets padded to multiples of 32 rows, as a row map (bucket_pad_kernel)
  const long long cap = pad_cap(R, N);
  int32_t* pad_off = pad;
  int32_t* pmap = pad + (N + 1);
  int32_t* qex = pmap + cap;
  // (already written by the router's scatter when pad_ready)
  if (!pad_ready) {
    const cudaError_t e = launch("bucket_pad", s, [&] {
      const int g = grid_for(cap, 256, sm_count() * 8);
      pdl_launch(bucket_pad_kernel, g, 256, static_cast<size_t>(N + 1) * 8, s, offsets, rows, idx, R, N, cap,
                 pad_off, pmap, qex);
    });
    if (e != cudaSuccess) return e;
  }
  const int grid = static_cast<int>(std::min<long long>(cap / kGemmBM, sm_count()));
  return launch("fused_expert", s, [&] {
    pdl_launch(fused_expert_kernel<D>, grid, kFusedThreads, C::SMEM_BYTES, s, tb, x, gates,
               static_cast<const int32_t*>(pmap), static_cast<const int32_t*>(qex),
               static_cast<const int32_t*>(pad_off + N), tq, pq, k, alpha, slot);
  });
}

// Gated combine of the slots: y_t = sum_j slot[t k + j], one rounding.
cudaError_t launch_combine(bool bf16, bool fast, const void* slot, int T, int k, int d, void* y, cudaStream_t s) {
  const long long nv = static_cast<long long>(T) * (d / ((bf16 && fast) ? 8 : 4));
  return launch("combine", s, [&] {
    const int g = grid_for(nv, 256, sm_count() * 16);
    if (bf16 && fast)
      pdl_launch(combine_kernel<__nv_bfloat16, __nv_bfloat16>, g, 256, 0, s,
                 static_cast<const __nv_bfloat16*>(slot), static_cast<long long>(T), k, d,
                 static_cast<__nv_bfloat16*>(y));
    else if (bf16)
      combine_kernel<float, __nv_bfloat16><<<g, 256, 0, s>>>(static_cast<const float*>(slot), T, k, d,
                                                             static_cast<__nv_bfloat16*>(y));
    else
      combine_kernel<float, float><<<g, 256, 0, s>>>(static_cast<const float*>(slot), T, k, d, static_cast<float*>(y));
  });
}

// Pre-rotation, ternary product, post-rotation with gates, combine.  `tabs`
// holds the weight tables (TabPlan), built per call or prepared once.
int forward_body(const bfmoe_layer* layer, const void* x, bool bf16, int T, int k, const int32_t* idx,
                 const float* gates, const int32_t* offsets, const int32_t* rows, void* y, const Plan& p, uint8_t* W,
                 const uint8_t* tabs, cudaStream_t s, bool pad_ready) {
  const int d = layer->d, N = layer->n_experts, L = ilog2(d);
  const TabPlan tp = make_tab_plan(d, N);
  const float2* tab_t = reinterpret_cast<const float2*>(tabs + tp.theta);
  const float2* tab_p = reinterpret_cast<const float2*>(tabs + tp.phi);
  const uint16_t* wbf = reinterpret_cast<const uint16_t*>(tabs + tp.w_bf16);
  void* slot = W + p.slot;
  const long long R = static_cast<long long>(T) * k;
  const int wpr = words_per_row(d);
  const bool fast = d >= 64;
  cudaError_t e;

  if (fused_path(bf16 ? BFMOE_BF16 : BFMOE_F32, d)) {
    CUtensorMap tb;
    if (!make_tmap_bf16(&tb, wbf, d, d, std::min(d, 128))) return fail(BFMOE_ECUDA, "forward: tensor map encoding failed");
    const auto* xb = static_cast<const __nv_bfloat16*>(x);
    const auto* tq = reinterpret_cast<const float4*>(tab_t);
    const auto* pq = reinterpret_cast<const float4*>(tabs + tp.phi_pq);
    auto* sb = static_cast<__nv_bfloat16*>(slot);
    int32_t* pad = reinterpret_cast<int32_t*>(W + p.pad);
    switch (d) {
      case 64: e = launch_fused<64>(tb, xb, idx, gates, rows, offsets, pad, tq, pq, R, k, N, layer->alpha, sb, pad_ready, s); break;
      case 128: e = launch_fused<128>(tb, xb, idx, gates, rows, offsets, pad, tq, pq, R, k, N, layer->alpha, sb, pad_ready, s); break;
      case 256: e = launch_fused<256>(tb, xb, idx, gates, rows, offsets, pad, tq, pq, R, k, N, layer->alpha, sb, pad_ready, s); break;
      default: e = launch_fused<512>(tb, xb, idx, gates, rows, offsets, pad, tq, pq, R, k, N, layer->alpha, sb, pad_ready, s); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "forward: fused expert kernel");
    e = launch_combine(true, true, slot, T, k, d, y, s);
    if (e != cudaSuccess) return cuda_fail(e, "forward: combine");
    return ok();
  }

  void* xrot = W + p.xrot;
  void* z = W + p.z;
  RotArgs ra{x, bf16, idx, gates, rows, tab_t, R, k, d, L, N, xrot, nullptr, s};
  e = fast ? dispatch_fast<PreRotateFast>(d, ra) : dispatch_e<PreRotate>(d, ra);
  if (e != cudaSuccess) return cuda_fail(e, "forward: pre-rotation");

  if (bf16 && d >= 64) {
    CUtensorMap ta, tb, tbh;
    const int BN = std::min(d, 256);
    if (!make_tmap_bf16(&ta, xrot, d, R, kGemmBM) || !make_tmap_bf16(&tb, wbf, d, d, BN) ||
        !make_tmap_bf16(&tbh, wbf, d, d, BN >= 128 ? BN / 2 : BN))
      return fail(BFMOE_ECUDA, "forward: tensor map encoding failed");
    __nv_bfloat16* zb = static_cast<__nv_bfloat16*>(z);
    const int Ri = static_cast<int>(R);
    switch (BN) {
      case 64: e = launch_gemm_tc<64, 8>(ta, tb, tbh, zb, Ri, d, layer->alpha, s); break;
      case 128: e = launch_gemm_tc<128, 6>(ta, tb, tbh, zb, Ri, d, layer->alpha, s); break;
      default: e = launch_gemm_tc<256, 4>(ta, tb, tbh, zb, Ri, d, layer->alpha, s); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "forward: tensor-core GEMM");
  } else {
    dim3 g((R + 63) / 64, (d + 63) / 64);
    e = launch("ternary_gemm_simt", s, [&] {
      if (bf16)
        ternary_gemm_simt_kernel<__nv_bfloat16><<<g, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(xrot),
                                                                  layer->w_packed, wpr, R, d, layer->alpha,
                                                                  static_cast<float*>(z));
      else
        ternary_gemm_simt_kernel<float><<<g, 256, 0, s>>>(static_cast<const float*>(xrot), layer->w_packed, wpr, R,
                                                          d, layer->alpha, static_cast<float*>(z));
    });
    if (e != cudaSuccess) return cuda_fail(e, "forward: SIMT ternary product");
  }

  RotArgs rb{nullptr, bf16, idx, gates, rows, tab_p, R, k, d, L, N, slot, z, s};
  e = fast ? dispatch_fast<PostRotateFast>(d, rb) : dispatch_e<PostRotate>(d, rb);
  if (e != cudaSuccess) return cuda_fail(e, "forward: post-rotation");

  e = launch_combine(bf16, fast, slot, T, k, d, y, s);
  if (e != cudaSuccess) return cuda_fail(e, "forward: combine");
  return ok();
}

// One side stream (and fork/join events) per device, created on first use,
// for the weight-only work of bfmoe_moe_forward.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_side_mu;
SideStream g_side[64];

int side_stream(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "moe_forward: cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(BFMOE_EUNSUPPORTED, "moe_forward: device %d", dev);
  std::lock_guard<std::mutex> lk(g_side_mu);
  SideStream& ss = g_side[dev];
  if (!ss.stream) {
    if ((e = cudaStreamCreateWithFlags(&ss.stream, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming)) != cudaSuccess)
      return cuda_fail(e, "moe_forward: side stream");
  }
  *out = &ss;
  return BFMOE_OK;
}

// Copy streams and events of bfmoe_moe_forward_host, one set per device,
// created on first use.
constexpr int kHostMaxChunks = 64;
// `lane1` is the second compute stream: odd chunks run there, even chunks on
// the caller's stream, so that one chunk's latency-bound kernels overlap the
// next chunk's.
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr, lane1 = nullptr;
  cudaEvent_t fork = nullptr, done = nullptr, lane1_go = nullptr, lane1_done = nullptr;
  cudaEvent_t ev_in[kHostMaxChunks] = {}, ev_out[kHostMaxChunks] = {};
};
std::mutex g_pipe_mu;
HostPipe g_pipe[64];

int host_pipe(HostPipe** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "moe_forward_host: cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(BFMOE_EUNSUPPORTED, "moe_forward_host: device %d", dev);
  std::lock_guard<std::mutex> lk(g_pipe_mu);
  HostPipe& hp = g_pipe[dev];
  if (!hp.in) {
    const unsigned ef = cudaEventDisableTiming;
    if ((e = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&hp.lane1, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&hp.fork, ef)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&hp.done, ef)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&hp.lane1_go, ef)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&hp.lane1_done, ef)) != cudaSuccess)
      return cuda_fail(e, "moe_forward_host: copy streams");
    for (int i = 0; i < kHostMaxChunks; ++i)
      if ((e = cudaEventCreateWithFlags(&hp.ev_in[i], ef)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&hp.ev_out[i], ef)) != cudaSuccess)
        return cuda_fail(e, "moe_forward_host: events");
  }
  *out = &hp;
  return BFMOE_OK;
}

// Workspace of bfmoe_moe_forward_host: device x and y, and per compute lane
// (two when there are two chunks or more) one chunk's routing and one
// chunk's bfmoe_moe_forward scratch; and the chunk schedule.
struct HostPlan {
  int chunk, nchunks, lanes;
  int start[kHostMaxChunks + 1];  // chunk c = tokens start[c] .. start[c+1]-1
  size_t x_dev, y_dev, parts, total;
  size_t idx[2], gates[2], counts[2], offsets[2], rows[2], moe[2];
};

// Chunks of `chunk` tokens (the last one takes the rest).  The default is
// T / 4096 about equal chunks, at least two and at most six, of at least
// 2048 tokens.  Measured end to end on B200: every chunk's work has a fixed
// cost of about 55 us (the kernels' latency chains, nearly independent of
// the chunk's size), so the best count balances that against the copies that
// cannot overlap at the start and the end; four chunks at T = 16384, d = 512
// (0.53 ms against 0.60 with six), six at T = 65536, d = 1024.
HostPlan make_host_plan(int d, int N, int T, int k, int xdt, int chunk) {
  HostPlan h{};
  if (chunk <= 0) {
    const int want = std::min(6, std::max(2, T / 4096));
    chunk = std::max(2048, (T + want - 1) / want);
  }
  chunk = (chunk + 127) / 128 * 128;
  if (T > 0 && chunk > T) chunk = T;
  if (T > 0 && (T + chunk - 1) / chunk > kHostMaxChunks) chunk = (T + kHostMaxChunks - 1) / kHostMaxChunks;
  h.chunk = std::max(1, chunk);
  int t = 0, c = 0;
  while (t < T) {
    const int left = T - t;
    int n = left > h.chunk ? h.chunk : left;
    if (c == kHostMaxChunks - 1) n = left;  // (the clamp above already keeps c below this)
    h.start[c++] = t;
    t += n;
  }
  h.start[c] = T;
  h.nchunks = c;
  const size_t es = xdt == BFMOE_BF16 ? 2 : 4;
  const size_t rc = static_cast<size_t>(h.chunk) * k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  h.x_dev = take(static_cast<size_t>(T) * d * es);
  h.y_dev = take(static_cast<size_t>(T) * d * es);
  h.parts = take(static_cast<size_t>(3) * N * d * 2);  // W_g split once per call (tensor-core router)
  const Plan p = make_plan(d, N, h.chunk, k, xdt);
  h.lanes = h.nchunks >= 2 ? 2 : 1;
  for (int l = 0; l < h.lanes; ++l) {
    h.idx[l] = take(rc * 4);
    h.gates[l] = take(rc * 4);
    h.counts[l] = take(static_cast<size_t>(N) * 4);
    h.offsets[l] = take(static_cast<size_t>(N + 1) * 4);
    h.rows[l] = take(rc * 4);
    h.moe[l] = take(p.fwd_end + p.rt_end);
  }
  h.total = off;
  return h;
}

}  // namespace

// ---------------------------------------------------------------------------
// Fixed scratch of bfmoe_router_topk_noalloc, for callers that cannot
// allocate device memory.  In host code the array's name only stands for the
// device symbol; its device address comes from cudaGetSymbolAddress, looked
// up once per device with that device current.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[BFMOE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.
int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "router_topk_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(BFMOE_EUNSUPPORTED, "router_topk_noalloc: device %d", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "router_topk_noalloc: cudaGetSymbolAddress");
    if (!p) return fail(BFMOE_ECUDA, "router_topk_noalloc: no device address for the scratch array");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return BFMOE_OK;
}

}  // namespace

namespace {

// Workspace of bfmoe_backward.
struct BwPlan {
  size_t tab_t, tab_p, wt, U, Z, dU, dg, dl, part, dapart, total;
  int slices, ra_blocks;
};

BwPlan make_bw_plan(int d, int N, long long T, int k) {
  BwPlan b{};
  const int L = ilog2(d);
  const long long R = T * k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  const size_t tab = static_cast<size_t>(N) * L * (d / 2) * sizeof(float2);
  b.tab_t = take(tab);
  b.tab_p = take(tab);
  b.wt = take(static_cast<size_t>(d) * words_per_row(d) * 4);
  b.U = take(static_cast<size_t>(R) * d * 4);
  b.Z = take(static_cast<size_t>(R) * d * 4);  // Z, then dZ in place, then the per-row dx
  b.dU = take(static_cast<size_t>(R) * d * 4);
  b.dg = take(static_cast<size_t>(R) * 4);
  b.dl = take(static_cast<size_t>(R) * 4);
  // the outer product dZ^T U in slices of the rows, at most 64 MB of partials
  long long sl = (R + 2047) / 2048;
  const long long cap = std::max(1LL, (64LL << 20) / (static_cast<long long>(d) * d * 4));
  sl = std::max(1LL, std::min({sl, 16LL, cap}));
  b.slices = static_cast<int>(sl);
  b.part = take(static_cast<size_t>(sl) * d * d * 4);
  b.ra_blocks = grid_for(static_cast<long long>(d) * d, 256, 1024);
  b.dapart = take(static_cast<size_t>(b.ra_blocks) * 4);
  b.total = off;
  return b;
}

template <int E>
struct BwRows {
  static cudaError_t run(const void* x, bool bf16, const int32_t* idx, const int32_t* rows, const int32_t* offsets,
                         const float* gates, const float* gy, const float2* tab_t, const float2* tab_p, long long R,
                         int k, int d, int L, int N, float* U, float* Z, float* dU, float* dg, float* dtheta,
                         float* dphi, int stage, cudaStream_t s) {
    const size_t smem = static_cast<size_t>(L) * (d / 2) * sizeof(float);
    static std::atomic<uint64_t> done{0};
    if (needs_attr(done)) {
      cudaFuncSetAttribute(bw_post_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, 12 * BFMOE_MAX_D * 2);
      cudaFuncSetAttribute(bw_pre_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, 12 * BFMOE_MAX_D * 2);
      attr_set(done);
    }
    if (stage == 0) {  // u = B(theta)^T x, bucket order, float32
      const int grid = grid_for(R, 8, sm_count() * 16);
      return launch("bw_pre_rotate", s, [&] {
        if (bf16)
          pre_rotate_kernel<E, __nv_bfloat16, float><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), idx,
                                                                          rows, tab_t, R, k, d, L, N, U);
        else
          pre_rotate_kernel<E, float, float><<<grid, 256, 0, s>>>(static_cast<const float*>(x), idx, rows, tab_t, R,
                                                                  k, d, L, N, U);
      });
    }
    // CTAs per expert: about 16 rows each on average (2 per warp)
    const long long per_expert = (R + N - 1) / N;
    const dim3 grid(N, static_cast<unsigned>(std::min<long long>(64, std::max<long long>(1, (per_expert + 15) / 16))));
    const size_t ang = static_cast<size_t>(N) * L * (d / 2) * sizeof(float);
    if (stage == 1) {
      cudaError_t e = cudaMemsetAsync(dphi, 0, ang, s);
      if (e != cudaSuccess) return e;
      return launch("bw_post", s, [&] {
        bw_post_kernel<E><<<grid, 256, smem, s>>>(Z, gy, rows, offsets, gates, tab_p, d, L, k, N, R, Z, dg, dphi);
      });
    }
    cudaError_t e = cudaMemsetAsync(dtheta, 0, ang, s);
    if (e != cudaSuccess) return e;
    return launch("bw_pre", s, [&] {
      bw_pre_kernel<E><<<grid, 256, smem, s>>>(U, dU, rows, offsets, tab_t, d, L, R, Z, dtheta);
    });
  }
};

template <int E, typename... A>
cudaError_t bw_rows(int d, A&&... a) {
  (void)d;
  return BwRows<E>::run(std::forward<A>(a)...);
}

cudaError_t bw_rows_dispatch(int d, const void* x, bool bf16, const int32_t* idx, const int32_t* rows,
                             const int32_t* offsets, const float* gates, const float* gy, const float2* tab_t,
                             const float2* tab_p, long long R, int k, int L, int N, float* U, float* Z, float* dU,
                             float* dg, float* dtheta, float* dphi, int stage, cudaStream_t s) {
#define BW_ARGS x, bf16, idx, rows, offsets, gates, gy, tab_t, tab_p, R, k, d, L, N, U, Z, dU, dg, dtheta, dphi, stage, s
  switch (d) {
    case 4: case 8: case 16: case 32: return BwRows<1>::run(BW_ARGS);
    case 64: return BwRows<2>::run(BW_ARGS);
    case 128: return BwRows<4>::run(BW_ARGS);
    case 256: return BwRows<8>::run(BW_ARGS);
    case 512: return BwRows<16>::run(BW_ARGS);
    case 1024: return BwRows<32>::run(BW_ARGS);
    case 2048: return BwRows<64>::run(BW_ARGS);
    case 4096: return BwRows<128>::run(BW_ARGS);
    default: return cudaErrorInvalidValue;
  }
#undef BW_ARGS
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* bfmoe_last_error(void) { return g_last_error; }

unsigned long long bfmoe_launch_count(void) { return g_launches.load(); }

size_t bfmoe_workspace_size(int d, int n_experts, int T, int k, int x_dtype) {
  if (check_sizes(d, n_experts, T, k) != BFMOE_OK || check_dtype(x_dtype) != BFMOE_OK) return 0;
  return make_plan(d, n_experts, T, k, x_dtype).total;
}

size_t bfmoe_router_scratch_size(int d, int n_experts, int T, int k, int x_dtype) {
  if (check_sizes(d, n_experts, T, k) != BFMOE_OK || check_dtype(x_dtype) != BFMOE_OK) return 0;
  return make_plan(d, n_experts, T, k, x_dtype).rt_end;
}

int bfmoe_pack_base(const int8_t* w, int d, uint32_t* w_packed, bfmoe_stream_t stream) {
  if (!w || !w_packed) return fail(BFMOE_EINVAL, "pack_base: NULL pointer");
  if (d < 4 || d > BFMOE_MAX_D || !is_pow2(d)) return fail(BFMOE_EINVAL, "pack_base: bad d=%d", d);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const unsigned zero = 0;
  cudaError_t e = cudaMemcpyToSymbolAsync(g_not_ternary, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "pack_base: reset flag");
  const int wpr = words_per_row(d);
  const long long n = static_cast<long long>(d) * wpr;
  e = launch("pack_base", s, [&] { pack_base_kernel<<<grid_for(n, 256, 4096), 256, 0, s>>>(w, d, wpr, w_packed); });
  if (e != cudaSuccess) return cuda_fail(e, "pack_base: launch");
  unsigned bad = 0;
  e = cudaMemcpyFromSymbolAsync(&bad, g_not_ternary, sizeof(bad), 0, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "pack_base: read flag");
  if (bad) return fail(BFMOE_ENOT_TERNARY, "pack_base: a weight is outside {-1, 0, +1}");
  return ok();
}

int bfmoe_unpack_base(const uint32_t* w_packed, int d, uint16_t* w_bf16, bfmoe_stream_t stream) {
  if (!w_packed || !w_bf16) return fail(BFMOE_EINVAL, "unpack_base: NULL pointer");
  if (d < 4 || d > BFMOE_MAX_D || !is_pow2(d)) return fail(BFMOE_EINVAL, "unpack_base: bad d=%d", d);
  if (!aligned16(w_bf16)) return fail(BFMOE_EINVAL, "unpack_base: output must be 16-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int wpr = words_per_row(d);
  const long long n = static_cast<long long>(d) * wpr;
  cudaError_t e = launch("expand_base_bf16", s, [&] {
    expand_base_bf16_kernel<<<grid_for(n, 256, 4096), 256, 0, s>>>(w_packed, d, wpr, w_bf16);
  });
  if (e != cudaSuccess) return cuda_fail(e, "unpack_base: launch");
  return ok();
}

namespace {

// The exact 3-way bf16 split of W_g ([3N][d]: hi, mid, lo parts per row block).
cudaError_t split_gate_weights(const float* w_gate, int N, int d, __nv_bfloat16* parts, cudaStream_t s) {
  const long long nw = static_cast<long long>(N) * d;
  return launch("router_split", s, [&] { pdl_launch(router_split_kernel, grid_for(nw, 256, 2048), 256, 0, s, w_gate, nw, parts); });
}

// Router + buckets; `parts_ready` (or null) is W_g already split by
// split_gate_weights, which a caller routing several token chunks with the
// same weights does once.
int router_topk_impl(const void* x, int x_dtype, int T, int d, const float* w_gate, const float* bias, int n_experts,
                     int k, int32_t* idx, float* gates, int32_t* counts, int32_t* offsets, int32_t* rows, void* ws,
                     size_t ws_bytes, cudaStream_t s, const __nv_bfloat16* parts_ready, int32_t* pad_out = nullptr);

}  // namespace

int bfmoe_router_topk(const void* x, int x_dtype, int T, int d, const float* w_gate, const float* bias,
                      int n_experts, int k, int32_t* idx, float* gates, int32_t* counts, int32_t* offsets,
                      int32_t* rows, void* ws, size_t ws_bytes, bfmoe_stream_t stream) {
  return router_topk_impl(x, x_dtype, T, d, w_gate, bias, n_experts, k, idx, gates, counts, offsets, rows, ws,
                          ws_bytes, reinterpret_cast<cudaStream_t>(stream), nullptr);
}

namespace {

int router_topk_impl(const void* x, int x_dtype, int T, int d, const float* w_gate, const float* bias, int n_experts,
                     int k, int32_t* idx, float* gates, int32_t* counts, int32_t* offsets, int32_t* rows, void* ws,
                     size_t ws_bytes, cudaStream_t s, const __nv_bfloat16* parts_ready, int32_t* pad_out) {
  int rc = check_sizes(d, n_experts, T, k);
  if (rc) return rc;
  if ((rc = check_dtype(x_dtype))) return rc;
  // the buckets are built when counts and offsets are given (rows too, unless
  // T = 0), skipped when all three are NULL
  const bool buckets = counts || offsets || rows;
  if (buckets && (!counts || !offsets || (!rows && T > 0)))
    return fail(BFMOE_EINVAL, "router_topk: counts, offsets and rows must be all given or all NULL");
  const int N = n_experts;
  cudaError_t e;
  if (T == 0) {
    if (!buckets) return ok();
    if ((e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * N, s)) != cudaSuccess) return cuda_fail(e, "router_topk: memset");
    if ((e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (N + 1), s)) != cudaSuccess) return cuda_fail(e, "router_topk: memset");
    return ok();
  }
  if (!x || !w_gate || !idx || !gates) return fail(BFMOE_EINVAL, "router_topk: NULL pointer");
  const Plan p = make_plan(d, N, T, k, x_dtype);
  if ((rc = check_ws(p, ws, ws_bytes, p.rt_end))) return rc;
  uint8_t* W = static_cast<uint8_t*>(ws);
  float* logits = reinterpret_cast<float*>(W + p.logits);
  int32_t* cc = reinterpret_cast<int32_t*>(W + p.chunk_counts);
  int32_t* totals = reinterpret_cast<int32_t*>(W + p.totals);
  int* unsure = reinterpret_cast<int*>(W + p.unsure);
  const long long R = static_cast<long long>(T) * k;
  // the float32 error band that leaves a top-k undecided (router.cuh)
  const float eps_c = 2e-5f * std::sqrt(static_cast<float>(d) / 2048.f);
  const bool tc_router = tc_router_path(x_dtype, d);
  if (!tc_router && (e = cudaMemsetAsync(unsure, 0, 8, s)) != cudaSuccess) return cuda_fail(e, "router_topk: memset");
  if (tc_router) {
    // tensor cores: exact 3-way bf16 split of W_g, top-k fused in the epilogue
    if (!aligned16(x)) return fail(BFMOE_EINVAL, "router_topk: x must be 16-byte aligned");
    const __nv_bfloat16* parts = parts_ready;
    if (!parts) {
      __nv_bfloat16* own = reinterpret_cast<__nv_bfloat16*>(W + p.wg_parts);
      if ((e = split_gate_weights(w_gate, N, d, own, s)) != cudaSuccess) return cuda_fail(e, "router_topk: split");
      parts = own;
    }
    const int BN = N >= 128 ? 128 : (N > 32 ? 64 : (N > 16 ? 32 : 16));
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    CUtensorMap tx, tw;
    if (!make_tmap_bf16(&tx, x, d, T, kGemmBM) || !make_tmap_bf16(&tw, parts, d, 3LL * N, BN))
      return fail(BFMOE_ECUDA, "router_topk: tensor map encoding failed");
    switch (BN) {
      case 16: e = launch_router_tc<16, 4>(tx, tw, bias, T, d, N, k, eps_c, logits, xb, w_gate, idx, gates, cc, s); break;
      case 32: e = launch_router_tc<32, 4>(tx, tw, bias, T, d, N, k, eps_c, logits, xb, w_gate, idx, gates, cc, s); break;
      case 64: e = launch_router_tc<64, 4>(tx, tw, bias, T, d, N, k, eps_c, logits, xb, w_gate, idx, gates, cc, s); break;
      default: e = launch_router_tc<128, 3>(tx, tw, bias, T, d, N, k, eps_c, logits, xb, w_gate, idx, gates, cc, s); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "router_topk: tensor-core router");
  } else {
    dim3 g1((T + 63) / 64, (N + 63) / 64);
    e = launch("router_logits_simt", s, [&] {
      if (x_dtype == BFMOE_BF16)
        router_logits_simt_kernel<__nv_bfloat16><<<g1, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), w_gate,
                                                                    bias, T, d, N, logits);
      else
        router_logits_simt_kernel<float><<<g1, 256, 0, s>>>(static_cast<const float*>(x), w_gate, bias, T, d, N,
                                                            logits);
    });
    if (e != cudaSuccess) return cuda_fail(e, "router_topk: logits");
    e = launch("router_topk", s, [&] {
      const int g = grid_for(T, 8, sm_count() * 32);
      if (x_dtype == BFMOE_BF16)
        router_topk_kernel<__nv_bfloat16><<<g, 256, 0, s>>>(logits, static_cast<const __nv_bfloat16*>(x), w_gate,
                                                            bias, T, d, N, k, eps_c, idx, gates, unsure);
      else
        router_topk_kernel<float><<<g, 256, 0, s>>>(logits, static_cast<const float*>(x), w_gate, bias, T, d, N, k,
                                                    eps_c, idx, gates, unsure);
    });
    if (e != cudaSuccess) return cuda_fail(e, "router_topk: top-k");
  }
  // the tokens left undecided by the float32 top-k, settled from exact
  // logits (usually a few per thousand; near ties always); the tensor-core
  // router settles its own in its epilogue
  if (!tc_router) {
    const int g = grid_for(T, kFixWarps, sm_count());
    int32_t* ccp = nullptr;
    e = launch("router_fixup", s, [&] {
      if (x_dtype == BFMOE_BF16)
        pdl_launch(router_fixup_kernel<__nv_bfloat16>, g, kFixWarps * 32, 0, s, static_cast<const __nv_bfloat16*>(x),
                   w_gate, bias, static_cast<const float*>(logits), T, d, N, k, eps_c,
                   static_cast<const int*>(unsure), idx, gates, ccp);
      else
        pdl_launch(router_fixup_kernel<float>, g, kFixWarps * 32, 0, s, static_cast<const float*>(x), w_gate, bias,
                   static_cast<const float*>(logits), T, d, N, k, eps_c, static_cast<const int*>(unsure), idx, gates,
                   ccp);
    });
    if (e != cudaSuccess) return cuda_fail(e, "router_topk: fix-up of undecided tokens");
  }

  const int chunk = bucket_chunk(k);
  if (!buckets) return ok();
  const int nchunks = static_cast<int>((R + chunk - 1) / chunk);
  static std::atomic<uint64_t> done{0};
  if (needs_attr(done)) {
    cudaFuncSetAttribute(bucket_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, BFMOE_MAX_EXPERTS * 4);
    cudaFuncSetAttribute(bucket_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         BFMOE_MAX_EXPERTS * 40 + 32);
    attr_set(done);
  }
  if (!tc_router) {  // the tensor-core router writes the chunk histograms itself
    e = launch("bucket_count", s, [&] { bucket_count_kernel<<<nchunks, chunk, N * 4, s>>>(idx, R, N, cc); });
    if (e != cudaSuccess) return cuda_fail(e, "router_topk: bucket count");
  }
  e = launch("bucket_scan", s, [&] { pdl_launch(bucket_scan_kernel, (N + 31) / 32, 1024, 0, s, cc, nchunks, N, totals); });
  if (e != cudaSuccess) return cuda_fail(e, "router_topk: bucket scan");
  const size_t scatter_smem = ((N + 1) * 4 + 15) / 16 * 16 + static_cast<size_t>(N) * 36 + 4;
  e = launch("bucket_scatter", s, [&] {
    pdl_launch(bucket_scatter_kernel, nchunks, chunk, scatter_smem, s, idx, R, N, static_cast<const int32_t*>(cc),
               static_cast<const int32_t*>(totals), counts, offsets, rows, pad_out, pad_cap(R, N));
  });
  if (e != cudaSuccess) return cuda_fail(e, "router_topk: bucket scatter");
  return ok();
}

}  // namespace

int bfmoe_router_topk_noalloc(const void* x, int x_dtype, int T, int d, const float* w_gate, const float* bias,
                              int n_experts, int k, int32_t* idx, float* gates, int32_t* counts, int32_t* offsets,
                              int32_t* rows, bfmoe_stream_t stream) {
  int rc = check_sizes(d, n_experts, T, k);
  if (rc) return rc;
  if ((rc = check_dtype(x_dtype))) return rc;
  const size_t need = make_plan(d, n_experts, T, k, x_dtype).rt_end;
  if (need > BFMOE_NOALLOC_SCRATCH_BYTES)
    return fail(BFMOE_EUNSUPPORTED,
                "router_topk_noalloc: these sizes need %zu bytes of scratch; the built-in array holds %u "
                "(use bfmoe_router_topk with a workspace)",
                need, static_cast<unsigned>(BFMOE_NOALLOC_SCRATCH_BYTES));
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch))) return rc;
  return bfmoe_router_topk(x, x_dtype, T, d, w_gate, bias, n_experts, k, idx, gates, counts, offsets, rows, scratch,
                           BFMOE_NOALLOC_SCRATCH_BYTES, stream);
}

int bfmoe_decode_forward(const bfmoe_layer* layer, const void* x, int x_dtype, int T, int k, const int32_t* idx,
                         const float* gates, void* y, bfmoe_stream_t stream) {
  if (!layer) return fail(BFMOE_EINVAL, "decode_forward: NULL layer");
  int rc = check_sizes(layer->d, layer->n_experts, T, k);
  if (rc) return rc;
  if ((rc = check_dtype(x_dtype))) return rc;
  if (T == 0) return ok();
  if (!layer->w_packed || !layer->theta || !layer->phi) return fail(BFMOE_EINVAL, "decode_forward: NULL layer weights");
  if (!x || !idx || !gates || !y) return fail(BFMOE_EINVAL, "decode_forward: NULL pointer");
  const int d = layer->d, L = ilog2(d), N = layer->n_experts;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t smem = static_cast<size_t>(2) * decode_rows(d, k) * d * sizeof(float);  // <= 128 KiB
  static std::atomic<uint64_t> done{0};
  if (needs_attr(done)) {
    const int most = 2 * 16384 * static_cast<int>(sizeof(float));
    cudaFuncSetAttribute(decode_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    cudaFuncSetAttribute(decode_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    attr_set(done);
  }
  const int grid = grid_for(T, 1, sm_count() * 8);
  const cudaError_t e = launch("decode", s, [&] {
    if (x_dtype == BFMOE_BF16)
      pdl_launch(decode_kernel<__nv_bfloat16>, grid, kDecodeThreads, smem, s, static_cast<const __nv_bfloat16*>(x),
                 T, d, L, k, idx, gates, layer->w_packed, layer->alpha, layer->theta, layer->phi, N,
                 static_cast<__nv_bfloat16*>(y));
    else
      pdl_launch(decode_kernel<float>, grid, kDecodeThreads, smem, s, static_cast<const float*>(x), T, d, L, k, idx,
                 gates, layer->w_packed, layer->alpha, layer->theta, layer->phi, N, static_cast<float*>(y));
  });
  if (e != cudaSuccess) return cuda_fail(e, "decode_forward");
  return ok();
}

int bfmoe_forward(const bfmoe_layer* layer, const void* x, int x_dtype, int T, int k, const int32_t* idx,
                  const float* gates, const int32_t* offsets, const int32_t* rows, void* y, void* ws,
                  size_t ws_bytes, bfmoe_stream_t stream) {
  int rc = check_forward_args(layer, x, x_dtype, T, k, idx, gates, offsets, rows, y);
  if (rc || T == 0) return rc ? rc : ok();
  const Plan p = make_plan(layer->d, layer->n_experts, T, k, x_dtype);
  if ((rc = check_ws(p, ws, ws_bytes, p.fwd_end))) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* W = static_cast<uint8_t*>(ws);
  const uint8_t* tabs = static_cast<const uint8_t*>(layer->tables);
  if (!tabs) {
    if ((rc = build_weight_tables(layer, W + p.tabs, s))) return rc;
    tabs = W + p.tabs;
  }
  return forward_body(layer, x, x_dtype == BFMOE_BF16, T, k, idx, gates, offsets, rows, y, p, W, tabs, s, false);
}

size_t bfmoe_moe_host_workspace_size(int d, int n_experts, int T, int k, int x_dtype, int chunk) {
  if (check_sizes(d, n_experts, T, k) != BFMOE_OK || check_dtype(x_dtype) != BFMOE_OK) return 0;
  return make_host_plan(d, n_experts, T, k, x_dtype, chunk).total;
}

int bfmoe_moe_forward_host(const bfmoe_layer* layer, const void* x_host, int x_dtype, int T, const float* w_gate,
                           const float* bias, int k, void* y_host, int chunk, void* ws, size_t ws_bytes,
                           bfmoe_stream_t stream) {
  if (!layer) return fail(BFMOE_EINVAL, "moe_forward_host: NULL layer");
  const int d = layer->d, N = layer->n_experts;
  int rc = check_sizes(d, N, T, k);
  if (rc) return rc;
  if ((rc = check_dtype(x_dtype))) return rc;
  if (T == 0) return ok();
  if (!layer->w_packed || !layer->theta || !layer->phi || !x_host || !y_host || !w_gate)
    return fail(BFMOE_EINVAL, "moe_forward_host: NULL pointer");
  const HostPlan hp = make_host_plan(d, N, T, k, x_dtype, chunk);
  if (!ws) return fail(BFMOE_EWORKSPACE, "moe_forward_host: NULL workspace");
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(BFMOE_EWORKSPACE, "moe_forward_host: workspace must be 256-byte aligned");
  if (ws_bytes < hp.total)
    return fail(BFMOE_EWORKSPACE, "moe_forward_host: workspace has %zu bytes, needs %zu", ws_bytes, hp.total);
  HostPipe* pipe = nullptr;
  SideStream* ss = nullptr;
  if ((rc = host_pipe(&pipe)) || (rc = side_stream(&ss))) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* W = static_cast<uint8_t*>(ws);
  const bool bf16 = x_dtype == BFMOE_BF16;
  const size_t row_bytes = static_cast<size_t>(d) * (bf16 ? 2 : 4);
  uint8_t* x_dev = W + hp.x_dev;
  uint8_t* y_dev = W + hp.y_dev;
  const Plan pc = make_plan(d, N, hp.chunk, k, x_dtype);
  const uint8_t* xh = static_cast<const uint8_t*>(x_host);
  uint8_t* yh = static_cast<uint8_t*>(y_host);
  // chunk c runs on lane c % lanes: lane 0 is `stream`, lane 1 the pipe's
  // second compute stream, each with its own routing buffers and scratch
  cudaStream_t lane_s[2] = {s, pipe->lane1};

  // the copy streams start after all earlier work on `stream` (so a previous
  // call's buffers are free); the weight tables build on the side stream
  cudaError_t e = cudaEventRecord(pipe->fork, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(pipe->in, pipe->fork, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(pipe->out, pipe->fork, 0);
  if (e == cudaSuccess) e = cudaEventRecord(ss->fork, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->stream, ss->fork, 0);
  if (e != cudaSuccess) return cuda_fail(e, "moe_forward_host: fork");
  const uint8_t* tabs = static_cast<const uint8_t*>(layer->tables);
  if (!tabs) {
    // (in lane 0's scratch; both lanes read them)
    rc = build_weight_tables(layer, W + hp.moe[0] + pc.tabs, ss->stream);
    tabs = W + hp.moe[0] + pc.tabs;
  }
  if ((e = cudaEventRecord(ss->join, ss->stream)) != cudaSuccess) return cuda_fail(e, "moe_forward_host: join record");
  // W_g is split once for all chunks, while the first chunk is copied in
  const __nv_bfloat16* parts = nullptr;
  if (rc == BFMOE_OK && tc_router_path(x_dtype, d)) {
    if (layer->gate_parts) {
      parts = static_cast<const __nv_bfloat16*>(layer->gate_parts);
    } else {
      auto* own = reinterpret_cast<__nv_bfloat16*>(W + hp.parts);
      if ((e = split_gate_weights(w_gate, N, d, own, s)) != cudaSuccess) rc = cuda_fail(e, "moe_forward_host: split");
      parts = own;
    }
  }
  // lane 1 starts after the split (and so after the fork)
  if (rc == BFMOE_OK && hp.lanes == 2 &&
      ((e = cudaEventRecord(pipe->lane1_go, s)) != cudaSuccess ||
       (e = cudaStreamWaitEvent(pipe->lane1, pipe->lane1_go, 0)) != cudaSuccess))
    rc = cuda_fail(e, "moe_forward_host: lane fork");
  const bool lane1_used = rc == BFMOE_OK && hp.lanes == 2;
  for (int c = 0; c < hp.nchunks && rc == BFMOE_OK; ++c) {
    const int l = c % hp.lanes;
    cudaStream_t ls = lane_s[l];
    int32_t* idx = reinterpret_cast<int32_t*>(W + hp.idx[l]);
    float* gates = reinterpret_cast<float*>(W + hp.gates[l]);
    int32_t* counts = reinterpret_cast<int32_t*>(W + hp.counts[l]);
    int32_t* offsets = reinterpret_cast<int32_t*>(W + hp.offsets[l]);
    int32_t* rows = reinterpret_cast<int32_t*>(W + hp.rows[l]);
    uint8_t* Wm = W + hp.moe[l];
    const int t0 = hp.start[c], Tc = hp.start[c + 1] - t0;
    const size_t o = static_cast<size_t>(t0) * row_bytes, n = static_cast<size_t>(Tc) * row_bytes;
    if ((e = cudaMemcpyAsync(x_dev + o, xh + o, n, cudaMemcpyHostToDevice, pipe->in)) != cudaSuccess ||
        (e = cudaEventRecord(pipe->ev_in[c], pipe->in)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(ls, pipe->ev_in[c], 0)) != cudaSuccess) {
      rc = cuda_fail(e, "moe_forward_host: copy in");
      break;
    }
    // the router's scatter also writes the fused kernel's padded bucket order
    const Plan pcur = make_plan(d, N, Tc, k, x_dtype);
    const bool fused = fused_path(x_dtype, d);
    rc = router_topk_impl(x_dev + o, x_dtype, Tc, d, w_gate, bias, N, k, idx, gates, counts, offsets, rows,
                          Wm + pc.fwd_end, pc.rt_end, ls, parts,
                          fused ? reinterpret_cast<int32_t*>(Wm + pcur.pad) : nullptr);
    // each lane's first forward waits for the weight tables
    if (c < hp.lanes && (e = cudaStreamWaitEvent(ls, ss->join, 0)) != cudaSuccess)
      rc = cuda_fail(e, "moe_forward_host: join");
    if (rc) break;
    rc = forward_body(layer, x_dev + o, bf16, Tc, k, idx, gates, offsets, rows, y_dev + o, pcur, Wm, tabs, ls, fused);
    if (rc) break;
    if ((e = cudaEventRecord(pipe->ev_out[c], ls)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(pipe->out, pipe->ev_out[c], 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(yh + o, y_dev + o, n, cudaMemcpyDeviceToHost, pipe->out)) != cudaSuccess)
      rc = cuda_fail(e, "moe_forward_host: copy out");
  }
  // join: later work on `stream` runs after every copy out, lane 1's work
  // and the side stream's tables (joined above or here when no chunk ran)
  if ((e = cudaEventRecord(pipe->done, pipe->out)) == cudaSuccess) e = cudaStreamWaitEvent(s, pipe->done, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ss->join, 0);
  if (e == cudaSuccess && lane1_used && (e = cudaEventRecord(pipe->lane1_done, pipe->lane1)) == cudaSuccess)
    e = cudaStreamWaitEvent(s, pipe->lane1_done, 0);
  if (e == cudaSuccess && (e = cudaEventRecord(pipe->fork, pipe->in)) == cudaSuccess)
    e = cudaStreamWaitEvent(s, pipe->fork, 0);
  if (e != cudaSuccess && rc == BFMOE_OK) rc = cuda_fail(e, "moe_forward_host: final join");
  return rc ? rc : ok();
}

size_t bfmoe_moe_workspace_size(int d, int n_experts, int T, int k, int x_dtype) {
  if (check_sizes(d, n_experts, T, k) != BFMOE_OK || check_dtype(x_dtype) != BFMOE_OK) return 0;
  const Plan p = make_plan(d, n_experts, T, k, x_dtype);
  return p.fwd_end + p.rt_end;
}

int bfmoe_moe_forward(const bfmoe_layer* layer, const void* x, int x_dtype, int T, const float* w_gate,
                      const float* bias, int k, int32_t* idx, float* gates, int32_t* counts, int32_t* offsets,
                      int32_t* rows, void* y, void* ws, size_t ws_bytes, bfmoe_stream_t stream) {
  int rc = check_forward_args(layer, x, x_dtype, T, k, idx, gates, offsets, rows, y);
  if (rc) return rc;
  if (!w_gate || !counts) return fail(BFMOE_EINVAL, "moe_forward: NULL pointer");
  const int d = layer->d, N = layer->n_experts;
  const Plan p = make_plan(d, N, T, k, x_dtype);
  const size_t need = p.fwd_end + p.rt_end;
  if (T > 0 && (rc = check_ws(p, ws, ws_bytes, need))) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* W = static_cast<uint8_t*>(ws);
  if (T == 0)
    return bfmoe_router_topk(x, x_dtype, T, d, w_gate, bias, N, k, idx, gates, counts, offsets, rows, nullptr, 0,
                             stream);
  const uint8_t* tabs = static_cast<const uint8_t*>(layer->tables);
  // the router's scatter also writes the fused kernel's padded bucket order
  const bool fused = fused_path(x_dtype, d);
  int32_t* pad = fused ? reinterpret_cast<int32_t*>(W + p.pad) : nullptr;
  const auto* gate_parts = static_cast<const __nv_bfloat16*>(layer->gate_parts);
  if (tabs) {
    // prepared tables: router and forward in stream order, nothing on the side
    rc = router_topk_impl(x, x_dtype, T, d, w_gate, bias, N, k, idx, gates, counts, offsets, rows, W + p.fwd_end,
                          p.rt_end, s, gate_parts, pad);
    if (rc) return rc;
    return forward_body(layer, x, x_dtype == BFMOE_BF16, T, k, idx, gates, offsets, rows, y, p, W, tabs, s, fused);
  }
  // fork: the weight-derived tables build on the side stream while the router runs
  SideStream* ss = nullptr;
  if ((rc = side_stream(&ss))) return rc;
  cudaError_t e = cudaEventRecord(ss->fork, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->stream, ss->fork, 0);
  if (e != cudaSuccess) return cuda_fail(e, "moe_forward: fork");
  if ((rc = build_weight_tables(layer, W + p.tabs, ss->stream))) return rc;
  if ((e = cudaEventRecord(ss->join, ss->stream)) != cudaSuccess) return cuda_fail(e, "moe_forward: join record");
  rc = router_topk_impl(x, x_dtype, T, d, w_gate, bias, N, k, idx, gates, counts, offsets, rows, W + p.fwd_end,
                        p.rt_end, s, gate_parts, pad);
  // join before anything else can fail, so the side stream never outlives the call's work
  if ((e = cudaStreamWaitEvent(s, ss->join, 0)) != cudaSuccess) return cuda_fail(e, "moe_forward: join");
  if (rc) return rc;
  return forward_body(layer, x, x_dtype == BFMOE_BF16, T, k, idx, gates, offsets, rows, y, p, W, W + p.tabs, s, fused);
}

size_t bfmoe_gate_parts_size(int n_experts, int d) {
  if (d < 4 || d > BFMOE_MAX_D || !is_pow2(d) || n_experts < 1 || n_experts > BFMOE_MAX_EXPERTS) return 0;
  return static_cast<size_t>(3) * n_experts * d * sizeof(__nv_bfloat16);
}

int bfmoe_prepare_gate(const float* w_gate, int n_experts, int d, void* parts, size_t bytes, bfmoe_stream_t stream) {
  if (!w_gate || !parts) return fail(BFMOE_EINVAL, "prepare_gate: NULL pointer");
  if (d < 4 || d > BFMOE_MAX_D || !is_pow2(d)) return fail(BFMOE_EINVAL, "prepare_gate: bad d=%d", d);
  if (n_experts < 1 || n_experts > BFMOE_MAX_EXPERTS) return fail(BFMOE_EINVAL, "prepare_gate: n_experts=%d", n_experts);
  if (reinterpret_cast<uintptr_t>(parts) & 255u) return fail(BFMOE_EWORKSPACE, "prepare_gate: parts must be 256-byte aligned");
  const size_t need = bfmoe_gate_parts_size(n_experts, d);
  if (bytes < need) return fail(BFMOE_EWORKSPACE, "prepare_gate: %zu bytes given, %zu needed", bytes, need);
  const cudaError_t e = split_gate_weights(w_gate, n_experts, d, static_cast<__nv_bfloat16*>(parts),
                                           reinterpret_cast<cudaStream_t>(stream));
  return e != cudaSuccess ? cuda_fail(e, "prepare_gate") : ok();
}

size_t bfmoe_layer_tables_size(int d, int n_experts) {
  if (d < 4 || d > BFMOE_MAX_D || !is_pow2(d) || n_experts < 1 || n_experts > BFMOE_MAX_EXPERTS) return 0;
  return make_tab_plan(d, n_experts).total;
}

int bfmoe_prepare_layer(const bfmoe_layer* layer, void* tables, size_t bytes, bfmoe_stream_t stream) {
  if (!layer || !tables) return fail(BFMOE_EINVAL, "prepare_layer: NULL pointer");
  const int d = layer->d, N = layer->n_experts;
  if (d < 4 || d > BFMOE_MAX_D || !is_pow2(d)) return fail(BFMOE_EINVAL, "prepare_layer: bad d=%d", d);
  if (N < 1 || N > BFMOE_MAX_EXPERTS) return fail(BFMOE_EINVAL, "prepare_layer: n_experts=%d", N);
  if (!layer->w_packed || !layer->theta || !layer->phi) return fail(BFMOE_EINVAL, "prepare_layer: NULL layer weights");
  if (reinterpret_cast<uintptr_t>(tables) & 255u) return fail(BFMOE_EWORKSPACE, "prepare_layer: tables must be 256-byte aligned");
  const size_t need = make_tab_plan(d, N).total;
  if (bytes < need) return fail(BFMOE_EWORKSPACE, "prepare_layer: %zu bytes given, %zu needed", bytes, need);
  int rc = build_weight_tables(layer, static_cast<uint8_t*>(tables), reinterpret_cast<cudaStream_t>(stream));
  return rc ? rc : ok();
}

int bfmoe_materialize_expert(const bfmoe_layer* layer, int e_idx, float* w_out, bfmoe_stream_t stream) {
  if (!layer || !w_out) return fail(BFMOE_EINVAL, "materialize: NULL pointer");
  const int d = layer->d, N = layer->n_experts;
  if (d < 4 || d > BFMOE_MAX_D || !is_pow2(d)) return fail(BFMOE_EINVAL, "materialize: bad d=%d", d);
  if (e_idx < 0 || e_idx >= N) return fail(BFMOE_EINVAL, "materialize: expert %d not in [0, %d)", e_idx, N);
  if (!layer->w_packed || !layer->theta || !layer->phi) return fail(BFMOE_EINVAL, "materialize: NULL layer weights");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int L = ilog2(d);
  const size_t per = static_cast<size_t>(L) * (d / 2);
  cudaError_t e = launch("materialize", s, [&] {
    materialize_kernel<<<d, 256, 2 * d * sizeof(float), s>>>(layer->w_packed, words_per_row(d), d, L, layer->alpha,
                                                             layer->theta + per * e_idx, layer->phi + per * e_idx,
                                                             w_out);
  });
  if (e != cudaSuccess) return cuda_fail(e, "materialize: launch");
  return ok();
}

size_t bfmoe_backward_workspace_size(int d, int n_experts, int T, int k) {
  if (check_sizes(d, n_experts, T, k) != BFMOE_OK) return 0;
  return make_bw_plan(d, n_experts, T, k).total;
}

int bfmoe_backward(const bfmoe_layer* layer, const void* x, int x_dtype, int T, int k, const float* w_gate,
                   const int32_t* idx, const float* gates, const int32_t* offsets, const int32_t* rows,
                   const float* gy, float* dx, float* dtheta, float* dphi, float* dw_base, float* dalpha,
                   float* dw_gate, float* dbias, void* ws, size_t ws_bytes, bfmoe_stream_t stream) {
  if (!layer) return fail(BFMOE_EINVAL, "backward: NULL layer");
  const int d = layer->d, N = layer->n_experts, L = ilog2(d);
  int rc = check_sizes(d, N, T, k);
  if (rc) return rc;
  if ((rc = check_dtype(x_dtype))) return rc;
  if (!layer->w_packed || !layer->theta || !layer->phi) return fail(BFMOE_EINVAL, "backward: NULL layer weights");
  if (!dtheta || !dphi || !dw_base || !dalpha || !dw_gate || !w_gate || !offsets)
    return fail(BFMOE_EINVAL, "backward: NULL pointer");
  if (T > 0 && (!x || !idx || !gates || !rows || !gy || !dx)) return fail(BFMOE_EINVAL, "backward: NULL pointer");
  const BwPlan b = make_bw_plan(d, N, T, k);
  if (!ws) return fail(BFMOE_EWORKSPACE, "backward: NULL workspace");
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(BFMOE_EWORKSPACE, "backward: workspace must be 256-byte aligned");
  if (ws_bytes < b.total) return fail(BFMOE_EWORKSPACE, "backward: workspace has %zu bytes, needs %zu", ws_bytes, b.total);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* W = static_cast<uint8_t*>(ws);
  float2* tab_t = reinterpret_cast<float2*>(W + b.tab_t);
  float2* tab_p = reinterpret_cast<float2*>(W + b.tab_p);
  uint32_t* wt = reinterpret_cast<uint32_t*>(W + b.wt);
  float* U = reinterpret_cast<float*>(W + b.U);
  float* Z = reinterpret_cast<float*>(W + b.Z);
  float* dU = reinterpret_cast<float*>(W + b.dU);
  float* dg = reinterpret_cast<float*>(W + b.dg);
  float* dl = reinterpret_cast<float*>(W + b.dl);
  float* part = reinterpret_cast<float*>(W + b.part);
  float* dapart = reinterpret_cast<float*>(W + b.dapart);
  const bool bf16 = x_dtype == BFMOE_BF16;
  const long long R = static_cast<long long>(T) * k;
  const long long nang = static_cast<long long>(N) * L * (d / 2);
  const int wpr = words_per_row(d);
  cudaError_t e;
  // cos/sin of both butterflies, the base's transpose
  e = launch("bw_tables", s, [&] { rot_table_kernel<<<grid_for(nang, 256, 8192), 256, 0, s>>>(layer->theta, nang, tab_t); });
  if (e == cudaSuccess)
    e = launch("bw_tables", s, [&] { rot_table_kernel<<<grid_for(nang, 256, 8192), 256, 0, s>>>(layer->phi, nang, tab_p); });
  if (e == cudaSuccess)
    e = launch("bw_transpose_base", s, [&] {
      transpose_packed_kernel<<<grid_for(static_cast<long long>(d) * wpr, 256, 4096), 256, 0, s>>>(layer->w_packed, d,
                                                                                                   wpr, wt);
    });
  if (e != cudaSuccess) return cuda_fail(e, "backward: tables");
  if (T == 0) {
    const size_t ang = static_cast<size_t>(nang) * 4;
    if ((e = cudaMemsetAsync(dtheta, 0, ang, s)) != cudaSuccess || (e = cudaMemsetAsync(dphi, 0, ang, s)) != cudaSuccess ||
        (e = cudaMemsetAsync(dw_base, 0, static_cast<size_t>(d) * d * 4, s)) != cudaSuccess ||
        (e = cudaMemsetAsync(dalpha, 0, 4, s)) != cudaSuccess ||
        (e = cudaMemsetAsync(dw_gate, 0, static_cast<size_t>(N) * d * 4, s)) != cudaSuccess ||
        (dbias && (e = cudaMemsetAsync(dbias, 0, static_cast<size_t>(N) * 4, s)) != cudaSuccess))
      return cuda_fail(e, "backward: memset");
    return ok();
  }
  // recompute the forward's rows in float32: u (bucket order), z = alpha W u
  if ((e = bw_rows_dispatch(d, x, bf16, idx, rows, offsets, gates, gy, tab_t, tab_p, R, k, L, N, U, Z, dU, dg, dtheta,
                            dphi, 0, s)) != cudaSuccess)
    return cuda_fail(e, "backward: pre-rotation");
  const dim3 gg((R + 63) / 64, (d + 63) / 64);
  e = launch("bw_gemm", s, [&] {
    ternary_gemm_simt_kernel<float><<<gg, 256, 0, s>>>(U, layer->w_packed, wpr, R, d, layer->alpha, Z);
  });
  if (e != cudaSuccess) return cuda_fail(e, "backward: product");
  // output side: dg, dz = B(phi)^T (g gy) (in place of z), dphi
  if ((e = bw_rows_dispatch(d, x, bf16, idx, rows, offsets, gates, gy, tab_t, tab_p, R, k, L, N, U, Z, dU, dg, dtheta,
                            dphi, 1, s)) != cudaSuccess)
    return cuda_fail(e, "backward: output rotation");
  // du = alpha W^T dz; M = dz^T u, dW = alpha M, dalpha = sum W .* M
  e = launch("bw_gemm", s, [&] {
    ternary_gemm_simt_kernel<float><<<gg, 256, 0, s>>>(Z, wt, wpr, R, d, layer->alpha, dU);
  });
  if (e == cudaSuccess)
    e = launch("bw_outer", s, [&] {
      const dim3 go((d + kOuterTile - 1) / kOuterTile, (d + kOuterTile - 1) / kOuterTile, b.slices);
      outer_tn_kernel<<<go, 256, 0, s>>>(Z, U, R, d, part);
    });
  if (e == cudaSuccess)
    e = launch("bw_outer_reduce", s, [&] {
      outer_reduce_kernel<<<b.ra_blocks, 256, 0, s>>>(part, b.slices, d, layer->alpha, layer->w_packed, wpr, dw_base,
                                                      dapart);
    });
  if (e == cudaSuccess) e = launch("bw_sum", s, [&] { sum_kernel<<<1, 32, 0, s>>>(dapart, b.ra_blocks, dalpha); });
  if (e != cudaSuccess) return cuda_fail(e, "backward: base gradient");
  // input side: per-row dx = B(theta) du (into the z buffer, row order), dtheta
  if ((e = bw_rows_dispatch(d, x, bf16, idx, rows, offsets, gates, gy, tab_t, tab_p, R, k, L, N, U, Z, dU, dg, dtheta,
                            dphi, 2, s)) != cudaSuccess)
    return cuda_fail(e, "backward: input rotation");
  // router and per-token sums
  e = launch("bw_token", s, [&] {
    const int g = grid_for(T, 8, sm_count() * 16);
    if (bf16)
      bw_token_kernel<__nv_bfloat16><<<g, 256, 0, s>>>(Z, dg, gates, idx, w_gate, T, k, d, N, dl, dx);
    else
      bw_token_kernel<float><<<g, 256, 0, s>>>(Z, dg, gates, idx, w_gate, T, k, d, N, dl, dx);
  });
  if (e == cudaSuccess)
    e = launch("bw_router", s, [&] {
      if (bf16)
        bw_router_kernel<__nv_bfloat16><<<N, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), dl, rows, offsets, k, d,
                                                         R, dw_gate, dbias);
      else
        bw_router_kernel<float><<<N, 256, 0, s>>>(static_cast<const float*>(x), dl, rows, offsets, k, d, R, dw_gate,
                                                 dbias);
    });
  if (e != cudaSuccess) return cuda_fail(e, "backward: router");
  return ok();
}

int bfmoe_check_device_error(bfmoe_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "check_device_error: synchronize");
  unsigned code = 0, info = 0;
  if ((e = cudaMemcpyFromSymbol(&code, g_err_code, sizeof(code))) != cudaSuccess) return cuda_fail(e, "read error word");
  if ((e = cudaMemcpyFromSymbol(&info, g_err_info, sizeof(info))) != cudaSuccess) return cuda_fail(e, "read error word");
  if (code == 0) return ok();
  const unsigned zero = 0;
  cudaMemcpyToSymbol(g_err_code, &zero, sizeof(zero));
  cudaMemcpyToSymbol(g_err_info, &zero, sizeof(zero));
  if (code == BFMOE_EDEVICE_TIMEOUT) return fail(BFMOE_EDEVICE_TIMEOUT, "device wait timed out (site 0x%x)", info);
  return fail(static_cast<int>(code), "device check failed (code %u, at %u)", code, info);
}

int bfmoe_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof) {
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_prof.clear();
  g_prof_on = on != 0;
  return ok();
}

int bfmoe_profile_collect(bfmoe_kernel_time* out, int max, int* n_out) {
  std::vector<ProfRec> recs;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    recs.swap(g_prof);
  }
  std::map<std::string, std::pair<int, double>> agg;
  std::vector<std::string> order;
  int rc = BFMOE_OK;
  for (auto& r : recs) {
    cudaError_t e = cudaEventSynchronize(r.b);
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess) rc = cuda_fail(e, "profile_collect");
    auto it = agg.find(r.name);
    if (it == agg.end()) {
      order.push_back(r.name);
      agg[r.name] = {1, ms};
    } else {
      it->second.first += 1;
      it->second.second += ms;
    }
  }
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (auto& r : recs) {
      g_event_pool.push_back(r.a);
      g_event_pool.push_back(r.b);
    }
  }
  int n = 0;
  for (auto& name : order) {
    if (n >= max) break;
    std::snprintf(out[n].name, sizeof(out[n].name), "%s", name.c_str());
    out[n].launches = agg[name].first;
    out[n].total_ms = agg[name].second;
    ++n;
  }
  if (n_out) *n_out = n;
  return rc == BFMOE_OK ? ok() : rc;
}

}  // extern "C"
