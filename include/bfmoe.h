/*
 * bfmoe.h - C ABI of the ButterflyMoE expert forward on NVIDIA B200 (sm_100a).
 *
 * The method (ButterflyMoE: sub-linear ternary experts via structured
 * butterfly orbits; gist.science technical summary, sections 2.1-2.3):
 * every expert is W_i = B(phi_i) . W_base . B(theta_i)^T, where W_base is one
 * d x d ternary {-1, 0, +1} matrix shared by all N experts (scaled here by one
 * float alpha) and B(.) is a butterfly of log2(d) stages of d/2 Givens
 * rotations, one angle per rotation.  Inference never forms W_i: a token x
 * routed to experts e_0..e_{k-1} with gates g_j gets
 *     y = sum_j g_j * B(phi_{e_j}) (alpha * W_base (B(theta_{e_j})^T x)).
 *
 * Conventions shared by every call (the pages leave them open):
 *  - stage s (stride h = 2^s) rotates the pairs (i, i+h) with bit s of i
 *    clear; its rotations are numbered by ascending i; the 2x2 block is
 *    [[cos a, -sin a], [sin a, cos a]]; B = S_{L-1} ... S_1 S_0, so stage 0
 *    acts first; B^T is the literal transpose (stages L-1 ... 0, blocks
 *    transposed).
 *  - W_base[o][i]: row o is the output, column i the input (y = W x).
 *  - angles are float32 [N][log2 d][d/2]; tokens and outputs are row-major
 *    [T][d] in float32 or bfloat16.
 *  - routed row r = t*k + j is slot j of token t.
 *
 * Memory: every pointer is caller-owned.  Pointers named "device" must be
 * device memory of the current device; the library allocates nothing per
 * call.  A call only enqueues work on `stream` (no host synchronisation)
 * unless its comment says it synchronises.
 *
 * Errors: every int-returning call returns a bfmoe_status.  Argument checks
 * run on the host before any launch; on failure nothing is launched and
 * bfmoe_last_error() (thread-local) describes the problem.  Device-side checks
 * (an index out of range in caller-provided routing arrays, a bounded wait
 * that ran out) never trap: the kernel skips the bad access, records a code
 * in a device error word and returns; bfmoe_check_device_error() reads it.
 */
#ifndef BFMOE_H
#define BFMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The same handle as cudaStream_t (NULL = the legacy default stream). */
typedef struct CUstream_st* bfmoe_stream_t;

typedef enum {
  BFMOE_OK = 0,
  BFMOE_EINVAL = 1,           /* null pointer, size or shape out of range      */
  BFMOE_ENOT_TERNARY = 2,     /* a base weight outside {-1, 0, +1}             */
  BFMOE_EUNSUPPORTED = 3,     /* well-formed but outside the supported range   */
  BFMOE_EWORKSPACE = 4,       /* workspace missing, too small or misaligned    */
  BFMOE_ECUDA = 5,            /* a CUDA runtime call failed                    */
  BFMOE_EDEVICE_TIMEOUT = 6,  /* a device-side bounded wait ran out            */
  BFMOE_EDEVICE_BOUNDS = 7    /* a device-side index check failed              */
} bfmoe_status;

typedef enum { BFMOE_F32 = 0, BFMOE_BF16 = 1 } bfmoe_dtype;

/* Supported ranges. */
#define BFMOE_MAX_D 4096        /* d: power of two, 4 <= d <= 4096         */
#define BFMOE_MAX_EXPERTS 4096  /* N: 1 <= N <= 4096                       */
#define BFMOE_MAX_K 8           /* k: 1 <= k <= min(8, N)                  */

/* One ButterflyMoE layer (all pointers device, caller-owned, read-only). */
typedef struct {
  int d;                      /* width; power of two in [4, BFMOE_MAX_D]           */
  int n_experts;              /* N                                                  */
  const uint32_t* w_packed;   /* [d][max(1, d/16)] 2-bit codes (bfmoe_pack_base)   */
  float alpha;                /* scale of the ternary base                          */
  const float* theta;         /* [N][log2 d][d/2] input-side angles  (B(theta)^T)  */
  const float* phi;           /* [N][log2 d][d/2] output-side angles (B(phi))      */
  const void* tables;         /* NULL, or this layer's weight tables written by
                                 bfmoe_prepare_layer (then the calls read them
                                 instead of rebuilding them per call)               */
  const void* gate_parts;     /* NULL, or the router weights passed to the
                                 bfmoe_moe_* calls split by bfmoe_prepare_gate
                                 (then those calls skip the per-call split)         */
} bfmoe_layer;

/*
 * Pack the shared ternary base (one-time weight load).
 * The pages store W_base at 1.58 bits per weight (technical summary, 2.1);
 * this storage spends 2 bits: 0 -> 00, +1 -> 01, -1 -> 11 (10 is never
 * written and reads as 0), 16 codes per uint32, row-major, column i of a word
 * at bits 2*(i mod 16).  Row length is max(1, d/16) words.
 *   w        device int8 [d][d], values in {-1, 0, +1}
 *   w_packed device uint32 [d][max(1, d/16)] (written)
 * Synchronises `stream` to report BFMOE_ENOT_TERNARY (then w_packed holds 0
 * for every invalid weight).
 */
int bfmoe_pack_base(const int8_t* w, int d, uint32_t* w_packed, bfmoe_stream_t stream);

/*
 * Expand the packed base to the exact bfloat16 matrix the tensor-core GEMM
 * multiplies by (checking aid for the 2-bit code).
 *   w_bf16   device uint16 [d][d] (bfloat16 bit patterns 0x0000, 0x3F80, 0xBF80)
 */
int bfmoe_unpack_base(const uint32_t* w_packed, int d, uint16_t* w_bf16, bfmoe_stream_t stream);

/*
 * Router: logits l = x W_g^T (+ b) in float32; top-k experts per token by
 * descending logit, the lower expert index first on equal logits (and NaN
 * below every number); gates g_j = exp(l_{e_j} - l_{e_0}) / sum_j' exp(...)
 * (softmax over all N, top-k, renormalised); then the token-to-expert
 * buckets.  The pages only define mixture-of-experts selection in general
 * (signalfieldnotes ButterflyMoE article, glossary "Mixtures of Experts").
 *   x         device [T][d], dtype x_dtype
 *   w_gate    device float [N][d];  bias: device float [N] or NULL
 *   idx       device int32 [T][k] (written): experts, slot order
 *   gates     device float [T][k] (written)
 *   counts    device int32 [N]    (written): rows per expert
 *   offsets   device int32 [N+1]  (written): exclusive prefix sum of counts
 *   rows      device int32 [T*k]  (written): expert by expert, that expert's
 *             routed rows r = t*k + j in ascending token order
 *   ws        device scratch of at least bfmoe_workspace_size(...) bytes,
 *             256-byte aligned
 * counts, offsets and rows may all three be NULL: the buckets are then not
 * built (bfmoe_decode_forward needs only idx and gates).  Otherwise counts
 * and offsets, and rows when T > 0, must all be given (else BFMOE_EINVAL).
 * T = 0 is allowed (counts and offsets, when given, are zeroed).
 */
int bfmoe_router_topk(const void* x, int x_dtype, int T, int d,
                      const float* w_gate, const float* bias, int n_experts, int k,
                      int32_t* idx, float* gates,
                      int32_t* counts, int32_t* offsets, int32_t* rows,
                      void* ws, size_t ws_bytes, bfmoe_stream_t stream);

/*
 * bfmoe_router_topk without a caller workspace (no counterpart on the pages:
 * it serves callers rather than the method).  Some callers cannot allocate
 * device memory when they call: a plug-in or kernel host that is handed only
 * its input and output buffers, code running while the framework's allocator
 * is locked or not reachable from the calling thread, or a runtime whose
 * memory is planned before execution.  This call computes exactly what
 * bfmoe_router_topk computes, using as scratch one fixed array inside the
 * library of BFMOE_NOALLOC_SCRATCH_BYTES (every GPU that loads the library
 * holds it until the process exits).  It allocates nothing.
 *   - Sizes whose router scratch (bfmoe_router_scratch_size for these sizes)
 *     exceeds the array are rejected with BFMOE_EUNSUPPORTED before any
 *     launch.
 *   - The first call on a device looks up the array's device address with that
 *     device current; make that first call before any stream capture.
 *   - Every call shares the array: calls whose work overlaps on the GPU (on
 *     different streams, or concurrent host threads on one device) race and
 *     give wrong results.  Calls ordered on one stream are safe.  No part of
 *     the array has to start at zero: each kernel writes its part before it
 *     is read.
 * Arguments and outputs as for bfmoe_router_topk.
 */
#define BFMOE_NOALLOC_SCRATCH_BYTES (32u << 20)
int bfmoe_router_topk_noalloc(const void* x, int x_dtype, int T, int d,
                              const float* w_gate, const float* bias, int n_experts, int k,
                              int32_t* idx, float* gates,
                              int32_t* counts, int32_t* offsets, int32_t* rows,
                              bfmoe_stream_t stream);

/*
 * Expert forward without forming any expert (technical summary, 2.3):
 * for every routed row, B(theta_e)^T x_t, then alpha * W_base (.), then
 * B(phi_e) (.), times the gate; the k rows of a token are summed in slot
 * order in float32 and rounded once to the output dtype.
 *   layer     weights (see bfmoe_layer)
 *   x         device [T][d], dtype x_dtype
 *   idx, gates, offsets, rows: as written by bfmoe_router_topk (any routing
 *             with k distinct experts per token and consistent buckets)
 *   y         device [T][d], dtype x_dtype (written)
 *   ws        device scratch, bfmoe_workspace_size(d, N, T, k, x_dtype) bytes
 * The bfloat16 path rounds B(theta)^T x to bfloat16 before the tensor-core
 * product (the ternary weights are exact in bfloat16); rotations, the
 * product's accumulation, the gates and the combine are float32.  The float32
 * path keeps every intermediate in float32.
 */
int bfmoe_forward(const bfmoe_layer* layer, const void* x, int x_dtype, int T, int k,
                  const int32_t* idx, const float* gates,
                  const int32_t* offsets, const int32_t* rows,
                  void* y, void* ws, size_t ws_bytes, bfmoe_stream_t stream);

/*
 * Router and expert forward in one call: the results of bfmoe_router_topk
 * followed by bfmoe_forward, bit for bit.  The work that depends on the
 * weights only (the cos/sin tables of theta and phi and the bf16 copy of the
 * base) runs on a library-owned side stream, forked from `stream` with an
 * event and joined back before the pre-rotation, so it overlaps the router.
 * The side stream and its two events are created once per device on first
 * use (make that first call before any stream capture); the fork and join
 * are stream-ordered and can be captured in a CUDA graph.  Calls from several
 * host threads on one device share that side stream and serialise their
 * weight-only work.
 *   ws        device scratch of bfmoe_moe_workspace_size(...) bytes, 256-byte
 *             aligned (the router and the tables need separate regions here)
 * Other arguments as for bfmoe_router_topk and bfmoe_forward.
 */
int bfmoe_moe_forward(const bfmoe_layer* layer, const void* x, int x_dtype, int T,
                      const float* w_gate, const float* bias, int k,
                      int32_t* idx, float* gates, int32_t* counts, int32_t* offsets, int32_t* rows,
                      void* y, void* ws, size_t ws_bytes, bfmoe_stream_t stream);

/*
 * Split the router weights once for the tensor-core router (no counterpart
 * on the pages).  The bf16 router multiplies x by an exact three-part bf16
 * split of the float32 W_g (hi + mid + lo == W_g); without prepared parts
 * every call makes it.  With `layer->gate_parts` pointing at memory written
 * here from the same w_gate, bfmoe_moe_forward and bfmoe_moe_forward_host
 * use it instead (results identical bit for bit); they ignore it on the
 * paths that do not split (float32 x, d not a multiple of 64).  Redo after
 * changing W_g.
 *   w_gate    device float [N][d]
 *   parts     device memory of bfmoe_gate_parts_size(N, d) bytes, 256-byte
 *             aligned (written: [3][N][d] bfloat16)
 * Returns BFMOE_EINVAL / BFMOE_EWORKSPACE on bad arguments (nothing launched).
 */
int bfmoe_prepare_gate(const float* w_gate, int n_experts, int d, void* parts, size_t bytes,
                       bfmoe_stream_t stream);

/* Bytes that bfmoe_prepare_gate writes (0 for invalid sizes). */
size_t bfmoe_gate_parts_size(int n_experts, int d);

/*
 * Build a layer's weight tables once (no counterpart on the pages, which store
 * only the ternary base and the angles: technical summary, 2.2).  Every
 * forward needs, besides the tokens, values that depend on the weights alone:
 * cos and sin of every angle of theta and phi in the orders the rotation
 * kernels read them, and the bf16 copy of the 2-bit base that the tensor cores
 * multiply by.  Without prepared tables each forward call rebuilds them in its
 * workspace; with `layer->tables` pointing at memory written by this call,
 * bfmoe_forward, bfmoe_moe_forward and bfmoe_moe_forward_host read them
 * instead (results identical bit for bit).  Rebuild after changing the
 * layer's angles or base.
 *   tables   device scratch of bfmoe_layer_tables_size(d, N) bytes, 256-byte
 *            aligned, caller-owned (written; its contents are opaque)
 * The layer's `tables` field is ignored by this call.  Returns BFMOE_EINVAL
 * for a bad layer, BFMOE_EWORKSPACE for a short or misaligned buffer.
 */
int bfmoe_prepare_layer(const bfmoe_layer* layer, void* tables, size_t bytes, bfmoe_stream_t stream);

/* Bytes of one layer's prepared weight tables (0 for invalid sizes). */
size_t bfmoe_layer_tables_size(int d, int n_experts);

/* Scratch bytes that bfmoe_moe_forward needs (0 for invalid sizes). */
size_t bfmoe_moe_workspace_size(int d, int n_experts, int T, int k, int x_dtype);

/*
 * Router and expert forward from and to HOST memory, the host <-> device
 * copies overlapped with the work.  The T tokens are cut into chunks of
 * `chunk` tokens, the last one taking the rest (chunk <= 0: T / 4096 about
 * equal chunks, at least two and at most six, of at least 2048 tokens; at
 * most 64 chunks).  Copies in run on a library-owned copy-in stream, copies
 * out on a library-owned copy-out stream; the router + forward of even
 * chunks run on `stream`, of odd chunks on a library-owned second compute
 * stream (each of the two with its own routing buffers and scratch in ws),
 * so that a chunk's copy in, the work of the two chunks before it and an
 * earlier chunk's copy out overlap; events order them.  Each token's output
 * is that of bfmoe_moe_forward on its chunk (tokens are independent; the
 * pages route every token on its own, summary 2.3).  The weight-only tables
 * are built once per call.  Pages have no counterpart for the host
 * interface.
 *   x_host    host [T][d] (read), best page-locked: pageable memory makes the
 *             copies synchronous
 *   y_host    host [T][d] (written), same dtype; complete once the work
 *             enqueued on `stream` by this call has finished (synchronise the
 *             stream before reading it)
 *   chunk     tokens per chunk, or <= 0 for the default
 *   ws        device scratch of bfmoe_moe_host_workspace_size(...) bytes (the
 *             device copies of x and y, the split gate weights, and per
 *             compute stream one chunk's routing and one chunk's
 *             bfmoe_moe_forward scratch), 256-byte aligned
 * The copy and compute streams and their events are created once per device
 * on first use (make that first call before any stream capture); after that
 * the whole call is stream-ordered and can be captured in a CUDA graph,
 * copies included.  Calls that overlap on one device share these streams and
 * serialise there.
 * Returns BFMOE_EINVAL for null pointers or bad sizes, BFMOE_EWORKSPACE for a
 * short workspace.
 */
int bfmoe_moe_forward_host(const bfmoe_layer* layer, const void* x_host, int x_dtype, int T,
                           const float* w_gate, const float* bias, int k, void* y_host, int chunk,
                           void* ws, size_t ws_bytes, bfmoe_stream_t stream);

/* Scratch bytes that bfmoe_moe_forward_host needs (0 for invalid sizes). */
size_t bfmoe_moe_host_workspace_size(int d, int n_experts, int T, int k, int x_dtype, int chunk);

/*
 * Backward pass of the layer (router included), for training the rotations
 * jointly with the ternary base (technical summary, 2.4; the pages give no
 * formula, so this is the chain rule of bfmoe_moe_forward's arithmetic).
 * Given dL/dy, with the routing of the forward:
 *   dg_r = <v_r, gy_t>, dv_r = g_r gy_t          (v_r = B(phi) alpha W u_r)
 *   dphi_e  = sum over e's rows of d<dv, B(phi) z>/dphi,  dz = B(phi)^T dv
 *   dw_base = alpha sum_r dz_r u_r^T   (straight-through: the gradient of W_base
 *             taken as a real matrix, for the trainer's latent weights)
 *   dalpha  = sum_r <dz_r, W_base u_r>,  du = alpha W_base^T dz
 *   dtheta_e = sum over e's rows of d<du, B(theta)^T x>/dtheta,  dx += B(theta) du
 *   router: dl_j = g_j (dg_j - sum_j' g_j' dg_j') for the k selected logits,
 *   dw_gate[e] = sum dl x_t, dbias[e] = sum dl, dx_t += sum_j dl_j w_gate[e_j].
 * Everything is computed in float32 on the CUDA cores (the forward's rows are
 * recomputed in float32 from x; rotations are inverted stage by stage instead
 * of storing their activations).  Angle gradients are summed with
 * shared-memory atomics, so their last bits may differ between runs.
 *   layer, x, x_dtype, T, k, w_gate: as for the forward (bias is not needed)
 *   idx, gates, offsets, rows: the forward's routing (bfmoe_router_topk)
 *   gy        device float [T][d]: dL/dy
 *   dx        device float [T][d] (written)
 *   dtheta, dphi  device float [N][log2 d][d/2] (written, zero for unused experts)
 *   dw_base   device float [d][d] (written);  dalpha: device float [1] (written)
 *   dw_gate   device float [N][d] (written);  dbias: device float [N] or NULL
 *   ws        device scratch of bfmoe_backward_workspace_size(d, N, T, k)
 *             bytes, 256-byte aligned
 * Returns BFMOE_EINVAL / BFMOE_EWORKSPACE on bad arguments (nothing launched);
 * routing indices out of range are reported through the device error word.
 */
int bfmoe_backward(const bfmoe_layer* layer, const void* x, int x_dtype, int T, int k, const float* w_gate,
                   const int32_t* idx, const float* gates, const int32_t* offsets, const int32_t* rows,
                   const float* gy, float* dx, float* dtheta, float* dphi, float* dw_base, float* dalpha,
                   float* dw_gate, float* dbias, void* ws, size_t ws_bytes, bfmoe_stream_t stream);

/* Scratch bytes that bfmoe_backward needs (0 for invalid sizes). */
size_t bfmoe_backward_workspace_size(int d, int n_experts, int T, int k);

/*
 * Add-only expert forward for small batches (decode).  The ternary product
 * of each expert is a signed sum of its inputs (technical summary, 2.3 step
 * 2): this call computes
 *   y_t = sum_j gates[t][j] * B(phi_e) (alpha * W_base (B(theta_e)^T x_t)),
 *   e = idx[t][j], j ascending,
 * decoding the 2-bit codes of W_base in registers and adding, subtracting or
 * skipping each rotated input (no multiplications in the product), with every
 * intermediate in float32 and one rounding of y to x_dtype.  One CTA per
 * token: meant for decode batches (T up to a few hundred), correct for any
 * T >= 0.
 *   layer     as for bfmoe_forward (the prepared tables are not used)
 *   x         device [T][d], dtype x_dtype
 *   idx, gates device [T][k] as written by bfmoe_router_topk (the bucket
 *             arrays are not needed)
 *   y         device [T][d], dtype x_dtype (written)
 * No workspace.  Returns BFMOE_EINVAL on bad arguments (nothing launched);
 * an expert id outside [0, N) is skipped and recorded as
 * BFMOE_EDEVICE_BOUNDS in the device error word.
 */
int bfmoe_decode_forward(const bfmoe_layer* layer, const void* x, int x_dtype, int T, int k,
                         const int32_t* idx, const float* gates, void* y, bfmoe_stream_t stream);

/*
 * Form expert e densely, alpha * B(phi_e) . W_base . B(theta_e)^T, in float32
 * (technical summary, 2.1).  For checking only.
 *   w_out     device float [d][d] (written), row = output
 */
int bfmoe_materialize_expert(const bfmoe_layer* layer, int e, float* w_out,
                             bfmoe_stream_t stream);

/* Scratch bytes that bfmoe_router_topk and bfmoe_forward need for these
 * sizes (one buffer serves both; calls on one stream may share it).
 * Returns 0 for invalid sizes. */
size_t bfmoe_workspace_size(int d, int n_experts, int T, int k, int x_dtype);

/* Scratch bytes that bfmoe_router_topk alone uses for these sizes (the part
 * of bfmoe_workspace_size the router touches; it depends on the path taken:
 * the CUDA-core router of float32 tokens, or of d not a multiple of 64, also
 * keeps the float32 logits [T][N]).  bfmoe_router_topk_noalloc accepts the
 * sizes for which this is at most BFMOE_NOALLOC_SCRATCH_BYTES.  Returns 0 for
 * invalid sizes. */
size_t bfmoe_router_scratch_size(int d, int n_experts, int T, int k, int x_dtype);

/* Thread-local description of the last failed call ("" if none). */
const char* bfmoe_last_error(void);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device.  Returns BFMOE_OK, BFMOE_EDEVICE_TIMEOUT,
 * BFMOE_EDEVICE_BOUNDS or BFMOE_ECUDA. */
int bfmoe_check_device_error(bfmoe_stream_t stream);

/* ---- tracing ------------------------------------------------------------ */

/* Number of kernels this library has launched in this process. */
unsigned long long bfmoe_launch_count(void);

typedef struct {
  char name[48];        /* kernel name                              */
  int launches;         /* launches recorded since profiling began  */
  double total_ms;      /* summed device time (CUDA events)          */
} bfmoe_kernel_time;

/* While enabled, every launch is bracketed by two CUDA events recorded on
 * its own stream.  Enabling discards earlier records. */
int bfmoe_profile_enable(int on);

/* Synchronises the recorded events and writes per-kernel totals
 * (at most `max` entries; *n_out = entries written).  Clears the records. */
int bfmoe_profile_collect(bfmoe_kernel_time* out, int max, int* n_out);

#ifdef __cplusplus
}
#endif

#endif /* BFMOE_H */
