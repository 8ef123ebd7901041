/*
 * bfmoe.h -- C ABI of the ButterflyMoE expert-layer forward for NVIDIA B200
 * (sm_100a).
 *
 * The method (ButterflyMoE: Sub-Linear Ternary Experts via Structured
 * Butterfly Orbits, gist.science summaries of paper 2601.13563, section 2
 * "Methodology" / 2.1 "Mathematical formulation"; ButterflyViT, paper
 * 2603.06746, section 2): every expert i is
 *
 *     W_i = alpha * B(phi_i) . W_base . B(theta_i)^T
 *
 * with ONE shared ternary matrix W_base (entries in {-1, 0, +1}) and two
 * orthogonal butterfly matrices per expert, each a product of log2 d layers
 * of Givens rotations ((d/2) log2 d angles).  W_i is never formed: a routed
 * token is rotated by B(theta)^T, multiplied by W_base, rotated by B(phi)
 * and weighted by its gate.  A standard top-k gate picks the experts
 * (ButterflyMoE summary, Dutch page, section 2 "Three phases").  alpha is not
 * on the pages; the packed base carries it.
 *
 * Conventions (fixed here once; the pages leave them open):
 *   L = log2 d.  Angle tables are fp32 [N][L][d/2], row major.
 *   Stage s (0 <= s < L) rotates the pairs (j, j + 2^s) for every j whose bit
 *   s is clear, with pair index p = (j >> (s+1)) * 2^s + (j & (2^s - 1)):
 *       y_j       = cos(a) x_j - sin(a) x_{j+2^s}
 *       y_{j+2^s} = sin(a) x_j + cos(a) x_{j+2^s},      a = angles[e][s][p].
 *   B = stage_{L-1} ... stage_0 (stage 0 acts first); B^T runs the stages
 *   from L-1 down to 0 with negated angles.
 *   Top-k: larger logit first, ties to the lower expert index (-0 == +0,
 *   +-inf ordinary values); a NaN logit is an error (BFMOE_ERR_NONFINITE).
 *   Gate g_{t,j}: softmax over the k selected logits (its limit if one is
 *   infinite: equal shares of the +inf entries; 1/k if all are -inf).
 *   Bucketing: the T*k routed rows i = t*k + j are sorted by (expert, t);
 *   perm[pos] = i and offsets[e] = first position of expert e,
 *   offsets[N] = T*k.
 *
 * Ownership and streams: every pointer argument is device memory owned by
 * the caller unless stated otherwise; the library never allocates device
 * memory and keeps no per-call state.  `stream` is a cudaStream_t passed as
 * void* (NULL = legacy default stream); every call is asynchronous on it
 * unless stated otherwise.
 *
 * Errors: argument checks run on the host before anything is launched and
 * return an error code at once.  Errors that only the device can see (NaN
 * logits, fp16 overflow of a rotated row, a malformed packed base, a wait
 * that timed out) are written to a status word at the start of the
 * workspace; read it with bfmoe_sync_status.  Each call clears the status
 * word when it starts.  A failed kernel launch returns BFMOE_ERR_CUDA.
 *
 * Workspaces: the first 32 bytes hold the status word and the routing's
 * grid-barrier words.  Their content on a workspace's first use does not
 * matter (the routing clears them on a launch it has not seen), and every
 * call leaves them ready for the next one, so no call clears them with a
 * separate copy.  Calls that share a workspace must be ordered (one stream,
 * or events).
 *
 * Launch overlap: the kernels of a call are chained with programmatic
 * dependent launch, and bfmoe_forward's first kernel (the weight
 * preparation) may start as soon as the previous kernel on the stream allows
 * its dependents to launch.  It reads theta, phi and the packed base (and
 * writes the workspace's cos/sin tables and decoded base, which only this
 * call's later kernels read) before it waits for that kernel; x, the logits
 * and the routing results are touched only after the wait (x is merely
 * prefetched into L2 before it).  So the kernel just before a forward must not write
 * theta, phi or the packed base if it triggers its dependents early
 * (griddepcontrol.launch_dependents); kernels that never do, and any
 * event, copy or other kernel in between, keep plain stream order.
 *
 * Limits: d is a power of two in [64, 4096]; 1 <= N <= 4096;
 * 1 <= k <= min(N, 8); 1 <= T <= 2^24 / k; x and y are fp32 or bf16,
 * 16-byte aligned; workspaces are 256-byte aligned.
 */
#ifndef BFMOE_H
#define BFMOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BFMOE_API __attribute__((visibility("default")))
#else
#define BFMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BFMOE_OK = 0,
    BFMOE_ERR_INVALID_ARG = 1,  /* bad size, pointer, alignment or value */
    BFMOE_ERR_UNSUPPORTED = 2,  /* valid but outside the supported limits */
    BFMOE_ERR_WORKSPACE = 3,    /* workspace too small */
    BFMOE_ERR_NONFINITE = 4,    /* NaN logit or fp16 overflow (device side) */
    BFMOE_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up */
    BFMOE_ERR_CUDA = 6          /* a CUDA runtime call or launch failed */
} bfmoe_status;

typedef enum { BFMOE_F32 = 0, BFMOE_BF16 = 1 } bfmoe_dtype;

/* Human-readable name of a status code (static string, never NULL). */
BFMOE_API const char *bfmoe_status_string(bfmoe_status s);

/* Library version as 10000*major + 100*minor + patch. */
BFMOE_API int bfmoe_version(void);

/* ------------------------------------------------------------ packing -- */

/* Bytes of a packed base for width d: 16-byte header + d*d/4 (2 bits per
 * weight).  Returns 0 for an unsupported d. */
BFMOE_API size_t bfmoe_packed_base_bytes(int d);

/* Pack the shared ternary substrate W_base (ButterflyMoE summaries, section
 * 2: one matrix of entries in {-1, 0, +1}, about 1.58 bits per weight) at 2
 * bits per weight, with the scale alpha.
 *   w:      device, int8 [d][d] row major, values in {-1, 0, +1}.
 *   packed: device, bfmoe_packed_base_bytes(d) bytes, 16-byte aligned.
 * Layout: header {u32 magic 0x32574642 "BFW2", u32 d, f32 alpha, u32 1},
 * then d*d/16 little-endian u32 words, row major; word w of row r holds
 * columns 16w..16w+15, column c in bits 2(c mod 16)+1..2(c mod 16);
 * codes 00 = 0, 01 = +1, 11 = -1 (10 is never written and reads as 0).
 * SYNCHRONISES `stream`: returns BFMOE_ERR_INVALID_ARG if any value of w is
 * outside {-1, 0, +1} (packed is then unspecified).  Done once per model. */
BFMOE_API bfmoe_status bfmoe_pack_base(const int8_t *w, int d, float alpha, void *packed, void *stream);

/* ------------------------------------------------------------ routing -- */

/* Workspace bytes for bfmoe_route. */
BFMOE_API size_t bfmoe_route_workspace_bytes(int T, int N, int k);

/* Top-k gate and bucketing over given router logits (the router network
 * that produces them is outside this library).
 *   logits:   device fp32 [T][N].
 *   topk_idx: device int32 [T][k] out, selection order (best first).
 *   gates:    device fp32 [T][k] out.
 *   perm:     device int32 [T*k] out; offsets: device int32 [N+1] out.
 *   ws:       device workspace of bfmoe_route_workspace_bytes(T, N, k);
 *             its first 4 bytes are the status word.
 * Device-side error: BFMOE_ERR_NONFINITE on a NaN logit (outputs are then
 * still a valid routing, with NaN treated as -inf). */
BFMOE_API bfmoe_status bfmoe_route(const float *logits, int T, int N, int k, int32_t *topk_idx, float *gates,
                         int32_t *perm, int32_t *offsets, void *ws, size_t ws_bytes, void *stream);

/* Routing for callers that cannot allocate device memory.  The paper has no
 * counterpart: this is a deployment variant of bfmoe_route.
 *
 * Some callers have no way to obtain device memory on the path where they
 * route: a plugin running inside a host framework that owns every
 * allocation, a real-time loop where allocation is forbidden, or code that
 * only receives device pointers for its inputs and outputs.  This entry
 * point takes no workspace: its scratch (status word, grid-barrier counter,
 * per-block histogram, expert totals) lives in a 1 MiB array inside the
 * library, which every GPU that loads the library holds until the process
 * exits.  It calls no cudaMalloc, cudaFree or allocating routine.
 *   Arguments and results are those of bfmoe_route (all device memory owned
 *   by the caller).
 *   Limits: N <= 510 experts (any T up to the bfmoe_route limit); larger N
 *   returns BFMOE_ERR_UNSUPPORTED.
 *   The first call on a device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   Every call shares the one array: calls that overlap on the GPU (on
 *   different streams, or from different threads) race and give undefined
 *   results; serialise them.  Each call clears the part that must start at
 *   zero.  Device-side errors (a NaN logit, a timed-out barrier) are not
 *   reported: a NaN logit ranks as -inf, so the outputs are still a valid
 *   routing. */
BFMOE_API bfmoe_status bfmoe_route_static(const float *logits, int T, int N, int k, int32_t *topk_idx, float *gates,
                                          int32_t *perm, int32_t *offsets, void *stream);

/* ---------------------------------------------------------- butterfly -- */

/* Workspace bytes for bfmoe_butterfly_apply (the cos/sin table). */
BFMOE_API size_t bfmoe_butterfly_workspace_bytes(int d, int N);

/* Apply each row's expert butterfly: y[r] = B(angles[e_r]) x[r], or
 * B(angles[e_r])^T x[r] when transpose != 0 (ButterflyMoE summaries, section
 * 2 / 2.2: layered Givens rotations; convention above).
 *   x, y:          device [rows][d] of dtype dt (may not alias).
 *   angles:        device fp32 [N][L][d/2].
 *   expert_of_row: device int32 [rows], values in [0, N); NULL means 0.
 *   ws:            device workspace of bfmoe_butterfly_workspace_bytes(d, N).
 * Arithmetic is fp32; the result is rounded to dt (nearest even). */
BFMOE_API bfmoe_status bfmoe_butterfly_apply(const void *x, bfmoe_dtype dt, int rows, int d, int N, const float *angles,
                                   const int32_t *expert_of_row, int transpose, void *y, void *ws,
                                   size_t ws_bytes, void *stream);

/* ------------------------------------------------------------ forward -- */

/* Workspace bytes for bfmoe_forward. */
BFMOE_API size_t bfmoe_forward_workspace_bytes(int T, int d, int N, int k);

/* Byte offsets, inside the forward workspace, of the routing results that
 * bfmoe_forward leaves there (same meaning as bfmoe_route's outputs). */
typedef struct {
    size_t status;    /* uint32 status word */
    size_t topk_idx;  /* int32 [T][k] */
    size_t gates;     /* fp32 [T][k] */
    size_t perm;      /* int32 [T*k] */
    size_t offsets;   /* int32 [N+1] */
    size_t total;     /* == bfmoe_forward_workspace_bytes */
} bfmoe_ws_layout;

BFMOE_API bfmoe_status bfmoe_forward_ws_layout(int T, int d, int N, int k, bfmoe_ws_layout *out /* host */);

/* The expert layer forward (ButterflyMoE summaries, section 2 / 2.1):
 *     y_t = sum_{j<k} g_{t,j} * alpha * B(phi_e) W_base B(theta_e)^T x_t,
 *     e = topk_idx[t][j].
 *   x:           device [T][d] of dtype dt; y: device [T][d] of dtype dt.
 *   logits:      device fp32 [T][N].
 *   packed_base: device, from bfmoe_pack_base with the same d.
 *   theta, phi:  device fp32 [N][L][d/2] (input and output butterflies).
 *   ws:          device workspace of bfmoe_forward_workspace_bytes(T,d,N,k).
 * Precision: rotations and accumulation in fp32; the rotated rows enter the
 * tensor-core contraction as fp16 (W_base's values are exact in fp16); each
 * product row, after the output stages that stay inside one GEMM column tile,
 * is scaled by alpha * g and held as fp16 until the last stages and the sum
 * over j; y is rounded to dt.  Device-side errors: NaN logit, fp16 overflow of
 * a rotated row (|x'| > 65504), non-finite y (fp16 overflow of a scaled
 * product row), malformed packed base, timeout. */
BFMOE_API bfmoe_status bfmoe_forward(const void *x, bfmoe_dtype dt, int T, int d, const float *logits, int N, int k,
                           const void *packed_base, const float *theta, const float *phi, void *y, void *ws,
                           size_t ws_bytes, void *stream);

/* Profiling variant of bfmoe_forward: the same launches, with a CUDA event
 * recorded on `stream` after each kernel; SYNCHRONISES `stream` and writes
 * the duration of each kernel in milliseconds to stage_ms (host array of at
 * least BFMOE_MAX_STAGES floats) and their count to *n_stages.  Stage names
 * come from bfmoe_stage_name.  Not for production use: the events add small
 * gaps between kernels. */
#define BFMOE_MAX_STAGES 16
BFMOE_API bfmoe_status bfmoe_forward_profile(const void *x, bfmoe_dtype dt, int T, int d, const float *logits, int N,
                                             int k, const void *packed_base, const float *theta, const float *phi,
                                             void *y, void *ws, size_t ws_bytes, void *stream,
                                             float *stage_ms /* host */, int *n_stages /* host */);

/* Name of profiling stage i of bfmoe_forward (static string; NULL when i is
 * out of range). */
BFMOE_API const char *bfmoe_stage_name(int i);

/* Test hooks (process-wide, not for production use).
 * BFMOE_DEBUG_SKIP_ARRIVE_BLOCK: the routing block with this index returns
 * before its first grid barrier (-1, the default, disables the hook), so
 * the other blocks' bounded waits run out and the call reports
 * BFMOE_ERR_TIMEOUT through the status word instead of hanging. */
#define BFMOE_DEBUG_SKIP_ARRIVE_BLOCK 1
BFMOE_API void bfmoe_debug_set(int key, int value);

/* Synchronise `stream`, then return (and clear) the status word at the start
 * of `ws` (a route, butterfly or forward workspace). */
BFMOE_API bfmoe_status bfmoe_sync_status(void *ws, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* BFMOE_H */
