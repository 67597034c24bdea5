/*
 * tileq.h — C ABI of the TileQ fused MoE-layer forward for NVIDIA B200 (sm_100a).
 *
 * What it computes (TileQ paper, "TileQ: Efficient Low-Rank Quantization of
 * Mixture-of-Experts with 2D Tiling"):
 *
 *   The K experts of a projection sit on an M x N tile grid.  Expert k at cell
 *   (m, n) applies  W_k = U_m diag(Sigma) V_n^T + deq(Q_k)  where U_m is the
 *   row-m block of the shared left (output-space) factor of the tiled block
 *   matrix W_big, V_n the column-n block of its shared right (input-space)
 *   factor, Sigma the shared diagonal, and deq(Q_k) the expert's 2-bit
 *   group-quantised residual (section 2.1, step 5 and the key technical
 *   insight).  The forward runs the fused low-rank inference of section 2.2
 *   ("Efficient Fused Sparse Low-Rank Inference", LoTileMoE): z = Sigma*(V_n^T x)
 *   is computed once per (token, grid column), U_m is applied per grid row
 *   through an in-place accumulation buffer, and the residual runs as one
 *   grouped GEMM instead of K small ones.
 *
 *   Routing (implicit on the pages: only a few experts are active per token):
 *   top-k of the fp32 router logits in descending order, equal logits -> the
 *   lower expert index first; weights = softmax over the k chosen logits
 *   (route_mode TILEQ_ROUTE_TOPK_SOFTMAX), or the k chosen entries of the
 *   softmax over all K logits, not renormalised (TILEQ_ROUTE_FULL_SOFTMAX).
 *   Section 2.2 ("Mechanism") only says that routing weights select the
 *   active tiles; both normalisations are readings of it.
 *   LINEAR layer:  out_t = sum_j w_j W_{e_j} x_t
 *   SWIGLU layer:  out_t = sum_j w_j W^down_{e_j} (silu(W^gate_{e_j} x_t) * (W^up_{e_j} x_t))
 *                  (+ an optional always-on dense bf16 SwiGLU shared expert, weight 1)
 *
 * Conventions for every call:
 *   - Tensors are caller-owned.  "device" pointers are CUDA global memory of
 *     the current device; "host" pointers are ordinary host memory.  Every
 *     device pointer must be 16-byte aligned.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream)
 *     unless stated otherwise.  Host-side validation errors are returned
 *     before anything is enqueued.  Launch failures return TILEQ_ERR_CUDA.
 *   - The library never allocates device memory: the packed weights and the
 *     workspace are sized by query and passed in.
 *   - Layers with a shared expert: tileq_moe_forward runs the shared expert on
 *     a non-blocking stream of the library's own (one per host thread and
 *     device, with two events, created by the first such call and kept for the
 *     life of the process), forked from `stream` by an event after the routing
 *     and permutation kernels and joined back into `stream` by an event before
 *     the output is formed.  The call's work therefore still follows earlier
 *     work on `stream` and precedes later work on it.  As with
 *     tileq_route_static, make the first such call on a thread and device
 *     before any stream capture begins.  If that stream cannot be created, the
 *     shared expert runs on `stream` itself.
 *   - Outputs are overwritten, never accumulated into.
 *   - Bounded device waits that give up write TILEQ_ERR_TIMEOUT into the
 *     workspace status word (read it with tileq_device_status).
 *   - Numeric range.  The forward computes in fp16 operands with fp32
 *     accumulation: x (bf16) is converted to fp16, and the projected vectors
 *     z and z', and the SwiGLU activation h = w * silu(g) * u, are stored in
 *     fp16.  fp16's finite range is |v| <= 65504 (normal down to 6.1e-5,
 *     subnormal to 6.0e-8).  Any of these values outside the finite range
 *     (including a NaN or infinite input) records TILEQ_ERR_RANGE in the
 *     workspace status word; the output of that forward is then not valid.
 *     Values below the normal range lose relative precision gradually, as
 *     fp16 subnormals.  The output is bf16 (fp32 range).
 */
#ifndef TILEQ_H_
#define TILEQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *tileq_stream_t;

typedef enum {
  TILEQ_OK = 0,
  TILEQ_ERR_INVALID_ARG = -1,  /* null pointer, bad size, non-injective grid, bad top_k   */
  TILEQ_ERR_UNSUPPORTED = -2,  /* shape outside the supported tiling (see tileq_proj)     */
  TILEQ_ERR_WORKSPACE = -3,    /* workspace or packed buffer smaller than the query says  */
  TILEQ_ERR_CUDA = -4,         /* a CUDA runtime call or kernel launch failed             */
  TILEQ_ERR_TIMEOUT = -5,      /* a bounded device wait gave up (device status word)      */
  TILEQ_ERR_RANGE = -6         /* an fp16 internal value left fp16's finite range (device
                                  status word): the output of that forward is not valid  */
} tileq_status;

enum { TILEQ_LINEAR = 0, TILEQ_SWIGLU = 1 };

/* One TileQ-compressed projection (d_out x d_in) of all K experts, in the
 * stored format (section 2.1, steps 4-5):
 *   grid_assign  HOST int32 [K]: cell m*N + n of expert k; must be injective.
 *   U            device bf16 [M*d_out, rank], row-major; block m = rows m*d_out..
 *   Sigma        device fp32 [rank]
 *   V            device bf16 [N*d_in, rank], row-major; block n = rows n*d_in..
 *   codes        device uint32 [K, d_out, d_in/16]; element j of a word at bits 2*(j%16)
 *   scales       device fp16 [K, d_out, d_in/group]
 *   zeros        device uint8 [K, d_out, ceil(d_in/group/4)]; group j at bits 2*(j%4)
 *                of byte j/4
 *   bits         2 (or 0: a zero-initialised struct) or 3 (the summary's section 4,
 *                "Experimental Results", evaluates 2-bit and 3-bit TileQ).  For 3: q = codes + 4 * (bit of codes_hi),
 *                zeros are device uint8 [K, d_out, ceil(d_in/group/2)] with group j
 *                at bits 4*(j%2) of byte j/2 (values 0..7), and
 *   codes_hi     device uint32 [K, d_out, d_in/32], element j at bit j%32 (3-bit only).
 *   Residual: w[o,i] = scales[o,i/group] * (q[o,i] - z[o,i/group]).
 * Supported: d_out % 16 == 0, d_in % 128 == 0, group == 64 or a multiple of 128,
 * d_in % group == 0,
 * 0 <= rank <= 256 and rank % 16 == 0 (rank 0 = residual only), bits in {0, 2, 3};
 * otherwise TILEQ_ERR_UNSUPPORTED. */
typedef struct {
  int d_in, d_out, rank, group;
  const int32_t *grid_assign;
  const void *U;
  const float *Sigma;
  const void *V;
  const uint32_t *codes;
  const void *scales;
  const uint8_t *zeros;
  int bits;
  const uint32_t *codes_hi;
} tileq_proj;

/* A TileQ MoE layer.
 *   kind = TILEQ_LINEAR: proj[0] only; x is [T, proj[0].d_in], out is [T, proj[0].d_out].
 *   kind = TILEQ_SWIGLU: proj[0] = gate (d_ff x d_model), proj[1] = up (d_ff x d_model),
 *                        proj[2] = down (d_model x d_ff); x and out are [T, d_model].
 *   shared_d_ff > 0 adds a dense SwiGLU shared expert (SWIGLU only):
 *   shared_w[0] gate, shared_w[1] up: device bf16 [shared_d_ff, d_model];
 *   shared_w[2] down: device bf16 [d_model, shared_d_ff]; shared_d_ff % 128 == 0.
 *   route_mode: TILEQ_ROUTE_TOPK_SOFTMAX (0, a zero-initialised struct) or
 *   TILEQ_ROUTE_FULL_SOFTMAX; any other value -> TILEQ_ERR_INVALID_ARG.
 *   tileq_route and tileq_route_static always route with mode 0. */
#define TILEQ_ROUTE_TOPK_SOFTMAX 0
#define TILEQ_ROUTE_FULL_SOFTMAX 1
typedef struct {
  int kind;
  int K, M, N;            /* experts and grid; K <= M*N; K, M, N <= 64 */
  int d_model, d_ff;      /* SWIGLU widths (ignored for LINEAR) */
  tileq_proj proj[3];
  int shared_d_ff;
  const void *shared_w[3];
  int route_mode;
} tileq_layer;

/* Optional copies of the routing results (device pointers, each may be NULL). */
typedef struct {
  int32_t *topk_idx;        /* [T, top_k] expert ids, descending logit               */
  float *topk_w;            /* [T, top_k] routing weights (per the layer's route_mode) */
  int32_t *expert_offsets;  /* [K+1] range of each expert in sorted_pairs             */
  int32_t *sorted_pairs;    /* [T*top_k] pair ids t*top_k+j, stably sorted by expert  */
} tileq_route_out;

/* Independent per-expert low-rank factors of one projection (the disjoint
 * per-expert layout the paper compares against, section 1 "Inference
 * Latency"): U_pe device bf16 [K, d_out, rank], V_pe device bf16 [K, d_in, rank]. */
typedef struct {
  const void *U_pe[3];
  const void *V_pe[3];
} tileq_per_expert_lr;

/* Human-readable name of a status code (static string, never NULL). */
const char *tileq_status_string(tileq_status s);

/* Bytes of the packed (kernel-layout) copy of `layer`.  Host only, synchronous. */
tileq_status tileq_packed_size(const tileq_layer *layer, size_t *bytes);

/* Repack `layer` into `packed` (device, packed_bytes >= tileq_packed_size).
 * Reads the layer's device arrays and host grid_assign; validates the grid is
 * injective.  Asynchronous on `stream`; the layer's arrays must stay valid
 * until the stream reaches this call.  Call once per set of weights. */
tileq_status tileq_pack(const tileq_layer *layer, void *packed, size_t packed_bytes,
                        tileq_stream_t stream);

/* Workspace bytes needed by tileq_moe_forward / tileq_route for T tokens. */
tileq_status tileq_workspace_size(const tileq_layer *layer, int T, int top_k, size_t *bytes);

/* The fused TileQ MoE-layer forward (section 2.2).
 *   layer, packed   the descriptor and its packed copy (from tileq_pack)
 *   x               device bf16 [T, d_x]       router_logits  device fp32 [T, K]
 *   out             device bf16 [T, d_y]       (overwritten)
 *   ws, ws_bytes    device workspace, ws_bytes >= tileq_workspace_size(layer, T, top_k)
 *   route           optional copies of the routing results (NULL = none)
 * 1 <= top_k <= K; T >= 0 (T == 0 enqueues nothing).  Asynchronous.
 * Kernel choice: experts averaging <= 32 slots run their residual GEMMs on
 * warp-level MMA, wider ones on tcgen05.  With the environment variable
 * TILEQ_DECODE_TC=1 set when the library makes its first plan, 2-bit layers
 * with groups of a multiple of 128 run the narrow case on the tcgen05 decode
 * kernel instead (same results within the parity bar, measured slower). */
tileq_status tileq_moe_forward(const tileq_layer *layer, const void *packed, const void *x,
                               int T, const float *router_logits, int top_k, void *out,
                               void *ws, size_t ws_bytes, tileq_route_out *route,
                               tileq_stream_t stream);

/* Bytes of the packed copy of a per-expert low-rank layout. */
tileq_status tileq_packed_per_expert_size(const tileq_layer *layer, size_t *bytes);

/* Repack the per-expert factors `pe` (same shapes as layer->proj) into `packed_pe`. */
tileq_status tileq_pack_per_expert(const tileq_layer *layer, const tileq_per_expert_lr *pe,
                                   void *packed_pe, size_t packed_pe_bytes,
                                   tileq_stream_t stream);

/* The unfused comparison path: the same residual GEMMs, but the low-rank term
 * of every expert runs as its own launches from the per-expert layout (K small
 * GEMMs per projection and stage, no sharing across grid rows or columns).
 * Same arguments and result as tileq_moe_forward plus `packed_pe`. */
tileq_status tileq_moe_forward_unfused(const tileq_layer *layer, const void *packed,
                                       const void *packed_pe, const void *x, int T,
                                       const float *router_logits, int top_k, void *out,
                                       void *ws, size_t ws_bytes, tileq_route_out *route,
                                       tileq_stream_t stream);

/* Routing and permutation alone: top-k, softmax weights and the stable
 * counting sort of the T*top_k pairs by expert.  Outputs as in tileq_route_out
 * (all four required).  ws as for tileq_moe_forward (tileq_workspace_size). */
tileq_status tileq_route(const float *router_logits, int T, int K, int top_k,
                         tileq_route_out *route, void *ws, size_t ws_bytes,
                         tileq_stream_t stream);

/* Largest T * top_k that tileq_route_static accepts. */
#define TILEQ_ROUTE_STATIC_MAX_PAIRS 8192

/* Routing and permutation with no workspace argument and no device allocation.
 * The pages have no counterpart for this call: it is a library convenience.
 *
 * Same computation and outputs as tileq_route (all four route outputs
 * required), but the scratch is a fixed 6 MiB array inside the library, one
 * per device, instead of a caller-supplied workspace.  It serves callers that
 * cannot allocate device memory at the point where they route: a C host
 * program that has no device allocator of its own, or a framework hook that
 * runs where its memory pool must not grow.  The call itself never calls
 * cudaMalloc, cudaFree or any other allocating routine.
 *
 *   router_logits  device fp32 [T, K]; 1 <= K <= 64, 1 <= top_k <= min(K, 8)
 *   route          device outputs as in tileq_route_out (all four non-NULL)
 * T * top_k > TILEQ_ROUTE_STATIC_MAX_PAIRS returns TILEQ_ERR_UNSUPPORTED before
 * anything is enqueued; T == 0 enqueues nothing.
 *
 * Set-up: the first call on a device (with that device current) looks up the
 * scratch address and zeroes it, synchronously; make that first call before
 * any stream capture begins.  Later calls are asynchronous on `stream`.
 * All calls on one device share the one scratch array: two calls whose work
 * overlaps on the device (different streams, or different host threads) race
 * and may return wrong results; order them on one stream or with events. */
tileq_status tileq_route_static(const float *router_logits, int T, int K, int top_k,
                                tileq_route_out *route, tileq_stream_t stream);

/* ---------------------------------------------------------------------------
 * Global low-rank decomposition of W_big by Gaussian sketching (TileQ summary,
 * section 2.1, step 5 "Quantization": one low-rank decomposition of the whole
 * tiled matrix, computed by a Gaussian sketch rather than a full SVD, yields
 * the shared factors U, Sigma, V that tileq_moe_forward reads).
 *
 * W_big [M*d_out, N*d_in] holds expert k's weights in grid block
 * (m, n) = (grid_assign[k] / N, grid_assign[k] % N).  Steps (randomised range
 * finder, then the SVD of the projected matrix):
 *   Y = W_big Omega;  Q = an orthonormal basis of range(Y);  B = Q^T W_big;
 *   B = U_B diag(s) V_B^T;  U = Q U_B[:, :r], Sigma = s[:r], V = V_B[:, :r].
 * U diag(Sigma) V^T is the rank-r truncated SVD of Q Q^T W_big.  The GPU
 * computes the basis and the SVD from fp64 Jacobi eigen-decompositions of the
 * l x l Gram matrices Y^T Y and B B^T; products are fp32.
 * ------------------------------------------------------------------------- */
#define TILEQ_SKETCH_MAX_L 160

typedef struct {
  int K, M, N;                  /* K == M * N <= 64: every grid cell holds one expert */
  int d_out, d_in;
  const void *w;                /* device, bf16 [K][d_out][d_in], expert k's weights */
  const int32_t *grid_assign;   /* host, [K], a bijection onto the cells 0..K-1 */
} tileq_wbig;

/* Workspace bytes of tileq_sketch_lowrank.  l: sketch width (even, 2..
 * TILEQ_SKETCH_MAX_L), r: rank (1..l).  TILEQ_ERR_UNSUPPORTED for shapes outside
 * these limits, TILEQ_ERR_INVALID_ARG for a grid_assign that is not a bijection. */
tileq_status tileq_sketch_workspace_size(const tileq_wbig *w, int l, int r, size_t *bytes);

/* omega_t: device bf16 [l][N*d_in], the transpose of the Gaussian test matrix
 * Omega (the caller draws it).  Outputs (device, overwritten): U fp32
 * [M*d_out][r], sigma fp32 [r] (descending), V fp32 [N*d_in][r]; the columns of
 * U and V pair up (the sign of each pair is arbitrary).  ws: device workspace
 * of at least the queried size (it holds, among others, a transposed copy of
 * the experts' weights).  d_out and d_in must be multiples of 128
 * (TILEQ_ERR_UNSUPPORTED).  Asynchronous on stream; the host validates before
 * any launch. */
tileq_status tileq_sketch_lowrank(const tileq_wbig *w, const void *omega_t, int l, int r, float *U,
                                  float *sigma, float *V, void *ws, size_t ws_bytes,
                                  tileq_stream_t stream);

/* ---------------------------------------------------------------------------
 * Expert placement on the M x N grid (TileQ summary, section 2.1, steps 2-4:
 * "Extracting" -- each expert's rank-r0 SVD factors (U_k, V_k), flattened and
 * scaled to unit norm, serve as its feature embeddings; "Clustering" -- K-Means
 * on the U side and on the V side picks a preferred cell (m, n) per expert;
 * "2D-Tiling Placement" -- a greedy pass settles experts that prefer the same
 * cell, keeping each one as near its preferred cell as it can).
 * The result is the grid_assign that W_big, tileq_sketch_lowrank and
 * tileq_pack take.
 *
 * Steps (the pages give no more detail; these are the plainest readings):
 *   embedding: each factor column is multiplied by the sign of its entry of
 *     largest magnitude (the first such row on ties), the factor is flattened
 *     row-major and divided by its L2 norm (a zero factor stays zero);
 *   rows: K-Means on the U-embeddings with min(M, K) clusters; columns:
 *     K-Means on the V-embeddings with min(N, K) clusters (rows of the grid
 *     share the left basis, columns the right basis);
 *   K-Means: Lloyd's algorithm on squared Euclidean distance; first centre =
 *     expert 0, each further centre = the expert farthest from the centres
 *     so far (ties -> lowest index); assignment to the nearest centre (ties
 *     -> lowest centre index); a centre with no experts keeps its place; stop
 *     when an update changes no assignment or after max_iter updates;
 *   greedy: repeatedly place the (unplaced expert, free cell) pair with the
 *     smallest squared grid distance (m - m*)^2 + (n - n*)^2 to the expert's
 *     ideal (m*, n*), ties -> lower expert index, then lower cell m*N + n.
 * The GPU evaluates the K-Means distances from the fp64 Gram matrix of the
 * embeddings, which it builds in one pass over the factors.
 * ------------------------------------------------------------------------- */
#define TILEQ_PLACE_MAX_R0 256
#define TILEQ_PLACE_MAX_ITER 65536

typedef struct {
  int K, M, N;          /* experts and grid: 1 <= K <= M*N; K, M, N <= 64 */
  int d_u, d_v, r0;     /* factor shapes: U_k [d_u][r0], V_k [d_v][r0]; 1 <= r0 <= TILEQ_PLACE_MAX_R0 */
  const float *u;       /* device fp32 [K][d_u][r0], row-major: the left (output-space) factors */
  const float *v;       /* device fp32 [K][d_v][r0]: the right (input-space) factors */
  int max_iter;         /* cap on the K-Means centre updates, 1..TILEQ_PLACE_MAX_ITER */
} tileq_place_in;

typedef struct {
  int32_t *grid_assign; /* device [K]: cell m*N + n of expert k (required) */
  int32_t *ideal;       /* device [K][2]: the ideal (m, n) from the two K-Means, or NULL */
  int32_t *iterations;  /* device [2]: centre updates run on the U side and the V side, or NULL */
} tileq_place_out;

/* Workspace bytes of tileq_place_experts (host only). */
tileq_status tileq_place_workspace_size(const tileq_place_in *in, size_t *bytes);

/* Embeddings, both K-Means and the greedy placement, asynchronous on stream.
 * Shapes outside the limits above -> TILEQ_ERR_UNSUPPORTED, NULL pointers or
 * max_iter < 1 -> TILEQ_ERR_INVALID_ARG, a short workspace ->
 * TILEQ_ERR_WORKSPACE; all checked on the host before any launch.  The factors
 * must stay valid until the stream reaches the call. */
tileq_status tileq_place_experts(const tileq_place_in *in, tileq_place_out *out, void *ws,
                                 size_t ws_bytes, tileq_stream_t stream);

/* Synchronously read (and clear) the device status word in `ws`.
 * *status receives TILEQ_OK or the first device error recorded. */
tileq_status tileq_device_status(void *ws, int *status, tileq_stream_t stream);

/* Self-test of the bounded device wait: launches one block that waits on an
 * mbarrier nothing arrives on, for at most `max_polls` polls, then records
 * TILEQ_ERR_TIMEOUT in the status word of `ws` and returns.  Never hangs. */
tileq_status tileq_selftest_bounded_wait(void *ws, size_t ws_bytes, int max_polls,
                                         tileq_stream_t stream);

/* Per-stage timing hook.  `events` holds n_events CUDA events (cudaEvent_t,
 * caller-created and owned) or is NULL to switch the hook off.  While set,
 * every tileq_moe_forward / tileq_moe_forward_unfused records event i on its
 * stream at stage boundary i: 0 before routing, 1 after routing, 2 after the
 * permutation, 3 after the column projection z = Sigma*(V_n^T x), 4 after the
 * gate/up GEMM (a linear layer: at 3 again), 5 after the down-side projection
 * z' = Sigma*(V_n^T h) (a linear layer: after the per-(token, grid row) sums
 * a_{t,m}), 6 after the shared expert, 7 after the residual GEMM of the down
 * (or linear) projection, 8 after the combine.  Where the shared expert runs
 * on the side stream (see the conventions above), 6 marks the point where
 * `stream` moves on without it: its time overlaps the stages after boundary
 * 2, and the wait for it falls between boundaries 6 and 7 (decode kernel with
 * the fused combine), else between 7 and 8.  tileq_place_experts records 0
 * before its first launch, 1 after the sign pass, 2 after the Gram pass, 3
 * after both K-Means, 4 after the greedy placement.  Events past n_events are
 * skipped.
 * Process-wide, not thread-safe; host only. */
tileq_status tileq_set_stage_events(void **events, int n_events);

/* Number of kernels the library has launched in this process so far. */
tileq_status tileq_launch_count(unsigned long long *count);

#ifdef __cplusplus
}
#endif
#endif /* TILEQ_H_ */
