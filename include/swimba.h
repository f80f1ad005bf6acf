/*
 * swimba.h -- C ABI of libswimba.so: the forward pass of one Swimba (Switch Mamba) token-mixer layer
 * on an NVIDIA B200 (sm_100a).
 *
 * The method ("Swimba: Switch Mamba Model Scales State Space Models", arXiv 2603.06938; the
 * papernotes.org NeurIPS 2026 notes, Method, key design 1, and the gist.science Technical Summary,
 * section 2 "Architecture Details"):
 *   router        g_t = W_r X_t,  K_t = top-k of g_t,  pi_t = softmax over K_t (renormalised)
 *   experts       z_t^(e) = W_exp[e] X_t, split into x^(e) (H x P), B^(e) (G x N), C^(e) (G x N)
 *   mixing        U~_t = sum_{e in K_t} pi_te B^(e) x^(e)T,   C~_t = sum_{e in K_t} pi_te C^(e)
 *   recurrence    h_t = a_t h_{t-1} + U~_t,  y_t = C~_t^T h_t,  a_t = exp(dt_t A_h) shared by all experts
 *   dt            dt_t,h = clamp(softplus(W_dt[h] . X_t + b_dt[h]), 1e-3, 0.1)
 *
 * Conventions for every entry point
 *  - Every pointer is caller-owned DEVICE memory unless stated; the library allocates no device memory
 *    (swimba_layer_fwd_host creates two copy streams and a few events once per device).
 *  - Tensors are dense, row-major (last index fastest) and 16-byte aligned.
 *  - M = batch * seqlen tokens; row m = b * seqlen + t.  W_e = H*P + 2*G*N.
 *  - dtype (swimba_dims.dtype) is the type of X, of the three weight matrices and of y.  dt, topk_w,
 *    b_dt, A and every SSM state are fp32.  The mixed streams (Bpi, Xs, Cpi) use the "stream dtype"
 *    (swimba_stream_dtype): fp32 when dtype is F32, fp16 when dtype is BF16 (fp16 keeps 11 bits,
 *    which the 2e-3 accuracy budget of bf16 outputs needs; bf16 streams would not meet it).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).  SWIMBA_OK
 *    means "validated and launched".  Device-side conditions (a bounded wait that gave up, an
 *    intermediate that left the fp16 range) are recorded in a sticky per-device status word and
 *    read with swimba_check_device_status.  No C++ exception crosses this boundary.
 *  - Invalid arguments return an error before anything is launched; unsupported shapes return
 *    SWIMBA_ERR_UNSUPPORTED (there is no fallback path).
 *  - Supported shapes: N, P in {16, 32, 64, 128}; chunk in {64, 128, 256}; 1 <= top_k <= min(E, 8);
 *    E <= 64; G divides H; d_model a multiple of 64 (bf16) or 8 (fp32); every size >= 1.
 *  - Supported values (bf16 layers): every mixed-stream value (x, pi*B, pi*C) and every carried state
 *    element must stay within the fp16 range (|v| <= 65504); a value outside it is recorded as
 *    SWIMBA_ERR_RANGE and the layer's outputs are then not valid.  There is no wider-range path.
 *  - Chunk length: `chunk` fixes where chunk_states are reported.  The tensor-core scan (bf16, N = 128,
 *    P in {64, 128}) always solves in 128-token sub-chunks, which gives the same result up to rounding
 *    for every chunk; the CUDA-core scan (fp32 layers and the other shapes) solves in `chunk`-token chunks.
 */
#ifndef SWIMBA_H_
#define SWIMBA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SWIMBA_OK = 0,
  SWIMBA_ERR_INVALID_ARG = 1,  /* null or misaligned pointer, non-positive size, inconsistent dims */
  SWIMBA_ERR_UNSUPPORTED = 2,  /* valid but outside the supported shapes listed above */
  SWIMBA_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed */
  SWIMBA_ERR_WORKSPACE = 4,    /* ws is NULL or smaller than swimba_workspace_size() */
  SWIMBA_ERR_TIMEOUT = 5,      /* device: a bounded wait gave up (read via swimba_check_device_status) */
  SWIMBA_ERR_RANGE = 6,        /* device: a mixed-stream value did not fit the stream dtype */
  SWIMBA_ERR_INDEX = 7,        /* device: a caller-given expert index lay outside [0, E) */
  SWIMBA_ERR_UNSTABLE = 8      /* device: an expert-mixed transition A~ was not negative (no contraction) */
} swimba_status;

typedef enum { SWIMBA_F32 = 0, SWIMBA_BF16 = 1, SWIMBA_F16 = 2 } swimba_dtype;

typedef struct {
  int32_t batch;      /* B: independent sequences */
  int32_t seqlen;     /* T: tokens per sequence (1 for swimba_step) */
  int32_t d_model;    /* D: width of X */
  int32_t nheads;     /* H */
  int32_t headdim;    /* P: width of x per head and of y per head */
  int32_t dstate;     /* N: state dimension (width of B and C) */
  int32_t ngroups;    /* G: heads h share the B/C of group h / (H/G); G = H gives every head its own */
  int32_t n_experts;  /* E */
  int32_t top_k;      /* k: active experts per token */
  int32_t chunk;      /* Q: SSD chunk length */
  int32_t dtype;      /* swimba_dtype of X, weights and y: SWIMBA_F32 or SWIMBA_BF16 */
} swimba_dims;

typedef struct {
  const void* w_router;  /* [E][D] dtype: router logits g = W_r X */
  const void* w_dt;      /* [H][D] dtype: shared dt projection */
  const float* b_dt;     /* [H] fp32 */
  const float* A;        /* [H] fp32, negative: a_t = exp(dt_t A_h) */
  const void* w_exp;     /* [E][W_e][D] dtype: expert projections, rows [x: H*P | B: G*N | C: G*N] */
  /* [E][H] fp32 or NULL.  When given, the transition is mixed in parameter space like B and C
   * (notes, limitations and outlook: the mixing extended to the diagonal of A under Lyapunov stability):
   * A~_t,h = sum_j pi_tj A_exp[K_tj][h] and a_t = exp(dt_t A~_t,h); A is then not read.  Every entry must
   * be negative, so that each A~ is negative and 0 < a_t < 1 (one contracting trajectory); an A~ that is
   * not negative is recorded as SWIMBA_ERR_UNSTABLE.  Read by swimba_layer_fwd, swimba_layer_fwd_host and
   * swimba_step; the stage entry points (swimba_ssd_scan, swimba_separated_scan) take the shared form
   * dt * A only: pass dt_t * A~_t as dt with A = 1 there. */
  const float* A_exp;
} swimba_weights;

/* Bytes of workspace that every entry point taking `ws` needs for these dims (0 if the dims are
 * invalid or unsupported).  The workspace is scratch owned by the caller; its contents need no
 * initialisation and are overwritten by each call.  Calls that share a workspace must not overlap. */
size_t swimba_workspace_size(const swimba_dims* dims);

/* Stream dtype of the mixed streams for these dims: SWIMBA_F32 or SWIMBA_F16 (-1 if invalid). */
int swimba_stream_dtype(const swimba_dims* dims);

/* Router and dt (one launch).  Paper: notes, Method, flowchart "token router R(X_t)" and key
 * design 1 (pi_t = softmax(g_t), active set K_t).
 *   X        [M][D] dtype
 *   topk_idx [M][k] int32 out: expert indices, largest logit first, equal logits -> lower index
 *   topk_w   [M][k] fp32 out: renormalised softmax weights over the k winners (sum to 1)
 *   dt       [M][H] fp32 out: clamp(softplus(W_dt X + b_dt), 1e-3, 0.1)
 * Logits are accumulated in fp32; the top-k decision is taken on those fp32 values. */
swimba_status swimba_router_topk(const swimba_dims* dims, const void* X, const swimba_weights* w,
                                 int32_t* topk_idx, float* topk_w, float* dt, void* stream);

/* Expert dispatch: a stable counting sort of the M*k (token, slot) pairs by expert (the token-level
 * routing the notes' efficiency discussion attributes Swimba's extra cost to).
 *   topk_idx       [M][k] int32 in, every value in [0, E)
 *   expert_offsets [E+1] int32 out: pairs of expert e are perm[expert_offsets[e] .. expert_offsets[e+1])
 *   perm           [M*k] int32 out: value m*k + j, in increasing m within each expert
 * A pair whose index lies outside [0, E) is left out of the sort (expert_offsets[E] then counts only the
 * valid pairs and perm's tail is not written) and SWIMBA_ERR_INDEX is recorded in the status word. */
swimba_status swimba_dispatch(const swimba_dims* dims, const int32_t* topk_idx, int32_t* expert_offsets,
                              int32_t* perm, void* ws, size_t ws_bytes, void* stream);

/* Expert dispatch that allocates nothing and takes no workspace.  The paper has no counterpart: this entry
 * point is for callers that cannot give the library scratch memory -- plugin-style hosts whose interface
 * hands an operator only its inputs and outputs, and runtimes that plan all device memory at start-up and
 * refuse allocations afterwards.  Same arguments (minus the workspace; topk_idx values in [0, E)), the
 * same status codes and the same results as swimba_dispatch.  Its scratch is one fixed 1 MiB array inside the library, held on every device that
 * loads the library until the process exits; a shape that needs more (about 0.56 * M * k bytes with 64
 * experts, 0.125 * M * k with 8) returns SWIMBA_ERR_WORKSPACE before launching anything.  The first call on
 * a device looks up the array's device address with that device current; make that first call before
 * any stream capture.  All calls share the array and it keeps the last call's contents (nothing in it
 * needs clearing: each call writes every word it reads); calls whose work overlaps on the GPU race. */
swimba_status swimba_dispatch_noalloc(const swimba_dims* dims, const int32_t* topk_idx, int32_t* expert_offsets,
                                      int32_t* perm, void* stream);

/* Expert projections of the active experts, unmixed (a stage probe; the fused path never writes them).
 * Paper: notes, key design 1 ("each expert applies its own linear projection to X_t").
 *   Z [M][k][W_e] fp32 out: Z[m][j] = W_exp[topk_idx[m][j]] X_m, accumulated in fp32. */
swimba_status swimba_expert_proj(const swimba_dims* dims, const void* X, const swimba_weights* w,
                                 const int32_t* topk_idx, float* Z, void* ws, size_t ws_bytes, void* stream);

#define SWIMBA_MIX_UNSCALED_B 1 /* flag: write B unscaled (the separated design's injection) */

/* Parameter-space mixing of unmixed projections (a stage probe of the epilogue the fused path runs).
 * Paper: notes, key design 1, first display equation.  U~ is kept factored per slot:
 *   Bpi [M][k][G][N] stream dtype out: pi_mj B^(j)  (B^(j) itself with SWIMBA_MIX_UNSCALED_B)
 *   Xs  [M][k][H][P] stream dtype out: x^(j)
 *   Cpi [M][k][G][N] stream dtype out: pi_mj C^(j)    (so C~_m = sum_j Cpi[m][j])
 * Values outside the stream dtype's range set SWIMBA_ERR_RANGE in the device status word. */
swimba_status swimba_mix(const swimba_dims* dims, const float* Z, const float* topk_w, int32_t flags,
                         void* Bpi, void* Xs, void* Cpi, void* stream);

/* The single shared-transition recurrence over the mixed streams, solved by chunks of `chunk` tokens.
 * Paper: notes, key design 1, second display equation; overall framework (chunked SSD, reused as is).
 *   Bpi, Xs, Cpi  as written by swimba_mix; dt [M][H] fp32; A [H] fp32
 *   init_state    [B][H][N][P] fp32 or NULL (zero initial state)
 *   y             [M][H][P] dtype out
 *   final_state   [B][H][N][P] fp32 out, or NULL
 *   chunk_states  [B][H][nc][N][P] fp32 out (state before each chunk, nc = ceil(T/chunk)), or NULL */
swimba_status swimba_ssd_scan(const swimba_dims* dims, const void* Bpi, const void* Xs, const void* Cpi,
                              const float* dt, const float* A, const float* init_state, void* y,
                              float* final_state, float* chunk_states, void* ws, size_t ws_bytes, void* stream);

/* Test hook for failure detection (no counterpart in the paper): runs the tensor-core scan as if the
 * first sub-chunk of every (sequence, head) had been lost -- the work counter starts past those
 * sub-chunks, so nothing ever publishes their end states.  Their successors' bounded waits run out
 * (about a second), record SWIMBA_ERR_TIMEOUT in the status word and continue from a zero state; the
 * later sub-chunks complete normally.  No fault, no hang: swimba_check_device_status() then returns
 * SWIMBA_ERR_TIMEOUT and the context stays usable.  Arguments as swimba_ssd_scan (no states); needs a
 * shape the tensor-core scan covers and seqlen > 128 (else SWIMBA_ERR_UNSUPPORTED). */
swimba_status swimba_debug_scan_lost_first_chunk(const swimba_dims* dims, const void* Bpi, const void* Xs,
                                                 const void* Cpi, const float* dt, const float* A, void* y,
                                                 void* ws, size_t ws_bytes, void* stream);

/* The whole layer: router -> dispatch -> expert projections with the mix fused into their epilogue
 * -> chunked scan.  Paper: notes, Method flowchart.
 *   X [M][D] dtype; init_state [B][H][N][P] fp32 or NULL; y [M][H][P] dtype out;
 *   final_state [B][H][N][P] fp32 out or NULL; topk_idx_out [M][k] / topk_w_out [M][k] or NULL. */
swimba_status swimba_layer_fwd(const swimba_dims* dims, const void* X, const swimba_weights* w,
                               const float* init_state, void* y, float* final_state, int32_t* topk_idx_out,
                               float* topk_w_out, void* ws, size_t ws_bytes, void* stream);

/* The whole layer for inputs and outputs in host memory (no counterpart in the paper; a serving
 * convenience).  The batch is split into `chunks` groups of consecutive sequences; group c's X rows are
 * copied host -> device, its layer forward runs on `stream`, and its y rows are copied device -> host,
 * the three kinds of work for different groups overlapping on library-owned copy streams (created once
 * per device) with events between them.  `stream` waits for the last copy before any later work on it.
 *   X_host [M][D] dtype, pinned host memory; y_host [M][H][P] dtype, pinned host memory, out
 *   X_dev, y_dev: device staging buffers of the same sizes (caller-owned)
 *   init_state / final_state: device [B][H][N][P] fp32 or NULL, as for swimba_layer_fwd
 *   ws: workspace sized for the full dims; chunks in [1, 16], clamped to the batch
 * With final_state given the groups are time segments instead: whole 128-token sub-chunks of every
 * sequence, chained through final_state (which then also carries the state between segments); the staging
 * buffers then hold the groups one after another ([batch][segment] rows each).
 * Returns SWIMBA_ERR_INVALID_ARG for null or misaligned pointers; the result is complete once `stream`
 * reaches the point after this call (synchronise `stream` before reading y_host).  The copy streams are
 * shared by all calls on a device: calls that may overlap in time must come from one host thread. */
swimba_status swimba_layer_fwd_host(const swimba_dims* dims, const void* X_host, const swimba_weights* w,
                                    const float* init_state, void* y_host, float* final_state, void* X_dev,
                                    void* y_dev, void* ws, size_t ws_bytes, int chunks, void* stream);

/* One recurrent decode step (dims.seqlen must be 1): each of `batch` sequences takes one token.
 * Paper: notes, key design 1, second display equation advanced by a single token (h_t = a_t h_{t-1} +
 * U~_t, y_t = C~_t^T h_t with the cached h_{t-1}); router, experts and mixing as in swimba_layer_fwd.
 *   X [B][D] dtype; state [B][H][N][P] fp32, updated in place (h <- a h + U~); y [B][H][P] dtype out;
 *   topk_idx_out [B][k] or NULL. */
swimba_status swimba_step(const swimba_dims* dims, const void* X, const swimba_weights* w, float* state,
                          void* y, int32_t* topk_idx_out, void* ws, size_t ws_bytes, void* stream);

/* The separated-trajectory contrast design restricted to the active slots ("k scans"): slot j keeps
 * its own state, driven by the unscaled injection B^(j) x^(j)T and read out with pi_j C^(j):
 *   h^(j)_t = a_t h^(j)_{t-1} + B_tj x_tj^T,   y_t = sum_j Cpi_tj^T h^(j)_t.
 * Paper: notes, key design 1 (separated SSMs cost O(T E C_step)) and the efficiency table.
 *   B [M][k][G][N] (swimba_mix with SWIMBA_MIX_UNSCALED_B), Xs, Cpi, dt, A as for swimba_ssd_scan
 *   init_states [k][B][H][N][P] fp32 or NULL; y [M][H][P] dtype out; final_states same shape or NULL. */
swimba_status swimba_separated_scan(const swimba_dims* dims, const void* B, const void* Xs, const void* Cpi,
                                    const float* dt, const float* A, const float* init_states, void* y,
                                    float* final_states, void* ws, size_t ws_bytes, void* stream);

/* Bytes of workspace swimba_layer_bwd needs for these dims (0 if invalid or unsupported): the layer's own
 * workspace followed by fp32 gradient buffers (about M*k*(W_e + G*N + H*P + D)*4 bytes more) and, for bf16
 * layers, the tensor-core products' operands (about (M*k + 64*E)*(2*W_e + D)*2 bytes). */
size_t swimba_layer_bwd_workspace_size(const swimba_dims* dims);

/* Gradients of the whole layer (swimba_layer_fwd with the shared A) for L = sum_t <dy_t, y_t>: the
 * vector-Jacobian product with the upstream gradient dy.  Paper: notes, Method flowchart differentiated
 * stage by stage in reverse (the notes train the model: loss function / training strategy).  The router's
 * active set is recomputed and held fixed (a top-k choice has no gradient); the dt clamp passes the gradient
 * only strictly inside [1e-3, 0.1].
 *   X [M][D] dtype, weights as for swimba_layer_fwd (A_exp must be NULL: SWIMBA_ERR_UNSUPPORTED otherwise),
 *   init_state [B][H][N][P] fp32 or NULL; dy [M][H][P] fp32
 *   dX [M][D], dW_router [E][D], dW_dt [H][D], db_dt [H], dA [H], dW_exp [E][W_e][D] fp32 out;
 *   d_init [B][H][N][P] fp32 out or NULL
 * Runs the forward's router, dispatch and projections again, the scan gradients, then fp32 kernels for the
 * mix, router and dt gradients.  The expert products dz W_e and dz^T X run on the tensor cores for bf16
 * layers (dz split into bf16 hi + lo, two MMAs into one fp32 accumulator: fp32-class accuracy) and on CUDA
 * cores in fp32 for fp32 layers; the router and dt products on CUDA cores.  ws must hold
 * swimba_layer_bwd_workspace_size(dims) bytes (SWIMBA_ERR_WORKSPACE otherwise); a device status of
 * SWIMBA_ERR_TIMEOUT means a bounded wait of the tensor-core kernel gave up (outputs invalid). */
swimba_status swimba_layer_bwd(const swimba_dims* dims, const void* X, const swimba_weights* w,
                               const float* init_state, const float* dy, float* dX, float* dW_router, float* dW_dt,
                               float* db_dt, float* dA, float* dW_exp, float* d_init, void* ws, size_t ws_bytes,
                               void* stream);

/* Gradients of the chunked scan (swimba_ssd_scan over all k key and read slots) for the loss
 * L = sum_t <dy_t, y_t>, i.e. the vector-Jacobian product with an upstream gradient dy.  Paper: notes,
 * key design 1, second display equation differentiated in reverse (the notes train the model: loss
 * function / training strategy); the adjoint state runs backwards through the same transition a_t.
 *   Bpi, Xs, Cpi, dt, A, init_state  as for swimba_ssd_scan (init_state may be NULL: zero)
 *   dy      [M][H][P] fp32: upstream gradient of y
 *   dBpi    [M][k][G][N] fp32 out     dXs [M][k][H][P] fp32 out
 *   dCt     [M][G][N] fp32 out: gradient of C~ = sum_j Cpi_j (every slot's Cpi receives it)
 *   d_dt    [M][H] fp32 out           dA [H] fp32 out (summed over tokens and sequences)
 *   d_init  [B][H][N][P] fp32 out or NULL
 * fp32 values and accumulation over 64-token sub-chunks: for fp16 streams with N = 128 and P in {64, 128} the
 * sub-chunk end states and adjoint sources run on the tensor cores (fp16 stream operands, the other operand as
 * an fp16 hi + lo pair under a power-of-two scale), everything else on CUDA cores (the gradient kernel takes
 * up to 226 KB of shared memory at N = P = 128); needs the layer workspace (the same dims'
 * swimba_workspace_size).  A device status of SWIMBA_ERR_TIMEOUT means a bounded wait of the tensor-core
 * kernels gave up (outputs invalid). */
swimba_status swimba_ssd_scan_bwd(const swimba_dims* dims, const void* Bpi, const void* Xs, const void* Cpi,
                                  const float* dt, const float* A, const float* init_state, const float* dy,
                                  float* dBpi, float* dXs, float* dCt, float* d_dt, float* dA, float* d_init,
                                  void* ws, size_t ws_bytes, void* stream);

/* The layer's output projection: out = y W_out^T, one projection shared by every expert (the layer has one
 * recurrence and one readout).  Paper: gist.science Technical Summary, Architecture Details (the shared
 * recurrence "followed by a single output projection").
 *   y      [M][H*P] dtype in, as written by swimba_layer_fwd / swimba_ssd_scan / swimba_step
 *   w_out  [D][H*P] dtype in (D = d_model)
 *   out    [M][D] dtype out
 * Only batch*seqlen, nheads*headdim, d_model and dtype are read from `dims`; the other fields must still be
 * valid.  bf16: tensor cores, bf16 operands, fp32 accumulation, one rounding to bf16 per output.  fp32: CUDA
 * cores in fp32.  Needs no workspace; y and out must not overlap.  Pointers must be non-NULL and 16-byte
 * aligned (SWIMBA_ERR_INVALID_ARG otherwise). */
swimba_status swimba_out_proj(const swimba_dims* dims, const void* y, const void* w_out, void* out, void* stream);

/* Synchronises `stream`, then reads and clears the current device's status word: SWIMBA_OK,
 * SWIMBA_ERR_TIMEOUT, SWIMBA_ERR_RANGE, SWIMBA_ERR_INDEX or SWIMBA_ERR_UNSTABLE, in that order of
 * precedence (SWIMBA_ERR_CUDA if the stream reports an error).  The word is sticky: it collects every flag raised on this device
 * since the previous check.  Its device address is looked up once per device; a device reset between
 * calls into the library is not supported. */
swimba_status swimba_check_device_status(void* stream);

/* Profiling support.  swimba_profile_enable(1) makes every later entry-point call record a CUDA
 * event on its stream after each kernel stage; swimba_profile_read then waits for the most recent
 * call's events and writes up to `max` stage names (static strings) and durations in milliseconds,
 * returning the number of stages (-1 on a CUDA error).  swimba_launch_count returns the number of
 * kernels this library has launched in the process so far (all devices). */
swimba_status swimba_profile_enable(int enable);
int swimba_profile_read(const char** names, float* ms, int max);
long long swimba_launch_count(void);

/* Static, human-readable name of a status code. */
const char* swimba_status_string(swimba_status s);

#ifdef __cplusplus
}
#endif

#endif /* SWIMBA_H_ */
