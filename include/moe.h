/*
 * moe.h - C ABI of libmoe.so, a B200 (sm_100a) MoE-layer forward pass.
 *
 * The layer (shared by DiT-MoE, EC-DiT, MMOE and the DES dLLM block):
 *   router GEMM + softmax      -> affinities A in R^{T x E}
 *   selection                  -> token-choice top-k | expert-choice top-C |
 *                                 DES-Vote or DES-Seq core set + restricted
 *                                 top-K
 *   dispatch                   -> stable permutation into per-expert groups
 *   grouped expert MLP         -> GELU or SwiGLU heavy experts (tcgen05 tensor
 *                                 cores for bf16), shared expert(s); the
 *                                 zero-computation experts issue no FLOPs
 *   combine                    -> y = r + shared + sum_j w_j * expert_j(x)
 *
 * Conventions for every entry point
 *   - Returns an int moe_status (MOE_OK == 0); moe_status_string() names it.
 *     Host-side argument checks run before anything is launched; a failing
 *     check launches nothing.
 *   - Tensor arguments are DEVICE pointers owned by the caller, row-major
 *     and contiguous, unless a parameter says "host". bf16 rows must start
 *     on 16-byte boundaries (row lengths d, h that are multiples of 8).
 *   - Calls are asynchronous on the given stream (NULL = legacy default
 *     stream) and never synchronise the host. Errors found on the device
 *     (an expert or token index out of range, a bounded wait that expired)
 *     are OR-ed into the caller's int32 status word `dev_status` (device
 *     memory, nullable) as MOE_DEV_* bits; the offending item is skipped,
 *     nothing traps.
 *   - The library allocates no memory on a call's path. Scratch comes from
 *     a caller workspace of at least moe_workspace_size() bytes, 256-byte
 *     aligned. Calls that share a workspace must not overlap on the device.
 *     Three exceptions, each documented at its entry point: the
 *     allocation-free dispatch (moe_dispatch_noalloc) keeps its scratch in
 *     one fixed library-owned device array per GPU, shared by all its
 *     calls; moe_forward_host creates two library-owned side streams and
 *     events per device on its first pipelined call; and moe_forward, for
 *     a bf16 layer with a shared expert and routed rows, creates one
 *     library-owned side stream and two events per device on first use.
 *     Both keep them for the life of the process.
 *   - Apart from those and from one-time lookups made safely on first
 *     use, there is no global mutable state: calls on different streams
 *     with different workspaces may run concurrently.
 *
 * Expert ids: heavy (MLP) experts occupy ids [0, n_heavy); ids
 * [n_heavy, E) are zero-computation experts whose kinds are listed in
 * moe_config.expert_kind (MMOE page, "MoE++ expert layer").
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef struct CUstream_st *moe_stream_t; /* a cudaStream_t */

enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, size out of range, misaligned pointer */
  MOE_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. E > 256, not sm_100) */
  MOE_ERR_WORKSPACE = 3,     /* workspace smaller than moe_workspace_size() */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE_STATUS = 5, /* reserved for callers reporting a nonzero dev_status */
  MOE_ERR_TIMEOUT = 6        /* reserved for callers reporting MOE_DEV_TIMEOUT */
};

/* Bits OR-ed into dev_status by kernels. */
#define MOE_DEV_BAD_EXPERT 1u /* a selected expert id outside [0, E) */
#define MOE_DEV_BAD_TOKEN 2u  /* a selected token id outside [0, T) */
#define MOE_DEV_TIMEOUT 4u    /* a bounded wait inside a kernel expired */
#define MOE_DEV_OVERFLOW 8u   /* more rows than the caller's buffers hold */
#define MOE_DEV_BAD_INDEX 16u /* MOE_DEBUG builds: a caller-supplied row offset, row or
                                 token-list index out of range (skipped) */

enum moe_dtype { MOE_F32 = 0, MOE_BF16 = 1 };
enum moe_routing { MOE_TOKEN_TOPK = 0, MOE_EXPERT_CHOICE = 1, MOE_DES_VOTE = 2, MOE_DES_SEQ = 3 };
enum moe_act { MOE_GELU_ERF = 0, MOE_SWIGLU = 1 };
enum moe_expert_kind { MOE_HEAVY = 0, MOE_IDENTITY = 1, MOE_ZERO = 2, MOE_CONST = 3 };

#define MOE_MAX_EXPERTS 256

/*
 * Layer configuration (host memory, read during the call only).
 *
 * T           tokens in the launch (for DES: the block's N tokens)
 * d           model width; h heavy-expert hidden width
 * E           routed experts of every kind (heavy + zero-computation)
 * n_heavy     heavy experts, ids [0, n_heavy)
 * k           token choice: experts per token; DES: the per-token K
 * n_shared, h_shared  shared experts and their hidden width; they are
 *             passed concatenated along the hidden dimension (n_shared *
 *             h_shared hidden units), which for GELU experts equals the sum
 *             of the separate experts exactly
 * dtype       moe_dtype of x, weights, residual, y (router/selection in fp32)
 * act         moe_act of the heavy experts (shared experts are GELU)
 * routing     moe_routing
 * group_size  expert choice: tokens S per routing group (T % S == 0)
 * capacity    expert choice: tokens C chosen per expert per group
 *             (EC-DiT page, "capacity factor": C = f_c * S / E)
 * M_core      DES-Vote core-set size (DES page, section 3.1: beta * M)
 * k_local     DES-Seq local budget: the core set is the union of every
 *             token's top-k_local experts (DES page, section 2.3)
 * const_mix   0: a constant expert returns its learned vector v; 1: it
 *             returns a0 x + a1 v with (a0, a1) = softmax(Wc x) (MMOE
 *             page, "Methodology": a learned-vector mixture); const_vecs
 *             then holds [n_const, 3, d]: v, then the two rows of Wc
 * gate_residual_scale  weight of the previous layer's logits z_prev
 * renorm      0: weights are the full-softmax affinities A (the pages'
 *             definition); 1: renormalised over each token's selection
 * expert_kind kinds of ids [0, E): MOE_HEAVY for ids < n_heavy, a
 *             zero-computation kind for the others
 */
typedef struct moe_config {
  int32_t T, d, h, E, n_heavy, k;
  int32_t n_shared, h_shared;
  int32_t dtype, act, routing;
  int32_t group_size, capacity, M_core;
  float gate_residual_scale;
  int32_t renorm;
  int32_t k_local;
  int32_t const_mix;
  int32_t expert_kind[MOE_MAX_EXPERTS];
} moe_config;

/* Human-readable name of a moe_status. Never NULL. */
MOE_API const char *moe_status_string(int status);

/* MOE_OK if `device` is an sm_100 GPU this library was built for, else
 * MOE_ERR_UNSUPPORTED (or MOE_ERR_CUDA if the device cannot be queried). */
MOE_API int moe_device_check(int device);

/* Number of routing assignments of a configuration: T*k for token choice
 * and DES, (T/S)*E*C for expert choice. */
MOE_API int moe_num_assignments(const moe_config *cfg, int64_t *n_assign);

/* Workspace bytes moe_forward / moe_forward_host need for `cfg`
 * (moe_dispatch and moe_grouped_mlp need at most this much). */
MOE_API int moe_workspace_size(const moe_config *cfg, size_t *bytes);

/*
 * Router GEMM, softmax and (optionally) token-choice top-k, fused.
 * EC-DiT page, section 3 "Expert-Choice routing formula": given x' in
 * R^{S x d}, A_{s,i} = exp((x' W_r)_{s,i}) / sum_j exp((x' W_r)_{s,j}).
 * MMOE page, "gate-residual routing": the previous expert layer's gate
 * logits are carried into the router: z = x W_r + b + scale * z_prev.
 *
 *   x        [T, d] (dtype)         W_r [E, d] (dtype; row e = expert e)
 *   bias     [E] fp32, nullable     z_prev [T, E] fp32, nullable
 *   logits   [T, E] fp32 out (z)    probs [T, E] fp32 out (A)
 *   k        0: no selection; else 1 <= k <= E and idx/w must be given
 *   idx      [T, k] int32 out: top-k expert ids by z, descending, ties to
 *            the lower id (EC-DiT page, "Token-Choice routing")
 *   w        [T, k] fp32 out: A[s, idx] (renormalised if renorm)
 * Limits: 1 <= E <= 128, d % 8 == 0 for bf16.
 */
MOE_API int moe_router(const void *x, const void *W_r, const float *bias,
               const float *z_prev, float z_prev_scale, int T, int d, int E,
               int dtype, float *logits, float *probs, int k, int renorm,
               int32_t *idx, float *w, moe_stream_t stream);

/*
 * Token-choice top-k from given fp32 logits (the selection half of
 * moe_router, for callers that hold their own logits).
 * EC-DiT page, section 3 "Token-Choice routing": each token selects its
 * top-k experts. Ranking key z, ties to the lower expert id; dropless.
 *   logits [T, E], probs [T, E] fp32 in; idx [T, k] int32, w [T, k] fp32 out.
 * Limits: 1 <= k <= E <= 128.
 */
MOE_API int moe_select_topk(const float *logits, const float *probs, int T, int E,
                    int k, int renorm, int32_t *idx, float *w,
                    moe_stream_t stream);

/*
 * Expert-choice top-C per expert column, by block radix select.
 * EC-DiT page, section 3 "Expert-Choice routing" (each expert picks its
 * top tokens) and "capacity factor" (Capacity = f_c * S / E). The routing
 * group is one sequence of S = group_size tokens.
 *   probs [T, E] fp32 in (A; T % S == 0)
 *   tok   [T/S, E, C] int32 out: GLOBAL token ids in ascending order
 *   w     [T/S, E, C] fp32 out: A[tok, e]
 * Ranking key A, ties to the lower token id. Limits: 1 <= C <= S <= 16384.
 */
MOE_API int moe_select_expert_choice(const float *probs, int T, int E, int group_size,
                             int C, int32_t *tok, float *w,
                             moe_stream_t stream);

/*
 * DES-Vote core set and restricted re-routing, for one block of N tokens.
 * Dynamic Expert Sharing page, section 2.4 "DES-Vote": each token masks to
 * its own top-K experts, votes with their routing weights, and the M_core
 * experts with the largest totals form the core set; section 4.3: tokens
 * then re-activate K experts from the core set.
 *   probs [N, M] fp32 in (P = A)
 *   votes [M] int64 out: sum over tokens of q(P) for each token's top-K,
 *         q(p) = round-half-even(p * 2^40) (exact, order-independent)
 *   core  [M_core] int32 out: elected experts in ascending id order
 *         (ranked by votes, ties to the lower id; always M_core entries)
 *   idx   [N, K] int32 out: each token's K largest P over the core set,
 *         descending, ties to the lower id;   w [N, K] fp32 out: P[n, idx]
 * Limits: 1 <= K <= M_core <= M <= 256, N <= 4096.
 */
MOE_API int moe_core_set_vote(const float *probs, int N, int M, int K, int M_core,
                      int64_t *votes, int32_t *core, int32_t *idx, float *w,
                      moe_stream_t stream);

/*
 * DES-Seq core set and restricted re-routing, for one block of N tokens.
 * Dynamic Expert Sharing page, section 2.3 "DES-Seq": every token selects
 * its k_local most salient experts (top-k_local by P) and the core set is
 * the union of these local selections; section 2.2: tokens then select
 * within the core set, at their original count K (section 4.3).
 *   probs  [N, M] fp32 in (P = A)
 *   core   [M] int32 out: the core set in ascending id order, then -1
 *   n_core [1] int32 out (device): the core-set size
 *   idx    [N, K] int32 out: each token's min(K, n_core) largest P over the
 *          core set, descending, ties to the lower id; slots past n_core
 *          are empty (-1)
 *   w      [N, K] fp32 out: P[n, idx] (0 for an empty slot)
 * Limits: 1 <= K <= M <= 256, 1 <= k_local <= M, N <= 4096.
 */
MOE_API int moe_core_set_union(const float *probs, int N, int M, int K, int k_local,
                               int32_t *core, int32_t *n_core, int32_t *idx, float *w,
                               moe_stream_t stream);

/*
 * Dispatch: a stable permutation of the heavy assignments into per-expert
 * groups (histogram, exclusive scan, scatter), plus the gather of x rows.
 * DICE page, "Conditional Communication" and the expert-parallel
 * dispatch/combine it schedules: tokens go to their experts, outputs come
 * back weighted by the routing score.
 *
 * Assignments in slot order a = 0..n_assign-1 come from `sel`:
 *   token choice / DES: sel = idx [T, k]; a = s*k + j has token s, expert sel[a]
 *   expert choice:      sel = tok [T/S, E, C]; a = (g*E + e)*C + c has
 *                       token sel[a], expert e
 * Outputs (device, caller-owned; sized for n_assign rows at most):
 *   offsets    [n_heavy + 1] int32: rows of expert e are offsets[e]..offsets[e+1]
 *   perm       [n_assign] int32: token of each row, ascending within an expert
 *   row_of     [n_assign] int32: row of assignment a, -1 if not heavy
 *   x_perm     [n_assign, d] (dtype), nullable: x_perm[r] = x[perm[r]]
 *   tok_ptr    [T + 1], tok_assign [n_assign] int32, nullable, expert choice
 *              only: each token's assignments in slot order (a CSR)
 * Expert id -1 marks an empty slot (DES-Seq with a core smaller than K):
 * no row, no flag. Other out-of-range ids set MOE_DEV_BAD_EXPERT /
 * MOE_DEV_BAD_TOKEN and are dropped.
 */
MOE_API int moe_dispatch(const moe_config *cfg, const int32_t *sel, const void *x,
                 void *x_perm, int32_t *offsets, int32_t *perm, int32_t *row_of,
                 int32_t *tok_ptr, int32_t *tok_assign, int32_t *dev_status,
                 void *ws, size_t ws_bytes, moe_stream_t stream);

/* Bytes of library-owned device scratch behind moe_dispatch_noalloc. */
#define MOE_NOALLOC_SCRATCH_BYTES (256u * 1024u)

/*
 * moe_dispatch without a workspace: the same dispatch, with the same
 * arguments, layouts and outputs as moe_dispatch minus ws / ws_bytes.
 * The pages have no counterpart of this entry point; it exists for callers
 * that cannot allocate device memory (for example a host framework that
 * owns all device memory and forbids allocation outside its own pool, or a
 * latency-critical path that cannot afford cudaMalloc's implicit
 * synchronisation) and so cannot hand over a workspace.
 *   - It allocates nothing. Its scratch (the per-block expert histograms)
 *     is a fixed file-scope __device__ array of MOE_NOALLOC_SCRATCH_BYTES
 *     that every GPU loading the library holds until the process exits.
 *   - Limit: max(1, ceil(n_assign / 1024)) * max(1, n_heavy) * 4 bytes
 *     must fit in MOE_NOALLOC_SCRATCH_BYTES; larger configurations return
 *     MOE_ERR_UNSUPPORTED before anything is launched (use moe_dispatch).
 *   - The first call on a device, made with that device current, looks up
 *     the array's device address once (cudaGetSymbolAddress) and caches
 *     it for that device's current CUDA context; make that first call
 *     before any stream capture. A device reset ends the context: the
 *     first call after it (in the new context) looks the address up again,
 *     so it too belongs before any capture.
 *   - All calls share the one array and it keeps the last call's contents
 *     (the kernels overwrite every entry they read, so nothing needs
 *     clearing). Calls that overlap on the GPU race on it: serialise them.
 */
MOE_API int moe_dispatch_noalloc(const moe_config *cfg, const int32_t *sel,
                                 const void *x, void *x_perm, int32_t *offsets,
                                 int32_t *perm, int32_t *row_of,
                                 int32_t *tok_ptr, int32_t *tok_assign,
                                 int32_t *dev_status, moe_stream_t stream);

/*
 * Grouped expert MLP over the dispatched rows, plus the shared expert(s).
 * MMOE page, "MoE++ expert layer" (heavy experts are standard MLPs) and
 * "shared experts" (one dense expert always active). For bf16 the GEMMs
 * run on tcgen05 tensor cores with TMEM accumulators fed by TMA; rows of
 * an expert with no tokens, and the zero-computation experts, issue no
 * MMA at all.
 *   x_perm  [n_assign, d] rows grouped by `offsets` (from moe_dispatch)
 *   W1      GELU: [n_heavy, h, d]; SwiGLU: [n_heavy, 2h, d] (gate rows, then up rows)
 *   W2      [n_heavy, d, h]
 *   x       [T, d], Ws1 [n_shared*h_shared, d], Ws2 [d, n_shared*h_shared]
 *           (all three nullable when n_shared == 0)
 *   y_perm  [n_assign, d] out (dtype): W2_e . act(W1_e . x_perm[r]) per row r
 *   y_shared [T, d] out (dtype; nullable when n_shared == 0)
 * Accumulation is fp32 in tensor memory; hidden activations and outputs are
 * rounded to `dtype` (bf16 layers: bf16).
 */
MOE_API int moe_grouped_mlp(const moe_config *cfg, const void *x_perm,
                    const int32_t *offsets, const void *W1, const void *W2,
                    const void *x, const void *Ws1, const void *Ws2,
                    void *y_perm, void *y_shared, int32_t *dev_status,
                    void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Combine back to token order, fused with the routing-weight scale and
 * the residual add. DICE page, "Conditional Communication": the output of
 * token i is the routing-score weighted sum of its experts' outputs.
 *   y_s = r_s + y_shared[s] + sum over s's assignments a (in slot order) of
 *         w[a] * { y_perm[row_of[a]] (heavy), x_s (identity), 0 (zero),
 *                  const_vecs[c] (c-th constant expert) }
 * summed in fp32 and rounded once to dtype. y_perm, y_shared are in dtype.
 * With cfg->const_mix a constant expert's term is a0 x_s + a1 v_c,
 * (a0, a1) = softmax(Wc_c x_s); its x part is added after the slots.
 * `residual` may be the same buffer as `y` (the sum is formed element by
 * element before y is written). A token with no assignment (expert choice
 * may leave a token unpicked) gets r_s + y_shared[s], 0 without either; an
 * assignment whose row_of is -1 or whose expert id is out of range adds
 * nothing.
 *   sel, w       the selection (as in moe_dispatch) and its [n_assign] weights
 *   row_of       from moe_dispatch;  tok_ptr/tok_assign: expert choice only
 *   x            [T, d] (identity experts); const_vecs [n_const, d]
 *                ([n_const, 3, d] with const_mix), nullable
 *   residual     [T, d] nullable (r = 0);  y [T, d] out (dtype)
 */
MOE_API int moe_combine(const moe_config *cfg, const void *y_perm,
                const void *y_shared, const int32_t *sel, const float *w,
                const int32_t *row_of, const int32_t *tok_ptr,
                const int32_t *tok_assign, const void *x,
                const void *const_vecs, const void *residual, void *y,
                int32_t *dev_status, moe_stream_t stream);

/*
 * The elementwise activation the heavy experts apply, on its own:
 * act == MOE_GELU_ERF: y = GELU(x) = x * Phi(x), the exact (erf) form;
 * act == MOE_SWIGLU:   y = SiLU(x) = x / (1 + exp(-x)), SwiGLU's gate.
 * MMOE page, "MoE++ expert layer" (heavy experts are standard MLPs). The
 * same device functions run in the GEMM epilogues; erf is evaluated by
 * Abramowitz & Stegun 7.1.26 (absolute error <= 1.5e-7), rearranged so
 * that GELU(x) = max(x, 0) - 0.5 |x| P(t) exp(-x^2/2) and evaluated two
 * values at a time on packed fp32x2 arithmetic: GELU(x) is within
 * 4e-7 max(1, |x|) of the exact value.
 *   x, y [n] fp32 device (y may alias x).
 */
MOE_API int moe_activation(const float *x, float *y, int64_t n, int act,
                           moe_stream_t stream);

/*
 * How this copy of the library was built (no counterpart on the pages):
 * MOE_BUILD_DEBUG is set in the MOE_DEBUG build (libmoe_debug.so), whose
 * kernels also range-check the row offsets, rows and token lists that a
 * caller hands to moe_grouped_mlp and moe_combine: an index out of range
 * sets MOE_DEV_BAD_INDEX in dev_status and its group, slot or token is
 * skipped, where the regular build (which trusts those arrays, as
 * moe_dispatch writes them) could read or write out of bounds.
 */
#define MOE_BUILD_DEBUG 1
MOE_API int moe_build_flags(void);

/*
 * Test hook for failure detection (no counterpart on the pages). Blocks of
 * at most 128 bf16 tokens with a shared expert finish their routing in one
 * cooperative kernel whose CTAs meet at grid barriers (software barriers
 * on a global counter, each wait bounded by 2 s). This sets, for every
 * later launch of that kernel in the process, the wait limit to `limit_ns`
 * (0 restores the 2 s default) and makes the barriers wait for
 * `extra_arrivals` arrivals beyond the grid (0 restores the default), so a
 * test can make a wait expire on purpose without faulting or hanging the
 * GPU. An expired barrier sets MOE_DEV_TIMEOUT in dev_status, and the
 * CTAs that gave up leave their tokens' slots empty (expert -1, weight 0,
 * no row) and zero row offsets (CTA 0), so the rest of the layer runs on
 * an empty routing for those tokens: y = residual + shared expert there.
 * Process-wide; set it only while no layer call is being enqueued.
 *   limit_ns        0 .. 2e9;  extra_arrivals  0 .. 1024
 * Returns MOE_ERR_INVALID_ARG outside those ranges.
 */
MOE_API int moe_test_set_barrier_wait(uint64_t limit_ns, int extra_arrivals);

/* Optional outputs of moe_forward (each pointer nullable; device memory). */
typedef struct moe_forward_aux {
  float *logits;     /* [T, E] fp32 */
  float *probs;      /* [T, E] fp32 */
  int32_t *sel;      /* [n_assign] idx (token choice, DES) or tok (expert choice) */
  float *w;          /* [n_assign] fp32 routing weights */
  int64_t *votes;    /* [E] DES-Vote only */
  int32_t *core;     /* DES-Vote: [M_core]; DES-Seq: [E], the core set then -1 */
  int32_t *offsets;  /* [n_heavy + 1] */
} moe_forward_aux;

/*
 * The whole layer: router -> selection -> dispatch -> grouped MLP ->
 * combine, every step a kernel of this library, no host synchronisation
 * (group sizes stay on the device). Everything runs on `stream`, except
 * that a bf16 layer with a shared expert and routed rows (not a small
 * block) runs the shared expert's up projection on a library-owned side
 * stream. That stream forks from `stream` after the routing and joins it
 * before the down projections, so the call is still ordered on `stream`
 * as a whole, and stream capture takes the side stream in. The first
 * such call on a device creates the side stream and its events; capture
 * that first call only in a capture mode that allows stream and event
 * creation. Concurrent callers on one device serialise on a host mutex
 * while they enqueue the layer.
 *   x [T, d], residual [T, d] nullable, z_prev [T, E] fp32 nullable,
 *   W_r [E, d], bias [E] fp32 nullable, W1, W2, Ws1, Ws2 as in
 *   moe_grouped_mlp, const_vecs [n_const, d] nullable, y [T, d] out.
 *   aux nullable: copies of the intermediate results for inspection.
 */
MOE_API int moe_forward(const moe_config *cfg, const void *x, const void *residual,
                const float *z_prev, const void *W_r, const float *bias,
                const void *W1, const void *W2, const void *Ws1,
                const void *Ws2, const void *const_vecs, void *y,
                const moe_forward_aux *aux, int32_t *dev_status, void *ws,
                size_t ws_bytes, moe_stream_t stream);

/*
 * moe_forward with the activations in HOST memory: copies x_host (and
 * residual_host, z_prev_host if given) to the device, runs the layer and
 * copies y back to y_host. Weights stay device pointers. For the copies to
 * be asynchronous the host buffers should be pinned; the caller
 * synchronises `stream` before reading y_host.
 *
 * Batches of at least 4096 tokens (token or expert choice) run as a
 * pipeline of 2 or 3 token chunks: chunk i's layer runs on `stream` while
 * chunk i+1 is copied in on one library-owned side stream and chunk i-1 is
 * copied out on another. The side streams fork from `stream` at entry and
 * join it before return, so work enqueued on `stream` afterwards sees y_host
 * complete, as in the one-chunk form. Chunks are whole routing units (whole
 * groups for expert choice; a DES block is never cut) and every later step
 * is per row or per token, so y is bit-identical to the unchunked layer.
 * Calls on a stream under CUDA graph capture take the one-chunk form. The
 * side streams and their events are made on first use per device and live
 * until process exit; concurrent callers serialise on a host mutex while
 * they enqueue.
 */
MOE_API int moe_forward_host(const moe_config *cfg, const void *x_host,
                     const void *residual_host, const float *z_prev_host,
                     const void *W_r, const float *bias, const void *W1,
                     const void *W2, const void *Ws1, const void *Ws2,
                     const void *const_vecs, void *y_host,
                     int32_t *dev_status, void *ws, size_t ws_bytes,
                     moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
