// Internal launch interface between the C ABI (moe_api.cu) and the kernel
// translation units. Every launcher enqueues on `stream`, returns a
// moe_status, and never synchronises the host.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

struct KindTable;

#define MOE_CUDA_TRY(expr)                                   \
  do {                                                       \
    cudaError_t moe_err_ = (expr);                           \
    if (moe_err_ != cudaSuccess) return MOE_ERR_CUDA;        \
  } while (0)

// Experts per layer the library takes (moe_config.E; larger is
// MOE_ERR_UNSUPPORTED).
constexpr int kMaxLayerExperts = 128;

inline int last_launch_status() {
  return cudaPeekAtLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int num_sms();

// router.cu: z = x W_r^T + bias + scale * z_prev; A = softmax(z); optional top-k.
// With `votes` (zeroed int64 [E]) the router also adds each token's DES
// top-k_vote votes into it (small bf16 blocks only: router_can_vote).
int launch_router(const void *x, const void *W_r, const float *bias,
                  const float *z_prev, float z_prev_scale, int T, int d, int E,
                  int dtype, float *logits, float *probs, int k, int renorm,
                  int32_t *idx, float *w, cudaStream_t stream,
                  int64_t *votes = nullptr, int k_vote = 0);
bool router_can_vote(int T, int dtype);
// Small bf16 blocks in the fused forward: the model width is split over
// n_part CTAs per 32-token tile (partial logits in `part`, [n_part][T][E]
// fp32), then one warp per token finishes (and optionally votes).
int router_split_parts(int T, int d, int dtype);  // 0: not used for this size
int launch_router_split(const void *x, const void *W_r, const float *bias, const float *z_prev,
                        float z_prev_scale, int T, int d, int E, float *part, int n_part,
                        float *logits, float *probs, int k, int renorm, int32_t *idx, float *w,
                        int64_t *votes, int k_vote, cudaStream_t stream);
// Words zeroed by the first CTA of the split router, for kernels later in
// the same stream (DES vote totals, a grid-barrier counter, counters).
struct ZeroList {
  int32_t *p[3];
  int n[3];
};
int launch_router_partial(const void *x, const void *W_r, int T, int d, int E, float *part,
                          int n_part, const ZeroList &zero, cudaStream_t stream);

// small_route.cu: router finish + DES election/re-route + dispatch + row
// gather for blocks of at most 128 tokens, one cooperative launch (one CTA
// per token, bounded grid barriers). Reads the split router's partials.
constexpr int kSmallRouteMaxTokens = 128;
constexpr int kSmallRouteMaxK = 32;
constexpr int kSmallRouteMaxAssign = 2048;
struct SmallRouteArgs {
  const float *part;     // [n_part][T][E] partial logits
  int n_part;
  const float *bias, *zprev;
  float zscale;
  int T, E, n_heavy, k, routing, renorm, M_core;
  int row_vecs;          // 16-byte vectors per x row
  const uint4 *x;        // [T][row_vecs]
  uint4 *x_perm;         // [rows][row_vecs]
  float *logits, *probs; // [T][E]
  int32_t *sel;          // [T*k] expert per slot
  float *w;              // [T*k] routing weight per slot
  unsigned long long *votes;  // [E] zeroed before the launch (DES)
  int32_t *core;         // [M_core] (DES)
  int32_t *offsets;      // [n_heavy + 1]
  int32_t *perm;         // [rows] token of each expert row
  int32_t *row_of;       // [T*k] expert row of each slot, -1 if none
  unsigned *barrier;     // grid-barrier counter, zeroed before the launch
  unsigned *gmask;       // [n_heavy][4] token bitmasks, zeroed before the launch
  int32_t *dev_status;
  // Set by launch_small_route: the grid barriers' wait limit and the
  // arrivals they wait for beyond the grid (0 except under the test hook).
  unsigned long long wait_ns;
  int extra_arrivals;
};
bool small_route_supported(int T, int E, int k, int routing, int dtype);
int launch_small_route(const SmallRouteArgs &args, cudaStream_t stream);
// Test hook behind moe_test_set_barrier_wait (0, 0 restores the defaults).
void set_small_route_test_wait(unsigned long long limit_ns, int extra_arrivals);

// block_sm100.cu: the whole layer for blocks of <= 128 bf16 tokens (token
// choice or DES-Vote, no shared expert) in one persistent cooperative
// kernel: router (K-sliced over the CTAs), selection, weight-streaming MLP
// (up projection over all tokens, no dispatch), combine. Its sync words,
// bitmasks, vote totals and counters sit in one workspace region that must
// be zero at launch (block_zero_bytes).
struct BlockArgs {
  const void *W_r;       // [E][d] bf16 router weights
  float *part;           // [n_slices][T][E] partial logits (workspace)
  int n_slices, kslice;  // router K slices over the CTAs, columns per slice
  const float *bias, *zprev;
  float zscale;
  int T, E, n_heavy, k, routing, renorm, M_core, k_local;
  int d, h;              // model width, expert hidden width
  int w1_rows_per_group; // h (GELU) or 2h (SwiGLU: gate rows, then up rows)
  const void *x;         // [T][d] bf16
  const void *residual;  // [T][d] bf16, may alias y
  const void *const_vecs;
  void *y;               // [T][d] bf16
  void *H, *Y;           // [T*k][h], [T*k][d] bf16 workspace
  float *logits, *probs;
  int32_t *sel;
  float *w;
  int64_t *votes_out;    // DES vote totals for the caller
  int32_t *core, *offsets, *perm, *row_of;
  // The zeroed region (block_zero_bytes), split by block_zero_layout:
  unsigned *sync;        // [0] barrier arrivals, [1] finished CTAs, [2] unit tickets,
                         // [3] tokens whose slots are out, [4] combine item tickets
  unsigned *gmask;       // [E][4] token bitmasks
  unsigned long long *votes;  // [E] DES-Vote totals (exact fixed point); DES-Seq: core bitmask
  int32_t *done;         // [n_heavy] up-unit arrivals per expert
  int32_t *dev_status;
};
bool moe_block_supported(const moe_config &c);
int block_router_slices(int d, int *kslice);  // K slices of the in-kernel router
size_t block_zero_bytes(int E, int n_heavy);
// Points a's sync / gmask / votes / done into the zeroed region `z`.
void block_zero_layout(BlockArgs &a, void *z, int E);
int launch_moe_block(const BlockArgs &a, const KindTable &kinds, const void *W1, const void *W2,
                     int act, cudaStream_t stream);

// small_f32.cu: the whole layer for a small fp32 token-choice layer without
// a shared expert, one CTA per token (router row, softmax, top-k, the
// experts' MLPs from L2-resident weights, combine), one launch. `counts`
// (small_f32_zero_bytes: one word per heavy expert, then a CTA counter)
// must be zero at launch.
struct SmallF32Args {
  const float *x, *residual, *W_r, *bias, *zprev, *W1, *W2, *const_vecs;
  float zscale;
  int T, d, h, E, n_heavy, k, renorm, gated;
  float *logits, *probs, *w, *y;
  int32_t *sel, *offsets;
  unsigned *counts;
};
bool small_f32_supported(const moe_config &c);
size_t small_f32_zero_bytes(int n_heavy);
int launch_small_f32(const SmallF32Args &a, const KindTable &kinds, cudaStream_t stream);

int launch_select_topk(const float *logits, const float *probs, int T, int E,
                       int k, int renorm, int32_t *idx, float *w,
                       cudaStream_t stream);

// select.cu: expert-choice radix select and the DES-Vote core set.
int launch_expert_choice(const float *probs, int T, int E, int S, int C,
                         int32_t *tok, float *w, cudaStream_t stream);
// Election recomputed per token-CTA from summed votes, then re-routing.
int launch_des_reroute(const float *probs, const int64_t *votes, int N, int M, int K,
                       int M_core, int32_t *core, int32_t *idx, float *w,
                       cudaStream_t stream);
// DES-Seq: core = union of every token's top-k_local; restricted re-route.
int launch_des_seq(const float *probs, int N, int M, int K, int k_local, int32_t *core,
                   int32_t *n_core, int32_t *idx, float *w, cudaStream_t stream);
int launch_des_vote(const float *probs, int N, int M, int K, int M_core,
                    int64_t *votes, int32_t *core, int32_t *idx, float *w,
                    cudaStream_t stream);

// dispatch.cu
struct DispatchArgs {
  int routing;     // moe_routing
  int T, E, n_heavy;
  int k;           // token choice / DES: slots per token
  int S, C;        // expert choice
  int64_t n_assign;
  const int32_t *sel;
  int32_t *offsets, *perm, *row_of, *tok_ptr, *tok_assign;
  int32_t *dev_status;
  int32_t *zero_words;  // optional: words the dispatch clears for a later kernel
  int n_zero_words;
};
size_t dispatch_workspace_bytes(int64_t n_assign, int n_heavy);
int launch_dispatch(const DispatchArgs &a, void *ws, cudaStream_t stream);
// Expert choice in one launch (the permutation in closed form, one CTA per
// routing group) for groups whose token ids fit in shared memory.
bool dispatch_ec_supported(int S, int E, int C);
int launch_dispatch_ec(const DispatchArgs &a, cudaStream_t stream);
// dispatch_noalloc.cu: the dispatch with library-owned scratch.
bool dispatch_fits_noalloc_scratch(int64_t n_assign, int n_heavy);
int launch_dispatch_noalloc(const DispatchArgs &a, cudaStream_t stream);
int launch_gather_rows(const void *x, void *x_perm, const int32_t *perm,
                       const int32_t *offsets, int n_heavy, int64_t max_rows,
                       int d, int elem_bytes, cudaStream_t stream);

// gemm_sm100.cu: grouped GEMM D = act(A . B^T) on tcgen05 (bf16 in, fp32 acc).
enum GemmAct { kActNone = 0, kActGelu = 1, kActSwiglu = 2 };
struct GemmProblem {
  const void *A;        // [rows, K] bf16
  int64_t a_rows;       // rows in the A tensor (TMA bound)
  const void *B;        // [n_groups * b_rows_per_group, K] bf16
  int b_rows_per_group; // N (none/GELU) or 2N (SwiGLU: gate rows then up rows)
  int n_groups;
  const int32_t *offsets;  // [n_groups + 1] device row offsets, or NULL: one group of a_rows rows
  int N, K;
  void *out;            // [rows, ld_out] (bf16 or fp32)
  int64_t ld_out;
  const void *residual; // optional [rows, ld_res] bf16 added before the output is rounded
  int64_t ld_res;
  int32_t *status;      // device status word for MOE_DEBUG range checks (fp32 path), nullable
};

// Upper bound of the m-tiles of height bm over all groups of a problem.
inline int64_t max_m_tiles(const GemmProblem &p, int bm) {
  return (p.a_rows + bm - 1) / bm + (p.offsets ? p.n_groups : 0);
}
// `also` (nullable): a problem of the same activation that would share this
// launch but runs in another one (moe_forward's shared up projection on its
// side stream, beside the routed one); the tile shape is chosen over both,
// so the two launches run the same kernel.
int launch_grouped_gemm_bf16(const GemmProblem *probs, int n_probs, int act,
                             bool out_f32, int32_t *dev_status,
                             cudaStream_t stream, const GemmProblem *also = nullptr);

// 2-D bf16 TMA descriptor [rows, cols] (cols contiguous), box {64, box_rows},
// 128-byte swizzle, zero fill outside the tensor.
bool make_tma_2d_bf16(CUtensorMap *map, const void *ptr, int64_t rows, int64_t cols, int box_rows);

// stream_sm100.cu: weight-streaming expert MLP for blocks of at most 128
// tokens (each expert's weights read from HBM once per layer).
bool stream_mlp_supported(int T);
size_t stream_mlp_workspace_bytes(int n_groups);
// `done` holds n_groups zeroed counters when counters_zeroed, else the
// launcher clears them first.
int launch_stream_mlp(const GemmProblem &up, int act, const GemmProblem &down,
                      int max_tokens, int32_t *done, bool counters_zeroed,
                      int32_t *dev_status, cudaStream_t stream);

// mlp_f32.cu: the same grouped GEMM in fp32 on CUDA cores (fp32 layers).
int launch_grouped_gemm_f32(const GemmProblem &p, int act,
                            cudaStream_t stream);

// activation.cu: the experts' elementwise activation on its own.
int launch_activation(const float *x, float *y, int64_t n, int act, cudaStream_t stream);

// combine.cu
struct CombineArgs {
  int routing, T, d, E, k, S, C, dtype;
  int const_mix;  // constant experts mix x and v (const_vecs is [n_const, 3, d])
  int fine;       // set by launch_combine: one 256-feature chunk per warp item
  const void *y_perm, *y_shared;  // expert outputs, in the layer dtype
  const int32_t *sel;
  const float *w;
  const int32_t *row_of, *tok_ptr, *tok_assign;
  const void *x, *const_vecs, *residual;
  void *y;
  int32_t *dev_status;
  int64_t y_rows;  // rows of y_perm (= assignments): the range MOE_DEBUG builds check rows against
};
int launch_combine(const CombineArgs &a, const KindTable &kinds,
                   cudaStream_t stream);

}  // namespace moe
