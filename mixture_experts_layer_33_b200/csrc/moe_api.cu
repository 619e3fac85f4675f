// The C ABI of libmoe.so: argument checks, workspace layout and the
// orchestration of the layer's kernels (declared in include/moe.h).
#include <string.h>

#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int elem_bytes(int dtype) { return dtype == MOE_BF16 ? 2 : 4; }

int64_t n_assign_of(const moe_config &c) {
  if (c.routing == MOE_EXPERT_CHOICE) return (int64_t)(c.T / c.group_size) * c.E * c.capacity;
  return (int64_t)c.T * c.k;
}

int check_config(const moe_config *c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_BF16 && c->dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->d < 8 || c->d % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (c->E < 1 || c->E > kMaxLayerExperts)
    return c->E > kMaxLayerExperts ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  if (c->n_heavy < 0 || c->n_heavy > c->E) return MOE_ERR_INVALID_ARG;
  if (c->n_heavy > 0 && (c->h < 8 || c->h % 8 != 0)) return MOE_ERR_INVALID_ARG;
  if (c->act != MOE_GELU_ERF && c->act != MOE_SWIGLU) return MOE_ERR_INVALID_ARG;
  for (int e = 0; e < c->E; ++e) {
    int k = c->expert_kind[e];
    if (e < c->n_heavy ? k != MOE_HEAVY : (k != MOE_IDENTITY && k != MOE_ZERO && k != MOE_CONST))
      return MOE_ERR_INVALID_ARG;
  }
  if (c->n_shared < 0) return MOE_ERR_INVALID_ARG;
  if (c->n_shared > 0 && (c->h_shared < 8 || c->h_shared % 8 != 0)) return MOE_ERR_INVALID_ARG;
  switch (c->routing) {
    case MOE_TOKEN_TOPK:
      if (c->k < 1 || c->k > c->E) return MOE_ERR_INVALID_ARG;
      break;
    case MOE_EXPERT_CHOICE:
      if (c->group_size < 1 || c->T % c->group_size != 0) return MOE_ERR_INVALID_ARG;
      if (c->capacity < 1 || c->capacity > c->group_size) return MOE_ERR_INVALID_ARG;
      if (c->group_size > 16384) return MOE_ERR_UNSUPPORTED;
      break;
    case MOE_DES_VOTE:
      if (c->k < 1 || c->k > c->M_core || c->M_core > c->E) return MOE_ERR_INVALID_ARG;
      if (c->T > 4096) return MOE_ERR_UNSUPPORTED;
      break;
    case MOE_DES_SEQ:
      if (c->k < 1 || c->k > c->E || c->k_local < 1 || c->k_local > c->E) return MOE_ERR_INVALID_ARG;
      if (c->T > 4096) return MOE_ERR_UNSUPPORTED;
      break;
    default:
      return MOE_ERR_INVALID_ARG;
  }
  if (c->renorm != 0 && c->renorm != 1) return MOE_ERR_INVALID_ARG;
  if (c->const_mix != 0 && c->const_mix != 1) return MOE_ERR_INVALID_ARG;
  if (n_assign_of(*c) > (int64_t)0x7fffffff) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

KindTable kind_table(const moe_config &c) {
  KindTable kt;
  memset(&kt, 0, sizeof(kt));
  int nc = 0;
  for (int e = 0; e < c.E; ++e) {
    kt.kind[e] = (int8_t)c.expert_kind[e];
    kt.cidx[e] = (int16_t)(c.expert_kind[e] == MOE_CONST ? nc++ : 0);
  }
  return kt;
}

int n_const_of(const moe_config &c) {
  int n = 0;
  for (int e = 0; e < c.E; ++e) n += c.expert_kind[e] == MOE_CONST;
  return n;
}

// Workspace layout shared by the entry points.
struct Layout {
  size_t logits, probs, sel, w, votes, core, offsets, perm, row_of, tok_ptr, tok_assign, dpart,
      x_perm, H, H_sh, Y, Y_sh, done, rpart, bzero, fzero, cbar, x_dev, res_dev, zp_dev, y_dev,
      total;
};

Layout layout_of(const moe_config &c) {
  Layout L;
  const int64_t na = n_assign_of(c);
  const size_t eb = elem_bytes(c.dtype);
  const int64_t hs = (int64_t)c.n_shared * c.h_shared;
  const int64_t h1 = c.h;  // hidden activations after the gate (SwiGLU halves 2h -> h)
  size_t o = kAlign;  // the first slot is reserved, so a workspace is never empty
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
  L.logits = take((size_t)c.T * c.E * 4);
  L.probs = take((size_t)c.T * c.E * 4);
  L.sel = take((size_t)na * 4);
  L.w = take((size_t)na * 4);
  L.votes = take((size_t)c.E * 8);
  L.core = take((size_t)c.E * 4);
  L.offsets = take((size_t)(c.n_heavy + 1) * 4);
  L.perm = take((size_t)na * 4);
  L.row_of = take((size_t)na * 4);
  L.tok_ptr = take((size_t)(c.T + 1) * 4);
  L.tok_assign = take((size_t)na * 4);
  L.dpart = take(dispatch_workspace_bytes(na, c.n_heavy));
  L.x_perm = take((size_t)na * c.d * eb);
  L.H = take((size_t)na * h1 * eb);
  L.H_sh = take((size_t)c.T * hs * eb);
  L.Y = take((size_t)na * c.d * eb);
  L.Y_sh = take(hs ? (size_t)c.T * c.d * eb : 0);
  L.done = take(stream_mlp_workspace_bytes(c.n_heavy + 1));  // routed groups, then the shared one
  {
    int ks = 0;
    const int parts = router_split_parts(c.T, c.d, c.dtype);
    const int slices = moe_block_supported(c) ? block_router_slices(c.d, &ks) : 0;
    L.rpart = take((size_t)(parts > slices ? parts : slices) * c.T * c.E * 4);
  }
  L.bzero = take(moe_block_supported(c) ? block_zero_bytes(c.E, c.n_heavy) : 0);
  L.fzero = take(small_f32_supported(c) ? small_f32_zero_bytes(c.n_heavy) : 0);
  // Small-block routing kernel: grid-barrier counter (16 B), then a 4-word
  // token bitmask per expert.
  L.cbar = take(16 + (size_t)c.E * 16);
  L.x_dev = take((size_t)c.T * c.d * eb);
  L.res_dev = take((size_t)c.T * c.d * eb);
  L.zp_dev = take((size_t)c.T * c.E * 4);
  L.y_dev = take((size_t)c.T * c.d * eb);
  L.total = o;
  return L;
}

template <typename T>
T *at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

int check_ws(const moe_config &c, void *ws, size_t ws_bytes) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < layout_of(c).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

// ---- host path: chunked copy / compute pipeline

constexpr int kHostMaxChunks = 4;
constexpr int64_t kHostMinChunkTokens = 2048;
// Relative chunk sizes: a small first chunk starts the layer early and a
// small last chunk ends the copy-out early. A chunk costs a fixed part (the
// fixed-latency kernels, the GEMMs' last wave, one more pass over the
// expert weights) on top of its per-token share, which bounds how many pay
// off: the third one re-reads the weights at HBM speed (~6.5 TB/s) to hide
// about a quarter of the activations' copies at PCIe speed (~55 GB/s each
// way), so it is taken while the weights stay under ~30x the activations.
constexpr int kHostPlan2[] = {1, 1};
constexpr int kHostPlan3[] = {1, 2, 1};
constexpr double kHostThirdChunkRatio = 30.0;

// Expert weight bytes one pass of the layer reads (routed and shared).
double layer_weight_bytes(const moe_config &c) {
  const double w1_rows = c.act == MOE_SWIGLU ? 2.0 * c.h : c.h;
  const double hs = (double)c.n_shared * c.h_shared;  // Ws1 [hs, d], Ws2 [d, hs]
  return ((double)c.n_heavy * (w1_rows + c.h) + 2.0 * hs) * c.d * elem_bytes(c.dtype);
}

// Chunk boundaries of moe_forward_host's token pipeline: bounds[0] = 0 <
// bounds[1] < ... < bounds[n] = T; returns n (1: no pipelining). A chunk is
// a whole number of routing units: token choice routes each token on its
// own (any cut; 128-token multiples keep the GEMM tiles full), expert
// choice routes whole groups, and DES elects one core set for the whole
// block, so a DES block is never cut. Every step after routing is per row
// or per token, so the chunked layer computes what the whole one does.
int host_chunk_plan(const moe_config &c, int64_t bounds[kHostMaxChunks + 1]) {
  bounds[0] = 0;
  bounds[1] = c.T;
  if (c.routing == MOE_DES_VOTE || c.routing == MOE_DES_SEQ) return 1;
  if (c.T < 2 * kHostMinChunkTokens) return 1;
  const double act_bytes = (double)c.T * c.d * elem_bytes(c.dtype);
  const bool two = c.T < 4 * kHostMinChunkTokens ||
                   layer_weight_bytes(c) > kHostThirdChunkRatio * act_bytes;
  const int *w = two ? kHostPlan2 : kHostPlan3;
  const int nw = (int)(two ? sizeof(kHostPlan2) : sizeof(kHostPlan3)) / (int)sizeof(int);
  const int64_t unit = c.routing == MOE_EXPERT_CHOICE ? c.group_size : 128;
  int total = 0;
  for (int i = 0; i < nw; ++i) total += w[i];
  int n = 0, acc = 0;
  for (int i = 0; i < nw; ++i) {
    acc += w[i];
    int64_t b = i == nw - 1 ? c.T : ((int64_t)c.T * acc / total + unit / 2) / unit * unit;
    if (b > c.T) b = c.T;
    if (b > bounds[n]) bounds[++n] = b;
  }
  return n;
}

// The host<->device copies of a token range [t0, t0 + nt).
struct HostCopy {
  const uint8_t *xh = nullptr, *rh = nullptr, *zh = nullptr;
  uint8_t *yh = nullptr;
  uint8_t *xd = nullptr, *rd = nullptr, *zd = nullptr, *yd = nullptr;
  size_t row = 0, zrow = 0;  // bytes per token of x / y / residual, of z_prev

  int in(int64_t t0, int64_t nt, cudaStream_t s) const {
    if (nt <= 0) return MOE_OK;
    MOE_CUDA_TRY(cudaMemcpyAsync(xd + t0 * row, xh + t0 * row, nt * row, cudaMemcpyHostToDevice, s));
    if (rh && rd)
      MOE_CUDA_TRY(cudaMemcpyAsync(rd + t0 * row, rh + t0 * row, nt * row, cudaMemcpyHostToDevice, s));
    if (zh && zd)
      MOE_CUDA_TRY(cudaMemcpyAsync(zd + t0 * zrow, zh + t0 * zrow, nt * zrow, cudaMemcpyHostToDevice, s));
    return MOE_OK;
  }
  int out(int64_t t0, int64_t nt, cudaStream_t s) const {
    if (nt <= 0) return MOE_OK;
    MOE_CUDA_TRY(cudaMemcpyAsync(yh + t0 * row, yd + t0 * row, nt * row, cudaMemcpyDeviceToHost, s));
    return MOE_OK;
  }
};

// Per-device side streams and events of the pipeline, made on first use
// and kept for the life of the process; callers hold g_host_pipe_mu from
// the first event record to the final join, so concurrent callers do not
// interleave their records and waits on the shared events.
constexpr int kHostMaxDevices = 64;
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t ev[2 + 2 * kHostMaxChunks] = {};
};
std::mutex g_host_pipe_mu;
HostPipe g_host_pipe[kHostMaxDevices];

int host_pipe(HostPipe **p) {
  int dev = 0;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kHostMaxDevices) return MOE_ERR_UNSUPPORTED;
  HostPipe &hp = g_host_pipe[dev];
  if (!hp.in) {
    if (!hp.out) MOE_CUDA_TRY(cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking));
    for (cudaEvent_t &e : hp.ev)
      if (!e) MOE_CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    MOE_CUDA_TRY(cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking));  // last: marks it ready
  }
  *p = &hp;
  return MOE_OK;
}

// moe_forward runs the shared expert's up projection (it needs only x) on a
// per-device side stream while the routed rows are dispatched and gathered
// on the caller's stream; the down projections wait for both. The stream
// and its two events are made on first use and kept for the life of the
// process. A forward holds g_side_mu from the fork's event record to the
// caller stream's wait on the join, so concurrent callers on one device do
// not interleave their records and waits.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_side_mu;
SideStream g_side[kHostMaxDevices];

// Fork of the side stream from a caller's stream, joined back (the caller's
// stream waits for the side stream's work) by join() or, on an early
// return, by the destructor, so a captured stream never ends with the side
// stream unjoined.
class SideFork {
 public:
  explicit SideFork(cudaStream_t stream) : stream_(stream) {}
  SideFork(const SideFork &) = delete;
  SideFork &operator=(const SideFork &) = delete;
  ~SideFork() { join(); }
  cudaStream_t side() const { return side_->s; }
  // Work enqueued on side() from here on runs after everything enqueued on
  // the caller's stream so far.
  int fork() {
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kHostMaxDevices) return MOE_ERR_UNSUPPORTED;
    lock_ = std::unique_lock<std::mutex>(g_side_mu);
    SideStream &ss = g_side[dev];
    if (!ss.s) {
      if (!ss.fork) MOE_CUDA_TRY(cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming));
      if (!ss.join) MOE_CUDA_TRY(cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming));
      MOE_CUDA_TRY(cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking));  // last: marks it ready
    }
    MOE_CUDA_TRY(cudaEventRecord(ss.fork, stream_));
    MOE_CUDA_TRY(cudaStreamWaitEvent(ss.s, ss.fork, 0));
    side_ = &ss;
    return MOE_OK;
  }
  // The caller's stream waits for the side stream's work so far.
  int join() {
    if (!side_) {
      if (lock_.owns_lock()) lock_.unlock();
      return MOE_OK;
    }
    SideStream *ss = side_;
    side_ = nullptr;
    cudaError_t e = cudaEventRecord(ss->join, ss->s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream_, ss->join, 0);
    lock_.unlock();
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }

 private:
  cudaStream_t stream_;
  SideStream *side_ = nullptr;
  std::unique_lock<std::mutex> lock_;
};

// The shared expert's up projection: H_sh = GELU(x Ws1^T) over all tokens
// (the shared experts concatenated along the hidden dimension).
GemmProblem shared_up_problem(const moe_config &c, const void *x, const void *Ws1, void *H_sh,
                              int32_t *dev_status) {
  const int64_t hs = (int64_t)c.n_shared * c.h_shared;
  GemmProblem g{};
  g.A = x; g.a_rows = c.T; g.B = Ws1; g.n_groups = 1; g.offsets = nullptr;
  g.N = (int)hs; g.b_rows_per_group = (int)hs; g.K = c.d; g.out = H_sh; g.ld_out = hs;
  g.status = dev_status;
  return g;
}

// The routed experts' up projection: H = act(x_perm W1_g^T) per group.
GemmProblem routed_up_problem(const moe_config &c, const void *x_perm, const int32_t *offsets,
                              const void *W1, void *H, int32_t *dev_status) {
  const bool gated = c.act == MOE_SWIGLU;
  GemmProblem g{};
  g.A = x_perm; g.a_rows = n_assign_of(c); g.B = W1; g.n_groups = c.n_heavy; g.offsets = offsets;
  g.N = c.h; g.b_rows_per_group = gated ? 2 * c.h : c.h; g.K = c.d;
  g.out = H; g.ld_out = c.h;
  g.status = dev_status;
  return g;
}

// `side`: the shared up projection already runs on a forked side stream;
// the routed up projection runs alone and the down projections wait for
// the side stream.
int run_grouped_mlp(const moe_config &c, const void *x_perm, const int32_t *offsets,
                    const void *W1, const void *W2, const void *x, const void *Ws1,
                    const void *Ws2, void *y_perm, void *y_shared, int32_t *dev_status,
                    void *ws, const Layout &L, cudaStream_t stream,
                    bool counters_zeroed = false, const void *shared_residual = nullptr,
                    SideFork *side = nullptr) {
  const int64_t na = n_assign_of(c);
  const int64_t hs = (int64_t)c.n_shared * c.h_shared;
  void *H = at<void>(ws, L.H);
  void *H_sh = at<void>(ws, L.H_sh);
  const int act1 = c.act == MOE_SWIGLU ? kActSwiglu : kActGelu;

  GemmProblem g1r{}, g1s{}, g2r{}, g2s{};
  g1r = routed_up_problem(c, x_perm, offsets, W1, H, dev_status);
  g2r.A = H; g2r.a_rows = na; g2r.B = W2; g2r.n_groups = c.n_heavy; g2r.offsets = offsets;
  g2r.N = c.d; g2r.b_rows_per_group = c.d; g2r.K = c.h; g2r.out = y_perm; g2r.ld_out = c.d;
  g1s = shared_up_problem(c, x, Ws1, H_sh, dev_status);
  g2s.A = H_sh; g2s.a_rows = c.T; g2s.B = Ws2; g2s.n_groups = 1; g2s.offsets = nullptr;
  g2s.N = c.d; g2s.b_rows_per_group = c.d; g2s.K = (int)hs; g2s.out = y_shared; g2s.ld_out = c.d;
  g2s.residual = shared_residual; g2s.ld_res = c.d;
  g1r.status = g1s.status = g2r.status = g2s.status = dev_status;
  const bool routed = c.n_heavy > 0 && na > 0;
  const bool shared = hs > 0 && c.T > 0;

  int st = MOE_OK;
  if (c.dtype == MOE_BF16 && stream_mlp_supported(c.T)) {
    // Small blocks (every expert serves <= T <= 128 tokens): stream each
    // used expert's weights once through the tensor cores.
    int32_t *done = at<int32_t>(ws, L.done);
    if (routed)
      st = launch_stream_mlp(g1r, act1, g2r, c.T, done, counters_zeroed, dev_status, stream);
    if (st == MOE_OK && shared)
      st = launch_stream_mlp(g1s, kActGelu, g2s, c.T, done + c.n_heavy, counters_zeroed,
                             dev_status, stream);
    return st;
  }
  if (c.dtype == MOE_BF16) {
    // GEMM1 (+activation): routed and shared in one tile stream when they share the activation.
    if (side) {
      if (routed)
        st = launch_grouped_gemm_bf16(&g1r, 1, act1, false, dev_status, stream,
                                      act1 == kActGelu ? &g1s : nullptr);
      if (st == MOE_OK) st = side->join();
    } else if (routed && shared && act1 == kActGelu) {
      GemmProblem p1[2] = {g1r, g1s};
      st = launch_grouped_gemm_bf16(p1, 2, kActGelu, false, dev_status, stream);
    } else {
      if (routed) st = launch_grouped_gemm_bf16(&g1r, 1, act1, false, dev_status, stream);
      if (st == MOE_OK && shared) st = launch_grouped_gemm_bf16(&g1s, 1, kActGelu, false, dev_status, stream);
    }
    if (st != MOE_OK) return st;
    // GEMM2: the longer-K shared problem first so the tile stream ends on short tiles.
    if (routed && shared) {
      GemmProblem p2[2] = {g2s, g2r};
      st = launch_grouped_gemm_bf16(p2, 2, kActNone, false, dev_status, stream);
    } else if (routed) {
      st = launch_grouped_gemm_bf16(&g2r, 1, kActNone, false, dev_status, stream);
    } else if (shared) {
      st = launch_grouped_gemm_bf16(&g2s, 1, kActNone, false, dev_status, stream);
    }
    return st;
  }
  if (routed) {
    st = launch_grouped_gemm_f32(g1r, act1, stream);
    if (st == MOE_OK) st = launch_grouped_gemm_f32(g2r, kActNone, stream);
  }
  if (st == MOE_OK && shared) {
    st = launch_grouped_gemm_f32(g1s, kActGelu, stream);
    if (st == MOE_OK) st = launch_grouped_gemm_f32(g2s, kActNone, stream);
  }
  return st;
}

DispatchArgs dispatch_args(const moe_config &c, const int32_t *sel, int32_t *offsets,
                           int32_t *perm, int32_t *row_of, int32_t *tok_ptr,
                           int32_t *tok_assign, int32_t *dev_status) {
  DispatchArgs a;
  a.routing = c.routing;
  a.T = c.T; a.E = c.E; a.n_heavy = c.n_heavy; a.k = c.k;
  a.S = c.group_size; a.C = c.capacity;
  a.n_assign = n_assign_of(c);
  a.sel = sel; a.offsets = offsets; a.perm = perm; a.row_of = row_of;
  a.tok_ptr = tok_ptr; a.tok_assign = tok_assign; a.dev_status = dev_status;
  a.zero_words = nullptr; a.n_zero_words = 0;
  return a;
}

CombineArgs combine_args(const moe_config &c, const void *y_perm, const void *y_shared,
                         const int32_t *sel, const float *w, const int32_t *row_of,
                         const int32_t *tok_ptr, const int32_t *tok_assign, const void *x,
                         const void *const_vecs, const void *residual, void *y,
                         int32_t *dev_status) {
  CombineArgs a;
  a.routing = c.routing; a.T = c.T; a.d = c.d; a.E = c.E; a.k = c.k;
  a.S = c.group_size; a.C = c.capacity; a.dtype = c.dtype; a.const_mix = c.const_mix;
  a.y_perm = y_perm; a.y_shared = y_shared; a.sel = sel; a.w = w; a.row_of = row_of;
  a.tok_ptr = tok_ptr; a.tok_assign = tok_assign; a.x = x; a.const_vecs = const_vecs;
  a.residual = residual; a.y = y; a.dev_status = dev_status;
  a.y_rows = n_assign_of(c);
  return a;
}

// NVTX range over a scope: names the layer's stages for a profiler
// (header-only NVTX; a no-op unless a tool is attached).
struct NvtxScope {
  explicit NvtxScope(const char *name) { nvtxRangePushA(name); }
  ~NvtxScope() { nvtxRangePop(); }
  NvtxScope(const NvtxScope &) = delete;
  NvtxScope &operator=(const NvtxScope &) = delete;
};
// Consecutive NVTX ranges: next() closes the open one and opens another.
struct NvtxStages {
  bool open = false;
  void next(const char *name) {
    if (open) nvtxRangePop();
    nvtxRangePushA(name);
    open = true;
  }
  ~NvtxStages() {
    if (open) nvtxRangePop();
  }
};

int forward_device(const moe_config &c, const void *x, const void *residual,
                   const float *z_prev, const void *W_r, const float *bias, const void *W1,
                   const void *W2, const void *Ws1, const void *Ws2, const void *const_vecs,
                   void *y, const moe_forward_aux *aux, int32_t *dev_status, void *ws,
                   const Layout &L, cudaStream_t stream) {
  float *logits = (aux && aux->logits) ? aux->logits : at<float>(ws, L.logits);
  float *probs = (aux && aux->probs) ? aux->probs : at<float>(ws, L.probs);
  int32_t *sel = (aux && aux->sel) ? aux->sel : at<int32_t>(ws, L.sel);
  float *w = (aux && aux->w) ? aux->w : at<float>(ws, L.w);
  int64_t *votes = (aux && aux->votes) ? aux->votes : at<int64_t>(ws, L.votes);
  int32_t *core = (aux && aux->core) ? aux->core : at<int32_t>(ws, L.core);
  int32_t *offsets = (aux && aux->offsets) ? aux->offsets : at<int32_t>(ws, L.offsets);
  int32_t *perm = at<int32_t>(ws, L.perm), *row_of = at<int32_t>(ws, L.row_of);
  int32_t *tok_ptr = at<int32_t>(ws, L.tok_ptr), *tok_assign = at<int32_t>(ws, L.tok_assign);
  const int64_t na = n_assign_of(c);
  const int64_t hs = (int64_t)c.n_shared * c.h_shared;
  void *Y = at<void>(ws, L.Y);
  void *Y_sh = hs ? at<void>(ws, L.Y_sh) : nullptr;
  void *x_perm = at<void>(ws, L.x_perm);
  NvtxScope layer_range("moe_forward");

  int st = MOE_OK;
  const int n_part = router_split_parts(c.T, c.d, c.dtype);
  const bool streaming = c.dtype == MOE_BF16 && stream_mlp_supported(c.T);
  bool routed_and_gathered = false;
  if (small_f32_supported(c)) {
    NvtxScope r("moe_forward/one_launch_f32");
    // Small fp32 token-choice layer without a shared expert: the whole layer
    // in one launch, a CTA per token (its per-expert row counts, and the
    // CTA counter that finds the last CTA, start at zero).
    MOE_CUDA_TRY(cudaMemsetAsync(at<void>(ws, L.fzero), 0, small_f32_zero_bytes(c.n_heavy), stream));
    SmallF32Args fa{};
    fa.x = static_cast<const float *>(x);
    fa.residual = static_cast<const float *>(residual);
    fa.W_r = static_cast<const float *>(W_r);
    fa.bias = bias; fa.zprev = z_prev; fa.zscale = c.gate_residual_scale;
    fa.W1 = static_cast<const float *>(W1); fa.W2 = static_cast<const float *>(W2);
    fa.const_vecs = static_cast<const float *>(const_vecs);
    fa.T = c.T; fa.d = c.d; fa.h = c.h; fa.E = c.E; fa.n_heavy = c.n_heavy; fa.k = c.k;
    fa.renorm = c.renorm; fa.gated = c.act == MOE_SWIGLU;
    fa.logits = logits; fa.probs = probs; fa.w = w; fa.y = static_cast<float *>(y);
    fa.sel = sel; fa.offsets = offsets; fa.counts = at<unsigned>(ws, L.fzero);
    return launch_small_f32(fa, kind_table(c), stream);
  }
  if (moe_block_supported(c)) {
    NvtxScope r("moe_forward/one_launch_block");
    // Small bf16 block without a shared expert: the whole layer in one
    // persistent kernel (router K-sliced over the CTAs, selection, a weight
    // stream that starts as soon as the experts to stream are known, the
    // combine). Its sync words, bitmasks, vote totals and counters start
    // at zero.
    BlockArgs ba{};
    MOE_CUDA_TRY(cudaMemsetAsync(at<void>(ws, L.bzero), 0, block_zero_bytes(c.E, c.n_heavy), stream));
    block_zero_layout(ba, at<void>(ws, L.bzero), c.E);
    ba.W_r = W_r; ba.part = at<float>(ws, L.rpart);
    ba.n_slices = block_router_slices(c.d, &ba.kslice);
    ba.bias = bias; ba.zprev = z_prev; ba.zscale = c.gate_residual_scale;
    ba.T = c.T; ba.E = c.E; ba.n_heavy = c.n_heavy; ba.k = c.k; ba.routing = c.routing;
    ba.renorm = c.renorm; ba.M_core = c.M_core; ba.k_local = c.k_local;
    ba.d = c.d; ba.h = c.h; ba.w1_rows_per_group = c.act == MOE_SWIGLU ? 2 * c.h : c.h;
    ba.x = x; ba.residual = residual; ba.const_vecs = const_vecs; ba.y = y;
    ba.H = at<void>(ws, L.H); ba.Y = at<void>(ws, L.Y);
    ba.logits = logits; ba.probs = probs; ba.sel = sel; ba.w = w;
    ba.votes_out = c.routing == MOE_DES_VOTE ? votes : nullptr; ba.core = core;
    ba.offsets = offsets; ba.perm = perm; ba.row_of = row_of;
    ba.dev_status = dev_status;
    return launch_moe_block(ba, kind_table(c), W1, W2, c.act, stream);
  }
  NvtxStages stage;
  stage.next("moe_forward/route");
  if (n_part > 0 && small_route_supported(c.T, c.E, c.k, c.routing, c.dtype)) {
    // Small bf16 block (<= 128 tokens): the router split over the model
    // width, then one cooperative kernel finishes the router, selects (DES:
    // votes, elects, re-routes), dispatches and gathers the rows. The split
    // router clears the vote totals, the barrier counter and the
    // weight-streaming kernel's counters on its way.
    const bool des = c.routing == MOE_DES_VOTE;
    ZeroList zero{};
    zero.p[0] = at<int32_t>(ws, L.cbar);
    zero.n[0] = 4 + 4 * c.E;
    if (des) { zero.p[1] = reinterpret_cast<int32_t *>(votes); zero.n[1] = 2 * c.E; }
    if (streaming) { zero.p[2] = at<int32_t>(ws, L.done); zero.n[2] = c.n_heavy + 1; }
    st = launch_router_partial(x, W_r, c.T, c.d, c.E, at<float>(ws, L.rpart), n_part, zero, stream);
    if (st != MOE_OK) return st;
    SmallRouteArgs sa{};
    sa.part = at<float>(ws, L.rpart); sa.n_part = n_part;
    sa.bias = bias; sa.zprev = z_prev; sa.zscale = c.gate_residual_scale;
    sa.T = c.T; sa.E = c.E; sa.n_heavy = c.n_heavy; sa.k = c.k; sa.routing = c.routing;
    sa.renorm = c.renorm; sa.M_core = c.M_core;
    sa.row_vecs = (int)((int64_t)c.d * elem_bytes(c.dtype) / 16);
    sa.x = static_cast<const uint4 *>(x); sa.x_perm = static_cast<uint4 *>(x_perm);
    sa.logits = logits; sa.probs = probs; sa.sel = sel; sa.w = w;
    sa.votes = reinterpret_cast<unsigned long long *>(votes); sa.core = core;
    sa.offsets = offsets; sa.perm = perm; sa.row_of = row_of;
    sa.barrier = at<unsigned>(ws, L.cbar); sa.gmask = at<unsigned>(ws, L.cbar) + 4;
    sa.dev_status = dev_status;
    st = launch_small_route(sa, stream);
    if (st != MOE_OK) return st;
    routed_and_gathered = true;
  } else if (n_part > 0 && (c.routing == MOE_TOKEN_TOPK || c.routing == MOE_DES_VOTE)) {
    // Small bf16 block: router split over the model width, then a per-token
    // finish that also selects (token choice) or sums the exact int64 DES
    // votes (cleared by the split router); DES then elects the core set and
    // re-routes per token.
    const bool des = c.routing == MOE_DES_VOTE;
    st = launch_router_split(x, W_r, bias, z_prev, c.gate_residual_scale, c.T, c.d, c.E,
                             at<float>(ws, L.rpart), n_part, logits, probs, des ? 0 : c.k,
                             c.renorm, des ? nullptr : sel, des ? nullptr : w,
                             des ? votes : nullptr, des ? c.k : 0, stream);
    if (st == MOE_OK && des)
      st = launch_des_reroute(probs, votes, c.T, c.E, c.k, c.M_core, core, sel, w, stream);
    if (st != MOE_OK) return st;
  } else {
    st = launch_router(x, W_r, bias, z_prev, c.gate_residual_scale, c.T, c.d, c.E, c.dtype, logits,
                       probs, c.routing == MOE_TOKEN_TOPK ? c.k : 0, c.renorm, sel, w, stream);
    if (st != MOE_OK) return st;
    if (c.routing == MOE_EXPERT_CHOICE)
      st = launch_expert_choice(probs, c.T, c.E, c.group_size, c.capacity, sel, w, stream);
    else if (c.routing == MOE_DES_VOTE)
      st = launch_des_vote(probs, c.T, c.E, c.k, c.M_core, votes, core, sel, w, stream);
    else if (c.routing == MOE_DES_SEQ)  // the core-set size goes to the (unused) vote slot
      st = launch_des_seq(probs, c.T, c.E, c.k, c.k_local, core,
                          reinterpret_cast<int32_t *>(at<int64_t>(ws, L.votes)), sel, w, stream);
    if (st != MOE_OK) return st;
  }
  // bf16 grouped-GEMM path with a shared expert: its down-projection epilogue
  // writes y = residual + shared(x) straight into y, and the combine then adds
  // the routed terms in place (no shared-output buffer round trip).
  const bool shared_into_y = hs > 0 && c.dtype == MOE_BF16 && !streaming && c.T > 0;
  // With routed rows too, the shared up projection runs on the side stream
  // during the dispatch and row gather (small launches that leave most of
  // each SM free), joined before the down projections.
  SideFork side(stream);
  const bool side_shared = shared_into_y && c.n_heavy > 0 && na > 0 && !routed_and_gathered;
  if (side_shared) {
    st = side.fork();
    if (st != MOE_OK) return st;
    const GemmProblem g1s = shared_up_problem(c, x, Ws1, at<void>(ws, L.H_sh), dev_status);
    const GemmProblem g1r = routed_up_problem(c, x_perm, offsets, W1, at<void>(ws, L.H), dev_status);
    st = launch_grouped_gemm_bf16(&g1s, 1, kActGelu, false, dev_status, side.side(),
                                  c.act == MOE_SWIGLU ? nullptr : &g1r);
    if (st != MOE_OK) return st;
  }
  stage.next("moe_forward/dispatch");
  if (!routed_and_gathered) {
    DispatchArgs da = dispatch_args(c, sel, offsets, perm, row_of, tok_ptr, tok_assign, dev_status);
    if (streaming) {  // the dispatch clears the weight-streaming kernel's counters
      da.zero_words = at<int32_t>(ws, L.done);
      da.n_zero_words = c.n_heavy + 1;
    }
    // The selection above is this library's own: under expert choice every
    // token id is in its group and every expert has exactly C of them.
    if (c.routing == MOE_EXPERT_CHOICE && dispatch_ec_supported(c.group_size, c.E, c.capacity))
      st = launch_dispatch_ec(da, stream);
    else
      st = launch_dispatch(da, at<void>(ws, L.dpart), stream);
    if (st != MOE_OK) return st;
    if (c.n_heavy > 0) {
      st = launch_gather_rows(x, x_perm, perm, offsets, c.n_heavy, na, c.d, elem_bytes(c.dtype), stream);
      if (st != MOE_OK) return st;
    }
  }
  stage.next("moe_forward/grouped_mlp");
  st = run_grouped_mlp(c, x_perm, offsets, W1, W2, x, Ws1, Ws2, Y, shared_into_y ? y : Y_sh,
                       dev_status, ws, L, stream, streaming, shared_into_y ? residual : nullptr,
                       side_shared ? &side : nullptr);
  if (st != MOE_OK) return st;
  CombineArgs ca = combine_args(c, Y, shared_into_y ? nullptr : Y_sh, sel, w, row_of, tok_ptr,
                                tok_assign, x, const_vecs, shared_into_y ? y : residual, y,
                                dev_status);
  stage.next("moe_forward/combine");
  return launch_combine(ca, kind_table(c), stream);
}

int check_forward_ptrs(const moe_config &c, const void *x, const void *W_r, const void *W1,
                       const void *W2, const void *Ws1, const void *Ws2,
                       const void *const_vecs, const void *y) {
  if (!W_r || !aligned16(W_r)) return MOE_ERR_INVALID_ARG;
  if (c.T > 0 && (!x || !y)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if (c.n_heavy > 0 && (!W1 || !W2 || !aligned16(W1) || !aligned16(W2))) return MOE_ERR_INVALID_ARG;
  if (c.n_shared > 0 && (!Ws1 || !Ws2 || !aligned16(Ws1) || !aligned16(Ws2))) return MOE_ERR_INVALID_ARG;
  if (n_const_of(c) > 0 && (!const_vecs || !aligned16(const_vecs))) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: valid but unsupported";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA call failed";
    case MOE_ERR_DEVICE_STATUS: return "MOE_ERR_DEVICE_STATUS: device status word set";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: bounded device wait expired";
    default: return "unknown moe_status";
  }
}

int moe_device_check(int device) {
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess)
    return MOE_ERR_CUDA;
  return (major == 10 && minor == 0) ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

int moe_num_assignments(const moe_config *cfg, int64_t *n_assign) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!n_assign) return MOE_ERR_INVALID_ARG;
  *n_assign = n_assign_of(*cfg);
  return MOE_OK;
}

int moe_workspace_size(const moe_config *cfg, size_t *bytes) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = layout_of(*cfg).total;
  return MOE_OK;
}

int moe_router(const void *x, const void *W_r, const float *bias, const float *z_prev,
               float z_prev_scale, int T, int d, int E, int dtype, float *logits, float *probs,
               int k, int renorm, int32_t *idx, float *w, moe_stream_t stream) {
  if (T < 0 || d < 8 || E < 1) return MOE_ERR_INVALID_ARG;
  if (E > 128) return MOE_ERR_UNSUPPORTED;
  if (dtype != MOE_BF16 && dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  if (dtype == MOE_BF16 && d % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (!W_r) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!x || !logits || !probs)) return MOE_ERR_INVALID_ARG;
  if (dtype == MOE_BF16 && (!aligned16(x) || !aligned16(W_r))) return MOE_ERR_INVALID_ARG;
  if (k < 0 || k > E || (k > 0 && (!idx || !w))) return MOE_ERR_INVALID_ARG;
  if (renorm != 0 && renorm != 1) return MOE_ERR_INVALID_ARG;
  return launch_router(x, W_r, bias, z_prev, z_prev_scale, T, d, E, dtype, logits, probs, k,
                       renorm, idx, w, stream);
}

int moe_select_topk(const float *logits, const float *probs, int T, int E, int k, int renorm,
                    int32_t *idx, float *w, moe_stream_t stream) {
  if (T < 0 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (E > 128) return MOE_ERR_UNSUPPORTED;
  if (!logits || !probs || !idx || !w) return MOE_ERR_INVALID_ARG;
  if (renorm != 0 && renorm != 1) return MOE_ERR_INVALID_ARG;
  return launch_select_topk(logits, probs, T, E, k, renorm, idx, w, stream);
}

int moe_select_expert_choice(const float *probs, int T, int E, int group_size, int C,
                             int32_t *tok, float *w, moe_stream_t stream) {
  if (T < 0 || E < 1 || group_size < 1 || T % group_size != 0) return MOE_ERR_INVALID_ARG;
  if (C < 1 || C > group_size) return MOE_ERR_INVALID_ARG;
  if (group_size > 16384) return MOE_ERR_UNSUPPORTED;
  if (!probs || !tok || !w) return MOE_ERR_INVALID_ARG;
  return launch_expert_choice(probs, T, E, group_size, C, tok, w, stream);
}

int moe_core_set_vote(const float *probs, int N, int M, int K, int M_core, int64_t *votes,
                      int32_t *core, int32_t *idx, float *w, moe_stream_t stream) {
  if (N < 0 || M < 1 || K < 1 || K > M_core || M_core > M) return MOE_ERR_INVALID_ARG;
  if (M > MOE_MAX_EXPERTS || N > 4096) return MOE_ERR_UNSUPPORTED;
  if (!probs || !votes || !core || !idx || !w) return MOE_ERR_INVALID_ARG;
  return launch_des_vote(probs, N, M, K, M_core, votes, core, idx, w, stream);
}

int moe_core_set_union(const float *probs, int N, int M, int K, int k_local, int32_t *core,
                       int32_t *n_core, int32_t *idx, float *w, moe_stream_t stream) {
  if (N < 0 || M < 1 || K < 1 || K > M || k_local < 1 || k_local > M) return MOE_ERR_INVALID_ARG;
  if (M > MOE_MAX_EXPERTS || N > 4096) return MOE_ERR_UNSUPPORTED;
  if (!probs || !core || !n_core || !idx || !w) return MOE_ERR_INVALID_ARG;
  return launch_des_seq(probs, N, M, K, k_local, core, n_core, idx, w, stream);
}

int moe_dispatch(const moe_config *cfg, const int32_t *sel, const void *x, void *x_perm,
                 int32_t *offsets, int32_t *perm, int32_t *row_of, int32_t *tok_ptr,
                 int32_t *tok_assign, int32_t *dev_status, void *ws, size_t ws_bytes,
                 moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (!offsets) return MOE_ERR_INVALID_ARG;
  if (n_assign_of(c) > 0 && (!sel || !perm || !row_of)) return MOE_ERR_INVALID_ARG;
  if (x_perm && (!x || !aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  if (c.routing == MOE_EXPERT_CHOICE && (!tok_ptr != !tok_assign)) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  const Layout L = layout_of(c);
  DispatchArgs da = dispatch_args(c, sel, offsets, perm, row_of, tok_ptr, tok_assign, dev_status);
  st = launch_dispatch(da, at<void>(ws, L.dpart), stream);
  if (st != MOE_OK || !x_perm || c.n_heavy == 0) return st;
  return launch_gather_rows(x, x_perm, perm, offsets, c.n_heavy, n_assign_of(c), c.d,
                            elem_bytes(c.dtype), stream);
}

int moe_dispatch_noalloc(const moe_config *cfg, const int32_t *sel, const void *x, void *x_perm,
                         int32_t *offsets, int32_t *perm, int32_t *row_of, int32_t *tok_ptr,
                         int32_t *tok_assign, int32_t *dev_status, moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (!offsets) return MOE_ERR_INVALID_ARG;
  if (n_assign_of(c) > 0 && (!sel || !perm || !row_of)) return MOE_ERR_INVALID_ARG;
  if (x_perm && (!x || !aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  if (c.routing == MOE_EXPERT_CHOICE && (!tok_ptr != !tok_assign)) return MOE_ERR_INVALID_ARG;
  if (!dispatch_fits_noalloc_scratch(n_assign_of(c), c.n_heavy)) return MOE_ERR_UNSUPPORTED;
  DispatchArgs da = dispatch_args(c, sel, offsets, perm, row_of, tok_ptr, tok_assign, dev_status);
  st = launch_dispatch_noalloc(da, stream);
  if (st != MOE_OK || !x_perm || c.n_heavy == 0) return st;
  return launch_gather_rows(x, x_perm, perm, offsets, c.n_heavy, n_assign_of(c), c.d,
                            elem_bytes(c.dtype), stream);
}

int moe_grouped_mlp(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                    const void *W1, const void *W2, const void *x, const void *Ws1,
                    const void *Ws2, void *y_perm, void *y_shared, int32_t *dev_status,
                    void *ws, size_t ws_bytes, moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (c.n_heavy > 0 && (!x_perm || !offsets || !W1 || !W2 || !y_perm)) return MOE_ERR_INVALID_ARG;
  if (c.n_heavy > 0 && (!aligned16(x_perm) || !aligned16(W1) || !aligned16(W2) || !aligned16(y_perm)))
    return MOE_ERR_INVALID_ARG;
  if (c.n_shared > 0 && (!x || !Ws1 || !Ws2 || !y_shared)) return MOE_ERR_INVALID_ARG;
  if (c.n_shared > 0 && (!aligned16(x) || !aligned16(Ws1) || !aligned16(Ws2) || !aligned16(y_shared)))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  return run_grouped_mlp(c, x_perm, offsets, W1, W2, x, Ws1, Ws2, y_perm, y_shared, dev_status,
                         ws, layout_of(c), stream);
}

int moe_combine(const moe_config *cfg, const void *y_perm, const void *y_shared,
                const int32_t *sel, const float *w, const int32_t *row_of,
                const int32_t *tok_ptr, const int32_t *tok_assign, const void *x,
                const void *const_vecs, const void *residual, void *y, int32_t *dev_status,
                moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (c.T > 0 && (!sel || !w || !row_of || !x || !y)) return MOE_ERR_INVALID_ARG;
  if (c.n_heavy > 0 && !y_perm) return MOE_ERR_INVALID_ARG;
  if (c.n_shared > 0 && !y_shared) return MOE_ERR_INVALID_ARG;
  if (c.routing == MOE_EXPERT_CHOICE && (!tok_ptr || !tok_assign)) return MOE_ERR_INVALID_ARG;
  if (n_const_of(c) > 0 && !const_vecs) return MOE_ERR_INVALID_ARG;
  const void *ptrs[6] = {y_perm, y_shared, x, const_vecs, residual, y};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  CombineArgs ca = combine_args(c, y_perm, c.n_shared > 0 ? y_shared : nullptr, sel, w, row_of,
                                tok_ptr, tok_assign, x, const_vecs, residual, y, dev_status);
  return launch_combine(ca, kind_table(c), stream);
}

int moe_activation(const float *x, float *y, int64_t n, int act, moe_stream_t stream) {
  if (n < 0 || (act != MOE_GELU_ERF && act != MOE_SWIGLU)) return MOE_ERR_INVALID_ARG;
  if (n > 0 && (!x || !y)) return MOE_ERR_INVALID_ARG;
  return launch_activation(x, y, n, act, stream);
}

int moe_build_flags(void) { return MOE_DEBUG ? MOE_BUILD_DEBUG : 0; }

int moe_test_set_barrier_wait(uint64_t limit_ns, int extra_arrivals) {
  if (limit_ns > 2000000000ull || extra_arrivals < 0 || extra_arrivals > 1024)
    return MOE_ERR_INVALID_ARG;
  set_small_route_test_wait((unsigned long long)limit_ns, extra_arrivals);
  return MOE_OK;
}

int moe_forward(const moe_config *cfg, const void *x, const void *residual, const float *z_prev,
                const void *W_r, const float *bias, const void *W1, const void *W2,
                const void *Ws1, const void *Ws2, const void *const_vecs, void *y,
                const moe_forward_aux *aux, int32_t *dev_status, void *ws, size_t ws_bytes,
                moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if ((st = check_forward_ptrs(c, x, W_r, W1, W2, Ws1, Ws2, const_vecs, y)) != MOE_OK) return st;
  if (residual && !aligned16(residual)) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  return forward_device(c, x, residual, z_prev, W_r, bias, W1, W2, Ws1, Ws2, const_vecs, y, aux,
                        dev_status, ws, layout_of(c), stream);
}

int moe_forward_host(const moe_config *cfg, const void *x_host, const void *residual_host,
                     const float *z_prev_host, const void *W_r, const float *bias,
                     const void *W1, const void *W2, const void *Ws1, const void *Ws2,
                     const void *const_vecs, void *y_host, int32_t *dev_status, void *ws,
                     size_t ws_bytes, moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config &c = *cfg;
  if (c.T > 0 && (!x_host || !y_host)) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  const Layout L = layout_of(c);
  void *xd = at<void>(ws, L.x_dev), *yd = at<void>(ws, L.y_dev);
  if ((st = check_forward_ptrs(c, xd, W_r, W1, W2, Ws1, Ws2, const_vecs, yd)) != MOE_OK) return st;
  HostCopy hc;
  hc.xh = static_cast<const uint8_t *>(x_host);
  hc.yh = static_cast<uint8_t *>(y_host);
  hc.rh = residual_host == x_host ? nullptr : static_cast<const uint8_t *>(residual_host);
  hc.zh = reinterpret_cast<const uint8_t *>(z_prev_host);
  hc.xd = static_cast<uint8_t *>(xd);
  hc.yd = static_cast<uint8_t *>(yd);
  hc.rd = residual_host == nullptr ? nullptr
          : residual_host == x_host ? hc.xd : at<uint8_t>(ws, L.res_dev);
  hc.zd = z_prev_host ? at<uint8_t>(ws, L.zp_dev) : nullptr;
  hc.row = (size_t)c.d * elem_bytes(c.dtype);
  hc.zrow = (size_t)c.E * 4;

  int64_t bounds[kHostMaxChunks + 1];
  const int n = host_chunk_plan(c, bounds);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  MOE_CUDA_TRY(cudaStreamIsCapturing(stream, &cap));
  bool pipelined = n > 1 && cap == cudaStreamCaptureStatusNone;
  // Every chunk's routing and MLP buffers must lie below the staging slots.
  for (int i = 0; pipelined && i < n; ++i) {
    moe_config ci = c;
    ci.T = (int32_t)(bounds[i + 1] - bounds[i]);
    pipelined = layout_of(ci).x_dev <= L.x_dev;
  }
  if (!pipelined) {
    if ((st = hc.in(0, c.T, stream)) != MOE_OK) return st;
    st = forward_device(c, xd, hc.rd, reinterpret_cast<const float *>(hc.zd), W_r, bias, W1, W2,
                        Ws1, Ws2, const_vecs, yd, nullptr, dev_status, ws, L, stream);
    if (st != MOE_OK) return st;
    return hc.out(0, c.T, stream);
  }

  // Copy-in on one side stream, copy-out on another, the layer on `stream`,
  // chunk by chunk: chunk i computes while chunk i+1 comes in and chunk i-1
  // goes out. The side streams fork from `stream` here and join it at the end.
  std::lock_guard<std::mutex> lock(g_host_pipe_mu);
  HostPipe *hp = nullptr;
  if ((st = host_pipe(&hp)) != MOE_OK) return st;
  MOE_CUDA_TRY(cudaEventRecord(hp->ev[0], stream));
  MOE_CUDA_TRY(cudaStreamWaitEvent(hp->in, hp->ev[0], 0));
  for (int i = 0; i < n; ++i) {
    const int64_t t0 = bounds[i], nt = bounds[i + 1] - bounds[i];
    if ((st = hc.in(t0, nt, hp->in)) != MOE_OK) return st;
    MOE_CUDA_TRY(cudaEventRecord(hp->ev[2 + 2 * i], hp->in));
  }
  for (int i = 0; i < n; ++i) {
    const int64_t t0 = bounds[i], nt = bounds[i + 1] - bounds[i];
    moe_config ci = c;
    ci.T = (int32_t)nt;
    MOE_CUDA_TRY(cudaStreamWaitEvent(stream, hp->ev[2 + 2 * i], 0));
    st = forward_device(ci, hc.xd + t0 * hc.row, hc.rd ? hc.rd + t0 * hc.row : nullptr,
                        hc.zd ? reinterpret_cast<const float *>(hc.zd + t0 * hc.zrow) : nullptr,
                        W_r, bias, W1, W2, Ws1, Ws2, const_vecs, hc.yd + t0 * hc.row, nullptr,
                        dev_status, ws, layout_of(ci), stream);
    if (st != MOE_OK) return st;
    MOE_CUDA_TRY(cudaEventRecord(hp->ev[3 + 2 * i], stream));
    MOE_CUDA_TRY(cudaStreamWaitEvent(hp->out, hp->ev[3 + 2 * i], 0));
    if ((st = hc.out(t0, nt, hp->out)) != MOE_OK) return st;
  }
  MOE_CUDA_TRY(cudaEventRecord(hp->ev[1], hp->out));
  MOE_CUDA_TRY(cudaStreamWaitEvent(stream, hp->ev[1], 0));
  return MOE_OK;
}

}  // extern "C"
