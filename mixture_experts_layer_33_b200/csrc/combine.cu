// Combine back to token order, fused with the routing-weight scale, the
// zero-computation experts, the shared expert and the residual add.
//
// DICE: Staleness-Centric Optimizations for Parallel Diffusion MoE
// Inference, "Conditional Communication": a token's output is the sum of
// its experts' outputs weighted by its routing scores.
// MMOE: Modernizing Diffusion Transformers with Efficient Expert Design,
// "MoE++ expert layer": identity experts return x, zero experts return 0,
// constant experts return a learned vector; "shared experts": one dense
// expert is always active (added with weight 1).
//
// One warp per token (or, when there are too few tokens to occupy the
// GPU that way, per 256-feature chunk of a token); each lane owns 8
// consecutive features of a chunk and reads them with 16-byte loads. The
// token's slot metadata is loaded once per item, one slot per lane (when
// its slots fit in a warp), and turned into a source row and weight per
// slot; the row then goes in passes of up to three chunks, each pass
// issuing the residual, shared-output and slot-row loads of all its chunks
// before any sum, so a token costs about one dependent round trip per pass
// after the metadata.
// The grid holds only resident blocks. Expert outputs arrive in the layer
// dtype; the sum runs in fp32 in slot order (no atomics, so the output is
// bitwise deterministic) and is rounded once. `residual` may alias `y`
// (the forward pass writes x + shared(x) into y first): each lane reads
// its own features of a chunk before it writes them.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 2;  // slots whose rows are in flight together
constexpr int kPass = 3;   // 256-feature chunks per pass

// 8 consecutive elements held raw until they are summed.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16 *p) { u = *reinterpret_cast<const uint4 *>(p); }
  __device__ __forceinline__ void fma_into(float wgt, float (&acc)[8]) const {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      acc[2 * i] = fmaf(wgt, f.x, acc[2 * i]);
      acc[2 * i + 1] = fmaf(wgt, f.y, acc[2 * i + 1]);
    }
  }
};
template <> struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float *p) {
    a = *reinterpret_cast<const float4 *>(p);
    b = *reinterpret_cast<const float4 *>(p + 4);
  }
  __device__ __forceinline__ void fma_into(float wgt, float (&acc)[8]) const {
    acc[0] = fmaf(wgt, a.x, acc[0]); acc[1] = fmaf(wgt, a.y, acc[1]);
    acc[2] = fmaf(wgt, a.z, acc[2]); acc[3] = fmaf(wgt, a.w, acc[3]);
    acc[4] = fmaf(wgt, b.x, acc[4]); acc[5] = fmaf(wgt, b.y, acc[5]);
    acc[6] = fmaf(wgt, b.z, acc[6]); acc[7] = fmaf(wgt, b.w, acc[7]);
  }
};

// (a0, a1) = softmax(Wc . x) of a mixed constant expert, Wc = rows 1..2 of
// its [3, d] block `vrow`; fp32 dot products by the whole warp. Out of
// line: the rare path keeps its registers to itself.
template <typename T>
__device__ __noinline__ float2 const_mix_weights(const T *xr, const T *vrow, int d) {
  const int lane = threadIdx.x & 31;
  float z0 = 0.f, z1 = 0.f;
  for (int c = lane * 8; c < d; c += 256) {
    float xv[8], w0[8], w1[8];
    load8(xr + c, xv);
    load8(vrow + d + c, w0);
    load8(vrow + 2 * d + c, w1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      z0 = fmaf(xv[i], w0[i], z0);
      z1 = fmaf(xv[i], w1[i], z1);
    }
  }
  z0 = warp_sum(z0);
  z1 = warp_sum(z1);
  const float mz = fmaxf(z0, z1);
  const float e0 = expf(z0 - mz), e1 = expf(z1 - mz);
  return make_float2(e0 / (e0 + e1), e1 / (e0 + e1));
}

// Slot j of token s, one per lane: its source row (the expert's output
// row, x_s for an identity expert, the learned vector for a constant
// expert) and weight, or no row (zero expert, a row the dispatch dropped,
// an id it flagged). *mix marks a mixed constant expert.
template <typename T>
__device__ __forceinline__ void slot_meta(const CombineArgs &a, const KindTable &kinds, bool ec,
                                          int s, int j, const T *x, const T *cv, const T *yp,
                                          const T *&src, float &wgt, bool &mix) {
  src = nullptr;
  wgt = 0.f;
  mix = false;
  const int asg = ec ? a.tok_assign[j] : j;
#if MOE_DEBUG
  if (asg < 0 || asg >= a.y_rows) {  // a token list entry out of range: skip the slot
    set_status(a.dev_status, MOE_DEV_BAD_INDEX);
    return;
  }
#endif
  const int e = ec ? (int)((asg / a.C) % a.E) : a.sel[asg];
  int row = a.row_of[asg];
#if MOE_DEBUG
  if (row >= a.y_rows) {  // a row past the expert outputs: no term
    set_status(a.dev_status, MOE_DEV_BAD_INDEX);
    row = -1;
  }
#endif
  const float wv = a.w[asg];
  if (e >= 0 && e < a.E) {
    const int kind = kinds.kind[e];
    if (kind == MOE_HEAVY) {
      if (row >= 0) src = yp + (size_t)row * a.d;
    } else if (kind == MOE_IDENTITY) {
      src = x + (size_t)s * a.d;
    } else if (kind == MOE_CONST) {
      src = cv + (size_t)kinds.cidx[e] * (a.const_mix ? 3 : 1) * a.d;
      mix = a.const_mix != 0;
    }
    wgt = wv;
  }
}

// Slots j0 .. j0+31 of token s (one per lane) with mixed constant experts
// resolved: the warp forms (a0, a1) = softmax(Wc x_s) for each such slot,
// which keeps w * a1 on v; w * a0 is added to *x_coef when it is given.
template <typename T>
__device__ __forceinline__ void slot_group(const CombineArgs &a, const KindTable &kinds, bool ec,
                                           int s, int j0, int a1, const T *x, const T *cv,
                                           const T *yp, const T *&src, float &wgt,
                                           float *x_coef) {
  const int lane = threadIdx.x & 31;
  bool mix = false;
  src = nullptr;
  wgt = 0.f;
  if (j0 + lane < a1) slot_meta(a, kinds, ec, s, j0 + lane, x, cv, yp, src, wgt, mix);
  for (unsigned mm = __ballot_sync(0xffffffffu, mix); mm; mm &= mm - 1u) {
    const int j = __ffs(mm) - 1;
    const T *vrow = reinterpret_cast<const T *>(
        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(src), j));
    const float2 m = const_mix_weights(x + (size_t)s * a.d, vrow, a.d);
    const float wj = __shfl_sync(0xffffffffu, wgt, j);
    if (x_coef) *x_coef = fmaf(wj, m.x, *x_coef);
    if (lane == j) wgt = wj * m.y;
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineArgs a, KindTable kinds) {
  const T *__restrict__ x = static_cast<const T *>(a.x);
  const T *res = static_cast<const T *>(a.residual);  // may alias y
  const T *__restrict__ cv = static_cast<const T *>(a.const_vecs);
  const T *__restrict__ yp = static_cast<const T *>(a.y_perm);
  const T *__restrict__ ysh = static_cast<const T *>(a.y_shared);
  T *y = static_cast<T *>(a.y);
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int nw = (gridDim.x * kThreads) >> 5;
  const bool ec = a.routing == MOE_EXPERT_CHOICE;
  const int chunks = (a.d + 255) / 256;
  // An item is a whole token (its metadata read once), or with few tokens
  // one 256-feature chunk of a token, so that every warp has work.
  const int per_item = a.fine ? 1 : chunks;
  const int items_per_tok = a.fine ? chunks : 1;
  const int64_t items = (int64_t)a.T * items_per_tok;
  for (int64_t it = gw; it < items; it += nw) {
    const int s = (int)(it / items_per_tok);
    const int c_begin = (int)(it - (int64_t)s * items_per_tok) * per_item;
    const int c_end = c_begin + per_item < chunks ? c_begin + per_item : chunks;
    int a0, a1;
    if (ec) { a0 = a.tok_ptr[s]; a1 = a.tok_ptr[s + 1]; }
    else { a0 = s * a.k; a1 = a0 + a.k; }
#if MOE_DEBUG
    if (a0 < 0 || a1 < a0 || a1 > a.y_rows) {  // a token list out of range: no slots
      if (lane == 0) set_status(a.dev_status, MOE_DEV_BAD_INDEX);
      a0 = a1 = 0;
    }
#endif
    const bool one_group = a1 - a0 <= 32;
    // Slot metadata (and the coefficient of x_s from mixed constant
    // experts) once per token; a token with more than 32 slots re-reads
    // its later groups' metadata in each pass.
    const T *m_src = nullptr;
    float m_w = 0.f, x_coef = 0.f;
    if (one_group) {
      slot_group(a, kinds, ec, s, a0, a1, x, cv, yp, m_src, m_w, &x_coef);
    } else if (a.const_mix) {
      for (int j0 = a0; j0 < a1; j0 += 32) {
        const T *q_src;
        float q_w;
        slot_group(a, kinds, ec, s, j0, a1, x, cv, yp, q_src, q_w, &x_coef);
      }
    }
    const size_t rb = (size_t)s * a.d;
    for (int cb = c_begin; cb < c_end; cb += kPass) {
      int c0[kPass];
      bool live[kPass];
      float acc[kPass][8];
#pragma unroll
      for (int q = 0; q < kPass; ++q) {
        c0[q] = (cb + q) * 256 + lane * 8;
        live[q] = cb + q < c_end && c0[q] < a.d;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[q][i] = 0.f;
        if (live[q] && res) load8(res + rb + c0[q], acc[q]);
        if (live[q] && ysh) {
          float t[8];
          load8(ysh + rb + c0[q], t);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[q][i] += t[i];
        }
      }
      for (int j0 = a0; j0 < a1; j0 += 32) {
        const T *g_src = m_src;
        float g_w = m_w;
        if (!one_group) slot_group(a, kinds, ec, s, j0, a1, x, cv, yp, g_src, g_w, nullptr);
        const int nj = min(32, a1 - j0);
        for (int jb = 0; jb < nj; jb += kBatch) {
          Raw8<T> raw[kBatch][kPass];
          const T *src[kBatch];
          float wgt[kBatch];
#pragma unroll
          for (int u = 0; u < kBatch; ++u) {
            const int j = (jb + u) & 31;
            src[u] = reinterpret_cast<const T *>(
                __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(g_src), j));
            wgt[u] = __shfl_sync(0xffffffffu, g_w, j);
            if (jb + u >= nj) src[u] = nullptr;
#pragma unroll
            for (int q = 0; q < kPass; ++q)
              if (src[u] && live[q]) raw[u][q].load(src[u] + c0[q]);
          }
#pragma unroll
          for (int u = 0; u < kBatch; ++u)
#pragma unroll
            for (int q = 0; q < kPass; ++q)
              if (src[u] && live[q]) raw[u][q].fma_into(wgt[u], acc[q]);
        }
      }
#pragma unroll
      for (int q = 0; q < kPass; ++q) {
        if (!live[q]) continue;
        if (x_coef != 0.f) {
          Raw8<T> xs;
          xs.load(x + rb + c0[q]);
          xs.fma_into(x_coef, acc[q]);
        }
        store8(y + rb + c0[q], acc[q]);
      }
    }
  }
}

}  // namespace

// Blocks of `kern` that are resident on one SM.
template <typename K>
int resident_blocks(K kern) {
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kThreads, 0) != cudaSuccess || nb < 1)
    nb = 1;
  return nb;
}

int launch_combine(const CombineArgs &a, const KindTable &kinds, cudaStream_t stream) {
  if (a.T == 0) return MOE_OK;
  // Asked once per kernel (function-local statics are initialised once,
  // safely under concurrent first calls).
  static const int nb_bf16 = resident_blocks(combine_kernel<__nv_bfloat16>);
  static const int nb_f32 = resident_blocks(combine_kernel<float>);
  const bool bf16 = a.dtype == MOE_BF16;
  const int nb = bf16 ? nb_bf16 : nb_f32;
  // Whole-token items unless that leaves most resident warps idle.
  const int64_t warps = (int64_t)num_sms() * nb * (kThreads / 32);
  const int chunks = (a.d + 255) / 256;
  const int64_t passes = (chunks + kPass - 1) / kPass;
  CombineArgs ka = a;
  ka.fine = (int64_t)a.T * passes < warps ? 1 : 0;
  const int64_t items = (int64_t)a.T * (ka.fine ? chunks : 1);
  int64_t blocks = (items + (kThreads / 32) - 1) / (kThreads / 32);  // a warp per item
  const int64_t cap = (int64_t)num_sms() * nb;
  if (blocks > cap) blocks = cap;
  const int grid = (int)blocks;
  if (bf16) combine_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(ka, kinds);
  else combine_kernel<float><<<grid, kThreads, 0, stream>>>(ka, kinds);
  return last_launch_status();
}

}  // namespace moe
