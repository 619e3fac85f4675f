// Dispatch: stable permutation of the heavy assignments into per-expert
// groups (histogram -> exclusive scan -> scatter) and the row gather.
//
// DICE: Staleness-Centric Optimizations for Parallel Diffusion MoE
// Inference, "Conditional Communication": tokens are dispatched to their
// experts and the outputs are combined back weighted by the routing score;
// this is the single-GPU form of that dispatch (rows grouped by expert in
// HBM instead of an all-to-all).
//
// Rows are ordered by (expert, assignment index). Assignments are numbered
// in slot order, which makes the rows of each expert ascend by token for
// token choice (a = s*k + j), DES (a = n*K + j) and expert choice
// (a = (g*E + e)*C + c, tokens ascending within a group).
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 4;
constexpr int kChunk = kThreads * kPerThread;  // assignments per block
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ bool decode(const DispatchArgs &a, int64_t i, int &tok, int &exp) {
  if (a.routing == MOE_EXPERT_CHOICE) {
    exp = (int)((i / a.C) % a.E);
    tok = a.sel[i];
    const int g = (int)(i / ((int64_t)a.E * a.C));
    if (tok < g * a.S || tok >= (g + 1) * a.S) {
      set_status(a.dev_status, MOE_DEV_BAD_TOKEN);
      return false;
    }
  } else {
    tok = (int)(i / a.k);
    exp = a.sel[i];
    if (exp == -1) return false;  // an empty slot (DES-Seq): no row, no flag
    if (exp < 0 || exp >= a.E) {
      set_status(a.dev_status, MOE_DEV_BAD_EXPERT);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void clear_words(const DispatchArgs &a) {
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < a.n_zero_words; i += blockDim.x) a.zero_words[i] = 0;
}

__global__ void __launch_bounds__(kThreads) dispatch_count_kernel(DispatchArgs a, int32_t *partial) {
  __shared__ int hist[MOE_MAX_EXPERTS];
  clear_words(a);
  for (int e = threadIdx.x; e < a.n_heavy; e += kThreads) hist[e] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kChunk;
  for (int r = 0; r < kPerThread; ++r) {
    int64_t i = base + r * kThreads + threadIdx.x;
    int tok, exp;
    if (i < a.n_assign && decode(a, i, tok, exp) && exp < a.n_heavy) atomicAdd(&hist[exp], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.n_heavy; e += kThreads)
    partial[(size_t)blockIdx.x * a.n_heavy + e] = hist[e];
}

// One block: offsets[e] = sum of counts of experts < e; partial[b][e]
// becomes the first row of block b's expert-e rows.
__global__ void __launch_bounds__(kThreads) dispatch_scan_kernel(DispatchArgs a, int32_t *partial, int nb) {
  __shared__ int scratch[33];
  const int e = threadIdx.x;
  int total_e = 0;
  if (e < a.n_heavy)
    for (int b = 0; b < nb; ++b) total_e += partial[(size_t)b * a.n_heavy + e];
  int all;
  int off = block_exclusive_scan(e < a.n_heavy ? total_e : 0, scratch, &all);
  if (e < a.n_heavy) {
    a.offsets[e] = off;
    int run = off;
    for (int b = 0; b < nb; ++b) {
      int c = partial[(size_t)b * a.n_heavy + e];
      partial[(size_t)b * a.n_heavy + e] = run;
      run += c;
    }
  }
  if (e == 0) a.offsets[a.n_heavy] = all;
}

// Stable scatter of one chunk of kChunk assignments starting at `base`;
// base_rows[e] is the first row of this chunk's expert-e rows.
__device__ __forceinline__ void scatter_chunk(const DispatchArgs &a, int64_t base,
                                              const int32_t *base_rows, int *run,
                                              int (*wcnt)[MOE_MAX_EXPERTS]) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < a.n_heavy; e += kThreads) {
    run[e] = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) wcnt[w][e] = 0;
  }
  __syncthreads();
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int r = 0; r < kPerThread; ++r) {
    const int64_t i = base + r * kThreads + tid;
    int tok = 0, exp = -1;
    bool valid = i < a.n_assign && decode(a, i, tok, exp);
    int key = (valid && exp < a.n_heavy) ? exp : -1;
    unsigned peers = __match_any_sync(0xffffffffu, key);
    int rank_w = __popc(peers & lt_mask);
    if (key >= 0 && rank_w == 0) wcnt[warp][key] = __popc(peers);
    __syncthreads();
    if (key >= 0) {
      int before = run[key] + rank_w;
      for (int w = 0; w < warp; ++w) before += wcnt[w][key];
      const int row = base_rows[key] + before;
      a.perm[row] = tok;
      a.row_of[i] = row;
    } else if (i < a.n_assign) {
      a.row_of[i] = -1;
    }
    __syncthreads();
    for (int e = tid; e < a.n_heavy; e += kThreads) {
      int s = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) { s += wcnt[w][e]; wcnt[w][e] = 0; }
      run[e] += s;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kThreads) dispatch_scatter_kernel(DispatchArgs a, const int32_t *base_rows) {
  __shared__ int run[MOE_MAX_EXPERTS];
  __shared__ int wcnt[kWarps][MOE_MAX_EXPERTS];
  scatter_chunk(a, (int64_t)blockIdx.x * kChunk, base_rows + (size_t)blockIdx.x * a.n_heavy, run,
                wcnt);
}

// All assignments fit one chunk: histogram, scan and scatter in one block.
__global__ void __launch_bounds__(kThreads) dispatch_single_block_kernel(DispatchArgs a) {
  __shared__ int hist[MOE_MAX_EXPERTS];
  __shared__ int32_t offs[MOE_MAX_EXPERTS];
  __shared__ int scratch[33];
  __shared__ int run[MOE_MAX_EXPERTS];
  __shared__ int wcnt[kWarps][MOE_MAX_EXPERTS];
  clear_words(a);
  for (int e = threadIdx.x; e < a.n_heavy; e += kThreads) hist[e] = 0;
  __syncthreads();
  for (int r = 0; r < kPerThread; ++r) {
    int64_t i = r * kThreads + threadIdx.x;
    int tok, exp;
    if (i < a.n_assign && decode(a, i, tok, exp) && exp < a.n_heavy) atomicAdd(&hist[exp], 1);
  }
  __syncthreads();
  const int e = threadIdx.x;
  int all;
  int off = block_exclusive_scan(e < a.n_heavy ? hist[e] : 0, scratch, &all);
  if (e < a.n_heavy) {
    offs[e] = off;
    a.offsets[e] = off;
  }
  if (e == 0) a.offsets[a.n_heavy] = all;
  __syncthreads();
  scatter_chunk(a, 0, offs, run, wcnt);
}

// Expert choice: each token's assignments in slot order, one block per
// routing group (the tokens and assignments of group g are contiguous).
__global__ void __launch_bounds__(kThreads) token_csr_kernel(DispatchArgs a) {
  extern __shared__ int sm[];
  int *cnt = sm;           // [S]
  int *ptr = sm + a.S;     // [S]
  __shared__ int scratch[33];
  const int g = blockIdx.x, S = a.S, E = a.E, C = a.C;
  const int64_t abase = (int64_t)g * E * C;
  for (int t = threadIdx.x; t < S; t += kThreads) cnt[t] = 0;
  __syncthreads();
  for (int j = threadIdx.x; j < E * C; j += kThreads) {
    int t = a.sel[abase + j] - g * S;
    if (t >= 0 && t < S) atomicAdd(&cnt[t], 1);
  }
  __syncthreads();
  const int per = (S + kThreads - 1) / kThreads;
  const int lo = threadIdx.x * per, hi = min(S, lo + per);
  int mine = 0;
  for (int t = lo; t < hi; ++t) mine += cnt[t];
  int total;
  int run = block_exclusive_scan(mine, scratch, &total);
  for (int t = lo; t < hi; ++t) {
    ptr[t] = run;
    a.tok_ptr[(size_t)g * S + t] = (int32_t)(abase + run);
    run += cnt[t];
    cnt[t] = 0;  // reused as the fill count
  }
  if (g == gridDim.x - 1 && threadIdx.x == 0) a.tok_ptr[(size_t)gridDim.x * S] = (int32_t)(abase + total);
  __syncthreads();
  for (int e = 0; e < E; ++e) {
    for (int c = threadIdx.x; c < C; c += kThreads) {
      const int64_t i = abase + (int64_t)e * C + c;
      int t = a.sel[i] - g * S;
      if (t >= 0 && t < S) {
        int slot = atomicAdd(&cnt[t], 1);
        a.tok_assign[abase + ptr[t] + slot] = (int32_t)i;
      }
    }
    __syncthreads();
  }
}

// Expert choice in one launch, one CTA per routing group. EC-DiT, section
// 3 (Expert-Choice routing): every expert takes exactly C tokens of every
// group, so the stable permutation by (expert, token) has a closed form:
// expert e's rows start at e*G*C, and the c-th token (ascending) that
// expert took from group g lands in row e*G*C + g*C + c (groups are
// consecutive token ranges, so rows stay in ascending token order within
// an expert). No histogram, scan or scatter; the group's token ids are
// staged in shared memory once, and the per-token assignment lists (in
// expert order, for the combine) are built from there.
__global__ void __launch_bounds__(kThreads) dispatch_ec_kernel(DispatchArgs a) {
  extern __shared__ int sm[];
  const int S = a.S, E = a.E, C = a.C, G = gridDim.x, g = blockIdx.x;
  int *cnt = sm;        // [S]
  int *ptr = sm + S;    // [S]
  int *tk = sm + 2 * S; // [E * C] token (within the group) of each assignment, or -1
  __shared__ int scratch[33];
  clear_words(a);
  const int64_t abase = (int64_t)g * E * C;
  const int64_t per_expert = (int64_t)G * C;
  if (g == 0)
    for (int e = threadIdx.x; e <= a.n_heavy; e += kThreads) a.offsets[e] = (int32_t)(e * per_expert);
  for (int t = threadIdx.x; t < S; t += kThreads) cnt[t] = 0;
  __syncthreads();
  for (int j = threadIdx.x; j < E * C; j += kThreads) {
    const int e = j / C, c = j - (j / C) * C;
    int t = a.sel[abase + j] - g * S;
    if (t < 0 || t >= S) {
      set_status(a.dev_status, MOE_DEV_BAD_TOKEN);
      t = -1;
    } else {
      atomicAdd(&cnt[t], 1);
    }
    tk[j] = t;
    if (e < a.n_heavy) {
      const int64_t row = e * per_expert + (int64_t)g * C + c;
      // A dropped token still owns its row (the layout is fixed): it
      // gathers the group's first token and no slot reads its output.
      a.perm[row] = g * S + (t >= 0 ? t : 0);
      a.row_of[abase + j] = t >= 0 ? (int32_t)row : -1;
    } else {
      a.row_of[abase + j] = -1;
    }
  }
  __syncthreads();
  if (a.tok_ptr && a.tok_assign) {
    const int per = (S + kThreads - 1) / kThreads;
    const int lo = threadIdx.x * per, hi = min(S, lo + per);
    int mine = 0;
    for (int t = lo; t < hi; ++t) mine += cnt[t];
    int total;
    int run = block_exclusive_scan(mine, scratch, &total);
    for (int t = lo; t < hi; ++t) {
      ptr[t] = run;
      a.tok_ptr[(size_t)g * S + t] = (int32_t)(abase + run);
      run += cnt[t];
      cnt[t] = 0;  // reused as the fill count
    }
    if (g == G - 1 && threadIdx.x == 0) a.tok_ptr[(size_t)G * S] = (int32_t)(abase + total);
    __syncthreads();
    for (int e = 0; e < E; ++e) {  // expert order: one expert's tokens are distinct
      for (int c = threadIdx.x; c < C; c += kThreads) {
        const int t = tk[e * C + c];
        if (t >= 0) {
          const int slot = atomicAdd(&cnt[t], 1);
          a.tok_assign[abase + ptr[t] + slot] = (int32_t)(abase + (int64_t)e * C + c);
        }
      }
      __syncthreads();
    }
  }
}

// x_perm[r] = x[perm[r]] for r < offsets[n_heavy], 16-byte vectors.
__global__ void __launch_bounds__(kThreads)
gather_rows_kernel(const uint4 *__restrict__ x, uint4 *__restrict__ xp, const int32_t *__restrict__ perm,
                   const int32_t *__restrict__ offsets, int n_heavy, int vec_per_row) {
  const int64_t rows = offsets[n_heavy];
  const int64_t total = rows * vec_per_row;
  for (int64_t v = (int64_t)blockIdx.x * kThreads + threadIdx.x; v < total;
       v += (int64_t)gridDim.x * kThreads) {
    const int64_t r = v / vec_per_row;
    const int c = (int)(v - r * vec_per_row);
    xp[v] = __ldg(x + (int64_t)perm[r] * vec_per_row + c);
  }
}

}  // namespace

size_t dispatch_workspace_bytes(int64_t n_assign, int n_heavy) {
  int64_t nb = (n_assign + kChunk - 1) / kChunk;
  if (nb < 1) nb = 1;
  return (size_t)nb * (size_t)(n_heavy > 0 ? n_heavy : 1) * sizeof(int32_t);
}

int launch_dispatch(const DispatchArgs &a, void *ws, cudaStream_t stream) {
  int32_t *partial = static_cast<int32_t *>(ws);
  const int nb = (int)((a.n_assign + kChunk - 1) / kChunk);
  if (nb == 0) {
    MOE_CUDA_TRY(cudaMemsetAsync(a.offsets, 0, (a.n_heavy + 1) * sizeof(int32_t), stream));
    if (a.n_zero_words > 0)
      MOE_CUDA_TRY(cudaMemsetAsync(a.zero_words, 0, a.n_zero_words * sizeof(int32_t), stream));
  } else if (nb == 1) {
    dispatch_single_block_kernel<<<1, kThreads, 0, stream>>>(a);
  } else {
    dispatch_count_kernel<<<nb, kThreads, 0, stream>>>(a, partial);
    dispatch_scan_kernel<<<1, kThreads, 0, stream>>>(a, partial, nb);
    dispatch_scatter_kernel<<<nb, kThreads, 0, stream>>>(a, partial);
  }
  int st = last_launch_status();
  if (st != MOE_OK) return st;
  if (a.routing == MOE_EXPERT_CHOICE && a.tok_ptr && a.tok_assign && a.T > 0) {
    const size_t smem = 2 * (size_t)a.S * sizeof(int);
    MOE_CUDA_TRY(cudaFuncSetAttribute(token_csr_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    token_csr_kernel<<<a.T / a.S, kThreads, smem, stream>>>(a);
    st = last_launch_status();
  }
  return st;
}

// Shared memory of dispatch_ec_kernel: two words per token of a group and
// one per assignment of a group.
static size_t dispatch_ec_smem(int S, int E, int C) {
  return (2 * (size_t)S + (size_t)E * C) * sizeof(int);
}

bool dispatch_ec_supported(int S, int E, int C) {
  return S >= 1 && C >= 1 && dispatch_ec_smem(S, E, C) <= 48 * 1024;
}

int launch_dispatch_ec(const DispatchArgs &a, cudaStream_t stream) {
  if (a.T == 0 || a.S < 1) {
    MOE_CUDA_TRY(cudaMemsetAsync(a.offsets, 0, (a.n_heavy + 1) * sizeof(int32_t), stream));
    if (a.n_zero_words > 0)
      MOE_CUDA_TRY(cudaMemsetAsync(a.zero_words, 0, a.n_zero_words * sizeof(int32_t), stream));
    if (a.tok_ptr) MOE_CUDA_TRY(cudaMemsetAsync(a.tok_ptr, 0, sizeof(int32_t), stream));
    return MOE_OK;
  }
  dispatch_ec_kernel<<<a.T / a.S, kThreads, dispatch_ec_smem(a.S, a.E, a.C), stream>>>(a);
  return last_launch_status();
}

int launch_gather_rows(const void *x, void *x_perm, const int32_t *perm, const int32_t *offsets,
                       int n_heavy, int64_t max_rows, int d, int elem_bytes,
                       cudaStream_t stream) {
  if (max_rows == 0) return MOE_OK;
  const int vec = (int)((int64_t)d * elem_bytes / 16);
  int64_t want = (max_rows * vec + kThreads - 1) / kThreads;
  int64_t cap = (int64_t)num_sms() * 8;
  int grid = (int)(want < cap ? want : cap);
  if (grid < 1) grid = 1;
  gather_rows_kernel<<<grid, kThreads, 0, stream>>>(static_cast<const uint4 *>(x),
                                                    static_cast<uint4 *>(x_perm), perm, offsets,
                                                    n_heavy, vec);
  return last_launch_status();
}

}  // namespace moe
