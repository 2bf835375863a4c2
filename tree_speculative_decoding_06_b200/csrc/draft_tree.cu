// tsd_draft_tree_init / _expand / _finalize: the EAGLE-2 draft tree built on the device.
//
// "Acelerando Sonar a traves de la especulacion", section "EAGLE": EAGLE-2 shapes the draft tree
// dynamically, expanding the Top-K candidates of every node and scoring the draft sequences.
// Reading of that passage (the pages give no more): a node's children are its K most likely
// draft tokens, a node's score is the cumulative draft log-probability of its root->node path,
// the next nodes to expand are the F best children, and the final tree keeps the root and the
// best keep-1 nodes by score, ordered by (depth, score desc, node index).
//
// Expansion is two launches: a vocabulary scan (one CTA per 16384-token chunk of every frontier
// row: chunk maximum, fp64 sum of fp32 exponentials, chunk top-K) and one CTA per sequence that
// merges the chunks (log-sum-exp, row top-K), appends the children and picks the new frontier by
// rank counting.  Finalisation is one CTA per sequence: rank every node by score, keep the best,
// renumber by (depth, score, index), remap parents.  Scores are fp64.
#include <climits>

#include "common.cuh"
#include "draft_tree.h"
#include "kernels.h"

namespace tsd {

namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 16384;           // vocabulary entries per scan CTA
constexpr int kMaxK = 16;               // children per node
constexpr int kMaxFinalNodes = 4096;    // tree capacity finalize stages on chip

__host__ __device__ inline int dt_chunks(int V) { return (V + kChunk - 1) / kChunk; }
// per (sequence, frontier row, chunk): fp64 sum, fp32 max, then K (value, index) pairs
__host__ __device__ inline size_t dt_rec_bytes(int K) { return ((size_t)16 + (size_t)8 * K + 15) & ~(size_t)15; }

struct ChunkRec {
  double s;
  float m;
  float pad;
};

__device__ __forceinline__ bool better_node(double sa, int ia, double sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

// Warp-cooperative top-K (K <= kMaxK <= 32): lane k < K holds the warp's k-th best (value, index)
// so far (best first; ties -> lower index).  A candidate enters only if it beats the K-th best, so
// after the first few hundred tokens almost every 32-token batch is dismissed by one ballot; an
// entry is placed by one ballot (its rank) and one shuffle (the lanes below it move down).
struct WarpTopK {
  float v;
  int i;
};

__device__ __forceinline__ void wtopk_insert(WarpTopK& me, int K, int lane, float x, int xi) {
  const bool ahead = lane < K && better(me.v, me.i, x, xi);
  const int pos = __popc(__ballot_sync(0xffffffffu, ahead));
  const float up_v = __shfl_up_sync(0xffffffffu, me.v, 1);
  const int up_i = __shfl_up_sync(0xffffffffu, me.i, 1);
  if (lane < K) {
    if (lane == pos) me.v = x, me.i = xi;
    else if (lane > pos) me.v = up_v, me.i = up_i;
  }
}

// Offer each lane's candidate (x, xi) to the warp list; `thr` (the K-th best) is kept current.
__device__ __forceinline__ void wtopk_offer(WarpTopK& me, WarpTopK& thr, int K, int lane, float x, int xi) {
  unsigned want = __ballot_sync(0xffffffffu, better(x, xi, thr.v, thr.i));
  while (want) {
    const int src = __ffs(want) - 1;
    const float cx = __shfl_sync(0xffffffffu, x, src);
    const int ci = __shfl_sync(0xffffffffu, xi, src);
    wtopk_insert(me, K, lane, cx, ci);
    thr.v = __shfl_sync(0xffffffffu, me.v, K - 1);
    thr.i = __shfl_sync(0xffffffffu, me.i, K - 1);
    want &= want - 1;
    want &= __ballot_sync(0xffffffffu, better(x, xi, thr.v, thr.i));
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) draft_row_stats(const T* __restrict__ logits, int V, int F, int K,
                                                            int chunks, uint8_t* __restrict__ ws, int vec) {
  pdl_trigger();
  const int c = blockIdx.x, f = blockIdx.y, b = blockIdx.z;
  const T* row = logits + ((size_t)b * F + f) * V;
  const int lo = c * kChunk, hi = min(V, lo + kChunk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WarpTopK me{-INFINITY, INT_MAX}, thr{-INFINITY, INT_MAX};
  float m = -INFINITY;
  // 16-byte path: the thread's 64 logits of the chunk are loaded at once (one round trip to
  // memory) and kept in registers for the maximum, the top-K offers and the exponential sum
  constexpr int kGroups = kChunk / (kThreads * 8);
  float xr[kGroups][8];
  if (vec) {
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi) {
      const int v = lo + (gi * kThreads + threadIdx.x) * 8;
      if (v < hi) {
        load8<T>(row, v, xr[gi]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) xr[gi][e] = -INFINITY;
      }
    }
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi) {
      const int v = lo + (gi * kThreads + threadIdx.x) * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        m = fmaxf(m, xr[gi][e]);
        wtopk_offer(me, thr, K, lane, xr[gi][e], v < hi ? v + e : INT_MAX);
      }
    }
  } else {
    for (int v0 = lo; v0 < hi; v0 += kThreads) {
      const int v = v0 + threadIdx.x;
      const float x = v < hi ? load1(row, v) : -INFINITY;
      m = fmaxf(m, x);
      wtopk_offer(me, thr, K, lane, x, v < hi ? v : INT_MAX);
    }
  }
  // chunk maximum
  __shared__ float s_m[kThreads / 32];
  __shared__ double s_s[kThreads / 32];
  __shared__ float s_wv[kThreads / 32][kMaxK];
  __shared__ int s_wi[kThreads / 32][kMaxK];
  float wm = warp_max(m);
  if (lane == 0) s_m[warp] = wm;
  if (lane < K) s_wv[warp][lane] = me.v, s_wi[warp][lane] = me.i;
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) M = fmaxf(M, s_m[w]);
  // fp64 sum of fp32 exponentials relative to the chunk maximum (second pass, cache-resident)
  double sum = 0.0;
  if (M != -INFINITY) {
    if (vec) {
#pragma unroll
      for (int gi = 0; gi < kGroups; ++gi) {
        float t = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) t += expf(xr[gi][e] - M);   // -inf padding adds 0
        sum += (double)t;
      }
    } else {
      for (int v = lo + threadIdx.x; v < hi; v += kThreads) sum += (double)expf(load1(row, v) - M);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) s_s[warp] = sum;
  // chunk top-K: warp 0 offers the other warps' lists to its own, K candidates per lane batch
  __shared__ float s_topv[kMaxK];
  __shared__ int s_topi[kMaxK];
  if (warp == 0) {
    for (int w = 1; w < kThreads / 32; ++w) {
      const float x = lane < K ? s_wv[w][lane] : -INFINITY;
      const int xi = lane < K ? s_wi[w][lane] : INT_MAX;
      wtopk_offer(me, thr, K, lane, x, xi);
    }
    if (lane < K) s_topv[lane] = me.v, s_topi[lane] = me.i;
  }
  __syncthreads();
  pdl_wait();   // the previous expansion may still be reading the workspace
  if (threadIdx.x == 0) {
    double S = 0.0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) S += s_s[w];
    uint8_t* rec = ws + (((size_t)b * F + f) * chunks + c) * dt_rec_bytes(K);
    ChunkRec cr;
    cr.s = S, cr.m = M, cr.pad = 0.f;
    *reinterpret_cast<ChunkRec*>(rec) = cr;
    float* vals = reinterpret_cast<float*>(rec + 16);
    int* idxs = reinterpret_cast<int*>(rec + 16 + 4 * K);
    for (int k = 0; k < K; ++k) vals[k] = s_topv[k], idxs[k] = s_topi[k];
  }
}

__global__ void __launch_bounds__(kThreads) draft_init_kernel(DraftTreeArgs t, const int32_t* __restrict__ root_token,
                                                              int32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= t.B) return;
  const size_t base = (size_t)b * t.max_nodes;
  t.parent[base] = -1;
  t.token[base] = root_token[b];
  t.score[base] = 0.0;
  t.depth[base] = 0;
  t.num_nodes[b] = 1;
  t.frontier[(size_t)b * t.F] = 0;
  t.num_frontier[b] = 1;
  status[b] = 0;
}

__global__ void __launch_bounds__(kThreads) draft_expand_kernel(DraftTreeArgs t, int K, int chunks,
                                                                const uint8_t* __restrict__ ws,
                                                                int32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) uint8_t s_recs[];
  __shared__ double s_sc[kMaxK * kMaxK];
  __shared__ int s_id[kMaxK * kMaxK];
  const int b = blockIdx.x;
  const int nf = t.num_frontier[b], n0 = t.num_nodes[b];
  const size_t base = (size_t)b * t.max_nodes;
  if (status[b] != 0 || nf <= 0) return;
  if (nf > t.F || (long long)n0 + (long long)nf * K > t.max_nodes) {
    if (threadIdx.x == 0) flag_status(status, b, TSD_ERR_CAPACITY);
    return;
  }
  // every chunk record of the sequence into shared memory with one coalesced read, so the row
  // merges below do not chain dependent global loads
  const size_t rb = dt_rec_bytes(K);
  {
    const uint4* src = reinterpret_cast<const uint4*>(ws + (size_t)b * t.F * chunks * rb);
    uint4* dst = reinterpret_cast<uint4*>(s_recs);
    const int n16 = (int)((size_t)nf * chunks * rb / 16);
    for (int i = threadIdx.x; i < n16; i += blockDim.x) dst[i] = src[i];
  }
  __syncthreads();
  // one thread per frontier row: merge the chunk records, append the row's K children
  const int f = threadIdx.x;
  if (f < nf) {
    const uint8_t* recs = s_recs + (size_t)f * chunks * rb;
    float M = -INFINITY;
    for (int c = 0; c < chunks; ++c) M = fmaxf(M, reinterpret_cast<const ChunkRec*>(recs + c * rb)->m);
    double S = 0.0;
    for (int c = 0; c < chunks; ++c) {
      const ChunkRec* cr = reinterpret_cast<const ChunkRec*>(recs + c * rb);
      if (cr->m != -INFINITY) S += cr->s * exp((double)cr->m - (double)M);
    }
    const double lse = (double)M + log(S);
    const int p = t.frontier[(size_t)b * t.F + f];
    const double sp = t.score[base + p];
    const int dp = t.depth[base + p];
    int head[64];   // per-chunk read position of the K-way merge (chunks <= 64)
    for (int c = 0; c < chunks; ++c) head[c] = 0;
    for (int k = 0; k < K; ++k) {
      float bv = -INFINITY;
      int bi = INT_MAX, bc = -1;
      for (int c = 0; c < chunks; ++c) {
        if (head[c] >= K) continue;
        const uint8_t* rec = recs + c * rb;
        const float v = reinterpret_cast<const float*>(rec + 16)[head[c]];
        const int i = reinterpret_cast<const int*>(rec + 16 + 4 * K)[head[c]];
        if (i != INT_MAX && better(v, i, bv, bi)) bv = v, bi = i, bc = c;
      }
      if (bc >= 0) ++head[bc];
      const int node = n0 + f * K + k;
      const double sc = sp + ((double)bv - lse);
      t.parent[base + node] = p;
      t.token[base + node] = bi == INT_MAX ? 0 : bi;
      t.score[base + node] = sc;
      t.depth[base + node] = dp + 1;
      s_sc[f * K + k] = sc;
      s_id[f * K + k] = node;
    }
  }
  __syncthreads();
  // new frontier: rank of every child among all children by (score desc, node index asc)
  const int nc = nf * K;
  for (int j = threadIdx.x; j < nc; j += blockDim.x) {
    int rank = 0;
    for (int i = 0; i < nc; ++i) rank += better_node(s_sc[i], s_id[i], s_sc[j], s_id[j]) ? 1 : 0;
    if (rank < t.F) t.frontier[(size_t)b * t.F + rank] = s_id[j];
  }
  if (threadIdx.x == 0) {
    t.num_nodes[b] = n0 + nc;
    t.num_frontier[b] = nc < t.F ? nc : t.F;
  }
}

__global__ void __launch_bounds__(kThreads) draft_finalize_kernel(DraftTreeArgs t, int keep,
                                                                  int32_t* __restrict__ parent_out,
                                                                  int32_t* __restrict__ tokens_out,
                                                                  int32_t* __restrict__ num_out,
                                                                  int32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) uint8_t smem[];
  const int b = blockIdx.x;
  const int n = t.num_nodes[b];
  const size_t base = (size_t)b * t.max_nodes;
  int32_t* prow = parent_out + (size_t)b * keep;
  int32_t* trow = tokens_out + (size_t)b * keep;
  const bool bad = status[b] != 0 || n < 1 || n > t.max_nodes;
  const int kept_n = bad ? 0 : min(keep, n);
  if (bad) {
    for (int i = threadIdx.x; i < keep; i += blockDim.x) prow[i] = -1, trow[i] = 0;
    if (threadIdx.x == 0) num_out[b] = 0;
    return;
  }
  double* s_sc = reinterpret_cast<double*>(smem);
  int* s_dep = reinterpret_cast<int*>(s_sc + n);
  int* s_map = s_dep + n;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    s_sc[i] = t.score[base + i];
    s_dep[i] = t.depth[base + i];
    s_map[i] = -1;
  }
  __syncthreads();
  // kept: the root and the kept_n - 1 best other nodes by (score desc, index asc)
  for (int i = 1 + threadIdx.x; i < n; i += blockDim.x) {
    int rank = 0;
    for (int j = 1; j < n; ++j) rank += better_node(s_sc[j], j, s_sc[i], i) ? 1 : 0;
    if (rank < kept_n - 1) s_map[i] = -2;   // kept, position below
  }
  __syncthreads();
  // position among the kept by (depth asc, score desc, index asc); the root is position 0
  for (int i = 1 + threadIdx.x; i < n; i += blockDim.x) {
    if (s_map[i] != -2) continue;
    int pos = 1;
    for (int j = 1; j < n; ++j) {
      if (j == i) continue;
      const int mj = s_map[j];
      if (mj == -1) continue;   // not kept (a kept node's entry is -2 or already its position)
      const bool before = s_dep[j] < s_dep[i] || (s_dep[j] == s_dep[i] && better_node(s_sc[j], j, s_sc[i], i));
      pos += before ? 1 : 0;
    }
    s_map[i] = -1000 - pos;     // kept marker that stays distinct from -1 while others still read
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    if (s_map[i] <= -1000) s_map[i] = -1000 - s_map[i];
  if (threadIdx.x == 0) s_map[0] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int pos = s_map[i];
    if (pos < 0) continue;
    const int p = t.parent[base + i];
    int np = -1;
    if (i > 0) {
      np = (p >= 0 && p < n) ? s_map[p] : -1;
      if (np < 0) flag_status(status, b, TSD_ERR_BAD_TREE, i);   // not ancestor-closed (never for scores)
    }
    prow[pos] = np;
    trow[pos] = t.token[base + i];
  }
  for (int i = kept_n + threadIdx.x; i < keep; i += blockDim.x) prow[i] = -1, trow[i] = 0;
  if (threadIdx.x == 0) num_out[b] = kept_n;
}

}  // namespace

size_t draft_expand_ws(int B, int F, int K, int V) { return (size_t)B * F * dt_chunks(V) * dt_rec_bytes(K); }

tsd_status launch_draft_init(const DraftTreeArgs& t, const int32_t* root_token, int32_t* status, cudaStream_t stream) {
  if (t.B == 0) return TSD_OK;
  launch_pdl(draft_init_kernel, dim3((t.B + kThreads - 1) / kThreads), dim3(kThreads), 0, stream, t, root_token, status);
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

tsd_status launch_draft_expand(const DraftTreeArgs& t, const void* logits, tsd_dtype dtype, int V, int K, void* ws,
                               int32_t* status, cudaStream_t stream) {
  if (t.B == 0) return TSD_OK;
  if (K < 1 || K > kMaxK || t.F < 1 || t.F > kMaxK || dt_chunks(V) > 64) return TSD_ERR_INVALID_ARG;
  const int chunks = dt_chunks(V);
  dim3 grid(chunks, t.F, t.B);
  const int vec = vec16_rows(logits, V) ? 1 : 0;
  if (dtype == TSD_BF16)
    launch_pdl(draft_row_stats<__nv_bfloat16>, grid, dim3(kThreads), 0, stream,
               reinterpret_cast<const __nv_bfloat16*>(logits), V, t.F, K, chunks, reinterpret_cast<uint8_t*>(ws), vec);
  else
    launch_pdl(draft_row_stats<float>, grid, dim3(kThreads), 0, stream, reinterpret_cast<const float*>(logits), V, t.F,
               K, chunks, reinterpret_cast<uint8_t*>(ws), vec);
  if (cudaGetLastError() != cudaSuccess) return TSD_ERR_CUDA;
  const size_t smem = (size_t)t.F * chunks * dt_rec_bytes(K);   // <= 16 x 64 x 144 B
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(draft_expand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch_pdl(draft_expand_kernel, dim3(t.B), dim3(kThreads), smem, stream, t, K, chunks, (const uint8_t*)ws, status);
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

tsd_status launch_draft_finalize(const DraftTreeArgs& t, int keep, int32_t* parent_out, int32_t* tokens_out,
                                 int32_t* num_out, int32_t* status, cudaStream_t stream) {
  if (t.B == 0) return TSD_OK;
  if (t.max_nodes > kMaxFinalNodes || keep < 1) return TSD_ERR_INVALID_ARG;
  const size_t smem = (size_t)t.max_nodes * (8 + 4 + 4);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(draft_finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch_pdl(draft_finalize_kernel, dim3(t.B), dim3(kThreads), smem, stream, t, keep, parent_out, tokens_out, num_out,
             status);
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

}  // namespace tsd
