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
constexpr int kMaxChunks = 64;          // vocabulary chunks per row (V <= 64 * kChunk)

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

// Offer each lane's candidate (x, xi) to the warp list.  `thr` is kept at the larger of the list's
// K-th best and the floor (floor_v, none): a candidate below it cannot make the top K.
__device__ __forceinline__ void wtopk_offer(WarpTopK& me, WarpTopK& thr, int K, int lane, float x, int xi,
                                            float floor_v) {
  unsigned want = __ballot_sync(0xffffffffu, better(x, xi, thr.v, thr.i));
  while (want) {
    const int src = __ffs(want) - 1;
    const float cx = __shfl_sync(0xffffffffu, x, src);
    const int ci = __shfl_sync(0xffffffffu, xi, src);
    wtopk_insert(me, K, lane, cx, ci);
    thr.v = __shfl_sync(0xffffffffu, me.v, K - 1);
    thr.i = __shfl_sync(0xffffffffu, me.i, K - 1);
    if (!better(thr.v, thr.i, floor_v, INT_MAX)) thr.v = floor_v, thr.i = INT_MAX;
    want &= want - 1;
    want &= __ballot_sync(0xffffffffu, better(x, xi, thr.v, thr.i));
  }
}

// The K-th largest of the 32 lane maxima (ties by lane): at least K tokens of the warp reach it, so
// it bounds the warp's K-th best from below.  -inf when no lane ranks K-th (NaN maxima).
__device__ __forceinline__ float kth_lane_max(float lm, int K, int lane) {
  int rank = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float o = __shfl_sync(0xffffffffu, lm, j);
    rank += (o > lm || (o == lm && j < lane)) ? 1 : 0;
  }
  const unsigned at = __ballot_sync(0xffffffffu, rank == K - 1);
  const float f = __shfl_sync(0xffffffffu, lm, at ? __ffs(at) - 1 : 0);
  return at ? f : -INFINITY;
}

constexpr float kLog2eHi = 1.44269502162933349609375f;            // fp32 part of log2(e)
constexpr float kLog2eLo = 1.925963033500011079198e-8f;           // log2(e) - kLog2eHi

__device__ __forceinline__ float exp_rel(float x, float m) {       // e^(x - m), x <= m
  const float d = x - m;
  return exp2f(fmaf(d, kLog2eHi, d * kLog2eLo));
}

// Offer a group of 8 consecutive tokens (v .. v+7) per lane.  Each lane marks the tokens that reach
// the threshold (the larger of the warp's K-th best and the floor); while any lane holds a mark,
// every such lane proposes its first one and the proposals enter the list one at a time (exact
// comparison, lowest lane first), after which the marks below the new threshold are dropped.  With
// a good floor a group usually costs one compare per token and one vote.
__device__ __forceinline__ void offer8(WarpTopK& me, WarpTopK& thr, int K, int lane, const float (&x)[8], int v,
                                       bool valid, float floor_v) {
  float m8 = x[0];
#pragma unroll
  for (int e = 1; e < 8; ++e) m8 = fmaxf(m8, x[e]);
  unsigned cand = 0;
  if (valid && m8 >= thr.v) {   // usually not: the floor dismisses the whole group
#pragma unroll
    for (int e = 0; e < 8; ++e) cand |= (x[e] >= thr.v ? 1u : 0u) << e;
  }
  while (__any_sync(0xffffffffu, cand != 0)) {
    const int e = __ffs(cand) - 1;
    float xv = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (e == j) xv = x[j];
    const int xi = cand ? v + e : INT_MAX;
    cand &= cand - 1;
    wtopk_offer(me, thr, K, lane, xv, xi, floor_v);
    if (cand) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (x[j] < thr.v) cand &= ~(1u << j);
    }
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
  // Pass 1: each lane's maximum; the warp's maximum is the reference of its exponential sum and the
  // K-th largest lane maximum is the floor of its top-K (at least K tokens reach it).  Pass 2 (the
  // chunk again, from cache): the exponentials and the offers of the tokens that reach the floor.
  float lm = -INFINITY;
  if (vec) {
    for (int v = lo + threadIdx.x * 8; v < hi; v += kThreads * 8) {
      float x[8];
      load8<T>(row, v, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) lm = fmaxf(lm, x[e]);
    }
  } else {
    for (int v = lo + threadIdx.x; v < hi; v += kThreads) lm = fmaxf(lm, load1(row, v));
  }
  const float wm = warp_max(lm);
  const float floor_v = kth_lane_max(lm, K, lane);
  thr.v = floor_v;
  double wsum = 0.0;
  if (vec) {
    // every lane of a warp runs the same trips (a lane past the end offers nothing)
    for (int g0 = lo; g0 < hi; g0 += kThreads * 8) {
      const int v = g0 + threadIdx.x * 8;
      const bool valid = v < hi;
      float x[8];
      if (valid) {
        load8<T>(row, v, x);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = -INFINITY;
      }
      if (wm != -INFINITY) wsum += (double)sum_ex2_8(x, wm, kLog2eHi, kLog2eLo);   // -inf adds 0
      offer8(me, thr, K, lane, x, v, valid, floor_v);
    }
  } else {
    for (int v0 = lo; v0 < hi; v0 += kThreads) {
      const int v = v0 + threadIdx.x;
      const float x = v < hi ? load1(row, v) : -INFINITY;
      if (wm != -INFINITY) wsum += (double)exp_rel(x, wm);
      wtopk_offer(me, thr, K, lane, x, v < hi ? v : INT_MAX, floor_v);
    }
  }
  // chunk maximum and sum: the warps' sums (relative to their maxima), then the block's maximum
  __shared__ float s_m[kThreads / 32];
  __shared__ double s_s[kThreads / 32];
  __shared__ float s_wv[kThreads / 32][kMaxK];
  __shared__ int s_wi[kThreads / 32][kMaxK];
  double sum = wsum;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) s_m[warp] = wm, s_s[warp] = sum;
  if (lane < K) s_wv[warp][lane] = me.v, s_wi[warp][lane] = me.i;
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) M = fmaxf(M, s_m[w]);
  // chunk top-K: each of the 8 K warp candidates counts the candidates that beat it and, if fewer
  // than K do, takes that slot (tokens are distinct across warps; unused slots keep (-inf, none))
  __shared__ float s_topv[kMaxK];
  __shared__ int s_topi[kMaxK];
  if (threadIdx.x < K) s_topv[threadIdx.x] = -INFINITY, s_topi[threadIdx.x] = INT_MAX;
  __syncthreads();
  if (threadIdx.x < (kThreads / 32) * K) {
    const int w = threadIdx.x / K, j = threadIdx.x % K;
    const float xv = s_wv[w][j];
    const int xi = s_wi[w][j];
    if (xi != INT_MAX) {
      int rank = 0;
      for (int w2 = 0; w2 < kThreads / 32; ++w2)
        for (int j2 = 0; j2 < K; ++j2) rank += better(s_wv[w2][j2], s_wi[w2][j2], xv, xi) ? 1 : 0;
      if (rank < K) s_topv[rank] = xv, s_topi[rank] = xi;
    }
  }
  __syncthreads();
  pdl_wait();   // the previous expansion may still be reading the workspace
  if (threadIdx.x == 0) {
    double S = 0.0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w)
      if (s_s[w] != 0.0) S += s_m[w] == M ? s_s[w] : s_s[w] * exp((double)s_m[w] - (double)M);
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
  // the row maxima, then every (row, chunk) sum rescaled to its row's maximum in fp64, then per row
  // the log-sum-exp (chunks summed in order)
  __shared__ float s_M[kMaxK];
  __shared__ double s_lse[kMaxK], s_psc[kMaxK];
  __shared__ int s_par[kMaxK], s_pdep[kMaxK];
  __shared__ double s_term[kMaxK * kMaxChunks];
  auto rec_at = [&](int f, int c) { return s_recs + ((size_t)f * chunks + c) * rb; };
  if (threadIdx.x < nf) {
    const int f = threadIdx.x;
    float M = -INFINITY;
    for (int c = 0; c < chunks; ++c) M = fmaxf(M, reinterpret_cast<const ChunkRec*>(rec_at(f, c))->m);
    s_M[f] = M;
    const int p = t.frontier[(size_t)b * t.F + f];
    s_par[f] = p, s_psc[f] = t.score[base + p], s_pdep[f] = t.depth[base + p];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < nf * chunks; idx += blockDim.x) {
    const int f = idx / chunks, c = idx % chunks;
    const ChunkRec* cr = reinterpret_cast<const ChunkRec*>(rec_at(f, c));
    s_term[f * kMaxChunks + c] = cr->m != -INFINITY ? cr->s * exp((double)cr->m - (double)s_M[f]) : 0.0;
  }
  __syncthreads();
  if (threadIdx.x < nf) {
    const int f = threadIdx.x;
    double S = 0.0;
    for (int c = 0; c < chunks; ++c) S += s_term[f * kMaxChunks + c];
    s_lse[f] = (double)s_M[f] + log(S);
  }
  __syncthreads();
  // the row's K children: each chunk candidate counts the candidates of its row that beat it and,
  // if fewer than K do, becomes that child (tokens are distinct across chunks, and the row holds
  // at least K candidates since K <= V)
  for (int idx = threadIdx.x; idx < nf * chunks * K; idx += blockDim.x) {
    const int f = idx / (chunks * K), rem = idx % (chunks * K), c = rem / K, k = rem % K;
    const uint8_t* rec = rec_at(f, c);
    const float xv = reinterpret_cast<const float*>(rec + 16)[k];
    const int xi = reinterpret_cast<const int*>(rec + 16 + 4 * K)[k];
    if (xi == INT_MAX) continue;
    int rank = 0;
    for (int c2 = 0; c2 < chunks; ++c2) {
      const uint8_t* r2 = rec_at(f, c2);
      const float* v2 = reinterpret_cast<const float*>(r2 + 16);
      const int* i2 = reinterpret_cast<const int*>(r2 + 16 + 4 * K);
      for (int k2 = 0; k2 < K; ++k2) rank += (i2[k2] != INT_MAX && better(v2[k2], i2[k2], xv, xi)) ? 1 : 0;
    }
    if (rank >= K) continue;
    const int node = n0 + f * K + rank;
    const double sc = s_psc[f] + ((double)xv - s_lse[f]);
    t.parent[base + node] = s_par[f];
    t.token[base + node] = xi;
    t.score[base + node] = sc;
    t.depth[base + node] = s_pdep[f] + 1;
    s_sc[f * K + rank] = sc;
    s_id[f * K + rank] = node;
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
