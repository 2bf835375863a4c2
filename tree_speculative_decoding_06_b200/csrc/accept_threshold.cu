// tsd_tree_accept_threshold: threshold acceptance over the draft tree.
//
// "Acelerando Sonar a traves de la especulacion" (Perplexity), section "Decodificacion
// especulativa": besides exact matching, the target may keep the longest prefix whose tokens stay
// above an acceptance threshold (the page gives no formula).  Reading: with
// p_n = softmax(target_logits[n] / T), a non-root node i is accepted iff its parent is and
// p_parent(i)(token[i]) >= tau; roots, the deepest-node rule and the emitted tokens (the target's
// own token is the argmax of the last accepted node's row) are those of greedy acceptance.
//
// Two launches: a vocabulary scan per (16384-token chunk, row) -- the argmax and, relative to the
// chunk's maximum, the fp64 sum of fp32 exponentials in one pass (16-byte loads; a thread's 64
// logits stay in registers) -- then one CTA per sequence merges the chunk statistics of every row,
// decides each edge p >= tau in fp64 from one gathered logit per node, and runs the greedy
// acceptance walk with those decisions.
#include <climits>

#include "accept_body.cuh"
#include "common.cuh"
#include "kernels.h"

namespace tsd {

namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 16384;
constexpr double kLog2eD = 1.4426950408889634074;

struct __align__(16) RowStat {
  float zm;   // chunk maximum (the argmax value), -inf if the chunk holds no number above -inf
  int bi;     // its lowest index
  double s;   // sum over the chunk of 2^((z - zm) log2(e) / T)
};

__host__ __device__ inline int num_chunks(int V) { return (V + kChunk - 1) / kChunk; }

__device__ __forceinline__ float expo(float z, float zm, float hi, float lo) {
  const float dz = z - zm;
  return exp2f(fmaf(dz, hi, dz * lo));
}

template <typename T>
__global__ void __launch_bounds__(kThreads) row_stats_chunks(const T* __restrict__ logits, int V, int rows_per_seq,
                                                             const int32_t* __restrict__ num_rows, int chunks,
                                                             float thi, float tlo, double cpow,
                                                             RowStat* __restrict__ part, int vec) {
  pdl_trigger();
  const int c = blockIdx.x, i = blockIdx.y, b = blockIdx.z;
  const int n = num_rows ? num_rows[b] : rows_per_seq;
  if (i >= n) {
    pdl_wait();
    return;
  }
  const T* row = logits + ((size_t)b * rows_per_seq + i) * V;
  const int lo = c * kChunk, hi = min(V, lo + kChunk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ float sm[kThreads / 32];
  __shared__ int si[kThreads / 32];
  __shared__ double ss[kThreads / 32];
  float lm = -INFINITY;   // the lane's maximum
  int li = INT_MAX;       // its lowest index (one-element path; the 16-byte path finds it on demand)
  double sum = 0.0;       // the lane's share of the chunk sum, relative to the warp's maximum
  constexpr int kGroups = kChunk / (kThreads * 8);
  float x[kGroups][8];
  float wm;
  if (vec) {
    // 16-byte path: the thread's 64 logits of the chunk are loaded at once and stay in registers:
    // the maximum, then the exponentials relative to the warp's maximum (paired instructions), and
    // the argmax index searched only by the lanes holding the chunk's maximum
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi) {
      const int v = lo + (gi * kThreads + threadIdx.x) * 8;
      if (v < hi) {
        load8<T>(row, v, x[gi]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[gi][e] = -INFINITY;
      }
    }
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi)
#pragma unroll
      for (int e = 0; e < 8; ++e) lm = fmaxf(lm, x[gi][e]);
    wm = warp_max(lm);
    if (wm != -INFINITY)
#pragma unroll
      for (int gi = 0; gi < kGroups; ++gi) sum += (double)sum_ex2_8(x[gi], wm, thi, tlo);
  } else {
    for (int v = lo + threadIdx.x; v < hi; v += kThreads) {
      const float xv = load1(row, v);
      if (better(xv, v, lm, li)) lm = xv, li = v;
    }
    wm = warp_max(lm);
    if (wm != -INFINITY)
      for (int v = lo + threadIdx.x; v < hi; v += kThreads) sum += (double)expo(load1(row, v), wm, thi, tlo);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) sm[warp] = wm;
  __syncthreads();
  float M = -INFINITY;
  for (int w = 0; w < kThreads / 32; ++w) M = fmaxf(M, sm[w]);
  // the lowest index holding the chunk maximum (ties -> lower index)
  int idx = INT_MAX;
  if (M != -INFINITY && lm == M) {
    if (vec) {
#pragma unroll
      for (int gi = kGroups - 1; gi >= 0; --gi) {
        const int v = lo + (gi * kThreads + threadIdx.x) * 8;
#pragma unroll
        for (int e = 7; e >= 0; --e)
          if (x[gi][e] == M) idx = v + e;
      }
    } else {
      idx = li;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) idx = min(idx, __shfl_xor_sync(0xffffffffu, idx, o));
  // each warp rescales its own sum to the chunk maximum (fp64, the warps in parallel)
  if (lane == 0) {
    si[warp] = idx;
    ss[warp] = (sum == 0.0 || wm == M) ? sum : sum * exp2(((double)wm - (double)M) * cpow);
  }
  __syncthreads();
  pdl_wait();   // the previous step's acceptance may still read the workspace
  if (threadIdx.x == 0) {
    double t = 0.0;
    int Mi = INT_MAX;
    for (int w = 0; w < kThreads / 32; ++w) t += ss[w], Mi = min(Mi, si[w]);
    RowStat r;
    r.zm = M;
    r.bi = (M == -INFINITY || Mi == INT_MAX) ? lo : Mi;
    r.s = t;
    part[((size_t)b * rows_per_seq + i) * chunks + c] = r;
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) tree_threshold_kernel(
    const T* __restrict__ logits, int V, const RowStat* __restrict__ part, int chunks, float thi, float tlo,
    double tau, const int32_t* __restrict__ tokens, const int32_t* __restrict__ parent_s,
    const int32_t* __restrict__ num_nodes, const int32_t* __restrict__ root_key, int Nmax, int Dmax,
    int32_t* __restrict__ accept_len, int32_t* __restrict__ path, int32_t* __restrict__ out_tokens,
    const int32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ double s_is[];                                            // Nmax: 1 / row sum
  int32_t* s_tstar = reinterpret_cast<int32_t*>(s_is + Nmax);                 // Nmax: row argmax
  float* s_zm = reinterpret_cast<float*>(s_tstar + Nmax);                     // Nmax: row maximum
  uint8_t* s_match = reinterpret_cast<uint8_t*>(s_zm + Nmax);                 // Nmax: edge passes
  __shared__ int32_t s_path[256];
  const int b = blockIdx.x;
  const int N = num_nodes ? num_nodes[b] : Nmax;
  const bool live = status[b] == 0 && N > 0 && N <= Nmax;
  const int32_t* ps = parent_s + (size_t)b * (Nmax + 1);
  const int32_t* tok = tokens + (size_t)b * Nmax;
  if (live) {
    // every row's merged statistics: argmax (ties -> lower index: chunks in order), max, 1 / sum
    for (int r = threadIdx.x; r < N; r += blockDim.x) {
      const RowStat* p = part + ((size_t)b * Nmax + r) * chunks;
      float M = -INFINITY;
      int Mi = INT_MAX;
      for (int c = 0; c < chunks; ++c)
        if (better(p[c].zm, p[c].bi, M, Mi)) M = p[c].zm, Mi = p[c].bi;
      double S = 0.0;
      if (M != -INFINITY)
        for (int c = 0; c < chunks; ++c)
          if (p[c].zm != -INFINITY) S += p[c].s * (double)expo(p[c].zm, M, thi, tlo);
      s_tstar[r] = Mi == INT_MAX ? 0 : Mi;
      s_zm[r] = M;
      s_is[r] = S > 0.0 ? 1.0 / S : 0.0;
    }
    __syncthreads();
    // edge decisions: p_parent(token) >= tau, in fp64 from the gathered logit
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
      const int p = ps[i + 1] - 1;
      bool m = false;
      const int x = tok[i];
      if (p >= 0 && p < i && x >= 0 && x < V && s_zm[p] != -INFINITY) {
        const float z = load1(logits + ((size_t)b * Nmax + p) * V, x);
        const double pv = (double)expo(z, s_zm[p], thi, tlo) * s_is[p];
        m = pv >= tau;
      }
      s_match[i] = m ? 1 : 0;
    }
  }
  acc::tree_accept_block(nullptr, chunks, tokens, parent_s, num_nodes, root_key, Nmax, Dmax, status, accept_len,
                         path, out_tokens, s_tstar, s_path, nullptr, nullptr, s_match, true);
}

}  // namespace

size_t accept_threshold_ws(int B, int Nmax, int V) { return (size_t)B * Nmax * num_chunks(V) * sizeof(RowStat); }

size_t accept_threshold_smem(int Nmax) { return (size_t)Nmax * (8 + 4 + 4 + 1); }

tsd_status launch_accept_threshold(const void* logits, tsd_dtype dtype, int V, const int32_t* tokens,
                                   const int32_t* parent_s, const int32_t* num_nodes, const int32_t* root_key,
                                   float tau, float T, int B, int Nmax, int Dmax, int32_t* accept_len,
                                   int32_t* path, int32_t* out_tokens, void* ws, int32_t* status,
                                   cudaStream_t stream) {
  if (B == 0) return TSD_OK;
  const int chunks = num_chunks(V);
  const double c = kLog2eD / (double)T;
  float thi, tlo;
  split_const(c, thi, tlo);
  RowStat* part = reinterpret_cast<RowStat*>(ws);
  const int vec = vec16_rows(logits, V) ? 1 : 0;
  const size_t smem = accept_threshold_smem(Nmax);
  if (dtype == TSD_BF16) {
    auto lg = reinterpret_cast<const __nv_bfloat16*>(logits);
    launch_pdl(row_stats_chunks<__nv_bfloat16>, dim3(chunks, Nmax, B), dim3(kThreads), 0, stream, lg, V, Nmax,
               num_nodes, chunks, thi, tlo, c, part, vec);
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(tree_threshold_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
    launch_pdl(tree_threshold_kernel<__nv_bfloat16>, dim3(B), dim3(kThreads), smem, stream, lg, V,
               (const RowStat*)part, chunks, thi, tlo, (double)tau, tokens, parent_s, num_nodes, root_key, Nmax,
               Dmax, accept_len, path, out_tokens, (const int32_t*)status);
  } else {
    auto lg = reinterpret_cast<const float*>(logits);
    launch_pdl(row_stats_chunks<float>, dim3(chunks, Nmax, B), dim3(kThreads), 0, stream, lg, V, Nmax, num_nodes,
               chunks, thi, tlo, c, part, vec);
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(tree_threshold_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_pdl(tree_threshold_kernel<float>, dim3(B), dim3(kThreads), smem, stream, lg, V, (const RowStat*)part,
               chunks, thi, tlo, (double)tau, tokens, parent_s, num_nodes, root_key, Nmax, Dmax, accept_len, path,
               out_tokens, (const int32_t*)status);
  }
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

}  // namespace tsd
