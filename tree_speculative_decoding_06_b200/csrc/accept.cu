// tsd_tree_accept_greedy and tsd_chain_accept_sample.
//
// Greedy: "Acelerando Sonar a traves de la especulacion", section "Decodificacion especulativa"
// (the longest accepted prefix is kept and the target supplies one more token, so n drafts give
// up to n+1 tokens) and section "EAGLE" (over a tree, the longest suitable branch continues);
// "Speculative Speculative Decoding", technical summary sec. 2 (a forest of pre-drafted outcomes
// is hit or missed by the real verify outcome).
// Sampling: section "Objetivo-Borrador" of the same Perplexity page (acceptance compares the full
// draft and target distributions, then one more target token is drawn), with the rule of the
// Leviathan et al. paper the page cites.
//
// Both scan the vocabulary, which is the HBM-bound part: the scans are split into chunks of
// kChunk tokens over many CTAs (16-byte loads), and small per-sequence kernels merge the chunk
// results.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace tsd {

namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 8192;          // vocab entries per scan CTA
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ inline int num_chunks(int V) { return (V + kChunk - 1) / kChunk; }

// Load 8 consecutive logits starting at element `v` of a row (v % 8 == 0, 16-byte aligned row).
template <typename T>
__device__ __forceinline__ void load8(const T* row, int v, float (&x)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* row, int v, float (&x)[8]) {
  const uint4 w = __ldg(reinterpret_cast<const uint4*>(row + v));
  x[0] = bf16_lo(w.x), x[1] = bf16_hi(w.x), x[2] = bf16_lo(w.y), x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z), x[5] = bf16_hi(w.z), x[6] = bf16_lo(w.w), x[7] = bf16_hi(w.w);
}
template <>
__device__ __forceinline__ void load8<float>(const float* row, int v, float (&x)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(row + v));
  const float4 c = __ldg(reinterpret_cast<const float4*>(row + v + 4));
  x[0] = a.x, x[1] = a.y, x[2] = a.z, x[3] = a.w, x[4] = c.x, x[5] = c.y, x[6] = c.z, x[7] = c.w;
}
__device__ __forceinline__ float load1(const __nv_bfloat16* row, int v) { return __bfloat162float(row[v]); }
__device__ __forceinline__ float load1(const float* row, int v) { return row[v]; }

// Block-wide argmax (value, index; NaN never wins, ties -> lower index).
__device__ __forceinline__ void block_argmax(float& bv, int& bi) {
  __shared__ float sv[kThreads / 32];
  __shared__ int si[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (better(ov, oi, bv, bi)) bv = ov, bi = oi;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sv[warp] = bv, si[warp] = bi;
  __syncthreads();
  if (warp == 0) {
    bv = lane < (int)(blockDim.x >> 5) ? sv[lane] : -INFINITY;
    bi = lane < (int)(blockDim.x >> 5) ? si[lane] : INT_MAX;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (better(ov, oi, bv, bi)) bv = ov, bi = oi;
    }
  }
}

// Argmax of one chunk of one row.  rows_per_seq rows per sequence; row i >= n_b is skipped.
template <typename T>
__global__ void __launch_bounds__(kThreads) row_argmax_chunks(const T* __restrict__ logits, int V, int rows_per_seq,
                                                              const int32_t* __restrict__ num_rows,
                                                              const int32_t* __restrict__ status, int chunks,
                                                              float2* __restrict__ part) {
  const int c = blockIdx.x, i = blockIdx.y, b = blockIdx.z;
  const int n = num_rows ? num_rows[b] : rows_per_seq;
  if (i >= n || (status && status[b] != 0)) return;
  const T* row = logits + ((size_t)b * rows_per_seq + i) * V;
  const int lo = c * kChunk, hi = min(V, lo + kChunk);
  float bv = -INFINITY;
  int bi = INT_MAX;
  if ((V & 7) == 0) {
    for (int v = lo + threadIdx.x * 8; v < hi; v += kThreads * 8) {
      float x[8];
      load8<T>(row, v, x);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (x[e] > bv) bv = x[e], bi = v + e;
    }
  } else {
    for (int v = lo + threadIdx.x; v < hi; v += kThreads) {
      const float x = load1(row, v);
      if (better(x, v, bv, bi)) bv = x, bi = v;
    }
  }
  block_argmax(bv, bi);
  if (threadIdx.x == 0) {
    if (bv == -INFINITY || bi == INT_MAX) bi = lo;   // nothing above -inf: the chunk's first index
    part[((size_t)b * rows_per_seq + i) * chunks + c] = make_float2(bv, __int_as_float(bi));
  }
}

__device__ __forceinline__ int merge_argmax(const float2* p, int chunks) {
  float bv = -INFINITY;
  int bi = INT_MAX;
  for (int c = 0; c < chunks; ++c) {
    const float v = p[c].x;
    const int i = __float_as_int(p[c].y);
    if (better(v, i, bv, bi)) bv = v, bi = i;
  }
  return bi == INT_MAX ? 0 : bi;
}

// Per-tree acceptance: t*(node), accepted set by walking each node's ancestors, deepest node.
__global__ void __launch_bounds__(kThreads) tree_accept_kernel(const float2* __restrict__ part, int chunks,
                                                               const int32_t* __restrict__ tokens,
                                                               const int32_t* __restrict__ parent_s,
                                                               const int32_t* __restrict__ num_nodes,
                                                               const int32_t* __restrict__ root_key, int Nmax,
                                                               int Dmax, int32_t* __restrict__ accept_len,
                                                               int32_t* __restrict__ path,
                                                               int32_t* __restrict__ out_tokens,
                                                               const int32_t* __restrict__ status) {
  extern __shared__ int32_t s_tstar[];
  __shared__ int s_hit, s_best;
  const int b = blockIdx.x;
  const int N = num_nodes ? num_nodes[b] : Nmax;
  const int32_t* tok = tokens + (size_t)b * Nmax;
  const int32_t* ps = parent_s + (size_t)b * (Nmax + 1);
  int32_t* prow = path + (size_t)b * (Dmax + 1);
  int32_t* orow = out_tokens + (size_t)b * (Dmax + 1);
  const bool live = status[b] == 0 && N > 0 && N <= Nmax;
  if (threadIdx.x == 0) s_hit = INT_MAX, s_best = -1;
  for (int i = threadIdx.x; live && i < N; i += blockDim.x)
    s_tstar[i] = merge_argmax(part + ((size_t)b * Nmax + i) * chunks, chunks);
  __syncthreads();
  if (live && root_key) {
    const int key = root_key[b];
    for (int i = threadIdx.x; i < N; i += blockDim.x)
      if (ps[i + 1] == 0 && tok[i] == key) atomicMin(&s_hit, i);
  }
  __syncthreads();
  for (int i = threadIdx.x; live && i < N; i += blockDim.x) {
    // accepted iff every edge on the root->i path matches and the root is accepted
    bool ok = true;
    int s = i + 1, d = 0;
    for (;;) {
      const int p = ps[s];
      if (p == 0) {
        if (root_key) ok = ok && (s - 1 == s_hit);
        break;
      }
      if (p >= s || d >= Dmax) {   // prepare guarantees neither; stay bounded anyway
        ok = false;
        break;
      }
      ok = ok && (tok[s - 1] == s_tstar[p - 1]);
      s = p;
      ++d;
      if (!ok) break;
    }
    if (ok) atomicMax(&s_best, (d << 20) | (0xFFFFF - i));
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  const int best = live ? s_best : -1;
  if (best < 0) {
    accept_len[b] = -1;
    for (int k = 0; k <= Dmax; ++k) prow[k] = 0, orow[k] = -1;
    return;
  }
  const int A = best >> 20, astar = 0xFFFFF - (best & 0xFFFFF);
  accept_len[b] = A;
  int s = astar + 1;
  for (int k = A; k >= 0; --k) {
    prow[k] = s;
    s = ps[s];
  }
  for (int k = A + 1; k <= Dmax; ++k) prow[k] = 0, orow[k] = -1;
  for (int k = 0; k < A; ++k) orow[k] = tok[prow[k + 1] - 1];
  orow[A] = s_tstar[astar];
}

// ---------------------------------------------------------------------------------------------
// Chain rejection sampling.  Row r of sequence b: r <= K target row r, r > K draft row r-K-1.
// Softmax statistics in the log2 domain: y = z * log2(e) / T, m = max y, s = sum 2^(y - m).
// ---------------------------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ const T* chain_row(const T* zp, const T* zq, int K, int V, int b, int r) {
  return r <= K ? zp + ((size_t)b * (K + 1) + r) * V : zq + ((size_t)b * K + (r - K - 1)) * V;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) chain_stats_kernel(const T* __restrict__ zp, const T* __restrict__ zq,
                                                               int V, int K, float c2, int chunks,
                                                               float2* __restrict__ part) {
  const int c = blockIdx.x, r = blockIdx.y, b = blockIdx.z;
  const T* row = chain_row(zp, zq, K, V, b, r);
  const int lo = c * kChunk, hi = min(V, lo + kChunk);
  float m = -INFINITY, s = 0.f;
  auto add = [&](float y) {
    if (y > m) {
      s = s * exp2f(m - y) + 1.f;
      m = y;
    } else if (m != -INFINITY) {
      s += exp2f(y - m);
    }
  };
  if ((V & 7) == 0) {
    for (int v = lo + threadIdx.x * 8; v < hi; v += kThreads * 8) {
      float x[8];
      load8<T>(row, v, x);
      float lm = x[0] * c2;
#pragma unroll
      for (int e = 1; e < 8; ++e) lm = fmaxf(lm, x[e] * c2);
      if (lm > m) {
        s *= exp2f(m - lm);
        m = lm;
      }
      if (m != -INFINITY) {
#pragma unroll
        for (int e = 0; e < 8; ++e) s += exp2f(x[e] * c2 - m);
      }
    }
  } else {
    for (int v = lo + threadIdx.x; v < hi; v += kThreads) add(load1(row, v) * c2);
  }
  // block merge of (m, s)
  __shared__ float sm[kThreads / 32], ss[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m, o), os = __shfl_xor_sync(0xffffffffu, s, o);
    const float nm = fmaxf(m, om);
    const float u = nm == -INFINITY ? 0.f : nm;
    s = s * exp2f(m - u) + os * exp2f(om - u);
    m = nm;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sm[warp] = m, ss[warp] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float M = -INFINITY, S = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) {
      const float nm = fmaxf(M, sm[w]);
      const float u = nm == -INFINITY ? 0.f : nm;
      S = S * exp2f(M - u) + ss[w] * exp2f(sm[w] - u);
      M = nm;
    }
    part[((size_t)b * (2 * K + 1) + r) * chunks + c] = make_float2(M, S);
  }
}

__device__ __forceinline__ float2 merge_stats(const float2* p, int chunks) {
  float M = -INFINITY, S = 0.f;
  for (int c = 0; c < chunks; ++c) {
    const float nm = fmaxf(M, p[c].x);
    const float u = nm == -INFINITY ? 0.f : nm;
    S = S * exp2f(M - u) + p[c].y * exp2f(p[c].x - u);
    M = nm;
  }
  return make_float2(M, S);
}

// Accept tests of one sequence, run by one warp: lanes merge the chunk statistics of the 2K+1
// rows and fetch the logits at the draft tokens in parallel, then lane 0 takes the K decisions
// in order.  Returns the first rejected position, or K when every draft is accepted.
template <typename T>
__device__ int chain_decide_warp(const T* zp, const T* zq, const int32_t* x, const float* u, const float2* part,
                                 int chunks, int V, int K, float c2, int b, float2* st, float* yx) {
  const int lane = threadIdx.x & 31;
  for (int r = lane; r < 2 * K + 1; r += 32) st[r] = merge_stats(part + ((size_t)b * (2 * K + 1) + r) * chunks, chunks);
  for (int k = lane; k < K; k += 32) {
    const int xk = x[(size_t)b * K + k];
    const bool in = xk >= 0 && xk < V;
    yx[2 * k] = in ? load1(chain_row(zp, zq, K, V, b, k), xk) * c2 : -INFINITY;
    yx[2 * k + 1] = in ? load1(chain_row(zp, zq, K, V, b, K + 1 + k), xk) * c2 : 0.f;
  }
  __syncwarp();
  int j = K;
  if (lane == 0) {
    for (int k = 0; k < K; ++k) {
      const float p = exp2f(yx[2 * k] - st[k].x) / st[k].y;               // an out-of-range draft has p = 0
      const float q = exp2f(yx[2 * k + 1] - st[K + 1 + k].x) / st[K + 1 + k].y;
      if (!(u[(size_t)b * (K + 1) + k] * q < p)) {
        j = k;
        break;
      }
    }
  }
  return __shfl_sync(0xffffffffu, j, 0);
}

// Mass of the final distribution at v: residual max(p_j - q_j, 0) after a rejection (or p_j
// when `plain`), p_K when everything was accepted.
template <typename T>
__device__ __forceinline__ float final_mass(const T* prow, const T* qrow, int v, float c2, float2 sp, float2 sq,
                                            bool residual) {
  const float p = exp2f(load1(prow, v) * c2 - sp.x) / sp.y;
  if (!residual) return p;
  const float q = exp2f(load1(qrow, v) * c2 - sq.x) / sq.y;
  return fmaxf(p - q, 0.f);
}

// Decide, then sum the final distribution over this CTA's chunk.
template <typename T>
__global__ void __launch_bounds__(kThreads) chain_mass_kernel(const T* __restrict__ zp, const T* __restrict__ zq,
                                                              const int32_t* __restrict__ x,
                                                              const float* __restrict__ u, int V, int K, float c2,
                                                              int chunks, const float2* __restrict__ part,
                                                              float* __restrict__ mass, int* __restrict__ jout) {
  extern __shared__ float2 s_st[];   // 2K+1 statistics, then 2K floats of logits at the drafts
  __shared__ int s_j;
  const int c = blockIdx.x, b = blockIdx.y;
  if (threadIdx.x < 32) {
    const int jj = chain_decide_warp(zp, zq, x, u, part, chunks, V, K, c2, b, s_st,
                                     reinterpret_cast<float*>(s_st + 2 * K + 1));
    if (threadIdx.x == 0) {
      s_j = jj;
      if (c == 0) jout[b] = jj;
    }
  }
  __syncthreads();
  const int j = s_j;
  const bool residual = j < K;
  const T* prow = chain_row(zp, zq, K, V, b, j);
  const T* qrow = residual ? chain_row(zp, zq, K, V, b, K + 1 + j) : prow;
  const float2 sp = s_st[j], sq = residual ? s_st[K + 1 + j] : s_st[j];
  const int lo = c * kChunk, hi = min(V, lo + kChunk);
  float acc = 0.f;
  for (int v = lo + threadIdx.x; v < hi; v += kThreads) acc += final_mass(prow, qrow, v, c2, sp, sq, residual);
  acc = warp_sum(acc);
  __shared__ float sw[kThreads / 32];
  if ((threadIdx.x & 31) == 0) sw[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) t += sw[w];
    mass[(size_t)b * chunks + c] = t;
  }
}

// Inverse CDF inside one CTA: the smallest v in [lo, hi) whose cumulative mass exceeds thr
// (cumulative counted from lo); each thread owns a contiguous run.  Returns -1 if not reached.
template <typename T>
__device__ int cta_inverse_cdf(const T* prow, const T* qrow, int lo, int hi, float thr, float c2, float2 sp,
                               float2 sq, bool residual, int* last_pos) {
  __shared__ float s_run[kThreads];
  __shared__ int s_tok, s_last;
  const int n = hi - lo, per = (n + kThreads - 1) / kThreads;
  const int a = lo + threadIdx.x * per, e = min(hi, a + per);
  float sum = 0.f;
  int lastp = -1;
  for (int v = a; v < e; ++v) {
    const float r = final_mass(prow, qrow, v, c2, sp, sq, residual);
    if (r > 0.f) lastp = v;
    sum += r;
  }
  s_run[threadIdx.x] = sum;
  if (threadIdx.x == 0) s_tok = INT_MAX, s_last = -1;
  __syncthreads();
  if (lastp >= 0) atomicMax(&s_last, lastp);
  if (threadIdx.x == 0) {   // sequential exclusive prefix over the thread runs
    float c = 0.f;
    for (int t = 0; t < kThreads; ++t) {
      const float nx = c + s_run[t];
      s_run[t] = c;
      c = nx;
    }
  }
  __syncthreads();
  float cum = s_run[threadIdx.x];
  if (cum <= thr && a < e) {
    for (int v = a; v < e; ++v) {
      cum += final_mass(prow, qrow, v, c2, sp, sq, residual);
      if (cum > thr) {
        atomicMin(&s_tok, v);
        break;
      }
    }
  }
  __syncthreads();
  *last_pos = s_last;
  return s_tok == INT_MAX ? -1 : s_tok;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) chain_select_kernel(const T* __restrict__ zp, const T* __restrict__ zq,
                                                                const int32_t* __restrict__ x,
                                                                const float* __restrict__ u, int V, int K, float c2,
                                                                int chunks, const float2* __restrict__ part,
                                                                const float* __restrict__ mass,
                                                                const int* __restrict__ jin,
                                                                int32_t* __restrict__ accept_len,
                                                                int32_t* __restrict__ out_tokens) {
  __shared__ float2 s_sp, s_sq;
  __shared__ int s_c;
  __shared__ float s_thr;
  const int b = blockIdx.x;
  const int j = jin[b];
  const bool residual = j < K;
  if (threadIdx.x == 0) {
    s_sp = merge_stats(part + ((size_t)b * (2 * K + 1) + j) * chunks, chunks);
    s_sq = residual ? merge_stats(part + ((size_t)b * (2 * K + 1) + K + 1 + j) * chunks, chunks) : s_sp;
    float R = 0.f;
    for (int c = 0; c < chunks; ++c) R += mass[(size_t)b * chunks + c];
    const float thr = u[(size_t)b * (K + 1) + K] * R;
    int cstar = -1;
    float cum = 0.f;
    for (int c = 0; c < chunks; ++c) {
      const float m = mass[(size_t)b * chunks + c];
      if (m > 0.f && cum + m > thr) {
        cstar = c;
        break;
      }
      cum += m;
    }
    if (R <= 0.f) cstar = -2;            // degenerate residual: draw from p_j over the whole row
    s_c = cstar;
    s_thr = cstar >= 0 ? fmaxf(thr - cum, 0.f) : thr;
  }
  __syncthreads();
  const T* prow = chain_row(zp, zq, K, V, b, j);
  const T* qrow = residual ? chain_row(zp, zq, K, V, b, K + 1 + j) : prow;
  int tok, lastp;
  if (s_c >= 0) {
    const int lo = s_c * kChunk, hi = min(V, lo + kChunk);
    tok = cta_inverse_cdf(prow, qrow, lo, hi, s_thr, c2, s_sp, s_sq, residual, &lastp);
  } else if (s_c == -2) {
    // total residual mass 0: sample p_j itself (threshold u * sum p over the whole row)
    __shared__ float s_tot;
    float acc = 0.f;
    for (int v = threadIdx.x; v < V; v += kThreads) acc += final_mass(prow, qrow, v, c2, s_sp, s_sq, false);
    acc = warp_sum(acc);
    __shared__ float sw[kThreads / 32];
    if ((threadIdx.x & 31) == 0) sw[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = 0.f;
      for (int w = 0; w < kThreads / 32; ++w) t += sw[w];
      s_tot = t * u[(size_t)b * (K + 1) + K];
    }
    __syncthreads();
    tok = cta_inverse_cdf(prow, prow, 0, V, s_tot, c2, s_sp, s_sp, false, &lastp);
  } else {
    // threshold at or past the rounded total: the last token with mass
    int clast = chunks - 1;
    while (clast > 0 && mass[(size_t)b * chunks + clast] <= 0.f) --clast;
    const int lo = clast * kChunk, hi = min(V, lo + kChunk);
    tok = cta_inverse_cdf(prow, qrow, lo, hi, INFINITY, c2, s_sp, s_sq, residual, &lastp);
  }
  if (threadIdx.x != 0) return;
  if (tok < 0) tok = lastp >= 0 ? lastp : 0;
  accept_len[b] = j;
  int32_t* orow = out_tokens + (size_t)b * (K + 1);
  for (int k = 0; k < j; ++k) orow[k] = x[(size_t)b * K + k];
  orow[j] = tok;
  for (int k = j + 1; k <= K; ++k) orow[k] = -1;
}

// Greedy chain (T == 0): accept while the draft equals the target argmax.
__global__ void chain_greedy_decide(const float2* __restrict__ part, int chunks, const int32_t* __restrict__ x,
                                    int B, int K, int32_t* __restrict__ accept_len,
                                    int32_t* __restrict__ out_tokens) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  int j = K;
  for (int k = 0; k < K; ++k)
    if (x[(size_t)b * K + k] != merge_argmax(part + ((size_t)b * (K + 1) + k) * chunks, chunks)) {
      j = k;
      break;
    }
  accept_len[b] = j;
  int32_t* orow = out_tokens + (size_t)b * (K + 1);
  for (int k = 0; k < j; ++k) orow[k] = x[(size_t)b * K + k];
  orow[j] = merge_argmax(part + ((size_t)b * (K + 1) + j) * chunks, chunks);
  for (int k = j + 1; k <= K; ++k) orow[k] = -1;
}

}  // namespace

size_t accept_greedy_ws(int B, int Nmax, int V) {
  return (size_t)B * Nmax * num_chunks(V) * sizeof(float2);
}

tsd_status launch_accept_greedy(const void* logits, tsd_dtype dtype, int V, const int32_t* tokens,
                                const int32_t* parent_s, const int32_t* num_nodes, const int32_t* root_key, int B,
                                int Nmax, int Dmax, int32_t* accept_len, int32_t* path, int32_t* out_tokens,
                                void* ws, int32_t* status, cudaStream_t stream) {
  if (B == 0) return TSD_OK;
  const int chunks = num_chunks(V);
  float2* part = reinterpret_cast<float2*>(ws);
  if (Nmax > 0) {
    dim3 grid(chunks, Nmax, B);
    if (dtype == TSD_BF16)
      row_argmax_chunks<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(
          reinterpret_cast<const __nv_bfloat16*>(logits), V, Nmax, num_nodes, status, chunks, part);
    else
      row_argmax_chunks<float><<<grid, kThreads, 0, stream>>>(reinterpret_cast<const float*>(logits), V, Nmax,
                                                              num_nodes, status, chunks, part);
    if (cudaGetLastError() != cudaSuccess) return TSD_ERR_CUDA;
  }
  const size_t smem = (size_t)(Nmax > 0 ? Nmax : 1) * sizeof(int32_t);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(tree_accept_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  tree_accept_kernel<<<B, kThreads, smem, stream>>>(part, chunks, tokens, parent_s, num_nodes, root_key, Nmax, Dmax,
                                                    accept_len, path, out_tokens, status);
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

size_t chain_sample_ws(int B, int K, int V) {
  const int chunks = num_chunks(V);
  size_t stats = (size_t)B * (2 * K + 1) * chunks * sizeof(float2);
  size_t mass = (size_t)B * chunks * sizeof(float);
  size_t j = (size_t)B * sizeof(int);
  return stats + mass + j + 64;
}

tsd_status launch_chain_sample(const void* zp, const void* zq, tsd_dtype dtype, int V, const int32_t* x,
                               const float* u, float T, int B, int K, int32_t* accept_len, int32_t* out_tokens,
                               void* ws, cudaStream_t stream) {
  if (B == 0) return TSD_OK;
  const int chunks = num_chunks(V);
  float2* part = reinterpret_cast<float2*>(ws);
  if (T == 0.f) {
    dim3 grid(chunks, K + 1, B);
    if (dtype == TSD_BF16)
      row_argmax_chunks<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(
          reinterpret_cast<const __nv_bfloat16*>(zp), V, K + 1, nullptr, nullptr, chunks, part);
    else
      row_argmax_chunks<float><<<grid, kThreads, 0, stream>>>(reinterpret_cast<const float*>(zp), V, K + 1,
                                                              nullptr, nullptr, chunks, part);
    chain_greedy_decide<<<(B + 127) / 128, 128, 0, stream>>>(part, chunks, x, B, K, accept_len, out_tokens);
    return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
  }
  float* mass = reinterpret_cast<float*>(part + (size_t)B * (2 * K + 1) * chunks);
  int* jbuf = reinterpret_cast<int*>(mass + (size_t)B * chunks);
  const float c2 = kLog2e / T;
  const size_t st_smem = (size_t)(2 * K + 1) * sizeof(float2) + (size_t)2 * K * sizeof(float) + 16;
  dim3 g1(chunks, 2 * K + 1, B), g2(chunks, B);
  if (dtype == TSD_BF16) {
    auto p = reinterpret_cast<const __nv_bfloat16*>(zp);
    auto q = reinterpret_cast<const __nv_bfloat16*>(zq);
    chain_stats_kernel<__nv_bfloat16><<<g1, kThreads, 0, stream>>>(p, q, V, K, c2, chunks, part);
    chain_mass_kernel<__nv_bfloat16><<<g2, kThreads, st_smem, stream>>>(p, q, x, u, V, K, c2, chunks, part, mass,
                                                                        jbuf);
    chain_select_kernel<__nv_bfloat16><<<B, kThreads, 0, stream>>>(p, q, x, u, V, K, c2, chunks, part, mass, jbuf,
                                                                   accept_len, out_tokens);
  } else {
    auto p = reinterpret_cast<const float*>(zp);
    auto q = reinterpret_cast<const float*>(zq);
    chain_stats_kernel<float><<<g1, kThreads, 0, stream>>>(p, q, V, K, c2, chunks, part);
    chain_mass_kernel<float><<<g2, kThreads, st_smem, stream>>>(p, q, x, u, V, K, c2, chunks, part, mass, jbuf);
    chain_select_kernel<float><<<B, kThreads, 0, stream>>>(p, q, x, u, V, K, c2, chunks, part, mass, jbuf,
                                                           accept_len, out_tokens);
  }
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

}  // namespace tsd
