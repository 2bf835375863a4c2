// tsd_chain_accept_sample with temperature > 0: rejection sampling of a linear draft.
//
// "Acelerando Sonar a traves de la especulacion" (Perplexity), section "Objetivo-Borrador": the
// verifier compares the complete draft and target distributions to decide how much of the draft
// to keep, then samples the target's logits after the accepted run for one more token.  The rule
// is that of the Leviathan et al. paper the page cites: accept x with probability min(1, p/q);
// after a rejection draw from max(p - q, 0) renormalised; with every draft accepted draw the bonus
// token from the next target distribution.
//
// Precision.  The accept decisions and the inverse-CDF draw are integer outcomes of real
// arithmetic; with a 128k vocabulary each token holds ~1e-5 of the mass, so the draw is sensitive
// to errors far below fp32's own rounding of a long sum.  Hence: exponent arguments
// (z - zmax) * log2(e) / T are formed with a two-term constant and rounded once; every sum, the
// normalisers, the acceptance products and the inverse-CDF scan run in fp64; only the
// exponentials themselves are fp32 (relative error ~1e-7, independent per token).
//
// Kernels: (1) per-chunk softmax statistics (row max, fp64 sum of exponentials) of all 2K+1 rows
// over many CTAs; (2) per-chunk mass of the final distribution, after a warp of each CTA has
// merged the statistics and taken the K accept tests; (3) one CTA per sequence locates the chunk
// holding the threshold and scans it.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace tsd {

namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 8192;
constexpr double kLog2eD = 1.4426950408889634074;

struct __align__(16) Stat {
  float zm;   // raw logit maximum of the chunk / row
  float pad;
  double s;   // sum of 2^((z - zm) * c), c = log2(e) / T
};

struct Temp {    // c = log2(e) / T as an unevaluated sum hi + lo, and in fp64
  float hi, lo;
  double c;
};

__host__ __device__ inline int num_chunks(int V) { return (V + kChunk - 1) / kChunk; }

__device__ __forceinline__ float expo(float z, float zm, const Temp& t) {
  const float dz = z - zm;                       // exact: both are bf16 / fp32 logits of one row
  return exp2f(fmaf(dz, t.hi, dz * t.lo));       // argument rounded once
}

template <typename T>
__device__ __forceinline__ const T* chain_row(const T* zp, const T* zq, int K, int V, int b, int r) {
  return r <= K ? zp + ((size_t)b * (K + 1) + r) * V : zq + ((size_t)b * K + (r - K - 1)) * V;
}

// Merge (zm_b, s_b) into (zm_a, s_a).
__device__ __forceinline__ void merge(float& zm, double& s, float zm2, double s2, double c) {
  if (zm2 == -INFINITY) return;
  if (zm == -INFINITY) {
    zm = zm2, s = s2;
    return;
  }
  if (zm2 > zm) {
    s = s * exp2((double)(zm - zm2) * c) + s2;
    zm = zm2;
  } else {
    s += s2 * exp2((double)(zm2 - zm) * c);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) stats_kernel(const T* __restrict__ zp, const T* __restrict__ zq, int V,
                                                         int K, Temp tc, int chunks, Stat* __restrict__ part,
                                                         int vec) {
  pdl_trigger();   // the scan reads inputs only; pdl_wait() comes before the partial is written
  const int c = blockIdx.x, r = blockIdx.y, b = blockIdx.z;
  const T* row = chain_row(zp, zq, K, V, b, r);
  const int lo = c * kChunk, hi = min(V, lo + kChunk);
  float zm = -INFINITY;
  double s = 0.0;
  if (vec) {
    for (int v = lo + threadIdx.x * 8; v < hi; v += kThreads * 8) {
      float x[8];
      load8<T>(row, v, x);
      float lm = x[0];
#pragma unroll
      for (int e = 1; e < 8; ++e) lm = fmaxf(lm, x[e]);
      if (lm > zm) {
        s = zm == -INFINITY ? 0.0 : s * exp2((double)(zm - lm) * tc.c);
        zm = lm;
      }
      if (zm != -INFINITY) {
        float t = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) t += expo(x[e], zm, tc);
        s += (double)t;
      }
    }
  } else {
    for (int v = lo + threadIdx.x; v < hi; v += kThreads) {
      const float x = load1(row, v);
      if (x > zm) {
        s = zm == -INFINITY ? 0.0 : s * exp2((double)(zm - x) * tc.c);
        zm = x;
      }
      if (zm != -INFINITY) s += (double)expo(x, zm, tc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float zm2 = __shfl_xor_sync(0xffffffffu, zm, o);
    const double s2 = __shfl_xor_sync(0xffffffffu, s, o);
    merge(zm, s, zm2, s2, tc.c);
  }
  __shared__ float szm[kThreads / 32];
  __shared__ double ss[kThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) szm[warp] = zm, ss[warp] = s;
  __syncthreads();
  pdl_wait();
  if (threadIdx.x == 0) {
    float M = -INFINITY;
    double S = 0.0;
    for (int w = 0; w < kThreads / 32; ++w) merge(M, S, szm[w], ss[w], tc.c);
    Stat st;
    st.zm = M, st.pad = 0.f, st.s = S;
    part[((size_t)b * (2 * K + 1) + r) * chunks + c] = st;
  }
}

__device__ __forceinline__ Stat merge_stats(const Stat* p, int chunks, double c) {
  float M = -INFINITY;
  double S = 0.0;
  for (int i = 0; i < chunks; ++i) merge(M, S, p[i].zm, p[i].s, c);
  Stat st;
  st.zm = M, st.pad = 0.f, st.s = S;
  return st;
}

// One warp: lanes merge the 2K+1 statistics and evaluate the drafts' exponentials in parallel,
// then lane 0 runs the K accept tests in order: accept iff u * q(x) < p(x), i.e.
// u * eq * s_p < ep * s_q in fp64.  Returns the first rejected position (K if none).
template <typename T>
__device__ int decide_warp(const T* zp, const T* zq, const int32_t* x, const float* u, const Stat* part, int chunks,
                           int V, int K, const Temp& tc, int b, Stat* st, float* ex) {
  const int lane = threadIdx.x & 31;
  for (int r = lane; r < 2 * K + 1; r += 32)
    st[r] = merge_stats(part + ((size_t)b * (2 * K + 1) + r) * chunks, chunks, tc.c);
  __syncwarp();
  for (int k = lane; k < K; k += 32) {
    const int xk = x[(size_t)b * K + k];
    const bool in = xk >= 0 && xk < V;
    ex[2 * k] = in ? expo(load1(chain_row(zp, zq, K, V, b, k), xk), st[k].zm, tc) : 0.f;
    ex[2 * k + 1] = in ? expo(load1(chain_row(zp, zq, K, V, b, K + 1 + k), xk), st[K + 1 + k].zm, tc) : 1.f;
  }
  __syncwarp();
  int j = K;
  if (lane == 0) {
    for (int k = 0; k < K; ++k) {
      const double lhs = (double)u[(size_t)b * (K + 1) + k] * (double)ex[2 * k + 1] * st[k].s;
      const double rhs = (double)ex[2 * k] * st[K + 1 + k].s;
      if (!(lhs < rhs)) {
        j = k;
        break;
      }
    }
  }
  return __shfl_sync(0xffffffffu, j, 0);
}

// Mass of the final distribution at token v: max(p_j - q_j, 0) after a rejection, p otherwise.
struct Final {
  float zmp, zmq;
  double ip, iq;   // 1 / s
  bool residual;
};

template <typename T>
__device__ __forceinline__ double final_mass(const T* prow, const T* qrow, int v, const Final& f, const Temp& tc) {
  const double p = (double)expo(load1(prow, v), f.zmp, tc) * f.ip;
  if (!f.residual) return p;
  const double q = (double)expo(load1(qrow, v), f.zmq, tc) * f.iq;
  return p > q ? p - q : 0.0;
}

__device__ __forceinline__ double block_sum_d(double v) {
  __shared__ double sw[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) sw[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < kThreads / 32; ++w) t += sw[w];
  __syncthreads();
  return t;   // valid in thread 0
}

template <typename T>
__global__ void __launch_bounds__(kThreads) mass_kernel(const T* __restrict__ zp, const T* __restrict__ zq,
                                                        const int32_t* __restrict__ x, const float* __restrict__ u,
                                                        int V, int K, Temp tc, int chunks,
                                                        const Stat* __restrict__ part, double* __restrict__ mass,
                                                        int* __restrict__ jout) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ Stat s_st[];     // 2K+1 statistics, then 2K floats of draft exponentials
  __shared__ int s_j;
  const int c = blockIdx.x, b = blockIdx.y;
  if (threadIdx.x < 32) {
    const int j = decide_warp(zp, zq, x, u, part, chunks, V, K, tc, b, s_st, reinterpret_cast<float*>(s_st + 2 * K + 1));
    if (threadIdx.x == 0) {
      s_j = j;
      if (c == 0) jout[b] = j;
    }
  }
  __syncthreads();
  const int j = s_j;
  Final f;
  f.residual = j < K;
  f.zmp = s_st[j].zm, f.ip = 1.0 / s_st[j].s;
  f.zmq = f.residual ? s_st[K + 1 + j].zm : 0.f;
  f.iq = f.residual ? 1.0 / s_st[K + 1 + j].s : 0.0;
  const T* prow = chain_row(zp, zq, K, V, b, j);
  const T* qrow = f.residual ? chain_row(zp, zq, K, V, b, K + 1 + j) : prow;
  const int lo = c * kChunk, hi = min(V, lo + kChunk);
  double acc = 0.0;
  for (int v = lo + threadIdx.x; v < hi; v += kThreads) acc += final_mass(prow, qrow, v, f, tc);
  const double t = block_sum_d(acc);
  if (threadIdx.x == 0) mass[(size_t)b * chunks + c] = t;
}

// Inverse CDF inside one CTA over [lo, hi): the smallest v whose cumulative mass (counted from lo)
// exceeds thr.  Each thread owns a contiguous run; run sums are prefixed in order by one thread.
// Returns -1 when the threshold is not reached; *last_pos = last token with mass in the range.
template <typename T>
__device__ int cta_inverse_cdf(const T* prow, const T* qrow, int lo, int hi, double thr, const Final& f,
                               const Temp& tc, int* last_pos) {
  __shared__ double s_run[kThreads];
  __shared__ int s_tok, s_last;
  const int n = hi - lo, per = (n + kThreads - 1) / kThreads;
  const int a = lo + threadIdx.x * per, e = min(hi, a + per);
  double sum = 0.0;
  int lastp = -1;
  for (int v = a; v < e; ++v) {
    const double r = final_mass(prow, qrow, v, f, tc);
    if (r > 0.0) lastp = v;
    sum += r;
  }
  s_run[threadIdx.x] = sum;
  if (threadIdx.x == 0) s_tok = INT_MAX, s_last = -1;
  __syncthreads();
  if (lastp >= 0) atomicMax(&s_last, lastp);
  if (threadIdx.x == 0) {
    double c = 0.0;
    for (int t = 0; t < kThreads; ++t) {
      const double nx = c + s_run[t];
      s_run[t] = c;
      c = nx;
    }
  }
  __syncthreads();
  double cum = s_run[threadIdx.x];
  if (cum <= thr && a < e) {
    for (int v = a; v < e; ++v) {
      cum += final_mass(prow, qrow, v, f, tc);
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
__global__ void __launch_bounds__(kThreads) select_kernel(const T* __restrict__ zp, const T* __restrict__ zq,
                                                          const int32_t* __restrict__ x, const float* __restrict__ u,
                                                          int V, int K, Temp tc, int chunks,
                                                          const Stat* __restrict__ part,
                                                          const double* __restrict__ mass,
                                                          const int* __restrict__ jin,
                                                          int32_t* __restrict__ accept_len,
                                                          int32_t* __restrict__ out_tokens) {
  pdl_trigger();
  pdl_wait();
  __shared__ Final s_f;
  __shared__ int s_c;
  __shared__ double s_thr;
  const int b = blockIdx.x;
  const int j = jin[b];
  if (threadIdx.x == 0) {
    Final f;
    f.residual = j < K;
    const Stat sp = merge_stats(part + ((size_t)b * (2 * K + 1) + j) * chunks, chunks, tc.c);
    f.zmp = sp.zm, f.ip = 1.0 / sp.s;
    if (f.residual) {
      const Stat sq = merge_stats(part + ((size_t)b * (2 * K + 1) + K + 1 + j) * chunks, chunks, tc.c);
      f.zmq = sq.zm, f.iq = 1.0 / sq.s;
    } else {
      f.zmq = 0.f, f.iq = 0.0;
    }
    double R = 0.0;
    for (int c = 0; c < chunks; ++c) R += mass[(size_t)b * chunks + c];
    const double thr = (double)u[(size_t)b * (K + 1) + K] * R;
    int cstar = -1;
    double cum = 0.0;
    for (int c = 0; c < chunks; ++c) {
      const double m = mass[(size_t)b * chunks + c];
      if (m > 0.0 && cum + m > thr) {
        cstar = c;
        break;
      }
      cum += m;
    }
    if (!(R > 0.0)) cstar = -2;          // residual with no mass: draw from p_j over the whole row
    if (cstar == -1) {                   // threshold at the rounded total: the last chunk with mass
      cstar = chunks - 1;
      while (cstar > 0 && !(mass[(size_t)b * chunks + cstar] > 0.0)) --cstar;
      cum = 1e300;
    }
    s_f = f;
    s_c = cstar;
    s_thr = cstar >= 0 ? (cum >= 1e299 ? 1e300 : thr - cum) : 0.0;
  }
  __syncthreads();
  Final f = s_f;
  const T* prow = chain_row(zp, zq, K, V, b, j);
  const T* qrow = f.residual ? chain_row(zp, zq, K, V, b, K + 1 + j) : prow;
  int tok, lastp;
  if (s_c >= 0) {
    const int lo = s_c * kChunk, hi = min(V, lo + kChunk);
    tok = cta_inverse_cdf(prow, qrow, lo, hi, s_thr, f, tc, &lastp);
  } else {
    f.residual = false;
    double acc = 0.0;
    for (int v = threadIdx.x; v < V; v += kThreads) acc += final_mass(prow, prow, v, f, tc);
    const double t = block_sum_d(acc);
    if (threadIdx.x == 0) s_thr = t * (double)u[(size_t)b * (K + 1) + K];
    __syncthreads();
    tok = cta_inverse_cdf(prow, prow, 0, V, s_thr, f, tc, &lastp);
  }
  if (threadIdx.x != 0) return;
  if (tok < 0) tok = lastp >= 0 ? lastp : 0;
  accept_len[b] = j;
  int32_t* orow = out_tokens + (size_t)b * (K + 1);
  for (int k = 0; k < j; ++k) orow[k] = x[(size_t)b * K + k];
  orow[j] = tok;
  for (int k = j + 1; k <= K; ++k) orow[k] = -1;
}

}  // namespace

size_t chain_sample_ws(int B, int K, int V) {
  const int chunks = num_chunks(V);
  const size_t stats = (size_t)B * (2 * K + 1) * chunks * sizeof(Stat);
  const size_t mass = (size_t)B * chunks * sizeof(double);
  return stats + mass + (size_t)B * sizeof(int) + 64;
}

tsd_status launch_chain_sample_stochastic(const void* zp, const void* zq, tsd_dtype dtype, int V, const int32_t* x,
                                          const float* u, float T, int B, int K, int32_t* accept_len,
                                          int32_t* out_tokens, void* ws, cudaStream_t stream) {
  const int chunks = num_chunks(V);
  Stat* part = reinterpret_cast<Stat*>(ws);
  double* mass = reinterpret_cast<double*>(part + (size_t)B * (2 * K + 1) * chunks);
  int* jbuf = reinterpret_cast<int*>(mass + (size_t)B * chunks);
  Temp tc;
  tc.c = kLog2eD / (double)T;
  tc.hi = (float)tc.c;
  tc.lo = (float)(tc.c - (double)tc.hi);
  const size_t st_smem = (size_t)(2 * K + 1) * sizeof(Stat) + (size_t)2 * K * sizeof(float) + 16;
  dim3 g1(chunks, 2 * K + 1, B), g2(chunks, B);
  const int vec = vec16_rows(zp, V) && (K == 0 || vec16_rows(zq, V)) ? 1 : 0;
  if (dtype == TSD_BF16) {
    auto p = reinterpret_cast<const __nv_bfloat16*>(zp);
    auto q = reinterpret_cast<const __nv_bfloat16*>(zq);
    launch_pdl(stats_kernel<__nv_bfloat16>, g1, dim3(kThreads), 0, stream, p, q, V, K, tc, chunks, part, vec);
    launch_pdl(mass_kernel<__nv_bfloat16>, g2, dim3(kThreads), st_smem, stream, p, q, x, u, V, K, tc, chunks,
               (const Stat*)part, mass, jbuf);
    launch_pdl(select_kernel<__nv_bfloat16>, dim3(B), dim3(kThreads), 0, stream, p, q, x, u, V, K, tc, chunks,
               (const Stat*)part, (const double*)mass, (const int*)jbuf, accept_len, out_tokens);
  } else {
    auto p = reinterpret_cast<const float*>(zp);
    auto q = reinterpret_cast<const float*>(zq);
    launch_pdl(stats_kernel<float>, g1, dim3(kThreads), 0, stream, p, q, V, K, tc, chunks, part, vec);
    launch_pdl(mass_kernel<float>, g2, dim3(kThreads), st_smem, stream, p, q, x, u, V, K, tc, chunks,
               (const Stat*)part, mass, jbuf);
    launch_pdl(select_kernel<float>, dim3(B), dim3(kThreads), 0, stream, p, q, x, u, V, K, tc, chunks, (const Stat*)part,
               (const double*)mass, (const int*)jbuf, accept_len, out_tokens);
  }
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

}  // namespace tsd
