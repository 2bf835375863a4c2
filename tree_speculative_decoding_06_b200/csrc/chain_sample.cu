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
// exponentials themselves are fp32 (relative error ~1e-7, independent per token); the chunk sums
// are combined with fp64 factors.
//
// Kernels (the first is the HBM-bound scan of all 2K+1 rows; the rest touch two rows at most):
//   1. chain_stats:  per (chunk, row): the chunk maximum, then the fp64 sum of the chunk's
//      exponentials relative to it (a second pass over the 16 KB chunk, from cache);
//   2. chain_decide: per sequence: the rows' statistics merged once, the K accept tests in order,
//      and the parameters of the final distribution (residual or bonus row);
//   3. chain_mass:   per (chunk, sequence): the chunk's mass under the final distribution;
//   4. chain_select: per sequence: the chunk holding the threshold, then an inverse CDF inside it
//      (each thread a contiguous run of tokens, block prefix of the run sums).
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace tsd {

namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 8192;
constexpr double kLog2eD = 1.4426950408889634074;

struct __align__(16) Stat {
  float zm;   // logit maximum of the chunk / row
  float pad;
  double s;   // sum of 2^((z - zm) * c), c = log2(e) / T
};

struct Temp {    // c = log2(e) / T as an unevaluated sum hi + lo, and in fp64
  float hi, lo;
  double c;
};

// Parameters of the final distribution of one sequence (written by chain_decide).
struct __align__(16) Final {
  float zmp, zmq;
  double ip, iq;   // 1 / row sums
  int j;           // first rejected position (K: all accepted -> bonus row K)
  int residual;    // 1: max(p_j - q_j, 0); 0: p_j
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

// Merge (zm2, s2) into (zm, s) with an fp64 factor.
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

__device__ __forceinline__ Stat merge_stats(const Stat* p, int chunks, double c) {
  float M = -INFINITY;
  double S = 0.0;
  for (int i = 0; i < chunks; ++i) merge(M, S, p[i].zm, p[i].s, c);
  Stat st;
  st.zm = M, st.pad = 0.f, st.s = S;
  return st;
}

__device__ __forceinline__ double block_sum_d(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) t += red[w];
  __syncthreads();
  return t;   // the same value in every thread
}

template <typename T>
__global__ void __launch_bounds__(kThreads) chain_stats(const T* __restrict__ zp, const T* __restrict__ zq, int V,
                                                        int K, Temp tc, int chunks, Stat* __restrict__ part,
                                                        int vec) {
  pdl_trigger();   // the scan reads inputs only; pdl_wait() comes before the partial is written
  const int c = blockIdx.x, r = blockIdx.y, b = blockIdx.z;
  const T* row = chain_row(zp, zq, K, V, b, r);
  const int lo = c * kChunk, hi = min(V, lo + kChunk);
  __shared__ float sm[kThreads / 32];
  __shared__ double sd[kThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // one read of the chunk: a thread's 32 logits stay in registers (16-byte path); each warp sums
  // its exponentials relative to its own maximum, then the warps' sums are rescaled (fp64) to the
  // chunk maximum
  float lm = -INFINITY, wm;
  double s = 0.0;
  if (vec) {
    constexpr int kGroups = kChunk / (kThreads * 8);
    float x[kGroups][8];
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
      for (int gi = 0; gi < kGroups; ++gi) s += (double)sum_exp2f_8(x[gi], wm, tc.hi, tc.lo);   // -inf adds 0
  } else {
    for (int v = lo + threadIdx.x; v < hi; v += kThreads) lm = fmaxf(lm, load1(row, v));
    wm = warp_max(lm);
    if (wm != -INFINITY)
      for (int v = lo + threadIdx.x; v < hi; v += kThreads) s += (double)expo(load1(row, v), wm, tc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) sm[warp] = wm;
  __syncthreads();
  float zm = -INFINITY;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) zm = fmaxf(zm, sm[w]);
  if (lane == 0) sd[warp] = (s == 0.0 || wm == zm) ? s : s * exp2(((double)wm - (double)zm) * tc.c);
  __syncthreads();
  s = 0.0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) s += sd[w];
  pdl_wait();
  if (threadIdx.x == 0) {
    Stat st;
    st.zm = zm, st.pad = 0.f, st.s = s;
    part[((size_t)b * (2 * K + 1) + r) * chunks + c] = st;
  }
}

// One CTA per sequence: row statistics merged (one thread per row), the drafts' exponentials (one
// thread per draft), then thread 0 takes the K tests in order -- accept iff u q(x) < p(x), i.e.
// u * eq * s_p < ep * s_q in fp64 -- and records the final distribution's parameters.
template <typename T>
__global__ void __launch_bounds__(kThreads) chain_decide(const T* __restrict__ zp, const T* __restrict__ zq,
                                                         const int32_t* __restrict__ x, const float* __restrict__ u,
                                                         int V, int K, Temp tc, int chunks,
                                                         const Stat* __restrict__ part, Final* __restrict__ fin,
                                                         int32_t* __restrict__ accept_len,
                                                         int32_t* __restrict__ out_tokens) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ Stat s_st[];                                  // 2K+1 row statistics
  float* s_ex = reinterpret_cast<float*>(s_st + 2 * K + 1);      // 2K draft exponentials
  __shared__ int s_j;
  const int b = blockIdx.x;
  for (int r = threadIdx.x; r < 2 * K + 1; r += blockDim.x)
    s_st[r] = merge_stats(part + ((size_t)b * (2 * K + 1) + r) * chunks, chunks, tc.c);
  __syncthreads();
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const int xk = x[(size_t)b * K + k];
    const bool in = xk >= 0 && xk < V;
    s_ex[2 * k] = in ? expo(load1(chain_row(zp, zq, K, V, b, k), xk), s_st[k].zm, tc) : 0.f;
    s_ex[2 * k + 1] = in ? expo(load1(chain_row(zp, zq, K, V, b, K + 1 + k), xk), s_st[K + 1 + k].zm, tc) : 1.f;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int j = K;
    for (int k = 0; k < K; ++k) {
      const double lhs = (double)u[(size_t)b * (K + 1) + k] * (double)s_ex[2 * k + 1] * s_st[k].s;
      const double rhs = (double)s_ex[2 * k] * s_st[K + 1 + k].s;
      if (!(lhs < rhs)) {
        j = k;
        break;
      }
    }
    Final f;
    f.j = j;
    f.residual = j < K ? 1 : 0;
    f.zmp = s_st[j].zm, f.ip = 1.0 / s_st[j].s;
    f.zmq = f.residual ? s_st[K + 1 + j].zm : 0.f;
    f.iq = f.residual ? 1.0 / s_st[K + 1 + j].s : 0.0;
    fin[b] = f;
    accept_len[b] = j;
    s_j = j;
  }
  __syncthreads();
  const int j = s_j;
  int32_t* orow = out_tokens + (size_t)b * (K + 1);
  for (int k = threadIdx.x; k <= K; k += blockDim.x) {
    if (k < j) orow[k] = x[(size_t)b * K + k];
    else if (k > j) orow[k] = -1;
  }
}

// Mass of the final distribution at token v: max(p_j - q_j, 0) after a rejection, p otherwise.
__device__ __forceinline__ double final_mass(float zp, float zq, const Final& f, const Temp& tc, bool residual) {
  const double p = (double)expo(zp, f.zmp, tc) * f.ip;
  if (!residual) return p;
  const double q = (double)expo(zq, f.zmq, tc) * f.iq;
  return p > q ? p - q : 0.0;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) chain_mass(const T* __restrict__ zp, const T* __restrict__ zq, int V,
                                                       int K, Temp tc, int chunks, const Final* __restrict__ fin,
                                                       double* __restrict__ mass, int vec) {
  pdl_trigger();
  pdl_wait();
  __shared__ double red[kThreads / 32];
  const int c = blockIdx.x, b = blockIdx.y;
  const Final f = fin[b];
  const bool res = f.residual != 0;
  const T* prow = chain_row(zp, zq, K, V, b, f.j);
  const T* qrow = res ? chain_row(zp, zq, K, V, b, K + 1 + f.j) : prow;
  const int lo = c * kChunk, hi = min(V, lo + kChunk);
  double acc = 0.0;
  if (vec) {
    for (int v = lo + threadIdx.x * 8; v < hi; v += kThreads * 8) {
      float xp[8], xq[8];
      load8<T>(prow, v, xp);
      if (res) load8<T>(qrow, v, xq);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc += final_mass(xp[e], res ? xq[e] : 0.f, f, tc, res);
    }
  } else {
    for (int v = lo + threadIdx.x; v < hi; v += kThreads)
      acc += final_mass(load1(prow, v), res ? load1(qrow, v) : 0.f, f, tc, res);
  }
  const double t = block_sum_d(acc, red);
  if (threadIdx.x == 0) mass[(size_t)b * chunks + c] = t;
}

// Inverse CDF inside [lo, hi): the smallest v whose cumulative mass (counted from lo) exceeds thr.
// Thread t owns a contiguous run of the range; run sums are prefixed with warp shuffles (fp64) and
// the thread whose run holds the threshold rescans it.  Returns -1 when the threshold is not
// reached; *last_pos = the last token with mass in the range.
template <typename T>
__device__ int cta_inverse_cdf(const T* prow, const T* qrow, int lo, int hi, double thr, const Final& f,
                               const Temp& tc, bool res, int* last_pos) {
  __shared__ double s_w[kThreads / 32];
  __shared__ int s_tok, s_last;
  const int n = hi - lo, run = (n + kThreads - 1) / kThreads;
  const int a = lo + min(n, (int)threadIdx.x * run), e = lo + min(n, ((int)threadIdx.x + 1) * run);
  double sum = 0.0;
  int lastp = -1;
  for (int v = a; v < e; ++v) {
    const double r = final_mass(load1(prow, v), res ? load1(qrow, v) : 0.f, f, tc, res);
    if (r > 0.0) lastp = v;
    sum += r;
  }
  if (threadIdx.x == 0) s_tok = INT_MAX, s_last = -1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  double incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_w[warp] = incl;
  __syncthreads();
  if (lastp >= 0) atomicMax(&s_last, lastp);
  double cum = incl - sum;   // exclusive prefix of this thread's run
  for (int w = 0; w < warp; ++w) cum += s_w[w];
  if (cum <= thr && a < e && cum + sum > thr) {
    for (int v = a; v < e; ++v) {
      cum += final_mass(load1(prow, v), res ? load1(qrow, v) : 0.f, f, tc, res);
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
__global__ void __launch_bounds__(kThreads) chain_select(const T* __restrict__ zp, const T* __restrict__ zq,
                                                         const float* __restrict__ u, int V, int K, Temp tc,
                                                         int chunks, const Final* __restrict__ fin,
                                                         const double* __restrict__ mass,
                                                         int32_t* __restrict__ out_tokens) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_c;
  __shared__ double s_thr;
  __shared__ double red[kThreads / 32];
  const int b = blockIdx.x;
  const Final f = fin[b];
  const bool res = f.residual != 0;
  if (threadIdx.x == 0) {
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
    s_c = cstar;
    s_thr = cstar >= 0 ? (cum >= 1e299 ? 1e300 : thr - cum) : 0.0;
  }
  __syncthreads();
  const T* prow = chain_row(zp, zq, K, V, b, f.j);
  const T* qrow = res ? chain_row(zp, zq, K, V, b, K + 1 + f.j) : prow;
  int tok, lastp;
  if (s_c >= 0) {
    const int lo = s_c * kChunk, hi = min(V, lo + kChunk);
    tok = cta_inverse_cdf(prow, qrow, lo, hi, s_thr, f, tc, res, &lastp);
  } else {
    double acc = 0.0;
    for (int v = threadIdx.x; v < V; v += kThreads) acc += final_mass(load1(prow, v), 0.f, f, tc, false);
    const double t = block_sum_d(acc, red);
    const double thr = t * (double)u[(size_t)b * (K + 1) + K];
    tok = cta_inverse_cdf(prow, prow, 0, V, thr, f, tc, false, &lastp);
  }
  if (threadIdx.x != 0) return;
  if (tok < 0) tok = lastp >= 0 ? lastp : 0;
  out_tokens[(size_t)b * (K + 1) + f.j] = tok;
}

}  // namespace

size_t chain_sample_ws(int B, int K, int V) {
  const int chunks = num_chunks(V);
  const size_t stats = (size_t)B * (2 * K + 1) * chunks * sizeof(Stat);
  const size_t fin = (size_t)B * sizeof(Final);
  const size_t mass = (size_t)B * chunks * sizeof(double);
  return stats + fin + mass + 64;
}

tsd_status launch_chain_sample_stochastic(const void* zp, const void* zq, tsd_dtype dtype, int V, const int32_t* x,
                                          const float* u, float T, int B, int K, int32_t* accept_len,
                                          int32_t* out_tokens, void* ws, cudaStream_t stream) {
  const int chunks = num_chunks(V);
  Stat* part = reinterpret_cast<Stat*>(ws);
  Final* fin = reinterpret_cast<Final*>(part + (size_t)B * (2 * K + 1) * chunks);
  double* mass = reinterpret_cast<double*>(fin + B);
  Temp tc;
  tc.c = kLog2eD / (double)T;
  split_const(tc.c, tc.hi, tc.lo);
  const size_t dsmem = (size_t)(2 * K + 1) * sizeof(Stat) + (size_t)2 * K * sizeof(float) + 16;
  dim3 g1(chunks, 2 * K + 1, B), g3(chunks, B);
  const int vec = vec16_rows(zp, V) && (K == 0 || vec16_rows(zq, V)) ? 1 : 0;
  if (dtype == TSD_BF16) {
    auto p = reinterpret_cast<const __nv_bfloat16*>(zp);
    auto q = reinterpret_cast<const __nv_bfloat16*>(zq);
    if (dsmem > 48 * 1024)
      cudaFuncSetAttribute(chain_decide<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsmem);
    launch_pdl(chain_stats<__nv_bfloat16>, g1, dim3(kThreads), 0, stream, p, q, V, K, tc, chunks, part, vec);
    launch_pdl(chain_decide<__nv_bfloat16>, dim3(B), dim3(kThreads), dsmem, stream, p, q, x, u, V, K, tc, chunks,
               (const Stat*)part, fin, accept_len, out_tokens);
    launch_pdl(chain_mass<__nv_bfloat16>, g3, dim3(kThreads), 0, stream, p, q, V, K, tc, chunks, (const Final*)fin,
               mass, vec);
    launch_pdl(chain_select<__nv_bfloat16>, dim3(B), dim3(kThreads), 0, stream, p, q, u, V, K, tc, chunks,
               (const Final*)fin, (const double*)mass, out_tokens);
  } else {
    auto p = reinterpret_cast<const float*>(zp);
    auto q = reinterpret_cast<const float*>(zq);
    if (dsmem > 48 * 1024)
      cudaFuncSetAttribute(chain_decide<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsmem);
    launch_pdl(chain_stats<float>, g1, dim3(kThreads), 0, stream, p, q, V, K, tc, chunks, part, vec);
    launch_pdl(chain_decide<float>, dim3(B), dim3(kThreads), dsmem, stream, p, q, x, u, V, K, tc, chunks,
               (const Stat*)part, fin, accept_len, out_tokens);
    launch_pdl(chain_mass<float>, g3, dim3(kThreads), 0, stream, p, q, V, K, tc, chunks, (const Final*)fin, mass,
               vec);
    launch_pdl(chain_select<float>, dim3(B), dim3(kThreads), 0, stream, p, q, u, V, K, tc, chunks, (const Final*)fin,
               (const double*)mass, out_tokens);
  }
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

}  // namespace tsd
