// tsd_tree_accept_sample: stochastic (multi-branch) acceptance of a draft tree at temperature > 0.
//
// "Acelerando Sonar a traves de la especulacion" (Perplexity), section "Objetivo-Borrador": the
// verifier accepts a draft token with the probability the rule of the cited Leviathan et al. paper
// gives, min(1, p/q), and after the accepted run samples one more token from the target; section
// "EAGLE": the draft is a tree of candidates.  Over a tree whose children were drawn independently
// from the draft distribution q of their parent, the plainest extension of that rule is taken:
// at the current node the children are tried in index order, child c (token x) is accepted iff
// u_c q(x) < p(x), and after a rejection the target is replaced by the normalised residual
// max(p - q, 0) / sum (left unchanged if the residual is empty), against which the next child is
// tested.  Acceptance moves to the accepted child and repeats; when every child of a node is
// rejected (or it is a leaf) the last token is drawn from the current target by the inverse CDF.
// With one child per node this is the chain rule of tsd_chain_accept_sample.
//
// Design.  The walk is sequential but each step is a vocabulary-wide reduction, so one sequence
// is one thread-block cluster of kC CTAs, each owning a slice of V / kC tokens: a step loads the
// current node's target and draft rows once from memory into the CTAs' shared memory (the only
// HBM traffic: two rows per node on the accepted path), and every later pass over them -- the
// softmax statistics, the residual mass after each rejection, the final inverse CDF -- runs from
// shared memory, with the slice results exchanged through distributed shared memory and a cluster
// barrier.  Every CTA merges the slice results in rank order, so every CTA of a cluster takes the
// same decisions and the same number of barriers.
//
// Precision as in the chain sampler: exponent arguments (z - zmax) log2(e) / T rounded once, fp32
// exponentials, everything else (sums, normalisers, the tests, the residual recursion, the CDF)
// in fp64.
#include <cooperative_groups.h>

#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace tsd {

namespace {

constexpr int kC = 8;           // CTAs per cluster (one sequence)
constexpr int kTS = 512;        // threads per CTA
constexpr int kMaxChildren = 256; // children tried at one node (a node with more flags the sequence)
constexpr double kLog2eD = 1.4426950408889634074;

struct Temp {
  float hi, lo;   // log2(e) / T as an unevaluated sum
};

struct TSArgs {
  const void* zp;           // [B, Nmax, V] target logits after each node
  const void* zq;           // [B, Nmax, V] draft logits each node's children were drawn from
  int V;
  const int32_t* tokens;    // [B, Nmax]
  const int32_t* parent_s;  // [B, Nmax + 1]
  const int32_t* num_nodes; // [B] or null
  const float* u;           // [B, Nmax]: u[c] tests node c, u[0] is the final draw
  Temp tc;
  int Nmax, Dmax;
  int slice;                // tokens per CTA (multiple of 8)
  int vec;                  // 16-byte loads of the rows
  int32_t* accept_len;
  int32_t* path;
  int32_t* out_tokens;
  int32_t* status;
};

struct Xch {      // one CTA's contribution to a cluster exchange
  float zmp, zmq;
  double sp, sq;  // sums of 2^((z - zm) c) over the slice
};

__device__ __forceinline__ float expo(float z, float zm, const Temp& t) {
  const float dz = z - zm;
  return exp2f(fmaf(dz, t.hi, dz * t.lo));
}

__device__ __forceinline__ float ldf(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float ldf(const float* p) { return *p; }

// Merge (zm2, s2) into (zm, s): sums relative to the larger maximum.
__device__ __forceinline__ void merge_stat(float& zm, double& s, float zm2, double s2, const Temp& t) {
  if (zm2 == -INFINITY) return;
  if (zm == -INFINITY) {
    zm = zm2, s = s2;
    return;
  }
  if (zm2 > zm) {
    s = s * (double)expo(zm, zm2, t) + s2;
    zm = zm2;
  } else {
    s += s2 * (double)expo(zm2, zm, t);
  }
}

__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < kTS / 32; ++i) m = fmaxf(m, red[i]);
  return m;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block sum in a fixed order (warp trees, then warps in order): the same value in every thread.
__device__ __forceinline__ double block_sum(double v, double* red) {
  v = warp_sum_d(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  double s = 0.0;
#pragma unroll
  for (int i = 0; i < kTS / 32; ++i) s += red[i];
  return s;
}

// Block maxima / sums of two values at once (one pair of barriers for both).
__device__ __forceinline__ void block_max2(float& a, float& b, float2* red) {
  a = warp_max(a), b = warp_max(b);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = make_float2(a, b);
  __syncthreads();
  a = -INFINITY, b = -INFINITY;
#pragma unroll
  for (int i = 0; i < kTS / 32; ++i) a = fmaxf(a, red[i].x), b = fmaxf(b, red[i].y);
}

__device__ __forceinline__ void block_sum2(double& a, double& b, double2* red) {
  a = warp_sum_d(a), b = warp_sum_d(b);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = make_double2(a, b);
  __syncthreads();
  a = 0.0, b = 0.0;
#pragma unroll
  for (int i = 0; i < kTS / 32; ++i) a += red[i].x, b += red[i].y;
}

// The running target after k rejections at a node: p_0 = softmax(zp / T) and
// p_j = max(p_{j-1} - q, 0) / R_j with R_j = sum_v max(p_{j-1} - q, 0).  By induction
// p_k = max(p_0 - C_k q, 0) * D_k with C_0 = 0, D_0 = 1, C_{j+1} = C_j + 1 / D_j, D_{j+1} = D_j / R_{j+1}
// (the same value as the step-by-step recursion up to rounding), so every level costs one
// multiply-subtract per token instead of k divisions.
struct Level {
  double C, D;
};

__device__ __forceinline__ double level_p(float zp, float zq, float Mp, double ip, float Mq, double iq,
                                          const Level& lv, const Temp& tc, double* q_out) {
  const double p = (double)expo(zp, Mp, tc) * ip;
  const bool need_q = lv.C != 0.0 || q_out;
  const double q = need_q ? (double)expo(zq, Mq, tc) * iq : 0.0;
  if (q_out) *q_out = q;
  const double r = p - lv.C * q;
  return r > 0.0 ? r * lv.D : 0.0;
}

template <typename T>
__global__ void __launch_bounds__(kTS, 1) tree_sample_kernel(const TSArgs a) {
  pdl_trigger();
  pdl_wait();
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int b = blockIdx.y;
  const int tid = threadIdx.x;
  extern __shared__ __align__(16) uint8_t smem[];
  T* sP = reinterpret_cast<T*>(smem);
  T* sQ = sP + a.slice;
  int32_t* sChild = reinterpret_cast<int32_t*>(sQ + a.slice);   // a.Nmax entries
  __shared__ float sCz[2 * kMaxChildren];                        // the children's (zp, zq) at their tokens
  __shared__ uint8_t sCin[kMaxChildren];
  __shared__ Xch s_x[2];            // exchange slots, alternating (one barrier per exchange)
  __shared__ double s_xd[2];        // exchange slots of scalar sums (residual / slice mass)
  __shared__ float s_redf[kTS / 32];
  __shared__ double s_redd[kTS / 32];
  __shared__ float2 s_redf2[kTS / 32];
  __shared__ double2 s_redd2[kTS / 32];
  __shared__ int s_wcnt[kTS / 32];
  __shared__ int s_path[256];
  __shared__ int s_nchild, s_acc, s_tok;
  __shared__ double s_run[kTS];

  const int V = a.V;
  // The entry verdict comes from rank 0 alone (published through distributed shared memory), so
  // the CTAs of a cluster agree on it even if another stream writes status[b] meanwhile.
  __shared__ int s_entry[2];
  if (rank == 0 && tid == 0) {
    s_entry[0] = a.num_nodes ? a.num_nodes[b] : a.Nmax;
    s_entry[1] = a.status[b];
  }
  cl.sync();
  if (tid == 0) {
    const int* e0 = cl.map_shared_rank(s_entry, 0);
    s_nchild = e0[0];
    s_acc = e0[1];
  }
  __syncthreads();
  const int N = s_nchild;
  const bool live = s_acc == 0 && N > 0 && N <= a.Nmax;
  __syncthreads();
  int32_t* prow_out = a.path + (size_t)b * (a.Dmax + 1);
  int32_t* orow_out = a.out_tokens + (size_t)b * (a.Dmax + 1);
  if (!live) {   // every CTA of the cluster takes this branch alike: no barrier is skipped by some
    if (rank == 0) {
      for (int j = tid; j <= a.Dmax; j += kTS) prow_out[j] = 0, orow_out[j] = -1;
      if (tid == 0) a.accept_len[b] = -1;
    }
    cl.sync();   // rank 0's entry words are read by its peers until here
    return;
  }
  const int32_t* ps = a.parent_s + (size_t)b * (a.Nmax + 1);
  const int32_t* tok = a.tokens + (size_t)b * a.Nmax;
  const float* ub = a.u + (size_t)b * a.Nmax;
  const int lo = rank * a.slice;
  const int cnt = max(0, min(V, lo + a.slice) - lo);
  int ph = 0;   // exchange phase

  // Cluster exchanges: thread 0 publishes this CTA's value, the cluster barrier orders it before
  // every peer's read, thread 0 reads all kC values in rank order and broadcasts the merge.  Slots
  // alternate between two phases, so one barrier per exchange suffices: a slot is rewritten only
  // after the next barrier, which every reader of its previous value has passed.
  __shared__ Xch s_merged;
  __shared__ double s_each[kC];
  auto exchange_stats = [&](float zmp, double sp, float zmq, double sq, float& Mp, double& Sp, float& Mq,
                            double& Sq) {
    if (tid == 0) s_x[ph] = Xch{zmp, zmq, sp, sq};
    cl.sync();
    if (tid == 0) {
      Xch x[kC];
#pragma unroll
      for (int r = 0; r < kC; ++r) x[r] = *cl.map_shared_rank(&s_x[ph], r);
      Xch m{-INFINITY, -INFINITY, 0.0, 0.0};
#pragma unroll
      for (int r = 0; r < kC; ++r) {
        merge_stat(m.zmp, m.sp, x[r].zmp, x[r].sp, a.tc);
        merge_stat(m.zmq, m.sq, x[r].zmq, x[r].sq, a.tc);
      }
      s_merged = m;
    }
    __syncthreads();
    Mp = s_merged.zmp, Sp = s_merged.sp, Mq = s_merged.zmq, Sq = s_merged.sq;
    __syncthreads();
    ph ^= 1;
  };
  // sum over the cluster of one double per CTA in rank order; s_each keeps each rank's value
  auto exchange_sum = [&](double v) -> double {
    if (tid == 0) s_xd[ph] = v;
    cl.sync();
    if (tid == 0) {
#pragma unroll
      for (int r = 0; r < kC; ++r) s_each[r] = *cl.map_shared_rank(&s_xd[ph], r);
    }
    __syncthreads();
    double s = 0.0;
#pragma unroll
    for (int r = 0; r < kC; ++r) s += s_each[r];
    ph ^= 1;
    return s;
  };

  int n = 0, depth = 0;
  bool too_wide = false;
  if (tid == 0) s_path[0] = 1;
  for (;;) {
    // ---- children of n in index order (ordered compaction of parent_s[i + 1] == n + 1)
    int nc = 0;
    for (int base = n + 1; base < N; base += kTS) {
      const int i = base + tid;
      const bool is = i < N && ps[i + 1] == n + 1;
      const unsigned m = __ballot_sync(0xffffffffu, is);
      const int w = tid >> 5, l = tid & 31;
      if (l == 0) s_wcnt[w] = __popc(m);
      __syncthreads();
      int before = nc;
      for (int k = 0; k < w; ++k) before += s_wcnt[k];
      if (is) sChild[before + __popc(m & ((1u << l) - 1u))] = i;
      int tot = 0;
      for (int k = 0; k < kTS / 32; ++k) tot += s_wcnt[k];
      nc += tot;
      __syncthreads();
    }
    if (nc > kMaxChildren) {   // more children than the walk tries: the sequence is flagged
      too_wide = true;
      break;
    }
    if (depth >= a.Dmax) nc = 0;   // the path cannot grow past Dmax
    const bool need_q = nc > 0;
    // ---- this node's target (and draft) rows: one read from memory into the CTA's slice
    {
      const T* gp = reinterpret_cast<const T*>(a.zp) + ((size_t)b * a.Nmax + n) * V + lo;
      const T* gq = reinterpret_cast<const T*>(a.zq) + ((size_t)b * a.Nmax + n) * V + lo;
      if (a.vec) {
        constexpr int E = 16 / sizeof(T);
        const int nv = cnt / E;
        for (int i = tid; i < nv; i += kTS) {
          reinterpret_cast<uint4*>(sP)[i] = __ldg(reinterpret_cast<const uint4*>(gp) + i);
          if (need_q) reinterpret_cast<uint4*>(sQ)[i] = __ldg(reinterpret_cast<const uint4*>(gq) + i);
        }
      } else {
        for (int i = tid; i < cnt; i += kTS) {
          sP[i] = gp[i];
          if (need_q) sQ[i] = gq[i];
        }
      }
    }
    __syncthreads();
    // ---- softmax statistics of both rows over the cluster
    float mp = -INFINITY, mq = -INFINITY;
    for (int i = tid; i < cnt; i += kTS) {
      mp = fmaxf(mp, ldf(sP + i));
      if (need_q) mq = fmaxf(mq, ldf(sQ + i));
    }
    block_max2(mp, mq, s_redf2);
    double sp = 0.0, sq = 0.0;
    for (int i = tid; i < cnt; i += kTS) {
      if (mp != -INFINITY) sp += (double)expo(ldf(sP + i), mp, a.tc);
      if (need_q && mq != -INFINITY) sq += (double)expo(ldf(sQ + i), mq, a.tc);
    }
    block_sum2(sp, sq, s_redd2);
    float Mp, Mq;
    double Sp, Sq;
    exchange_stats(mp, sp, mq, sq, Mp, Sp, Mq, Sq);
    const double ip = Sp > 0.0 ? 1.0 / Sp : 0.0, iq = Sq > 0.0 ? 1.0 / Sq : 0.0;
    // ---- children in order against the running residual
    Level lv{0.0, 1.0};
    int accepted = -1;
    const T* gp = reinterpret_cast<const T*>(a.zp) + ((size_t)b * a.Nmax + n) * V;
    const T* gq = reinterpret_cast<const T*>(a.zq) + ((size_t)b * a.Nmax + n) * V;
    // every child's token and two logits are gathered at once (one round trip), then tested in order
    for (int ci = tid; ci < nc; ci += kTS) {
      const int c = sChild[ci];
      const int x = tok[c];
      const bool in = x >= 0 && x < V;
      sCz[2 * ci] = in ? ldf(gp + x) : 0.f;
      sCz[2 * ci + 1] = in ? ldf(gq + x) : 0.f;
      sCin[ci] = in ? 1 : 0;
    }
    __syncthreads();
    for (int ci = 0; ci < nc; ++ci) {
      const int c = sChild[ci];
      if (tid == 0) {
        bool acc = false;
        if (sCin[ci]) {
          double qx;
          const double px = level_p(sCz[2 * ci], sCz[2 * ci + 1], Mp, ip, Mq, iq, lv, a.tc, &qx);
          acc = (double)ub[c] * qx < px;
        }
        s_acc = acc ? 1 : 0;
      }
      __syncthreads();
      const bool acc = s_acc != 0;
      __syncthreads();
      if (acc) {
        accepted = c;
        break;
      }
      // residual mass of the current level over the vocabulary
      double r = 0.0;
      for (int i = tid; i < cnt; i += kTS) {
        double q;
        const double p = level_p(ldf(sP + i), ldf(sQ + i), Mp, ip, Mq, iq, lv, a.tc, &q);
        r += p > q ? p - q : 0.0;
      }
      r = block_sum(r, s_redd);
      const double R = exchange_sum(r);
      __syncthreads();   // s_each is rewritten by the next exchange
      if (R > 0.0) lv = Level{lv.C + 1.0 / lv.D, lv.D / R};
    }
    if (accepted >= 0) {
      ++depth;
      if (tid == 0) s_path[depth] = accepted + 1;
      n = accepted;
      __syncthreads();
      continue;
    }
    // ---- final draw from the current level by the inverse CDF: slice masses, then the CTA
    // holding the threshold scans its slice (each thread owns a contiguous run)
    const int per = (cnt + kTS - 1) / kTS;
    const int ra = min(cnt, tid * per), re = min(cnt, ra + per);
    double run = 0.0;
    int lastp = -1;
    for (int i = ra; i < re; ++i) {
      const double p = level_p(ldf(sP + i), need_q ? ldf(sQ + i) : 0.f, Mp, ip, Mq, iq, lv, a.tc, nullptr);
      if (p > 0.0) lastp = i;
      run += p;
    }
    // exclusive prefix of the runs in thread order
    double incl = run;
    const int w = tid >> 5, l = tid & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (l >= o) incl += y;
    }
    if (l == 31) s_redd[w] = incl;
    __syncthreads();
    double wbase = 0.0, mass = 0.0;
    for (int i = 0; i < kTS / 32; ++i) {
      if (i < w) wbase += s_redd[i];
      mass += s_redd[i];
    }
    s_run[tid] = wbase + incl - run;
    if (tid == 0) s_tok = INT_MAX;
    __syncthreads();
    const double total = exchange_sum(mass);
    double each[kC];
#pragma unroll
    for (int r = 0; r < kC; ++r) each[r] = s_each[r];
    const double thr = (double)ub[0] * total;
    int cstar = -1;
    double cum = 0.0;
    for (int r = 0; r < kC; ++r) {
      if (each[r] > 0.0 && cum + each[r] > thr) {
        cstar = r;
        break;
      }
      cum += each[r];
    }
    bool fallback = false;
    if (cstar < 0) {   // threshold at or past the rounded total: the last token with mass
      for (int r = kC - 1; r >= 0; --r)
        if (each[r] > 0.0) {
          cstar = r;
          break;
        }
      fallback = true;
    }
    if (rank == (cstar < 0 ? 0 : cstar)) {
      if (cstar >= 0 && !fallback) {
        const double t = thr - cum;
        double c0 = s_run[tid];
        if (c0 <= t && ra < re && c0 + run > t) {
          for (int i = ra; i < re; ++i) {
            c0 += level_p(ldf(sP + i), need_q ? ldf(sQ + i) : 0.f, Mp, ip, Mq, iq, lv, a.tc, nullptr);
            if (c0 > t) {
              atomicMin(&s_tok, lo + i);
              break;
            }
          }
        }
      }
      __syncthreads();
      if (s_tok == INT_MAX) {   // rounding left the threshold past the run sums: last token with mass
        __shared__ int s_last;
        if (tid == 0) s_last = -1;
        __syncthreads();
        if (lastp >= 0) atomicMax(&s_last, lo + lastp);
        __syncthreads();
        if (tid == 0) s_tok = s_last >= 0 ? s_last : 0;
        __syncthreads();
      }
      for (int j = tid; j <= a.Dmax; j += kTS) {
        prow_out[j] = j <= depth ? s_path[j] : 0;
        orow_out[j] = j < depth ? tok[s_path[j + 1] - 1] : (j == depth ? s_tok : -1);
      }
      if (tid == 0) a.accept_len[b] = depth;
    }
    break;
  }
  cl.sync();   // no CTA leaves while a peer may still read its shared memory
  // status is written only here, after every CTA of the cluster has read it at entry
  if (too_wide && rank == 0) {
    for (int j = tid; j <= a.Dmax; j += kTS) prow_out[j] = 0, orow_out[j] = -1;
    if (tid == 0) {
      a.accept_len[b] = -1;
      flag_status(a.status, b, TSD_ERR_INVALID_ARG, n);
    }
  }
}

}  // namespace

int tree_sample_cluster() { return kC; }

tsd_status launch_tree_sample(const void* zp, const void* zq, tsd_dtype dtype, int V, const int32_t* tokens,
                              const int32_t* parent_s, const int32_t* num_nodes, const float* u, float T, int B,
                              int Nmax, int Dmax, int32_t* accept_len, int32_t* path, int32_t* out_tokens,
                              int32_t* status, cudaStream_t stream) {
  if (B == 0) return TSD_OK;
  TSArgs a{};
  a.zp = zp, a.zq = zq, a.V = V, a.tokens = tokens, a.parent_s = parent_s, a.num_nodes = num_nodes, a.u = u;
  const double c = kLog2eD / (double)T;
  split_const(c, a.tc.hi, a.tc.lo);
  a.Nmax = Nmax, a.Dmax = Dmax;
  a.slice = ((V + kC - 1) / kC + 7) / 8 * 8;
  a.vec = vec16_rows(zp, V) && vec16_rows(zq, V) ? 1 : 0;
  a.accept_len = accept_len, a.path = path, a.out_tokens = out_tokens, a.status = status;
  const size_t es = dtype == TSD_BF16 ? 2 : 4;
  const size_t smem = 2 * (size_t)a.slice * es + (size_t)Nmax * 4;
  if (smem > 200 * 1024) return TSD_ERR_INVALID_ARG;
  auto kernel = dtype == TSD_BF16 ? tree_sample_kernel<__nv_bfloat16> : tree_sample_kernel<float>;
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kC, B);
  cfg.blockDim = dim3(kTS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kC, attr[0].val.clusterDim.y = 1, attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, kernel, a) != cudaSuccess) return TSD_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

size_t tree_sample_smem(int V, int Nmax, tsd_dtype dtype) {
  const size_t slice = ((size_t)(V + kC - 1) / kC + 7) / 8 * 8;
  return 2 * slice * (dtype == TSD_BF16 ? 2 : 4) + (size_t)Nmax * 4;
}

}  // namespace tsd
