// tsd_ssd_cache_build: the SSD / Saguaro outcome cache of one verification round.
//
// "Speculative Speculative Decoding", technical summary sec. 2 and sec. 3 A-B: while the target
// verifies, the draft predicts the verification outcome -- how many draft tokens will be accepted
// and which bonus token the target adds -- and pre-drafts a continuation for each likely outcome
// (the outcome cache; a hit sends the pre-drafted continuation straight to verification).  The
// budget of cache slots is spread by a geometric fan-out over the accepted lengths the acceptance
// rate makes likely, and Saguaro sampling lowers, while drafting, the draft probability of the
// tokens the cache holds, which raises the residual mass the target's bonus draw puts on them.
//
// Reading (the page gives the ideas, not formulas): with per-token acceptance rate alpha the
// accepted length a in 0..K has P(a) = alpha^a (1 - alpha) (a < K), P(K) = alpha^K; the S slots
// are apportioned by the largest-remainder rule (floor(S P(a)), then one more slot to the largest
// remainders, ties -> shorter length); the n_a slots of length a hold the n_a most likely tokens
// of the draft distribution at position a+1 (the token a rejection at a+1 would be replaced by, or
// the free token at a = K), ties -> lower id; the draft token of position j+1 (j < K) is drawn by
// the inverse CDF from q' proportional to q times beta on the tokens cached for length j.
//
// Design: the K+1 rows of a sequence are independent, so each (sequence, row) is one cluster of
// kC CTAs that loads the row once into shared-memory slices.  The n_a-th largest logit is found
// by a radix select on order-preserving integer keys (8-bit digits, cluster-wide histograms
// exchanged through distributed shared memory), ties at the threshold go to the lowest ids in
// slice order, the selected tokens are ordered by (logit desc, id asc) -- softmax preserves the
// order -- and the Saguaro draw runs over the slices as in the tree sampler: fp32 exponentials,
// fp64 sums, slice masses exchanged in rank order, the CTA holding the threshold scans its slice.
#include <cooperative_groups.h>

#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace tsd {

namespace {

constexpr int kC = 8;
constexpr int kTS = 512;
constexpr int kMaxS = 256;     // slots per sequence
constexpr int kMaxK = 63;      // draft length
constexpr double kLog2eD = 1.4426950408889634074;

struct SSDArgs {
  const void* zq;          // [B, K+1, V] draft logits (row a = the draft distribution at position a+1)
  int V, K, S;
  const float* alpha;      // [B]
  float beta;
  const float* u;          // [B, K]
  float thi, tlo;          // log2(e) / T as an unevaluated sum
  int slice;
  int vec;
  int32_t* slots;          // [B, K+1]
  int32_t* key_len;        // [B, S]
  int32_t* key_tok;        // [B, S]
  int32_t* draft_tokens;   // [B, K]
};

__device__ __forceinline__ float expo(float z, float zm, float hi, float lo) {
  const float dz = z - zm;
  return exp2f(fmaf(dz, hi, dz * lo));
}

// Order-preserving unsigned keys of the logits (larger value -> larger key; NaN -> 0, never kept
// ahead of a number).
__device__ __forceinline__ uint32_t okey(__nv_bfloat16 x) {
  const uint32_t b = __bfloat16_as_ushort(x);
  if ((b & 0x7fffu) > 0x7f80u) return 0u;
  return (b & 0x8000u) ? (~b & 0xffffu) : (b | 0x8000u);
}
__device__ __forceinline__ uint32_t okey(float x) {
  const uint32_t b = __float_as_uint(x);
  if ((b & 0x7fffffffu) > 0x7f800000u) return 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
template <typename T>
constexpr int key_bits() { return sizeof(T) * 8; }

__device__ __forceinline__ float ldf(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float ldf(float x) { return x; }

// Largest-remainder apportionment of S slots over the lengths 0..K (every thread computes it).
__device__ void fanout(float alpha_in, int K, int S, int* n) {
  double alpha = alpha_in;
  alpha = alpha < 0.0 ? 0.0 : (alpha > 1.0 ? 1.0 : alpha);
  double share[kMaxK + 1], rem[kMaxK + 1];
  double pw = 1.0;   // alpha^a by repeated multiplication
  int used = 0;
  for (int a = 0; a <= K; ++a) {
    const double P = a < K ? pw * (1.0 - alpha) : pw;
    share[a] = (double)S * P;
    n[a] = (int)floor(share[a]);
    rem[a] = share[a] - (double)n[a];
    used += n[a];
    pw *= alpha;
  }
  const int left = S - used;
  for (int a = 0; a <= K; ++a) {   // rank of a among the remainders (larger first, then shorter)
    int rank = 0;
    for (int c = 0; c <= K; ++c) rank += (rem[c] > rem[a]) || (rem[c] == rem[a] && c < a);
    if (rank < left) ++n[a];
  }
}

template <typename T>
__global__ void __launch_bounds__(kTS, 2) ssd_cache_kernel(const SSDArgs a) {
  pdl_trigger();
  pdl_wait();
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int row = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ __align__(16) uint8_t smem[];
  T* sZ = reinterpret_cast<T*>(smem);
  __shared__ int s_n[kMaxK + 1];
  __shared__ uint32_t s_hist[256];
  __shared__ uint32_t s_xh[2][256];      // histogram exchange slots
  __shared__ double s_xd[2];             // scalar exchange slots
  __shared__ double2 s_xd2[2], s_xd2m;
  __shared__ float s_xf[2];
  __shared__ int s_xi[2];
  __shared__ uint32_t s_sel_key[kMaxS];  // this CTA's selected tokens
  __shared__ int s_sel_tok[kMaxS];
  __shared__ int s_nsel;
  __shared__ double s_redd[kTS / 32];
  __shared__ float s_redf[kTS / 32];
  __shared__ int s_wcnt[kTS / 32];
  __shared__ double s_each[kC];
  __shared__ int s_eachi[kC];
  __shared__ double s_run[kTS];
  __shared__ int s_tok, s_digit, s_above;
  const int V = a.V, K = a.K;
  const int lo = rank * a.slice;
  const int cnt = max(0, min(V, lo + a.slice) - lo);
  int ph = 0;

  if (tid == 0) fanout(a.alpha[b], K, a.S, s_n);
  // this CTA's slice of the row, read once
  {
    const T* g = reinterpret_cast<const T*>(a.zq) + ((size_t)b * (K + 1) + row) * V + lo;
    if (a.vec) {
      constexpr int E = 16 / sizeof(T);
      for (int i = tid; i < cnt / E; i += kTS) reinterpret_cast<uint4*>(sZ)[i] = __ldg(reinterpret_cast<const uint4*>(g) + i);
    } else {
      for (int i = tid; i < cnt; i += kTS) sZ[i] = g[i];
    }
  }
  __syncthreads();
  const int na = s_n[row];
  int off = 0;
  for (int c = 0; c < row; ++c) off += s_n[c];
  if (row == 0 && rank == 0)
    for (int c = tid; c <= K; c += kTS) a.slots[(size_t)b * (K + 1) + c] = s_n[c];

  auto sum_d = [&](double v) -> double {   // cluster sum in rank order; s_each keeps the terms
    if (tid == 0) s_xd[ph] = v;
    cl.sync();
    if (tid == 0)
      for (int r = 0; r < kC; ++r) s_each[r] = *cl.map_shared_rank(&s_xd[ph], r);
    __syncthreads();
    double s = 0.0;
    for (int r = 0; r < kC; ++r) s += s_each[r];
    __syncthreads();
    ph ^= 1;
    return s;
  };
  auto sum_d2 = [&](double v0, double v1, double& t0, double& t1) {   // two cluster sums, one barrier
    if (tid == 0) s_xd2[ph] = make_double2(v0, v1);
    cl.sync();
    if (tid == 0) {
      double2 t = make_double2(0.0, 0.0);
      for (int r = 0; r < kC; ++r) {
        const double2 x = *cl.map_shared_rank(&s_xd2[ph], r);
        t.x += x.x, t.y += x.y;
      }
      s_xd2m = t;
    }
    __syncthreads();
    t0 = s_xd2m.x, t1 = s_xd2m.y;
    __syncthreads();
    ph ^= 1;
  };
  auto sum_i = [&](int v) -> int {         // cluster sum; s_eachi keeps the terms
    if (tid == 0) s_xi[ph] = v;
    cl.sync();
    if (tid == 0)
      for (int r = 0; r < kC; ++r) s_eachi[r] = *cl.map_shared_rank(&s_xi[ph], r);
    __syncthreads();
    int s = 0;
    for (int r = 0; r < kC; ++r) s += s_eachi[r];
    __syncthreads();
    ph ^= 1;
    return s;
  };
  auto max_f = [&](float v) -> float {
    if (tid == 0) s_xf[ph] = v;
    cl.sync();
    if (tid == 0) {
      float m = -INFINITY;
      for (int r = 0; r < kC; ++r) m = fmaxf(m, *cl.map_shared_rank(&s_xf[ph], r));
      s_redf[0] = m;
    }
    __syncthreads();
    const float m = s_redf[0];
    __syncthreads();
    ph ^= 1;
    return m;
  };
  auto block_sum = [&](double v) -> double {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_redd[warp] = v;
    __syncthreads();
    double s = 0.0;
    for (int i = 0; i < kTS / 32; ++i) s += s_redd[i];
    __syncthreads();
    return s;
  };

  // ---------------------------------------------------------------- keys: the na largest logits
  uint32_t kth = 0;     // key of the na-th largest
  int tie_cut = 0;      // selected ties: key == kth at slice positions < tie_cut
  if (na > 0) {
    uint32_t prefix = 0;
    int want = na;      // rank (1-based, from the top) still to locate inside the current prefix
    for (int shift = key_bits<T>() - 8; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kTS) s_hist[i] = 0u;
      __syncthreads();
      const uint32_t hmask = shift + 8 >= 32 ? 0u : (0xffffffffu << (shift + 8));
      // warp-aggregated counting: logits crowd into a few high digits, so lanes with the same
      // digit are grouped and their leader adds the group's size
      for (int base = 0; base < cnt; base += kTS) {
        const int i = base + tid;
        int bin = -1;
        if (i < cnt) {
          const uint32_t k = okey(sZ[i]);
          if ((k & hmask) == (prefix & hmask)) bin = (int)((k >> shift) & 0xffu);
        }
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&s_hist[bin], (uint32_t)__popc(peers));
      }
      __syncthreads();
      for (int i = tid; i < 256; i += kTS) s_xh[ph][i] = s_hist[i];
      cl.sync();
      for (int i = tid; i < 256; i += kTS) {
        uint32_t t = 0;
        for (int r = 0; r < kC; ++r) t += cl.map_shared_rank(&s_xh[ph][0], r)[i];
        s_hist[i] = t;
      }
      __syncthreads();
      // digit holding the want-th largest, scanning from the top digit down
      if (tid == 0) {
        int acc = 0, d = 255;
        for (; d > 0; --d) {
          if (acc + (int)s_hist[d] >= want) break;
          acc += (int)s_hist[d];
        }
        s_digit = d;
        s_above = acc;
      }
      __syncthreads();
      prefix |= (uint32_t)s_digit << shift;
      want -= s_above;
      __syncthreads();
      ph ^= 1;
    }
    kth = prefix;
    // elements strictly above kth, then (na - above) ties in id order over the cluster
    int gt = 0, eq = 0;
    for (int i = tid; i < cnt; i += kTS) {
      const uint32_t k = okey(sZ[i]);
      gt += k > kth;
      eq += k == kth;
    }
    gt = (int)block_sum((double)gt);
    eq = (int)block_sum((double)eq);
    const int gt_all = sum_i(gt);
    int eq_before = 0;
    {   // eq counts of the lower ranks
      const int eq_all = sum_i(eq);
      (void)eq_all;
      for (int r = 0; r < rank; ++r) eq_before += s_eachi[r];
    }
    const int take = max(0, min(eq, na - gt_all - eq_before));
    // position after this CTA's take-th tie (ordered scan with ballots)
    tie_cut = 0;
    if (take > 0) {
      int seen = 0;
      for (int base = 0; base < cnt && seen < take; base += kTS) {
        const int i = base + tid;
        const bool is = i < cnt && okey(sZ[i]) == kth;
        const unsigned m = __ballot_sync(0xffffffffu, is);
        if (lane == 0) s_wcnt[warp] = __popc(m);
        __syncthreads();
        int before = seen;
        for (int w = 0; w < warp; ++w) before += s_wcnt[w];
        const int my = before + __popc(m & ((1u << lane) - 1u));
        if (is && my == take - 1) s_tok = i + 1;
        int tot = 0;
        for (int w = 0; w < kTS / 32; ++w) tot += s_wcnt[w];
        seen += tot;
        __syncthreads();
      }
      tie_cut = s_tok;
      __syncthreads();
    }
    // this CTA's selected tokens
    if (tid == 0) s_nsel = 0;
    __syncthreads();
    for (int i = tid; i < cnt; i += kTS) {
      const uint32_t k = okey(sZ[i]);
      if (k > kth || (k == kth && i < tie_cut)) {
        const int p = atomicAdd(&s_nsel, 1);
        if (p < kMaxS) s_sel_key[p] = k, s_sel_tok[p] = lo + i;
      }
    }
    cl.sync();   // every CTA's selection is complete
    if (rank == 0) {
      // gather all selections and order them by (key desc, token asc): rank by counting
      __shared__ uint32_t g_key[kMaxS];
      __shared__ int g_tok[kMaxS];
      if (tid == 0) {
        int m = 0;
        for (int r = 0; r < kC; ++r) {
          const int nr = *cl.map_shared_rank(&s_nsel, r);
          const uint32_t* kr = cl.map_shared_rank(s_sel_key, r);
          const int* tr = cl.map_shared_rank(s_sel_tok, r);
          for (int j = 0; j < nr && m < kMaxS; ++j, ++m) g_key[m] = kr[j], g_tok[m] = tr[j];
        }
        s_tok = m;
      }
      __syncthreads();
      const int m = s_tok;
      for (int j = tid; j < m; j += kTS) {
        int r = 0;
        for (int c = 0; c < m; ++c)
          r += g_key[c] > g_key[j] || (g_key[c] == g_key[j] && g_tok[c] < g_tok[j]);
        if (r < na) {
          a.key_len[(size_t)b * a.S + off + r] = row;
          a.key_tok[(size_t)b * a.S + off + r] = g_tok[j];
        }
      }
    }
    cl.sync();   // rank 0 has read every peer's selection
  }
  if (row == K) return;   // the free-token row holds keys only; no draw

  // ---------------------------------------------------------------- Saguaro draw at position row+1
  float mx = -INFINITY;
  for (int i = tid; i < cnt; i += kTS) mx = fmaxf(mx, ldf(sZ[i]));
  mx = warp_max(mx);
  if (lane == 0) s_redf[warp] = mx;
  __syncthreads();
  mx = -INFINITY;
  for (int i = 0; i < kTS / 32; ++i) mx = fmaxf(mx, s_redf[i]);
  __syncthreads();
  const float M = max_f(mx);
  const double beta = a.beta;
  auto weight = [&](int i) -> double {
    const uint32_t k = okey(sZ[i]);
    return (na > 0 && (k > kth || (k == kth && i < tie_cut))) ? beta : 1.0;
  };
  // With e = 2^((z - M) log2(e) / T): q = e / sum(e) and q' = q w / sum(q w) = e w / sum(e w), so
  // both sums come from one pass (q itself when the weighted sum is 0).
  double se = 0.0, sw = 0.0;
  for (int i = tid; i < cnt; i += kTS) {
    const double e = (double)expo(ldf(sZ[i]), M, a.thi, a.tlo);
    se += e;
    sw += e * weight(i);
  }
  double Sq, Sw;
  sum_d2(block_sum(se), block_sum(sw), Sq, Sw);
  const bool plain = !(Sw > 0.0);
  const double inv = plain ? (Sq > 0.0 ? 1.0 / Sq : 0.0) : 1.0 / Sw;
  auto qprime = [&](int i) -> double {
    const double e = (double)expo(ldf(sZ[i]), M, a.thi, a.tlo);
    return (plain ? e : e * weight(i)) * inv;
  };
  const int per = (cnt + kTS - 1) / kTS;
  const int ra = min(cnt, tid * per), re = min(cnt, ra + per);
  double run = 0.0;
  int lastp = -1;
  for (int i = ra; i < re; ++i) {
    const double x = qprime(i);
    if (x > 0.0) lastp = i;
    run += x;
  }
  double incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_redd[warp] = incl;
  __syncthreads();
  double wbase = 0.0, mass = 0.0;
  for (int i = 0; i < kTS / 32; ++i) {
    if (i < warp) wbase += s_redd[i];
    mass += s_redd[i];
  }
  s_run[tid] = wbase + incl - run;
  if (tid == 0) s_tok = INT_MAX;
  __syncthreads();
  const double total = sum_d(mass);
  const double thr = (double)a.u[(size_t)b * K + row] * total;
  int cstar = -1;
  double cum = 0.0;
  for (int r = 0; r < kC; ++r) {
    if (s_each[r] > 0.0 && cum + s_each[r] > thr) {
      cstar = r;
      break;
    }
    cum += s_each[r];
  }
  bool fallback = false;
  if (cstar < 0) {
    for (int r = kC - 1; r >= 0; --r)
      if (s_each[r] > 0.0) {
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
          c0 += qprime(i);
          if (c0 > t) {
            atomicMin(&s_tok, lo + i);
            break;
          }
        }
      }
    }
    __syncthreads();
    if (s_tok == INT_MAX) {
      __shared__ int s_last;
      if (tid == 0) s_last = -1;
      __syncthreads();
      if (lastp >= 0) atomicMax(&s_last, lo + lastp);
      __syncthreads();
      if (tid == 0) s_tok = s_last >= 0 ? s_last : 0;
      __syncthreads();
    }
    if (tid == 0) a.draft_tokens[(size_t)b * K + row] = s_tok;
  }
  cl.sync();   // no CTA leaves while a peer may still read its shared memory
}

}  // namespace

size_t ssd_cache_smem(int V, tsd_dtype dtype) {
  const size_t slice = ((size_t)(V + kC - 1) / kC + 7) / 8 * 8;
  return slice * (dtype == TSD_BF16 ? 2 : 4);
}

int ssd_cache_max_slots() { return kMaxS; }
int ssd_cache_max_k() { return kMaxK; }

tsd_status launch_ssd_cache(const void* zq, tsd_dtype dtype, int V, int K, int S, const float* alpha, float beta,
                            const float* u, float T, int B, int32_t* slots, int32_t* key_len, int32_t* key_tok,
                            int32_t* draft_tokens, cudaStream_t stream) {
  if (B == 0) return TSD_OK;
  SSDArgs a{};
  a.zq = zq, a.V = V, a.K = K, a.S = S, a.alpha = alpha, a.beta = beta, a.u = u;
  const double c = kLog2eD / (double)T;
  split_const(c, a.thi, a.tlo);
  a.slice = ((V + kC - 1) / kC + 7) / 8 * 8;
  a.vec = vec16_rows(zq, V) ? 1 : 0;
  a.slots = slots, a.key_len = key_len, a.key_tok = key_tok, a.draft_tokens = draft_tokens;
  const size_t smem = ssd_cache_smem(V, dtype);
  auto kernel = dtype == TSD_BF16 ? ssd_cache_kernel<__nv_bfloat16> : ssd_cache_kernel<float>;
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kC, K + 1, B);
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

}  // namespace tsd
