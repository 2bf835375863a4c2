// Device helpers shared by the attention kernels (mma.sync / FFMA paths in attn.cu and the
// tcgen05 path in attn_umma.cu): the per-sequence view, key addressing, ancestor-bit masks.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace tsd {
namespace attn {

// Per-CTA view of one sequence: lengths, tile ranges and the early-exit verdicts.
struct SeqView {
  int N, R, L, nPT, T, nsplit;
  bool skip, zero;   // skip: nothing to do; zero: write zeros (flagged / out of capacity)
  bool cap;          // out of capacity (decided by the inputs alone, unlike the status word)
};

__device__ __forceinline__ SeqView seq_view(const AttnArgs& a, int b, int G, int BN, int tps) {
  SeqView v;
  v.N = a.num_nodes ? a.num_nodes[b] : a.Nmax;
  v.skip = (v.N <= 0 || v.N > a.Nmax);
  v.R = G * v.N;
  v.L = a.prefix_len[b];
  const bool in_cache = (a.k_tree == nullptr);
  const bool cap_bad = (v.L < 0) || ((long long)v.L + (in_cache ? v.N : 0) > a.Lcap);
  v.cap = cap_bad;
  v.zero = cap_bad || (a.status[b] != 0);
  v.nPT = cap_bad ? 0 : (v.L + BN - 1) / BN;
  v.T = v.nPT + (v.N + BN - 1) / BN;
  v.nsplit = (v.T + tps - 1) / tps;
  return v;
}

// Element offset of cache row `pos` of KV head g of sequence b; ok=false on a bad block id.
__device__ __forceinline__ size_t cache_row(const AttnArgs& a, int b, int g, int pos, bool& ok) {
  if (a.block_table == nullptr) return (((size_t)b * a.Hkv + g) * a.Lcap + pos) * a.d;
  int blk = a.block_table[(size_t)b * a.max_blocks + (pos >> a.block_shift)];
  if (blk < 0 || blk >= a.num_blocks) {
    ok = false;
    blk = 0;
  }
  const int off = pos & ((1 << a.block_shift) - 1);
  return ((((size_t)blk * a.Hkv + g) << a.block_shift) + off) * a.d;
}

// Element offset (into k/v_cache or k/v_tree) of key `c` of tile t; sets from_tree.
__device__ __forceinline__ size_t key_row(const AttnArgs& a, const SeqView& v, int b, int g, int t, int BN,
                                          int c, bool& valid, bool& from_tree, bool& ok) {
  if (t < v.nPT) {
    const int k = t * BN + c;
    valid = k < v.L;
    from_tree = false;
    return valid ? cache_row(a, b, g, k, ok) : 0;
  }
  const int j = (t - v.nPT) * BN + c;
  valid = j < v.N;
  if (a.k_tree == nullptr) {
    from_tree = false;
    return valid ? cache_row(a, b, g, v.L + j, ok) : 0;
  }
  from_tree = true;
  return valid ? (((size_t)b * a.Nmax + j) * a.Hkv + g) * a.d : 0;
}

// Ancestor bits of the CTA's nodes i_lo..i_lo+cnt-1 over tree nodes, one row of W words each.
// Rows of nodes at or past N (padding of the last row tile) are left zero and never walked.
__device__ __forceinline__ void build_mask(const AttnArgs& a, int b, int i_lo, int cnt, int W, uint32_t* smask,
                                           int N, int t0 = -1, int tstride = 0) {
  const int32_t* ps = a.parent_s + (size_t)b * (a.Nmax + 1);
  if (t0 < 0) t0 = threadIdx.x, tstride = blockDim.x;
  for (int n = t0; n < cnt; n += tstride) {
    uint32_t* row = smask + (size_t)n * W;
    for (int w = 0; w < W; ++w) row[w] = 0u;
    if (i_lo + n >= N) continue;
    int s = i_lo + n + 1;
    for (int step = 0; step <= a.Dmax && s != 0; ++step) {
      const int j = s - 1;
      row[j >> 5] |= 1u << (j & 31);
      const int p = ps[s];
      if (p >= s || p < 0) break;   // prepare rejects such trees; never walk upward-out-of-range
      s = p;
    }
  }
}

// build_mask by one warp from a shared-memory copy of the sequence's parent slots (s_ps holds
// N + 1 ints): one coalesced read, then the ancestor walks are chains of shared-memory loads.
__device__ __forceinline__ void build_mask_staged(const AttnArgs& a, int b, int i_lo, int cnt, int W, uint32_t* smask,
                                                  int N, int32_t* s_ps, int lane) {
  const int32_t* ps = a.parent_s + (size_t)b * (a.Nmax + 1);
  for (int s = lane; s <= N; s += 32) s_ps[s] = ps[s];
  __syncwarp();
  for (int n = lane; n < cnt; n += 32) {
    uint32_t* row = smask + (size_t)n * W;
    for (int w = 0; w < W; ++w) row[w] = 0u;
    if (i_lo + n >= N) continue;
    int s = i_lo + n + 1;
    for (int step = 0; step <= a.Dmax && s != 0; ++step) {
      const int j = s - 1;
      row[j >> 5] |= 1u << (j & 31);
      const int p = s_ps[s];
      if (p >= s || p < 0) break;   // prepare rejects such trees; never walk upward-out-of-range
      s = p;
    }
  }
}

template <typename OutT>
__device__ __forceinline__ void store_out(OutT* o, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* o, float v) { *o = v; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* o, float v) { *o = __float2bfloat16_rn(v); }

// Zero the output (and lse) rows [r_lo, r_hi) of (b, g).
template <typename OutT>
__device__ void zero_rows(const AttnArgs& a, int b, int g, int G, int r_lo, int r_hi) {
  OutT* out = reinterpret_cast<OutT*>(a.out);
  const int D = a.d;
  for (int idx = threadIdx.x; idx < (r_hi - r_lo) * D; idx += blockDim.x) {
    const int r = r_lo + idx / D, c = idx % D;
    const int i = r / G, hh = r % G;
    store_out(out + (((size_t)b * a.Nmax + i) * a.Hq + g * G + hh) * D + c, 0.f);
  }
  if (a.lse)
    for (int r = r_lo + threadIdx.x; r < r_hi; r += blockDim.x) {
      const int i = r / G, hh = r % G;
      a.lse[((size_t)b * a.Nmax + i) * a.Hq + g * G + hh] = 0.f;
    }
}


}  // namespace attn
}  // namespace tsd
