// Greedy acceptance of one draft tree by one CTA, shared by tsd_tree_accept_greedy and the fused
// acceptance + commit kernel.
//
// "Acelerando Sonar a traves de la especulacion", section "EAGLE": over a tree, the target keeps
// the longest branch whose every token equals the target's own next token, then adds one token of
// its own; "Speculative Speculative Decoding", technical summary sec. 2: in a forest, the real
// outcome token selects the subtree (a miss accepts nothing).
#pragma once

#include <climits>

#include "common.cuh"

namespace tsd {
namespace acc {

// Merge of the per-chunk (value, index) argmax partials of one row (ties -> lower index).
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

// Warp-parallel merge of the chunk partials of rows [0, n) held in shared memory (chunks <= 32):
// one row per warp at a time, lane c holds chunk c, a shuffle tree keeps the best (ties -> lower
// index).  Writes s_tstar[row].
__device__ __forceinline__ void merge_rows_warp(const float2* s_part, int chunks, int n, int32_t* s_tstar) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int r = warp; r < n; r += nw) {
    float bv = -INFINITY;
    int bi = INT_MAX;
    if (lane < chunks) {
      const float2 p = s_part[(size_t)r * chunks + lane];
      bv = p.x, bi = __float_as_int(p.y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (better(ov, oi, bv, bi)) bv = ov, bi = oi;
    }
    if (lane == 0) s_tstar[r] = bi == INT_MAX ? 0 : bi;
  }
}

// Acceptance of sequence b by the whole CTA.  s_tstar holds >= Nmax ints of shared memory
// (already filled when tstar_ready); match, if not null, holds one byte per node: edge
// parent(i) -> i passes iff match[i] != 0, instead of the greedy token test;
// s_stage, if not null, >= 2 * Nmax + 1 more, into which the tree's parent slots and tokens are
// copied first (one coalesced read each) so that the ancestor walks run on shared memory;
// s_part, if not null, holds Nmax * chunks float2: every row's argmax partials are read into it
// at once (one round trip to memory instead of one per chunk) before the rows are merged.
// Writes accept_len[b], the path row (slots root..a*, 0 beyond) and the emitted tokens (the
// accepted drafts below the root, then the target's token at a*, -1 beyond), leaves the path
// slots in s_path[0..A] and returns A to every thread (-1: a forest miss, or a sequence that is
// flagged / empty, whose outputs are then the miss outputs).
__device__ __forceinline__ int tree_accept_block(const float2* __restrict__ part, int chunks,
                                                 const int32_t* __restrict__ tokens,
                                                 const int32_t* __restrict__ parent_s,
                                                 const int32_t* __restrict__ num_nodes,
                                                 const int32_t* __restrict__ root_key, int Nmax, int Dmax,
                                                 const int32_t* __restrict__ status, int32_t* __restrict__ accept_len,
                                                 int32_t* __restrict__ path, int32_t* __restrict__ out_tokens,
                                                 int32_t* s_tstar, int32_t* s_path, int32_t* s_stage,
                                                 float2* s_part, const uint8_t* match = nullptr,
                                                 bool tstar_ready = false) {
  __shared__ int s_hit, s_best, s_A;
  const int b = blockIdx.x;
  const int N = num_nodes ? num_nodes[b] : Nmax;
  const int32_t* tok = tokens + (size_t)b * Nmax;
  const int32_t* ps = parent_s + (size_t)b * (Nmax + 1);
  int32_t* prow = path + (size_t)b * (Dmax + 1);
  int32_t* orow = out_tokens + (size_t)b * (Dmax + 1);
  const bool live = status[b] == 0 && N > 0 && N <= Nmax;
  // the staging reads cover all Nmax rows (in bounds whatever N is), so they are issued together
  // with the reads of N and the status instead of after them
  if (s_stage != nullptr) {   // visible after the __syncthreads below
    for (int i = threadIdx.x; i <= Nmax; i += blockDim.x) s_stage[i] = ps[i];
    for (int i = threadIdx.x; i < Nmax; i += blockDim.x) s_stage[Nmax + 1 + i] = tok[i];
    ps = s_stage;
    tok = s_stage + Nmax + 1;
  }
  if (threadIdx.x == 0) s_hit = INT_MAX, s_best = -1;
  if (tstar_ready) {
    // the caller filled s_tstar[0..N) (visible after the __syncthreads below)
  } else if (s_part != nullptr) {
    const float2* src = part + (size_t)b * Nmax * chunks;
    for (int k = threadIdx.x; k < Nmax * chunks; k += blockDim.x) s_part[k] = src[k];
    __syncthreads();
    if (chunks <= 32) {
      if (live) merge_rows_warp(s_part, chunks, N, s_tstar);
    } else {
      for (int i = threadIdx.x; live && i < N; i += blockDim.x)
        s_tstar[i] = merge_argmax(s_part + (size_t)i * chunks, chunks);
    }
  } else {
    for (int i = threadIdx.x; live && i < N; i += blockDim.x)
      s_tstar[i] = merge_argmax(part + ((size_t)b * Nmax + i) * chunks, chunks);
  }
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
      // greedy: the token is the parent's argmax; with a match table (threshold acceptance) the
      // caller decided every edge
      ok = ok && (match ? match[s - 1] != 0 : tok[s - 1] == s_tstar[p - 1]);
      s = p;
      ++d;
      if (!ok) break;
    }
    if (ok) atomicMax(&s_best, (d << 20) | (0xFFFFF - i));
  }
  __syncthreads();
  // thread 0 walks the path into shared memory; then every thread writes its entries
  if (threadIdx.x == 0) {
    const int best = live ? s_best : -1;
    if (best < 0) {
      s_A = -1;
    } else {
      const int A = best >> 20, astar = 0xFFFFF - (best & 0xFFFFF);
      int s = astar + 1;
      for (int k = A; k >= 0; --k) {
        s_path[k] = s;
        s = ps[s];
      }
      s_A = A;
    }
  }
  __syncthreads();
  const int A = s_A;
  if (threadIdx.x == 0) accept_len[b] = A;
  for (int k = threadIdx.x; k <= Dmax; k += blockDim.x) {
    if (k <= A) {
      prow[k] = s_path[k];
      orow[k] = k < A ? tok[s_path[k + 1] - 1] : s_tstar[s_path[A] - 1];
    } else {
      prow[k] = 0;
      orow[k] = -1;
    }
  }
  return A;
}

}  // namespace acc
}  // namespace tsd
