// Commit of one sequence's accepted rows by one CTA, shared by tsd_kv_commit[_paged] and the
// fused acceptance + commit kernel.
//
// "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs", technical summary
// sec. 2 (branchable KV cache): only the rows of the accepted path reach the cache.
//
// All checks (capacity, path range, block ids) run before any write, so a flagged sequence keeps
// its cache and prefix length untouched.  In-place mode compacts rows inside the cache: sources
// sit at or after their destinations, so rows are moved in ascending batches, each batch read
// completely into shared memory before any of it is written back.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace tsd {
namespace commit {

constexpr int kThreads = 256;
constexpr int kStageBytes = 32 * 1024;

__device__ __forceinline__ size_t row_off(const CommitArgs& a, int b, int h, int pos, bool& ok) {
  const size_t row_elems = (size_t)a.d;
  if (a.block_table == nullptr) return ((((size_t)b * a.Hkv + h) * a.Lcap) + pos) * row_elems;
  int blk = a.block_table[(size_t)b * a.max_blocks + (pos >> a.block_shift)];
  if (blk < 0 || blk >= a.num_blocks) {
    ok = false;
    blk = 0;
  }
  const int off = pos & ((1 << a.block_shift) - 1);
  return ((((size_t)blk * a.Hkv + h) << a.block_shift) + off) * row_elems;
}

// Items (16-byte chunks of one K row and one V row) a thread holds in registers in the gather copy.
constexpr int kRegItems = 8;
constexpr int kMaxDstBlocks = 40;   // blocks spanned by Dmax + 1 <= 256 rows of block size >= 8

// Commits rows 0..A of sequence b (A >= 0), N = num_nodes[b] (or Nmax), L = prefix_len[b] as
// the caller read them.  path_row: the A+1 path slots (global or shared memory; unused in LENGTH
// mode).  s_stage: the in-place staging buffer (kStageBytes, or one row of every head if larger).
// Returns true iff the rows were written and prefix_len[b] advanced; false after flagging
// status[b].  Every thread of the CTA must call it.
__device__ __forceinline__ bool commit_block(const CommitArgs& a, int b, int A, int N, int L, const int32_t* path_row,
                                             uint8_t* s_stage) {
  __shared__ int s_src[257];
  __shared__ int s_blk[kMaxDstBlocks];
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  if (A > a.Dmax || A >= N || N > a.Nmax) {
    if (threadIdx.x == 0) flag_status(a.status, b, TSD_ERR_INVALID_ARG);
    return false;
  }
  if (L < 0 || (long long)L + A + 1 > a.Lcap) {
    if (threadIdx.x == 0) flag_status(a.status, b, TSD_ERR_CAPACITY);
    return false;
  }
  // source node of every committed row
  for (int j = threadIdx.x; j <= A; j += blockDim.x) {
    const int node = a.mode == TSD_COMMIT_LENGTH ? j : path_row[j] - 1;
    if (node < 0 || node >= N) atomicOr(&s_bad, 1);
    s_src[j] = node;
  }
  // block ids of every touched cache position (destinations, and in-place sources)
  if (a.block_table) {
    const int hi = a.mode == TSD_COMMIT_INPLACE ? L + N : L + A + 1;
    if ((long long)hi > a.Lcap) {
      if (a.mode == TSD_COMMIT_INPLACE && threadIdx.x == 0) atomicOr(&s_bad, 2);
    } else {
      const int p0 = L >> a.block_shift;
      for (int p = p0 + threadIdx.x; p <= ((hi - 1) >> a.block_shift); p += blockDim.x) {
        const int blk = a.block_table[(size_t)b * a.max_blocks + p];
        if (blk < 0 || blk >= a.num_blocks) atomicOr(&s_bad, 2);
        if (p - p0 < kMaxDstBlocks) s_blk[p - p0] = blk;   // destination blocks, kept for the copy
      }
    }
  } else if (a.mode == TSD_COMMIT_INPLACE && (long long)L + N > a.Lcap) {
    if (threadIdx.x == 0) atomicOr(&s_bad, 2);
  }
  __syncthreads();
  if (s_bad) {
    if (threadIdx.x == 0) flag_status(a.status, b, (s_bad & 1) ? TSD_ERR_INVALID_ARG : TSD_ERR_CAPACITY);
    return false;
  }
  const int es = a.esize;
  const int CH = a.d * es / 16;            // 16-byte chunks per row
  uint8_t* kc = reinterpret_cast<uint8_t*>(a.k_cache);
  uint8_t* vc = reinterpret_cast<uint8_t*>(a.v_cache);
  bool ok = true;
  if (a.mode != TSD_COMMIT_INPLACE) {
    const uint8_t* kt = reinterpret_cast<const uint8_t*>(a.k_tree);
    const uint8_t* vt = reinterpret_cast<const uint8_t*>(a.v_tree);
    const int total = (A + 1) * a.Hkv * CH;
    const int p0 = L >> a.block_shift;
    const bool blk_ok = a.block_table == nullptr || ((L + A) >> a.block_shift) - p0 < kMaxDstBlocks;
    if (total <= kRegItems * (int)blockDim.x && blk_ok) {
      // gather: every source chunk is loaded before any is stored, so the loads of a thread
      // are in flight together (one round trip to memory instead of one per chunk)
      uint4 kr[kRegItems], vr[kRegItems];
#pragma unroll
      for (int r = 0; r < kRegItems; ++r) {
        const int idx = threadIdx.x + r * blockDim.x;
        if (idx < total) {
          const int ch = idx % CH, h = (idx / CH) % a.Hkv, j = idx / (CH * a.Hkv);
          const size_t src = ((((size_t)b * a.Nmax + s_src[j]) * a.Hkv + h) * a.d) * es + (size_t)ch * 16;
          kr[r] = *reinterpret_cast<const uint4*>(kt + src);
          vr[r] = *reinterpret_cast<const uint4*>(vt + src);
        }
      }
#pragma unroll
      for (int r = 0; r < kRegItems; ++r) {
        const int idx = threadIdx.x + r * blockDim.x;
        if (idx < total) {
          const int ch = idx % CH, h = (idx / CH) % a.Hkv, j = idx / (CH * a.Hkv);
          const int pos = L + j;
          size_t row;
          if (a.block_table == nullptr) {
            row = (((size_t)b * a.Hkv + h) * a.Lcap) + pos;
          } else {
            const int blk = s_blk[(pos >> a.block_shift) - p0];
            row = (((size_t)blk * a.Hkv + h) << a.block_shift) + (pos & ((1 << a.block_shift) - 1));
          }
          const size_t dst = row * a.d * es + (size_t)ch * 16;
          *reinterpret_cast<uint4*>(kc + dst) = kr[r];
          *reinterpret_cast<uint4*>(vc + dst) = vr[r];
        }
      }
    } else
    for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
      const int ch = idx % CH, h = (idx / CH) % a.Hkv, j = idx / (CH * a.Hkv);
      const size_t src = ((((size_t)b * a.Nmax + s_src[j]) * a.Hkv + h) * a.d) * es + (size_t)ch * 16;
      const size_t dst = row_off(a, b, h, L + j, ok) * es + (size_t)ch * 16;
      *reinterpret_cast<uint4*>(kc + dst) = *reinterpret_cast<const uint4*>(kt + src);
      *reinterpret_cast<uint4*>(vc + dst) = *reinterpret_cast<const uint4*>(vt + src);
    }
  } else {
    // rows per batch so that K and V of every head of the batch fit the staging buffer
    const int row_bytes = a.d * es * a.Hkv * 2;
    int per = kStageBytes / row_bytes;
    if (per < 1) per = 1;
    uint4* st = reinterpret_cast<uint4*>(s_stage);
    for (int j0 = 0; j0 <= A; j0 += per) {
      const int j1 = min(A + 1, j0 + per);
      const int total = (j1 - j0) * a.Hkv * CH;
      for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
        const int ch = idx % CH, h = (idx / CH) % a.Hkv, j = j0 + idx / (CH * a.Hkv);
        if (s_src[j] == j) continue;     // already in place
        const size_t src = row_off(a, b, h, L + s_src[j], ok) * es + (size_t)ch * 16;
        st[2 * idx] = *reinterpret_cast<const uint4*>(kc + src);
        st[2 * idx + 1] = *reinterpret_cast<const uint4*>(vc + src);
      }
      __syncthreads();
      for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
        const int ch = idx % CH, h = (idx / CH) % a.Hkv, j = j0 + idx / (CH * a.Hkv);
        if (s_src[j] == j) continue;
        const size_t dst = row_off(a, b, h, L + j, ok) * es + (size_t)ch * 16;
        *reinterpret_cast<uint4*>(kc + dst) = st[2 * idx];
        *reinterpret_cast<uint4*>(vc + dst) = st[2 * idx + 1];
      }
      __syncthreads();
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) a.prefix_len[b] = L + A + 1;
  return true;
}

}  // namespace commit
}  // namespace tsd
