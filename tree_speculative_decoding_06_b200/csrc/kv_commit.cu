// tsd_kv_commit / tsd_kv_commit_paged: copy only the accepted path's K/V rows into the cache.
//
// "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs", technical summary
// sec. 2 (branchable KV cache): the committed prefix is kept apart from per-branch speculative
// state, and a commit either keeps the first A steps (length mode) or follows the path indices,
// moving only the rows that must move.  The speculative rows live in a separate tree buffer, so
// rows of rejected branches never reach the cache.
//
// One CTA per sequence.  All checks (miss, capacity, path range, block ids) run before any
// write, so a flagged sequence keeps its cache and prefix length untouched.  In-place mode
// compacts rows inside the cache: sources sit at or after their destinations, so rows are moved
// in ascending batches, each batch read completely into shared memory before any of it is
// written back.
#include "common.cuh"
#include "kernels.h"

namespace tsd {

namespace {

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

__global__ void __launch_bounds__(kThreads) kv_commit_kernel(const CommitArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) uint8_t s_stage[];
  __shared__ int s_src[257];
  __shared__ int s_bad;
  const int b = blockIdx.x;
  const int A = a.accept_len[b];
  if (a.status[b] != 0 || A < 0) return;
  const int N = a.num_nodes ? a.num_nodes[b] : a.Nmax;
  const int L = a.prefix_len[b];
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  if (A > a.Dmax || A >= N || N > a.Nmax) {
    if (threadIdx.x == 0) flag_status(a.status, b, TSD_ERR_INVALID_ARG);
    return;
  }
  if (L < 0 || (long long)L + A + 1 > a.Lcap) {
    if (threadIdx.x == 0) flag_status(a.status, b, TSD_ERR_CAPACITY);
    return;
  }
  // source node of every committed row
  for (int j = threadIdx.x; j <= A; j += blockDim.x) {
    const int node = a.mode == TSD_COMMIT_LENGTH ? j : a.path[(size_t)b * (a.Dmax + 1) + j] - 1;
    if (node < 0 || node >= N) atomicOr(&s_bad, 1);
    s_src[j] = node;
  }
  // block ids of every touched cache position (destinations, and in-place sources)
  if (a.block_table) {
    const int hi = a.mode == TSD_COMMIT_INPLACE ? L + N : L + A + 1;
    if ((long long)hi > a.Lcap) {
      if (a.mode == TSD_COMMIT_INPLACE && threadIdx.x == 0) atomicOr(&s_bad, 2);
    } else {
      for (int p = (L >> a.block_shift) + threadIdx.x; p <= ((hi - 1) >> a.block_shift); p += blockDim.x) {
        const int blk = a.block_table[(size_t)b * a.max_blocks + p];
        if (blk < 0 || blk >= a.num_blocks) atomicOr(&s_bad, 2);
      }
    }
  } else if (a.mode == TSD_COMMIT_INPLACE && (long long)L + N > a.Lcap) {
    if (threadIdx.x == 0) atomicOr(&s_bad, 2);
  }
  __syncthreads();
  if (s_bad) {
    if (threadIdx.x == 0) flag_status(a.status, b, (s_bad & 1) ? TSD_ERR_INVALID_ARG : TSD_ERR_CAPACITY);
    return;
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
}

}  // namespace

tsd_status launch_kv_commit(const CommitArgs& a, cudaStream_t stream) {
  if (a.B == 0) return TSD_OK;
  size_t smem = 0;
  if (a.mode == TSD_COMMIT_INPLACE) {
    const size_t row_bytes = (size_t)a.d * a.esize * a.Hkv * 2;
    smem = row_bytes > (size_t)kStageBytes ? row_bytes : (size_t)kStageBytes;
    if (smem > 200 * 1024) return TSD_ERR_INVALID_ARG;   // one row of every head must fit on chip
    if (smem > 48 * 1024) cudaFuncSetAttribute(kv_commit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  }
  return launch_pdl(kv_commit_kernel, dim3(a.B), dim3(kThreads), smem, stream, a) == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

}  // namespace tsd
