// tsd_kv_commit / tsd_kv_commit_paged: copy only the accepted path's K/V rows into the cache.
//
// "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs", technical summary
// sec. 2 (branchable KV cache): the committed prefix is kept apart from per-branch speculative
// state, and a commit either keeps the first A steps (length mode) or follows the path indices,
// moving only the rows that must move.  The speculative rows live in a separate tree buffer, so
// rows of rejected branches never reach the cache.
//
// One CTA per sequence; the per-sequence body (checks before any write, in-place staging) is in
// commit_body.cuh.
#include "commit_body.cuh"

namespace tsd {

namespace {

__global__ void __launch_bounds__(commit::kThreads) kv_commit_kernel(const CommitArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) uint8_t s_stage[];
  const int b = blockIdx.x;
  const int A = a.accept_len[b];
  const int st = a.status[b];
  const int N = a.num_nodes ? a.num_nodes[b] : a.Nmax;
  const int L = a.prefix_len[b];
  if (st != 0 || A < 0) return;
  commit::commit_block(a, b, A, N, L, a.path ? a.path + (size_t)b * (a.Dmax + 1) : nullptr, s_stage);
}

}  // namespace

tsd_status launch_kv_commit(const CommitArgs& a, cudaStream_t stream) {
  if (a.B == 0) return TSD_OK;
  size_t smem = 0;
  if (a.mode == TSD_COMMIT_INPLACE) {
    const size_t row_bytes = (size_t)a.d * a.esize * a.Hkv * 2;
    smem = row_bytes > (size_t)commit::kStageBytes ? row_bytes : (size_t)commit::kStageBytes;
    if (smem > 200 * 1024) return TSD_ERR_INVALID_ARG;   // one row of every head must fit on chip
    if (smem > 48 * 1024) cudaFuncSetAttribute(kv_commit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  }
  return launch_pdl(kv_commit_kernel, dim3(a.B), dim3(commit::kThreads), smem, stream, a) == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

}  // namespace tsd
