// tsd_tree_accept_commit: greedy tree acceptance and the commit of the accepted path in one
// kernel, with an optional splice of the emitted tokens into a device-resident token history.
//
// "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs", technical summary
// sec. 2 (branchable KV cache: commit follows the accepted path) and "Acelerando Sonar a traves
// de la especulacion", section "EAGLE" (longest target-matching branch plus one target token):
// the same acceptance and the same commit as tsd_tree_accept_greedy followed by tsd_kv_commit,
// but the path never leaves the CTA that found it.  Accepted lengths drive the cache length and
// the token history on the device, so a decoding loop needs no host round trip per step.
//
// Launches: the vocabulary argmax scan (many CTAs, HBM-bound), then one CTA per sequence that
// merges the scan, picks the deepest accepted node, copies its path's K/V rows into the cache,
// advances prefix_len and appends the emitted tokens to the history.
#include "accept_body.cuh"
#include "commit_body.cuh"

namespace tsd {

namespace {

__host__ __device__ inline int tstar_bytes(int Nmax) { return ((Nmax > 0 ? Nmax : 1) * 4 + 15) & ~15; }
// staging of the tree's parent slots and tokens for the acceptance walks (2 Nmax + 1 ints), then
// of the argmax partials (Nmax x chunks float2)
__host__ __device__ inline int tree_stage_bytes(int Nmax) { return ((2 * Nmax + 1) * 4 + 15) & ~15; }
__host__ __device__ inline int part_stage_bytes(int Nmax, int chunks) { return (Nmax * chunks * 8 + 15) & ~15; }

__global__ void __launch_bounds__(commit::kThreads) accept_commit_kernel(
    const float2* __restrict__ part, int chunks, const int32_t* __restrict__ tokens,
    const int32_t* __restrict__ parent_s, const int32_t* __restrict__ root_key, int32_t* __restrict__ accept_len,
    int32_t* __restrict__ path, int32_t* __restrict__ out_tokens, const CommitArgs a, const SpliceArgs sp,
    int staged) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int32_t s_path[256];
  int32_t* s_tstar = reinterpret_cast<int32_t*>(smem);
  int32_t* s_tree = staged ? reinterpret_cast<int32_t*>(smem + tstar_bytes(a.Nmax)) : nullptr;
  float2* s_part = staged ? reinterpret_cast<float2*>(smem + tstar_bytes(a.Nmax) + tree_stage_bytes(a.Nmax)) : nullptr;
  uint8_t* s_stage = smem + tstar_bytes(a.Nmax) +
                     (staged ? tree_stage_bytes(a.Nmax) + part_stage_bytes(a.Nmax, chunks) : 0);
  const int b = blockIdx.x;
  const int L = a.prefix_len[b];   // read now: its latency overlaps the acceptance
  const int A = acc::tree_accept_block(part, chunks, tokens, parent_s, a.num_nodes, root_key, a.Nmax, a.Dmax,
                                       a.status, accept_len, path, out_tokens, s_tstar, s_path, s_tree, s_part);
  if (A < 0) return;   // a miss, or a flagged sequence: nothing to commit
  int h0 = 0;
  if (sp.history) {
    h0 = sp.history_len[b];
    if (h0 < 0 || (long long)h0 + A + 1 > sp.cap) {
      if (threadIdx.x == 0) flag_status(a.status, b, TSD_ERR_CAPACITY);
      return;
    }
  }
  if (!commit::commit_block(a, b, A, a.num_nodes ? a.num_nodes[b] : a.Nmax, L, s_path, s_stage)) return;
  if (sp.history && threadIdx.x == 0) {
    const int32_t* orow = out_tokens + (size_t)b * (a.Dmax + 1);   // written by this thread above
    int32_t* hrow = sp.history + (size_t)b * sp.cap;
    for (int k = 0; k <= A; ++k) hrow[h0 + k] = orow[k];
    sp.history_len[b] = h0 + A + 1;
  }
}

}  // namespace

tsd_status launch_accept_commit(const void* logits, tsd_dtype dtype, int V, const int32_t* tokens,
                                const int32_t* parent_s, const int32_t* root_key, int32_t* accept_len,
                                int32_t* path, int32_t* out_tokens, const CommitArgs& a, const SpliceArgs& sp,
                                void* ws, cudaStream_t stream) {
  if (a.B == 0) return TSD_OK;
  size_t smem = (size_t)tstar_bytes(a.Nmax);
  const size_t stage = (size_t)tree_stage_bytes(a.Nmax) + part_stage_bytes(a.Nmax, argmax_chunks(V));
  const int staged = smem + stage <= 96 * 1024 ? 1 : 0;
  if (staged) smem += stage;
  if (a.mode == TSD_COMMIT_INPLACE) {
    const size_t row_bytes = (size_t)a.d * a.esize * a.Hkv * 2;
    smem += row_bytes > (size_t)commit::kStageBytes ? row_bytes : (size_t)commit::kStageBytes;
  }
  if (smem > 200 * 1024) return TSD_ERR_INVALID_ARG;
  if (launch_row_argmax(logits, dtype, V, a.Nmax, a.num_nodes, a.B, ws, stream) != TSD_OK) return TSD_ERR_CUDA;
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(accept_commit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch_pdl(accept_commit_kernel, dim3(a.B), dim3(commit::kThreads), smem, stream, (const float2*)ws,
             argmax_chunks(V), tokens, parent_s, root_key, accept_len, path, out_tokens, a, sp, staged);
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

}  // namespace tsd
