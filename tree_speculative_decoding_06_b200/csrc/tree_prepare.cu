// tsd_tree_prepare: validate each draft tree and build its shifted-index tables.
//
// "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs", technical summary
// sec. 2 (accelerator-safe tree tensor semantics): the root's -1 placeholder becomes a dummy row
// 0 so every gather index is valid, ancestor index tables are built for structured gathers, and
// range / acyclicity / depth-consistency checks run before the fused kernels launch.
//
// One CTA per sequence; one thread per node.  Each node's check depends only on its own parent
// and its ancestors, so the first offending node (smallest index) is found with an atomicMin on
// (node << 4 | code): if every node below it is valid, its own verdict is exact.  The parent
// array is first copied into shared memory with one coalesced read (when it fits), so the
// ancestor walks are chains of shared-memory loads rather than of dependent global loads.
#include "common.cuh"
#include "kernels.h"

namespace tsd {

__global__ void tree_prepare_kernel(const int32_t* __restrict__ parent, const int32_t* __restrict__ num_nodes,
                                    int Nmax, int Dmax, int forest, int32_t* __restrict__ parent_s,
                                    int32_t* __restrict__ depth_s, int32_t* __restrict__ anc,
                                    uint32_t* __restrict__ anc_bits, int32_t* __restrict__ status, int staged) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int32_t s_par[];
  const int b = blockIdx.x;
  const int N = num_nodes ? num_nodes[b] : Nmax;
  const int32_t* par = parent + (size_t)b * Nmax;
  if (staged) {   // all Nmax entries (in bounds whatever N is): the copy need not wait for N
    for (int i = threadIdx.x; i < Nmax; i += blockDim.x) s_par[i] = par[i];
    par = s_par;   // made visible by the __syncthreads below
  }
  const int S = Nmax + 1;                  // slots per sequence
  const int AW = Dmax + 1;                 // ancestor-table width
  const int W = (S + 31) >> 5;             // ancestor-bit words per slot
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = INT_MAX;
  __syncthreads();

  const bool n_ok = (N >= 0 && N <= Nmax);
  if (n_ok) {
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
      const int p = par[i];
      int code = 0;
      if (p < -1 || p >= i) {
        code = TSD_ERR_BAD_TREE;
      } else if (p == -1) {
        if (!forest && i > 0) code = TSD_ERR_TREE_ROOTS;
      } else {
        int d = 1, s = p;
        bool walk_ok = true;
        while (d <= Dmax) {
          const int ps = par[s];
          if (ps == -1) break;
          if (ps < -1 || ps >= s) { walk_ok = false; break; }  // a lower node carries the error
          s = ps;
          ++d;
        }
        if (walk_ok && d > Dmax) code = TSD_ERR_TREE_DEPTH;
      }
      if (code) atomicMin(&s_bad, (i << 4) | code);
    }
  }
  __syncthreads();
  const int bad = s_bad;
  const bool ok = n_ok && bad == INT_MAX;
  if (threadIdx.x == 0) {
    if (!n_ok)
      status[b] = TSD_ERR_INVALID_ARG;
    else if (!ok)
      status[b] = (bad & 15) | ((bad >> 4) << 8);
    else
      status[b] = 0;
  }

  int32_t* ps_out = parent_s + (size_t)b * S;
  int32_t* d_out = depth_s + (size_t)b * S;
  int32_t* a_out = anc + (size_t)b * S * AW;
  uint32_t* bits_out = anc_bits ? anc_bits + (size_t)b * S * W : nullptr;
  for (int s = threadIdx.x; s < S; s += blockDim.x) {
    const int i = s - 1;
    int32_t* arow = a_out + (size_t)s * AW;
    uint32_t* brow = bits_out ? bits_out + (size_t)s * W : nullptr;
    if (brow)
      for (int w = 0; w < W; ++w) brow[w] = 0u;
    if (!ok || s == 0 || i >= N) {
      ps_out[s] = 0;
      d_out[s] = 0;
      for (int k = 0; k < AW; ++k) arow[k] = 0;
      continue;
    }
    // depth by walking up (valid tree: terminates within Dmax steps)
    int d = 0;
    for (int j = par[i]; j >= 0; j = par[j]) ++d;
    ps_out[s] = par[i] + 1;
    d_out[s] = d;
    for (int k = d + 1; k < AW; ++k) arow[k] = 0;
    int k = d;
    for (int j = i; j >= 0; j = par[j], --k) {
      arow[k] = j + 1;
      if (brow) brow[(j + 1) >> 5] |= 1u << ((j + 1) & 31);
    }
  }
}

tsd_status launch_tree_prepare(const int32_t* parent, const int32_t* num_nodes, int B, int Nmax, int Dmax,
                               int forest, int32_t* parent_s, int32_t* depth, int32_t* anc, uint32_t* anc_bits,
                               int32_t* status, cudaStream_t stream) {
  if (B == 0) return TSD_OK;
  const int threads = Nmax + 1 >= 256 ? 256 : ((Nmax + 1 + 31) / 32) * 32;
  const size_t smem = (size_t)Nmax * sizeof(int32_t);
  const int staged = smem <= 48 * 1024 ? 1 : 0;
  if (launch_pdl(tree_prepare_kernel, dim3(B), dim3(threads), staged ? smem : 0, stream, parent, num_nodes, Nmax, Dmax,
                 forest, parent_s, depth, anc, anc_bits, status, staged) != cudaSuccess)
    return TSD_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

}  // namespace tsd
