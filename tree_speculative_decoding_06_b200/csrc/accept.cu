// tsd_tree_accept_greedy and tsd_chain_accept_sample.
//
// Greedy: "Acelerando Sonar a traves de la especulacion", section "Decodificacion especulativa"
// (the longest accepted prefix is kept and the target supplies one more token, so n drafts give
// up to n+1 tokens) and section "EAGLE" (over a tree, the longest suitable branch continues);
// "Speculative Speculative Decoding", technical summary sec. 2 (a forest of pre-drafted outcomes
// is hit or missed by the real verify outcome).
// The stochastic chain sampler (temperature > 0) lives in chain_sample.cu; the greedy chain
// (temperature 0) is an argmax test and shares the argmax scan below.
//
// Both scan the vocabulary, which is the HBM-bound part: the scans are split into chunks of
// kChunk tokens over many CTAs (16-byte loads), and small per-sequence kernels merge the chunk
// results.
#include <climits>
#include <mutex>

#include "accept_body.cuh"
#include "common.cuh"
#include "kernels.h"

namespace tsd {

namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 8192;          // vocab entries per scan CTA
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ inline int num_chunks(int V) { return (V + kChunk - 1) / kChunk; }

// Block-wide argmax (value, index; NaN never wins, ties -> lower index).
__device__ __forceinline__ void block_argmax(float& bv, int& bi) {
  __shared__ float sv[kThreads / 32];
  __shared__ int si[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (better(ov, oi, bv, bi)) bv = ov, bi = oi;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sv[warp] = bv, si[warp] = bi;
  __syncthreads();
  if (warp == 0) {
    bv = lane < (int)(blockDim.x >> 5) ? sv[lane] : -INFINITY;
    bi = lane < (int)(blockDim.x >> 5) ? si[lane] : INT_MAX;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (better(ov, oi, bv, bi)) bv = ov, bi = oi;
    }
  }
}

// Argmax of one chunk of one row.  rows_per_seq rows per sequence; row i >= n_b is skipped.
// The scan reads only the logits (inputs), so it runs before pdl_wait(); the partial is written
// after it (the previous step's acceptance may still be reading the workspace).
template <typename T>
__global__ void __launch_bounds__(kThreads) row_argmax_chunks(const T* __restrict__ logits, int V, int rows_per_seq,
                                                              const int32_t* __restrict__ num_rows, int chunks,
                                                              float2* __restrict__ part, int vec) {
  pdl_trigger();
  const int c = blockIdx.x, i = blockIdx.y, b = blockIdx.z;
  const int n = num_rows ? num_rows[b] : rows_per_seq;
  if (i >= n) {
    pdl_wait();
    return;
  }
  const T* row = logits + ((size_t)b * rows_per_seq + i) * V;
  const int lo = c * kChunk, hi = min(V, lo + kChunk);
  float bv = -INFINITY;
  int bi = INT_MAX;
  if (vec) {
    for (int v = lo + threadIdx.x * 8; v < hi; v += kThreads * 8) {
      float x[8];
      load8<T>(row, v, x);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (x[e] > bv) bv = x[e], bi = v + e;
    }
  } else {
    for (int v = lo + threadIdx.x; v < hi; v += kThreads) {
      const float x = load1(row, v);
      if (better(x, v, bv, bi)) bv = x, bi = v;
    }
  }
  block_argmax(bv, bi);
  pdl_wait();
  if (threadIdx.x == 0) {
    if (bv == -INFINITY || bi == INT_MAX) bi = lo;   // nothing above -inf: the chunk's first index
    part[((size_t)b * rows_per_seq + i) * chunks + c] = make_float2(bv, __int_as_float(bi));
  }
}

// Per-tree acceptance: t*(node), accepted set by walking each node's ancestors, deepest node.
__global__ void __launch_bounds__(kThreads) tree_accept_kernel(const float2* __restrict__ part, int chunks,
                                                               const int32_t* __restrict__ tokens,
                                                               const int32_t* __restrict__ parent_s,
                                                               const int32_t* __restrict__ num_nodes,
                                                               const int32_t* __restrict__ root_key, int Nmax,
                                                               int Dmax, int32_t* __restrict__ accept_len,
                                                               int32_t* __restrict__ path,
                                                               int32_t* __restrict__ out_tokens,
                                                               const int32_t* __restrict__ status, int staged) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int32_t s_tstar[];
  __shared__ int32_t s_path[256];
  acc::tree_accept_block(part, chunks, tokens, parent_s, num_nodes, root_key, Nmax, Dmax, status, accept_len, path,
                         out_tokens, s_tstar, s_path, staged ? s_tstar + Nmax : nullptr,
                         staged ? reinterpret_cast<float2*>(s_tstar + 3 * Nmax + 2) : nullptr);
}

// Greedy chain (T == 0): accept while the draft equals the target argmax.
__global__ void chain_greedy_decide(const float2* __restrict__ part, int chunks, const int32_t* __restrict__ x,
                                    int B, int K, int32_t* __restrict__ accept_len,
                                    int32_t* __restrict__ out_tokens) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  int j = K;
  for (int k = 0; k < K; ++k)
    if (x[(size_t)b * K + k] != acc::merge_argmax(part + ((size_t)b * (K + 1) + k) * chunks, chunks)) {
      j = k;
      break;
    }
  accept_len[b] = j;
  int32_t* orow = out_tokens + (size_t)b * (K + 1);
  for (int k = 0; k < j; ++k) orow[k] = x[(size_t)b * K + k];
  orow[j] = acc::merge_argmax(part + ((size_t)b * (K + 1) + j) * chunks, chunks);
  for (int k = j + 1; k <= K; ++k) orow[k] = -1;
}

}  // namespace

size_t accept_greedy_ws(int B, int Nmax, int V) {
  return (size_t)B * Nmax * num_chunks(V) * sizeof(float2);
}

tsd_status launch_row_argmax(const void* logits, tsd_dtype dtype, int V, int rows_per_seq, const int32_t* num_rows,
                             int B, void* ws, cudaStream_t stream) {
  if (B == 0 || rows_per_seq == 0) return TSD_OK;
  const int chunks = num_chunks(V);
  float2* part = reinterpret_cast<float2*>(ws);
  dim3 grid(chunks, rows_per_seq, B);
  const int vec = vec16_rows(logits, V) ? 1 : 0;
  if (dtype == TSD_BF16)
    launch_pdl(row_argmax_chunks<__nv_bfloat16>, grid, dim3(kThreads), 0, stream,
               reinterpret_cast<const __nv_bfloat16*>(logits), V, rows_per_seq, num_rows, chunks, part, vec);
  else
    launch_pdl(row_argmax_chunks<float>, grid, dim3(kThreads), 0, stream, reinterpret_cast<const float*>(logits), V,
               rows_per_seq, num_rows, chunks, part, vec);
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

int argmax_chunks(int V) { return num_chunks(V); }

tsd_status launch_accept_greedy(const void* logits, tsd_dtype dtype, int V, const int32_t* tokens,
                                const int32_t* parent_s, const int32_t* num_nodes, const int32_t* root_key, int B,
                                int Nmax, int Dmax, int32_t* accept_len, int32_t* path, int32_t* out_tokens,
                                void* ws, int32_t* status, cudaStream_t stream) {
  if (B == 0) return TSD_OK;
  const int chunks = num_chunks(V);
  if (launch_row_argmax(logits, dtype, V, Nmax, num_nodes, B, ws, stream) != TSD_OK) return TSD_ERR_CUDA;
  size_t smem = (size_t)(Nmax > 0 ? Nmax : 1) * sizeof(int32_t);
  // parent slots and tokens (2 Nmax + 1 ints, padded to 8 bytes) and the argmax partials copied on chip
  const size_t stage = (size_t)(2 * Nmax + 2) * sizeof(int32_t) + (size_t)Nmax * chunks * sizeof(float2);
  const int staged = (Nmax & 1) == 0 && smem + stage <= 96 * 1024 ? 1 : 0;
  if (staged) smem += stage;
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(tree_accept_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch_pdl(tree_accept_kernel, dim3(B), dim3(kThreads), smem, stream, (const float2*)ws, chunks, tokens, parent_s,
             num_nodes, root_key, Nmax, Dmax, accept_len, path, out_tokens, (const int32_t*)status, staged);
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

tsd_status launch_chain_sample(const void* zp, const void* zq, tsd_dtype dtype, int V, const int32_t* x,
                               const float* u, float T, int B, int K, int32_t* accept_len, int32_t* out_tokens,
                               void* ws, cudaStream_t stream) {
  if (B == 0) return TSD_OK;
  if (T > 0.f)
    return launch_chain_sample_stochastic(zp, zq, dtype, V, x, u, T, B, K, accept_len, out_tokens, ws, stream);
  // T == 0: greedy chain -- accept while the draft equals the target argmax
  const int chunks = num_chunks(V);
  float2* part = reinterpret_cast<float2*>(ws);
  dim3 grid(chunks, K + 1, B);
  const int vec = vec16_rows(zp, V) ? 1 : 0;
  if (dtype == TSD_BF16)
    launch_pdl(row_argmax_chunks<__nv_bfloat16>, grid, dim3(kThreads), 0, stream,
               reinterpret_cast<const __nv_bfloat16*>(zp), V, K + 1, (const int32_t*)nullptr, chunks, part, vec);
  else
    launch_pdl(row_argmax_chunks<float>, grid, dim3(kThreads), 0, stream, reinterpret_cast<const float*>(zp), V, K + 1,
               (const int32_t*)nullptr, chunks, part, vec);
  launch_pdl(chain_greedy_decide, dim3((B + 127) / 128), dim3(128), 0, stream, (const float2*)part, chunks, x, B, K,
             accept_len, out_tokens);
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}


// ---------------------------------------------------------------------------------------------
// tsd_tree_accept_greedy_noalloc: the same acceptance with its scratch in a fixed device array.
//
// Some callers cannot allocate device memory for scratch: a serving engine that handed all free
// device memory to its KV-cache pool at start-up, or a plug-in that a host runtime gives device
// pointers but no allocator.  This variant needs no workspace argument: the argmax partials live
// in g_accept_scratch, a file-scope array that every device loading this library holds until the
// process exits.  Host code cannot pass the array's name to a kernel (in host code it names a
// host-side stand-in), so the device address is fetched once per device with
// cudaGetSymbolAddress, with that device current, on the first call made on it, and cached.
// All calls share the array and it keeps the previous call's contents; nothing in it needs to
// start at zero, because every entry the final kernel reads is written earlier in the same call.
// Calls that overlap on the GPU (two streams, or two host threads) race on the array.
// ---------------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_accept_scratch[TSD_ACCEPT_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
}  // namespace

tsd_status accept_noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TSD_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_accept_scratch) != cudaSuccess || p == nullptr) return TSD_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return TSD_OK;
}

}  // namespace tsd
