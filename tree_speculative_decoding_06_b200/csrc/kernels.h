// Internal launch entry points of the kernels (host side); the C ABI in api.cu validates
// arguments and calls these.
#pragma once
#include <cmath>

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "tsd.h"

namespace tsd {

// The vocabulary scans read 8 logits (16 bytes of bf16, two 16-byte words of fp32) per load when
// every row starts on a 16-byte boundary: V a multiple of 8 and the base pointer 16-byte aligned.
// Decided on the host from the actual pointer, so a view at an odd storage offset takes the
// scalar path instead of faulting.
inline bool vec16_rows(const void* base, int V) {
  return V % 8 == 0 && (reinterpret_cast<uintptr_t>(base) & 15) == 0;
}
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// A positive constant c as an unevaluated sum hi + lo of floats with lo > 0 (hi rounded toward
// zero; a tiny lo when c is itself a float), so that d * hi + d * lo is -inf, not -inf + inf, for
// d = -inf (a -inf logit, or -inf padding).
inline void split_const(double c, float& hi, float& lo) {
  hi = (float)c;
  if ((double)hi > c) hi = std::nextafter(hi, 0.0f);
  lo = (float)(c - (double)hi);
  if (!(lo > 0.f)) lo = 1e-30f;
}

// Launch with programmatic stream serialisation (see pdl_wait / pdl_trigger in common.cuh).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The attention workspace starts with the split-merge ticket words (one int32 per (sequence, KV
// head, row block) of the tcgen05 kernel, at most kAttnTicketBytes / 4 of them), zero between calls;
// the partials follow.
constexpr size_t kAttnTicketBytes = 65536;

// Split-KV plan of one attention launch: a CTA covers BM query rows of one (sequence, KV head)
// and `tps` key tiles of BN keys; the keys of sequence b are its prefix tiles followed by its
// tree tiles.  Partials of (max, sum, unnormalised output) go to the workspace when a sequence
// needs more than one split.
struct AttnPlan {
  int G = 1, Rmax = 0;      // query rows per (sequence, KV head) = G * Nmax
  int BM = 0, mtiles = 0;   // rows per CTA, row tiles
  int BN = 64;              // keys per tile
  int max_tiles = 0;        // prefix tiles at capacity + tree tiles
  int tps = 1, splits = 1;  // tiles per split, splits per (sequence, KV head, row tile)
  bool dual = false;        // tcgen05 kernel: two 128-row query tiles per CTA
  int umtiles = 0;          // tcgen05 kernel: row blocks per (sequence, KV head)
  int usplits = 1;          // tcgen05 kernel: CTAs splitting a row block's keys (equal shares)
  int threads = 128;
  size_t smem = 0;
  size_t ws_bytes = 0;
};

struct AttnArgs {
  const void* q;
  const void* k_cache;      // contiguous [B,Hkv,Lmax,d] or pages [num_blocks,Hkv,bs,d]
  const void* v_cache;
  const int32_t* block_table;  // null = contiguous
  int max_blocks, block_shift, num_blocks;
  int Lcap;                 // Lmax or max_blocks * bs
  const int32_t* prefix_len;
  const void* k_tree;       // null = tree rows in the cache after the prefix
  const void* v_tree;
  const int32_t* parent_s;
  const int32_t* num_nodes;
  int B, Nmax, Hq, Hkv, d, Dmax;
  float scale;
  void* out;
  float* lse;
  void* workspace;
  size_t ws_bytes;
  int32_t* status;
};

AttnPlan plan_attention(int B, int Nmax, int Hq, int Hkv, int d, int Lcap, tsd_dtype dtype, bool paged);
tsd_status launch_attention(const AttnArgs& a, tsd_dtype dtype, cudaStream_t stream);
// tcgen05 path (attn_umma.cu): bf16, d = 128, tree K/V in their own buffer, G a power of two.
bool umma_eligible(const AttnArgs& a, tsd_dtype dtype);
// Shared-memory layout of one tcgen05 attention CTA (rings, staged epilogue rows).
struct UmmaLayout {
  int rows = 0, W = 0, ks = 0, vs = 0, stage = 0;
  uint32_t k_off = 0, v_off = 0, mask_off = 0, ps_off = 0;
  size_t smem = 0;
};
bool umma_layout(const AttnPlan& p, int G, int Nmax, UmmaLayout& L);
bool umma_merges_in_kernel(const AttnPlan& p, const UmmaLayout& L, int B, int Hkv);
// Kernels one attention call launches (split kernel, plus the merge kernel when the keys are split
// and not merged in the kernel), for 16-byte-aligned tensors and a workspace of the queried size.
// (*ctas, if given: the CTAs of the split kernel's grid.)
int attention_launch_count(int B, int Nmax, int Hq, int Hkv, int d, int Lcap, tsd_dtype dtype, bool paged,
                           bool tree_in_cache, long long* ctas = nullptr);

// `tickets` (may be null) enables the split merge inside the kernel; *merged says whether it ran
// there (otherwise the caller launches the merge kernel).
tsd_status launch_attention_umma(const AttnArgs& a, const AttnPlan& p, int* tickets, bool* merged,
                                 cudaStream_t stream);

tsd_status launch_tree_prepare(const int32_t* parent, const int32_t* num_nodes, int B, int Nmax, int Dmax,
                               int forest, int32_t* parent_s, int32_t* depth, int32_t* anc, uint32_t* anc_bits,
                               int32_t* status, cudaStream_t stream);

size_t accept_greedy_ws(int B, int Nmax, int V);
tsd_status launch_accept_greedy(const void* logits, tsd_dtype dtype, int V, const int32_t* tokens,
                                const int32_t* parent_s, const int32_t* num_nodes, const int32_t* root_key, int B,
                                int Nmax, int Dmax, int32_t* accept_len, int32_t* path, int32_t* out_tokens,
                                void* ws, int32_t* status, cudaStream_t stream);

tsd_status accept_noalloc_scratch(void** out);

size_t chain_sample_ws(int B, int K, int V);
tsd_status launch_chain_sample_stochastic(const void* zp, const void* zq, tsd_dtype dtype, int V, const int32_t* x,
                                          const float* u, float T, int B, int K, int32_t* accept_len,
                                          int32_t* out_tokens, void* ws, cudaStream_t stream);
tsd_status launch_chain_sample(const void* zp, const void* zq, tsd_dtype dtype, int V, const int32_t* x,
                               const float* u, float T, int B, int K, int32_t* accept_len, int32_t* out_tokens,
                               void* ws, cudaStream_t stream);

// Stochastic tree acceptance (tree_sample.cu): one cluster of CTAs per sequence.
size_t tree_sample_smem(int V, int Nmax, tsd_dtype dtype);
tsd_status launch_tree_sample(const void* zp, const void* zq, tsd_dtype dtype, int V, const int32_t* tokens,
                              const int32_t* parent_s, const int32_t* num_nodes, const float* u, float T, int B,
                              int Nmax, int Dmax, int32_t* accept_len, int32_t* path, int32_t* out_tokens,
                              int32_t* status, cudaStream_t stream);

// SSD / Saguaro outcome cache (ssd_cache.cu): one cluster of CTAs per (sequence, row).
size_t ssd_cache_smem(int V, tsd_dtype dtype);
int ssd_cache_max_slots();
int ssd_cache_max_k();
tsd_status launch_ssd_cache(const void* zq, tsd_dtype dtype, int V, int K, int S, const float* alpha, float beta,
                            const float* u, float T, int B, int32_t* slots, int32_t* key_len, int32_t* key_tok,
                            int32_t* draft_tokens, cudaStream_t stream);

// Threshold acceptance (accept_threshold.cu).
size_t accept_threshold_ws(int B, int Nmax, int V);
size_t accept_threshold_smem(int Nmax);
tsd_status launch_accept_threshold(const void* logits, tsd_dtype dtype, int V, const int32_t* tokens,
                                   const int32_t* parent_s, const int32_t* num_nodes, const int32_t* root_key,
                                   float tau, float T, int B, int Nmax, int Dmax, int32_t* accept_len,
                                   int32_t* path, int32_t* out_tokens, void* ws, int32_t* status,
                                   cudaStream_t stream);

struct CommitArgs {
  void* k_cache;
  void* v_cache;
  const int32_t* block_table;  // null = contiguous [B,Hkv,Lmax,d]
  int max_blocks, block_shift, num_blocks;
  int Lcap;
  int32_t* prefix_len;
  const void* k_tree;
  const void* v_tree;
  const int32_t* path;
  const int32_t* accept_len;
  const int32_t* num_nodes;
  int B, Nmax, Hkv, d, Dmax, esize;
  int mode;
  int32_t* status;
};
tsd_status launch_kv_commit(const CommitArgs& a, cudaStream_t stream);

// Vocabulary argmax scan of rows_per_seq rows per sequence into ws (float2 per (row, chunk)).
tsd_status launch_row_argmax(const void* logits, tsd_dtype dtype, int V, int rows_per_seq, const int32_t* num_rows,
                             int B, void* ws, cudaStream_t stream);
int argmax_chunks(int V);
// Greedy tree acceptance fused with the commit of the accepted path (and an optional splice of
// the emitted tokens into a device token history).  a.accept_len / a.path are unused.
struct SpliceArgs {
  int32_t* history;      // [B, cap] or null
  int cap;
  int32_t* history_len;  // [B]
};
tsd_status launch_accept_commit(const void* logits, tsd_dtype dtype, int V, const int32_t* tokens,
                                const int32_t* parent_s, const int32_t* root_key, int32_t* accept_len,
                                int32_t* path, int32_t* out_tokens, const CommitArgs& a, const SpliceArgs& sp,
                                void* ws, cudaStream_t stream);

int device_sm_count();

}  // namespace tsd
