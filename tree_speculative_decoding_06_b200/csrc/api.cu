// The C ABI (include/tsd.h): host-side argument checks, then one launch sequence per call on the
// caller's stream.  No allocation, no synchronisation, no state kept between calls.
#include <cstdio>

#include "draft_tree.h"
#include "kernels.h"
#include "tsd.h"

using namespace tsd;

namespace {

constexpr int kAbiVersion = 2;

inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
inline int log2i(int x) {
  int s = 0;
  while ((1 << s) < x) ++s;
  return s;
}
inline bool dtype_ok(tsd_dtype t) { return t == TSD_F32 || t == TSD_BF16; }

tsd_status check_attn_common(const void* q, const int32_t* prefix_len, const void* k_tree, const void* v_tree,
                             const int32_t* parent_s, int B, int Nmax, int Hq, int Hkv, int d, int Dmax,
                             tsd_dtype dtype, const void* out, int32_t* status) {
  if (!dtype_ok(dtype)) return TSD_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || B > 65535 || Nmax < 0 || Nmax > 4096 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Hkv > 65535)
    return TSD_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return TSD_ERR_INVALID_ARG;
  if (Dmax < 0 || Dmax > 255) return TSD_ERR_INVALID_ARG;
  if ((k_tree == nullptr) != (v_tree == nullptr)) return TSD_ERR_INVALID_ARG;
  if (B > 0 && Nmax > 0 && (!q || !prefix_len || !parent_s || !out || !status)) return TSD_ERR_INVALID_ARG;
  // the kernels move Q, K, V and O rows in 16-byte pieces
  if (!aligned16(q) || !aligned16(k_tree) || !aligned16(v_tree) || !aligned16(out)) return TSD_ERR_INVALID_ARG;
  return TSD_OK;
}

}  // namespace

extern "C" {

const char* tsd_status_str(int code) {
  switch (code & 0xff) {
    case TSD_OK: return "TSD_OK";
    case TSD_ERR_INVALID_ARG: return "TSD_ERR_INVALID_ARG";
    case TSD_ERR_UNSUPPORTED_DTYPE: return "TSD_ERR_UNSUPPORTED_DTYPE";
    case TSD_ERR_BAD_TREE: return "TSD_ERR_BAD_TREE";
    case TSD_ERR_TREE_DEPTH: return "TSD_ERR_TREE_DEPTH";
    case TSD_ERR_TREE_ROOTS: return "TSD_ERR_TREE_ROOTS";
    case TSD_ERR_CAPACITY: return "TSD_ERR_CAPACITY";
    case TSD_ERR_TIMEOUT: return "TSD_ERR_TIMEOUT";
    case TSD_ERR_CUDA: return "TSD_ERR_CUDA";
    case TSD_ERR_WORKSPACE: return "TSD_ERR_WORKSPACE";
    default: return "TSD_ERR_UNKNOWN";
  }
}

int tsd_abi_version(void) { return kAbiVersion; }

tsd_status tsd_tree_prepare(const int32_t* parent, const int32_t* num_nodes, int B, int Nmax, int Dmax, int forest,
                            int32_t* parent_s, int32_t* depth, int32_t* anc, uint32_t* anc_bits, int32_t* status,
                            void* stream) {
  if (B < 0 || Nmax < 0 || Dmax < 0 || Dmax > 255 || (forest != 0 && forest != 1)) return TSD_ERR_INVALID_ARG;
  if (B == 0) return TSD_OK;
  if (!parent_s || !depth || !anc || !status || (Nmax > 0 && !parent)) return TSD_ERR_INVALID_ARG;
  return launch_tree_prepare(parent, num_nodes, B, Nmax, Dmax, forest, parent_s, depth, anc, anc_bits, status,
                             S(stream));
}

size_t tsd_tree_verify_attn_workspace_size(int B, int Nmax, int Hq, int Hkv, int d, int Lmax, tsd_dtype dtype) {
  if (B <= 0 || Nmax <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Lmax < 0 || !dtype_ok(dtype)) return 0;
  return plan_attention(B, Nmax, Hq, Hkv, d, Lmax, dtype, false).ws_bytes;
}

size_t tsd_tree_verify_attn_ticket_bytes(void) { return kAttnTicketBytes; }

int tsd_tree_verify_attn_kernels(int B, int Nmax, int Hq, int Hkv, int d, int Lmax, int block_size, int tree_in_cache,
                                 tsd_dtype dtype) {
  if (B <= 0 || Nmax <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Lmax < 0 || block_size < 0 || !dtype_ok(dtype)) return 0;
  return attention_launch_count(B, Nmax, Hq, Hkv, d, Lmax, dtype, block_size > 0, tree_in_cache != 0);
}

long long tsd_tree_verify_attn_ctas(int B, int Nmax, int Hq, int Hkv, int d, int Lmax, int block_size,
                                    int tree_in_cache, tsd_dtype dtype) {
  if (B <= 0 || Nmax <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Lmax < 0 || block_size < 0 || !dtype_ok(dtype)) return 0;
  long long n = 0;
  attention_launch_count(B, Nmax, Hq, Hkv, d, Lmax, dtype, block_size > 0, tree_in_cache != 0, &n);
  return n;
}

size_t tsd_tree_verify_attn_paged_workspace_size(int B, int Nmax, int Hq, int Hkv, int d, int max_blocks,
                                                 int block_size, tsd_dtype dtype) {
  if (max_blocks < 0 || block_size <= 0) return 0;
  if (B <= 0 || Nmax <= 0 || Hkv <= 0 || Hq % Hkv != 0 || !dtype_ok(dtype)) return 0;
  return plan_attention(B, Nmax, Hq, Hkv, d, max_blocks * block_size, dtype, true).ws_bytes;
}

tsd_status tsd_tree_verify_attn(const void* q, const void* k_cache, const void* v_cache, int Lmax,
                                const int32_t* prefix_len, const void* k_tree, const void* v_tree,
                                const int32_t* parent_s, const int32_t* num_nodes, int B, int Nmax, int Hq, int Hkv,
                                int d, int Dmax, tsd_dtype dtype, float scale, void* out, float* lse,
                                void* workspace, size_t ws_bytes, int32_t* status, void* stream) {
  tsd_status e = check_attn_common(q, prefix_len, k_tree, v_tree, parent_s, B, Nmax, Hq, Hkv, d, Dmax, dtype, out,
                                   status);
  if (e != TSD_OK) return e;
  if (Lmax < 0) return TSD_ERR_INVALID_ARG;
  if (B == 0 || Nmax == 0) return TSD_OK;
  if (Lmax > 0 && (!k_cache || !v_cache)) return TSD_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return TSD_ERR_INVALID_ARG;
  const size_t need = tsd_tree_verify_attn_workspace_size(B, Nmax, Hq, Hkv, d, Lmax, dtype);
  if (need > 0 && (workspace == nullptr || ws_bytes < need || !aligned16(workspace))) return TSD_ERR_WORKSPACE;
  AttnArgs a{};
  a.q = q, a.k_cache = k_cache, a.v_cache = v_cache, a.block_table = nullptr;
  a.max_blocks = 0, a.block_shift = 0, a.num_blocks = 0, a.Lcap = Lmax, a.prefix_len = prefix_len;
  a.k_tree = k_tree, a.v_tree = v_tree, a.parent_s = parent_s, a.num_nodes = num_nodes;
  a.B = B, a.Nmax = Nmax, a.Hq = Hq, a.Hkv = Hkv, a.d = d, a.Dmax = Dmax, a.scale = scale;
  a.out = out, a.lse = lse, a.workspace = workspace, a.ws_bytes = ws_bytes, a.status = status;
  return launch_attention(a, dtype, S(stream));
}

tsd_status tsd_tree_verify_attn_paged(const void* q, const void* k_pages, const void* v_pages, int num_blocks,
                                      int block_size, const int32_t* block_table, int max_blocks,
                                      const int32_t* prefix_len, const void* k_tree, const void* v_tree,
                                      const int32_t* parent_s, const int32_t* num_nodes, int B, int Nmax, int Hq,
                                      int Hkv, int d, int Dmax, tsd_dtype dtype, float scale, void* out, float* lse,
                                      void* workspace, size_t ws_bytes, int32_t* status, void* stream) {
  tsd_status e = check_attn_common(q, prefix_len, k_tree, v_tree, parent_s, B, Nmax, Hq, Hkv, d, Dmax, dtype, out,
                                   status);
  if (e != TSD_OK) return e;
  if (!pow2(block_size) || block_size < 8 || block_size > 256 || max_blocks < 0 || num_blocks < 0)
    return TSD_ERR_INVALID_ARG;
  if ((long long)max_blocks * block_size > 0x7fffffffLL) return TSD_ERR_INVALID_ARG;
  if (B == 0 || Nmax == 0) return TSD_OK;
  if (max_blocks > 0 && (!k_pages || !v_pages || !block_table)) return TSD_ERR_INVALID_ARG;
  if (!aligned16(k_pages) || !aligned16(v_pages)) return TSD_ERR_INVALID_ARG;
  const size_t need =
      tsd_tree_verify_attn_paged_workspace_size(B, Nmax, Hq, Hkv, d, max_blocks, block_size, dtype);
  if (need > 0 && (workspace == nullptr || ws_bytes < need || !aligned16(workspace))) return TSD_ERR_WORKSPACE;
  AttnArgs a{};
  a.q = q, a.k_cache = k_pages, a.v_cache = v_pages, a.block_table = block_table;
  a.max_blocks = max_blocks, a.block_shift = log2i(block_size), a.num_blocks = num_blocks;
  a.Lcap = max_blocks * block_size, a.prefix_len = prefix_len;
  a.k_tree = k_tree, a.v_tree = v_tree, a.parent_s = parent_s, a.num_nodes = num_nodes;
  a.B = B, a.Nmax = Nmax, a.Hq = Hq, a.Hkv = Hkv, a.d = d, a.Dmax = Dmax, a.scale = scale;
  a.out = out, a.lse = lse, a.workspace = workspace, a.ws_bytes = ws_bytes, a.status = status;
  return launch_attention(a, dtype, S(stream));
}

size_t tsd_tree_accept_greedy_workspace_size(int B, int Nmax, int V) {
  if (B <= 0 || Nmax <= 0 || V <= 0) return 0;
  return accept_greedy_ws(B, Nmax, V);
}

tsd_status tsd_tree_accept_greedy(const void* logits, tsd_dtype dtype, int V, const int32_t* tokens,
                                  const int32_t* parent_s, const int32_t* num_nodes, const int32_t* root_key, int B,
                                  int Nmax, int Dmax, int32_t* accept_len, int32_t* path, int32_t* out_tokens,
                                  void* workspace, size_t ws_bytes, int32_t* status, void* stream) {
  if (!dtype_ok(dtype)) return TSD_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || B > 65535 || Nmax < 0 || Nmax > 65535 || V <= 0 || Dmax < 0 || Dmax > 255) return TSD_ERR_INVALID_ARG;
  if ((long long)Nmax * 4 > 200 * 1024) return TSD_ERR_INVALID_ARG;
  if (B == 0) return TSD_OK;
  if (!accept_len || !path || !out_tokens || !status || !parent_s || (Nmax > 0 && (!logits || !tokens)))
    return TSD_ERR_INVALID_ARG;
  const size_t need = tsd_tree_accept_greedy_workspace_size(B, Nmax, V);
  if (need > 0 && (workspace == nullptr || ws_bytes < need || !aligned16(workspace))) return TSD_ERR_WORKSPACE;
  return launch_accept_greedy(logits, dtype, V, tokens, parent_s, num_nodes, root_key, B, Nmax, Dmax, accept_len,
                              path, out_tokens, workspace, status, S(stream));
}

size_t tsd_tree_accept_threshold_workspace_size(int B, int Nmax, int V) {
  if (B <= 0 || Nmax <= 0 || V <= 0) return 0;
  return accept_threshold_ws(B, Nmax, V);
}

tsd_status tsd_tree_accept_threshold(const void* logits, tsd_dtype dtype, int V, const int32_t* tokens,
                                     const int32_t* parent_s, const int32_t* num_nodes, const int32_t* root_key,
                                     float tau, float temperature, int B, int Nmax, int Dmax, int32_t* accept_len,
                                     int32_t* path, int32_t* out_tokens, void* workspace, size_t ws_bytes,
                                     int32_t* status, void* stream) {
  if (!dtype_ok(dtype)) return TSD_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || B > 65535 || Nmax < 0 || Nmax > 4096 || V <= 0 || Dmax < 0 || Dmax > 255) return TSD_ERR_INVALID_ARG;
  if (!(tau >= 0.f && tau <= 1.f) || !(temperature > 0.f) || !(temperature < 3.0e38f)) return TSD_ERR_INVALID_ARG;
  if (B == 0) return TSD_OK;
  if (!accept_len || !path || !out_tokens || !status || !parent_s || (Nmax > 0 && (!logits || !tokens)))
    return TSD_ERR_INVALID_ARG;
  const size_t need = tsd_tree_accept_threshold_workspace_size(B, Nmax, V);
  if (need > 0 && (workspace == nullptr || ws_bytes < need || !aligned16(workspace))) return TSD_ERR_WORKSPACE;
  return launch_accept_threshold(logits, dtype, V, tokens, parent_s, num_nodes, root_key, tau, temperature, B, Nmax,
                                 Dmax, accept_len, path, out_tokens, workspace, status, S(stream));
}

tsd_status tsd_tree_accept_greedy_noalloc(const void* logits, tsd_dtype dtype, int V, const int32_t* tokens,
                                          const int32_t* parent_s, const int32_t* num_nodes,
                                          const int32_t* root_key, int B, int Nmax, int Dmax,
                                          int32_t* accept_len, int32_t* path, int32_t* out_tokens, int32_t* status,
                                          void* stream) {
  if (!dtype_ok(dtype)) return TSD_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || B > 65535 || Nmax < 0 || Nmax > 65535 || V <= 0 || Dmax < 0 || Dmax > 255) return TSD_ERR_INVALID_ARG;
  if ((long long)Nmax * 4 > 200 * 1024) return TSD_ERR_INVALID_ARG;
  if (B == 0) return TSD_OK;
  if (!accept_len || !path || !out_tokens || !status || !parent_s || (Nmax > 0 && (!logits || !tokens)))
    return TSD_ERR_INVALID_ARG;
  const size_t need = tsd_tree_accept_greedy_workspace_size(B, Nmax, V);
  if (need > (size_t)TSD_ACCEPT_NOALLOC_SCRATCH_BYTES) return TSD_ERR_WORKSPACE;
  void* scratch = nullptr;
  const tsd_status e = accept_noalloc_scratch(&scratch);
  if (e != TSD_OK) return e;
  return launch_accept_greedy(logits, dtype, V, tokens, parent_s, num_nodes, root_key, B, Nmax, Dmax, accept_len,
                              path, out_tokens, scratch, status, S(stream));
}

size_t tsd_tree_accept_greedy_noalloc_scratch_bytes(void) { return (size_t)TSD_ACCEPT_NOALLOC_SCRATCH_BYTES; }

size_t tsd_chain_accept_sample_workspace_size(int B, int K, int V) {
  if (B <= 0 || K < 0 || V <= 0) return 0;
  return chain_sample_ws(B, K, V);
}

tsd_status tsd_chain_accept_sample(const void* target_logits, const void* draft_logits, tsd_dtype dtype, int V,
                                   const int32_t* draft_tokens, const float* uniforms, float temperature, int B, int K,
                                   int32_t* accept_len, int32_t* out_tokens, void* workspace, size_t ws_bytes,
                                   void* stream) {
  if (!dtype_ok(dtype)) return TSD_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || B > 65535 || K < 0 || K > 1024 || V <= 0 || !(temperature >= 0.f)) return TSD_ERR_INVALID_ARG;
  if (B == 0) return TSD_OK;
  if (!target_logits || !uniforms || !accept_len || !out_tokens || (K > 0 && (!draft_logits || !draft_tokens)))
    return TSD_ERR_INVALID_ARG;
  const size_t need = tsd_chain_accept_sample_workspace_size(B, K, V);
  if (workspace == nullptr || ws_bytes < need || !aligned16(workspace)) return TSD_ERR_WORKSPACE;
  return launch_chain_sample(target_logits, draft_logits, dtype, V, draft_tokens, uniforms, temperature, B, K,
                             accept_len, out_tokens, workspace, S(stream));
}

tsd_status tsd_tree_accept_sample(const void* target_logits, const void* draft_logits, tsd_dtype dtype, int V,
                                  const int32_t* tokens, const int32_t* parent_s, const int32_t* num_nodes,
                                  const float* uniforms, float temperature, int B, int Nmax, int Dmax,
                                  int32_t* accept_len, int32_t* path, int32_t* out_tokens, int32_t* status,
                                  void* stream) {
  if (!dtype_ok(dtype)) return TSD_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || B > 65535 || Nmax < 0 || Nmax > 4096 || V <= 0 || Dmax < 0 || Dmax > 255) return TSD_ERR_INVALID_ARG;
  if (!(temperature > 0.f) || !(temperature < 3.0e38f)) return TSD_ERR_INVALID_ARG;
  if (tree_sample_smem(V, Nmax, dtype) > 200 * 1024) return TSD_ERR_INVALID_ARG;
  if (B == 0) return TSD_OK;
  if (!accept_len || !path || !out_tokens || !status || !parent_s || !uniforms ||
      (Nmax > 0 && (!target_logits || !draft_logits || !tokens)))
    return TSD_ERR_INVALID_ARG;
  return launch_tree_sample(target_logits, draft_logits, dtype, V, tokens, parent_s, num_nodes, uniforms,
                            temperature, B, Nmax, Dmax, accept_len, path, out_tokens, status, S(stream));
}

tsd_status tsd_ssd_cache_build(const void* draft_logits, tsd_dtype dtype, int V, int K, int S, const float* alpha,
                               float beta, const float* uniforms, float temperature, int B, int32_t* slots,
                               int32_t* key_len, int32_t* key_tok, int32_t* draft_tokens, void* stream) {
  if (!dtype_ok(dtype)) return TSD_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || B > 65535 || V <= 0 || K < 0 || K > ssd_cache_max_k() || S < 1 || S > ssd_cache_max_slots() || S > V)
    return TSD_ERR_INVALID_ARG;
  if (!(beta >= 0.f && beta <= 1.f) || !(temperature > 0.f) || !(temperature < 3.0e38f)) return TSD_ERR_INVALID_ARG;
  if (ssd_cache_smem(V, dtype) > 200 * 1024) return TSD_ERR_INVALID_ARG;
  if (B == 0) return TSD_OK;
  if (!draft_logits || !alpha || !slots || !key_len || !key_tok || (K > 0 && (!uniforms || !draft_tokens)))
    return TSD_ERR_INVALID_ARG;
  return launch_ssd_cache(draft_logits, dtype, V, K, S, alpha, beta, uniforms, temperature, B, slots, key_len,
                          key_tok, draft_tokens, ::S(stream));
}

static tsd_status commit_common(CommitArgs& a, const void* k_tree, const void* v_tree, const int32_t* path,
                                const int32_t* accept_len, tsd_dtype dtype, tsd_commit_mode mode) {
  if (!dtype_ok(dtype)) return TSD_ERR_UNSUPPORTED_DTYPE;
  if (mode != TSD_COMMIT_PATH && mode != TSD_COMMIT_LENGTH && mode != TSD_COMMIT_INPLACE) return TSD_ERR_INVALID_ARG;
  if (a.B < 0 || a.B > 2147483647 || a.Nmax < 0 || a.Hkv <= 0 || (a.d != 64 && a.d != 128) || a.Dmax < 0 ||
      a.Dmax > 255)
    return TSD_ERR_INVALID_ARG;
  if (a.B == 0) return TSD_OK;
  if (!a.k_cache || !a.v_cache || !a.prefix_len || !accept_len || !a.status) return TSD_ERR_INVALID_ARG;
  if (mode != TSD_COMMIT_LENGTH && !path) return TSD_ERR_INVALID_ARG;
  if (mode != TSD_COMMIT_INPLACE && (!k_tree || !v_tree)) return TSD_ERR_INVALID_ARG;
  // rows are copied in 16-byte pieces
  if (!aligned16(a.k_cache) || !aligned16(a.v_cache) || !aligned16(k_tree) || !aligned16(v_tree))
    return TSD_ERR_INVALID_ARG;
  a.k_tree = k_tree, a.v_tree = v_tree, a.path = path, a.accept_len = accept_len;
  a.esize = dtype == TSD_BF16 ? 2 : 4;
  a.mode = (int)mode;
  return TSD_OK;
}

tsd_status tsd_kv_commit(void* k_cache, void* v_cache, int Lmax, int32_t* prefix_len, const void* k_tree,
                         const void* v_tree, const int32_t* path, const int32_t* accept_len, const int32_t* num_nodes,
                         int B, int Nmax, int Hkv, int d, int Dmax, tsd_dtype dtype, tsd_commit_mode mode,
                         int32_t* status, void* stream) {
  CommitArgs a{};
  a.k_cache = k_cache, a.v_cache = v_cache, a.block_table = nullptr, a.Lcap = Lmax, a.prefix_len = prefix_len;
  a.num_nodes = num_nodes, a.B = B, a.Nmax = Nmax, a.Hkv = Hkv, a.d = d, a.Dmax = Dmax, a.status = status;
  if (Lmax < 0) return TSD_ERR_INVALID_ARG;
  tsd_status e = commit_common(a, k_tree, v_tree, path, accept_len, dtype, mode);
  if (e != TSD_OK || B == 0) return e;
  return launch_kv_commit(a, S(stream));
}

tsd_status tsd_kv_commit_paged(void* k_pages, void* v_pages, int num_blocks, int block_size, const int32_t* block_table,
                               int max_blocks, int32_t* prefix_len, const void* k_tree, const void* v_tree,
                               const int32_t* path, const int32_t* accept_len, const int32_t* num_nodes, int B,
                               int Nmax, int Hkv, int d, int Dmax, tsd_dtype dtype, tsd_commit_mode mode,
                               int32_t* status, void* stream) {
  if (!pow2(block_size) || block_size < 8 || block_size > 256 || max_blocks < 0 || num_blocks < 0)
    return TSD_ERR_INVALID_ARG;
  if ((long long)max_blocks * block_size > 0x7fffffffLL) return TSD_ERR_INVALID_ARG;
  CommitArgs a{};
  a.k_cache = k_pages, a.v_cache = v_pages, a.block_table = block_table, a.max_blocks = max_blocks;
  a.block_shift = log2i(block_size), a.num_blocks = num_blocks, a.Lcap = max_blocks * block_size;
  a.prefix_len = prefix_len, a.num_nodes = num_nodes, a.B = B, a.Nmax = Nmax, a.Hkv = Hkv, a.d = d, a.Dmax = Dmax;
  a.status = status;
  tsd_status e = commit_common(a, k_tree, v_tree, path, accept_len, dtype, mode);
  if (e != TSD_OK || B == 0) return e;
  if (!block_table) return TSD_ERR_INVALID_ARG;
  return launch_kv_commit(a, S(stream));
}

tsd_status tsd_tree_accept_commit(const void* logits, tsd_dtype logits_dtype, int V, const int32_t* tokens,
                                  const int32_t* parent_s, const int32_t* num_nodes, const int32_t* root_key, int B,
                                  int Nmax, int Dmax, const tsd_kv_cache* cache, const void* k_tree,
                                  const void* v_tree, int Hkv, int d, tsd_dtype kv_dtype, tsd_commit_mode mode,
                                  int32_t* history, int history_cap, int32_t* history_len, int32_t* accept_len,
                                  int32_t* path, int32_t* out_tokens, void* workspace, size_t ws_bytes,
                                  int32_t* status, void* stream) {
  // acceptance checks, as tsd_tree_accept_greedy
  if (!dtype_ok(logits_dtype)) return TSD_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || B > 65535 || Nmax < 0 || Nmax > 65535 || V <= 0 || Dmax < 0 || Dmax > 255) return TSD_ERR_INVALID_ARG;
  if ((long long)Nmax * 4 > 160 * 1024) return TSD_ERR_INVALID_ARG;
  if (!cache) return TSD_ERR_INVALID_ARG;
  // commit checks, as tsd_kv_commit[_paged]
  CommitArgs a{};
  a.k_cache = cache->k, a.v_cache = cache->v, a.prefix_len = cache->prefix_len, a.block_table = cache->block_table;
  if (cache->block_table) {
    if (!pow2(cache->block_size) || cache->block_size < 8 || cache->block_size > 256 || cache->max_blocks < 0 ||
        cache->num_blocks < 0)
      return TSD_ERR_INVALID_ARG;
    if ((long long)cache->max_blocks * cache->block_size > 0x7fffffffLL) return TSD_ERR_INVALID_ARG;
    a.max_blocks = cache->max_blocks, a.block_shift = log2i(cache->block_size), a.num_blocks = cache->num_blocks;
    a.Lcap = cache->max_blocks * cache->block_size;
  } else {
    if (cache->Lmax < 0) return TSD_ERR_INVALID_ARG;
    a.Lcap = cache->Lmax;
  }
  a.num_nodes = num_nodes, a.B = B, a.Nmax = Nmax, a.Hkv = Hkv, a.d = d, a.Dmax = Dmax, a.status = status;
  // the path is produced in the kernel; commit_common only checks it is given in PATH / INPLACE
  tsd_status e = commit_common(a, k_tree, v_tree, path, accept_len, kv_dtype, mode);
  if (e != TSD_OK || B == 0) return e;
  if (!accept_len || !path || !out_tokens || !status || !parent_s || (Nmax > 0 && (!logits || !tokens)))
    return TSD_ERR_INVALID_ARG;
  if (history && (history_cap < 0 || !history_len)) return TSD_ERR_INVALID_ARG;
  const size_t need = tsd_tree_accept_greedy_workspace_size(B, Nmax, V);
  if (need > 0 && (workspace == nullptr || ws_bytes < need || !aligned16(workspace))) return TSD_ERR_WORKSPACE;
  SpliceArgs sp{history, history_cap, history_len};
  return launch_accept_commit(logits, logits_dtype, V, tokens, parent_s, root_key, accept_len, path, out_tokens, a, sp,
                              workspace, S(stream));
}

static bool draft_args(const tsd_draft_tree* tree, int B, DraftTreeArgs& t) {
  if (!tree || B < 0 || B > 65535 || tree->max_nodes < 1 || tree->F < 1 || tree->F > 16) return false;
  if (B > 0 && (!tree->parent || !tree->token || !tree->score || !tree->depth || !tree->num_nodes ||
                !tree->frontier || !tree->num_frontier))
    return false;
  t.parent = tree->parent, t.token = tree->token, t.score = tree->score, t.depth = tree->depth;
  t.num_nodes = tree->num_nodes, t.frontier = tree->frontier, t.num_frontier = tree->num_frontier;
  t.max_nodes = tree->max_nodes, t.F = tree->F, t.B = B;
  return true;
}

tsd_status tsd_draft_tree_init(const tsd_draft_tree* tree, const int32_t* root_token, int B, int32_t* status,
                               void* stream) {
  DraftTreeArgs t{};
  if (!draft_args(tree, B, t)) return TSD_ERR_INVALID_ARG;
  if (B == 0) return TSD_OK;
  if (!root_token || !status) return TSD_ERR_INVALID_ARG;
  return launch_draft_init(t, root_token, status, S(stream));
}

size_t tsd_draft_tree_expand_workspace_size(int B, int F, int K, int V) {
  if (B <= 0 || F <= 0 || K <= 0 || V <= 0) return 0;
  return draft_expand_ws(B, F, K, V);
}

tsd_status tsd_draft_tree_expand(const tsd_draft_tree* tree, const void* draft_logits, tsd_dtype dtype, int V, int K,
                                 int B, void* workspace, size_t ws_bytes, int32_t* status, void* stream) {
  if (!dtype_ok(dtype)) return TSD_ERR_UNSUPPORTED_DTYPE;
  DraftTreeArgs t{};
  if (!draft_args(tree, B, t)) return TSD_ERR_INVALID_ARG;
  if (V <= 0 || V > 64 * 16384 || K < 1 || K > 16 || K > V) return TSD_ERR_INVALID_ARG;
  if (B == 0) return TSD_OK;
  if (!draft_logits || !status) return TSD_ERR_INVALID_ARG;
  const size_t need = draft_expand_ws(B, t.F, K, V);
  if (workspace == nullptr || ws_bytes < need || !aligned16(workspace)) return TSD_ERR_WORKSPACE;
  return launch_draft_expand(t, draft_logits, dtype, V, K, workspace, status, S(stream));
}

tsd_status tsd_draft_tree_finalize(const tsd_draft_tree* tree, int B, int keep, int32_t* parent_out,
                                   int32_t* tokens_out, int32_t* num_nodes_out, int32_t* status, void* stream) {
  DraftTreeArgs t{};
  if (!draft_args(tree, B, t)) return TSD_ERR_INVALID_ARG;
  if (keep < 1 || tree->max_nodes > 4096) return TSD_ERR_INVALID_ARG;
  if (B == 0) return TSD_OK;
  if (!parent_out || !tokens_out || !num_nodes_out || !status) return TSD_ERR_INVALID_ARG;
  return launch_draft_finalize(t, keep, parent_out, tokens_out, num_nodes_out, status, S(stream));
}

}  // extern "C"
