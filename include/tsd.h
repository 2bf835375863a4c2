/*
 * tsd.h -- C ABI of the tree speculative decoding verify library (sm_100a, B200).
 *
 * One verify step of the target model, as the source pages state the problem:
 *   1. tsd_tree_prepare       validate the draft tree and build its shifted indices;
 *   2. tsd_tree_verify_attn   tree-masked GQA attention of every tree node over the committed
 *                             prefix plus its own ancestors (contiguous or paged cache);
 *   3. tsd_tree_accept_greedy longest target-matching root->leaf path + the free target token,
 *      tsd_chain_accept_sample rejection sampling of a linear draft;
 *   4. tsd_kv_commit          copy only the accepted path's K/V rows into the cache.
 *
 * Sources (cited by page title and section):
 *   [EP]  "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs",
 *         technical summary sec. 2 (methodology) and sec. 4 (results: verification and cache
 *         commit dominate the step; mask and tree tensorisation cost milliseconds).
 *   [SO]  "Acelerando Sonar a traves de la especulacion" (Perplexity): sections
 *         "Decodificacion especulativa", "Objetivo-Borrador", "EAGLE" and
 *         "Programacion MTP para un solo token"; its cited reference by Leviathan et al.
 *   [SSD] "Speculative Speculative Decoding", technical summary sec. 2 (hit / miss).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE memory owned by the caller; the library allocates
 *     nothing and keeps no state between calls.  Scratch ("workspace") is passed in; its size
 *     comes from the matching *_workspace_size() query, which is a pure host function.  (The
 *     attention's workspace is the one that carries something from call to call: ticket
 *     words that every call returns to zero.)
 *   - Every call takes a CUDA stream (cudaStream_t passed as void*; NULL = legacy default
 *     stream), only enqueues work on it and returns without synchronising.  Accepted lengths
 *     and prefix lengths stay in device memory: nothing forces a device->host round trip
 *     between steps ([SO], "Inferencia con decodificacion especulativa": the accepted count
 *     is the hard CPU-GPU sync point of speculative decoding).
 *   - Node numbering: nodes 0..N_b-1 of sequence b are in topological order
 *     (parent[i] < i; a root has parent -1).  The kernels never see the -1: the internal
 *     SLOT of node i is i+1 and slot 0 is a dummy row ([EP] sec. 2, shifted indexing with a
 *     dummy row 0 for the root).  parent_s[s] is the parent slot of slot s (0 for roots and
 *     for slot 0), so every gather index is in range.
 *   - Row-major layouts (d = head dim, G = Hq / Hkv query heads per KV head):
 *       q, out        [B, Nmax, Hq, d]         (dtype)
 *       k_tree,v_tree [B, Nmax, Hkv, d]        (dtype)  K/V of the tree nodes
 *       k/v_cache     [B, Hkv, Lmax, d]        (dtype)  contiguous committed cache
 *       k/v_pages     [num_blocks, Hkv, block_size, d] + block_table [B, max_blocks] (int32)
 *       logits        [B, Nmax, V]             (dtype)
 *     Q and K are taken after the positional encoding (RoPE) has been applied by the caller.
 *   - Alignment: every tensor pointer an entry point moves in 16-byte pieces (Q, K, V, O and
 *     the caches of the attention, the caches and tree K/V of the commit, every workspace) must
 *     be 16-byte aligned, else the call returns TSD_ERR_INVALID_ARG (TSD_ERR_WORKSPACE for a
 *     workspace) before any launch.  Logits may start anywhere: the vocabulary scans take their
 *     16-byte path only when the base pointer is 16-byte aligned and V % 8 == 0, and read one
 *     element at a time otherwise.
 *   - Return value: host-detected problems (null pointers, bad sizes, unsupported dtypes, a
 *     too small workspace, launch failures).  Problems that only the device can see
 *     (a malformed tree, a prefix past the cache capacity, a bad block-table entry, a bad
 *     path entry) are written to the per-sequence device word status[b] and never trap:
 *       status[b] = code | (detail << 8),  code = a tsd_status value, detail = the offending
 *       node (tree errors) or 0.
 *     A sequence whose status is non-zero on entry is skipped by every later call (its
 *     outputs are zero-filled where the call has outputs).  An error a call detects itself is
 *     stored into status[b] only if status[b] is still 0 (the first error wins); that
 *     sequence's outputs of that call are then zero-filled.
 *   - Environment knobs of the attention, read at each call (A/B runs and tests; the defaults
 *     are the measured choices): TSD_ATTN_PATH=mma (the warp-level mma.sync kernel where the
 *     tcgen05 kernel applies), TSD_ATTN_DUAL=0 (one query tile per CTA), TSD_ATTN_SPLITS=n (the
 *     tcgen05 kernel's key splits, when the workspace holds n partials), TSD_ATTN_MERGE=kernel|fused
 *     (where the splits are merged), TSD_ATTN_L2HINT=0 (no evict-first L2 policy on K/V tiles read
 *     once), TSD_TEST_WITHHOLD_TILE=t (test hook: the K producer skips
 *     key tile t and the bounded waits give up after 1e5 cycles, reporting TSD_ERR_TIMEOUT).
 */
#ifndef TSD_H_
#define TSD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tsd_status {
    TSD_OK = 0,
    TSD_ERR_INVALID_ARG = 1,       /* null pointer, bad size, Hq % Hkv != 0, d not 64/128, bad path entry */
    TSD_ERR_UNSUPPORTED_DTYPE = 2,
    TSD_ERR_BAD_TREE = 3,          /* parent[i] outside [-1, i): range / acyclicity ([EP] sec. 2) */
    TSD_ERR_TREE_DEPTH = 4,        /* depth(i) > Dmax: depth consistency ([EP] sec. 2) */
    TSD_ERR_TREE_ROOTS = 5,        /* a second root outside forest mode */
    TSD_ERR_CAPACITY = 6,          /* prefix + rows beyond the cache (or block table) capacity */
    TSD_ERR_TIMEOUT = 7,           /* a bounded device wait gave up (tcgen05 attention pipeline) */
    TSD_ERR_CUDA = 8,              /* a kernel launch failed (cudaGetLastError) */
    TSD_ERR_WORKSPACE = 9          /* workspace pointer null or smaller than the query said */
} tsd_status;

typedef enum tsd_dtype { TSD_F32 = 0, TSD_BF16 = 1 } tsd_dtype;

typedef enum tsd_commit_mode {
    TSD_COMMIT_PATH = 0,    /* gather tree rows path[j]-1 from the separate tree K/V buffer   */
    TSD_COMMIT_LENGTH = 1,  /* chain: tree rows 0..A (path ignored, may be NULL)               */
    TSD_COMMIT_INPLACE = 2  /* tree K/V already sits at cache positions L..L+N-1: compact it  */
} tsd_commit_mode;

#define TSD_STATUS_CODE(w) ((w) & 0xff)
#define TSD_STATUS_DETAIL(w) ((int32_t)((uint32_t)(w) >> 8))

/* Name of a status code (a static string). */
const char *tsd_status_str(int code);

/* ABI version of this header (bumped on any signature or contract change; 2: the attention
 * workspace starts with split-merge ticket words that must be zero before its first use). */
int tsd_abi_version(void);

/* ---------------------------------------------------------------------------------------
 * tsd_tree_prepare -- validate each draft tree and build its shifted-index tables
 * ([EP] sec. 2: shifted indexing with a dummy row 0, ancestor index tables, and range /
 * acyclicity / depth checks run before the fused kernels launch).
 *
 *   parent     [B, Nmax] int32   parent node of node i, -1 for a root; entries i >= N_b ignored
 *   num_nodes  [B] int32 or NULL N_b per sequence (NULL: every sequence has Nmax nodes);
 *                                N_b = 0 is allowed (an idle batch slot)
 *   Dmax                         deepest allowed depth (root depth 0), 0 <= Dmax <= 255
 *   forest                       0: exactly one root per tree; 1: any number of roots (an SSD
 *                                set of pre-drafted outcome subtrees, [SSD] sec. 2)
 *   parent_s   [B, Nmax+1] int32 out: parent slot of every slot (slot 0 and roots -> 0)
 *   depth      [B, Nmax+1] int32 out: depth of every slot (slot 0 -> 0)
 *   anc        [B, Nmax+1, Dmax+1] int32 out: anc[b][s][k] = slot of the depth-k ancestor of
 *                                slot s (k = depth(s) gives s itself), 0 beyond; row s is the
 *                                root->node path of s
 *   anc_bits   [B, Nmax+1, W] uint32 or NULL, W = ceil((Nmax+1)/32): bit t of row s set iff
 *                                slot t is an ancestor-or-self of slot s (slot 0 never set)
 *   status     [B] int32 out: 0, or TSD_ERR_BAD_TREE / _TREE_DEPTH / _TREE_ROOTS with the
 *                                first offending node as detail (checks run in node order:
 *                                range, then roots, then depth); TSD_ERR_INVALID_ARG when
 *                                N_b is outside [0, Nmax].  A flagged sequence's tables are
 *                                zero-filled.
 * --------------------------------------------------------------------------------------- */
tsd_status tsd_tree_prepare(const int32_t *parent, const int32_t *num_nodes, int B, int Nmax, int Dmax,
                            int forest, int32_t *parent_s, int32_t *depth, int32_t *anc, uint32_t *anc_bits,
                            int32_t *status, void *stream);

/* ---------------------------------------------------------------------------------------
 * tsd_tree_verify_attn -- tree-masked GQA attention of the verify step
 * ([EP] sec. 2: the 4D tree mask lets a token attend only to its ancestors on its own
 * branch, so branches cannot leak into each other; [SO] "EAGLE": tree verify needs a custom
 * mask, and masking a whole sequence costs up to half the attention speed, so here the mask
 * touches only the tree's own keys).
 *
 * For every sequence b, node i < N_b and query head h (KV head g = h / G):
 *   out[b,i,h,:] = softmax(scale * q[b,i,h,:] . K^T) V
 * over the keys {cache rows 0 .. L_b-1} U {tree node j : j is an ancestor of i or i itself}.
 *
 *   q                 [B, Nmax, Hq, d]  dtype
 *   k_cache, v_cache  [B, Hkv, Lmax, d] dtype, committed prefix of L_b = prefix_len[b] rows
 *   prefix_len        [B] int32 (device), 0 <= L_b; L_b > Lmax flags TSD_ERR_CAPACITY
 *   k_tree, v_tree    [B, Nmax, Hkv, d] dtype; both NULL = the tree K/V sit in the cache
 *                     at positions L_b .. L_b+N_b-1 (the layout TSD_COMMIT_INPLACE compacts)
 *   parent_s          [B, Nmax+1] int32 from tsd_tree_prepare; the mask is rebuilt from it in
 *                     shared memory by every CTA (walks are bounded by Dmax+1 steps)
 *   num_nodes         [B] int32 or NULL (NULL = Nmax)
 *   Hq, Hkv, d        Hq % Hkv == 0, d in {64, 128}
 *   dtype             TSD_BF16 (tensor-core path, fp32 accumulation) or TSD_F32 (FFMA path)
 *   scale             score scale, usually 1/sqrt(d)
 *   out               [B, Nmax, Hq, d] dtype; rows of nodes i >= N_b are not written
 *   lse               [B, Nmax, Hq] fp32 or NULL: log-sum-exp of the scaled scores (natural log)
 *   workspace         device scratch of at least tsd_tree_verify_attn_workspace_size() bytes;
 *                     may be NULL when that size is 0.  Its first
 *                     tsd_tree_verify_attn_ticket_bytes() bytes are split-merge ticket words
 *                     (the CTAs of one query block count themselves out and the last one
 *                     merges the key splits): zero the workspace once (cudaMemset) before its
 *                     first use; every call, error paths included, leaves them zero again.  A
 *                     ticket word holding a count no call leaves flags TSD_ERR_WORKSPACE in
 *                     status[b] and those rows are not written.  The rest holds the split-KV
 *                     partials.  Calls in flight at the same time need separate workspaces.
 *                     After a TSD_ERR_TIMEOUT, query blocks that had finished before the time-out
 *                     may keep their rows: status[b] is what marks the sequence.
 *   status            [B] int32 (see the conventions above)
 * --------------------------------------------------------------------------------------- */
size_t tsd_tree_verify_attn_workspace_size(int B, int Nmax, int Hq, int Hkv, int d, int Lmax, tsd_dtype dtype);

/* Size of the ticket region at the start of an attention workspace (a constant). */
size_t tsd_tree_verify_attn_ticket_bytes(void);

/* Number of kernels one tsd_tree_verify_attn[_paged] call launches on its stream for these sizes
 * (1: the split kernel alone, its key splits merged inside it or not split; 2: followed by the
 * merge kernel), for 16-byte-aligned tensors and a workspace of the queried size.  Lmax is the
 * capacity (max_blocks * block_size for the paged call), block_size 0 for the contiguous cache,
 * tree_in_cache 1 when k_tree / v_tree are NULL.  A host function; 0 for invalid sizes. */
int tsd_tree_verify_attn_kernels(int B, int Nmax, int Hq, int Hkv, int d, int Lmax, int block_size, int tree_in_cache,
                                 tsd_dtype dtype);

/* CTAs of the attention call's split kernel for the same arguments (its grid: a caller that runs
 * other work beside the attention can tell whether the grid alone fills the GPU).  0 for invalid
 * sizes. */
long long tsd_tree_verify_attn_ctas(int B, int Nmax, int Hq, int Hkv, int d, int Lmax, int block_size,
                                    int tree_in_cache, tsd_dtype dtype);

tsd_status tsd_tree_verify_attn(const void *q, const void *k_cache, const void *v_cache, int Lmax,
                                const int32_t *prefix_len, const void *k_tree, const void *v_tree,
                                const int32_t *parent_s, const int32_t *num_nodes, int B, int Nmax, int Hq,
                                int Hkv, int d, int Dmax, tsd_dtype dtype, float scale, void *out, float *lse,
                                void *workspace, size_t ws_bytes, int32_t *status, void *stream);

/* Paged-cache variant: the cache is k_pages/v_pages [num_blocks, Hkv, block_size, d] and
 * position p of sequence b lives in block block_table[b][p / block_size] at row
 * p % block_size.  block_size must be a power of two in [8, 256].  The capacity of sequence
 * b is max_blocks * block_size; a block id outside [0, num_blocks) flags
 * TSD_ERR_CAPACITY.  Everything else is as in tsd_tree_verify_attn. */
size_t tsd_tree_verify_attn_paged_workspace_size(int B, int Nmax, int Hq, int Hkv, int d, int max_blocks,
                                                 int block_size, tsd_dtype dtype);

tsd_status tsd_tree_verify_attn_paged(const void *q, const void *k_pages, const void *v_pages, int num_blocks,
                                      int block_size, const int32_t *block_table, int max_blocks,
                                      const int32_t *prefix_len, const void *k_tree, const void *v_tree,
                                      const int32_t *parent_s, const int32_t *num_nodes, int B, int Nmax,
                                      int Hq, int Hkv, int d, int Dmax, tsd_dtype dtype, float scale, void *out,
                                      float *lse, void *workspace, size_t ws_bytes, int32_t *status,
                                      void *stream);

/* ---------------------------------------------------------------------------------------
 * tsd_tree_accept_greedy -- greedy acceptance over the tree
 * ([SO] "Decodificacion especulativa": the longest accepted prefix wins and the target
 * gives one extra token, so n drafted tokens can yield n+1; "EAGLE": among tree branches the
 * longest suitable one continues, plus the target's extra token; [SSD] sec. 2: with a forest
 * of pre-drafted outcomes the real verify outcome either hits one of them or misses).
 *
 * t*(i) = argmax_v logits[b,i,v] (ties -> lowest v; NaN never wins; an all -inf/NaN row -> 0).
 * A root is accepted unconditionally when root_key is NULL; otherwise only the lowest-index
 * root with tokens[b,root] == root_key[b] is accepted (hit) and none when no root matches
 * (miss).  A non-root i is accepted iff its parent p is and tokens[b,i] == t*(p).
 * a* = the accepted node of greatest depth (ties -> lowest index).
 *
 *   logits      [B, Nmax, V] dtype; V % 8 == 0 is fastest (any V >= 1 works)
 *   tokens      [B, Nmax] int32 draft token of every node (a root's token is the token it stands for)
 *   parent_s    [B, Nmax+1] int32 from tsd_tree_prepare
 *   root_key    [B] int32 or NULL
 *   accept_len  [B] int32 out: depth(a*), or -1 on a miss / N_b == 0 / a flagged sequence
 *   path        [B, Dmax+1] int32 out: slots of the root->a* path (path[0] = root slot), 0 beyond
 *   out_tokens  [B, Dmax+1] int32 out: tokens of path nodes 1..A then t*(a*), -1 beyond
 *   workspace   >= tsd_tree_accept_greedy_workspace_size(B, Nmax, V) bytes
 * --------------------------------------------------------------------------------------- */
size_t tsd_tree_accept_greedy_workspace_size(int B, int Nmax, int V);

tsd_status tsd_tree_accept_greedy(const void *logits, tsd_dtype dtype, int V, const int32_t *tokens,
                                  const int32_t *parent_s, const int32_t *num_nodes, const int32_t *root_key,
                                  int B, int Nmax, int Dmax, int32_t *accept_len, int32_t *path,
                                  int32_t *out_tokens, void *workspace, size_t ws_bytes, int32_t *status,
                                  void *stream);

/* ---------------------------------------------------------------------------------------
 * tsd_tree_accept_threshold -- threshold acceptance over the tree
 * ([SO] "Decodificacion especulativa": besides exact matching, the target may keep the longest
 * prefix whose tokens stay above an acceptance threshold; the page gives no formula).  Reading:
 * with p_n = softmax(logits[b,n] / T), a non-root node i is accepted iff its parent is accepted
 * and p_parent(i)(tokens[b,i]) >= tau (fp64 comparison); roots, the deepest-node rule, the path
 * and the emitted tokens (the last one = argmax of the deepest accepted node's row) are exactly
 * those of tsd_tree_accept_greedy.  tau = 0 accepts every node; tau > 1/2 accepts only argmax
 * tokens.
 *
 *   logits, tokens, parent_s, num_nodes, root_key, outputs, status: as tsd_tree_accept_greedy
 *   tau           threshold in [0, 1];  temperature > 0
 *   workspace     >= tsd_tree_accept_threshold_workspace_size(B, Nmax, V) bytes
 * Two launches (the vocabulary scan, then one CTA per sequence); Nmax <= 4096.
 * --------------------------------------------------------------------------------------- */
size_t tsd_tree_accept_threshold_workspace_size(int B, int Nmax, int V);

tsd_status tsd_tree_accept_threshold(const void *logits, tsd_dtype dtype, int V, const int32_t *tokens,
                                     const int32_t *parent_s, const int32_t *num_nodes, const int32_t *root_key,
                                     float tau, float temperature, int B, int Nmax, int Dmax,
                                     int32_t *accept_len, int32_t *path, int32_t *out_tokens, void *workspace,
                                     size_t ws_bytes, int32_t *status, void *stream);

/* ---------------------------------------------------------------------------------------
 * tsd_tree_accept_greedy_noalloc -- tsd_tree_accept_greedy for callers that cannot allocate.
 * The pages have no counterpart of this call; it exists for library users whose code may not
 * call cudaMalloc: a serving engine that gave all free device memory to its KV-cache pool at
 * start-up, or a plug-in that a host runtime hands device pointers but no allocator.
 *
 * Same arguments, outputs and results as tsd_tree_accept_greedy, without the workspace: the
 * scratch is a fixed array of TSD_ACCEPT_NOALLOC_SCRATCH_BYTES inside the library, present on
 * every device that loads it until the process exits.  The call allocates nothing.
 *   - A batch whose scratch need, tsd_tree_accept_greedy_workspace_size(B, Nmax, V), exceeds
 *     TSD_ACCEPT_NOALLOC_SCRATCH_BYTES is refused with TSD_ERR_WORKSPACE before any launch
 *     (1 MiB holds e.g. B*Nmax = 8192 rows of a 128256-token vocabulary).
 *   - The first call on a device looks up the array's device address (with that device
 *     current) and caches it; make that first call before any stream capture.  The cached
 *     address belongs to the device's primary context: after cudaDeviceReset on that device
 *     the library must be reloaded before this call is used again.
 *   - Every call shares the one array: calls that overlap on the GPU (other streams, other
 *     host threads) race and must be serialised by the caller.
 * --------------------------------------------------------------------------------------- */
#define TSD_ACCEPT_NOALLOC_SCRATCH_BYTES (1u << 20)

/* Size of that fixed array as compiled into the loaded library (equals
 * TSD_ACCEPT_NOALLOC_SCRATCH_BYTES of the header it was built with). */
size_t tsd_tree_accept_greedy_noalloc_scratch_bytes(void);

tsd_status tsd_tree_accept_greedy_noalloc(const void *logits, tsd_dtype dtype, int V, const int32_t *tokens,
                                          const int32_t *parent_s, const int32_t *num_nodes,
                                          const int32_t *root_key, int B, int Nmax, int Dmax,
                                          int32_t *accept_len, int32_t *path, int32_t *out_tokens,
                                          int32_t *status, void *stream);

/* ---------------------------------------------------------------------------------------
 * tsd_chain_accept_sample -- rejection sampling of a linear draft of K tokens
 * ([SO] "Objetivo-Borrador": acceptance compares the full draft and target distributions and
 * the target's logits after the accepted run are sampled for one more token; the rule is the
 * one of the Leviathan et al. paper the page cites).
 *
 * With p_k = softmax(target_logits[b,k]/T) and q_k = softmax(draft_logits[b,k]/T) (fp32):
 * for k = 0..K-1 accept draft_tokens[b,k] iff u[b,k] * q_k(x) < p_k(x) (probability
 * min(1, p/q)); at the first rejection j the last token is the smallest t with
 * sum_{v<=t} r_v > u[b,K] * sum_v r_v for r = max(p_j - q_j, 0) (p_j if r sums to 0); with all
 * K accepted it is drawn the same way from p_K.  T == 0 is greedy (argmax tests, argmax token).
 *
 *   target_logits [B, K+1, V] dtype (row k: target logits after the k-th chain node, root first)
 *   draft_logits  [B, K, V]   dtype (row k: the distribution draft token k was drawn from)
 *   draft_tokens  [B, K] int32;  uniforms [B, K+1] fp32 in [0,1)
 *   accept_len    [B] int32 out: accepted drafts A (0..K)
 *   out_tokens    [B, K+1] int32 out: the A accepted drafts then the drawn token, -1 beyond
 *   workspace     >= tsd_chain_accept_sample_workspace_size(B, K, V) bytes
 * The chain's tree is the path 0..K, so the commit that follows is TSD_COMMIT_LENGTH.
 * --------------------------------------------------------------------------------------- */
size_t tsd_chain_accept_sample_workspace_size(int B, int K, int V);

tsd_status tsd_chain_accept_sample(const void *target_logits, const void *draft_logits, tsd_dtype dtype, int V,
                                   const int32_t *draft_tokens, const float *uniforms, float temperature, int B,
                                   int K, int32_t *accept_len, int32_t *out_tokens, void *workspace,
                                   size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------------------
 * tsd_tree_accept_sample -- stochastic acceptance of a draft tree (temperature > 0)
 * ([SO] "Objetivo-Borrador": accept a draft token with probability min(1, p/q), the rule of the
 * cited Leviathan et al. paper, and sample one more token from the target after the accepted
 * run; [SO] "EAGLE": the draft is a tree of candidates).  Reading for a tree whose children were
 * drawn independently from their parent's draft distribution: starting at the root (node 0), the
 * children of the current node are tried in index order; child c with token x is accepted iff
 *   u[b,c] * q(x) < p(x),
 * and after each rejection p is replaced by max(p - q, 0) / sum (kept when that sum is 0), so
 * the next child is tested against the residual the earlier rejections left.  Acceptance moves
 * to the accepted child and repeats; when no child is accepted (or the node is a leaf, or depth
 * Dmax is reached) the last token is the smallest t with sum_{v<=t} p(v) > u[b,0] * sum_v p(v)
 * for the current p.  p = softmax(target_logits[b,n] / T), q = softmax(draft_logits[b,n] / T)
 * at node n.  With one child per node this is tsd_chain_accept_sample's rule.
 *
 *   target_logits [B, Nmax, V] dtype: row n = the target distribution after node n
 *   draft_logits  [B, Nmax, V] dtype: row n = the draft distribution node n's children were drawn
 *                 from (rows of leaves are not read)
 *   tokens        [B, Nmax] int32; parent_s [B, Nmax+1] from tsd_tree_prepare (single-root trees:
 *                 forest = 0)
 *   uniforms      [B, Nmax] fp32 in [0,1): entry c (c >= 1) for the test of node c, entry 0 for
 *                 the final draw
 *   temperature   > 0 (use tsd_tree_accept_greedy for T = 0)
 *   accept_len, path, out_tokens as in tsd_tree_accept_greedy (path = slots of the accepted nodes,
 *                 out_tokens = the accepted drafts below the root, then the drawn token, -1 beyond)
 *   status        [B] int32: a flagged sequence is skipped (accept_len -1); a node on the walk with
 *                 more than 256 children flags TSD_ERR_INVALID_ARG (detail = that node)
 * V is bounded by shared memory: 2 * ceil(V / 8) * sizeof(dtype) + 4 * Nmax <= 200 KiB.
 * One launch (a cluster of 8 CTAs per sequence), no workspace.
 * --------------------------------------------------------------------------------------- */
tsd_status tsd_tree_accept_sample(const void *target_logits, const void *draft_logits, tsd_dtype dtype, int V,
                                  const int32_t *tokens, const int32_t *parent_s, const int32_t *num_nodes,
                                  const float *uniforms, float temperature, int B, int Nmax, int Dmax,
                                  int32_t *accept_len, int32_t *path, int32_t *out_tokens, int32_t *status,
                                  void *stream);

/* ---------------------------------------------------------------------------------------
 * tsd_ssd_cache_build -- the outcome cache of one SSD / Saguaro verification round
 * ([SSD] sec. 2 and sec. 3 A-B: while the target verifies, the draft predicts the outcome --
 * the accepted length and the bonus token -- and pre-drafts for the likely outcomes; the cache
 * budget follows a geometric fan-out over the likely accepted lengths; Saguaro sampling lowers
 * the draft probability of the cached tokens while drafting).  Reading of those passages:
 *   P(a) = alpha^a (1 - alpha) for a < K, P(K) = alpha^K   (accepted length a of K drafts);
 *   slots[b,a] = the largest-remainder apportionment of S slots in proportion to P(a)
 *     (floor(S P(a)), then +1 to the largest remainders, ties -> shorter length);
 *   the slots[b,a] outcome keys of length a are the most likely tokens of the draft distribution
 *     at position a+1, q_a = softmax(draft_logits[b,a] / T) (ties -> lower id);
 *   draft_tokens[b,j] (j < K) = the smallest t with sum_{v<=t} q'(v) > u[b,j] * sum_v q'(v),
 *     q' = q_j * (beta on the keys of length j, 1 elsewhere), renormalised (q_j if that sum is 0).
 *
 *   draft_logits  [B, K+1, V] dtype: row a = the draft logits at position a+1 (row K: the free
 *                 token after K accepted drafts; keys only)
 *   alpha         [B] fp32 per-sequence acceptance rate (clamped to [0, 1])
 *   beta          in [0, 1];  uniforms [B, K] fp32 in [0, 1);  temperature > 0
 *   slots         [B, K+1] int32 out: slots per accepted length (sum S)
 *   key_len, key_tok [B, S] int32 out: the outcome keys (accepted length, bonus token), ordered by
 *                 length, then by draft probability (desc), then token id
 *   draft_tokens  [B, K] int32 out
 * Limits: 1 <= S <= 256, S <= V, 0 <= K <= 63, ceil(V / 8) * sizeof(dtype) <= 200 KiB.
 * One launch (a cluster of 8 CTAs per (sequence, row)), no workspace.
 * --------------------------------------------------------------------------------------- */
tsd_status tsd_ssd_cache_build(const void *draft_logits, tsd_dtype dtype, int V, int K, int S, const float *alpha,
                               float beta, const float *uniforms, float temperature, int B, int32_t *slots,
                               int32_t *key_len, int32_t *key_tok, int32_t *draft_tokens, void *stream);

/* ---------------------------------------------------------------------------------------
 * tsd_kv_commit -- commit the accepted path's K/V rows into the contiguous cache
 * ([EP] sec. 2, branchable KV cache: committed prefix state is kept apart from per-branch
 * speculative state; commit either keeps the first A steps (length) or follows the path
 * indices, moving only what must move).  Here the speculative state is the separate tree
 * K/V buffer, so nothing outside the accepted path is ever written to the cache.
 *
 * For every sequence with A = accept_len[b] >= 0 and status[b] == 0, L = prefix_len[b]:
 *   cache[b, :, L+j, :] <- source row j  for j = 0..A   (K and V, every KV head), then
 *   prefix_len[b] = L + A + 1   (on the device).
 * Source row j: PATH: k_tree[b, path[b][j]-1]; LENGTH: k_tree[b, j]; INPLACE: the cache
 * row at L + path[b][j]-1 (all sources are read before any row is written; rows already in
 * place are skipped).  A miss (A < 0) is a no-op.  L + A + 1 > Lmax flags TSD_ERR_CAPACITY, a
 * path entry outside 1..N_b flags TSD_ERR_INVALID_ARG, and A > Dmax flags TSD_ERR_INVALID_ARG;
 * a flagged sequence's cache and prefix_len are left untouched.
 *
 *   path          [B, Dmax+1] int32 slots (tsd_tree_accept_greedy's output); NULL in LENGTH mode
 *   num_nodes     [B] int32 or NULL (NULL = Nmax), bounds the path entries
 *   k_tree/v_tree unused (may be NULL) in INPLACE mode
 * --------------------------------------------------------------------------------------- */
tsd_status tsd_kv_commit(void *k_cache, void *v_cache, int Lmax, int32_t *prefix_len, const void *k_tree,
                         const void *v_tree, const int32_t *path, const int32_t *accept_len,
                         const int32_t *num_nodes, int B, int Nmax, int Hkv, int d, int Dmax, tsd_dtype dtype,
                         tsd_commit_mode mode, int32_t *status, void *stream);

/* Paged-cache variant (layout as in tsd_tree_verify_attn_paged; capacity max_blocks *
 * block_size; a block id outside [0, num_blocks) flags TSD_ERR_CAPACITY). */
tsd_status tsd_kv_commit_paged(void *k_pages, void *v_pages, int num_blocks, int block_size,
                               const int32_t *block_table, int max_blocks, int32_t *prefix_len,
                               const void *k_tree, const void *v_tree, const int32_t *path,
                               const int32_t *accept_len, const int32_t *num_nodes, int B, int Nmax, int Hkv,
                               int d, int Dmax, tsd_dtype dtype, tsd_commit_mode mode, int32_t *status,
                               void *stream);

/* ---------------------------------------------------------------------------------------
 * tsd_tree_accept_commit -- greedy tree acceptance and the commit of the accepted path in one
 * step, with an optional splice of the emitted tokens into a device token history
 * ([EP] sec. 2: commit follows the accepted path's indices; [SO] "EAGLE": longest matching
 * branch plus the target's own token; the accepted length drives the next step's cache length
 * on the device, with no host synchronisation).
 *
 * Same results as tsd_tree_accept_greedy followed by tsd_kv_commit[_paged] with the same
 * arguments: accept_len, path and out_tokens as there, the cache rows and prefix_len as there.
 * In addition, when history is not NULL, for every committed sequence
 *   history[b, H .. H+A] <- out_tokens[b, 0 .. A],  history_len[b] = H + A + 1,
 * with H = history_len[b]; H < 0 or H + A + 1 > history_cap flags TSD_ERR_CAPACITY before any
 * cache write (the acceptance outputs are still written).
 *
 *   cache       the committed K/V cache (struct below: contiguous when block_table is NULL,
 *               else paged with the layout of tsd_tree_verify_attn_paged); prefix_len in/out
 *   mode        TSD_COMMIT_PATH or TSD_COMMIT_INPLACE (LENGTH commits the first A+1 tree rows)
 *   history     [B, history_cap] int32 device memory, or NULL (no splice; history_len unused)
 *   workspace   >= tsd_tree_accept_greedy_workspace_size(B, Nmax, V) bytes
 * Errors as the two calls it replaces.  Two kernel launches on `stream` (the vocabulary scan,
 * then one CTA per sequence for acceptance, commit and splice); nothing is allocated.
 * --------------------------------------------------------------------------------------- */
typedef struct tsd_kv_cache {
  void *k;                     /* [B, Hkv, Lmax, d] or [num_blocks, Hkv, block_size, d] */
  void *v;
  int32_t *prefix_len;         /* [B] committed lengths, advanced on the device */
  int Lmax;                    /* contiguous capacity per sequence (ignored when paged) */
  const int32_t *block_table;  /* [B, max_blocks] block ids, or NULL for the contiguous layout */
  int max_blocks;
  int block_size;              /* power of two in [8, 256] when paged */
  int num_blocks;
} tsd_kv_cache;

tsd_status tsd_tree_accept_commit(const void *logits, tsd_dtype logits_dtype, int V, const int32_t *tokens,
                                  const int32_t *parent_s, const int32_t *num_nodes, const int32_t *root_key,
                                  int B, int Nmax, int Dmax, const tsd_kv_cache *cache, const void *k_tree,
                                  const void *v_tree, int Hkv, int d, tsd_dtype kv_dtype, tsd_commit_mode mode,
                                  int32_t *history, int history_cap, int32_t *history_len, int32_t *accept_len,
                                  int32_t *path, int32_t *out_tokens, void *workspace, size_t ws_bytes,
                                  int32_t *status, void *stream);

/* ---------------------------------------------------------------------------------------
 * Device-side draft tree build (EAGLE-2 style): tsd_draft_tree_init / _expand / _finalize
 * ([SO] "EAGLE": EAGLE-2 shapes the tree dynamically from the Top-K candidates of every node
 * and scores the draft sequences).  Reading of that passage: a node's children are its K most
 * likely draft tokens (ties -> lower token id), a node's score is the cumulative draft
 * log-probability of its root->node path, the next nodes to expand are the F best children
 * (score desc, then node index), and the final tree keeps the root plus the keep-1 best nodes
 * (same order), renumbered by (depth, score desc, node index) with parents remapped -- the
 * parent[] / tokens the verify step takes.  The tree lives on the device between draft steps.
 *
 * tsd_draft_tree holds caller-owned device arrays:
 *   parent, token, depth [B, max_nodes] int32; score [B, max_nodes] fp64;
 *   num_nodes [B]; frontier [B, F] (node ids, best first); num_frontier [B];
 *   F <= 16 frontier width.
 * init: node 0 = root (token root_token[b], score 0), frontier = [0]; status[b] = 0.
 * expand: draft_logits [B, F, V] (row f = the draft distribution after frontier node f; rows
 *   past num_frontier[b] are ignored), K <= min(16, V) children per node, V <= 64 * 16384; appends
 *   num_frontier * K nodes (in frontier order, then rank order) and replaces the frontier.
 *   Scores: fp32 exponentials summed in fp64, log-sum-exp and scores in fp64.  Capacity
 *   overflow flags TSD_ERR_CAPACITY in status[b] and leaves the tree unchanged.
 *   workspace >= tsd_draft_tree_expand_workspace_size(B, F, K, V) bytes.  Two launches.
 * finalize: parent_out [B, keep] int32 (root -1, padding -1), tokens_out [B, keep] (padding 0),
 *   num_nodes_out [B] = min(keep, nodes); max_nodes <= 4096.  One launch.
 * A flagged sequence (status[b] != 0) is skipped by expand and finalised empty.
 * --------------------------------------------------------------------------------------- */
typedef struct tsd_draft_tree {
  int32_t *parent;
  int32_t *token;
  double *score;
  int32_t *depth;
  int32_t *num_nodes;
  int32_t *frontier;
  int32_t *num_frontier;
  int max_nodes;
  int F;
} tsd_draft_tree;

tsd_status tsd_draft_tree_init(const tsd_draft_tree *tree, const int32_t *root_token, int B, int32_t *status,
                               void *stream);
size_t tsd_draft_tree_expand_workspace_size(int B, int F, int K, int V);
tsd_status tsd_draft_tree_expand(const tsd_draft_tree *tree, const void *draft_logits, tsd_dtype dtype, int V, int K,
                                 int B, void *workspace, size_t ws_bytes, int32_t *status, void *stream);
tsd_status tsd_draft_tree_finalize(const tsd_draft_tree *tree, int B, int keep, int32_t *parent_out,
                                   int32_t *tokens_out, int32_t *num_nodes_out, int32_t *status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TSD_H_ */
