// Tree-verify attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Same operation and work decomposition as the split kernels in attn.cu ("EAGLE-Pangu", technical
// summary sec. 2: a tree token attends to the committed prefix and to its own ancestors only;
// "Acelerando Sonar a traves de la especulacion", section "EAGLE": the mask touches only the
// tree's keys), built for Blackwell:
//   * a CTA owns 128 query rows (G heads x 128/G tree nodes of one KV head), or two such tiles
//     when a KV head has more than 128 rows, and a range of 64-key tiles of one sequence; every
//     K/V tile is read from memory once per CTA;
//   * two producer threads stream K and V tiles with TMA (128-byte swizzled boxes; paged caches
//     box by block, the tree's K/V by node for one KV head) into separate rings: a K slot is
//     released as soon as S = Q K^T has read it, a V slot after P V, so loads run several tiles
//     ahead of the math;
//   * warp 3 issues tcgen05.mma warp-collectively (one elected lane; descriptors built once and
//     advanced by constants): S into TMEM tiles of 128 lanes x 64 fp32 columns (two per softmax
//     warpgroup with one query tile, so the tensor cores compute a warpgroup's next S while it
//     is still exponentiating the current one) and O += P V into two 128 x 128 fp32 TMEM
//     accumulators;
//   * P never touches shared memory: the softmax writes it as bf16 over the first half of its S
//     tile in TMEM and the P V product reads its A operand from there; with two query tiles the
//     tiles themselves live in TMEM too (the A operand of S), so shared memory carries only the
//     TMA writes and the K and V operand reads;
//   * one query tile: two softmax warpgroups take alternate key tiles (even / odd), each with its
//     own S tiles, O accumulator and running (max, sum) -- a split of the key range inside the
//     CTA, merged by log-sum-exp in the epilogue; two query tiles: warpgroup w owns query tile w
//     over every key tile.  In a warpgroup each warp owns one TMEM lane quarter, one query row
//     per thread: a row's 64 scores come out of TMEM with one tcgen05.ld, so its max and sum need
//     no shuffles.  The ancestor mask is applied only on tree tiles (bits built in shared memory
//     by warp 1 from the staged parent slots while the first prefix tiles stream in); full
//     prefix tiles take a lean path (no mask work, paired fp32 instructions).  The running max is
//     raised lazily (only past a 2^8 growth), so O is rescaled in TMEM rarely;
//   * the epilogue stages finished rows in the idle K/V rings and writes them out with coalesced
//     16-byte stores.
// Every mbarrier wait is bounded: on time-out the CTA records TSD_ERR_TIMEOUT, drains its own
// TMA copies (again bounded) and frees its TMEM before returning.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cstdlib>
#include <mutex>

#include "attn_common.cuh"
#include "common.cuh"
#include "kernels.h"
#include "umma.cuh"

namespace tsd {

namespace {

using namespace attn;
using namespace umma;

constexpr int kBM = 128, kBN = 64, kD = 128;
constexpr int kThreadsU = 384;                    // 12 warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256;         // O_w at 128*w; S of tile i at 256 + 64*(i%4)
constexpr int kSBufs = 4;                          // S tiles in TMEM: two per softmax warpgroup
// Two-query-tile CTAs: S_w at 256 + 64*w (one per warpgroup) and the query tile Q_w itself at
// 384 + 64*w (bf16 pairs), the A operand of S = Q K^T read from TMEM instead of shared memory.
constexpr uint32_t kColQ = 384;
// Epilogue staging rows in shared memory (the K/V rings are idle by then), padded by 16 bytes so
// that the 32 rows a warp writes at once spread over all banks.
constexpr uint32_t kStageF = kD * 4 + 16;   // fp32 split partial row
constexpr uint32_t kStageH = kD * 2 + 16;   // bf16 output row
constexpr uint32_t kHalf = kBN * 128;              // one 64-column half of a K or V tile: 8 KB
constexpr uint32_t kSlot = 2 * kHalf;              // one K or V tile: 16 KB
constexpr uint32_t kQBytes = kBM * 256;            // 32 KB
constexpr int kMaxRing = 6;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;               // lazy max: rescale only past a 2^8 growth

struct UParams {
  int splits;          // CTAs splitting one (sequence, KV head, row block)'s keys, equal shares
  int Rmax;            // query rows per (sequence, KV head): the partials' row stride
  int mtiles;
  long long wait;      // cycles after which an mbarrier wait gives up (TSD_ERR_TIMEOUT)
  int withhold;        // test hook: the K producer never issues this tile (-1: off)
  int lpt;             // map blockIdx.z to sequences by decreasing prefix length (B <= threads)
  int ks, vs;          // K and V ring depths
  int box_rows;        // rows per TMA box of the cache (64 contiguous, min(block, 64) paged)
  int W;               // ancestor-bit words per node
  int stage;           // epilogue rows go through shared memory (the ring region is large enough)
  int* tickets;        // split merge in the kernel: one ticket word per row block (null: merge kernel)
  int evict_first;     // the cache's K/V tiles are read once: load them with an evict-first L2 policy
  uint32_t k_off, v_off, mask_off, ps_off;   // shared-memory offsets
};

struct __align__(8) Bars {
  uint64_t q_full;
  uint64_t k_full[kMaxRing], k_empty[kMaxRing];
  uint64_t v_full[kMaxRing], v_empty[kMaxRing];
  uint64_t s_full[kSBufs];  // S tile of key tile i (buffer i % 4) is in TMEM
  uint64_t p_full[2];    // warpgroup w: its P tile is in shared memory (and its S tile was read)
  uint64_t pv_done[2];   // warpgroup w: its last P V product finished (P buffer free, O current)
  uint64_t mask_full;    // the ancestor bits of the tree tiles are in shared memory
  uint64_t fin;
};

// 2^x with the hardware approximation (flush-to-zero; 2^-inf = 0).  P is rounded to bf16 anyway.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Paired fp32 arithmetic of sm_100 (one instruction for two lanes of work) and the three-input
// maximum: the lean full-tile softmax issues a third fewer instructions with them.
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0, float c1) {
  asm("{\n"
      ".reg .b64 ra, rb, rc, rd;\n"
      "mov.b64 ra, {%2, %3};\n"
      "mov.b64 rb, {%4, %5};\n"
      "mov.b64 rc, {%6, %7};\n"
      "fma.rn.f32x2 rd, ra, rb, rc;\n"
      "mov.b64 {%0, %1}, rd;\n"
      "}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n"
      ".reg .b64 ra, rb, rd;\n"
      "mov.b64 ra, {%2, %3};\n"
      "mov.b64 rb, {%4, %5};\n"
      "add.rn.f32x2 rd, ra, rb;\n"
      "mov.b64 {%0, %1}, rd;\n"
      "}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ void abort_cta(const AttnArgs& a, int b, volatile int* s_abort) {
  if (*s_abort == 0) {
    *s_abort = 1;
    flag_status(a.status, b, TSD_ERR_TIMEOUT);
  }
}

// Block ids of the boxes of prefix tile t (paged caches): loaded one tile ahead by the producers so
// the table reads never wait in line behind the TMA issues.
struct TileBlocks {
  int blk[8];
};
__device__ __forceinline__ void fetch_blocks(const AttnArgs& a, const SeqView& v, const UParams& u, int b, int t,
                                             TileBlocks& tb) {
  if (a.block_table == nullptr || t >= v.nPT) return;
  const int pos0 = t * kBN;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int seg = k * u.box_rows;
    if (seg < kBN) tb.blk[k] = a.block_table[(size_t)b * a.max_blocks + min((pos0 + seg) >> a.block_shift,
                                                                             a.max_blocks - 1)];
  }
}

// TMA loads of one 64-key tile (K or V half pair) of sequence b, KV head g into `dst`.
__device__ __forceinline__ void load_tile(const AttnArgs& a, const SeqView& v, const UParams& u, int b, int g,
                                          int t, uint8_t* dst, const CUtensorMap* cache_map,
                                          const CUtensorMap* tree_map, uint64_t* bar, int* s_err,
                                          const TileBlocks& tb, uint64_t pol) {
  // cache tiles go in under the producer's L2 policy: evict-first when the whole grid reads each
  // tile once (the split partials written meanwhile then stay in L2 for the merge)
  auto load2 = [&](uint8_t* d, int x, int y) { tma_load_2d_hint(d, cache_map, x, y, bar, pol); };
  if (t < v.nPT) {
    const int pos0 = t * kBN;
    if (a.block_table == nullptr) {
      const int y = (b * a.Hkv + g) * a.Lcap + pos0;
      load2(dst, 0, y);
      load2(dst + kHalf, 64, y);
    } else {
      const int bs_mask = (1 << a.block_shift) - 1;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int seg = k * u.box_rows;
        if (seg >= kBN) break;
        const int pos = pos0 + seg;
        int blk = tb.blk[k];
        if (blk < 0 || blk >= a.num_blocks) {
          if (pos < v.L) *s_err = 1;
          blk = 0;
        }
        const int y = (blk * a.Hkv + g) * (1 << a.block_shift) + (pos & bs_mask);
        const uint32_t off = (uint32_t)seg * 128;
        load2(dst + off, 0, y);
        load2(dst + kHalf + off, 64, y);
      }
    }
  } else {
    const int z = b * a.Nmax + (t - v.nPT) * kBN;
    tma_load_3d(dst, tree_map, 0, g, z, bar);
    tma_load_3d(dst + kHalf, tree_map, 64, g, z, bar);
  }
}

// kDual: the CTA owns two 128-row query tiles of the same KV head and streams every K/V tile once
// for both (warpgroup w owns query tile w over all key tiles); otherwise one query tile whose key
// tiles alternate between the two warpgroups.
// Split merge inside the kernel.  Every CTA of a (sequence, KV head, row block) publishes its
// partial, then takes a ticket from the row block's word; the CTA that draws the last ticket merges
// the partials and writes the output, and returns the word to zero for the next call.  No CTA
// waits for another.  Returns 1 to the last CTA, 2 when the word held a count no call leaves
// behind (the workspace was not zeroed before its first use), else 0.
__device__ __forceinline__ int take_ticket(int* word, int splits, int* s_flag) {
  __threadfence();   // this thread's partial stores, before the ticket
  __syncthreads();
  if (threadIdx.x == 0) {
    const int old = atomicAdd(word, 1);
    const int r = old == splits - 1 ? 1 : ((old < 0 || old >= splits) ? 2 : 0);
    if (r == 1) atomicExch(word, 0);
    __threadfence();
    *s_flag = r;
  }
  __syncthreads();
  return *s_flag;
}

// The last CTA's merge (all threads).  (1) Every split's (max, sum) of every row into shared memory
// with independent loads; (2) per row the largest split maximum, the splits' weights
// 2^(M_s - M) / sum (s_w[s][row]) and the log-sum-exp; (3) every (row, 8 columns) the weighted sum
// of the partial rows, two such pieces per thread and two splits per round so that several loads are
// in flight, written as bf16.  This CTA's own partial is read from its staged rows in shared memory,
// the others' from L2 (.cg: written by other SMs).  A split with no mass (M = -inf) has weight 0 and
// its rows are never read.  Zero rows when the sequence is flagged or out of capacity.
__device__ void merge_splits(const AttnArgs& a, const UParams& u, int b, int g, int G, int r0, int r_hi, int own,
                             bool zero, const uint8_t* sStage, float* s_w, int rows_cap) {
  if (zero) {
    zero_rows<__nv_bfloat16>(a, b, g, G, r0, r_hi);
    return;
  }
  const int nrows = r_hi - r0, ns = u.splits, bd = blockDim.x;
  const float* wo = reinterpret_cast<const float*>(a.workspace);
  const float* wml = wo + (size_t)a.B * a.Hkv * ns * u.Rmax * kD;
  const size_t base = ((size_t)b * a.Hkv + g) * ns * u.Rmax + r0;   // + s * Rmax + row
  float2* s_ml = reinterpret_cast<float2*>(s_w + ns * rows_cap);      // [s][row]
  const int npairs = ns * nrows;
  for (int i0 = threadIdx.x; i0 < npairs; i0 += 4 * bd) {
    float2 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int idx = i0 + j * bd, sp = idx / nrows, cr = idx - sp * nrows;
      if (idx < npairs) v[j] = __ldcg(reinterpret_cast<const float2*>(wml + (base + (size_t)sp * u.Rmax + cr) * 2));
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int idx = i0 + j * bd, sp = idx / nrows, cr = idx - sp * nrows;
      if (idx < npairs) s_ml[sp * rows_cap + cr] = v[j];
    }
  }
  __syncthreads();
  for (int cr = threadIdx.x; cr < nrows; cr += bd) {
    float M = -INFINITY;
    for (int sp = 0; sp < ns; ++sp) M = fmaxf(M, s_ml[sp * rows_cap + cr].x);
    const float Mu = M == -INFINITY ? 0.f : M;
    float l = 0.f;
    for (int sp = 0; sp < ns; ++sp) {
      const float2 ml = s_ml[sp * rows_cap + cr];
      const float w = ml.x == -INFINITY ? 0.f : exp2f(ml.x - Mu);
      l += ml.y * w;
      s_w[sp * rows_cap + cr] = w;
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    for (int sp = 0; sp < ns; ++sp) s_w[sp * rows_cap + cr] *= inv;
    if (a.lse) {
      const int r = r0 + cr;
      a.lse[((size_t)b * a.Nmax + r / G) * a.Hq + g * G + r % G] = (M + __log2f(l)) * kLn2;
    }
  }
  __syncthreads();
  const int ntask = nrows * (kD / 8);
  constexpr int kT = 2;   // pieces per thread per round (registers stay near the main loop's count)
  for (int t0 = threadIdx.x; t0 < ntask; t0 += kT * bd) {
    float acc[kT][8];
#pragma unroll
    for (int j = 0; j < kT; ++j) {
      const int t = t0 + j * bd, cr = t / (kD / 8), c8 = t % (kD / 8);
      const float w = t < ntask ? s_w[own * rows_cap + cr] : 0.f;
      float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0;
      if (t < ntask && w != 0.f) {
        const float4* src = reinterpret_cast<const float4*>(sStage + (size_t)cr * kStageF + c8 * 32);
        x0 = src[0], x1 = src[1];
      }
      acc[j][0] = w * x0.x, acc[j][1] = w * x0.y, acc[j][2] = w * x0.z, acc[j][3] = w * x0.w;
      acc[j][4] = w * x1.x, acc[j][5] = w * x1.y, acc[j][6] = w * x1.z, acc[j][7] = w * x1.w;
    }
    for (int s0 = 0; s0 < ns; s0 += 2) {
      float4 x[2][kT][2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int sp = s0 + q;
#pragma unroll
        for (int j = 0; j < kT; ++j) {
          const int t = t0 + j * bd, cr = t / (kD / 8), c8 = t % (kD / 8);
          if (sp < ns && sp != own && t < ntask) {
            const float4* p4 = reinterpret_cast<const float4*>(wo + (base + (size_t)sp * u.Rmax + cr) * kD + c8 * 8);
            x[q][j][0] = __ldcg(p4), x[q][j][1] = __ldcg(p4 + 1);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int sp = s0 + q;
#pragma unroll
        for (int j = 0; j < kT; ++j) {
          const int t = t0 + j * bd, cr = t / (kD / 8);
          if (sp < ns && sp != own && t < ntask) {
            const float w = s_w[sp * rows_cap + cr];
            if (w != 0.f) {
              const float4 a0 = x[q][j][0], a1 = x[q][j][1];
              acc[j][0] = fmaf(w, a0.x, acc[j][0]), acc[j][1] = fmaf(w, a0.y, acc[j][1]);
              acc[j][2] = fmaf(w, a0.z, acc[j][2]), acc[j][3] = fmaf(w, a0.w, acc[j][3]);
              acc[j][4] = fmaf(w, a1.x, acc[j][4]), acc[j][5] = fmaf(w, a1.y, acc[j][5]);
              acc[j][6] = fmaf(w, a1.z, acc[j][6]), acc[j][7] = fmaf(w, a1.w, acc[j][7]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kT; ++j) {
      const int t = t0 + j * bd, cr = t / (kD / 8), c8 = t % (kD / 8);
      if (t < ntask) {
        const int r = r0 + cr;
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) +
                              (((size_t)b * a.Nmax + r / G) * a.Hq + g * G + r % G) * kD;
        *reinterpret_cast<uint4*>(orow + c8 * 8) =
            make_uint4(pack_bf16x2(acc[j][0], acc[j][1]), pack_bf16x2(acc[j][2], acc[j][3]),
                       pack_bf16x2(acc[j][4], acc[j][5]), pack_bf16x2(acc[j][6], acc[j][7]));
      }
    }
  }
}

template <bool kDual>
__global__ void __launch_bounds__(kThreadsU, 1)
    attn_umma_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKt,
                     const __grid_constant__ CUtensorMap tmVt, const AttnArgs a, const UParams u) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ Bars bars;
  __shared__ uint32_t s_tmem;
  __shared__ int s_err;
  __shared__ int s_ticket;
  __shared__ volatile int s_abort;
  __shared__ int s_k_issued, s_v_issued, s_k_consumed, s_v_consumed;
  __shared__ float2 s_ml1[kBM];   // warpgroup 1's (max, sum) per row, for the epilogue merge
  constexpr int kRows = kDual ? 2 * kBM : kBM;   // query rows of this CTA

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // ---------------------------------------------------------------- set-up
  // Barriers, tensor memory and the tensor-map descriptors need nothing an earlier kernel writes,
  // so they are set up before the wait on the previous launch (programmatic dependent launch):
  // under a chain of kernels this prologue overlaps the previous kernel's tail.
  if (tid == 0) {
    mbar_init(&bars.q_full, kDual ? 8 : 1);   // two query tiles: each softmax warp stores its rows
    for (int s = 0; s < u.ks; ++s) mbar_init(&bars.k_full[s], 1), mbar_init(&bars.k_empty[s], 1);
    for (int s = 0; s < u.vs; ++s) mbar_init(&bars.v_full[s], 1), mbar_init(&bars.v_empty[s], 1);
    for (int sb = 0; sb < kSBufs; ++sb) mbar_init(&bars.s_full[sb], 1);
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars.p_full[w], 4);
      mbar_init(&bars.pv_done[w], 1);
    }
    mbar_init(&bars.mask_full, 1);
    mbar_init(&bars.fin, 1);
    s_err = 0;
    s_abort = 0;
    s_k_issued = s_v_issued = s_k_consumed = s_v_consumed = 0;
    fence_barrier_init();
    fence_proxy_async();
    prefetch_tmap(&tmQ), prefetch_tmap(&tmK), prefetch_tmap(&tmV), prefetch_tmap(&tmKt), prefetch_tmap(&tmVt);
  }
  if (warp == 3) {
    tmem_alloc(&s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  pdl_wait();
  // every early return below frees the tensor memory first (nothing has used it yet)
  auto leave = [&]() {
    if (warp == 3) tmem_dealloc(tmem, kTmemCols);
  };

  // CTA `split` of a (sequence, KV head, row block) takes an equal share of that sequence's own key
  // tiles (so ragged lengths stay balanced across its splits)
  const int split = blockIdx.x % u.splits, mt = blockIdx.x / u.splits;
  const int g = blockIdx.y;
  // Sequences are taken longest prefix first (ties by index): blocks start in z order, so the
  // longest sequences' CTAs start in the first wave and a ragged batch does not end on one long
  // sequence.  Every CTA ranks the prefix lengths itself.
  int b = blockIdx.z;
  if (u.lpt) {
    __shared__ int s_b;
    __shared__ int s_len[kThreadsU];
    if (tid < a.B) s_len[tid] = a.prefix_len[tid];   // one read each, then ranks from shared memory
    __syncthreads();
    if (tid < a.B) {
      const int L = s_len[tid];
      int rank = 0;
      for (int o = 0; o < a.B; ++o) {
        const int Lo = s_len[o];
        rank += (Lo > L) || (Lo == L && o < tid);
      }
      if (rank == (int)blockIdx.z) s_b = tid;
    }
    __syncthreads();
    b = s_b;
  }
  const int G = a.Hq / a.Hkv;
  SeqView v = seq_view(a, b, G, kBN, 1 << 30);
  // the status word can be flagged by another CTA while this one starts: one read, shared by every
  // thread, so the CTA takes one branch below
  __shared__ int s_status;
  if (tid == 0) s_status = __ldcg(a.status + b);
  __syncthreads();
  v.zero = v.cap || s_status != 0;
  const int r0 = mt * kRows;
  if (v.skip || r0 >= v.R) {
    leave();
    return;
  }
  const int r_hi = min(r0 + kRows, v.R);
  // a flagged or over-capacity sequence: zero rows (the split merge zeroes them too, as it reads
  // the status after every split has finished)
  // (the status word may be flagged while the launch runs, so with the merge in the kernel these
  // CTAs still take their tickets: the row block's count must reach its split count)
  if (v.zero) {
    if (split == 0 && mt == 0 && g == 0 && tid == 0 && s_status == 0 && v.cap)
      flag_status(a.status, b, TSD_ERR_CAPACITY);
    if (u.splits > 1 && u.tickets != nullptr) {
      int* word = u.tickets + ((size_t)b * a.Hkv + g) * u.mtiles + mt;
      const int t = take_ticket(word, u.splits, &s_ticket);
      if (t == 1) zero_rows<__nv_bfloat16>(a, b, g, G, r0, r_hi);
      else if (t == 2 && tid == 0) flag_status(a.status, b, TSD_ERR_WORKSPACE);
    } else if (split == 0) {
      zero_rows<__nv_bfloat16>(a, b, g, G, r0, r_hi);
    }
    leave();
    return;
  }
  const bool direct = (u.splits == 1);
  const int t_begin = (int)((long long)split * v.T / u.splits);
  const int nt = (int)((long long)(split + 1) * v.T / u.splits) - t_begin;   // 0 when T < splits
  const int nodes_per_tile = kRows / G;
  const int node0 = mt * nodes_per_tile;

  uint8_t* sQ = smem;
  uint8_t* sK = smem + u.k_off;
  uint8_t* sV = smem + u.v_off;
  uint32_t* sMask = reinterpret_cast<uint32_t*>(smem + u.mask_off);

  float row_m = -INFINITY, row_l = 0.f;   // softmax threads: the row's final (max, sum) for their warpgroup

  if (warp == 0) {
    // ------------------------------------------------------------ K producer (one thread), Q first
    if (lane == 0) {
      if (!kDual) {
        mbar_expect_tx(&bars.q_full, kQBytes);
        const int zq = b * a.Nmax + node0;
        tma_load_3d(sQ, &tmQ, 0, g * G, zq, &bars.q_full);
        tma_load_3d(sQ + kQBytes / 2, &tmQ, 64, g * G, zq, &bars.q_full);
      }
      int issued = 0;
      const uint64_t pol = u.evict_first ? l2_evict_first_policy() : l2_evict_normal_policy();
      TileBlocks nxt;
      fetch_blocks(a, v, u, b, t_begin, nxt);
      for (int i = 0; i < nt && !s_abort; ++i) {
        if (t_begin + i == u.withhold) break;   // test hook: this tile never arrives
        const TileBlocks cur = nxt;
        if (i + 1 < nt) fetch_blocks(a, v, u, b, t_begin + i + 1, nxt);
        const int st = i % u.ks;
        if (i >= u.ks && !mbar_wait(&bars.k_empty[st], ((i / u.ks) - 1) & 1, u.wait)) {
          abort_cta(a, b, &s_abort);
          break;
        }
        mbar_expect_tx(&bars.k_full[st], kSlot);
        load_tile(a, v, u, b, g, t_begin + i, sK + (size_t)st * kSlot, &tmK, &tmKt, &bars.k_full[st], &s_err, cur,
                  pol);
        ++issued;
      }
      s_k_issued = issued;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ ancestor bits of the tree tiles
    // built while the first prefix tiles stream in; the softmax waits for them at its first tree tile
    if (t_begin + nt > v.nPT) {
      build_mask_staged(a, b, node0, nodes_per_tile, u.W, sMask, v.N, reinterpret_cast<int32_t*>(smem + u.ps_off),
                        lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.mask_full);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ V producer (one thread)
    if (lane == 0) {
      int issued = 0;
      const uint64_t pol = u.evict_first ? l2_evict_first_policy() : l2_evict_normal_policy();
      TileBlocks nxt;
      fetch_blocks(a, v, u, b, t_begin, nxt);
      for (int i = 0; i < nt && !s_abort; ++i) {
        const TileBlocks cur = nxt;
        if (i + 1 < nt) fetch_blocks(a, v, u, b, t_begin + i + 1, nxt);
        const int st = i % u.vs;
        if (i >= u.vs && !mbar_wait(&bars.v_empty[st], ((i / u.vs) - 1) & 1, u.wait)) {
          abort_cta(a, b, &s_abort);
          break;
        }
        mbar_expect_tx(&bars.v_full[st], kSlot);
        load_tile(a, v, u, b, g, t_begin + i, sV + (size_t)st * kSlot, &tmV, &tmVt, &bars.v_full[st], &s_err, cur,
                  pol);
        ++issued;
      }
      s_v_issued = issued;
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ MMA issuer (one thread)
    // Warp 3 shares its SM sub-partition with row quarter 3, which is padding in small-row tiles.
    // Descriptors are built once; a k-step advances the 14-bit start-address field by a constant.
    const uint32_t idesc_s = idesc_bf16(kBM, kBN, false);
    const uint32_t idesc_o = idesc_bf16(kBM, kD, true);
    const uint64_t dq = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dk = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t dv = sdesc_sw128(smem_u32(sV), kHalf, 1024);
    // every lane waits and the verdict is made warp-uniform: the MMA issue below is
    // warp-collective (elect.sync) and needs the whole warp converged
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, u.wait)) != 0;
    };
    bool ok = wait_all(&bars.q_full, 0);
    int k_consumed = 0, v_consumed = 0;
    // S(j) = Q K(j)^T into S buffer j % 4 (warpgroup j & 1); frees the K slot when done
    auto issue_s = [&](int j) -> bool {
      const int st = j % u.ks;
      if (!wait_all(&bars.k_full[st], (j / u.ks) & 1)) return false;
      ++k_consumed;
      tc_fence_after();
      const uint64_t bk = dk + (uint64_t)((st * kSlot) >> 4);
      const uint32_t d = tmem + kColS + (uint32_t)(j % kSBufs) * kBN;
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t off_q = ((kk >> 2) * (kQBytes / 2) + (kk & 3) * 32) >> 4;
        const uint32_t off_k = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
        mma_bf16_ss_warp(d, dq + off_q, bk + off_k, idesc_s, kk > 0 ? 1u : 0u);
      }
      tc_commit_warp(&bars.k_empty[st]);
      tc_commit_warp(&bars.s_full[j % kSBufs]);
      return true;
    };
    // zero V rows past the valid keys of a partial tile (its TMA box may hold stale rows)
    auto zero_v_tail = [&](int i, int st) {
      const int t = t_begin + i;
      const int nv = t < v.nPT ? min(kBN, v.L - t * kBN) : min(kBN, v.N - (t - v.nPT) * kBN);
      if (nv < kBN) {
        uint8_t* dV = sV + (size_t)st * kSlot;
        const int nchunks = (kBN - nv) * 8;   // 16-byte chunks per half
        for (int c = lane; c < 2 * nchunks; c += 32) {
          const int half = c / nchunks, cc = c % nchunks;
          *reinterpret_cast<uint4*>(dV + half * kHalf + (size_t)nv * 128 + (size_t)cc * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async();
      }
      __syncwarp();
    };
    if constexpr (kDual) {
      // S_w(j) = Q_w K(j)^T into warpgroup w's S tile, A = Q_w from TMEM (8 columns per k-step);
      // the K slot is freed after both
      auto issue_s_w = [&](int j, int w) -> bool {
        const int st = j % u.ks;
        if (w == 0) {
          if (!wait_all(&bars.k_full[st], (j / u.ks) & 1)) return false;
          ++k_consumed;
        }
        tc_fence_after();
        const uint64_t bk = dk + (uint64_t)((st * kSlot) >> 4);
        const uint32_t aq = tmem + kColQ + (uint32_t)w * 64;
        const uint32_t d = tmem + kColS + (uint32_t)w * kBN;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off_k = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
          mma_bf16_ts_warp(d, aq + (uint32_t)(kk * 8), bk + off_k, idesc_s, kk > 0 ? 1u : 0u);
        }
        if (w == 1) tc_commit_warp(&bars.k_empty[st]);
        tc_commit_warp(&bars.s_full[w]);
        return true;
      };
      if (ok && nt > 0) {
        ok = issue_s_w(0, 0);
        if (ok) ok = issue_s_w(0, 1);
      }
      for (int i = 0; ok && i < nt; ++i) {
        const int st = i % u.vs;
        if (!wait_all(&bars.v_full[st], (i / u.vs) & 1)) {
          ok = false;
          break;
        }
        ++v_consumed;
        zero_v_tail(i, st);
        const uint64_t bv = dv + (uint64_t)((st * kSlot) >> 4);
        for (int w = 0; ok && w < 2; ++w) {
          if (!wait_all(&bars.p_full[w], i & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ap = tmem + kColS + (uint32_t)w * kBN;   // P_w(i) over S_w(i)
          const uint32_t d = tmem + kColO + (uint32_t)w * kD;
#pragma unroll
          for (int kb = 0; kb < kBN / 16; ++kb)
            mma_bf16_ts_warp(d, ap + (uint32_t)(kb * 8), bv + (uint32_t)(kb * 128), idesc_o, (i > 0 || kb > 0) ? 1u : 0u);
          if (w == 1) tc_commit_warp(&bars.v_empty[st]);
          tc_commit_warp(&bars.pv_done[w]);
          // S_w(i+1) overwrites P_w(i): tcgen05.mma of one thread execute in issue order, so the
          // P V product just issued has read its A operand first
          if (i + 1 < nt) ok = issue_s_w(i + 1, w);
        }
      }
    } else {
    for (int j = 0; ok && j < kSBufs && j < nt; ++j) ok = issue_s(j);
    for (int i = 0; ok && i < nt; ++i) {
      const int w = i & 1;
      if (!wait_all(&bars.p_full[w], (i >> 1) & 1)) {
        ok = false;
        break;
      }
      const int st = i % u.vs;
      if (!wait_all(&bars.v_full[st], (i / u.vs) & 1)) {
        ok = false;
        break;
      }
      ++v_consumed;
      zero_v_tail(i, st);
      tc_fence_after();
      const uint64_t bv = dv + (uint64_t)((st * kSlot) >> 4);
      const uint32_t ap = tmem + kColS + (uint32_t)(i % kSBufs) * kBN;   // P(i) over S(i)
      const uint32_t d = tmem + kColO + (uint32_t)w * kD;
#pragma unroll
      for (int kb = 0; kb < kBN / 16; ++kb)
        mma_bf16_ts_warp(d, ap + (uint32_t)(kb * 8), bv + (uint32_t)(kb * 128), idesc_o, (i >= 2 || kb > 0) ? 1u : 0u);
      tc_commit_warp(&bars.v_empty[st]);
      tc_commit_warp(&bars.pv_done[w]);
      if (i + kSBufs < nt) ok = issue_s(i + kSBufs);   // warpgroup w has read S(i): its buffer is free
    }
    }
    if (!ok) abort_cta(a, b, &s_abort);
    if (lane == 0) s_k_consumed = k_consumed, s_v_consumed = v_consumed;
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = (warp - 4) >> 2;
    const int q4 = warp & 3;                       // TMEM lane quarter of this warp
    const int row = q4 * 32 + lane;                // TMEM lane = row of the query tile
    const int qrow = (kDual ? wg * kBM : 0) + row;  // row within the CTA's query rows
    const int r = r0 + qrow;
    const bool row_ok = r < r_hi;
    // a warp whose 32 rows are all padding skips the softmax; its P rows are never read into an
    // output row (each output row depends on its own P row only)
    const bool warp_live = r0 + qrow - lane < r_hi;
    const int nl = qrow / G;
    const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
    const uint32_t o_col = kColO + (uint32_t)wg * kD;
    const float sl2 = a.scale * kLog2e;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    bool mask_ready = false;
    if constexpr (kDual) {
      // this thread's query row into TMEM as bf16 pairs (64 columns of Q_w): the A operand of
      // S = Q K^T; rows past the sequence's rows are zero
      const int i_node = r / G, hh = r % G;
      const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.q) +
                                                        (((size_t)b * a.Nmax + (row_ok ? i_node : 0)) * a.Hq +
                                                         g * G + hh) * kD);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t qv[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 x = row_ok ? src[half * 8 + c] : make_uint4(0, 0, 0, 0);
          qv[4 * c] = x.x, qv[4 * c + 1] = x.y, qv[4 * c + 2] = x.z, qv[4 * c + 3] = x.w;
        }
        tmem_st32(lane_addr + kColQ + (uint32_t)wg * 64 + (uint32_t)half * 32, qv);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.q_full);
    }
    for (int i = kDual ? 0 : wg; i < nt; i += kDual ? 1 : 2) {
      const int k = kDual ? i : i >> 1;            // this warpgroup's k-th tile
      const int buf = kDual ? wg : wg + 2 * (k & 1);
      const uint32_t s_col = kColS + (uint32_t)buf * kBN;
      const int t = t_begin + i;
      const bool tree = t >= v.nPT;
      const int kbase = tree ? (t - v.nPT) * kBN : t * kBN;
      if (ok && !mbar_wait(&bars.s_full[buf], kDual ? (k & 1) : ((k >> 1) & 1), u.wait)) ok = false;
      if (ok && tree && !mask_ready) {
        if (mbar_wait(&bars.mask_full, 0, u.wait)) mask_ready = true;
        else ok = false;
      }
      // one verdict per warp: the TMEM accesses below are warp-collective
      ok = __all_sync(0xffffffffu, ok) != 0;
      if (!ok) break;
      tc_fence_after();
      float alpha = 1.f;
      bool resc = false;
      uint32_t pk[32];
      if (warp_live) {
        uint32_t s0[32], s1[32];
        tmem_ld32(lane_addr + s_col, s0);
        tmem_ld32(lane_addr + s_col + 32, s1);
        tmem_wait_ld();
        float mx;
        const bool full = !tree && kbase + kBN <= v.L;
        if (full) {
          // a full prefix tile: every key is visible to every row, no mask work
          float ma[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) ma[q] = fmaxf(__uint_as_float(s0[q]), __uint_as_float(s1[q]));
#pragma unroll
          for (int c = 8; c < 32; ++c) ma[c & 7] = max3f(ma[c & 7], __uint_as_float(s0[c]), __uint_as_float(s1[c]));
          mx = max3f(max3f(ma[0], ma[1], ma[2]), max3f(ma[3], ma[4], ma[5]), fmaxf(ma[6], ma[7]));
          mx = row_ok ? mx * sl2 : -INFINITY;
        } else {
          const int lim = tree ? v.N : v.L;
          uint32_t w0 = 0xffffffffu, w1 = 0xffffffffu;
          if (tree) {
            const int wi = kbase >> 5;
            w0 = sMask[nl * u.W + wi];
            w1 = (wi + 1 < u.W) ? sMask[nl * u.W + wi + 1] : 0u;
          }
          // fold the key limit into the bit words: bit c survives iff kbase + c < lim
          const int n0 = lim - kbase;
          if (n0 < 32) w0 &= n0 <= 0 ? 0u : ((1u << n0) - 1u);
          if (n0 < 64) w1 &= n0 <= 32 ? 0u : ((1u << (n0 - 32)) - 1u);
          if (!row_ok) w0 = w1 = 0u;
          float ma[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) ma[q] = -INFINITY;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float x0 = ((w0 >> c) & 1u) ? __uint_as_float(s0[c]) : -INFINITY;
            const float x1 = ((w1 >> c) & 1u) ? __uint_as_float(s1[c]) : -INFINITY;
            s0[c] = __float_as_uint(x0);
            s1[c] = __float_as_uint(x1);
            ma[c & 7] = fmaxf(ma[c & 7], fmaxf(x0, x1));
          }
          mx = fmaxf(fmaxf(fmaxf(ma[0], ma[1]), fmaxf(ma[2], ma[3])), fmaxf(fmaxf(ma[4], ma[5]), fmaxf(ma[6], ma[7])));
          mx = mx * sl2;   // -inf stays -inf (sl2 > 0)
        }
        if (mx != -INFINITY && (m_used == -INFINITY || mx > m_used + kRescaleLog2)) {
          if (m_used != -INFINITY) {
            alpha = exp2f(m_used - mx);
            resc = true;
          }
          m_used = mx;
        }
        const float nmu = m_used == -INFINITY ? 0.f : -m_used;
        float suma[4] = {0.f, 0.f, 0.f, 0.f};
        if (full) {
#pragma unroll
          // pair sums: suma[0..1] gather the even/odd keys of s0, suma[2..3] those of s1
          for (int c = 0; c < 32; c += 2) {
            float x0, x1, x2, x3;
            fma2(x0, x1, __uint_as_float(s0[c]), __uint_as_float(s0[c + 1]), sl2, sl2, nmu, nmu);
            fma2(x2, x3, __uint_as_float(s1[c]), __uint_as_float(s1[c + 1]), sl2, sl2, nmu, nmu);
            const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            const float p2 = fast_exp2(x2), p3 = fast_exp2(x3);
            add2(suma[0], suma[1], suma[0], suma[1], p0, p1);
            add2(suma[2], suma[3], suma[2], suma[3], p2, p3);
            pk[c / 2] = pack_bf16x2(p0, p1);
            pk[16 + c / 2] = pack_bf16x2(p2, p3);
          }
        } else {
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          // p = 2^(s * scale * log2(e) - m): one FFMA feeds the exponential (masked s = -inf gives 0)
          const float p0 = fast_exp2(fmaf(__uint_as_float(s0[c]), sl2, nmu));
          const float p1 = fast_exp2(fmaf(__uint_as_float(s0[c + 1]), sl2, nmu));
          const float p2 = fast_exp2(fmaf(__uint_as_float(s1[c]), sl2, nmu));
          const float p3 = fast_exp2(fmaf(__uint_as_float(s1[c + 1]), sl2, nmu));
          suma[(c >> 1) & 3] += (p0 + p1) + (p2 + p3);
          pk[c / 2] = pack_bf16x2(p0, p1);
          pk[16 + c / 2] = pack_bf16x2(p2, p3);
        }
        }
        l = l * alpha + ((suma[0] + suma[1]) + (suma[2] + suma[3]));
      }
      // this warpgroup's previous P V must be done before O is rescaled (one verdict per warp: the
      // TMEM accesses below are warp-collective)
      bool pv_ok = k < 1 || mbar_wait(&bars.pv_done[wg], (k - 1) & 1, u.wait);
      if (!__all_sync(0xffffffffu, pv_ok)) {
        ok = false;
        break;
      }
      if (warp_live && __any_sync(0xffffffffu, resc)) {   // warp-collective TMEM read-modify-write of O
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < kD / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(lane_addr + o_col + ch * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(lane_addr + o_col + ch * 32, o);
        }
        tmem_wait_st();
      }
      if (warp_live) {   // P row (bf16 pairs) over the first 32 columns of its S tile
        tmem_st32(lane_addr + s_col, pk);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[wg]);
    }
    // the warpgroup's last P V product
    const int kn = kDual ? nt : (nt - wg + 1) >> 1;   // tiles this warpgroup processed
    if (ok && kn > 0 && !mbar_wait(&bars.pv_done[wg], (kn - 1) & 1, u.wait)) ok = false;
    if (!ok) abort_cta(a, b, &s_abort);
    row_m = m_used;
    row_l = l;
    if (!kDual && wg == 1) s_ml1[row] = make_float2(m_used, l);
  }

  // ---------------------------------------------------------------- epilogue / teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  uint8_t* sStage = smem + u.k_off;   // the K/V rings, idle once every P V product is done
  if (!s_abort && u.stage) fence_proxy_async();   // last read there by the tensor cores
  if (!s_abort) {
    if (kDual ? warp >= 4 : (warp >= 4 && warp < 8)) {
      // one query tile: merge the two warpgroups' partial results of this row (log-sum-exp);
      // two query tiles: each warpgroup holds its rows' complete result.  Then write the row.
      const int wg = (warp - 4) >> 2;
      const int q4 = warp & 3;
      const int row = q4 * 32 + lane;
      const int crow = (kDual ? wg * kBM : 0) + row;   // row within this CTA's rows
      const int r = r0 + crow;
      const bool row_ok = r < r_hi;
      const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
      const uint32_t o_first = kColO + (kDual ? (uint32_t)wg * kD : 0u);
      const bool two = !kDual && nt > 1;   // a second accumulator (warpgroup 1's) to merge
      const float2 ml1 = two ? s_ml1[row] : make_float2(-INFINITY, 0.f);
      const float M = fmaxf(row_m, ml1.x);
      const float Mu = M == -INFINITY ? 0.f : M;
      const float a0 = exp2f(row_m - Mu);
      const float a1 = two ? exp2f(ml1.x - Mu) : 0.f;
      const float l = row_l * a0 + ml1.y * a1;
      const bool err = s_err != 0;
      const int i_node = r / G, hh = r % G;
      if (direct) {
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) +
                              (((size_t)b * a.Nmax + (row_ok ? i_node : 0)) * a.Hq + g * G + hh) * kD;
        const float inv = (l > 0.f && !err) ? 1.f / l : 0.f;
        const float c0 = a0 * inv, c1 = a1 * inv;
#pragma unroll
        for (int ch = 0; ch < kD / 32; ++ch) {
          uint32_t o0[32], o1[32];
          tmem_ld32(lane_addr + o_first + ch * 32, o0);
          if (two) tmem_ld32(lane_addr + kColO + kD + ch * 32, o1);
          tmem_wait_ld();
          float f[32];
#pragma unroll
          for (int e = 0; e < 32; ++e)
            f[e] = __uint_as_float(o0[e]) * c0 + (two ? __uint_as_float(o1[e]) * c1 : 0.f);
          if (row_ok) {
            uint4* dst = u.stage ? reinterpret_cast<uint4*>(sStage + (size_t)crow * kStageH + ch * 64)
                                 : reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(pack_bf16x2(f[8 * q], f[8 * q + 1]), pack_bf16x2(f[8 * q + 2], f[8 * q + 3]),
                                  pack_bf16x2(f[8 * q + 4], f[8 * q + 5]), pack_bf16x2(f[8 * q + 6], f[8 * q + 7]));
          }
        }
        if (row_ok && a.lse)
          a.lse[((size_t)b * a.Nmax + i_node) * a.Hq + g * G + hh] = err ? 0.f : (M + __log2f(l)) * kLn2;
      } else {
        // split partial: unnormalised O relative to M, with (M, l); a split with no keys (or no
        // mass) writes M = -inf, which the merge skips without reading its O
        float* wo = reinterpret_cast<float*>(a.workspace);
        const size_t base = (((size_t)b * a.Hkv + g) * u.splits + split) * u.Rmax;
        float* wml = wo + (size_t)a.B * a.Hkv * u.splits * u.Rmax * kD;
#pragma unroll
        for (int ch = 0; ch < kD / 32; ++ch) {
          uint32_t o0[32], o1[32];
          tmem_ld32(lane_addr + o_first + ch * 32, o0);
          if (two) tmem_ld32(lane_addr + kColO + kD + ch * 32, o1);
          tmem_wait_ld();
          if (row_ok) {
            float4* dst = u.stage ? reinterpret_cast<float4*>(sStage + (size_t)crow * kStageF + ch * 128)
                                  : reinterpret_cast<float4*>(wo + (base + r) * kD + ch * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float f[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                f[e] = __uint_as_float(o0[4 * q + e]) * a0 + (two ? __uint_as_float(o1[4 * q + e]) * a1 : 0.f);
              dst[q] = make_float4(f[0], f[1], f[2], f[3]);
            }
          }
        }
        if (row_ok) *reinterpret_cast<float2*>(wml + (base + r) * 2) = make_float2(l > 0.f ? M : -INFINITY, l);
      }
      if (err && tid == 128) flag_status(a.status, b, TSD_ERR_CAPACITY);
    }
    if (u.stage) {
      // every thread copies staged rows out with coalesced 16-byte stores
      __syncthreads();
      const int nrows = r_hi - r0;
      if (direct) {
        for (int idx = tid; idx < nrows * (kD / 8); idx += kThreadsU) {
          const int cr = idx / (kD / 8), c = idx % (kD / 8);
          const int rr = r0 + cr, node = rr / G, hh = rr % G;
          __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) +
                                (((size_t)b * a.Nmax + node) * a.Hq + g * G + hh) * kD;
          reinterpret_cast<uint4*>(orow)[c] = *reinterpret_cast<const uint4*>(sStage + (size_t)cr * kStageH + c * 16);
        }
      } else {
        float* wo = reinterpret_cast<float*>(a.workspace);
        const size_t base = (((size_t)b * a.Hkv + g) * u.splits + split) * u.Rmax + r0;
        for (int idx = tid; idx < nrows * (kD / 4); idx += kThreadsU) {
          const int cr = idx / (kD / 4), c = idx % (kD / 4);
          reinterpret_cast<float4*>(wo + (base + cr) * kD)[c] =
              *reinterpret_cast<const float4*>(sStage + (size_t)cr * kStageF + c * 16);
        }
      }
    }
  } else {
    // time-out: let this CTA's own TMA copies and MMAs land (bounded) before freeing TMEM
    if (tid == 0) {
      for (int i = s_k_consumed; i < s_k_issued; ++i) mbar_wait(&bars.k_full[i % u.ks], (i / u.ks) & 1, u.wait);
      for (int i = s_v_consumed; i < s_v_issued; ++i) mbar_wait(&bars.v_full[i % u.vs], (i / u.vs) & 1, u.wait);
    }
    if (warp == 3 && lane == 0) {
      tc_commit(&bars.fin);
      mbar_wait(&bars.fin, 0, u.wait);
    }
    if (direct) {
      zero_rows<__nv_bfloat16>(a, b, g, G, r0, r_hi);
    } else {   // an unusable partial: the merge skips it (and zeroes the rows: status is flagged)
      float* wml = reinterpret_cast<float*>(a.workspace) + (size_t)a.B * a.Hkv * u.splits * u.Rmax * kD;
      const size_t base = (((size_t)b * a.Hkv + g) * u.splits + split) * u.Rmax;
      for (int r = r0 + tid; r < r_hi; r += kThreadsU)
        *reinterpret_cast<float2*>(wml + (base + r) * 2) = make_float2(-INFINITY, 0.f);
    }
  }
  if (!direct && u.tickets != nullptr) {
    int* word = u.tickets + ((size_t)b * a.Hkv + g) * u.mtiles + mt;
    const int t = take_ticket(word, u.splits, &s_ticket);
    if (t == 1) {
      // one read of the status word for the whole CTA (another row block may flag it meanwhile);
      // the staged rows hold this CTA's partial (none after a time-out: the status is flagged then)
      __threadfence();
      if (tid == 0) s_status = __ldcg(a.status + b);
      __syncthreads();
      merge_splits(a, u, b, g, G, r0, r_hi, split, s_abort != 0 || s_status != 0, sStage,
                   reinterpret_cast<float*>(sStage + (size_t)kRows * kStageF), kRows);
    } else if (t == 2 && tid == 0) {
      flag_status(a.status, b, TSD_ERR_WORKSPACE);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// -------------------------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 tensor map with 128-byte swizzle; dims/box innermost first; strides in bytes for dims 1..
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
              const uint32_t* box) {
  auto fn = encoder();
  if (!fn) return false;
  uint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool umma_eligible(const AttnArgs& a, tsd_dtype dtype) {
  const int G = a.Hq / a.Hkv;
  if (dtype != TSD_BF16 || a.d != kD || a.k_tree == nullptr) return false;
  if (G < 1 || G > 128 || (G & (G - 1)) != 0) return false;
  if ((reinterpret_cast<uintptr_t>(a.q) | reinterpret_cast<uintptr_t>(a.k_cache) |
       reinterpret_cast<uintptr_t>(a.v_cache) | reinterpret_cast<uintptr_t>(a.k_tree) |
       reinterpret_cast<uintptr_t>(a.v_tree)) & 15)
    return false;
  if (a.Lcap <= 0) return false;
  return encoder() != nullptr;
}

bool umma_layout(const AttnPlan& p, int G, int Nmax, UmmaLayout& L) {
  L.rows = p.dual ? 2 * kBM : kBM;                     // query rows per CTA
  const uint32_t q_bytes = p.dual ? 0u : kQBytes;      // two query tiles live in TMEM, not shared memory
  L.W = (Nmax + 31) / 32;
  const uint32_t mask_bytes = (uint32_t)(L.rows / G) * L.W * 4;
  const uint32_t ps_bytes = (uint32_t)(Nmax + 1) * 4;   // the tree's parent slots, staged for the mask
  auto total = [&](int ks, int vs) {
    return 1024 + q_bytes + (uint32_t)(ks + vs) * kSlot + ((mask_bytes + 15) & ~15u) + ps_bytes;
  };
  L.ks = 6, L.vs = 5;   // K is consumed first (by S = Q K^T), so its ring runs further ahead
  const uint32_t limit = 227 * 1024 - 4096;   // leave room for the static shared variables
  while (total(L.ks, L.vs) > limit && L.vs > 2) {
    if (L.ks > L.vs) --L.ks; else --L.vs;
  }
  if (total(L.ks, L.vs) > limit) return false;
  L.k_off = q_bytes;
  L.v_off = L.k_off + (uint32_t)L.ks * kSlot;
  L.mask_off = L.v_off + (uint32_t)L.vs * kSlot;
  L.ps_off = L.mask_off + ((mask_bytes + 15) & ~15u);
  L.stage = (uint32_t)(L.ks + L.vs) * kSlot >= (uint32_t)L.rows * kStageF ? 1 : 0;
  L.smem = total(L.ks, L.vs);
  return true;
}

// Split merge in the kernel: the last CTA's staged rows and the splits' weights fit in the rings,
// and the ticket words fit their region.  Measured on B200: it pays for the two-tile kernel (256
// rows per CTA: the merge kernel re-reads large partials from DRAM after the grid ends), not for
// one-tile CTAs (many short CTAs pay the fence and ticket round trips; many splits leave one CTA a
// long merge), which keep the merge kernel.  TSD_ATTN_MERGE=kernel / =fused force either choice
// (A/B runs).
bool umma_merges_in_kernel(const AttnPlan& p, const UmmaLayout& L, int B, int Hkv) {
  const char* merge_env = getenv("TSD_ATTN_MERGE");
  const long long groups = (long long)B * Hkv * p.umtiles;
  const bool want = merge_env != nullptr ? merge_env[0] == 'f' : p.dual;
  return want && p.usplits > 1 && L.stage &&
         (size_t)(L.ks + L.vs) * kSlot >= (size_t)L.rows * kStageF + (size_t)p.usplits * L.rows * 12 &&
         groups * 4 <= (long long)kAttnTicketBytes;
}

tsd_status launch_attention_umma(const AttnArgs& a, const AttnPlan& p, int* tickets, bool* merged,
                                 cudaStream_t stream) {
  const int G = a.Hq / a.Hkv;
  UParams u{};
  u.splits = p.usplits, u.Rmax = p.Rmax, u.mtiles = p.umtiles;
  u.wait = kWaitCycles;
  u.withhold = -1;
  u.lpt = a.B > 1 && a.B <= kThreadsU ? 1 : 0;
  // one row block per KV head: every cache tile is read once by the whole grid (TSD_ATTN_L2HINT=0
  // turns the evict-first policy off, for A/B runs)
  const char* l2_env = getenv("TSD_ATTN_L2HINT");
  u.evict_first = (p.umtiles == 1 && !(l2_env != nullptr && l2_env[0] == '0')) ? 1 : 0;
  // Test hook for the bounded waits: TSD_TEST_WITHHOLD_TILE=t makes the K producer of every CTA
  // skip key tile t (and every later one), so the waits on it give up after 10^5 cycles and the
  // call reports TSD_ERR_TIMEOUT in status[] instead of stalling.
  if (const char* w = getenv("TSD_TEST_WITHHOLD_TILE")) {
    u.withhold = atoi(w);
    u.wait = 100000;
  }
  UmmaLayout L;
  if (!umma_layout(p, G, a.Nmax, L)) return TSD_ERR_INVALID_ARG;
  u.W = L.W, u.ks = L.ks, u.vs = L.vs, u.stage = L.stage;
  u.k_off = L.k_off, u.v_off = L.v_off, u.mask_off = L.mask_off, u.ps_off = L.ps_off;
  const bool fuse = tickets != nullptr && umma_merges_in_kernel(p, L, a.B, a.Hkv);
  u.tickets = fuse ? tickets : nullptr;
  *merged = fuse;
  const size_t smem = L.smem;

  CUtensorMap mq, mk, mv, mkt, mvt;
  {  // Q [B*Nmax rows][Hq][128] -> box (64, G, 128/G)
    uint64_t dims[3] = {(uint64_t)kD, (uint64_t)a.Hq, (uint64_t)a.B * a.Nmax};
    uint64_t str[2] = {(uint64_t)kD * 2, (uint64_t)a.Hq * kD * 2};
    uint32_t box[3] = {64, (uint32_t)G, (uint32_t)(kBM / G)};
    if (!make_map(&mq, a.q, 3, dims, str, box)) return TSD_ERR_CUDA;
  }
  if (a.block_table == nullptr) {  // cache [B*Hkv*Lmax rows][128]
    u.box_rows = kBN;
    uint64_t dims[2] = {(uint64_t)kD, (uint64_t)a.B * a.Hkv * a.Lcap};
    uint64_t str[1] = {(uint64_t)kD * 2};
    uint32_t box[2] = {64, (uint32_t)kBN};
    if (!make_map(&mk, a.k_cache, 2, dims, str, box) || !make_map(&mv, a.v_cache, 2, dims, str, box))
      return TSD_ERR_CUDA;
  } else {  // pages [num_blocks*Hkv*bs rows][128]
    const int bs = 1 << a.block_shift;
    u.box_rows = bs < kBN ? bs : kBN;
    uint64_t dims[2] = {(uint64_t)kD, (uint64_t)a.num_blocks * a.Hkv * bs};
    uint64_t str[1] = {(uint64_t)kD * 2};
    uint32_t box[2] = {64, (uint32_t)u.box_rows};
    if (!make_map(&mk, a.k_cache, 2, dims, str, box) || !make_map(&mv, a.v_cache, 2, dims, str, box))
      return TSD_ERR_CUDA;
  }
  {  // tree K/V [B*Nmax][Hkv][128] -> box (64, 1, 64)
    uint64_t dims[3] = {(uint64_t)kD, (uint64_t)a.Hkv, (uint64_t)a.B * a.Nmax};
    uint64_t str[2] = {(uint64_t)kD * 2, (uint64_t)a.Hkv * kD * 2};
    uint32_t box[3] = {64, 1, (uint32_t)kBN};
    if (!make_map(&mkt, a.k_tree, 3, dims, str, box) || !make_map(&mvt, a.v_tree, 3, dims, str, box))
      return TSD_ERR_CUDA;
  }
  auto kernel = p.dual ? attn_umma_kernel<true> : attn_umma_kernel<false>;
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid(u.mtiles * u.splits, a.Hkv, a.B);
  if (launch_pdl(kernel, grid, dim3(kThreadsU), smem, stream, mq, mk, mv, mkt, mvt, a, u) != cudaSuccess)
    return TSD_ERR_CUDA;
  return TSD_OK;
}

}  // namespace tsd
