// Tree-verify attention on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Same operation and work decomposition as the split kernels in attn.cu ("EAGLE-Pangu", technical
// summary sec. 2: a tree token attends to the committed prefix and to its own ancestors only;
// "Acelerando Sonar a traves de la especulacion", section "EAGLE": the mask touches only the
// tree's keys), built for Blackwell:
//   * a CTA owns 128 query rows (G heads x 128/G tree nodes of one KV head) and a range of 64-key
//     tiles of one sequence; every K/V tile is read from memory once per 128 rows;
//   * warp 0 streams the tiles with TMA (128-byte swizzled boxes; paged caches box by block, the
//     tree's K/V by node for one KV head) through a 4-deep ring of shared-memory stages;
//   * warp 1 issues tcgen05.mma from one thread: S = Q K^T into a double-buffered TMEM tile
//     (128 lanes x 64 fp32 columns), then O += P V into a 128 x 128 fp32 TMEM accumulator;
//   * warps 4-7 each own one TMEM lane quarter, one query row per thread: a row's 64 scores come
//     out of TMEM with one tcgen05.ld, so its max and sum need no shuffles; the ancestor mask is
//     applied only on tree tiles (bits rebuilt in shared memory by warps 2-3); P is written back
//     as bf16 into a swizzled shared tile for the P V product.  The running max is raised
//     lazily (only when a row's max grows by more than 2^8), so O is rescaled in TMEM rarely.
// Every mbarrier wait is bounded: on time-out the CTA records TSD_ERR_TIMEOUT, drains its own
// TMA copies (again bounded) and frees its TMEM before returning.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <climits>
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
constexpr int kThreadsU = 256;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 0, kColS = 128;        // S buffers at columns 128 and 192
constexpr uint32_t kHalf = kBN * 128;              // one 64-column half of a K or V tile: 8 KB
constexpr uint32_t kStageBytes = 4 * kHalf;        // K halves + V halves: 32 KB
constexpr uint32_t kQBytes = kBM * 256;            // 32 KB
constexpr uint32_t kPBytes = kBM * 128;            // 16 KB
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;               // lazy max: rescale only past a 2^8 growth

struct UParams {
  int tps, splits, Rmax, mtiles, stages;
  int box_rows;        // rows per TMA box of the cache (64 contiguous, min(block, 64) paged)
  int W;               // ancestor-bit words per node
  uint32_t mask_off;   // shared-memory offsets
  uint32_t p_off;
};

struct __align__(8) Bars {
  uint64_t q_full;
  uint64_t s_full[2];
  uint64_t p_full;
  uint64_t pv_done;
  uint64_t kv_full[4];
  uint64_t kv_empty[4];
  uint64_t fin;
};

__device__ __forceinline__ void abort_cta(const AttnArgs& a, int b, volatile int* s_abort) {
  if (*s_abort == 0) {
    *s_abort = 1;
    flag_status(a.status, b, TSD_ERR_TIMEOUT);
  }
}

__global__ void __launch_bounds__(kThreadsU, 1)
    attn_umma_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKt,
                     const __grid_constant__ CUtensorMap tmVt, const AttnArgs a, const UParams u) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ Bars bars;
  __shared__ uint32_t s_tmem;
  __shared__ int s_err;
  __shared__ volatile int s_abort;
  __shared__ int s_issued, s_consumed;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int mt = blockIdx.x % u.mtiles, split = blockIdx.x / u.mtiles;
  const int g = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const SeqView v = seq_view(a, b, G, kBN, u.tps);
  const int r0 = mt * kBM;
  if (v.skip || r0 >= v.R) return;
  const int r_hi = min(r0 + kBM, v.R);
  if (v.zero) {
    if (split == 0) zero_rows<__nv_bfloat16>(a, b, g, G, r0, r_hi);
    if (split == 0 && mt == 0 && g == 0 && tid == 0 && a.status[b] == 0) flag_status(a.status, b, TSD_ERR_CAPACITY);
    return;
  }
  if (split >= v.nsplit) return;
  const bool direct = (v.nsplit == 1);
  const int t_begin = split * u.tps;
  const int nt = min(v.T, t_begin + u.tps) - t_begin;
  const int nodes_per_tile = kBM / G;
  const int node0 = mt * nodes_per_tile;

  uint8_t* sQ = smem;
  uint8_t* sKV = smem + kQBytes;
  uint8_t* sP = smem + u.p_off;
  uint32_t* sMask = reinterpret_cast<uint32_t*>(smem + u.mask_off);

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.s_full[0], 1);
    mbar_init(&bars.s_full[1], 1);
    mbar_init(&bars.p_full, 4);
    mbar_init(&bars.pv_done, 1);
    mbar_init(&bars.fin, 1);
    for (int s = 0; s < u.stages; ++s) {
      mbar_init(&bars.kv_full[s], 1);
      mbar_init(&bars.kv_empty[s], 1);
    }
    s_err = 0;
    s_abort = 0;
    s_issued = 0;
    s_consumed = 0;
    fence_barrier_init();
    fence_proxy_async();
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 2 || warp == 3) {
    if (t_begin + nt > v.nPT) build_mask(a, b, node0, nodes_per_tile, u.W, sMask, v.N, tid - 64, 64);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  float row_state_m = -INFINITY, row_state_l = 0.f;   // softmax threads: the row's final max and sum

  if (warp == 0) {
    // ------------------------------------------------------------ producer (one thread)
    if (lane == 0) {
      mbar_expect_tx(&bars.q_full, kQBytes);
      const int zq = b * a.Nmax + node0;
      tma_load_3d(sQ, &tmQ, 0, g * G, zq, &bars.q_full);
      tma_load_3d(sQ + kQBytes / 2, &tmQ, 64, g * G, zq, &bars.q_full);
      int issued = 0;
      for (int i = 0; i < nt; ++i) {
        const int st = i % u.stages;
        if (i >= u.stages && !mbar_wait(&bars.kv_empty[st], ((i / u.stages) - 1) & 1)) {
          abort_cta(a, b, &s_abort);
          break;
        }
        if (s_abort) break;
        uint8_t* dK = sKV + (size_t)st * kStageBytes;
        uint8_t* dV = dK + 2 * kHalf;
        mbar_expect_tx(&bars.kv_full[st], kStageBytes);
        const int t = t_begin + i;
        if (t < v.nPT) {
          const int pos0 = t * kBN;
          if (a.block_table == nullptr) {
            const int y = (b * a.Hkv + g) * a.Lcap + pos0;
            tma_load_2d(dK, &tmK, 0, y, &bars.kv_full[st]);
            tma_load_2d(dK + kHalf, &tmK, 64, y, &bars.kv_full[st]);
            tma_load_2d(dV, &tmV, 0, y, &bars.kv_full[st]);
            tma_load_2d(dV + kHalf, &tmV, 64, y, &bars.kv_full[st]);
          } else {
            const int bs_mask = (1 << a.block_shift) - 1;
            for (int seg = 0; seg < kBN; seg += u.box_rows) {
              const int pos = pos0 + seg;
              const int bi = min(pos >> a.block_shift, a.max_blocks - 1);
              int blk = a.block_table[(size_t)b * a.max_blocks + bi];
              if (blk < 0 || blk >= a.num_blocks) {
                if (pos < v.L) s_err = 1;
                blk = 0;
              }
              const int y = (blk * a.Hkv + g) * (1 << a.block_shift) + (pos & bs_mask);
              const uint32_t off = (uint32_t)seg * 128;
              tma_load_2d(dK + off, &tmK, 0, y, &bars.kv_full[st]);
              tma_load_2d(dK + kHalf + off, &tmK, 64, y, &bars.kv_full[st]);
              tma_load_2d(dV + off, &tmV, 0, y, &bars.kv_full[st]);
              tma_load_2d(dV + kHalf + off, &tmV, 64, y, &bars.kv_full[st]);
            }
          }
        } else {
          const int z = b * a.Nmax + (t - v.nPT) * kBN;
          tma_load_3d(dK, &tmKt, 0, g, z, &bars.kv_full[st]);
          tma_load_3d(dK + kHalf, &tmKt, 64, g, z, &bars.kv_full[st]);
          tma_load_3d(dV, &tmVt, 0, g, z, &bars.kv_full[st]);
          tma_load_3d(dV + kHalf, &tmVt, 64, g, z, &bars.kv_full[st]);
        }
        ++issued;
      }
      s_issued = issued;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (one thread)
    const uint32_t idesc_s = idesc_bf16(kBM, kBN, false);
    const uint32_t idesc_o = idesc_bf16(kBM, kD, true);
    const uint32_t q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
    bool ok = mbar_wait(&bars.q_full, 0);
    int consumed = 0;
    // zero V rows past the valid keys of a partial tile (its TMA box may hold stale rows)
    auto ready_tile = [&](int i) -> bool {
      const int st = i % u.stages;
      if (!mbar_wait(&bars.kv_full[st], (i / u.stages) & 1)) return false;
      ++consumed;
      const int t = t_begin + i;
      const int nv = t < v.nPT ? min(kBN, v.L - t * kBN) : min(kBN, v.N - (t - v.nPT) * kBN);
      if (nv < kBN) {
        uint8_t* dV = sKV + (size_t)st * kStageBytes + 2 * kHalf;
        const int nchunks = (kBN - nv) * 8;   // 16-byte chunks per half
        for (int c = lane; c < 2 * nchunks; c += 32) {
          const int half = c / nchunks, cc = c % nchunks;
          *reinterpret_cast<uint4*>(dV + half * kHalf + (size_t)nv * 128 + (size_t)cc * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async();
      }
      __syncwarp();
      return true;
    };
    auto issue_s = [&](int i) {
      const int st = i % u.stages;
      const uint32_t k_addr = smem_u32(sKV + (size_t)st * kStageBytes);
      const uint32_t d = tmem + kColS + (uint32_t)(i & 1) * kBN;
      if (lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t half = (uint32_t)(kk >> 2), within = (uint32_t)(kk & 3) * 32;
          const uint64_t ad = sdesc_sw128(q_addr + half * (kQBytes / 2) + within, 16, 1024);
          const uint64_t bd = sdesc_sw128(k_addr + half * kHalf + within, 16, 1024);
          mma_bf16_ss(d, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars.s_full[i & 1]);
      }
      __syncwarp();
    };
    if (ok && nt > 0) {
      ok = ready_tile(0);
      if (ok) issue_s(0);
    }
    for (int i = 0; ok && i < nt; ++i) {
      if (i + 1 < nt) {
        ok = ready_tile(i + 1);
        if (!ok) break;
        issue_s(i + 1);
      }
      if (!mbar_wait(&bars.p_full, i & 1)) {
        ok = false;
        break;
      }
      const int st = i % u.stages;
      const uint32_t v_addr = smem_u32(sKV + (size_t)st * kStageBytes + 2 * kHalf);
      if (lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int kb = 0; kb < kBN / 16; ++kb) {
          const uint64_t ad = sdesc_sw128(p_addr + (uint32_t)kb * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(v_addr + (uint32_t)kb * 2048, kHalf, 1024);
          mma_bf16_ss(tmem + kColO, ad, bd, idesc_o, (i > 0 || kb > 0) ? 1u : 0u);
        }
        tc_commit(&bars.kv_empty[st]);
        tc_commit(&bars.pv_done);
      }
      __syncwarp();
    }
    if (!ok) abort_cta(a, b, &s_abort);
    if (lane == 0) s_consumed = consumed;
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp - 4;
    const int row = q4 * 32 + lane;
    const int r = r0 + row;
    const bool row_ok = r < r_hi;
    const int nl = row / G;
    const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
    const float sl2 = a.scale * kLog2e;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < nt; ++i) {
      if (!mbar_wait(&bars.s_full[i & 1], (i >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s0[32], s1[32];
      tmem_ld32(lane_addr + kColS + (uint32_t)(i & 1) * kBN, s0);
      tmem_ld32(lane_addr + kColS + (uint32_t)(i & 1) * kBN + 32, s1);
      tmem_wait_ld();
      const int t = t_begin + i;
      const bool tree = t >= v.nPT;
      const int kbase = tree ? (t - v.nPT) * kBN : t * kBN;
      const int lim = tree ? v.N : v.L;
      uint32_t w0 = 0xffffffffu, w1 = 0xffffffffu;
      if (tree) {
        const int wi = kbase >> 5;
        w0 = sMask[nl * u.W + wi];
        w1 = (wi + 1 < u.W) ? sMask[nl * u.W + wi + 1] : 0u;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const bool v0 = row_ok && (kbase + c < lim) && ((w0 >> c) & 1u);
        const bool v1 = row_ok && (kbase + 32 + c < lim) && ((w1 >> c) & 1u);
        const float x0 = v0 ? __uint_as_float(s0[c]) * sl2 : -INFINITY;
        const float x1 = v1 ? __uint_as_float(s1[c]) * sl2 : -INFINITY;
        s0[c] = __float_as_uint(x0);
        s1[c] = __float_as_uint(x1);
        mx = fmaxf(mx, fmaxf(x0, x1));
      }
      float alpha = 1.f;
      bool resc = false;
      if (mx != -INFINITY && (m_used == -INFINITY || mx > m_used + kRescaleLog2)) {
        if (m_used != -INFINITY) {
          alpha = exp2f(m_used - mx);
          resc = true;
        }
        m_used = mx;
      }
      const float mu = m_used == -INFINITY ? 0.f : m_used;
      float sum = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float p0 = exp2f(__uint_as_float(s0[c]) - mu), p1 = exp2f(__uint_as_float(s0[c + 1]) - mu);
        const float p2 = exp2f(__uint_as_float(s1[c]) - mu), p3 = exp2f(__uint_as_float(s1[c + 1]) - mu);
        sum += (p0 + p1) + (p2 + p3);
        pk[c / 2] = pack_bf16x2(p0, p1);
        pk[16 + c / 2] = pack_bf16x2(p2, p3);
      }
      l = l * alpha + sum;
      if (i > 0 && !mbar_wait(&bars.pv_done, (i - 1) & 1)) {
        ok = false;
        break;
      }
      if (__any_sync(0xffffffffu, resc)) {   // warp-collective TMEM read-modify-write of O
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < kD / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(lane_addr + kColO + ch * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(lane_addr + kColO + ch * 32, o);
        }
        tmem_wait_st();
      }
      // P row -> swizzled shared tile (row = TMEM lane), then hand it to the MMA warp
      uint8_t* prow = sP + (size_t)row * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full);
    }
    if (ok && nt > 0 && !mbar_wait(&bars.pv_done, (nt - 1) & 1)) ok = false;
    if (!ok) abort_cta(a, b, &s_abort);
    row_state_m = m_used;
    row_state_l = l;
  }
  // ---------------------------------------------------------------- epilogue / teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (!s_abort) {
    if (warp >= 4) {
      const int q4 = warp - 4;
      const int row = q4 * 32 + lane;
      const int r = r0 + row;
      const bool row_ok = r < r_hi;
      const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
      const float m_used = row_state_m, l = row_state_l;
      const bool err = s_err != 0;
      const int i_node = r / G, hh = r % G;
      if (direct) {
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) +
                              (((size_t)b * a.Nmax + (row_ok ? i_node : 0)) * a.Hq + g * G + hh) * kD;
        const float inv = (l > 0.f && !err) ? 1.f / l : 0.f;
#pragma unroll
        for (int ch = 0; ch < kD / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(lane_addr + kColO + ch * 32, o);
          tmem_wait_ld();
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              dst[q] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * q]) * inv, __uint_as_float(o[8 * q + 1]) * inv),
                                  pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv),
                                  pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv),
                                  pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv));
            }
          }
        }
        if (row_ok && a.lse)
          a.lse[((size_t)b * a.Nmax + i_node) * a.Hq + g * G + hh] = err ? 0.f : (m_used + __log2f(l)) * kLn2;
      } else {
        float* wo = reinterpret_cast<float*>(a.workspace);
        const size_t base = (((size_t)b * a.Hkv + g) * u.splits + split) * u.Rmax;
        float* wml = wo + (size_t)a.B * a.Hkv * u.splits * u.Rmax * kD;
#pragma unroll
        for (int ch = 0; ch < kD / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(lane_addr + kColO + ch * 32, o);
          tmem_wait_ld();
          if (row_ok) {
            float4* dst = reinterpret_cast<float4*>(wo + (base + r) * kD + ch * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(__uint_as_float(o[4 * q]), __uint_as_float(o[4 * q + 1]),
                                   __uint_as_float(o[4 * q + 2]), __uint_as_float(o[4 * q + 3]));
          }
        }
        if (row_ok) *reinterpret_cast<float2*>(wml + (base + r) * 2) = make_float2(m_used, l);
      }
      if (err && split == 0 && mt == 0 && g == 0 && tid == 128) flag_status(a.status, b, TSD_ERR_CAPACITY);
    }
  } else {
    // time-out: let this CTA's own TMA copies and MMAs land (bounded) before freeing TMEM
    if (tid == 0)
      for (int i = s_consumed; i < s_issued; ++i) mbar_wait(&bars.kv_full[i % u.stages], (i / u.stages) & 1);
    if (warp == 1 && lane == 0) {
      tc_commit(&bars.fin);
      mbar_wait(&bars.fin, 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
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

tsd_status launch_attention_umma(const AttnArgs& a, const AttnPlan& p, cudaStream_t stream) {
  const int G = a.Hq / a.Hkv;
  UParams u{};
  u.tps = p.tps, u.splits = p.splits, u.Rmax = p.Rmax, u.mtiles = p.mtiles;
  u.W = (a.Nmax + 31) / 32;
  const uint32_t mask_bytes = (uint32_t)(kBM / G) * u.W * 4;
  u.stages = 4;
  auto total = [&](int st) { return 1024 + kQBytes + (uint32_t)st * kStageBytes + kPBytes + mask_bytes; };
  if (total(u.stages) > 227 * 1024) u.stages = 3;
  if (total(u.stages) > 227 * 1024) return TSD_ERR_INVALID_ARG;
  u.p_off = kQBytes + (uint32_t)u.stages * kStageBytes;
  u.mask_off = u.p_off + kPBytes;
  const size_t smem = total(u.stages);

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
  cudaFuncSetAttribute(attn_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid(p.mtiles * p.splits, a.Hkv, a.B);
  attn_umma_kernel<<<grid, kThreadsU, smem, stream>>>(mq, mk, mv, mkt, mvt, a, u);
  return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
}

}  // namespace tsd
