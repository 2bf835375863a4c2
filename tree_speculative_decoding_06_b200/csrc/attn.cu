// tsd_tree_verify_attn: tree-masked GQA split-KV attention of the verify step.
//
// "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs", technical summary
// sec. 2 (fused tree-mask teacher execution): a tree token attends only to its ancestors on its
// own branch, so branches cannot leak.  "Acelerando Sonar a traves de la especulacion", section
// "EAGLE": a custom mask over the whole sequence costs up to half the attention speed -- here the
// committed prefix is attended without any mask and the ancestor mask touches only the tree's own
// key tiles.  Section "Programacion MTP para un solo token": matrix instructions tile the token
// dimension, so the G query heads of a KV head and the N tree nodes are stacked into one M
// dimension of G*N rows that share every K/V tile read from memory.
//
// Work decomposition: CTA = (row tile of BM query rows, key split) x KV head x sequence.  The
// keys of sequence b are its ceil(L/BN) prefix tiles followed by ceil(N/BN) tree tiles; a split
// covers `tps` consecutive tiles.  Every CTA rebuilds the ancestor bits of its own nodes in shared
// memory from the sentinel-shifted parent_s[] (walks bounded by Dmax+1 steps).  One split writes
// the normalised output directly; several write (max, sum, unnormalised output) partials that the
// combine kernel merges by log-sum-exp.
#include <climits>
#include <cstdio>
#include <cstdlib>

#include "attn_common.cuh"
#include "common.cuh"
#include "kernels.h"

namespace tsd {

namespace {

using namespace attn;

constexpr int kStages = 3;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            const void* p) {
  uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(s));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                                  const void* p) {
  uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(s));
}
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------------------------------
// bf16 path: warp-level tensor-core tiles (m16n8k16), 16 query rows per warp, K/V tiles of
// 64 keys in 128B-swizzled shared memory, 3-stage cp.async pipeline.
// ------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256, 1)
    attn_bf16_kernel(const AttnArgs a, int BM, int mtiles, int tps, int splits, int Rmax) {
  pdl_trigger();
  pdl_wait();
  constexpr int BN = 64;
  constexpr int CH = D / 8;   // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sK = sQ + (size_t)BM * D;
  __nv_bfloat16* sV = sK + (size_t)kStages * BN * D;
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sV + (size_t)kStages * BN * D);
  __shared__ int s_err;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int mt = blockIdx.x % mtiles, split = blockIdx.x / mtiles;
  const int g = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const SeqView v = seq_view(a, b, G, BN, tps);
  const int r0 = mt * BM;
  if (v.skip || r0 >= v.R) return;
  const int r_hi = min(r0 + BM, v.R);
  if (v.zero) {
    if (split == 0) zero_rows<__nv_bfloat16>(a, b, g, G, r0, r_hi);
    if (split == 0 && mt == 0 && g == 0 && tid == 0 && a.status[b] == 0) flag_status(a.status, b, TSD_ERR_CAPACITY);
    return;
  }
  if (split >= v.nsplit) return;
  const bool direct = (v.nsplit == 1);
  const int t_begin = split * tps, t_end = min(v.T, t_begin + tps), nt = t_end - t_begin;
  const int W = (a.Nmax + 31) >> 5;
  const int i_lo = r0 / G, i_cnt = (r_hi - 1) / G - i_lo + 1;
  if (tid == 0) s_err = 0;
  __syncthreads();

  const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* kc = reinterpret_cast<const __nv_bfloat16*>(a.k_cache);
  const __nv_bfloat16* vc = reinterpret_cast<const __nv_bfloat16*>(a.v_cache);
  const __nv_bfloat16* kt = reinterpret_cast<const __nv_bfloat16*>(a.k_tree);
  const __nv_bfloat16* vt = reinterpret_cast<const __nv_bfloat16*>(a.v_tree);

  // Q rows of this tile (rows past R are zero-filled).
  for (int c = tid; c < BM * CH; c += blockDim.x) {
    const int row = c / CH, ch = c % CH, r = r0 + row;
    const bool ok = r < v.R;
    const int i = ok ? r / G : 0, hh = ok ? r % G : 0;
    const __nv_bfloat16* src = q + (((size_t)b * a.Nmax + i) * a.Hq + g * G + hh) * D + ch * 8;
    cp_async_16(sQ + row * D + ((ch ^ (row & 7)) * 8), ok ? (const void*)src : (const void*)q, ok ? 16 : 0);
  }
  auto load_tile = [&](int t, int stage) {
    __nv_bfloat16* dK = sK + (size_t)stage * BN * D;
    __nv_bfloat16* dV = sV + (size_t)stage * BN * D;
    bool ok_all = true;
    for (int c = tid; c < BN * CH; c += blockDim.x) {
      const int row = c / CH, ch = c % CH;
      bool valid, from_tree, ok = true;
      const size_t off = key_row(a, v, b, g, t, BN, row, valid, from_tree, ok);
      ok_all &= ok;
      valid &= ok;
      const __nv_bfloat16* bk = from_tree ? kt : kc;
      const __nv_bfloat16* bv = from_tree ? vt : vc;
      const int dst = row * D + ((ch ^ (row & 7)) * 8);
      // a zero-fill copy reads nothing; q is only a valid placeholder address
      cp_async_16(dK + dst, valid ? (const void*)(bk + off + ch * 8) : (const void*)q, valid ? 16 : 0);
      cp_async_16(dV + dst, valid ? (const void*)(bv + off + ch * 8) : (const void*)q, valid ? 16 : 0);
    }
    if (!ok_all) s_err = 1;
  };
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < nt) load_tile(t_begin + s, s);
    cp_async_commit();
  }
  if (t_end > v.nPT) build_mask(a, b, i_lo, i_cnt, W, sMask, v.N);

  // per-thread rows: A = lane/4, B = lane/4 + 8 of this warp's 16
  const int wr0 = r0 + warp * 16;
  const bool warp_on = wr0 < r_hi;
  const int rowA = wr0 + (lane >> 2), rowB = rowA + 8;
  const bool okA = rowA < r_hi, okB = rowB < r_hi;
  const int nodeA = okA ? rowA / G - i_lo : 0, nodeB = okB ? rowB / G - i_lo : 0;
  const float sl2 = a.scale * kLog2e;

  uint32_t qf[D / 16][4];
  float o[D / 8][4];
#pragma unroll
  for (int nd = 0; nd < D / 8; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
  float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;

  for (int it = 0; it < nt; ++it) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (it + kStages - 1 < nt) load_tile(t_begin + it + kStages - 1, (it + kStages - 1) % kStages);
    cp_async_commit();
    if (it == 0 && warp_on) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int row = warp * 16 + (lane & 15), ch = 2 * kk + (lane >> 4);
        ldmatrix_x4(qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], sQ + row * D + ((ch ^ (row & 7)) * 8));
      }
    }
    if (!warp_on) continue;
    const int t = t_begin + it, stage = it % kStages;
    const __nv_bfloat16* tK = sK + (size_t)stage * BN * D;
    const __nv_bfloat16* tV = sV + (size_t)stage * BN * D;

    float s[BN / 8][4];
#pragma unroll
    for (int nb = 0; nb < BN / 8; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int nb2 = 0; nb2 < BN / 16; ++nb2) {
        const int key = nb2 * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int ch = 2 * kk + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(b0, b1, b2, b3, tK + key * D + ((ch ^ (key & 7)) * 8));
        mma_bf16_16816(s[2 * nb2], qf[kk], b0, b1);
        mma_bf16_16816(s[2 * nb2 + 1], qf[kk], b2, b3);
      }
    }
    // scale + mask (prefix: key < L; tree: node < N and ancestor bit set)
    const bool tree_tile = t >= v.nPT;
    const int kbase = tree_tile ? (t - v.nPT) * BN : t * BN;
    const int lim = tree_tile ? v.N : v.L;
    uint32_t wA0 = 0xffffffffu, wA1 = 0xffffffffu, wB0 = 0xffffffffu, wB1 = 0xffffffffu;
    if (tree_tile) {
      const int w0 = kbase >> 5;
      wA0 = sMask[nodeA * W + w0];
      wB0 = sMask[nodeB * W + w0];
      wA1 = (w0 + 1 < W) ? sMask[nodeA * W + w0 + 1] : 0u;
      wB1 = (w0 + 1 < W) ? sMask[nodeB * W + w0 + 1] : 0u;
    }
    float mxA = -INFINITY, mxB = -INFINITY;
#pragma unroll
    for (int nb = 0; nb < BN / 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = nb * 8 + 2 * (lane & 3) + e;
        const bool kin = kbase + col < lim;
        const uint32_t bitA = col < 32 ? (wA0 >> col) : (wA1 >> (col - 32));
        const uint32_t bitB = col < 32 ? (wB0 >> col) : (wB1 >> (col - 32));
        const bool vA = okA && kin && (bitA & 1u);
        const bool vB = okB && kin && (bitB & 1u);
        s[nb][e] = vA ? s[nb][e] * sl2 : -INFINITY;
        s[nb][2 + e] = vB ? s[nb][2 + e] * sl2 : -INFINITY;
        mxA = fmaxf(mxA, s[nb][e]);
        mxB = fmaxf(mxB, s[nb][2 + e]);
      }
    }
    mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 1));
    mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 2));
    mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 1));
    mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 2));
    const float nA = fmaxf(mA, mxA), nB = fmaxf(mB, mxB);
    const float uA = nA == -INFINITY ? 0.f : nA, uB = nB == -INFINITY ? 0.f : nB;
    const float alA = exp2f(mA - uA), alB = exp2f(mB - uB);
    mA = nA;
    mB = nB;
    float sumA = 0.f, sumB = 0.f;
#pragma unroll
    for (int nb = 0; nb < BN / 8; ++nb) {
      s[nb][0] = exp2f(s[nb][0] - uA);
      s[nb][1] = exp2f(s[nb][1] - uA);
      s[nb][2] = exp2f(s[nb][2] - uB);
      s[nb][3] = exp2f(s[nb][3] - uB);
      sumA += s[nb][0] + s[nb][1];
      sumB += s[nb][2] + s[nb][3];
    }
    lA = lA * alA + sumA;
    lB = lB * alB + sumB;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
      o[nd][0] *= alA;
      o[nd][1] *= alA;
      o[nd][2] *= alB;
      o[nd][3] *= alB;
    }
    // O += P V
#pragma unroll
    for (int kb = 0; kb < BN / 16; ++kb) {
      uint32_t pa[4];
      pa[0] = pack_bf16x2(s[2 * kb][0], s[2 * kb][1]);
      pa[1] = pack_bf16x2(s[2 * kb][2], s[2 * kb][3]);
      pa[2] = pack_bf16x2(s[2 * kb + 1][0], s[2 * kb + 1][1]);
      pa[3] = pack_bf16x2(s[2 * kb + 1][2], s[2 * kb + 1][3]);
#pragma unroll
      for (int nd2 = 0; nd2 < D / 16; ++nd2) {
        const int key = kb * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int ch = 2 * nd2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(b0, b1, b2, b3, tV + key * D + ((ch ^ (key & 7)) * 8));
        mma_bf16_16816(o[2 * nd2], pa, b0, b1);
        mma_bf16_16816(o[2 * nd2 + 1], pa, b2, b3);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  const bool err = s_err != 0;
  if (err && tid == 0) flag_status(a.status, b, TSD_ERR_CAPACITY);
  if (!warp_on) return;
  lA += __shfl_xor_sync(0xffffffffu, lA, 1);
  lA += __shfl_xor_sync(0xffffffffu, lA, 2);
  lB += __shfl_xor_sync(0xffffffffu, lB, 1);
  lB += __shfl_xor_sync(0xffffffffu, lB, 2);
  const int hA = okA ? rowA % G : 0, hB = okB ? rowB % G : 0;
  const int iA = okA ? rowA / G : 0, iB = okB ? rowB / G : 0;
  if (direct) {
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
    const float invA = (lA > 0.f && !err) ? 1.f / lA : 0.f, invB = (lB > 0.f && !err) ? 1.f / lB : 0.f;
    __nv_bfloat16* oA = out + (((size_t)b * a.Nmax + iA) * a.Hq + g * G + hA) * D;
    __nv_bfloat16* oB = out + (((size_t)b * a.Nmax + iB) * a.Hq + g * G + hB) * D;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
      const int col = nd * 8 + 2 * (lane & 3);
      if (okA) *reinterpret_cast<uint32_t*>(oA + col) = pack_bf16x2(o[nd][0] * invA, o[nd][1] * invA);
      if (okB) *reinterpret_cast<uint32_t*>(oB + col) = pack_bf16x2(o[nd][2] * invB, o[nd][3] * invB);
    }
    if (a.lse && (lane & 3) == 0) {
      if (okA)
        a.lse[((size_t)b * a.Nmax + iA) * a.Hq + g * G + hA] = err ? 0.f : (mA + __log2f(lA)) * kLn2;
      if (okB)
        a.lse[((size_t)b * a.Nmax + iB) * a.Hq + g * G + hB] = err ? 0.f : (mB + __log2f(lB)) * kLn2;
    }
  } else {
    float* wo = reinterpret_cast<float*>(a.workspace);
    const size_t base = (((size_t)b * a.Hkv + g) * splits + split) * Rmax;
    float* wml = wo + (size_t)a.B * a.Hkv * splits * Rmax * D;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
      const int col = nd * 8 + 2 * (lane & 3);
      if (okA) *reinterpret_cast<float2*>(wo + (base + rowA) * D + col) = make_float2(o[nd][0], o[nd][1]);
      if (okB) *reinterpret_cast<float2*>(wo + (base + rowB) * D + col) = make_float2(o[nd][2], o[nd][3]);
    }
    if ((lane & 3) == 0) {
      if (okA) *reinterpret_cast<float2*>(wml + (base + rowA) * 2) = make_float2(mA, lA);
      if (okB) *reinterpret_cast<float2*>(wml + (base + rowB) * 2) = make_float2(mB, lB);
    }
  }
}

// ------------------------------------------------------------------------------------------
// fp32 path (FFMA; the fp32 tolerance excludes tf32 tensor cores): one warp per query row at
// a time, one key per lane, 32-key tiles in padded shared memory.
// ------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) attn_f32_kernel(const AttnArgs a, int BM, int mtiles, int tps, int splits,
                                                       int Rmax) {
  pdl_trigger();
  pdl_wait();
  constexpr int BN = 32, RPW = 4, E = D / 32, LD = D + 1;
  extern __shared__ __align__(128) uint8_t smem[];
  float* sQ = reinterpret_cast<float*>(smem);
  float* sK = sQ + 16 * D;
  float* sV = sK + BN * LD;
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sV + BN * LD);
  __shared__ int s_err;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int mt = blockIdx.x % mtiles, split = blockIdx.x / mtiles;
  const int g = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const SeqView v = seq_view(a, b, G, BN, tps);
  const int r0 = mt * BM;
  if (v.skip || r0 >= v.R) return;
  const int r_hi = min(r0 + BM, v.R);
  if (v.zero) {
    if (split == 0) zero_rows<float>(a, b, g, G, r0, r_hi);
    if (split == 0 && mt == 0 && g == 0 && tid == 0 && a.status[b] == 0) flag_status(a.status, b, TSD_ERR_CAPACITY);
    return;
  }
  if (split >= v.nsplit) return;
  const bool direct = (v.nsplit == 1);
  const int t_begin = split * tps, t_end = min(v.T, t_begin + tps);
  const int W = (a.Nmax + 31) >> 5;
  const int i_lo = r0 / G, i_cnt = (r_hi - 1) / G - i_lo + 1;
  const float* q = reinterpret_cast<const float*>(a.q);
  const float* kc = reinterpret_cast<const float*>(a.k_cache);
  const float* vc = reinterpret_cast<const float*>(a.v_cache);
  const float* kt = reinterpret_cast<const float*>(a.k_tree);
  const float* vt = reinterpret_cast<const float*>(a.v_tree);
  if (tid == 0) s_err = 0;
  for (int idx = tid; idx < BM * D; idx += blockDim.x) {
    const int row = idx / D, c = idx % D, r = r0 + row;
    float x = 0.f;
    if (r < v.R) x = q[(((size_t)b * a.Nmax + r / G) * a.Hq + g * G + r % G) * D + c];
    sQ[row * D + c] = x;
  }
  if (t_end > v.nPT) build_mask(a, b, i_lo, i_cnt, W, sMask, v.N);
  const float sl2 = a.scale * kLog2e;
  float m[RPW], l[RPW], o[RPW][E];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[rr][e] = 0.f;
  }
  for (int t = t_begin; t < t_end; ++t) {
    __syncthreads();
    bool ok_all = true;
    for (int idx = tid; idx < BN * D; idx += blockDim.x) {
      const int row = idx / D, c = idx % D;
      bool valid, from_tree, ok = true;
      const size_t off = key_row(a, v, b, g, t, BN, row, valid, from_tree, ok);
      ok_all &= ok;
      valid &= ok;
      sK[row * LD + c] = valid ? (from_tree ? kt : kc)[off + c] : 0.f;
      sV[row * LD + c] = valid ? (from_tree ? vt : vc)[off + c] : 0.f;
    }
    if (!ok_all) s_err = 1;
    __syncthreads();
    const bool tree_tile = t >= v.nPT;
    const int kbase = tree_tile ? (t - v.nPT) * BN : t * BN;
    const int lim = tree_tile ? v.N : v.L;
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      const int lr = warp * RPW + rr, r = r0 + lr;
      if (r >= r_hi) continue;
      float s = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) s = fmaf(sQ[lr * D + c], sK[lane * LD + c], s);
      bool valid = kbase + lane < lim;
      if (tree_tile && valid) {
        const int node = r / G - i_lo, j = kbase + lane;
        valid = (sMask[node * W + (j >> 5)] >> (j & 31)) & 1u;
      }
      s = valid ? s * sl2 : -INFINITY;
      const float nm = fmaxf(m[rr], warp_max(s));
      const float use = nm == -INFINITY ? 0.f : nm;
      const float al = exp2f(m[rr] - use);
      const float p = exp2f(s - use);
      l[rr] = l[rr] * al + warp_sum(p);
      m[rr] = nm;
#pragma unroll
      for (int e = 0; e < E; ++e) o[rr][e] *= al;
      for (int k = 0; k < BN; ++k) {
        const float pk = __shfl_sync(0xffffffffu, p, k);
#pragma unroll
        for (int e = 0; e < E; ++e) o[rr][e] = fmaf(pk, sV[k * LD + lane + 32 * e], o[rr][e]);
      }
    }
  }
  __syncthreads();
  const bool err = s_err != 0;
  if (err && tid == 0) flag_status(a.status, b, TSD_ERR_CAPACITY);
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int r = r0 + warp * RPW + rr;
    if (r >= r_hi) continue;
    const int i = r / G, hh = r % G;
    if (direct) {
      float* out = reinterpret_cast<float*>(a.out) + (((size_t)b * a.Nmax + i) * a.Hq + g * G + hh) * D;
      const float inv = (l[rr] > 0.f && !err) ? 1.f / l[rr] : 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) out[lane + 32 * e] = o[rr][e] * inv;
      if (a.lse && lane == 0)
        a.lse[((size_t)b * a.Nmax + i) * a.Hq + g * G + hh] = err ? 0.f : (m[rr] + __log2f(l[rr])) * kLn2;
    } else {
      float* wo = reinterpret_cast<float*>(a.workspace);
      const size_t base = (((size_t)b * a.Hkv + g) * splits + split) * Rmax + r;
      float* wml = wo + (size_t)a.B * a.Hkv * splits * Rmax * D;
#pragma unroll
      for (int e = 0; e < E; ++e) wo[base * D + lane + 32 * e] = o[rr][e];
      if (lane == 0) *reinterpret_cast<float2*>(wml + base * 2) = make_float2(m[rr], l[rr]);
    }
  }
}

// ------------------------------------------------------------------------------------------
// Split merge: o = sum_s o_s 2^(m_s - M) / sum_s l_s 2^(m_s - M), one warp per query row.
// ------------------------------------------------------------------------------------------
constexpr int kFastSplits = 16;   // merges of up to this many splits load everything at once

// equal != 0: every sequence has `splits` partials (the tcgen05 kernel's equal shares, where a
// split with no keys wrote M = -inf); else ceil(tiles / tps) of them.  A partial whose weight is 0
// is skipped without reading its O.
template <int D, typename OutT>
__global__ void attn_combine_kernel(const AttnArgs a, int BN, int tps, int splits, int Rmax, int equal) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * (blockDim.x >> 5) + warp;
  const int g = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  SeqView v = seq_view(a, b, G, BN, tps);
  if (equal) v.nsplit = splits;
  if (v.skip || r >= v.R) return;
  const int i = r / G, hh = r % G;
  OutT* orow = reinterpret_cast<OutT*>(a.out) + (((size_t)b * a.Nmax + i) * a.Hq + g * G + hh) * D;
  float* lrow = a.lse ? a.lse + ((size_t)b * a.Nmax + i) * a.Hq + g * G + hh : nullptr;
  if (v.zero) {
#pragma unroll
    for (int e = 0; e < D / 32; ++e) store_out(orow + lane + 32 * e, 0.f);
    if (lrow && lane == 0) *lrow = 0.f;
    return;
  }
  if (v.nsplit <= 1) return;
  const float* wo = reinterpret_cast<const float*>(a.workspace);
  const float* wml = wo + (size_t)a.B * a.Hkv * splits * Rmax * D;
  const size_t base = ((size_t)b * a.Hkv + g) * splits * Rmax + r;
  if (v.nsplit <= kFastSplits) {
    // every load is issued up front (lane s holds split s's (max, sum); each lane holds its four
    // columns of every split's partial row), so the merge waits for one round trip to memory
    float2 ml = make_float2(-INFINITY, 0.f);
    if (lane < v.nsplit) ml = *reinterpret_cast<const float2*>(wml + (base + (size_t)lane * Rmax) * 2);
    const bool use = ml.x != -INFINITY;   // lanes >= nsplit hold (-inf, 0) too
    const unsigned live = __ballot_sync(0xffffffffu, use);
    float ov[kFastSplits][D / 32];
#pragma unroll
    for (int s = 0; s < kFastSplits; ++s) {
      const float* src = wo + (base + (size_t)s * Rmax) * D + lane;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) ov[s][e] = (live >> s) & 1u ? src[32 * e] : 0.f;
    }
    const float M = warp_max(ml.x);
    const float Mu = M == -INFINITY ? 0.f : M;
    const float w = use ? exp2f(ml.x - Mu) : 0.f;
    const float lsum = warp_sum(ml.y * w);
    float acc[D / 32];
#pragma unroll
    for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;
#pragma unroll
    for (int s = 0; s < kFastSplits; ++s) {
      const float ws = __shfl_sync(0xffffffffu, w, s);
#pragma unroll
      for (int e = 0; e < D / 32; ++e) acc[e] = fmaf(ov[s][e], ws, acc[e]);
    }
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) store_out(orow + lane + 32 * e, acc[e] * inv);
    if (lrow && lane == 0) *lrow = (M + __log2f(lsum)) * kLn2;
    return;
  }
  // lane s holds split s's (max, sum): all of them are fetched at once, not one after another
  float M = -INFINITY;
  for (int s0 = 0; s0 < v.nsplit; s0 += 32) {
    const int s = s0 + lane;
    if (s < v.nsplit) M = fmaxf(M, wml[(base + (size_t)s * Rmax) * 2]);
  }
  M = warp_max(M);
  const float Mu = M == -INFINITY ? 0.f : M;
  float lsum = 0.f, acc[D / 32];
#pragma unroll
  for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;
  for (int s0 = 0; s0 < v.nsplit; s0 += 32) {
    const int s = s0 + lane;
    float w = 0.f;
    if (s < v.nsplit) {
      const float2 ml = *reinterpret_cast<const float2*>(wml + (base + (size_t)s * Rmax) * 2);
      w = ml.x == -INFINITY ? 0.f : exp2f(ml.x - Mu);
      lsum += ml.y * w;
    }
    const int n = min(32, v.nsplit - s0);
#pragma unroll 4
    for (int k = 0; k < n; ++k) {
      const float wk = __shfl_sync(0xffffffffu, w, k);
      if (wk == 0.f) continue;
      const float* src = wo + (base + (size_t)(s0 + k) * Rmax) * D + lane;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) acc[e] = fmaf(src[32 * e], wk, acc[e]);
    }
  }
  lsum = warp_sum(lsum);
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) store_out(orow + lane + 32 * e, acc[e] * inv);
  if (lrow && lane == 0) *lrow = (M + __log2f(lsum)) * kLn2;
}

template <typename K>
void set_smem_attr(K kernel, size_t bytes) {
  // cheap and idempotent; needed once per kernel for > 48 KB of dynamic shared memory
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

int device_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

AttnPlan plan_attention(int B, int Nmax, int Hq, int Hkv, int d, int Lcap, tsd_dtype dtype, bool paged) {
  AttnPlan p;
  p.G = Hq / Hkv;
  p.Rmax = p.G * Nmax;
  const int W = (Nmax + 31) / 32;
  if (dtype == TSD_BF16) {
    p.BN = 64;
    p.BM = p.Rmax >= 128 ? 128 : ((p.Rmax + 15) / 16) * 16;
    p.threads = p.BM / 16 * 32;
    p.smem = (size_t)p.BM * d * 2 + (size_t)2 * kStages * p.BN * d * 2 + (size_t)(p.BM / p.G + 2) * W * 4;
  } else {
    p.BN = 32;
    p.BM = 16;
    p.threads = 128;
    p.smem = (size_t)16 * d * 4 + (size_t)2 * 32 * (d + 1) * 4 + (size_t)(16 / p.G + 2) * W * 4;
  }
  if (p.BM <= 0) p.BM = 16;
  p.mtiles = (p.Rmax + p.BM - 1) / p.BM;
  p.max_tiles = (Lcap + p.BN - 1) / p.BN + (Nmax + p.BN - 1) / p.BN;
  // the tcgen05 kernel (bf16, d = 128, power-of-two groups) takes two 128-row query tiles per CTA
  // when a KV head has more than 128 query rows, streaming each K/V tile once for both
  const bool umma_shape = dtype == TSD_BF16 && d == 128 && p.G <= 128 && (p.G & (p.G - 1)) == 0;
  // (TSD_ATTN_DUAL=0 keeps one query tile per CTA: an A/B knob)
  const char* dual_env = getenv("TSD_ATTN_DUAL");
  p.dual = umma_shape && p.Rmax > 128 && !(dual_env != nullptr && dual_env[0] == '0');
  p.umtiles = p.dual ? (p.Rmax + 255) / 256 : p.mtiles;
  const long long base = (long long)B * Hkv * (umma_shape ? p.umtiles : p.mtiles);
  const int sms = device_sm_count();
  // Split count: the CTAs of one launch run in waves of one CTA per SM, a CTA costs its tiles plus a
  // fixed overhead (set-up, pipeline fill, epilogue) of about two tiles, and every split adds
  // partials to write and merge.
  // Minimise waves * (tiles per split + overhead) over the split counts that keep a split at least
  // min_tps tiles long (partials must stay small next to the K/V they summarise).
  const int min_tps = dtype == TSD_BF16 ? 2 : (3 * p.BM / 2 + p.BN - 1) / p.BN;
  const double overhead = 2.0;
  int best_tps = p.max_tiles > 0 ? p.max_tiles : 1;
  double best_cost = 1e300;
  for (int s = 1; s <= 64; ++s) {
    int tps = (p.max_tiles + s - 1) / s;
    if (tps < 1) tps = 1;
    if (s > 1 && tps < min_tps) break;
    const int splits = (p.max_tiles + tps - 1) / tps;
    const long long ctas = base * splits;
    const double waves = (double)((ctas + sms - 1) / sms);
    // each extra split adds a partial row set to write and merge
    const double cost = waves * (tps + overhead) + (splits > 1 ? 0.35 * splits : 0.0);
    if (cost < best_cost - 1e-9) best_cost = cost, best_tps = tps;
  }
  p.tps = best_tps;
  p.splits = (p.max_tiles + p.tps - 1) / p.tps;
  if (p.splits < 1) p.splits = 1;
  // tcgen05 kernel: CTA s of a row block's `usplits` takes the equal share [s T / n, (s+1) T / n)
  // of its own sequence's T tiles and sequences are taken longest first, so a ragged batch stays
  // balanced.  The host does not see the lengths: contiguous caches are costed at the capacity
  // length (waves x tiles per CTA); paged caches, whose sequences are usually ragged, by the mean
  // of that and a spread-lengths model (half the capacity on average: the larger of the longest
  // CTA and the total work over the SMs).  Each split adds partials to write and merge.
  if (umma_shape) {
    const long long ubase = (long long)B * Hkv * p.umtiles;
    // a two-tile CTA's fixed cost (Q rows into TMEM, the first K/V tiles through the block table,
    // the epilogue and the in-kernel merge) measured ~8 key tiles; a one-tile CTA's ~2
    const double uover = p.dual ? 8.0 : overhead;
    double best = 1e300;
    for (int c = 1; c <= 32; ++c) {
      const double per = (double)((p.max_tiles + c - 1) / c) + uover;
      const double waves = (double)((ubase * c + sms - 1) / sms);
      double cost = waves * per;
      if (paged) {
        const double spread = fmax(per, (double)ubase * (0.5 * p.max_tiles + c * uover) / sms);
        cost = 0.5 * (cost + spread);
      }
      cost += c > 1 ? 0.35 * c : 0.0;
      if (cost < best - 1e-9) best = cost, p.usplits = c;
    }
  }
  const int wsplits = p.splits > p.usplits ? p.splits : p.usplits;   // either kernel may run
  p.ws_bytes = wsplits > 1 ? kAttnTicketBytes + (size_t)B * Hkv * wsplits * p.Rmax * (d + 2) * sizeof(float) : 0;
  return p;
}

int attention_launch_count(int B, int Nmax, int Hq, int Hkv, int d, int Lcap, tsd_dtype dtype, bool paged,
                           bool tree_in_cache, long long* ctas) {
  if (ctas) *ctas = 0;
  if (B <= 0 || Nmax <= 0 || Hkv <= 0) return 0;
  const AttnPlan p = plan_attention(B, Nmax, Hq, Hkv, d, Lcap, dtype, paged);
  const char* path_env = getenv("TSD_ATTN_PATH");
  const bool force_mma = path_env != nullptr && path_env[0] == 'm' && path_env[1] == 'm';
  const int G = Hq / Hkv;
  // the tcgen05 kernel's conditions (umma_eligible), for aligned tensors
  const bool umma = dtype == TSD_BF16 && d == 128 && !tree_in_cache && G >= 1 && G <= 128 && (G & (G - 1)) == 0 &&
                    Lcap > 0 && !force_mma;
  if (ctas) {
    *ctas = umma ? (long long)B * Hkv * p.umtiles * p.usplits : (long long)B * Hkv * p.mtiles * p.splits;
  }
  if (!umma) return p.splits > 1 ? 2 : 1;
  if (p.usplits <= 1) return 1;
  UmmaLayout L;
  if (!umma_layout(p, G, Nmax, L)) return 0;
  return umma_merges_in_kernel(p, L, B, Hkv) ? 1 : 2;
}

tsd_status launch_attention(const AttnArgs& a_in, tsd_dtype dtype, cudaStream_t stream) {
  if (a_in.B == 0 || a_in.Nmax == 0) return TSD_OK;
  AttnPlan p = plan_attention(a_in.B, a_in.Nmax, a_in.Hq, a_in.Hkv, a_in.d, a_in.Lcap, dtype,
                              a_in.block_table != nullptr);
  // TSD_ATTN_SPLITS=n overrides the tcgen05 kernel's split count (a tuning knob for sweeps), when
  // the workspace the caller passed holds n partials
  if (const char* e = getenv("TSD_ATTN_SPLITS")) {
    const int n = atoi(e);
    const size_t need = kAttnTicketBytes + (size_t)a_in.B * a_in.Hkv * (size_t)n * p.Rmax * (a_in.d + 2) * sizeof(float);
    if (n >= 1 && n <= 64 && (n == 1 || need <= a_in.ws_bytes)) p.usplits = n;
  }
  // the kernels see the partials; the ticket words stay at the start of the workspace
  AttnArgs a = a_in;
  int* tickets = nullptr;
  if (a_in.workspace != nullptr && a_in.ws_bytes > kAttnTicketBytes) {
    tickets = reinterpret_cast<int*>(a_in.workspace);
    a.workspace = reinterpret_cast<uint8_t*>(a_in.workspace) + kAttnTicketBytes;
    a.ws_bytes = a_in.ws_bytes - kAttnTicketBytes;
  }
  dim3 grid(p.mtiles * p.splits, a.Hkv, a.B);
  // TSD_ATTN_PATH=mma selects the warp-level kernel even where the tcgen05 kernel applies (A/B runs)
  const char* path_env = getenv("TSD_ATTN_PATH");
  const bool force_mma = path_env != nullptr && path_env[0] == 'm' && path_env[1] == 'm';
  if (dtype == TSD_BF16 && !force_mma && umma_eligible(a, dtype)) {
    bool merged = false;
    const tsd_status st = launch_attention_umma(a, p, tickets, &merged, stream);
    if (st != TSD_OK || p.usplits <= 1 || merged) return st;
    const int rows_per_block = 8;
    dim3 cg((p.Rmax + rows_per_block - 1) / rows_per_block, a.Hkv, a.B);
    launch_pdl(attn_combine_kernel<128, __nv_bfloat16>, cg, dim3(256), 0, stream, a, p.BN, p.tps, p.usplits, p.Rmax,
               1);
    return cudaGetLastError() == cudaSuccess ? TSD_OK : TSD_ERR_CUDA;
  } else if (dtype == TSD_BF16) {
    if (a.d == 128) {
      set_smem_attr(attn_bf16_kernel<128>, p.smem);
      launch_pdl(attn_bf16_kernel<128>, grid, dim3(p.threads), p.smem, stream, a, p.BM, p.mtiles, p.tps, p.splits, p.Rmax);
    } else {
      set_smem_attr(attn_bf16_kernel<64>, p.smem);
      launch_pdl(attn_bf16_kernel<64>, grid, dim3(p.threads), p.smem, stream, a, p.BM, p.mtiles, p.tps, p.splits, p.Rmax);
    }
  } else {
    if (a.d == 128) {
      set_smem_attr(attn_f32_kernel<128>, p.smem);
      launch_pdl(attn_f32_kernel<128>, grid, dim3(p.threads), p.smem, stream, a, p.BM, p.mtiles, p.tps, p.splits, p.Rmax);
    } else {
      set_smem_attr(attn_f32_kernel<64>, p.smem);
      launch_pdl(attn_f32_kernel<64>, grid, dim3(p.threads), p.smem, stream, a, p.BM, p.mtiles, p.tps, p.splits, p.Rmax);
    }
  }
  if (cudaGetLastError() != cudaSuccess) return TSD_ERR_CUDA;
  if (p.splits > 1) {
    const int rows_per_block = 8;
    dim3 cg((p.Rmax + rows_per_block - 1) / rows_per_block, a.Hkv, a.B);
    if (dtype == TSD_BF16) {
      if (a.d == 128)
        launch_pdl(attn_combine_kernel<128, __nv_bfloat16>, cg, dim3(256), 0, stream, a, p.BN, p.tps, p.splits, p.Rmax, 0);
      else
        launch_pdl(attn_combine_kernel<64, __nv_bfloat16>, cg, dim3(256), 0, stream, a, p.BN, p.tps, p.splits, p.Rmax, 0);
    } else {
      if (a.d == 128)
        launch_pdl(attn_combine_kernel<128, float>, cg, dim3(256), 0, stream, a, p.BN, p.tps, p.splits, p.Rmax, 0);
      else
        launch_pdl(attn_combine_kernel<64, float>, cg, dim3(256), 0, stream, a, p.BN, p.tps, p.splits, p.Rmax, 0);
    }
    if (cudaGetLastError() != cudaSuccess) return TSD_ERR_CUDA;
  }
  return TSD_OK;
}

}  // namespace tsd
