// a3: attention on tcgen05.  One CTA = (query tile of 128 rows, query head j,
// batch element b, key split z).  Keys are the concatenation of segment A (the
// cached prompt window) and segment B (the pass's own keys: the canvas, or the
// prompt itself in the causal prefill).  Per key tile of 128:
//   S = Q K^T          (TMEM, fp32)             — tcgen05.mma, operands by TMA
//   P = exp(S/sqrt(h) - m) (bf16, 128B-swizzled smem, written by the row's thread)
//   O_t = P V          (TMEM)                   — V cached transposed (h x keys)
//   O = O * e^(m_old - m_new) + O_t, l likewise (registers, one row per thread)
// Each split writes its unnormalised O, m and l; attn_combine merges the splits
// in a fixed order.  Grouped-query: head j reads key/value head j / (Hq/Hkv).
//
// Passages: bidirectional attention inside the canvas and attention to the
// prompt's KV cache — "DiffusionGemma 技术报告" (full translation page), §3.1
// (canvas conditioned on the cache) and §3.2 (decoder forward); causal context
// pass with sliding window 1024 — §3.1 and the explainer page "DiffusionGemma
// 深度解析", list "核心架构参数".
#pragma once

#include "k_tc_gemm.cuh"

namespace dg {

struct AttnParams {
  int nq;          // queries per batch element (rows b*nq .. b*nq + nq - 1 of Q)
  int qpos0;       // absolute position of query 0
  int Hq, Hkv;
  int nA, kposA, rowsA, vrowsA;  // segment A: keys, first position, K rows per (b,g), V^T rows base
  int nB, kposB, rowsB;          // segment B
  int causal, window;
  int tiles_per_split;
  int layer_rowA;   // first K row of this layer's segment A for (b=0, g=0)
  int layer_vrowA;  // first V^T row of this layer's segment A for (b=0, g=0)
  float* part_o;    // [splits, B*nq, Hq, 128]
  float* part_ml;   // [splits, B*nq, Hq, 2]
  int B;
  float scale_log2;  // log2(e) / sqrt(h)
};

constexpr int AT_KT = 128;  // keys per tile
constexpr uint32_t AT_SUB = 128 * 64 * 2;
constexpr size_t AT_SMEM = 1024 + 2 * AT_SUB /*Q*/ + 2 * (4 * AT_SUB) /*K,V x2*/ + 2 * AT_SUB /*P*/ + 256;

// h = 128 only (two 64-wide swizzle atoms along the head dimension).
__global__ void __launch_bounds__(128, 1)
    tc_attn_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mKA,
                   const __grid_constant__ CUtensorMap mVA, const __grid_constant__ CUtensorMap mKB,
                   const __grid_constant__ CUtensorMap mVB, AttnParams p, int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem;                       // 2 sub-tiles
  uint8_t* sKV = sQ + 2 * AT_SUB;           // stage s: K (2 sub) then V^T (2 sub)
  uint8_t* sP = sKV + 2 * 4 * AT_SUB;       // 2 sub-tiles
  uint64_t* bar = reinterpret_cast<uint64_t*>(sP + 2 * AT_SUB);
  uint64_t* q_full = bar;
  uint64_t* kv_full = bar + 1;  // [2]
  uint64_t* s_done = bar + 3;
  uint64_t* o_done = bar + 4;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 5);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hq = p.Hq;
  const int qt = blockIdx.x / Hq, j = blockIdx.x % Hq;
  const int b = blockIdx.y, z = blockIdx.z;
  const int g = j / (Hq / p.Hkv);
  const int q0 = qt * 128;
  const int row = q0 + tid;  // this thread's query (within the batch element)
  const int qp = p.qpos0 + row;

  // key tiles of this split
  const int TA = (p.nA + AT_KT - 1) / AT_KT, TB = (p.nB + AT_KT - 1) / AT_KT;
  int t_lo = 0, t_hi = TA + TB;
  if (p.causal) {  // only segment B; tiles meeting [q0 - window + 1, q0 + 127]
    const int lo_pos = max(p.kposB, p.qpos0 + q0 - p.window + 1);
    const int hi_pos = min(p.kposB + p.nB - 1, p.qpos0 + min(q0 + 127, p.nq - 1));
    t_lo = TA + (lo_pos - p.kposB) / AT_KT;
    t_hi = TA + (hi_pos - p.kposB) / AT_KT + 1;
  }
  const int my_lo = t_lo + z * p.tiles_per_split;
  const int my_hi = min(t_hi, my_lo + p.tiles_per_split);
  const int nt = max(0, my_hi - my_lo);

  if (tid == 0) {
    tc::mbar_init(q_full, 1);
    tc::mbar_init(kv_full, 1);
    tc::mbar_init(kv_full + 1, 1);
    tc::mbar_init(s_done, 1);
    tc::mbar_init(o_done, 1);
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tslot, 256);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
  pdl_enter();  // global memory is touched only from here on

  auto load_tile = [&](int i) {  // tile index i within this split -> stage i & 1
    const int t = my_lo + i;
    uint8_t* st = sKV + (i & 1) * 4 * AT_SUB;
    uint64_t* fb = kv_full + (i & 1);
    tc::mbar_expect_tx(fb, 4 * AT_SUB);
    if (t < TA) {
      const int t0 = t * AT_KT;
      const int krow = p.layer_rowA + (b * p.Hkv + g) * p.rowsA + t0;
      const int vrow = p.layer_vrowA + (b * p.Hkv + g) * 128;
      tc::tma_load_2d(st, &mKA, fb, 0, krow);
      tc::tma_load_2d(st + AT_SUB, &mKA, fb, 64, krow);
      tc::tma_load_2d(st + 2 * AT_SUB, &mVA, fb, t0, vrow);
      tc::tma_load_2d(st + 3 * AT_SUB, &mVA, fb, t0 + 64, vrow);
    } else {
      const int t0 = (t - TA) * AT_KT;
      const int krow = (b * p.Hkv + g) * p.rowsB + t0;
      const int vrow = (b * p.Hkv + g) * 128;
      tc::tma_load_2d(st, &mKB, fb, 0, krow);
      tc::tma_load_2d(st + AT_SUB, &mKB, fb, 64, krow);
      tc::tma_load_2d(st + 2 * AT_SUB, &mVB, fb, t0, vrow);
      tc::tma_load_2d(st + 3 * AT_SUB, &mVB, fb, t0 + 64, vrow);
    }
  };

  bool ok = true;
  if (tid == 0 && nt > 0) {
    tc::mbar_expect_tx(q_full, 2 * AT_SUB);
    const int qrow = b * p.nq + q0;
    tc::tma_load_2d(sQ, &mQ, q_full, j * 128, qrow);
    tc::tma_load_2d(sQ + AT_SUB, &mQ, q_full, j * 128 + 64, qrow);
    load_tile(0);
    if (nt > 1) load_tile(1);
  }

  float o[128];
#pragma unroll
  for (int d = 0; d < 128; ++d) o[d] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  constexpr uint32_t idesc = tc::idesc_bf16(128, 128);

  for (int i = 0; i < nt && ok; ++i) {
    const int t = my_lo + i;
    const bool segA = t < TA;
    const int t0 = segA ? t * AT_KT : (t - TA) * AT_KT;
    const int nseg = segA ? p.nA : p.nB;
    const int kpos0 = (segA ? p.kposA : p.kposB) + t0;
    uint8_t* st = sKV + (i & 1) * 4 * AT_SUB;
    // ---- S = Q K^T
    if (tid == 0) {
      bool w1 = i > 0 || tc::mbar_wait(q_full, 0);
      bool w2 = w1 && tc::mbar_wait(kv_full + (i & 1), (i >> 1) & 1);
      if (!w2) {
        atomicOr(err, ERR_TIMEOUT);
      } else {
        tc::fence_after_sync();
        const uint32_t qa = tc::smem_addr(sQ), ka = tc::smem_addr(st);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_bf16(tS, tc::sdesc_k128(qa + kb * AT_SUB + k * 32),
                         tc::sdesc_k128(ka + kb * AT_SUB + k * 32), idesc, (kb | k) != 0);
        tc::mma_commit(s_done);
      }
    }
    __syncwarp();
    bool ready = true;
    if (lane == 0) ready = tc::mbar_wait(s_done, i & 1);
    ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
    if (!__syncthreads_and(ready ? 1 : 0)) {
      if (tid == 0) atomicOr(err, ERR_TIMEOUT);
      ok = false;
      break;
    }
    tc::fence_after_sync();
    // ---- softmax of this row over the tile (two passes over TMEM)
    float mt = -INFINITY;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float v[32];
      tc::tmem_ld32(tS + lane_base + c * 32, v);
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const int kk = t0 + c * 32 + q;
        const int kp = kpos0 + c * 32 + q;
        bool valid = kk < nseg;
        if (p.causal) valid = valid && kp <= qp && kp > qp - p.window;
        if (valid) mt = fmaxf(mt, v[q] * p.scale_log2);
      }
    }
    const float m_new = fmaxf(m_run, mt);
    const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_run - m_new);
    float lsum = 0.f;
    const int r7 = tid & 7;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float v[32];
      tc::tmem_ld32(tS + lane_base + c * 32, v);
      uint32_t pk[16];
#pragma unroll
      for (int q = 0; q < 32; q += 2) {
        float e2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int kk = t0 + c * 32 + q + u;
          const int kp = kpos0 + c * 32 + q + u;
          bool valid = kk < nseg;
          if (p.causal) valid = valid && kp <= qp && kp > qp - p.window;
          e2[u] = valid ? exp2f(v[q + u] * p.scale_log2 - m_new) : 0.f;
          lsum += e2[u];
        }
        __nv_bfloat162 b2 = __floats2bfloat162_rn(e2[0], e2[1]);
        pk[q >> 1] = *reinterpret_cast<uint32_t*>(&b2);
      }
      // keys c*32 .. c*32+31 -> sub-tile c/2, 16-byte chunks (c%2)*4 .. +3, swizzled by row
      uint8_t* base = sP + (c >> 1) * AT_SUB + tid * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int chunk = (c & 1) * 4 + q;
        *reinterpret_cast<uint4*>(base + ((chunk ^ r7) << 4)) =
            make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
    }
    l_run = l_run * alpha + lsum;
    m_run = m_new;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc::fence_before_sync();
    __syncthreads();
    // ---- O_t = P V
    if (tid == 0) {
      tc::fence_after_sync();
      const uint32_t pa = tc::smem_addr(sP), va = tc::smem_addr(st + 2 * AT_SUB);
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc::mma_bf16(tO, tc::sdesc_k128(pa + kb * AT_SUB + k * 32),
                       tc::sdesc_k128(va + kb * AT_SUB + k * 32), idesc, (kb | k) != 0);
      tc::mma_commit(o_done);
    }
    __syncwarp();
    ready = true;
    if (lane == 0) ready = tc::mbar_wait(o_done, i & 1);
    ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
    if (!__syncthreads_and(ready ? 1 : 0)) {
      if (tid == 0) atomicOr(err, ERR_TIMEOUT);
      ok = false;
      break;
    }
    tc::fence_after_sync();
    // stage i & 1 is free again: prefetch tile i + 2
    if (tid == 0 && i + 2 < nt) load_tile(i + 2);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float v[32];
      tc::tmem_ld32(tO + lane_base + c * 32, v);
#pragma unroll
      for (int q = 0; q < 32; ++q) o[c * 32 + q] = o[c * 32 + q] * alpha + v[q];
    }
    tc::fence_before_sync();
    __syncthreads();
  }

  // ---- partial results of this split
  if (row < p.nq) {
    const size_t tok = (size_t)b * p.nq + row;
    const size_t ntok = (size_t)p.B * p.nq;
    float* po = p.part_o + (((size_t)z * ntok + tok) * Hq + j) * 128;
#pragma unroll
    for (int d = 0; d < 128; d += 4)
      *reinterpret_cast<float4*>(po + d) = make_float4(o[d], o[d + 1], o[d + 2], o[d + 3]);
    float* pm = p.part_ml + (((size_t)z * ntok + tok) * Hq + j) * 2;
    pm[0] = (nt > 0 && ok) ? m_run : -INFINITY;
    pm[1] = (nt > 0 && ok) ? l_run : 0.f;
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, 256);
}

// Merge of the key splits (fixed order): out[tok, j, :] = sum_z e^(m_z - M) O_z /
// sum_z e^(m_z - M) l_z  (m in log2 units).  One warp per (token, head).
__global__ void attn_combine_kernel(const float* __restrict__ part_o,
                                    const float* __restrict__ part_ml, int splits, int ntok,
                                    int Hq, bf16* __restrict__ out) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const long w = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= (long)ntok * Hq) return;
  float M = -INFINITY;
  for (int z = 0; z < splits; ++z) M = fmaxf(M, part_ml[((size_t)z * ntok * Hq + w) * 2]);
  float L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int z = 0; z < splits; ++z) {
    const float mz = part_ml[((size_t)z * ntok * Hq + w) * 2];
    if (mz == -INFINITY) continue;
    const float s = exp2f(mz - M);
    L += s * part_ml[((size_t)z * ntok * Hq + w) * 2 + 1];
    const float4 v = reinterpret_cast<const float4*>(part_o + ((size_t)z * ntok * Hq + w) * 128)[lane];
    acc[0] += s * v.x;
    acc[1] += s * v.y;
    acc[2] += s * v.z;
    acc[3] += s * v.w;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  __nv_bfloat162 a = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
  __nv_bfloat162 c = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
  uint2 pk = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&c));
  reinterpret_cast<uint2*>(out + (size_t)w * 128)[lane] = pk;
}

}  // namespace dg
