// a3: attention on tcgen05.  One CTA = (query tile of 128 rows, query head j,
// batch element b, key split z); the splits of a (tile, head, b) form one thread
// block cluster.  Keys are the concatenation of segment A (the cached prompt
// window) and segment B (the pass's own keys: the canvas, or the prompt itself
// in the causal prefill).  Per key tile of 128:
//   S = Q K^T          (TMEM, two buffers: S of the next tile is computed while
//                       this tile's softmax runs)  — tcgen05.mma, operands by TMA
//   P = exp(S/sqrt(h) - m) (bf16, 128B-swizzled smem)
//   O_t = P V          (TMEM)                     — V cached transposed (h x keys)
//   O = O * e^(m_old - m_new) + O_t, l likewise   (registers)
// Eight warps: warps w and w + 4 share a TMEM lane quarter (32 query rows) and
// split the tile's keys (softmax) and the head dimension (O) in halves.  At the
// end the splits of the cluster merge through distributed shared memory in
// rank order and the owning CTA writes the normalised bf16 output rows.
// Grouped-query: head j reads key/value head j / (Hq/Hkv).
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
  int nA, kposA, rowsA;  // segment A: keys, first position, K rows per (b, g)
  int nB, kposB, rowsB;  // segment B
  int causal, window;
  int tiles_per_split;
  int layer_rowA;   // first K row of this layer's segment A for (b=0, g=0)
  int layer_vrowA;  // first V^T row of this layer's segment A for (b=0, g=0)
  int B;
  float scale_log2;  // log2(e) / sqrt(h)
  bf16* out;         // [B*nq, Hq, 128]
};

constexpr int AT_KT = 128;  // keys per tile
constexpr int AT_THREADS = 256;
constexpr uint32_t AT_SUB = 128 * 64 * 2;
constexpr int AT_RS = 132;  // merge staging row stride (floats)
constexpr size_t AT_SMEM =
    1024 + 2 * AT_SUB /*Q*/ + 2 * (4 * AT_SUB) /*K,V x2*/ + 2 * AT_SUB /*P*/ + 256 /*barriers*/ +
    2 * 128 * 4 /*row max halves*/ + 128 * 4 * 4 /*m, l halves for the merge*/;
static_assert(128 * AT_RS * 4 <= 2 * 4 * AT_SUB, "merge staging fits the K/V buffers");

// h = 128 only (two 64-wide swizzle atoms along the head dimension).
__global__ void __launch_bounds__(AT_THREADS, 1)
    tc_attn_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mKA,
                   const __grid_constant__ CUtensorMap mVA, const __grid_constant__ CUtensorMap mKB,
                   const __grid_constant__ CUtensorMap mVB, AttnParams p, int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem;                       // 2 sub-tiles
  uint8_t* sKV = sQ + 2 * AT_SUB;           // stage s: K (2 sub) then V^T (2 sub)
  uint8_t* sP = sKV + 2 * 4 * AT_SUB;       // 2 sub-tiles (keys 0..63, 64..127)
  uint64_t* bar = reinterpret_cast<uint64_t*>(sP + 2 * AT_SUB);
  uint64_t* q_full = bar;
  uint64_t* kv_full = bar + 1;  // [2]
  uint64_t* s_done = bar + 3;   // [2]
  uint64_t* o_done = bar + 5;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 6);
  float* xmax = reinterpret_cast<float*>(smem + 2 * AT_SUB + 8 * AT_SUB + 2 * AT_SUB + 256);  // [2][128]
  float* mlst = xmax + 256;  // [128][4]: m, l of half 0, l of half 1, unused

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, hf = warp >> 2;
  const int Hq = p.Hq;
  const int qt = blockIdx.x / Hq, j = blockIdx.x % Hq;
  const int b = blockIdx.y, z = blockIdx.z;
  const int splits = gridDim.z;
  const int g = j / (Hq / p.Hkv);
  const int q0 = qt * 128;
  const int r = 32 * quarter + lane;  // this thread's query row within the tile
  const int qp = p.qpos0 + q0 + r;

  // key tiles of this split
  const int TA = (p.nA + AT_KT - 1) / AT_KT, TB = (p.nB + AT_KT - 1) / AT_KT;
  int t_lo = 0, t_hi = TA + TB;
  if (p.causal) {
    // tiles meeting the key positions [q - window + 1, q] of the tile's queries: the
    // cached segment A (positions before segment B) from its first tile in reach, then
    // segment B up to the last query
    const int lo_pos = p.qpos0 + q0 - p.window + 1;
    const int hi_pos = min(p.kposB + p.nB - 1, p.qpos0 + min(q0 + 127, p.nq - 1));
    if (TA > 0 && p.kposA + p.nA - 1 >= lo_pos)
      t_lo = max(0, lo_pos - p.kposA) / AT_KT;
    else
      t_lo = TA + max(0, lo_pos - p.kposB) / AT_KT;
    t_hi = TA + (hi_pos - p.kposB) / AT_KT + 1;
  }
  const int my_lo = t_lo + z * p.tiles_per_split;
  const int my_hi = min(t_hi, my_lo + p.tiles_per_split);
  const int nt = max(0, my_hi - my_lo);

  if (tid == 0) {
    tc::mbar_init(q_full, 1);
    for (int k = 0; k < 2; ++k) {
      tc::mbar_init(kv_full + k, 1);
      tc::mbar_init(s_done + k, 1);
    }
    tc::mbar_init(o_done, 1);
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tslot, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;
  const uint32_t tO = tmem + 256;  // S buffers at columns 0 and 128
  const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;

  int n_loaded = 0;  // tiles requested so far (thread 0): tiles 0 .. n_loaded - 1
  auto load_tile = [&](int i) {  // tile index i within this split -> stage i & 1
    const int t = my_lo + i;
    ++n_loaded;
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
  constexpr uint32_t idesc = tc::idesc_bf16(128, 128);
  // S(i) = Q K_i^T into S buffer i & 1 (thread 0); false on a timeout
  auto issue_s = [&](int i) -> bool {
    if (i == 0 && !tc::mbar_wait(q_full, 0)) return false;
    if (!tc::mbar_wait(kv_full + (i & 1), (i >> 1) & 1)) return false;
    tc::fence_after_sync();
    const uint32_t qa = tc::smem_addr(sQ), ka = tc::smem_addr(sKV + (i & 1) * 4 * AT_SUB);
#pragma unroll
    for (int kb = 0; kb < 2; ++kb)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        tc::mma_bf16(tmem + (i & 1) * 128, tc::sdesc_k128(qa + kb * AT_SUB + k * 32),
                     tc::sdesc_k128(ka + kb * AT_SUB + k * 32), idesc, (kb | k) != 0);
    tc::mma_commit(s_done + (i & 1));
    return true;
  };
  // every warp's lane 0 waits on `bar`; false everywhere if any wait gave up
  auto wait_all = [&](uint64_t* bar_, uint32_t ph) -> bool {
    bool ok_ = true;
    if (lane == 0) ok_ = tc::mbar_wait(bar_, ph);
    ok_ = __shfl_sync(0xffffffffu, ok_ ? 1 : 0, 0) != 0;
    return __syncthreads_and(ok_ ? 1 : 0) != 0;
  };

  // the cached prompt window (segment A) was written before this forward began, so its
  // first tiles are requested before the preceding kernel has finished
  const int n_first = min(nt, 2);
  if (tid == 0)
    for (int i = 0; i < n_first; ++i)
      if (my_lo + i < TA) load_tile(i);
  pdl_enter();  // q and the pass's own keys / values are read only from here on

  bool ok = true;
  if (tid == 0 && nt > 0) {
    tc::mbar_expect_tx(q_full, 2 * AT_SUB);
    const int qrow = b * p.nq + q0;
    tc::tma_load_2d(sQ, &mQ, q_full, j * 128, qrow);
    tc::tma_load_2d(sQ + AT_SUB, &mQ, q_full, j * 128 + 64, qrow);
    for (int i = 0; i < n_first; ++i)
      if (my_lo + i >= TA) load_tile(i);
    if (!issue_s(0)) atomicOr(err, ERR_TIMEOUT);
  }

  float o[64];  // head dims 64 hf .. 64 hf + 63 of this row
#pragma unroll
  for (int d = 0; d < 64; ++d) o[d] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;  // l over this half's keys

  for (int i = 0; i < nt && ok; ++i) {
    const int t = my_lo + i;
    const bool segA = t < TA;
    const int t0 = segA ? t * AT_KT : (t - TA) * AT_KT;
    const int nseg = segA ? p.nA : p.nB;
    const int kpos0 = (segA ? p.kposA : p.kposB) + t0;
    // ---- S of the next tile runs on the tensor cores during this tile's softmax
    if (tid == 0 && i + 1 < nt && !issue_s(i + 1)) atomicOr(err, ERR_TIMEOUT);
    __syncwarp();
    if (!wait_all(s_done + (i & 1), (i >> 1) & 1)) {
      if (tid == 0) atomicOr(err, ERR_TIMEOUT);
      ok = false;
      break;
    }
    tc::fence_after_sync();
    const uint32_t tS = tmem + (i & 1) * 128 + 64 * hf;
    // ---- softmax over this half's 64 keys; the row max is shared with the other half
    float sv[64];
    tc::tmem_ld64(tS + lane_base, sv);
    float mt = -INFINITY;
#pragma unroll
    for (int q = 0; q < 64; ++q) {
      const int kk = t0 + 64 * hf + q;
      const int kp = kpos0 + 64 * hf + q;
      bool valid = kk < nseg;
      if (p.causal) valid = valid && kp <= qp && kp > qp - p.window;
      sv[q] = valid ? sv[q] * p.scale_log2 : -INFINITY;
      mt = fmaxf(mt, sv[q]);
    }
    xmax[hf * 128 + r] = mt;
    __syncthreads();
    mt = fmaxf(xmax[r], xmax[128 + r]);
    const float m_new = fmaxf(m_run, mt);
    const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_run - m_new);
    float lsum = 0.f;
    const int r7 = r & 7;
    uint8_t* prow = sP + hf * AT_SUB + r * 128;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t pk[16];
#pragma unroll
      for (int q = 0; q < 32; q += 2) {
        float e2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float x = sv[c * 32 + q + u];
          e2[u] = x == -INFINITY ? 0.f : exp2f(x - m_new);
          lsum += e2[u];
        }
        __nv_bfloat162 b2 = __floats2bfloat162_rn(e2[0], e2[1]);
        pk[q >> 1] = *reinterpret_cast<uint32_t*>(&b2);
      }
      // keys 32c .. 32c + 31 of this half -> 16-byte chunks 4c .. 4c + 3, swizzled by row
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int chunk = c * 4 + q;
        *reinterpret_cast<uint4*>(prow + ((chunk ^ r7) << 4)) =
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
      const uint32_t pa = tc::smem_addr(sP), va = tc::smem_addr(sKV + (i & 1) * 4 * AT_SUB + 2 * AT_SUB);
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc::mma_bf16(tO, tc::sdesc_k128(pa + kb * AT_SUB + k * 32),
                       tc::sdesc_k128(va + kb * AT_SUB + k * 32), idesc, (kb | k) != 0);
      tc::mma_commit(o_done);
    }
    __syncwarp();
    if (!wait_all(o_done, i & 1)) {
      if (tid == 0) atomicOr(err, ERR_TIMEOUT);
      ok = false;
      break;
    }
    tc::fence_after_sync();
    // stage i & 1 is free again (S(i) and O_t(i) done): prefetch tile i + 2
    if (tid == 0 && i + 2 < nt) load_tile(i + 2);
    {
      float ov[64];
      tc::tmem_ld64(tO + lane_base + 64 * hf, ov);
#pragma unroll
      for (int q = 0; q < 64; ++q) o[q] = o[q] * alpha + ov[q];
    }
    tc::fence_before_sync();
  }

  // ---- merge of the cluster's splits: stage (m, l, O) rows in this CTA's K/V buffers
  // (all loads have landed, all MMAs are done), then the owner of each row sums the
  // splits in rank order and writes the normalised bf16 row.  After a timed-out wait,
  // thread 0 first waits (bounded) for the copies it requested.
  if (tid == 0 && nt > 0 &&
      !(tc::mbar_wait(q_full, 0) && tc::drain_slots(kv_full, 2, n_loaded)))
    atomicOr(err, ERR_TIMEOUT);
  __syncthreads();
  const uint32_t stg = tc::smem_addr(sKV);
  {
    const uint32_t dst = stg + (uint32_t)((r * AT_RS + 64 * hf) * 4);
#pragma unroll
    for (int d = 0; d < 64; d += 4) cl::sts4(dst + d * 4, o[d], o[d + 1], o[d + 2], o[d + 3]);
    const bool have = nt > 0 && ok;
    mlst[r * 4 + 1 + hf] = have ? l_run : 0.f;
    if (hf == 0) mlst[r * 4] = have ? m_run : -INFINITY;
  }
  if (splits > 1) cl::sync();
  else __syncthreads();
  {
    const int R = 128 / splits;  // rows owned by this CTA (splits: 1, 2, 4 or 8)
    const uint32_t mls = tc::smem_addr(mlst);
#pragma unroll 1
    for (int lr = warp; lr < R; lr += AT_THREADS / 32) {
      const int row = z * R + lr;  // row within the tile
      if (q0 + row >= p.nq) break;
      float ms[8], ls[8];
      float4 os[8];
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2) {
        if (s2 < splits) {
          const uint32_t base_ml = (splits > 1 ? cl::map(mls, (uint32_t)s2) : mls) + row * 16;
          const uint32_t base_o = (splits > 1 ? cl::map(stg, (uint32_t)s2) : stg) +
                                  (uint32_t)((row * AT_RS + 4 * lane) * 4);
          if (splits > 1) {
            ms[s2] = cl::ldc(base_ml);
            ls[s2] = cl::ldc(base_ml + 4) + cl::ldc(base_ml + 8);
            os[s2] = cl::ldc4(base_o);
          } else {
            ms[s2] = cl::lds(base_ml);
            ls[s2] = cl::lds(base_ml + 4) + cl::lds(base_ml + 8);
            os[s2] = cl::lds4(base_o);
          }
        }
      }
      float M = -INFINITY;
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        if (s2 < splits) M = fmaxf(M, ms[s2]);
      float L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        if (s2 < splits && ms[s2] > -INFINITY) {
          const float w = exp2f(ms[s2] - M);
          L += w * ls[s2];
          acc.x += w * os[s2].x;
          acc.y += w * os[s2].y;
          acc.z += w * os[s2].z;
          acc.w += w * os[s2].w;
        }
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&lo);
      pk.y = *reinterpret_cast<const uint32_t*>(&hi);
      const size_t tok = (size_t)b * p.nq + q0 + row;
      *reinterpret_cast<uint2*>(p.out + (tok * Hq + j) * 128 + 4 * lane) = pk;
    }
  }
  if (splits > 1) cl::sync();  // peers may still read this CTA's staged rows
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

}  // namespace dg
