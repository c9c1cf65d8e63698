// Grouped routed-expert GEMM with FP8 E4M3 expert weights (one fp32 scale per
// weight row and 128 consecutive input columns) and bf16 activations.
//
// Work unit = token chunk x 128 weight rows, weights on the MMA's M side, tokens on
// N (as in the bf16 routed-expert kernel), gate/up and down as two launches.  Per stage of 64 input columns:
// TMA brings the FP8 weight tile(s) [128 rows x 64 bytes] and the bf16 token rows;
// eight converter warps turn each FP8 tile into the 128-byte-swizzled bf16 tile the
// MMA reads (value = code * scale, rounded to bf16); the MMA warp then issues
// tcgen05.mma as in the bf16 kernel.  Roles (576 threads): warp 0 TMA, warp 1 MMA,
// warps 2..9 epilogue (warps w and w + 4 share a TMEM lane quarter and split the
// token chunks), warps 10..17 converters.
//
// Passage: FP8 serving of the MoE experts — "DiffusionGemma 技术报告" (full
// translation page), §6 (FP8 on H100, MoE memory-bound at batch 1).
#pragma once

#include <cuda_fp8.h>

#include "k_tc_gemm.cuh"

namespace dg {

template <bool GATEUP, int ST>
struct ExpertF8Cfg {
  static constexpr int NW = GATEUP ? 2 : 1;
  static constexpr uint32_t F8_TILE = 128 * 64;           // 8 KB staging per weight
  static constexpr uint32_t B_MAX = 128 * TC_KB * 2;      // token rows
  static constexpr uint32_t STAGE = NW * F8_TILE + NW * TC_SUB_A + B_MAX;
  static constexpr uint32_t TCOLS = GATEUP ? 256 : 128;
  static constexpr size_t SMEM = 1024 + (size_t)ST * STAGE + 512;
};

// bf16 pair from two E4M3 bytes times a scale
__device__ __forceinline__ uint32_t f8x2_scaled(uint32_t two, float sc) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<__half2*>(&h));
  __nv_bfloat162 b = __floats2bfloat162_rn(f.x * sc, f.y * sc);
  return *reinterpret_cast<uint32_t*>(&b);
}

constexpr int TC_F8_THREADS = 576;

template <bool GATEUP, int ST>
__global__ void __launch_bounds__(TC_F8_THREADS, 1)
    tc_expert_f8_kernel(const __grid_constant__ CUtensorMap mW, const __grid_constant__ CUtensorMap mW2,
                        const __grid_constant__ CUtensorMap mX, const float* __restrict__ sW,
                        const float* __restrict__ sW2, const int32_t* __restrict__ chunk_e,
                        const int32_t* __restrict__ chunk_r0, const int32_t* __restrict__ n_chunks,
                        const int32_t* __restrict__ offsets, int w_rows_per_expert, int K, int FT,
                        void* __restrict__ out, int ldo, const float* __restrict__ gate_of,
                        int32_t* err) {
  typedef ExpertF8Cfg<GATEUP, ST> Cfg;
  pdl_enter();  // the routing tables come from the preceding kernels
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * Cfg::STAGE);
  uint64_t* conv = full + ST;     // converted tiles ready (8 converter warps)
  uint64_t* empty = conv + ST;
  uint64_t* tfull = empty + ST;
  uint64_t* tempty = tfull + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(tempty + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_units = *n_chunks * FT;
  const int nk = (K + TC_KB - 1) / TC_KB;
  const int kscale = K / 128;  // scales per weight row

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      tc::mbar_init(full + s, 1);
      tc::mbar_init(conv + s, 8);
      tc::mbar_init(empty + s, 1);
    }
    tc::mbar_init(tfull, 1);
    tc::mbar_init(tempty, 8);
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tslot, Cfg::TCOLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;

  auto unit_rows = [&](int u, int& e, int& r0, int& n, int& f) {
    const int c = u / FT;
    f = u % FT;
    e = chunk_e[c];
    r0 = chunk_r0[c];
    n = min(128, offsets[e + 1] - r0);
  };
  // per-stage buffers: [FP8 staging x NW][bf16 tile x NW][token rows]
  auto f8_at = [&](int s, int w) { return smem + s * Cfg::STAGE + w * Cfg::F8_TILE; };
  auto bf_at = [&](int s, int w) {
    return smem + s * Cfg::STAGE + Cfg::NW * Cfg::F8_TILE + w * TC_SUB_A;
  };
  auto x_at = [&](int s) {
    return smem + s * Cfg::STAGE + Cfg::NW * Cfg::F8_TILE + Cfg::NW * TC_SUB_A;
  };

  if (warp == 0) {
    if (lane == 0) {
      tc::prefetch_tmap(&mW);
      if (GATEUP) tc::prefetch_tmap(&mW2);
      tc::prefetch_tmap(&mX);
      int it = 0;
      for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        int e, r0, n, f;
        unit_rows(u, e, r0, n, f);
        const int nb = (n + 31) >> 5;
        const uint32_t bytes = Cfg::NW * Cfg::F8_TILE + (uint32_t)nb * 32 * TC_KB * 2;
        const int wrow = e * w_rows_per_expert + f * 128;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % ST;
          const uint32_t ph = (it / ST) & 1;
          if (it >= ST && !tc::mbar_wait(empty + s, ph ^ 1)) {
            atomicOr(err, ERR_TIMEOUT);
            u = n_units;
            break;
          }
          const int kx = ((kb + f) % nk) * TC_KB;
          tc::mbar_expect_tx(full + s, bytes);
          tc::tma_load_2d(f8_at(s, 0), &mW, full + s, kx, wrow);
          if (GATEUP) tc::tma_load_2d(f8_at(s, 1), &mW2, full + s, kx, wrow);
          for (int j = 0; j < nb; ++j)
            tc::tma_load_2d(x_at(s) + j * 32 * TC_KB * 2, &mX, full + s, kx, r0 + 32 * j);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0, ui = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ui) {
        int e, r0, n, f;
        unit_rows(u, e, r0, n, f);
        const int npad = ((n + 31) >> 5) << 5;
        const uint32_t idesc = tc::idesc_bf16(128, npad);
        if (ui > 0 && !tc::mbar_wait(tempty, (ui - 1) & 1)) {
          atomicOr(err, ERR_TIMEOUT);
          break;
        }
        tc::fence_after_sync();
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % ST;
          const uint32_t ph = (it / ST) & 1;
          if (!tc::mbar_wait(conv + s, ph)) {
            atomicOr(err, ERR_TIMEOUT);
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t a0 = tc::smem_addr(bf_at(s, 0));
          const uint32_t b0 = tc::smem_addr(x_at(s));
#pragma unroll
          for (int k = 0; k < TC_KB / 16; ++k) {
            const uint32_t acc = (kb | k) != 0;
            const uint64_t bd = tc::sdesc_k128(b0 + k * 32);
            tc::mma_bf16(tmem, tc::sdesc_k128(a0 + k * 32), bd, idesc, acc);
            if (GATEUP) tc::mma_bf16(tmem + 128, tc::sdesc_k128(a0 + TC_SUB_A + k * 32), bd, idesc, acc);
          }
          tc::mma_commit(empty + s);
        }
        if (ok) tc::mma_commit(tfull);
      }
    }
  } else if (warp >= 10) {
    // converters: thread t handles 16-byte chunk (t % 4) of FP8 rows (t / 4) + 64 i
    const int t = threadIdx.x - 320;  // 0..255
    const int chunk = t & 3;
    int it = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
      int e, r0, n, f;
      unit_rows(u, e, r0, n, f);
      const int wrow = e * w_rows_per_expert + f * 128;
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % ST;
        const uint32_t ph = (it / ST) & 1;
        const int kx = ((kb + f) % nk) * TC_KB;
        // the scales do not depend on the staged tile: request them before waiting
        float scl[Cfg::NW][2];
#pragma unroll
        for (int w = 0; w < Cfg::NW; ++w)
#pragma unroll
          for (int i = 0; i < 2; ++i)
            scl[w][i] = (w == 0 ? sW : sW2)[(size_t)(wrow + (t >> 2) + 64 * i) * kscale + kx / 128];
        bool ready = true;
        if (lane == 0) ready = tc::mbar_wait(full + s, ph);
        ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
        if (!ready) {
          if (lane == 0) atomicOr(err, ERR_TIMEOUT);
          ok = false;
          break;
        }
#pragma unroll
        for (int w = 0; w < Cfg::NW; ++w) {
          const uint8_t* src = f8_at(s, w);
          uint8_t* dst = bf_at(s, w);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int r = (t >> 2) + 64 * i;
            const float scale = scl[w][i];
            const uint4 q = *reinterpret_cast<const uint4*>(src + r * 64 + chunk * 16);
            const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              o[2 * j] = f8x2_scaled(qw[j] & 0xffffu, scale);
              o[2 * j + 1] = f8x2_scaled(qw[j] >> 16, scale);
            }
            // 16 bf16 values = two 16-byte chunks (2 chunk, 2 chunk + 1) of row r
            uint8_t* rowp = dst + r * 128;
            const int c0 = (2 * chunk) ^ (r & 7), c1 = (2 * chunk + 1) ^ (r & 7);
            *reinterpret_cast<uint4*>(rowp + c0 * 16) = make_uint4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<uint4*>(rowp + c1 * 16) = make_uint4(o[4], o[5], o[6], o[7]);
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0)
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_addr(conv + s))
                       : "memory");
      }
      if (!ok) break;
    }
  } else {
    // epilogue warps 2..9 -> TMEM lane quarter (warp % 4), token chunks of parity hf
    const int q = warp & 3, hf = (warp - 2) >> 2;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    int ui = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++ui) {
      int e, r0, n, f;
      unit_rows(u, e, r0, n, f);
      bool ready = true;
      if (lane == 0) ready = tc::mbar_wait(tfull, ui & 1);
      ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
      if (!ready) {
        if (lane == 0) atomicOr(err, ERR_TIMEOUT);
        break;
      }
      tc::fence_after_sync();
      const int fr = f * 128 + 32 * q + lane;
      const int nch = (n + 31) >> 5;
#pragma unroll 1
      for (int c = hf; c < nch; c += 2) {
        float v[32];
        tc::tmem_ld32(tmem + lane_base + c * 32, v);
        if (GATEUP) {
          float g2[32];
          tc::tmem_ld32(tmem + lane_base + 128 + c * 32, g2);
          bf16* o = reinterpret_cast<bf16*>(out);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tt = c * 32 + j;
            if (tt < n) o[(size_t)(r0 + tt) * ldo + fr] = __float2bfloat16_rn(silu(v[j]) * g2[j]);
          }
        } else {
          float* o = reinterpret_cast<float*>(out);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tt = c * 32 + j;
            if (tt < n) o[(size_t)(r0 + tt) * ldo + fr] = gate_of[r0 + tt] * v[j];
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0)
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_addr(tempty))
                     : "memory");
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, Cfg::TCOLS);
}

}  // namespace dg
