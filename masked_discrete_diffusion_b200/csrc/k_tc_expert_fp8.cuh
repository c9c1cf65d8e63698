// Routed experts with FP8 E4M3 expert weights (one fp32 scale per weight row and 128
// consecutive input columns), or NVFP4 expert weights (E2M1 codes two per byte, one
// E4M3 scale per weight row and 16 consecutive input columns, one fp32 power-of-two
// scale per tensor), and bf16 activations: gate/up SwiGLU and down in one persistent
// launch, with the schedule and device-side chunk counters of the bf16 routed-expert
// kernel (tc_moe_kernel).
//
// Weights sit on the MMA's M side, tokens on N.  Per stage of 64 input columns TMA
// brings two FP8 weight tiles [128 rows x 64 bytes] and the bf16 token rows; eight
// converter warps turn each FP8 tile into the 128-byte-swizzled bf16 tile the MMA
// reads (value = code * scale, rounded to bf16); the MMA warp then issues tcgen05.mma.
// A unit's scales are staged in shared memory once per unit.  NVFP4: TMA brings two
// tiles [128 rows x 32 bytes] of packed codes and the converters write value =
// e2m1(code) * (block scale * tensor scale), exact in fp32, rounded to bf16.
//
// Passages: FP8 serving of the MoE experts — "DiffusionGemma 技术报告" (full
// translation page), §6 (FP8 on H100, MoE memory-bound at batch 1); NVFP4 — the
// agentlenshq page on DiffusionGemma (NVFP4 kernels for Hopper and Blackwell).  The
// block-scaled tensor-core MMA is not used: the codes are widened to bf16 in shared
// memory and the MMA is the bf16 one of the other expert kernels.
#pragma once

#include <cuda_fp8.h>

#include "k_tc_gemm.cuh"

namespace dg {

// bf16 pair from two E4M3 bytes times a scale
__device__ __forceinline__ uint32_t f8x2_scaled(uint32_t two, float sc) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<__half2*>(&h));
  __nv_bfloat162 b = __floats2bfloat162_rn(f.x * sc, f.y * sc);
  return *reinterpret_cast<uint32_t*>(&b);
}

constexpr int TC_F8_THREADS = 576;

// NVFP4 scales of one layer: E4M3 block scales [rows, K / 16] and fp32 tensor scales [1]
struct F4Scales {
  const uint8_t *g = nullptr, *u = nullptr, *d = nullptr;
  const float *tg = nullptr, *tu = nullptr, *td = nullptr;
};

// value of a 4-bit E2M1 code: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 for codes 0..7 (in
// half units 0, 1, 2, 3, 4, 6, 8, 12, one nibble each of 0xC8643210), bit 3 the sign
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const float mag = (float)((0xC8643210u >> (4 * (c & 7u))) & 0xFu) * 0.5f;
  return (c & 8u) ? -mag : mag;
}

__device__ __forceinline__ float e4m3_value(uint8_t b) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3);
  return __half2float(*reinterpret_cast<__half*>(&h));
}

// ---------------------------------------------------------------------------
// Both phases of the routed experts with FP8 weights in one persistent launch (the
// schedule and the device-side chunk counters of tc_moe_kernel).  Per stage: TMA
// brings two FP8 weight tiles [128 rows x 64 bytes] and the bf16 token rows; the
// eight converter warps write the two bf16 tiles; the MMA warp issues two MMAs.
//   phase 1, unit u = c * FT1 + f: gate rows and up rows f*128 .. +127 (K = d);
//   phase 2, unit v = c * FT2 + f: down rows f*256 .. +127 and +128 .. +255 (K = I).
// Roles (576 threads): warp 0 TMA, warp 1 MMA, warps 2..9 epilogue, warps 10..17
// converters.
// ---------------------------------------------------------------------------
template <int ST, bool FP4>
struct MoeLowpCfg {
  static constexpr uint32_t F8_TILE = FP4 ? 128 * 32 : 128 * 64;  // weight bytes per tile
  static constexpr uint32_t B_MAX = 128 * TC_KB * 2;
  static constexpr uint32_t STAGE = 2 * F8_TILE + 2 * TC_SUB_A + B_MAX;
  static_assert(STAGE % 1024 == 0 && (2 * F8_TILE) % 1024 == 0, "swizzled tiles 1024-aligned");
  static constexpr uint32_t TCOLS = 256;
  static constexpr size_t SMEM = 1024 + (size_t)ST * STAGE + 512;  // + the unit's scales
  // a unit's scales: 256 weight rows (gate then up, or the two down tiles) x K / 128
  // fp32 (FP8) or x K / 16 E4M3 bytes (NVFP4), then (NVFP4) the 256-entry table of a
  // byte's two E2M1 values as a bf16 pair
  static size_t smem_bytes(int d, int I) {
    const size_t K = d > I ? d : I;
    return SMEM + (FP4 ? 16 * K + 1024 : 8 * K);
  }
};
template <int ST> using MoeF8Cfg = MoeLowpCfg<ST, false>;

template <int ST, bool FP4>
__device__ __forceinline__ void moe_lowp_body(
    const CUtensorMap& mWg, const CUtensorMap& mWu, const CUtensorMap& mX,
    const CUtensorMap& mWd, const CUtensorMap& mH, const float* __restrict__ sWg,
    const float* __restrict__ sWu, const float* __restrict__ sWd, const F4Scales& f4,
    const int32_t* __restrict__ chunk_e, const int32_t* __restrict__ chunk_r0,
    const int32_t* __restrict__ n_chunks, const int32_t* __restrict__ offsets, int I, int d,
    bf16* __restrict__ hb, float* __restrict__ yb, const float* __restrict__ gate_of,
    int32_t* __restrict__ ready, int32_t* __restrict__ next, int32_t* err) {
  typedef MoeLowpCfg<ST, FP4> Cfg;
  pdl_enter();  // the routing tables come from the preceding kernels
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * Cfg::STAGE);
  uint64_t* conv = full + ST;     // converted tiles ready (8 converter warps)
  uint64_t* empty = conv + ST;
  uint64_t* tfull = empty + ST;
  uint64_t* tempty = tfull + 1;   // 8 epilogue arrivals
  // units taken by the TMA thread, in order, for the MMA thread, the epilogue leader and
  // the converter leader (the schedule of tc_moe_kernel)
  constexpr int QD = 4;
  uint64_t* qfull = tempty + 1;   // [QD] unit id written (TMA thread)
  uint64_t* qempty = qfull + QD;  // [QD] unit id read (three readers)
  int32_t* qid = reinterpret_cast<int32_t*>(qempty + QD);  // [QD]
  int32_t* ubc = qid + QD;        // the epilogue leader's broadcast of the unit id
  int32_t* cbc = ubc + 1;         // the converter leader's broadcast
  uint32_t* tslot = reinterpret_cast<uint32_t*>(cbc + 1);
  float* sscl = reinterpret_cast<float*>(smem + ST * Cfg::STAGE + 512);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nc = *n_chunks;
  const int FT1 = I / 128, FT2 = d / 256;
  const int U1 = nc * FT1, n_units = U1 + nc * FT2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      tc::mbar_init(full + s, 1);
      tc::mbar_init(conv + s, 8);
      tc::mbar_init(empty + s, 1);
    }
    tc::mbar_init(tfull, 1);
    tc::mbar_init(tempty, 8);
    for (int k = 0; k < QD; ++k) {
      tc::mbar_init(qfull + k, 1);
      tc::mbar_init(qempty + k, 3);
    }
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tslot, Cfg::TCOLS);
  // NVFP4: byte b -> (e2m1(b & 15), e2m1(b >> 4)) as bf16, exact (at most 2 significant bits)
  uint32_t* f4tab = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(sscl) +
                                                16 * (size_t)(d > I ? d : I));
  if (FP4 && threadIdx.x < 256) {
    __nv_bfloat162 v2 = __floats2bfloat162_rn(e2m1_value(threadIdx.x & 15u),
                                              e2m1_value(threadIdx.x >> 4));
    f4tab[threadIdx.x] = *reinterpret_cast<uint32_t*>(&v2);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;

  struct Unit {
    bool down;
    int c, e, r0, n, f, w1, nk;
  };
  auto unit_of = [&](int u) {
    Unit x;
    x.down = u >= U1;
    const int v = x.down ? u - U1 : u, ft = x.down ? FT2 : FT1;
    x.c = v / ft;
    x.f = v % ft;
    x.e = chunk_e[x.c];
    x.r0 = chunk_r0[x.c];
    x.n = min(128, offsets[x.e + 1] - x.r0);
    x.w1 = x.down ? x.e * d + x.f * 256 : x.e * I + x.f * 128;  // first weight row of tile 0
    x.nk = (x.down ? I : d) / TC_KB;
    return x;
  };
  // the ui-th unit id of this block (n_units when there is none, or on a timeout)
  auto take = [&](int ui) -> int {
    const int k = ui % QD;
    if (!tc::mbar_wait(qfull + k, (ui / QD) & 1)) {
      atomicOr(err, ERR_TIMEOUT);
      return n_units;
    }
    const int u = *reinterpret_cast<volatile int32_t*>(qid + k);
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_addr(qempty + k))
                 : "memory");
    return u;
  };
  auto f8_at = [&](int s, int w) { return smem + s * Cfg::STAGE + w * Cfg::F8_TILE; };
  auto bf_at = [&](int s, int w) { return smem + s * Cfg::STAGE + 2 * Cfg::F8_TILE + w * TC_SUB_A; };
  auto x_at = [&](int s) { return smem + s * Cfg::STAGE + 2 * Cfg::F8_TILE + 2 * TC_SUB_A; };

  if (warp == 0) {
    if (lane == 0) {
      tc::prefetch_tmap(&mWg);
      tc::prefetch_tmap(&mWu);
      tc::prefetch_tmap(&mX);
      tc::prefetch_tmap(&mWd);
      tc::prefetch_tmap(&mH);
      int it = 0;
      bool ok = true;
      for (int qi = 0;; ++qi) {
        // blocks take the next unit when they are ready for it (gate/up units first,
        // so a down unit only ever waits for units that running blocks have taken)
        const int k = qi % QD;
        if (qi >= QD && !tc::mbar_wait(qempty + k, ((qi / QD) & 1) ^ 1)) {
          atomicOr(err, ERR_TIMEOUT);
          break;  // the readers give up on their own bounded waits
        }
        const int u = ok ? atomicAdd(next, 1) : n_units;
        qid[k] = u < n_units ? u : n_units;
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_addr(qfull + k))
                     : "memory");
        if (u >= n_units) break;
        const Unit x = unit_of(u);
        if (x.down) {
          const uint64_t t0 = tc::global_ns();
          while (ld_acquire(ready + x.c) < FT1) {
            __nanosleep(64);
            if (tc::global_ns() - t0 > 2000000000ull) {
              atomicOr(err, ERR_TIMEOUT);
              ok = false;
              break;
            }
          }
          if (!ok) continue;  // publish the end of the work next
          asm volatile("fence.proxy.async.global;" ::: "memory");  // before the TMA reads
        }
        const int nb = (x.n + 31) >> 5;
        const uint32_t bytes = 2 * Cfg::F8_TILE + (uint32_t)nb * 32 * TC_KB * 2;
        for (int kb = 0; kb < x.nk; ++kb, ++it) {
          const int s = it % ST;
          const uint32_t ph = (it / ST) & 1;
          if (it >= ST && !tc::mbar_wait(empty + s, ph ^ 1)) {
            atomicOr(err, ERR_TIMEOUT);
            ok = false;
            break;
          }
          const int kx = ((kb + x.f) % x.nk) * TC_KB;
          const int kw = FP4 ? kx / 2 : kx;  // byte column of the weight tiles
          tc::mbar_expect_tx(full + s, bytes);
          if (x.down) {
            tc::tma_load_2d(f8_at(s, 0), &mWd, full + s, kw, x.w1);
            tc::tma_load_2d(f8_at(s, 1), &mWd, full + s, kw, x.w1 + 128);
          } else {
            tc::tma_load_2d(f8_at(s, 0), &mWg, full + s, kw, x.w1);
            tc::tma_load_2d(f8_at(s, 1), &mWu, full + s, kw, x.w1);
          }
          for (int j = 0; j < nb; ++j)
            tc::tma_load_2d(x_at(s) + j * 32 * TC_KB * 2, x.down ? &mH : &mX, full + s, kx,
                            x.r0 + 32 * j);
        }
      }
      if (!tc::drain_slots(full, ST, it)) atomicOr(err, ERR_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int ui = 0; ok; ++ui) {
        const int u = take(ui);
        if (u >= n_units) break;
        const Unit x = unit_of(u);
        const int npad = ((x.n + 31) >> 5) << 5;
        const uint32_t idesc = tc::idesc_bf16(128, npad);
        if (ui > 0 && !tc::mbar_wait(tempty, (ui - 1) & 1)) {
          atomicOr(err, ERR_TIMEOUT);
          break;
        }
        tc::fence_after_sync();
        for (int kb = 0; kb < x.nk; ++kb, ++it) {
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
            tc::mma_bf16(tmem + 128, tc::sdesc_k128(a0 + TC_SUB_A + k * 32), bd, idesc, acc);
          }
          tc::mma_commit(empty + s);
        }
        if (ok) tc::mma_commit(tfull);
      }
    }
  } else if (warp >= 10) {
    // converters: thread t handles 16-byte chunk (t % 4) of FP8 rows (t / 4) + 64 i.
    // A unit's scales (256 rows x K/128) are brought into shared memory once; after a
    // timed-out wait the warp skips the waits but keeps step with the other converters.
    const int t = threadIdx.x - 320;  // 0..255
    const int chunk = t & 3;
    int it = 0;
    bool dead = false;
    uint8_t* sscl8 = reinterpret_cast<uint8_t*>(sscl);
    for (int ui = 0;; ++ui) {
      // warp 10 takes the unit id for the eight converter warps; the barrier also keeps
      // the previous unit's scales until every converter has read them
      if (warp == 10 && lane == 0) *reinterpret_cast<volatile int32_t*>(cbc) = take(ui);
      asm volatile("bar.sync 2, 256;" ::: "memory");
      const int u = *reinterpret_cast<volatile int32_t*>(cbc);
      if (u >= n_units) break;
      const Unit x = unit_of(u);
      const int kscale = (x.down ? I : d) / (FP4 ? 16 : 128);
      const int half = 128 * kscale;
      float tsc[2] = {1.f, 1.f};
      if constexpr (FP4) {
        // E4M3 bytes: gate rows then up rows, or the 256 down rows (16 bytes at a time)
        for (int i = 16 * t; i < 2 * half; i += 4096) {
          const uint8_t* src = x.down ? f4.d + (size_t)x.w1 * kscale + i
                               : i < half ? f4.g + (size_t)x.w1 * kscale + i
                                          : f4.u + (size_t)x.w1 * kscale + (i - half);
          *reinterpret_cast<uint4*>(sscl8 + i) = __ldg(reinterpret_cast<const uint4*>(src));
        }
        tsc[0] = x.down ? __ldg(f4.td) : __ldg(f4.tg);
        tsc[1] = x.down ? __ldg(f4.td) : __ldg(f4.tu);
      } else {
        for (int i = 4 * t; i < 2 * half; i += 1024) {
          const float* src = x.down ? sWd + (size_t)x.w1 * kscale + i
                             : i < half ? sWg + (size_t)x.w1 * kscale + i
                                        : sWu + (size_t)x.w1 * kscale + (i - half);
          *reinterpret_cast<float4*>(sscl + i) = __ldg(reinterpret_cast<const float4*>(src));
        }
      }
      asm volatile("bar.sync 2, 256;" ::: "memory");
      for (int kb = 0; kb < x.nk; ++kb, ++it) {
        const int s = it % ST;
        const uint32_t ph = (it / ST) & 1;
        const int kx = ((kb + x.f) % x.nk) * TC_KB;
        if (!dead) {
          bool rdy = true;
          if (lane == 0) rdy = tc::mbar_wait(full + s, ph);
          rdy = __shfl_sync(0xffffffffu, rdy ? 1 : 0, 0) != 0;
          if (!rdy) {
            if (lane == 0) atomicOr(err, ERR_TIMEOUT);
            dead = true;
          }
        }
        if (!dead && FP4) {
          // thread t (0..255) converts, in tile w = 0 and 1, row t / 2 and 16-byte chunk
          // t % 2 of the row's 32 bytes (64 codes): codes 32 ch .. 32 ch + 31, scale
          // blocks (kx + 32 ch) / 16 and the next
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const int r = t >> 1, ch = t & 1;
            const uint4 q = *reinterpret_cast<const uint4*>(f8_at(s, w) + r * 32 + ch * 16);
            const uint8_t* srow = sscl8 + (size_t)(128 * w + r) * kscale + ((kx + 32 * ch) >> 4);
            // block scale * tensor scale: at most 4 significant bits times a power of
            // two, exact in bf16, so the bf16 products below are exact
            const __nv_bfloat162 sc2[2] = {
                __float2bfloat162_rn(e4m3_value(srow[0]) * tsc[w]),
                __float2bfloat162_rn(e4m3_value(srow[1]) * tsc[w])};
            const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
            uint32_t o[16];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint32_t t2 = f4tab[(qw[b] >> (8 * i)) & 0xffu];
                __nv_bfloat162 v2 = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&t2),
                                            sc2[b >> 1]);
                o[4 * b + i] = *reinterpret_cast<uint32_t*>(&v2);
              }
            }
            uint8_t* rowp = bf_at(s, w) + r * 128;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              *reinterpret_cast<uint4*>(rowp + (((4 * ch + k) ^ (r & 7)) << 4)) =
                  make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
          }
        }
        if (!dead && !FP4) {
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const uint8_t* src = f8_at(s, w);
            uint8_t* dst = bf_at(s, w);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int r = (t >> 2) + 64 * i;
              const float scale = sscl[(128 * w + r) * kscale + kx / 128];
              const uint4 q = *reinterpret_cast<const uint4*>(src + r * 64 + chunk * 16);
              const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
              uint32_t o[8];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                o[2 * j] = f8x2_scaled(qw[j] & 0xffffu, scale);
                o[2 * j + 1] = f8x2_scaled(qw[j] >> 16, scale);
              }
              uint8_t* rowp = dst + r * 128;
              const int c0 = (2 * chunk) ^ (r & 7), c1 = (2 * chunk + 1) ^ (r & 7);
              *reinterpret_cast<uint4*>(rowp + c0 * 16) = make_uint4(o[0], o[1], o[2], o[3]);
              *reinterpret_cast<uint4*>(rowp + c1 * 16) = make_uint4(o[4], o[5], o[6], o[7]);
            }
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0)
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_addr(conv + s))
                       : "memory");
      }
    }
  } else {
    // epilogue warps 2..9 -> TMEM lane quarter (warp % 4), token chunks of parity hf
    const int q = warp & 3, hf = (warp - 2) >> 2;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    for (int ui = 0;; ++ui) {
      // warp 2 takes the unit id for the eight epilogue warps
      if (warp == 2 && lane == 0) *reinterpret_cast<volatile int32_t*>(ubc) = take(ui);
      asm volatile("bar.sync 1, 256;" ::: "memory");
      const int u = *reinterpret_cast<volatile int32_t*>(ubc);
      asm volatile("bar.sync 1, 256;" ::: "memory");  // read by all before the next take
      if (u >= n_units) break;
      const Unit x = unit_of(u);
      bool rdy = true;
      if (lane == 0) rdy = tc::mbar_wait(tfull, ui & 1);
      rdy = __shfl_sync(0xffffffffu, rdy ? 1 : 0, 0) != 0;
      // on a timeout the warp records it and keeps step with the other epilogue warps
      if (!rdy && lane == 0) atomicOr(err, ERR_TIMEOUT);
      tc::fence_after_sync();
      const int nch = rdy ? (x.n + 31) >> 5 : 0;
      if (!x.down) {
        const int fr = x.f * 128 + 32 * q + lane;
#pragma unroll 1
        for (int c = hf; c < nch; c += 2) {
          float g[32], v[32];
          tc::tmem_ld32(tmem + lane_base + c * 32, g);
          tc::tmem_ld32(tmem + lane_base + 128 + c * 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tt = c * 32 + j;
            if (tt < x.n) hb[(size_t)(x.r0 + tt) * I + fr] = __float2bfloat16_rn(silu(g[j]) * v[j]);
          }
        }
      } else {
#pragma unroll 1
        for (int half2 = 0; half2 < 2; ++half2) {
          const int fr = x.f * 256 + half2 * 128 + 32 * q + lane;
#pragma unroll 1
          for (int c = hf; c < nch; c += 2) {
            float v[32];
            tc::tmem_ld32(tmem + lane_base + half2 * 128 + c * 32, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int tt = c * 32 + j;
              if (tt < x.n) yb[(size_t)(x.r0 + tt) * d + fr] = gate_of[x.r0 + tt] * v[j];
            }
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_addr(tempty)) : "memory");
      if (!x.down) {
        __threadfence();
        asm volatile("bar.sync 1, 256;" ::: "memory");  // the eight epilogue warps
        if (warp == 2 && lane == 0) atomicAdd(ready + x.c, 1);
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, Cfg::TCOLS);
}

template <int ST>
__global__ void __launch_bounds__(TC_F8_THREADS, 1)
    tc_moe_f8_kernel(const __grid_constant__ CUtensorMap mWg, const __grid_constant__ CUtensorMap mWu,
                     const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mWd,
                     const __grid_constant__ CUtensorMap mH, const float* __restrict__ sWg,
                     const float* __restrict__ sWu, const float* __restrict__ sWd,
                     const int32_t* __restrict__ chunk_e, const int32_t* __restrict__ chunk_r0,
                     const int32_t* __restrict__ n_chunks, const int32_t* __restrict__ offsets,
                     int I, int d, bf16* __restrict__ hb, float* __restrict__ yb,
                     const float* __restrict__ gate_of, int32_t* __restrict__ ready,
                     int32_t* __restrict__ next, int32_t* err) {
  moe_lowp_body<ST, false>(mWg, mWu, mX, mWd, mH, sWg, sWu, sWd, F4Scales{}, chunk_e, chunk_r0,
                           n_chunks, offsets, I, d, hb, yb, gate_of, ready, next, err);
}

template <int ST>
__global__ void __launch_bounds__(TC_F8_THREADS, 1)
    tc_moe_f4_kernel(const __grid_constant__ CUtensorMap mWg, const __grid_constant__ CUtensorMap mWu,
                     const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mWd,
                     const __grid_constant__ CUtensorMap mH, const F4Scales f4,
                     const int32_t* __restrict__ chunk_e, const int32_t* __restrict__ chunk_r0,
                     const int32_t* __restrict__ n_chunks, const int32_t* __restrict__ offsets,
                     int I, int d, bf16* __restrict__ hb, float* __restrict__ yb,
                     const float* __restrict__ gate_of, int32_t* __restrict__ ready,
                     int32_t* __restrict__ next, int32_t* err) {
  moe_lowp_body<ST, true>(mWg, mWu, mX, mWd, mH, nullptr, nullptr, nullptr, f4, chunk_e,
                          chunk_r0, n_chunks, offsets, I, d, hb, yb, gate_of, ready, next, err);
}

}  // namespace dg
