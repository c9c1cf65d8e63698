// tcgen05 (5th-generation tensor core) kernels for the bf16 dense contractions:
//   * tc_dense_kernel  — D[M, N] = A[M, K] W[N, K]^T, activations as the MMA
//     A operand (128-row sub-tiles, up to MT per CTA so each weight tile is read
//     from HBM once), weights as the B operand; fused epilogues: fp32 store,
//     residual add, SwiGLU (two weight operands), and the LM-head per-row
//     softmax statistics (the logits never leave the SM).
//   * tc_expert_kernel — grouped routed-expert GEMM, weights as the MMA A operand
//     (128 weight rows per tile) and the expert's gathered token rows as the B
//     operand (N = tokens rounded up to 32, <= 128), persistent over work units
//     (token chunk, weight-row tile); SwiGLU or gate-weighted epilogue.
// Operands are staged by TMA (no multicast) into 128-byte-swizzled K-major
// tiles; accumulators live in TMEM and are read back with tcgen05.ld.
//
// Passages: routed MoE with top-8 of 128 experts plus a shared expert and the
// 262K-vocabulary LM head — explainer page "DiffusionGemma 深度解析", list
// "核心架构参数"; logits per canvas position and the entropy-ordered sampler —
// "DiffusionGemma 技术报告" (full translation page), §3.2 and §3.3.
#pragma once

#include <unordered_map>

#include "dg_internal.h"
#include "k_common.cuh"
#include "tc_ptx.cuh"

namespace dg {

constexpr int TC_KB = 64;                 // K elements per stage (one 128-byte swizzle row)
constexpr uint32_t TC_SUB_A = 128 * 64 * 2;  // one 128-row operand sub-tile (16 KB)

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int COLS> struct TmemCols {
  static constexpr uint32_t value =
      COLS <= 32 ? 32 : COLS <= 64 ? 64 : COLS <= 128 ? 128 : COLS <= 256 ? 256 : 512;
};

// ---------------------------------------------------------------------------
// epilogues of the dense kernel: run(row, valid, n0, ld) with ld(acc, chunk, v)
// loading 32 fp32 columns of accumulator `acc` (0, or 1 for the second weight).
// ---------------------------------------------------------------------------
// Chunk epilogues: chunk(row, col, v, u) consumes 32 consecutive columns of one row
// (v: the accumulator, u: the second weight's accumulator for dual GEMMs).
template <class Derived, bool DUAL>
struct EpiChunked {
  static constexpr bool kChunked = true, kRowWise = false;
  template <int NCH, class Ld>
  __device__ void run(int row, bool valid, int n0, Ld&& ld) const {
#pragma unroll 1
    for (int c = 0; c < NCH; ++c) {
      float v[32], u[32];
      ld(0, c, v);
      if (DUAL) ld(1, c, u);
      static_cast<const Derived*>(this)->chunk(row, valid, n0 + c * 32, v, u);
    }
  }
};

struct EpiStoreF32 : EpiChunked<EpiStoreF32, false> {
  float* out;
  int ldo, N;
  EpiStoreF32(float* o, int l, int n) : out(o), ldo(l), N(n) {}
  __device__ void chunk(int row, bool valid, int col, const float* v, const float*) const {
    if (!valid || col >= N) return;
    float4* p = reinterpret_cast<float4*>(out + (size_t)row * ldo + col);
#pragma unroll
    for (int j = 0; j < 8; ++j) p[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  }
};

struct EpiAddF32 : EpiChunked<EpiAddF32, false> {
  float* out;
  int ldo, N;
  EpiAddF32(float* o, int l, int n) : out(o), ldo(l), N(n) {}
  __device__ void chunk(int row, bool valid, int col, const float* v, const float*) const {
    if (!valid || col >= N) return;
    float4* p = reinterpret_cast<float4*>(out + (size_t)row * ldo + col);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float4 o = p[j];
      o.x += v[4 * j];
      o.y += v[4 * j + 1];
      o.z += v[4 * j + 2];
      o.w += v[4 * j + 3];
      p[j] = o;
    }
  }
};

struct EpiSwigluBf16 : EpiChunked<EpiSwigluBf16, true> {
  bf16* out;
  int ldo, N;
  EpiSwigluBf16(bf16* o, int l, int n) : out(o), ldo(l), N(n) {}
  __device__ void chunk(int row, bool valid, int col, const float* g, const float* u) const {
    if (!valid || col >= N) return;
    uint4* p = reinterpret_cast<uint4*>(out + (size_t)row * ldo + col);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = 8 * j + 2 * q;
        __nv_bfloat162 b2 = __floats2bfloat162_rn(silu(g[i]) * u[i], silu(g[i + 1]) * u[i + 1]);
        w[q] = *reinterpret_cast<uint32_t*>(&b2);
      }
      p[j] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
};

// QKV projection epilogue (N-tile = one head of h = 128): rotate query and key
// heads (pairs (j, j + 64) by pos * theta_j, cos/sin from the table
// rope[pos, 64] / rope[max_pos + pos, 64]) and scatter: q -> q[row, head, :],
// k -> kc[b, g, i, :], v -> vc[b, g, :, i] (transposed); all bf16.  Row = b * n_seq + i
// sits at position pos0 + i.
struct EpiQkvRope {
  static constexpr bool kChunked = false, kRowWise = true;
  bf16 *q, *kc, *vc;
  const float* rope;
  int max_pos, n_seq, np, pos0, Hq, Hkv;
  template <int NCH, class Ld>
  __device__ void run(int row, bool valid, int n0, Ld&& ld) const {
    static_assert(NCH == 4, "one head of 128 per tile");
    const int head = n0 / 128;
    const int b = valid ? row / n_seq : 0, i = valid ? row % n_seq : 0, pos = pos0 + i;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      float lo[32], hi[32];
      ld(0, c, lo);
      ld(0, c + 2, hi);
      if (!valid) continue;
      if (head < Hq + Hkv) {
        const float* cs = rope + (size_t)pos * 64 + c * 32;
        const float* sn = rope + ((size_t)max_pos + pos) * 64 + c * 32;
        bf16* dst = head < Hq ? q + ((size_t)row * Hq + head) * 128
                              : kc + (((size_t)b * Hkv + (head - Hq)) * np + i) * 128;
        uint32_t w1[16], w2[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float c0 = cs[j], s0 = sn[j], c1 = cs[j + 1], s1 = sn[j + 1];
          __nv_bfloat162 a = __floats2bfloat162_rn(lo[j] * c0 - hi[j] * s0, lo[j + 1] * c1 - hi[j + 1] * s1);
          __nv_bfloat162 bb = __floats2bfloat162_rn(hi[j] * c0 + lo[j] * s0, hi[j + 1] * c1 + lo[j + 1] * s1);
          w1[j >> 1] = *reinterpret_cast<uint32_t*>(&a);
          w2[j >> 1] = *reinterpret_cast<uint32_t*>(&bb);
        }
        uint4* d1 = reinterpret_cast<uint4*>(dst + c * 32);
        uint4* d2 = reinterpret_cast<uint4*>(dst + 64 + c * 32);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          d1[j] = make_uint4(w1[4 * j], w1[4 * j + 1], w1[4 * j + 2], w1[4 * j + 3]);
          d2[j] = make_uint4(w2[4 * j], w2[4 * j + 1], w2[4 * j + 2], w2[4 * j + 3]);
        }
      } else {
        const int g = head - Hq - Hkv;
        bf16* vt = vc + ((size_t)b * Hkv + g) * 128 * np + i;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          vt[(size_t)(c * 32 + j) * np] = __float2bfloat16_rn(lo[j]);
          vt[(size_t)(64 + c * 32 + j) * np] = __float2bfloat16_rn(hi[j]);
        }
      }
    }
  }
};

// Per-row statistics of logits l = scale * acc over this CTA's vocabulary tile
// (columns n0 .. n0 + 32 NCH - 1, those < N): m = max, s = sum exp(l - m),
// u = sum exp(l - m) (l - m), a = lowest id attaining m.  part[(tile, row)] = (m, s, u, a).
struct EpiLmStats {
  static constexpr bool kChunked = false, kRowWise = false;
  float* part;
  int M, N;
  float scale;
  template <int NCH, class Ld>
  __device__ void run(int row, bool valid, int n0, Ld&& ld) const {
    float mx = -INFINITY;
    int am = 0x7fffffff;
#pragma unroll 1
    for (int c = 0; c < NCH; ++c) {
      float v[32];
      ld(0, c, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int col = n0 + c * 32 + j;
        const float l = scale * v[j];
        if (col < N && l > mx) {
          mx = l;
          am = col;
        }
      }
    }
    float s = 0.f, u = 0.f;
#pragma unroll 1
    for (int c = 0; c < NCH; ++c) {
      float v[32];
      ld(0, c, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int col = n0 + c * 32 + j;
        const float z = scale * v[j] - mx;
        const float e = col < N ? __expf(z) : 0.f;
        s += e;
        u += e * z;
      }
    }
    if (valid) {
      const int tile = n0 / (NCH * 32);
      reinterpret_cast<float4*>(part)[(size_t)tile * M + row] =
          make_float4(mx, s, u, (float)am);
    }
  }
};

// ---------------------------------------------------------------------------
// dense kernel: grid (ceil(M / (128 MT)), ceil(N / BN), ksplit); 128 threads.
// warp 0 lane 0: TMA producer; warp 1 lane 0: MMA issuer; warp 2: TMEM owner;
// all four warps: epilogue (warp w reads accumulator lanes 32w .. 32w + 31).
// ksplit > 1 (launched as clusters of ksplit CTAs along z): CTA r accumulates the
// r-th slice of K; the partial tiles are then reduced through distributed shared
// memory: CTA r owns rows [r R, (r+1) R) of the tile (R = 128 MT / ksplit),
// receives every CTA's partial rows into slot [source rank], sums the slots in
// rank order (deterministic) and runs the epilogue for its rows.
// ---------------------------------------------------------------------------
namespace cl {
__device__ __forceinline__ uint32_t ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t map(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}
}  // namespace cl

template <int BN, int MT, bool DUAL, int ST>
struct DenseCfg {
  static constexpr int NACC = DUAL ? 2 : 1;
  static constexpr uint32_t B_BYTES = BN * TC_KB * 2;
  static constexpr uint32_t STAGE = MT * TC_SUB_A + NACC * B_BYTES;
  static constexpr uint32_t TCOLS = TmemCols<MT * NACC * BN>::value;
  static constexpr size_t SMEM = 1024 + (size_t)ST * STAGE + 256;
  static_assert(MT * NACC * BN <= 512, "accumulators exceed TMEM");
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
};

template <int BN, int MT, bool DUAL, int ST, class Epi>
__global__ void __launch_bounds__(128, 1)
    tc_dense_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB,
                    const __grid_constant__ CUtensorMap mB2, int M, int K, int ksplit, Epi epi,
                    int32_t* err) {
  typedef DenseCfg<BN, MT, DUAL, ST> Cfg;
  // split-K needs the whole fp32 tile in the (drained) pipeline buffers and a chunk epilogue
  constexpr int RS = Cfg::NACC * BN + 4;  // reduction row stride (floats): padded against bank conflicts
  constexpr bool kSplitOK =
      MT * 128 * RS * 4 <= ST * Cfg::STAGE && (Epi::kChunked || Epi::kRowWise);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * Cfg::STAGE);
  uint64_t* empty = full + ST;
  uint64_t* done = empty + ST;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * (MT * 128), n0 = blockIdx.y * BN;
  const int nk_all = (K + TC_KB - 1) / TC_KB;
  const int rank = ksplit > 1 ? (int)cl::ctarank() : 0;
  const int kb_lo = (int)((long)nk_all * rank / ksplit);
  const int nk = (int)((long)nk_all * (rank + 1) / ksplit) - kb_lo;
  const int rot = nk > 0 ? (int)(blockIdx.y % nk) : 0;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < ST; ++s) {
      tc::mbar_init(full + s, 1);
      tc::mbar_init(empty + s, 1);
    }
    tc::mbar_init(done, 1);
    tc::fence_mbar_init();
  }
  if (warp == 2) tc::tmem_alloc(tslot, Cfg::TCOLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;
  pdl_enter();  // global memory is touched only from here on

  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&mA);
    tc::prefetch_tmap(&mB);
    if (DUAL) tc::prefetch_tmap(&mB2);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % ST;
      const uint32_t ph = (kb / ST) & 1;
      if (kb >= ST && !tc::mbar_wait(empty + s, ph ^ 1)) {
        atomicOr(err, ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      uint8_t* st = smem + s * Cfg::STAGE;
      tc::mbar_expect_tx(full + s, Cfg::STAGE);
#pragma unroll
      // CTAs start their K walk at different offsets so that they do not all read
      // the same activation tile from the same L2 slices at the same time
      const int kx = (kb_lo + (kb + rot) % nk) * TC_KB;
      for (int mt = 0; mt < MT; ++mt)
        tc::tma_load_2d(st + mt * TC_SUB_A, &mA, full + s, kx, m0 + mt * 128);
      tc::tma_load_2d(st + MT * TC_SUB_A, &mB, full + s, kx, n0);
      if (DUAL) tc::tma_load_2d(st + MT * TC_SUB_A + Cfg::B_BYTES, &mB2, full + s, kx, n0);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = tc::idesc_bf16(128, BN);
    bool ok = true;
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int s = kb % ST;
      const uint32_t ph = (kb / ST) & 1;
      if (!tc::mbar_wait(full + s, ph)) {
        atomicOr(err, ERR_TIMEOUT);
        *abort_flag = 1;
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint32_t a0 = tc::smem_addr(smem + s * Cfg::STAGE);
      const uint32_t b0 = a0 + MT * TC_SUB_A;
#pragma unroll
      for (int k = 0; k < TC_KB / 16; ++k) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const uint64_t ad = tc::sdesc_k128(a0 + mt * TC_SUB_A + k * 32);
          const uint32_t acc = (kb | k) != 0;
          tc::mma_bf16(tmem + (mt * Cfg::NACC) * BN, ad, tc::sdesc_k128(b0 + k * 32), idesc, acc);
          if (DUAL)
            tc::mma_bf16(tmem + (mt * Cfg::NACC + 1) * BN, ad,
                         tc::sdesc_k128(b0 + Cfg::B_BYTES + k * 32), idesc, acc);
        }
      }
      tc::mma_commit(empty + s);
    }
    if (ok) tc::mma_commit(done);
  }
  __syncwarp();

  // epilogue: wait for the accumulators
  bool ready = true;
  if (lane == 0) ready = nk == 0 || tc::mbar_wait(done, 0);
  ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
  if (!ready && lane == 0) atomicOr(err, ERR_TIMEOUT);
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
  if (ksplit == 1) {
    if (ready) {
      tc::fence_after_sync();
#pragma unroll 1
      for (int mt = 0; mt < MT; ++mt) {
        const int row = m0 + mt * 128 + 32 * warp + lane;
        auto ld = [&](int a, int c, float* v) {
          tc::tmem_ld32(tmem + lane_base + (mt * Cfg::NACC + a) * BN + c * 32, v);
        };
        epi.template run<BN / 32>(row, row < M, n0, ld);
      }
    }
  } else if constexpr (kSplitOK) {
    // every thread of every CTA passes both cluster barriers, whatever happened above
    const int R = MT * 128 / ksplit;         // rows owned per CTA
    cl::sync();                              // all pipelines drained: smem reusable
    if (ready) {
      tc::fence_after_sync();
      const uint32_t recv = tc::smem_addr(smem);
#pragma unroll 1
      for (int mt = 0; mt < MT; ++mt) {
        const int trow = mt * 128 + 32 * warp + lane;  // row within the tile
        const int owner = trow / R, lr = trow % R;
        const uint32_t dst = cl::map(recv, owner) + (uint32_t)(((rank * R + lr) * RS) * 4);
#pragma unroll 1
        for (int a = 0; a < Cfg::NACC; ++a)
#pragma unroll 1
          for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            tc::tmem_ld32(tmem + lane_base + (mt * Cfg::NACC + a) * BN + c * 32, v);
            const uint32_t o = dst + (uint32_t)((a * BN + c * 32) * 4);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              cl::st4(o + 16 * j, v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          }
      }
    }
    cl::sync();                              // all partial rows delivered
    const float* buf = reinterpret_cast<const float*>(smem);
    if constexpr (Epi::kRowWise) {  // one thread per owned row, chunks summed on demand
      for (int lr = threadIdx.x; lr < R; lr += blockDim.x) {
        auto ld = [&](int a, int c, float* v) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
          for (int src = 0; src < ksplit; ++src) {
            const float* p = buf + (size_t)(src * R + lr) * RS + a * BN + c * 32;
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += p[j];
          }
        };
        const int row = m0 + rank * R + lr;
        epi.template run<BN / 32>(row, row < M, n0, ld);
      }
    } else
    for (int item = threadIdx.x; item < R * (BN / 32); item += blockDim.x) {
      const int lr = item / (BN / 32), c = item % (BN / 32);
      float v[32], u[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        v[j] = 0.f;
        u[j] = 0.f;
      }
      for (int src = 0; src < ksplit; ++src) {
        const float* p = buf + (size_t)(src * R + lr) * RS + c * 32;
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += p[j];
        if (DUAL) {
#pragma unroll
          for (int j = 0; j < 32; ++j) u[j] += p[BN + j];
        }
      }
      const int row = m0 + rank * R + lr;
      epi.chunk(row, row < M, n0 + c * 32, v, u);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 2) tc::tmem_dealloc(tmem, Cfg::TCOLS);
}

// ---------------------------------------------------------------------------
// grouped expert kernel (persistent).  Work unit u = chunk * FT + f: token chunk
// `chunk` (expert e = chunk_e[chunk], permuted rows r0 = chunk_r0[chunk] ..
// r0 + n - 1, n <= 128) times weight-row tile f (128 rows of the expert's
// weight).  GATEUP: two weights (gate, up) [E*I, d] -> hb[r, f*128 + i] =
// silu(g) * u (bf16).  Otherwise: down [E*d, I] -> yb[r, f*128 + i] =
// gate_of[r] * acc (fp32).
// 192 threads: warp 0 TMA, warp 1 MMA, warps 2..5 epilogue (TMEM lanes
// 32 (w % 4) .. +31).  One accumulator set; the MMA warp waits for the epilogue
// to drain it before the next unit, while the producer keeps streaming.
// ---------------------------------------------------------------------------
template <bool GATEUP, int ST>
struct ExpertCfg {
  static constexpr int NW = GATEUP ? 2 : 1;
  static constexpr uint32_t B_MAX = 128 * TC_KB * 2;
  static constexpr uint32_t STAGE = NW * TC_SUB_A + B_MAX;
  static constexpr uint32_t TCOLS = GATEUP ? 256 : 128;
  static constexpr size_t SMEM = 1024 + (size_t)ST * STAGE + 256;
};

template <bool GATEUP, int ST>
__global__ void __launch_bounds__(192, 1)
    tc_expert_kernel(const __grid_constant__ CUtensorMap mW, const __grid_constant__ CUtensorMap mW2,
                     const __grid_constant__ CUtensorMap mX, const int32_t* __restrict__ chunk_e,
                     const int32_t* __restrict__ chunk_r0, const int32_t* __restrict__ n_chunks,
                     const int32_t* __restrict__ offsets, int w_rows_per_expert, int K, int FT,
                     void* __restrict__ out, int ldo, const float* __restrict__ gate_of,
                     int32_t* err) {
  typedef ExpertCfg<GATEUP, ST> Cfg;
  pdl_enter();  // the routing tables come from the preceding kernels
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * Cfg::STAGE);
  uint64_t* empty = full + ST;
  uint64_t* tfull = empty + ST;   // accumulator ready (MMA -> epilogue)
  uint64_t* tempty = tfull + 1;   // accumulator drained (epilogue -> MMA), 4 arrivals
  uint32_t* tslot = reinterpret_cast<uint32_t*>(tempty + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_units = *n_chunks * FT;
  const int nk = (K + TC_KB - 1) / TC_KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      tc::mbar_init(full + s, 1);
      tc::mbar_init(empty + s, 1);
    }
    tc::mbar_init(tfull, 1);
    tc::mbar_init(tempty, 4);
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
        const uint32_t bytes = Cfg::NW * TC_SUB_A + (uint32_t)nb * 32 * TC_KB * 2;
        const int wrow = e * w_rows_per_expert + f * 128;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % ST;
          const uint32_t ph = (it / ST) & 1;
          if (it >= ST && !tc::mbar_wait(empty + s, ph ^ 1)) {
            atomicOr(err, ERR_TIMEOUT);
            u = n_units;
            break;
          }
          uint8_t* st = smem + s * Cfg::STAGE;
          // units of one token chunk start their K walk at different offsets
          const int kx = ((kb + f) % nk) * TC_KB;
          tc::mbar_expect_tx(full + s, bytes);
          tc::tma_load_2d(st, &mW, full + s, kx, wrow);
          if (GATEUP) tc::tma_load_2d(st + TC_SUB_A, &mW2, full + s, kx, wrow);
          uint8_t* bt = st + Cfg::NW * TC_SUB_A;
          for (int j = 0; j < nb; ++j)
            tc::tma_load_2d(bt + j * 32 * TC_KB * 2, &mX, full + s, kx, r0 + 32 * j);
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
        // wait until the epilogue has drained the previous unit's accumulators
        if (ui > 0 && !tc::mbar_wait(tempty, (ui - 1) & 1)) {
          atomicOr(err, ERR_TIMEOUT);
          break;
        }
        tc::fence_after_sync();
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % ST;
          const uint32_t ph = (it / ST) & 1;
          if (!tc::mbar_wait(full + s, ph)) {
            atomicOr(err, ERR_TIMEOUT);
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t a0 = tc::smem_addr(smem + s * Cfg::STAGE);
          const uint32_t b0 = a0 + Cfg::NW * TC_SUB_A;
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
  } else {
    // epilogue warps 2..5 -> TMEM lane quarter (warp % 4)
    const int q = warp & 3;
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
      const int fr = f * 128 + 32 * q + lane;  // weight row within the expert = output column
      const int nch = (n + 31) >> 5;
#pragma unroll 1
      for (int c = 0; c < nch; ++c) {
        float v[32];
        tc::tmem_ld32(tmem + lane_base + c * 32, v);
        if (GATEUP) {
          float g2[32];
          tc::tmem_ld32(tmem + lane_base + 128 + c * 32, g2);
          bf16* o = reinterpret_cast<bf16*>(out);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = c * 32 + j;
            if (t < n) o[(size_t)(r0 + t) * ldo + fr] = __float2bfloat16_rn(silu(v[j]) * g2[j]);
          }
        } else {
          float* o = reinterpret_cast<float*>(out);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = c * 32 + j;
            if (t < n) o[(size_t)(r0 + t) * ldo + fr] = gate_of[r0 + t] * v[j];
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_addr(tempty)) : "memory");
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, Cfg::TCOLS);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
dg_status tc_prepare(dg_model* m);
void tc_release(dg_model* m);
inline int tc_group_rows() { return 128; }
dg_status tc_gemm_store_f32(dg_model* m, const bf16* A, const void* W, float* out, int M, int N,
                            int K, cudaStream_t st);
dg_status tc_gemm_qkv_rope(dg_model* m, const bf16* A, const void* W, int M, int n_seq, int np,
                           int pos0, bf16* q, bf16* kc, bf16* vc, cudaStream_t st);
dg_status tc_gemm_f32_rows(dg_model* m, const bf16* A, int a_rows, const void* W, float* out,
                           int M, int N, int K, cudaStream_t st);
dg_status tc_gemm_add_residual(dg_model* m, const bf16* A, const void* W, float* x, int M, int N,
                               int K, cudaStream_t st);
dg_status tc_gemm_swiglu(dg_model* m, const bf16* A, const void* Wg, const void* Wu, bf16* out,
                         int M, int N, int K, cudaStream_t st);
dg_status tc_moe_gate_up(dg_model* m, int l, const bf16* X, bf16* hb, int grid_y, cudaStream_t st);
dg_status tc_moe_down(dg_model* m, int l, const bf16* H, float* yb, int grid_y, cudaStream_t st);
dg_status tc_lmhead_stats(dg_model* m, const bf16* xn, int M, float* ent, int32_t* amax,
                          cudaStream_t st);
dg_status tc_attention(dg_model* m, const bf16* q, int B, int nq, int qpos0, const dg_kv* kv,
                       int l, const bf16* kB, const bf16* vB, int nB, int kposB, int npB,
                       bool causal, bf16* out, cudaStream_t st);

}  // namespace dg
