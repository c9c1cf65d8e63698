// tcgen05 (5th-generation tensor core) kernels for the bf16 dense contractions:
//   * tc_dense_kernel  — D[M, N] = A[M, K] W[N, K]^T, activations as the MMA
//     A operand (128-row sub-tiles, up to MT per CTA so each weight tile is read
//     from HBM once), weights as the B operand; fused epilogues: fp32 store,
//     residual add, SwiGLU (two weight operands), and the LM-head per-row
//     softmax statistics (the logits never leave the SM).
//   * tc_moe_kernel — the routed experts (gate/up SwiGLU, then gate-weighted down)
//     in one persistent launch: weights as the MMA A operand (two 128-row tiles
//     per unit) and the expert's gathered token rows as the B operand (N = tokens
//     rounded up to 32, <= 128); down units of a token chunk wait, on the device,
//     for the chunk's gate/up units.
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
#include "k_anneal.cuh"
#include "k_common.cuh"
#include "k_selfcond.cuh"
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
// Epilogues of the dense kernel.
//
// Staged epilogues (kStaged): the kernel stages the fp32 accumulator tile in
// shared memory, sums the split-K partials of the cluster there in a fixed order
// and hands the result over with lane = column, so that every store of a warp
// covers consecutive columns:
//   col4(row, col, v, u): four consecutive elements from col (a multiple of 4;
//   u: the second weight's accumulator, DUAL);
//   warp_rows<NQ, RB>(row0, M, n0, v, lane) (kWarpRows): RB whole rows, lane l
//   holding columns n0 + l + 32 q.
// Direct epilogues (!kStaged) read TMEM rows themselves: run(row, valid, n0, ld)
// with ld(acc, chunk, v) loading 32 fp32 columns of one row; never split.
// ---------------------------------------------------------------------------
struct EpiStoreF32 {
  static constexpr bool kStaged = true, kWarpRows = false;
  static constexpr size_t kExtraSmem = 0;
  __device__ void prefill(uint8_t*, int, int, int, int, int, int) const {}
  __device__ const float* cache() const { return nullptr; }
  float* out;
  int ldo, N;
  EpiStoreF32(float* o, int l, int n) : out(o), ldo(l), N(n) {}
  __device__ void col4(int row, int c, float4 v, float4) const {
    float* p = out + (size_t)row * ldo + c;
    if (c + 4 <= N) {
      *reinterpret_cast<float4*>(p) = v;
    } else {
      const float a[4] = {v.x, v.y, v.z, v.w};
      for (int j = 0; j < 4 && c + j < N; ++j) p[j] = a[j];
    }
  }
};

struct EpiAddF32 {
  // the residual rows this CTA owns ([R <= 64][64 columns] fp32) are read into shared
  // memory by the warps idle during the main loop; col4 then adds from there
  static constexpr bool kStaged = true, kWarpRows = false;
  static constexpr int kCacheRows = 64, kCacheCols = 64;
  static constexpr size_t kExtraSmem = (size_t)kCacheRows * kCacheCols * 4;
  float* out;
  int ldo, N;
  EpiAddF32(float* o, int l, int n) : out(o), ldo(l), N(n) {}
  __device__ void prefill(uint8_t* extra, int row_base, int R, int M, int n0, int t,
                          int nt) const {
    if (R > kCacheRows || n0 + kCacheCols > N) return;
    float4* dst = reinterpret_cast<float4*>(extra);
    const int units = R * (kCacheCols / 4);
    constexpr int U = 8;
    for (int base = t; base < units; base += nt * U) {
      float4 x[U];
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const int idx = base + k * nt, r = idx / (kCacheCols / 4), c = idx % (kCacheCols / 4);
        if (idx < units && row_base + r < M)
          x[k] = reinterpret_cast<const float4*>(out + (size_t)(row_base + r) * ldo + n0)[c];
      }
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const int idx = base + k * nt;
        if (idx < units && row_base + idx / (kCacheCols / 4) < M) dst[idx] = x[k];
      }
    }
  }
  // residual rows from the cache when it holds them (R <= 64 and a full 64-column tile)
  __device__ void col4_cached(const uint8_t* extra, int row_base, int R, int n0, int row, int c,
                              float4 v) const {
    if (R <= kCacheRows && n0 + kCacheCols <= N) {
      float4 o = reinterpret_cast<const float4*>(extra)[(row - row_base) * (kCacheCols / 4) +
                                                        (c - n0) / 4];
      o.x += v.x;
      o.y += v.y;
      o.z += v.z;
      o.w += v.w;
      *reinterpret_cast<float4*>(out + (size_t)row * ldo + c) = o;
    } else {
      col4(row, c, v, v);
    }
  }
  __device__ void col4(int row, int c, float4 v, float4) const {
    float* p = out + (size_t)row * ldo + c;
    if (c + 4 <= N) {
      float4 o = *reinterpret_cast<float4*>(p);
      o.x += v.x;
      o.y += v.y;
      o.z += v.z;
      o.w += v.w;
      *reinterpret_cast<float4*>(p) = o;
    } else {
      const float a[4] = {v.x, v.y, v.z, v.w};
      for (int j = 0; j < 4 && c + j < N; ++j) p[j] += a[j];
    }
  }
};

struct EpiSwigluBf16 {
  static constexpr bool kStaged = true, kWarpRows = false;
  static constexpr size_t kExtraSmem = 0;
  __device__ void prefill(uint8_t*, int, int, int, int, int, int) const {}
  bf16* out;
  int ldo, N;
  EpiSwigluBf16(bf16* o, int l, int n) : out(o), ldo(l), N(n) {}
  __device__ void col4(int row, int c, float4 g, float4 u) const {
    bf16* p = out + (size_t)row * ldo + c;
    const __nv_bfloat162 lo = __floats2bfloat162_rn(silu(g.x) * u.x, silu(g.y) * u.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(silu(g.z) * u.z, silu(g.w) * u.w);
    if (c + 4 <= N) {
      uint2 w;
      w.x = *reinterpret_cast<const uint32_t*>(&lo);
      w.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(p) = w;
    } else {
      const bf16 a[4] = {lo.x, lo.y, hi.x, hi.y};
      for (int j = 0; j < 4 && c + j < N; ++j) p[j] = a[j];
    }
  }
};

// Warp-row epilogues: a warp owns one output row; lane l holds the columns
// n0 + l + 32 q (q < BN / 32) of the summed accumulator.  The kernel stages the
// accumulator rows in shared memory (and sums split-K partials there) first.
//
// QKV projection (N-tile = one head of h = 128): rotate query and key heads
// (pairs (j, j + 64) by pos * theta_j; cos / sin from the table rope[pos, 64] /
// rope[max_pos + pos, 64]) and scatter: q -> q[row, head, :], k -> kc[b, g, i, :],
// v -> vc[b, g, :, i] (transposed); all bf16.  Row = b * n_seq + i sits at
// position pos0 + i.
struct EpiQkvRope {
  static constexpr bool kStaged = true, kWarpRows = true;
  // cos / sin (fp32) of the positions of up to kCacheRows owned rows, filled by the
  // warps that are idle during the main loop
  static constexpr int kCacheRows = 64;
  static constexpr size_t kExtraSmem = (size_t)kCacheRows * 64 * 2 * 4;
  static constexpr int kVtStride = 66;  // bf16 per transposed row: conflict-free columns
  bf16 *q, *kc, *vc;
  const float* rope;
  int max_pos, n_seq, np, pos0, Hq, Hkv;

  __device__ bool cached(int R) const { return R <= kCacheRows; }
  // owned rows of a value head go through a transposed tile in shared memory
  __device__ bool v_tile(int n0, int row_base, int R) const {
    return n0 / 128 >= Hq + Hkv && R <= kCacheRows && (row_base % n_seq) + R <= n_seq &&
           ((row_base % n_seq) & 1) == 0;
  }
  __device__ void prefill(uint8_t* extra, int row_base, int R, int M, int, int t, int nt) const {
    if (!cached(R)) return;
    // 16-byte units: rows of 64 floats = 16 units, cos then sin; all loads of a round
    // are issued before its stores
    float4* dst = reinterpret_cast<float4*>(extra);
    const int units = R * 16 * 2;
    constexpr int U = 8;
    for (int base = t; base < units; base += nt * U) {
      float4 x[U];
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const int idx = base + k * nt;
        if (idx < units) {
          const int tab = idx / (R * 16), rem = idx % (R * 16), r = rem >> 4, c = rem & 15;
          const int row = row_base + r;
          const int pos = pos0 + (row < M ? row % n_seq : 0);
          x[k] = reinterpret_cast<const float4*>(rope + ((size_t)tab * max_pos + pos) * 64)[c];
        }
      }
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const int idx = base + k * nt;
        if (idx < units) {
          const int tab = idx / (R * 16), rem = idx % (R * 16);
          dst[tab * kCacheRows * 16 + rem] = x[k];
        }
      }
    }
  }
  // rows row0 .. row0 + RB - 1 (those < M)
  template <int NQ, int RB>
  __device__ void warp_rows(int row0, int M, int n0, const float (*v)[NQ], int lane,
                            const uint8_t* extra, int row_base, int R, uint8_t* vt_s) const {
    static_assert(NQ == 4, "one head of 128 per tile");
    const int head = n0 / 128;
    if (head < Hq + Hkv) {
      float cs[RB][2], sn[RB][2];
      const bool hit = cached(R);
      const float* ccs = reinterpret_cast<const float*>(extra);
      const float* csn = ccs + kCacheRows * 64;
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        const int pos = pos0 + (row0 + r < M ? (row0 + r) % n_seq : 0);
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          const int j = lane + 32 * q2;
          if (hit) {
            cs[r][q2] = ccs[(row0 + r - row_base) * 64 + j];
            sn[r][q2] = csn[(row0 + r - row_base) * 64 + j];
          } else {
            cs[r][q2] = rope[(size_t)pos * 64 + j];
            sn[r][q2] = rope[((size_t)max_pos + pos) * 64 + j];
          }
        }
      }
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        const int row = row0 + r;
        if (row >= M) break;
        const int b = row / n_seq, i = row % n_seq;
        bf16* dst = head < Hq ? q + ((size_t)row * Hq + head) * 128
                              : kc + (((size_t)b * Hkv + (head - Hq)) * np + i) * 128;
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          const int j = lane + 32 * q2;
          const float x1 = v[r][q2], x2 = v[r][q2 + 2];
          dst[j] = __float2bfloat16_rn(x1 * cs[r][q2] - x2 * sn[r][q2]);
          dst[j + 64] = __float2bfloat16_rn(x2 * cs[r][q2] + x1 * sn[r][q2]);
        }
      }
    } else if (v_tile(n0, row_base, R)) {
      bf16* t = reinterpret_cast<bf16*>(vt_s);  // [128 dims][kVtStride]
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        if (row0 + r >= M) break;
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2)
          t[(lane + 32 * q2) * kVtStride + (row0 + r - row_base)] = __float2bfloat16_rn(v[r][q2]);
      }
    } else {
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        const int row = row0 + r;
        if (row >= M) break;
        const int b = row / n_seq, i = row % n_seq;
        bf16* vt = vc + ((size_t)b * Hkv + (head - Hq - Hkv)) * 128 * np + i;
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2)
          vt[(size_t)(lane + 32 * q2) * np] = __float2bfloat16_rn(v[r][q2]);
      }
    }
  }
  // after every warp's rows: the transposed value tile -> vc rows of 2 R contiguous bytes
  __device__ void tail(uint8_t* vt_s, int row_base, int R, int M, int n0) const {
    if (!v_tile(n0, row_base, R)) return;
    const int g = n0 / 128 - Hq - Hkv;
    const int b = row_base / n_seq, i0 = row_base % n_seq;
    const int n_ok = min(R, M - row_base);
    const uint32_t* t = reinterpret_cast<const uint32_t*>(vt_s);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int d = warp; d < 128; d += blockDim.x >> 5) {
      bf16* dst = vc + (((size_t)b * Hkv + g) * 128 + d) * np + i0;
      for (int pr = lane; 2 * pr < n_ok; pr += 32) {
        const uint32_t two = t[(d * kVtStride) / 2 + pr];
        if (2 * pr + 1 < n_ok) {
          *reinterpret_cast<uint32_t*>(dst + 2 * pr) = two;
        } else {
          dst[2 * pr] = *reinterpret_cast<const bf16*>(&two);
        }
      }
    }
  }
};

// Router (N-tile = all E <= 32 NQ experts of a row): softmax over the E logits,
// the top_k experts by probability (ties -> lower id) and their gates
// renormalised over the selection: idx / gate [row, top_k]; lane k keeps the
// k-th selection.
struct EpiRouterTopk {
  static constexpr bool kStaged = true, kWarpRows = true;
  static constexpr size_t kExtraSmem = 0;
  __device__ void prefill(uint8_t*, int, int, int, int, int, int) const {}
  __device__ void tail(uint8_t*, int, int, int, int) const {}
  int32_t* idx;
  float* gate;
  int E, top_k;
  // the warp's RB rows side by side (each row's arithmetic as for a single row), so that
  // the warp reductions of the rows overlap
  template <int NQ, int RB>
  __device__ void warp_rows(int row0, int M, int n0, const float (*v)[NQ], int lane,
                            const uint8_t*, int, int, uint8_t*) const {
    float p[RB][NQ];
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      float mx = -INFINITY;
#pragma unroll
      for (int q2 = 0; q2 < NQ; ++q2) {
        p[r][q2] = lane + 32 * q2 < E ? v[r][q2] : -INFINITY;
        mx = fmaxf(mx, p[r][q2]);
      }
      mx = warp_max(mx);
      float z = 0.f;
#pragma unroll
      for (int q2 = 0; q2 < NQ; ++q2) {
        p[r][q2] = lane + 32 * q2 < E ? expf(p[r][q2] - mx) : 0.f;
        z += p[r][q2];
      }
      z = warp_sum(z);
#pragma unroll
      for (int q2 = 0; q2 < NQ; ++q2) p[r][q2] /= z;
    }
    unsigned taken[RB];
    float gsum[RB], my_p[RB];
    int my_e[RB];
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      taken[r] = 0;
      gsum[r] = 0.f;
      my_p[r] = 0.f;
      my_e[r] = 0;
    }
    for (int k = 0; k < top_k; ++k) {
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        // this lane's best untaken probability (lowest id on ties), then the warp's: the
        // probabilities are >= 0, so their bit patterns order like the values
        float bp = -1.f;
        int be = 0x7fffffff;
#pragma unroll
        for (int q2 = 0; q2 < NQ; ++q2) {
          const int e = lane + 32 * q2;
          if (e < E && !((taken[r] >> q2) & 1u) && p[r][q2] > bp) {
            bp = p[r][q2];
            be = e;
          }
        }
        const unsigned bits = bp >= 0.f ? __float_as_uint(bp) : 0u;
        const unsigned top = __reduce_max_sync(0xffffffffu, bits);
        be = (unsigned)__reduce_min_sync(0xffffffffu, bits == top && bp >= 0.f ? (unsigned)be
                                                                                : 0x7fffffffu);
        bp = __uint_as_float(top);
        if ((be & 31) == lane) taken[r] |= 1u << (be >> 5);
        if (lane == k) {
          my_e[r] = be;
          my_p[r] = bp;
        }
        gsum[r] += bp;
      }
    }
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int row = row0 + r;
      if (row < M && lane < top_k) {
        idx[(size_t)row * top_k + lane] = my_e[r];
        gate[(size_t)row * top_k + lane] = my_p[r] / gsum[r];
      }
    }
  }
};

// Partial tiles of a K-sliced GEMM (launched with ksplit < 0): thread per row, the
// CTA's accumulator rows stored to out + blockIdx.z * zstride ([M, N] fp32 per slice).
struct EpiPartialRows {
  static constexpr bool kStaged = false, kWarpRows = false;
  static constexpr size_t kExtraSmem = 0;
  float* out;
  int M, N;
  size_t zstride;
  template <int NCH, class Ld>
  __device__ void run(int row, bool valid, int n0, Ld&& ld) const {
    float* o = out + (size_t)blockIdx.z * zstride + (size_t)row * N;
#pragma unroll 1
    for (int c = 0; c < NCH; ++c) {
      float v[32];
      ld(0, c, v);  // warp-collective: every lane loads
      const int c0 = n0 + c * 32;
      if (!valid || c0 >= N) continue;
      if (c0 + 32 <= N) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          reinterpret_cast<float4*>(o + c0)[q] =
              make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      } else {
        for (int j = 0; j < 32 && c0 + j < N; ++j) o[c0 + j] = v[j];
      }
    }
  }
};

// Per-row statistics of logits l = scale * acc over this CTA's vocabulary tile
// (columns n0 .. n0 + 32 NCH - 1, those < N): m = max, s = sum exp(l - m),
// u = sum exp(l - m) (l - m), a = lowest id attaining m.  part[(tile, row)] = (m, s, u, a).
// With an.N > 0 the logits are tempered (l = scale acc / tau) and, with an.seeds, the
// tile's winner of the Gumbel-max race goes to an.gpart[(tile, row)] = (l / tau - log E,
// id).  With sc.P, the tile's values exp(l1 - ref) at temperature 1 (l1 = scale acc,
// ref = its largest) go to sc.P as bf16 and (ref, their sum) to sc.ref (self-conditioning).
// Pass 1 finds the largest accumulator (a max tree per 32-column chunk; the index is
// searched only in a chunk that raises the maximum).  Pass 2 works in base-2 units,
// z2 = (l - m) log2 e, e = 2^z2 (ex2.approx.ftz), with two interleaved sums; columns
// >= N hold a large negative finite value, so that no column test is needed per element.
struct EpiLmStats {
  static constexpr bool kStaged = false, kWarpRows = false;
  static constexpr size_t kExtraSmem = 0;
  float* part;
  int M, N;
  float scale;
  AnnealDev an = {};
  ScDev sc = {};

  static __device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
  }

  template <int NCH, class Ld>
  __device__ void run(int row, bool valid, int n0, Ld&& ld) const {
    constexpr float kLog2e = 1.4426950408889634f;
    const float tau = an.N > 0 ? (float)an.tau() : 1.f;
    const float sc_ = an.N > 0 ? (float)((double)scale / an.tau()) : scale;
    const float sc2 = sc_ * kLog2e;
    auto load = [&](int c, float* v) {
      ld(0, c, v);
      if (n0 + c * 32 + 32 > N) {  // the ragged last tile (uniform across the warp)
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (n0 + c * 32 + j >= N) v[j] = -1e30f;
      }
    };
    // pass 1
    float mv = -INFINITY;
    int am = 0x7fffffff;
#pragma unroll 1
    for (int c = 0; c < NCH; ++c) {
      float v[32];
      load(c, v);
      float t[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) t[j] = fmaxf(v[j], v[j + 16]);
#pragma unroll
      for (int w = 8; w > 0; w >>= 1)
#pragma unroll
        for (int j = 0; j < w; ++j) t[j] = fmaxf(t[j], t[j + w]);
      if (t[0] > mv) {  // strict: an equal maximum in a later chunk keeps the earlier id
        int idx = 31;
#pragma unroll
        for (int j = 30; j >= 0; --j)
          if (v[j] == t[0]) idx = j;
        mv = t[0];
        am = n0 + c * 32 + idx;
      }
    }
    const bool draw = an.seeds != nullptr, scp = sc.P != nullptr;
    if (!draw && !scp) pass2<NCH, false, false>(row, valid, n0, load, mv, am, sc_, sc2, tau);
    else if (!draw) pass2<NCH, false, true>(row, valid, n0, load, mv, am, sc_, sc2, tau);
    else if (!scp) pass2<NCH, true, false>(row, valid, n0, load, mv, am, sc_, sc2, tau);
    else pass2<NCH, true, true>(row, valid, n0, load, mv, am, sc_, sc2, tau);
  }

  template <int NCH, bool DRAW, bool SC, class Load>
  __device__ void pass2(int row, bool valid, int n0, Load& load, float mv, int am, float sc_,
                        float sc2, float tau) const {
    constexpr float kLn2 = 0.6931471805599453f;
    const float mx = sc_ * mv, mx2 = sc2 * mv;
    const int tile = n0 / (NCH * 32);
    float s0 = 0.f, s1 = 0.f, u0 = 0.f, u1 = 0.f, p0 = 0.f, p1 = 0.f;
    // Gumbel-max race of this tile (DRAW): it starts from the tile's argmax (z = 0,
    // e = 1); a chunk where no row of the warp has e >= E_argmax^-1 E_min draws nothing
    // (no column there can beat the argmax).  Otherwise each output of the stream serves
    // a column pair, and since E = -log u >= 1 - u a column can beat the argmax (hence
    // the best so far) only if 1 - u < e E_argmax (the margin 2^-10 covers every
    // rounding): only those columns take the log, in a branch the warp skips when none of
    // its rows has one.
    GumbelBest<float> gb;
    unsigned long long st = 0;
    float lim = 0.f, tcap = 0.f;
    if constexpr (DRAW) {
      st = an.pair_state(valid ? row : 0, N, n0 >> 1);
      if (am < N)
        gb.offer(1.f,
                 sm64_expo(sm64_field(sm64_mix(st + (unsigned long long)((am - n0) >> 1) * SM64_G),
                                      am & 1),
                           0.f),
                 0.f, am);
      lim = gb.e * SM64_EMIN_LO / gb.E;
      tcap = gb.E * (1.f + 1.f / 1024.f);
    }
    // p0 tile values at temperature 1: 2^(z2 tau) (= e when tau = 1)
    bf16* prow = SC ? reinterpret_cast<bf16*>(sc.P) + (size_t)(valid ? row : 0) * sc.ldp : nullptr;
#pragma unroll 1
    for (int c = 0; c < NCH; ++c) {
      float v[32];
      load(c, v);
      bool cand = false;
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float z0 = fmaf(v[j], sc2, -mx2), z1 = fmaf(v[j + 1], sc2, -mx2);
        const float e0 = ex2(z0), e1 = ex2(z1);
        s0 += e0;
        s1 += e1;
        u0 = fmaf(e0, z0, u0);
        u1 = fmaf(e1, z1, u1);
        if constexpr (SC) {
          const float q0 = tau == 1.f ? e0 : ex2(z0 * tau), q1 = tau == 1.f ? e1 : ex2(z1 * tau);
          p0 += q0;
          p1 += q1;
          v[j] = q0;  // the p0 values are stored below, then z is recomputed if drawing
          v[j + 1] = q1;
        } else if constexpr (DRAW) {
          v[j] = z0;
          v[j + 1] = z1;
        }
        if constexpr (DRAW) cand |= fmaxf(e0, e1) >= lim;
      }
      if constexpr (SC) {
        if (valid && n0 + c * 32 < N) {
          uint4* dst = reinterpret_cast<uint4*>(prow + n0 + c * 32);
          const bool full = n0 + c * 32 + 32 <= N;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * q + 2 * h], v[8 * q + 2 * h + 1]);
              wp[h] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            if (full) {
              dst[q] = w;
            } else {
              const bf16* wb = reinterpret_cast<const bf16*>(&w);
              for (int h = 0; h < 8; ++h)
                if (n0 + c * 32 + 8 * q + h < N) prow[n0 + c * 32 + 8 * q + h] = wb[h];
            }
          }
        }
      }
      if constexpr (DRAW) {
        if (!__any_sync(0xffffffffu, cand)) continue;
        if constexpr (SC) {  // v holds the p0 values: bring back the tempered z2
          load(c, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = fmaf(v[j], sc2, -mx2);
        }
        const unsigned long long stc = st + (unsigned long long)(c * 16) * SM64_G;
        float uu[32];
        unsigned fm = 0;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const unsigned long long zz = sm64_mix(stc + (unsigned long long)q * SM64_G);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int j = 2 * q + h;
            const float uj = ((float)sm64_field(zz, h) + 0.5f) * 1.1920928955078125e-07f;
            uu[j] = uj;
            if (1.f - uj < ex2(v[j]) * tcap) fm |= 1u << j;
          }
        }
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (__any_sync(0xffffffffu, (fm >> j) & 1u) && ((fm >> j) & 1u))
            gb.offer(ex2(v[j]), -logf(uu[j]), v[j] * kLn2, n0 + c * 32 + j);
      }
    }
    if (valid) {
      if constexpr (DRAW)
        reinterpret_cast<float2*>(an.gpart)[(size_t)tile * M + row] =
            make_float2(gb.value(mx), (float)gb.id);  // ids < 2^24: exact
      if constexpr (SC)
        reinterpret_cast<float2*>(sc.ref)[(size_t)tile * M + row] = make_float2(scale * mv, p0 + p1);
      reinterpret_cast<float4*>(part)[(size_t)tile * M + row] =
          make_float4(mx, s0 + s1, (u0 + u1) * kLn2, (float)am);
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
__device__ __forceinline__ float lds(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float ldc(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float4 lds4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ float4 ldc4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void sts4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
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

// 256 threads: warp 0 lane 0 issues the TMA loads, warp 1 lane 0 the MMAs; all eight
// warps share the epilogue (warps w and w + 4 read the same TMEM lane quarter).
constexpr int TC_DENSE_THREADS = 256;

template <int BN, int MT, bool DUAL, int ST, class Epi>
__global__ void __launch_bounds__(TC_DENSE_THREADS, 1)
    tc_dense_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB,
                    const __grid_constant__ CUtensorMap mB2, int M, int K, int ksplit, Epi epi,
                    int32_t* err, int kwrap, int b_early) {
  // kwrap > 0: the B operand's K coordinate is taken modulo kwrap (A = [a1 | a2]
  // against B = [w | w] without storing w twice).
  // b_early != 0: B is a model weight, constant while the model runs, so its first
  // stages are requested before the preceding kernel has finished.
  typedef DenseCfg<BN, MT, DUAL, ST> Cfg;
  // staged epilogues reuse the drained pipeline buffers for the fp32 tile
  constexpr int RS = Cfg::NACC * BN + 4;  // staging row stride (floats): padded against bank conflicts
  static_assert(!Epi::kStaged || MT * 128 * RS * 4 <= ST * Cfg::STAGE, "staging buffer");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * Cfg::STAGE);
  uint64_t* empty = full + ST;
  uint64_t* done = empty + ST;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tslot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * (MT * 128), n0 = blockIdx.y * BN;
  // ksplit > 1: the K slices of a cluster, reduced through DSMEM; ksplit < 0: -ksplit
  // independent K slices along grid z, each leaving its own partial tile (the epilogue
  // writes it to slice blockIdx.z)
  const int nk_all = (K + TC_KB - 1) / TC_KB;
  const int nparts = ksplit < 0 ? -ksplit : ksplit;
  const int rank = ksplit > 1 ? (int)cl::ctarank() : (ksplit < 0 ? (int)blockIdx.z : 0);
  const int kb_lo = (int)((long)nk_all * rank / nparts);
  const int nk = (int)((long)nk_all * (rank + 1) / nparts) - kb_lo;
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
  // CTAs start their K walk at different offsets so that they do not all read the
  // same activation tile from the same L2 slices at the same time
  auto kcoord = [&](int kb) { return (kb_lo + (kb + rot) % nk) * TC_KB; };
  auto load_b = [&](int kb, int s) {
    const int kx = kcoord(kb), kxb = kwrap > 0 ? kx % kwrap : kx;
    uint8_t* st = smem + s * Cfg::STAGE;
    tc::tma_load_2d(st + MT * TC_SUB_A, &mB, full + s, kxb, n0);
    if (DUAL) tc::tma_load_2d(st + MT * TC_SUB_A + Cfg::B_BYTES, &mB2, full + s, kxb, n0);
  };
  const int early = b_early ? min(ST, nk) : 0;
  if (warp == 0 && lane == 0 && early > 0) {
    tc::prefetch_tmap(&mB);
    if (DUAL) tc::prefetch_tmap(&mB2);
    for (int kb = 0; kb < early; ++kb) {
      tc::mbar_expect_tx(full + kb, Cfg::STAGE);  // the whole stage: B now, A below
      load_b(kb, kb);
    }
  }
  pdl_enter();  // the activations (A) are read only from here on

  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&mA);
    if (early == 0) {
      tc::prefetch_tmap(&mB);
      if (DUAL) tc::prefetch_tmap(&mB2);
    }
    int kb = 0;
    for (; kb < nk; ++kb) {
      const int s = kb % ST;
      const uint32_t ph = (kb / ST) & 1;
      if (kb >= ST && !tc::mbar_wait(empty + s, ph ^ 1)) {
        atomicOr(err, ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      uint8_t* st = smem + s * Cfg::STAGE;
      if (kb >= early) {
        tc::mbar_expect_tx(full + s, Cfg::STAGE);
        load_b(kb, s);
      }
      const int kx = kcoord(kb);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
        tc::tma_load_2d(st + mt * TC_SUB_A, &mA, full + s, kx, m0 + mt * 128);
    }
    if (!tc::drain_slots(full, ST, kb)) atomicOr(err, ERR_TIMEOUT);
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
  } else if constexpr (Epi::kExtraSmem > 0) {
    // warps 2.. are idle during the main loop: they fill the epilogue's table cache
    if (warp >= 2)
      epi.prefill(smem + ST * Cfg::STAGE + 256, m0 + rank * (MT * 128 / ksplit),
                  MT * 128 / ksplit, M, n0, threadIdx.x - 64, TC_DENSE_THREADS - 64);
  }
  __syncwarp();

  // epilogue: wait for the accumulators
  bool ready = true;
  if (lane == 0) ready = nk == 0 || tc::mbar_wait(done, 0);
  ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
  if (!ready && lane == 0) atomicOr(err, ERR_TIMEOUT);
  const int quarter = warp & 3, half = warp >> 2;  // TMEM lane quarter; column half
  const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
  if constexpr (!Epi::kStaged) {
    // thread per row; with two 128-row blocks the two warp groups take one each
    if (ready && (MT == 2 || half == 0)) {
      tc::fence_after_sync();
#pragma unroll 1
      for (int mt = MT == 2 ? half : 0; mt < MT; mt += MT == 2 ? 2 : 1) {
        const int row = m0 + mt * 128 + 32 * quarter + lane;
        auto ld = [&](int a, int c, float* v) {
          tc::tmem_ld32(tmem + lane_base + (mt * Cfg::NACC + a) * BN + c * 32, v);
        };
        epi.template run<BN / 32>(row, row < M, n0, ld);
      }
    }
  } else {
    // 1. this CTA's partial tile -> its own shared memory, row-major (stride RS)
    const uint32_t stg = tc::smem_addr(smem);
    if (ready) {
      tc::fence_after_sync();
#pragma unroll 1
      for (int mt = 0; mt < MT; ++mt) {
        const uint32_t dst = stg + (uint32_t)((mt * 128 + 32 * quarter + lane) * RS * 4);
#pragma unroll 1
        for (int a = 0; a < Cfg::NACC; ++a)
#pragma unroll 1
          for (int c = half; c < BN / 32; c += 2) {
            float v[32];
            tc::tmem_ld32(tmem + lane_base + (mt * Cfg::NACC + a) * BN + c * 32, v);
            const uint32_t o = dst + (uint32_t)((a * BN + c * 32) * 4);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              cl::sts4(o + 16 * j, v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          }
      }
    }
    // every thread of every CTA passes the cluster barriers, whatever happened above
    if (ksplit > 1) cl::sync();
    else __syncthreads();
    // 2. this CTA owns rows [rank R, rank R + R) of the tile: sum the partials of the
    //    cluster's CTAs in rank order (lane = column), RB rows per warp at a time
    // Every instruction latency is exposed here (two warps per scheduler), so a warp
    // issues all loads of a pass (every source CTA) before it sums them.
    constexpr int NW = TC_DENSE_THREADS / 32;
    const int R = MT * 128 / ksplit;
    if constexpr (Epi::kWarpRows) {
      // lane = column; RB whole rows per warp at a time
      constexpr int NQ = Cfg::NACC * BN / 32;
      constexpr int RB = NQ >= 4 ? 2 : 4;
      static_assert(16 % RB == 0, "warp-row tiling");  // R is a multiple of 16
#pragma unroll 1
      for (int lr0 = warp * RB; lr0 < R; lr0 += NW * RB) {
        const int row0 = m0 + rank * R + lr0;
        if (row0 >= M) break;
        const uint32_t off = (uint32_t)(((rank * R + lr0) * RS + lane) * 4);
        float t[8][RB][NQ];
#pragma unroll
        for (int src = 0; src < 8; ++src) {
          if (src < ksplit) {
            const uint32_t rb = off + (src == rank ? stg : cl::map(stg, (uint32_t)src));
#pragma unroll
            for (int r = 0; r < RB; ++r)
#pragma unroll
              for (int q = 0; q < NQ; ++q) {
                const uint32_t ad = rb + (uint32_t)((r * RS + q * 32) * 4);
                t[src][r][q] = src == rank ? cl::lds(ad) : cl::ldc(ad);
              }
          }
        }
        float v[RB][NQ];
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            v[r][q] = 0.f;  // sources in rank order
#pragma unroll
            for (int src = 0; src < 8; ++src)
              if (src < ksplit) v[r][q] += t[src][r][q];
          }
        epi.template warp_rows<BN / 32, RB>(row0, M, n0, v, lane, smem + ST * Cfg::STAGE + 256,
                                            m0 + rank * R, R, smem + MT * 128 * RS * 4);
      }
      if constexpr (Epi::kExtraSmem > 0) {
        static_assert(MT * 128 * RS * 4 + 128 * 66 * 2 <= ST * Cfg::STAGE, "transposed tile");
        __syncthreads();  // every warp's rows are in the transposed tile
        epi.tail(smem + MT * 128 * RS * 4, m0 + rank * R, R, M, n0);
      }
    } else {
      // lane -> (row, 4 consecutive columns): a warp instruction covers RPW rows of BN
      constexpr int LPR = BN / 4, RPW = 32 / LPR;
      constexpr int IB = Cfg::NACC == 2 ? 1 : 2;  // warp instructions per pass
      // R is a multiple of 16, so a warp's RPW * IB rows lie wholly inside or outside it
      static_assert(BN <= 128 && 16 % (RPW * IB) == 0, "column epilogue tiling");
      const int rsub = lane / LPR, c4 = (lane % LPR) * 4;
#pragma unroll 1
      for (int lr0 = warp * RPW * IB; lr0 < R; lr0 += NW * RPW * IB) {
        if (m0 + rank * R + lr0 >= M) break;
        const uint32_t off = (uint32_t)(((rank * R + lr0 + rsub) * RS + c4) * 4);
        float4 t[8][IB][Cfg::NACC];
#pragma unroll
        for (int src = 0; src < 8; ++src) {
          if (src < ksplit) {
            const uint32_t rb = off + (src == rank ? stg : cl::map(stg, (uint32_t)src));
#pragma unroll
            for (int i = 0; i < IB; ++i)
#pragma unroll
              for (int a = 0; a < Cfg::NACC; ++a) {
                const uint32_t ad = rb + (uint32_t)((i * RPW * RS + a * BN) * 4);
                t[src][i][a] = src == rank ? cl::lds4(ad) : cl::ldc4(ad);
              }
          }
        }
#pragma unroll
        for (int i = 0; i < IB; ++i) {
          float4 v[Cfg::NACC];
#pragma unroll
          for (int a = 0; a < Cfg::NACC; ++a) {
            v[a] = make_float4(0.f, 0.f, 0.f, 0.f);  // sources in rank order
#pragma unroll
            for (int src = 0; src < 8; ++src)
              if (src < ksplit) {
                v[a].x += t[src][i][a].x;
                v[a].y += t[src][i][a].y;
                v[a].z += t[src][i][a].z;
                v[a].w += t[src][i][a].w;
              }
          }
          const int row = m0 + rank * R + lr0 + i * RPW + rsub;
          if (row < M) {
            if constexpr (Epi::kExtraSmem > 0)
              epi.col4_cached(smem + ST * Cfg::STAGE + 256, m0 + rank * R, R, n0, row, n0 + c4,
                              v[0]);
            else
              epi.col4(row, n0 + c4, v[0], v[Cfg::NACC - 1]);
          }
        }
      }
    }
    if (ksplit > 1) cl::sync();  // peers may still read this CTA's tile
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 2) tc::tmem_dealloc(tmem, Cfg::TCOLS);
}

// ---------------------------------------------------------------------------
// Routed experts in one persistent launch.  Token chunk `c` = expert e =
// chunk_e[c], permuted rows r0 = chunk_r0[c] .. r0 + n - 1 (n <= 128).
//   phase 1, unit u = c * FT1 + f (FT1 = I / 128): gate and up rows f*128 .. +127
//     of expert e against the chunk's rows X -> hb[r, f*128 + i] = silu(g) * u (bf16);
//   phase 2, unit v = c * FT2 + f (FT2 = d / 256): down rows f*256 .. +255 of
//     expert e (two 128-row tiles) against hb -> yb[r, f*256 + i] = gate_of[r] * acc.
// Units are numbered phase 1 first.  A block's TMA thread takes the next number from
// the device counter `next` (zeroed with `ready` before the launch) once it has issued
// the loads of its current unit, and passes it to the MMA thread and the epilogue
// through a small queue in shared memory.  A phase-2 unit waits for its chunk's
// phase-1 units (counted in ready[c]); those were taken earlier by running blocks,
// whose progress never depends on a waiting block, so every wait ends.
// Both phases run two MMAs per k-step (weights on the MMA's M side, tokens on N)
// into TMEM columns 0 and 128.  576 threads: warp 0 TMA, warp 1 MMA, warps 2..17
// epilogue (warps w, w + 4, w + 8 and w + 12 share a TMEM lane quarter and take one
// 32-token chunk each, so that each thread's share of the SwiGLU and of the stores is
// a quarter of a unit's).
// ---------------------------------------------------------------------------
template <int ST>
struct MoeCfg {
  static constexpr uint32_t B_MAX = 128 * TC_KB * 2;
  static constexpr uint32_t STAGE = 2 * TC_SUB_A + B_MAX;
  static constexpr uint32_t TCOLS = 256;
  static constexpr size_t SMEM = 1024 + (size_t)ST * STAGE + 256;
};
constexpr int MOE_EPI_WARPS = 16;
constexpr int TC_MOE_THREADS = 64 + 32 * MOE_EPI_WARPS;

template <int ST>
__global__ void __launch_bounds__(TC_MOE_THREADS, 1)
    tc_moe_kernel(const __grid_constant__ CUtensorMap mWg, const __grid_constant__ CUtensorMap mWu,
                  const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mWd,
                  const __grid_constant__ CUtensorMap mH, const int32_t* __restrict__ chunk_e,
                  const int32_t* __restrict__ chunk_r0, const int32_t* __restrict__ n_chunks,
                  const int32_t* __restrict__ offsets, int I, int d, bf16* __restrict__ hb,
                  float* __restrict__ yb, const float* __restrict__ gate_of,
                  int32_t* __restrict__ ready, int32_t* __restrict__ next, int32_t* err,
                  uint64_t limit_ns, int stall) {
  // limit_ns: how long any wait of this launch may last before it gives up (records
  // ERR_TIMEOUT and unwinds); stall != 0 (tests of that path only): a down unit waits for
  // one more gate/up unit than its chunk has, so every such wait runs out
  typedef MoeCfg<ST> Cfg;
  pdl_enter();  // the routing tables come from the preceding kernels
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * Cfg::STAGE);
  uint64_t* empty = full + ST;
  uint64_t* tfull = empty + ST;   // accumulators ready (MMA -> epilogue)
  uint64_t* tempty = tfull + 1;   // accumulators drained (epilogue -> MMA), one per epilogue warp
  // units taken by the TMA thread, in order, for the MMA thread and the epilogue leader
  constexpr int QD = 4;
  uint64_t* qfull = tempty + 1;   // [QD] unit id written (TMA thread)
  uint64_t* qempty = qfull + QD;  // [QD] unit id read (MMA thread + epilogue leader)
  int32_t* qid = reinterpret_cast<int32_t*>(qempty + QD);  // [QD]
  int32_t* ubc = qid + QD;        // the epilogue leader's broadcast of the unit id
  uint32_t* tslot = reinterpret_cast<uint32_t*>(ubc + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nc = *n_chunks;
  const int FT1 = I / 128, FT2 = d / 256;
  const int U1 = nc * FT1, n_units = U1 + nc * FT2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      tc::mbar_init(full + s, 1);
      tc::mbar_init(empty + s, 1);
    }
    tc::mbar_init(tfull, 1);
    tc::mbar_init(tempty, MOE_EPI_WARPS);
    for (int k = 0; k < QD; ++k) {
      tc::mbar_init(qfull + k, 1);
      tc::mbar_init(qempty + k, 2);
    }
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tslot, Cfg::TCOLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;

  struct Unit {
    bool down;
    int c, e, r0, n, f;
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
    return x;
  };
  // the ui-th unit id of this block (n_units when there is none, or on a timeout)
  auto take = [&](int ui) -> int {
    const int k = ui % QD;
    if (!tc::mbar_wait(qfull + k, (ui / QD) & 1, limit_ns)) {
      atomicOr(err, ERR_TIMEOUT);
      return n_units;
    }
    const int u = *reinterpret_cast<volatile int32_t*>(qid + k);
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_addr(qempty + k))
                 : "memory");
    return u;
  };

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
        if (qi >= QD && !tc::mbar_wait(qempty + k, ((qi / QD) & 1) ^ 1, limit_ns)) {
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
          // the chunk's hidden rows are complete once all its phase-1 units have counted
          const uint64_t t0 = tc::global_ns();
          const int need = FT1 + (stall ? 1 : 0);
          while (ld_acquire(ready + x.c) < need) {
            __nanosleep(64);
            if (tc::global_ns() - t0 > limit_ns) {
              atomicOr(err, ERR_TIMEOUT);
              ok = false;
              break;
            }
          }
          if (!ok) continue;  // publish the end of the work next
          asm volatile("fence.proxy.async.global;" ::: "memory");  // before the TMA reads
        }
        const int nk = (x.down ? I : d) / TC_KB;
        const int nb = (x.n + 31) >> 5;
        const uint32_t bytes = 2 * TC_SUB_A + (uint32_t)nb * 32 * TC_KB * 2;
        const int w1 = x.down ? x.e * d + x.f * 256 : x.e * I + x.f * 128;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % ST;
          const uint32_t ph = (it / ST) & 1;
          if (it >= ST && !tc::mbar_wait(empty + s, ph ^ 1, limit_ns)) {
            atomicOr(err, ERR_TIMEOUT);
            ok = false;
            break;
          }
          uint8_t* st = smem + s * Cfg::STAGE;
          // units of one chunk start their K walk at different offsets
          const int kx = ((kb + x.f) % nk) * TC_KB;
          tc::mbar_expect_tx(full + s, bytes);
          if (x.down) {
            tc::tma_load_2d(st, &mWd, full + s, kx, w1);
            tc::tma_load_2d(st + TC_SUB_A, &mWd, full + s, kx, w1 + 128);
          } else {
            tc::tma_load_2d(st, &mWg, full + s, kx, w1);
            tc::tma_load_2d(st + TC_SUB_A, &mWu, full + s, kx, w1);
          }
          uint8_t* bt = st + 2 * TC_SUB_A;
          for (int j = 0; j < nb; ++j)
            tc::tma_load_2d(bt + j * 32 * TC_KB * 2, x.down ? &mH : &mX, full + s, kx,
                            x.r0 + 32 * j);
        }
      }
      if (!tc::drain_slots(full, ST, it, limit_ns)) atomicOr(err, ERR_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int ui = 0; ok; ++ui) {
        const int u = take(ui);
        if (u >= n_units) break;
        const Unit x = unit_of(u);
        const int nk = (x.down ? I : d) / TC_KB;
        const int npad = ((x.n + 31) >> 5) << 5;
        const uint32_t idesc = tc::idesc_bf16(128, npad);
        // wait until the epilogue has drained the previous unit's accumulators
        if (ui > 0 && !tc::mbar_wait(tempty, (ui - 1) & 1, limit_ns)) {
          atomicOr(err, ERR_TIMEOUT);
          break;
        }
        tc::fence_after_sync();
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % ST;
          const uint32_t ph = (it / ST) & 1;
          if (!tc::mbar_wait(full + s, ph, limit_ns)) {
            atomicOr(err, ERR_TIMEOUT);
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t a0 = tc::smem_addr(smem + s * Cfg::STAGE);
          const uint32_t b0 = a0 + 2 * TC_SUB_A;
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
  } else {
    // epilogue warps 2..17 -> TMEM lane quarter (warp % 4), token chunks part, part + 4, ..
    constexpr int NP = MOE_EPI_WARPS / 4;
    const int q = warp & 3, part = (warp - 2) >> 2;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    for (int ui = 0;; ++ui) {
      // warp 2 takes the unit id for the epilogue warps
      if (warp == 2 && lane == 0) *reinterpret_cast<volatile int32_t*>(ubc) = take(ui);
      asm volatile("bar.sync 1, %0;" ::"n"(32 * MOE_EPI_WARPS) : "memory");
      const int u = *reinterpret_cast<volatile int32_t*>(ubc);
      asm volatile("bar.sync 1, %0;" ::"n"(32 * MOE_EPI_WARPS) : "memory");  // read by all before the next take
      if (u >= n_units) break;
      const Unit x = unit_of(u);
      bool rdy = true;
      if (lane == 0) rdy = tc::mbar_wait(tfull, ui & 1, limit_ns);
      rdy = __shfl_sync(0xffffffffu, rdy ? 1 : 0, 0) != 0;
      // on a timeout the warp records it and keeps step with the other epilogue warps
      // (same barriers, no TMEM reads), so that nothing waits forever
      if (!rdy && lane == 0) atomicOr(err, ERR_TIMEOUT);
      tc::fence_after_sync();
      const int nch = rdy ? (x.n + 31) >> 5 : 0;
      if (!x.down) {
        const int fr = x.f * 128 + 32 * q + lane;  // hidden column
#pragma unroll 1
        for (int c = part; c < nch; c += NP) {
          float g[32], v[32];
          tc::tmem_ld32(tmem + lane_base + c * 32, g);
          tc::tmem_ld32(tmem + lane_base + 128 + c * 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = c * 32 + j;
            if (t < x.n) hb[(size_t)(x.r0 + t) * I + fr] = __float2bfloat16_rn(silu(g[j]) * v[j]);
          }
        }
      } else {
#pragma unroll 1
        for (int half2 = 0; half2 < 2; ++half2) {
          const int fr = x.f * 256 + half2 * 128 + 32 * q + lane;  // output column
#pragma unroll 1
          for (int c = part; c < nch; c += NP) {
            float v[32];
            tc::tmem_ld32(tmem + lane_base + half2 * 128 + c * 32, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int t = c * 32 + j;
              if (t < x.n) yb[(size_t)(x.r0 + t) * d + fr] = gate_of[x.r0 + t] * v[j];
            }
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_addr(tempty)) : "memory");
      if (!x.down) {
        // this unit's hidden columns are written: count it for the chunk's phase-2 units
        __threadfence();
        asm volatile("bar.sync 1, %0;" ::"n"(32 * MOE_EPI_WARPS) : "memory");  // the epilogue warps
        if (warp == 2 && lane == 0) atomicAdd(ready + x.c, 1);
      }
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
dg_status tc_router_topk(dg_model* m, const bf16* u2, const void* Wr, int M, int32_t* idx,
                         float* gate, cudaStream_t st);
dg_status tc_gemm_f32_rows(dg_model* m, const bf16* A, int a_rows, const void* W, float* out,
                           int M, int N, int K, cudaStream_t st);
dg_status tc_gemm_add_residual(dg_model* m, const bf16* A, const void* W, float* x, int M, int N,
                               int K, cudaStream_t st);
dg_status tc_gemm_swiglu(dg_model* m, const bf16* A, const void* Wg, const void* Wu, bf16* out,
                         int M, int N, int K, cudaStream_t st);
dg_status tc_moe_experts(dg_model* m, int l, const bf16* X, bf16* hb, float* yb, cudaStream_t st);
dg_status tc_moe_experts_f4(dg_model* m, int l, const bf16* X, bf16* hb, float* yb,
                            cudaStream_t st);
dg_status tc_moe_experts_f8(dg_model* m, int l, const bf16* X, bf16* hb, float* yb,
                            cudaStream_t st);
dg_status tc_lmhead_stats(dg_model* m, const bf16* xn, int M, float* ent, int32_t* amax,
                          cudaStream_t st, const AnnealDev& an = AnnealDev{},
                          int32_t* sampled = nullptr, const ScDev& sc = ScDev{});
// y = p0 E for the n rows the LM head left in the workspace (self-conditioning): a
// K-sliced tcgen05 GEMM against the transposed embedding, partials added in slice order.
dg_status tc_selfcond_mix(dg_model* m, int n, cudaStream_t st);
dg_status tc_attention(dg_model* m, const bf16* q, int B, int nq, int qpos0, const dg_kv* kv,
                       int l, const bf16* kB, const bf16* vB, int nB, int kposB, int npB,
                       bool causal, bf16* out, cudaStream_t st);

}  // namespace dg
