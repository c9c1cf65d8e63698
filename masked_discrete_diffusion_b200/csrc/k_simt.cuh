// CUDA-core kernels of the denoise forward (all precisions).
//
// These carry the whole path for the fp32 tiny model (activations and sums in
// fp64) and every step that is not a dense contraction for the bf16 models.
// The dense contractions of the bf16 models run on tcgen05 (k_tc_gemm.cuh).
//
// Model passages: "DiffusionGemma 技术报告" (full translation page) §3.1-§3.2
// (causal context pass, bidirectional canvas decoder, logits per position);
// explainer page "DiffusionGemma 深度解析", list "核心架构参数" (MoE top-8 of 128
// plus one shared expert, sliding window 1024, timestep embedding).
#pragma once

#include "k_anneal.cuh"
#include "k_common.cuh"
#include "k_selfcond.cuh"

namespace dg {

// ---------------------------------------------------------------------------
// a1: embedding gather (+ sinusoidal timestep embedding for canvas rows)
// x[t, :] = E[ids[t], :] + temb(tau); temb[i] = sin(1000 tau w_i),
// temb[d/2 + i] = cos(1000 tau w_i), w_i = 10000^(-i / (d/2)).  tau < 0: none.
// With s_dev set, tau = *s_dev / T (steps left read from device memory).  With z set
// (self-conditioning), z[t, :] is added as well.
// ---------------------------------------------------------------------------
template <class TW, class TR, class TZ>
__global__ void embed_kernel(const int32_t* __restrict__ ids, const TW* __restrict__ emb,
                             TR* __restrict__ x, int n_tok, int d, int max_id, double tau,
                             int32_t* err, const int32_t* __restrict__ s_dev, int T,
                             const TZ* __restrict__ z) {
  pdl_enter();
  if (s_dev) tau = (double)*s_dev / (double)T;
  const int t = blockIdx.x;
  if (t >= n_tok) return;
  int id = ids[t];
  if (id < 0 || id > max_id) {
    if (threadIdx.x == 0) atomicOr(err, 1);
    id = 0;
  }
  const TW* row = emb + (size_t)id * d;
  const int half = d / 2;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    double v = (double)widen(row[c]);
    if (tau >= 0.0) {
      const int i = c < half ? c : c - half;
      const double w = pow(10000.0, -(double)i / (double)half);
      const double a = 1000.0 * tau * w;
      v += c < half ? sin(a) : cos(a);
    }
    if (z) v += (double)z[(size_t)t * d + c];
    x[(size_t)t * d + c] = narrow<TR>(v);
  }
}

// ---------------------------------------------------------------------------
// RMSNorm, gain 1: y = x / sqrt(mean(x^2) + eps)
// Optional u2 [n, 2d]: the two-term split of u = x / rms into y (first d
// columns) and lo = narrow(u - y) (last d columns); y + lo carries u to about
// twice the precision of TA, so that a TA x TA contraction of [y | lo] against
// [w | w] reproduces u . w at nearly fp32 accuracy (router logits on tensor cores).
// ---------------------------------------------------------------------------
template <class TR, class TA, class Acc>
__global__ void rmsnorm_kernel(const TR* __restrict__ x, TA* __restrict__ y, int n, int d,
                               float eps, Acc* __restrict__ inv_out = nullptr,
                               TA* __restrict__ u2 = nullptr) {
  pdl_enter();
  __shared__ Acc red[32];
  const int t = blockIdx.x;
  if (t >= n) return;
  const TR* r = x + (size_t)t * d;
  Acc ss = 0;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    Acc v = (Acc)widen(r[c]);
    ss += v * v;
  }
  ss = block_sum(ss, red);
  const Acc inv = Acc(1) / dsqrt(ss / (Acc)d + (Acc)eps);
  if (inv_out && threadIdx.x == 0) inv_out[t] = inv;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const Acc u = (Acc)widen(r[c]) * inv;
    const TA hi = narrow<TA>(u);
    y[(size_t)t * d + c] = hi;
    if (u2) {
      u2[(size_t)t * 2 * d + c] = hi;
      u2[(size_t)t * 2 * d + d + c] = narrow<TA>(u - (Acc)widen(hi));
    }
  }
}

// ---------------------------------------------------------------------------
// Tiled CUDA-core GEMM  C[M, N] = A[M, K] W[N, K]^T with an epilogue functor.
// GROUPED: blockIdx.y walks a tile table (expert e, first permuted row m0);
// rows [m0, min(m0 + 64, offsets[e + 1])) use weight slab W + e * w_slab.
// DUAL: a second weight W2 is accumulated alongside (gate and up projections).
// ---------------------------------------------------------------------------
struct GroupInfo {
  const int32_t* tile_e = nullptr;
  const int32_t* tile_m0 = nullptr;
  const int32_t* n_tiles = nullptr;
  const int32_t* offsets = nullptr;
  size_t w_slab = 0;
};

constexpr int SG_BM = 64, SG_BN = 64, SG_BK = 16;

template <class TA, class TW, class Acc, bool GROUPED, bool DUAL, class Epi>
__global__ void __launch_bounds__(256)
    gemm_simt_kernel(const TA* __restrict__ A, int lda, const TW* __restrict__ W,
                     const TW* __restrict__ W2, int ldw, int M, int N, int K, GroupInfo g,
                     Epi epi) {
  pdl_enter();
  __shared__ Acc As[SG_BK][SG_BM + 1];
  __shared__ Acc Ws[SG_BK][SG_BN + 1];
  __shared__ Acc Ws2[DUAL ? SG_BK : 1][DUAL ? SG_BN + 1 : 1];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int n0 = blockIdx.x * SG_BN;
  int m0 = blockIdx.y * SG_BM, m_end = M;
  int e = 0;
  if (GROUPED) {
    if ((int)blockIdx.y >= *g.n_tiles) return;
    e = g.tile_e[blockIdx.y];
    m0 = g.tile_m0[blockIdx.y];
    m_end = g.offsets[e + 1];
    W += (size_t)e * g.w_slab;
    if (DUAL) W2 += (size_t)e * g.w_slab;
  }
  const int m_lim = min(m0 + SG_BM, m_end);
  Acc acc[4][4], acc2[DUAL ? 4 : 1][DUAL ? 4 : 1];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc[i][j] = 0;
      if (DUAL) acc2[DUAL ? i : 0][DUAL ? j : 0] = 0;
    }
  for (int k0 = 0; k0 < K; k0 += SG_BK) {
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int el = tid + it * 256, r = el >> 4, kk = el & 15;
      const int gm = m0 + r, gk = k0 + kk, gn = n0 + r;
      As[kk][r] = (gm < m_lim && gk < K) ? (Acc)widen(A[(size_t)gm * lda + gk]) : Acc(0);
      Ws[kk][r] = (gn < N && gk < K) ? (Acc)widen(W[(size_t)gn * ldw + gk]) : Acc(0);
      if (DUAL)
        Ws2[DUAL ? kk : 0][DUAL ? r : 0] =
            (gn < N && gk < K) ? (Acc)widen(W2[(size_t)gn * ldw + gk]) : Acc(0);
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      Acc a[4], b[4], b2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b[j] = Ws[kk][tx + 16 * j];
        if (DUAL) b2[j] = Ws2[DUAL ? kk : 0][DUAL ? tx + 16 * j : 0];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] += a[i] * b[j];
          if (DUAL) acc2[DUAL ? i : 0][DUAL ? j : 0] += a[i] * b2[j];
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = m0 + ty + 16 * i, c = n0 + tx + 16 * j;
      if (r < m_lim && c < N) {
        if (DUAL)
          epi(r, c, acc[i][j], acc2[DUAL ? i : 0][DUAL ? j : 0]);
        else
          epi(r, c, acc[i][j], acc[i][j]);
      }
    }
}

template <class TO, class Acc> struct EpiStore {
  TO* out;
  int ldo;
  __device__ void operator()(int r, int c, Acc v, Acc) const {
    out[(size_t)r * ldo + c] = narrow<TO>(v);
  }
};

template <class TR, class Acc> struct EpiAddResidual {
  TR* res;
  int ldr;
  __device__ void operator()(int r, int c, Acc v, Acc) const {
    TR* p = res + (size_t)r * ldr + c;
    *p = narrow<TR>((Acc)widen(*p) + v);
  }
};

template <class TO, class Acc> struct EpiSwiglu {
  TO* out;
  int ldo;
  __device__ void operator()(int r, int c, Acc g, Acc u) const {
    out[(size_t)r * ldo + c] = narrow<TO>(silu(g) * u);
  }
};

template <class TO, class Acc> struct EpiRowScale {
  TO* out;
  int ldo;
  const Acc* scale;
  __device__ void operator()(int r, int c, Acc v, Acc) const {
    out[(size_t)r * ldo + c] = narrow<TO>(scale[r] * v);
  }
};

// ---------------------------------------------------------------------------
// a2 (RoPE part): rotate q and k of the raw projection, scatter q / k / v.
// qkv: [n_tok, (Hq + 2 Hkv) h] raw projections.  Token t = b * n_seq + i sits at
// absolute position pos0 + i.  q -> q_out [n_tok, Hq, h]; k -> kc [b, Hkv, np, h];
// v -> vc transposed [b, Hkv, h, np] (np >= n_seq, padded).
// Pair (j, j + h/2) rotates by pos*theta_j.
// rope: [max_pos, h/2] cos values followed by [max_pos, h/2] sin values.
// ---------------------------------------------------------------------------
template <class Acc, class TA, class TKV>
__global__ void rope_scatter_kernel(const Acc* __restrict__ qkv, TA* __restrict__ q_out,
                                    TKV* __restrict__ kc, TKV* __restrict__ vc, int n_tok,
                                    int n_seq, int np, int pos0, int Hq, int Hkv, int h,
                                    const Acc* __restrict__ rope, int max_pos) {
  pdl_enter();
  const int t = blockIdx.x;
  if (t >= n_tok) return;
  const int b = t / n_seq, i = t % n_seq, pos = pos0 + i;
  const int half = h / 2, heads = Hq + 2 * Hkv;
  const Acc* row = qkv + (size_t)t * heads * h;
  const Acc* cs = rope + (size_t)pos * half;
  const Acc* sn = rope + (size_t)max_pos * half + (size_t)pos * half;
  for (int e = threadIdx.x; e < heads * half; e += blockDim.x) {
    const int hd = e / half, j = e % half;
    const Acc x1 = row[hd * h + j], x2 = row[hd * h + j + half];
    if (hd < Hq + Hkv) {
      const Acc c = cs[j], s = sn[j];
      const Acc y1 = x1 * c - x2 * s, y2 = x2 * c + x1 * s;
      if (hd < Hq) {
        TA* qo = q_out + ((size_t)t * Hq + hd) * h;
        qo[j] = narrow<TA>(y1);
        qo[j + half] = narrow<TA>(y2);
      } else {
        TKV* ko = kc + (((size_t)b * Hkv + (hd - Hq)) * np + i) * h;
        ko[j] = narrow<TKV>(y1);
        ko[j + half] = narrow<TKV>(y2);
      }
    } else {
      TKV* vo = vc + ((size_t)b * Hkv + (hd - Hq - Hkv)) * h * np + i;
      vo[(size_t)j * np] = narrow<TKV>(x1);
      vo[(size_t)(j + half) * np] = narrow<TKV>(x2);
    }
  }
}

// ---------------------------------------------------------------------------
// a3: attention, one warp per (batch b, query i, query head j).
// Keys: segment A (the cached prompt window, nA keys, absolute positions
// kposA..) followed by segment B (the pass's own keys, nB keys at kposB..).
// causal != 0: key at position p is visible to the query at position qp iff
// qp - window < p <= qp; otherwise every key is visible.  One online softmax
// over both segments; scores scaled by 1/sqrt(h).  DPL = ceil(h / 32).
// K layout [b, Hkv, n_pad, h]; V transposed [b, Hkv, h, n_pad]; q/o: [b * nq + i, Hq, h].
// ---------------------------------------------------------------------------
template <class TA, class TKV, class Acc, int DPL>
__global__ void attention_simt_kernel(const TA* __restrict__ q, TA* __restrict__ o,
                                      const TKV* __restrict__ kA, const TKV* __restrict__ vA,
                                      int nA, int padA, int kposA, const TKV* __restrict__ kB,
                                      const TKV* __restrict__ vB, int nB, int padB, int kposB, int B,
                                      int nq, int qpos0, int Hq, int Hkv, int h, int causal,
                                      int window) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const long wid = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long total = (long)B * nq * Hq;
  if (wid >= total) return;
  const int j = (int)(wid % Hq);
  const long ti = wid / Hq;  // b * nq + i
  const int b = (int)(ti / nq), i = (int)(ti % nq);
  const int kvh = j / (Hq / Hkv);
  const int qp = qpos0 + i;
  const Acc scale = Acc(1) / dsqrt((Acc)h);
  Acc qv[DPL], acc[DPL];
  const TA* qrow = q + ((size_t)ti * Hq + j) * h;
#pragma unroll
  for (int u = 0; u < DPL; ++u) {
    const int dd = lane + 32 * u;
    qv[u] = dd < h ? (Acc)widen(qrow[dd]) * scale : Acc(0);
    acc[u] = 0;
  }
  Acc mrun = -INFINITY, lrun = 0;
  for (int seg = 0; seg < 2; ++seg) {
    const TKV* K = seg == 0 ? kA : kB;
    const TKV* V = seg == 0 ? vA : vB;
    const int n = seg == 0 ? nA : nB;
    const int npad = seg == 0 ? padA : padB;
    const int p0 = seg == 0 ? kposA : kposB;
    if (n == 0 || K == nullptr) continue;
    const size_t base = ((size_t)b * Hkv + kvh) * npad * h;
    int lo = 0, hi = n;
    if (causal) {
      lo = max(0, qp - window + 1 - p0);
      hi = min(n, qp - p0 + 1);
    }
    for (int t = lo; t < hi; ++t) {
      const TKV* kr = K + base + (size_t)t * h;
      Acc s = 0;
#pragma unroll
      for (int u = 0; u < DPL; ++u) {
        const int dd = lane + 32 * u;
        if (dd < h) s += qv[u] * (Acc)widen(kr[dd]);
      }
      s = warp_sum(s);
      const Acc mnew = max(mrun, s);
      const Acc corr = dexp(mrun - mnew), pexp = dexp(s - mnew);
      lrun = lrun * corr + pexp;
      const TKV* vr = V + base + t;
#pragma unroll
      for (int u = 0; u < DPL; ++u) {
        const int dd = lane + 32 * u;
        if (dd < h) acc[u] = acc[u] * corr + pexp * (Acc)widen(vr[(size_t)dd * npad]);
      }
      mrun = mnew;
    }
  }
  TA* orow = o + ((size_t)ti * Hq + j) * h;
  const Acc inv = Acc(1) / lrun;
#pragma unroll
  for (int u = 0; u < DPL; ++u) {
    const int dd = lane + 32 * u;
    if (dd < h) orow[dd] = narrow<TA>(acc[u] * inv);
  }
}

// ---------------------------------------------------------------------------
// a5: router.  logits = RMSNorm(x) Wr^T computed at the accumulation precision
// from the residual: router_logits_kernel forms split-K partial dot products
// x . w (tile of 32 tokens x 128 experts per CTA, K range per blockIdx.y);
// router_topk_kernel (one warp per token) sums the splits in a fixed order,
// scales by the row's 1/rms, takes the softmax over all E experts, the top-k by
// probability (ties -> lower expert id) and renormalises the k gates.
// ---------------------------------------------------------------------------
template <class TR, class TW, class Acc>
__global__ void __launch_bounds__(256)
    router_logits_kernel(const TR* __restrict__ x, const TW* __restrict__ wr, int n, int d, int E,
                         int k_per_split, Acc* __restrict__ part) {
  pdl_enter();
  __shared__ Acc Xs[32][33];
  __shared__ Acc Ws[32][129];
  const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;
  const int t0 = blockIdx.x * 32, e0 = blockIdx.z * 128;
  const int k_lo = blockIdx.y * k_per_split, k_hi = min(d, k_lo + k_per_split);
  Acc acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0;
  for (int k0 = k_lo; k0 < k_hi; k0 += 32) {
#pragma unroll
    for (int it = 0; it < 4; ++it) {  // x tile: 32 tokens x 32 k
      const int el = tid + it * 256, r = el >> 5, kk = el & 31;
      const int gt = t0 + r, gk = k0 + kk;
      Xs[kk][r] = (gt < n && gk < k_hi) ? (Acc)widen(x[(size_t)gt * d + gk]) : Acc(0);
    }
#pragma unroll
    for (int it = 0; it < 16; ++it) {  // w tile: 128 experts x 32 k
      const int el = tid + it * 256, r = el >> 5, kk = el & 31;
      const int ge = e0 + r, gk = k0 + kk;
      Ws[kk][r] = (ge < E && gk < k_hi) ? (Acc)widen(wr[(size_t)ge * d + gk]) : Acc(0);
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      Acc a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Xs[kk][ty + 8 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Ws[kk][tx + 32 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += a[i] * b[j];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + ty + 8 * i, e = e0 + tx + 32 * j;
      if (t < n && e < E) part[((size_t)blockIdx.y * n + t) * E + e] = acc[i][j];
    }
}

template <class Acc, int MAXE>  // MAXE experts per lane: E <= 32 * MAXE
__global__ void router_topk_kernel(const Acc* __restrict__ part, int splits,
                                   const Acc* __restrict__ inv_rms, int n, int E, int top_k,
                                   int32_t* __restrict__ idx, Acc* __restrict__ gate,
                                   int32_t* __restrict__ load) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= n) return;
  Acc pr[MAXE];
  const Acc inv = inv_rms[t];
  Acc mx = -INFINITY;
#pragma unroll
  for (int q = 0; q < MAXE; ++q) {
    const int e = lane + 32 * q;
    pr[q] = -INFINITY;
    if (e < E) {
      Acc s = 0;
      for (int z = 0; z < splits; ++z) s += part[((size_t)z * n + t) * E + e];
      pr[q] = s * inv;
      mx = max(mx, pr[q]);
    }
  }
  mx = warp_max(mx);
  Acc z = 0;
#pragma unroll
  for (int q = 0; q < MAXE; ++q) {
    const int e = lane + 32 * q;
    pr[q] = e < E ? dexp(pr[q] - mx) : Acc(0);
    z += pr[q];
  }
  z = warp_sum(z);
#pragma unroll
  for (int q = 0; q < MAXE; ++q) pr[q] /= z;
  unsigned taken = 0;  // bit q: expert lane + 32 q already selected
  Acc gsum = 0;
  int my_e = 0;   // lane k keeps the k-th selection
  Acc my_p = 0;
  for (int k = 0; k < top_k; ++k) {
    Acc bp = -1;
    int be = 0x7fffffff;
#pragma unroll
    for (int q = 0; q < MAXE; ++q) {
      const int e = lane + 32 * q;
      if (e < E && !((taken >> q) & 1u) && (pr[q] > bp || (pr[q] == bp && e < be))) {
        bp = pr[q];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const Acc op = __shfl_xor_sync(0xffffffffu, bp, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (op > bp || (op == bp && oe < be)) {
        bp = op;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == k) {
      my_e = be;
      my_p = bp;
    }
    gsum += bp;
  }
  if (lane < top_k) {
    idx[(size_t)t * top_k + lane] = my_e;
    gate[(size_t)t * top_k + lane] = my_p / gsum;
    if (load) atomicAdd(&load[my_e], 1);
  }
}

// The whole permutation of the (token, slot) entries into expert-contiguous rows,
// by one block (any multiple of 32 threads <= 1024): ranks by warp-level match
// plus per-(warp, expert) counts scanned in warp order (entry order is kept within
// an expert), counts, offsets, the tile table (bm rows per tile), the
// streamed-expert counter, per-expert load, and the scatter of (row, token, gate).
// Shared memory `psm`: (32 + 1) * E + 2 * blockDim.x ints.  rank [n_entries] and
// tok [n_entries] (the token of every permuted row) are the caller's (shared or
// global memory); `write` selects the block that stores the permutation.
struct PermuteArgs {
  const int32_t* idx;
  int n_entries, top_k, E, bm;
  int32_t *rank, *offsets, *tile_e, *tile_m0, *n_tiles;
  int max_tiles;
  unsigned long long* used;
  int32_t *load, *row_of, *tok_of;
  int32_t* ready;  // per-tile counters of the routed-expert kernel and, after them, its
                   // unit counter; all zeroed here (nullable)
};

template <class Acc>
__device__ void block_permute(const PermuteArgs& a, const Acc* __restrict__ gate,
                              Acc* __restrict__ gate_of, int* psm, int* rank, int* tok,
                              bool write) {
  const int E = a.E, nthr = blockDim.x, nw = nthr >> 5;
  int* hist = psm;             // [nw][E]: counts, then exclusive offsets per warp
  int* carry = psm + 32 * E;   // [E]: entries of each expert in earlier chunks, then offsets
  int* sc = carry + E;         // [nthr] scan scratch (entries)
  int* stl = sc + nthr;        // [nthr] scan scratch (tiles)
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int e = tid; e < E; e += nthr) carry[e] = 0;
  for (int base = 0; base < a.n_entries; base += nthr) {
    for (int i = tid; i < nw * E; i += nthr) hist[i] = 0;
    __syncthreads();
    const int j = base + tid;
    const bool valid = j < a.n_entries;
    const int e = valid ? __ldcg(a.idx + j) : -1;  // written by other blocks: read at L2
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int before = __popc(same & ((1u << lane) - 1u));
    if (valid && before == 0) hist[w * E + e] = __popc(same);
    __syncthreads();
    for (int e2 = tid; e2 < E; e2 += nthr) {
      int s0 = carry[e2];
      for (int w2 = 0; w2 < nw; ++w2) {
        const int c = hist[w2 * E + e2];
        hist[w2 * E + e2] = s0;
        s0 += c;
      }
      carry[e2] = s0;
    }
    __syncthreads();
    if (valid) rank[j] = hist[w * E + e] + before;
    __syncthreads();
  }
  // counts -> offsets and tile table: thread t scans experts [t * per, t * per + per)
  const int per = (E + nthr - 1) / nthr, e0 = tid * per;
  int c_sum = 0, t_sum = 0, used_n = 0;
  for (int e = e0; e < min(E, e0 + per); ++e) {
    const int c = carry[e];
    c_sum += c;
    t_sum += (c + a.bm - 1) / a.bm;
    used_n += c > 0;
    if (write && a.load) a.load[e] += c;
  }
  if (write && a.used && used_n) atomicAdd(a.used, (unsigned long long)used_n);
  sc[tid] = c_sum;
  stl[tid] = t_sum;
  __syncthreads();
  for (int off = 1; off < nthr; off <<= 1) {  // inclusive scans over the threads
    const int x = tid >= off ? sc[tid - off] : 0, y = tid >= off ? stl[tid - off] : 0;
    __syncthreads();
    sc[tid] += x;
    stl[tid] += y;
    __syncthreads();
  }
  int off_e = sc[tid] - c_sum, t_e = stl[tid] - t_sum;
  for (int e = e0; e < min(E, e0 + per); ++e) {
    const int c = carry[e], nt = (c + a.bm - 1) / a.bm;
    carry[e] = off_e;
    if (write) {
      a.offsets[e] = off_e;
      for (int r = 0; r < nt; ++r)
        if (t_e + r < a.max_tiles) {
          a.tile_e[t_e + r] = e;
          a.tile_m0[t_e + r] = off_e + r * a.bm;
        }
    }
    off_e += c;
    t_e += nt;
  }
  if (write && tid == nthr - 1) {
    a.offsets[E] = sc[tid];
    *a.n_tiles = min(stl[tid], a.max_tiles);
  }
  if (write && a.ready)
    for (int t = tid; t <= a.max_tiles; t += nthr) a.ready[t] = 0;  // and the unit counter
  __syncthreads();
  for (int j = tid; j < a.n_entries; j += nthr) {
    const int pos = carry[__ldcg(a.idx + j)] + rank[j];
    tok[pos] = j / a.top_k;
    if (write) {
      a.row_of[j] = pos;
      a.tok_of[pos] = j / a.top_k;
      gate_of[pos] = __ldcg(gate + j);
    }
  }
  __syncthreads();
}

inline size_t permute_smem_bytes(int E, int threads, int n_entries_in_smem) {
  return ((size_t)33 * E + 2 * (size_t)threads + 2 * (size_t)n_entries_in_smem) * sizeof(int);
}

// The permutation alone (one block; rank scratch and tok_of in global memory), for
// entry counts whose ranks do not fit in shared memory.
template <class Acc>
__global__ void __launch_bounds__(1024)
    moe_permute_kernel(PermuteArgs a, const Acc* __restrict__ gate, Acc* __restrict__ gate_of) {
  pdl_enter();
  extern __shared__ int psm[];
  block_permute(a, gate, gate_of, psm, a.rank, a.tok_of, true);
}

// Permutation and gather in one launch: every block derives the permutation (so that
// no block waits for another), block 0 stores it, and block z copies its share of
// the permuted rows dst[r] = src[token of row r] (rows of d elements, 16-byte units).
template <class Acc, class TA>
__global__ void __launch_bounds__(1024)
    moe_permute_gather_kernel(PermuteArgs a, const Acc* __restrict__ gate,
                              Acc* __restrict__ gate_of, const TA* __restrict__ src, int d,
                              TA* __restrict__ dst) {
  pdl_enter();
  extern __shared__ int psm[];
  int* rank = psm + 33 * a.E + 2 * blockDim.x;
  int* tok = rank + a.n_entries;
  block_permute(a, gate, gate_of, psm, rank, tok, blockIdx.x == 0);
  const int units = d * (int)sizeof(TA) / 16;  // 16-byte units per row
  const int per = (a.n_entries + gridDim.x - 1) / gridDim.x;
  const int r0 = blockIdx.x * per, r1 = min(a.n_entries, r0 + per);
  for (long u = threadIdx.x; u < (long)(r1 - r0) * units; u += blockDim.x) {
    const int r = r0 + (int)(u / units), c = (int)(u % units);
    reinterpret_cast<uint4*>(dst + (size_t)r * d)[c] =
        reinterpret_cast<const uint4*>(src + (size_t)tok[r] * d)[c];
  }
}

template <class TA>
__global__ void gather_rows_kernel(const TA* __restrict__ src, const int32_t* __restrict__ tok_of,
                                   const int32_t* __restrict__ n_rows_dev, int d,
                                   TA* __restrict__ dst) {
  pdl_enter();
  const int r = blockIdx.x;
  if (r >= *n_rows_dev) return;
  const TA* s = src + (size_t)tok_of[r] * d;
  TA* o = dst + (size_t)r * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) o[c] = s[c];
}

// Combine fused with the next RMSNorm: x[t] += ys[t] + sum over slots of
// yb[row_of[t * k + slot]] (slot order fixed), then y[t] = RMSNorm(x[t]).
// One block per token; each thread owns 8 consecutive columns (d % 8 == 0) and
// issues the loads of all slots before summing.
template <class TR, class TA, class TY, class Acc>
__global__ void moe_combine_norm_kernel(TR* __restrict__ x, const TY* __restrict__ ys,
                                        const TY* __restrict__ yb,
                                        const int32_t* __restrict__ row_of, int n_tok, int d,
                                        int top_k, float eps, TA* __restrict__ y) {
  pdl_enter();
  constexpr int KB = 8;  // slots loaded together
  __shared__ Acc red[32];
  __shared__ int rows[64];
  const int t = blockIdx.x;
  if (t >= n_tok) return;
  for (int k = threadIdx.x; k < top_k; k += blockDim.x) rows[k] = row_of[(size_t)t * top_k + k];
  __syncthreads();
  TR* xr = x + (size_t)t * d;
  Acc ss = 0;
  // rows are 16-byte aligned (d % 8 == 0): every access moves 8 columns at once; the
  // sums keep their order (shared expert, then the slots in k order, then the residual)
  TR keep[8];  // the thread's first column group, kept for the norm pass
  int g = 0;
  for (int c0 = threadIdx.x * 8; c0 < d; c0 += blockDim.x * 8, ++g) {
    Acc v[8];
    {
      TY a[8];
      ld8(ys + (size_t)t * d + c0, a);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = (Acc)widen(a[j]);
    }
    for (int k0 = 0; k0 < top_k; k0 += KB) {
      TY u[KB][8];
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        if (k0 + k < top_k) {
          ld8(yb + (size_t)rows[k0 + k] * d + c0, u[k]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) u[k][j] = TY(0);
        }
      }
#pragma unroll
      for (int k = 0; k < KB; ++k)
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] += (Acc)widen(u[k][j]);
    }
    TR xo[8], nx[8];
    ld8(xr + c0, xo);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      nx[j] = narrow<TR>((Acc)widen(xo[j]) + v[j]);
      const Acc a = (Acc)widen(nx[j]);
      ss += a * a;
    }
    st8(xr + c0, nx);
    if (g == 0) {
#pragma unroll
      for (int j = 0; j < 8; ++j) keep[j] = nx[j];
    }
  }
  ss = block_sum(ss, red);
  const Acc inv = Acc(1) / dsqrt(ss / (Acc)d + (Acc)eps);
  g = 0;
  for (int c0 = threadIdx.x * 8; c0 < d; c0 += blockDim.x * 8, ++g) {
    TR xv[8];
    if (g == 0) {
#pragma unroll
      for (int j = 0; j < 8; ++j) xv[j] = keep[j];
    } else {
      ld8(xr + c0, xv);
    }
    TA o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] = narrow<TA>((Acc)widen(xv[j]) * inv);
    if constexpr ((sizeof(TA) * 8) % 16 == 0) {
      st8(y + (size_t)t * d + c0, o);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) y[(size_t)t * d + c0 + j] = o[j];
    }
  }
}

// ---------------------------------------------------------------------------
// a8 (CUDA-core form): logits tile = scale * xn W_lm^T for 64 rows x 64 vocab
// entries, reduced per row to partial statistics over the tile:
//   m = max logit, s = sum exp(l - m), u = sum exp(l - m) (l - m), a = argmax
// (lowest id among equal maxima).  Partials: [n_vtiles, n_rows, 4].
// Optional logits output [n_rows, V] (test hook).  With an.N > 0 the logits are
// tempered (l = scale acc / tau) and, with an.seeds, each row's winner of the tile's
// Gumbel-max race goes to an.gpart [n_vtiles, n_rows, 2] = (l / tau - log E, id).
// ---------------------------------------------------------------------------
template <class TA, class TW, class Acc>
__global__ void __launch_bounds__(256)
    lmhead_simt_kernel(const TA* __restrict__ xn, const TW* __restrict__ wlm, int n_rows, int V,
                       int d, float scale, Acc* __restrict__ part, float* __restrict__ logits,
                       AnnealDev an, ScDev sc) {
  pdl_enter();
  const Acc tau = an.N > 0 ? (Acc)an.tau() : Acc(1);
  // the logits tile T reuses the operand staging buffers once the K loop is done
  constexpr int kStage = 2 * SG_BK * (SG_BM + 1), kTile = SG_BM * (SG_BN + 1);
  __shared__ Acc smem[kStage > kTile ? kStage : kTile];
  Acc(*As)[SG_BM + 1] = reinterpret_cast<Acc(*)[SG_BM + 1]>(smem);
  Acc(*Ws)[SG_BN + 1] = reinterpret_cast<Acc(*)[SG_BN + 1]>(smem + SG_BK * (SG_BM + 1));
  Acc(*T)[SG_BN + 1] = reinterpret_cast<Acc(*)[SG_BN + 1]>(smem);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int n0 = blockIdx.x * SG_BN, m0 = blockIdx.y * SG_BM;
  Acc acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0;
  for (int k0 = 0; k0 < d; k0 += SG_BK) {
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int el = tid + it * 256, r = el >> 4, kk = el & 15;
      const int gm = m0 + r, gk = k0 + kk, gn = n0 + r;
      As[kk][r] = (gm < n_rows && gk < d) ? (Acc)widen(xn[(size_t)gm * d + gk]) : Acc(0);
      Ws[kk][r] = (gn < V && gk < d) ? (Acc)widen(wlm[(size_t)gn * d + gk]) : Acc(0);
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      Acc a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Ws[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += a[i] * b[j];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      Acc l = (Acc)scale * acc[i][j];
      if (an.N > 0) l = l / tau;
      T[ty + 16 * i][tx + 16 * j] = l;
      const int r = m0 + ty + 16 * i, c = n0 + tx + 16 * j;
      if (logits && r < n_rows && c < V) logits[(size_t)r * V + c] = (float)l;
    }
  __syncthreads();
  const int lane = tid & 31, wid = tid >> 5;
  for (int rr = wid; rr < SG_BM; rr += 8) {
    const int r = m0 + rr;
    if (r >= n_rows) continue;
    Acc mx = -INFINITY;
    int am = 0x7fffffff;
    for (int c = lane; c < SG_BN; c += 32) {
      if (n0 + c >= V) continue;
      const Acc l = T[rr][c];
      if (l > mx || (l == mx && n0 + c < am)) {
        mx = l;
        am = n0 + c;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const Acc om = __shfl_xor_sync(0xffffffffu, mx, off);
      const int oa = __shfl_xor_sync(0xffffffffu, am, off);
      if (om > mx || (om == mx && oa < am)) {
        mx = om;
        am = oa;
      }
    }
    Acc s = 0, u = 0;
    for (int c = lane; c < SG_BN; c += 32) {
      if (n0 + c >= V) continue;
      const Acc z = T[rr][c] - mx, e = dexp(z);
      s += e;
      u += e * z;
    }
    s = warp_sum(s);
    u = warp_sum(u);
    if (lane == 0) {
      Acc* pp = part + ((size_t)blockIdx.x * n_rows + r) * 4;
      pp[0] = mx;
      pp[1] = s;
      pp[2] = u;
      pp[3] = (Acc)am;
    }
    if (sc.P) {  // self-conditioning: exp(l1 - ref) at temperature 1, ref = the tile's max
      TA* prow = reinterpret_cast<TA*>(sc.P) + (size_t)r * sc.ldp;
      Acc p = 0;
      for (int c = lane; c < SG_BN; c += 32) {
        if (n0 + c >= V) continue;
        const Acc q = dexp((T[rr][c] - mx) * tau);
        prow[n0 + c] = narrow<TA>(q);
        p += q;
      }
      p = warp_sum(p);
      if (lane == 0) {
        Acc* rp = reinterpret_cast<Acc*>(sc.ref) + ((size_t)blockIdx.x * n_rows + r) * 2;
        rp[0] = mx * tau;
        rp[1] = p;
      }
    }
    if (an.seeds) {  // this tile's winner of the race, lane by lane then across the warp
      GumbelBest<Acc> gb;
      const unsigned long long st = an.pair_state(r, V, 0);
      for (int c = lane; c < SG_BN; c += 32) {
        const int col = n0 + c;
        if (col >= V) continue;
        const Acc z = T[rr][c] - mx;
        const unsigned long long zz = sm64_mix(st + (unsigned long long)(col >> 1) * SM64_G);
        gb.offer(dexp(z), sm64_expo(sm64_field(zz, col & 1), Acc(0)), z, col);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const Acc oe = __shfl_xor_sync(0xffffffffu, gb.e, off);
        const Acc oE = __shfl_xor_sync(0xffffffffu, gb.E, off);
        const Acc oz = __shfl_xor_sync(0xffffffffu, gb.z, off);
        const int oi = __shfl_xor_sync(0xffffffffu, gb.id, off);
        gb.offer(oe, oE, oz, oi);
      }
      if (lane == 0) {
        Acc* gp = reinterpret_cast<Acc*>(an.gpart) + ((size_t)blockIdx.x * n_rows + r) * 2;
        gp[0] = gb.value(mx);
        gp[1] = (Acc)gb.id;
      }
    }
  }
}

// Merge of per-tile statistics (fixed order and shape), one warp per row:
//   M = max m_i, S = sum s_i e^(m_i - M),
//   H = log S - (1/S) sum e^(m_i - M) (u_i + (m_i - M) s_i)   (clamped at 0),
//   argmax = the id of the first tile (lowest vocab) attaining M.
//   sampled (with gpart) = the id of the best (value, lowest id) race winner over tiles;
//   with sc.P: each tile's factor exp(ref_t - M) / S (M = max ref_t,
//   S = sum_t s_t exp(ref_t - M)) replaces ref_t, for selfcond_scale_kernel.
template <class Acc, class TP>
__global__ void __launch_bounds__(128)
    lm_merge_kernel(const Acc* __restrict__ part, int n_vt, int n_rows, float* __restrict__ H,
                    int32_t* __restrict__ amax, const Acc* __restrict__ gpart,
                    int32_t* __restrict__ sampled, ScDev sc) {
  // one block per row; the tiles are split over the threads, each thread merges
  // its tiles online (running max M_t; S and U rescaled when M_t rises), then the
  // block merges the threads in a fixed order
  pdl_enter();
  __shared__ Acc sm_m[128], sm_s[128], sm_u[128], sm_i[128];
  const int r = blockIdx.x, tid = threadIdx.x;
  if (r >= n_rows) return;
  Acc M = -INFINITY, S = 0, U = 0, id = 0;
  for (int i0 = tid; i0 < n_vt; i0 += 4 * blockDim.x) {
    Acc pm[4], ps[4], pu[4], pi[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // independent loads first
      const int i = i0 + q * blockDim.x;
      if (i < n_vt) {
        const Acc* p = part + ((size_t)i * n_rows + r) * 4;
        pm[q] = p[0];
        ps[q] = p[1];
        pu[q] = p[2];
        pi[q] = p[3];
      } else {
        pm[q] = -INFINITY;
        ps[q] = pu[q] = pi[q] = 0;
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (!(pm[q] > -INFINITY)) continue;
      if (pm[q] > M) {  // tiles come in increasing id order per thread: ties keep the first
        const Acc w = dexp(M - pm[q]);
        U = w * (U + (M - pm[q]) * S);
        S = w * S;
        if (!(M > -INFINITY)) U = S = 0;
        M = pm[q];
        id = pi[q];
      }
      const Acc w = dexp(pm[q] - M);
      S += ps[q] * w;
      U += w * (pu[q] + (pm[q] - M) * ps[q]);
    }
  }
  sm_m[tid] = M;
  sm_s[tid] = S;
  sm_u[tid] = U;
  sm_i[tid] = id;
  __syncthreads();
  if (tid < 32) {
    // lane l merges threads l, l + 32, ... in order, then a fixed butterfly
    Acc m2 = -INFINITY, s2 = 0, u2 = 0, i2 = 0;
    for (int t = tid; t < blockDim.x; t += 32) {
      const Acc mt = sm_m[t];
      if (!(mt > -INFINITY)) continue;
      if (mt > m2 || (mt == m2 && sm_i[t] < i2)) {
        if (mt > m2) {
          const Acc w = dexp(m2 - mt);
          u2 = (m2 > -INFINITY) ? w * (u2 + (m2 - mt) * s2) : Acc(0);
          s2 = (m2 > -INFINITY) ? w * s2 : Acc(0);
          m2 = mt;
        }
        i2 = sm_i[t];
      }
      const Acc w = dexp(mt - m2);
      s2 += sm_s[t] * w;
      u2 += w * (sm_u[t] + (mt - m2) * sm_s[t]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const Acc om = __shfl_xor_sync(0xffffffffu, m2, off);
      const Acc os = __shfl_xor_sync(0xffffffffu, s2, off);
      const Acc ou = __shfl_xor_sync(0xffffffffu, u2, off);
      const Acc oi = __shfl_xor_sync(0xffffffffu, i2, off);
      const Acc mm = om > m2 ? om : m2;
      if (mm > -INFINITY) {
        const Acc wa = dexp(m2 - mm), wb = dexp(om - mm);
        const Acc sa = m2 > -INFINITY ? s2 : Acc(0), sb = om > -INFINITY ? os : Acc(0);
        const Acc ua = m2 > -INFINITY ? wa * (u2 + (m2 - mm) * s2) : Acc(0);
        const Acc ub = om > -INFINITY ? wb * (ou + (om - mm) * os) : Acc(0);
        const Acc ni = (om > m2 || (om == m2 && oi < i2)) ? oi : i2;
        s2 = wa * sa + wb * sb;
        u2 = ua + ub;
        i2 = ni;
        m2 = mm;
      }
    }
    if (tid == 0) {
      Acc h = dlog(s2) - u2 / s2;
      if (!(h > Acc(0))) h = 0;
      H[r] = (float)h;
      amax[r] = (int32_t)i2;
    }
  }
  if (gpart) {  // (value, id) is a total order (ids are distinct): any merge order agrees
    __syncthreads();
    Acc bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = tid; i < n_vt; i += blockDim.x) {
      const Acc* g = gpart + ((size_t)i * n_rows + r) * 2;
      const Acc v = g[0];
      const int id = (int)g[1];
      if (v > bv || (v == bv && id < bi)) {
        bv = v;
        bi = id;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const Acc ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if ((tid & 31) == 0) {
      sm_m[tid >> 5] = bv;
      sm_i[tid >> 5] = (Acc)bi;
    }
    __syncthreads();
    if (tid == 0) {
      for (int w = 1; w < (int)(blockDim.x >> 5); ++w) {
        const Acc ov = sm_m[w];
        const int oi = (int)sm_i[w];
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      sampled[r] = bi;
    }
  }
  if (sc.P) {
    // M = max ref_t, S = sum_t s_t exp(ref_t - M) (per-thread partial sums over strided
    // tiles, then added in thread order), and each tile's factor exp(ref_t - M) / S
    // written over its ref_t for selfcond_scale_kernel
    __syncthreads();
    Acc* rp = reinterpret_cast<Acc*>(sc.ref);
    Acc Mt = -INFINITY;
    for (int i = tid; i < n_vt; i += blockDim.x) Mt = fmax(Mt, rp[((size_t)i * n_rows + r) * 2]);
    sm_m[tid] = Mt;
    __syncthreads();
    Acc Mx = -INFINITY;
    for (int t = 0; t < (int)blockDim.x; ++t) Mx = fmax(Mx, sm_m[t]);
    Acc St = 0;
    for (int i = tid; i < n_vt; i += blockDim.x) {
      const Acc* q = rp + ((size_t)i * n_rows + r) * 2;
      St += q[1] * dexp(q[0] - Mx);
    }
    sm_s[tid] = St;
    __syncthreads();
    Acc S = 0;
    for (int t = 0; t < (int)blockDim.x; ++t) S += sm_s[t];
    const Acc inv = Acc(1) / S;
    for (int i = tid; i < n_vt; i += blockDim.x) {
      Acc* q = rp + ((size_t)i * n_rows + r) * 2;
      q[0] = dexp(q[0] - Mx) * inv;
    }
  }
}

// p0 from the tile values: P[r, c] *= factor of (row r, tile c >> tw_shift) (the
// merge left the factors at ref[(tile, r)][0]).  One thread per 16 bytes of a row.
template <class TP, class Acc>
__global__ void selfcond_scale_kernel(TP* __restrict__ P, const Acc* __restrict__ ref, int n_rows,
                                      int V, int tw_shift) {
  pdl_enter();
  constexpr int kVec = 16 / sizeof(TP);
  const int per_row = V / kVec;  // V % kVec == 0
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)n_rows * per_row) return;
  const int r = (int)(i / per_row), c0 = (int)(i - (size_t)r * per_row) * kVec;
  const Acc f = ref[((size_t)(c0 >> tw_shift) * n_rows + r) * 2];
  uint4 w = *reinterpret_cast<const uint4*>(P + (size_t)r * V + c0);
  TP* e = reinterpret_cast<TP*>(&w);
#pragma unroll
  for (int j = 0; j < kVec; ++j) e[j] = narrow<TP>((Acc)widen(e[j]) * f);
  *reinterpret_cast<uint4*>(P + (size_t)r * V + c0) = w;
}

// Cache K [blocks, Wp, h] and V^T [blocks, h, Wp] -> K, V [blocks, W, h].
template <class T>
__global__ void kv_unpack_kernel(const T* __restrict__ k, const T* __restrict__ vt,
                                 T* __restrict__ ko, T* __restrict__ vo, size_t blocks, int W,
                                 int Wp, int h) {
  pdl_enter();
  const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i >= blocks * W * h) return;
  const size_t bl = i / ((size_t)W * h);
  const int t = (int)(i / h % W), dd = (int)(i % h);
  ko[i] = k[(bl * Wp + t) * h + dd];
  vo[i] = vt[(bl * h + dd) * Wp + t];
}

template <class T>
__global__ void widen_f32_kernel(const float* __restrict__ src, T* __restrict__ dst, long n) {
  pdl_enter();
  const long i = blockIdx.x * (long)blockDim.x + threadIdx.x;
  if (i < n) dst[i] = (T)src[i];
}

template <class T>
__global__ void to_f32_kernel(const T* __restrict__ src, float* __restrict__ dst, long n) {
  pdl_enter();
  const long i = blockIdx.x * (long)blockDim.x + threadIdx.x;
  if (i < n) dst[i] = (float)widen(src[i]);
}

// Start of a block: canvas all [MASK], mask all 1, counters cleared, steps left = T.
static __global__ void block_init_kernel(int32_t* __restrict__ canvas, uint8_t* __restrict__ mask,
                                         int n, int32_t mask_id, int32_t* __restrict__ nfwd,
                                         int B, int32_t* __restrict__ load, int n_load,
                                         int32_t* __restrict__ s_dev, int T) {
  pdl_enter();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    canvas[i] = mask_id;
    mask[i] = 1;
  }
  if (nfwd && i < B) nfwd[i] = 0;
  if (load && i < n_load) load[i] = 0;
  if (i == 0) *s_dev = T;
}

// End of one loop iteration of the captured block: steps left -= 1; run the next
// iteration only if steps remain and some canvas still has masked positions.
static __global__ void block_step_kernel(cudaGraphConditionalHandle handle,
                                         int32_t* __restrict__ s_dev,
                                         const int32_t* __restrict__ remaining, int B) {
  pdl_enter();
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const int s = *s_dev - 1;
  *s_dev = s;
  int any = 0;
  for (int b = 0; b < B; ++b) any |= remaining[b] > 0;
  cudaGraphSetConditional(handle, (s > 0 && any) ? 1u : 0u);
}

static __global__ void fill_i32_kernel(int32_t* __restrict__ p, int n, int32_t v) {
  pdl_enter();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}

}  // namespace dg
