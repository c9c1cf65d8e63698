// The Report's default sampler on the device: entropy-bounded refinement with
// temperature annealing and adaptive stopping over a uniform-noise canvas
// ("DiffusionGemma 技术报告" (full translation page), §3.2 "画布初始化" and
// "多项式扩散", §3.3 "熵有界的 token 精炼", "温度退火", "自适应停止启发式").
//
// Readings (the same list stands beside the oracle):
//  * step k (0-based) runs at t = (N - k) / N, tau = tau_min + (tau_max - tau_min) t in
//    fp64; the entropies ordered, bounded and averaged are those of softmax(l / tau);
//  * accepted set: the longest prefix of the ascending (entropy, position) order whose
//    entropies satisfy sum - max <= b (mutual-information bound), i.e. one more than
//    the number of leading fixed-point entropies that sum to <= b (at most C); the
//    accepted positions keep the token drawn for them, every other position takes a
//    fresh uniform token;
//  * stop after a step when sum_i q(H_i) < C q(e_stop) and the argmax sequence equals
//    the previous step's (never at the first step); then, or after step N - 1, the
//    canvas becomes that step's argmax sequence;
//  * draws: SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) used counter-wise, the
//    c-th output after state key being mix64(key + (c + 1) G); per canvas seed three
//    stream keys mix64(seed + j G), j = 1 initial canvas (c = i), 2 Gumbel noise
//    (c = (k C + i) ceil(V / 2) + floor(v / 2): one output per token pair, the even
//    token taking bits 63..41 and the odd one bits 31..9), 3 re-noising (c = k C + i);
//    token = hi32(z) V >> 32; Gumbel noise -log E, E = -log u, u = (f + 1/2) 2^-23
//    for the 23-bit field f; the drawn token is argmax_v (l_v / tau - log E_v), the
//    lowest id on ties.
#pragma once

#include "k_common.cuh"
#include "k_sampler.cuh"

namespace dg {

constexpr unsigned long long SM64_G = 0x9E3779B97F4A7C15ull;
enum { SM64_INIT = 1, SM64_GUMBEL = 2, SM64_RENOISE = 3 };

__host__ __device__ __forceinline__ unsigned long long sm64_mix(unsigned long long z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__host__ __device__ __forceinline__ unsigned long long sm64_key(unsigned long long seed,
                                                                int stream) {
  return sm64_mix(seed + (unsigned long long)stream * SM64_G);
}
__host__ __device__ __forceinline__ unsigned long long sm64_draw(unsigned long long key,
                                                                 unsigned long long c) {
  return sm64_mix(key + (c + 1) * SM64_G);
}
__device__ __forceinline__ int32_t sm64_token(unsigned long long z, int V) {
  return (int32_t)(((z >> 32) * (unsigned long long)(unsigned)V) >> 32);
}
// the 23-bit field of output z for the even (odd = 0) or odd token of a pair
__device__ __forceinline__ unsigned sm64_field(unsigned long long z, int odd) {
  return odd ? (unsigned)(z >> 9) & 0x7FFFFFu : (unsigned)(z >> 41);
}
// E = -log u with u = (f + 1/2) 2^-23, u exact in fp32 and fp64
__device__ __forceinline__ float sm64_expo(unsigned f, float) {
  return -logf(((float)f + 0.5f) * 1.1920928955078125e-07f);
}
__device__ __forceinline__ double sm64_expo(unsigned f, double) {
  return -log(((double)f + 0.5) * 1.1920928955078125e-07);
}

// Per-launch parameters of the tempered LM-head statistics and the Gumbel-max draw.
// N == 0: statistics at temperature 1 and no draw (the Entropy-Bound path).
struct AnnealDev {
  const unsigned long long* seeds = nullptr;  // [B] per-canvas seeds
  const int32_t* s_dev = nullptr;             // steps left on the device (loop), else s
  int s = 0, N = 0, C = 1;
  float tau_max = 1.f, tau_min = 1.f;
  void* gpart = nullptr;  // [tiles, rows] (best l / tau - log E, id) in the accumulate type
  __device__ __forceinline__ int steps_left() const { return s_dev ? *s_dev : s; }
  __device__ __forceinline__ double tau() const {
    return (double)tau_min +
           ((double)tau_max - (double)tau_min) * ((double)steps_left() / (double)N);
  }
  // the Gumbel stream's state for token pair `pair` of row `row`: key + (c + 1) G with
  // c = (k C + i) ceil(V / 2) + pair
  __device__ __forceinline__ unsigned long long pair_state(int row, int V, int pair) const {
    const int b = row / C, i = row - b * C;
    const unsigned long long key = sm64_key(seeds[b], SM64_GUMBEL);
    const unsigned long long k = (unsigned long long)(N - steps_left());
    const unsigned long long c =
        (k * C + i) * (unsigned long long)((V + 1) >> 1) + (unsigned)pair;
    return key + (c + 1) * SM64_G;
  }
};

// A candidate of the Gumbel-max race kept as (e = exp(z), E, z, id) with z the
// tempered logit minus the tile maximum: candidate a beats b when e_a / E_a > e_b / E_b
// (compared as e_a E_b > e_b E_a), or equally and with the lower id.
template <class Acc> struct GumbelBest {
  Acc e = 0, E = 1, z = 0;
  int id = 0x7fffffff;
  __device__ __forceinline__ bool offer(Acc e2, Acc E2, Acc z2, int id2) {
    const Acc l = e2 * E, r = e * E2;
    if (l > r || (l == r && id2 < id)) {
      e = e2;
      E = E2;
      z = z2;
      id = id2;
      return true;
    }
    return false;
  }
  // the candidate's value on the absolute scale: m + z - log E = l / tau + Gumbel noise
  __device__ __forceinline__ Acc value(Acc m) const { return m + z - dlog(E); }
};

// The smallest E a draw can give is -log(1 - 2^-24) = 5.96e-8; a candidate with
// e < e_best * SM64_EMIN_LO / E_best therefore cannot beat the best (SM64_EMIN_LO is a
// little below that minimum, so the test never discards a possible winner).
constexpr float SM64_EMIN_LO = 5.9e-8f;

// x_1: uniform tokens (stream 1); previous argmax -1; per-canvas stop state 0; the
// loop's steps-left counter N.
static __global__ void anneal_init_kernel(int32_t* __restrict__ canvas,
                                          int32_t* __restrict__ prev, int32_t* __restrict__ state,
                                          int32_t* __restrict__ nfwd, int B, int C, int V,
                                          const unsigned long long* __restrict__ seeds,
                                          int32_t* __restrict__ s_dev, int N) {
  pdl_enter();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < B * C) {
    const int b = t / C, i = t - b * C;
    canvas[t] = sm64_token(sm64_draw(sm64_key(seeds[b], SM64_INIT), (unsigned)i), V);
    if (prev) prev[t] = -1;
  }
  if (t < B) {
    if (state) state[t] = 0;
    if (nfwd) nfwd[t] = 0;
  }
  if (t == 0 && s_dev) *s_dev = N;
}

// One refinement step of every canvas (one CTA of NP threads per canvas, NP a power of
// two >= max(C, 32), <= 1024).  H, amax, sampled: [B, C] from the step's forward;
// canvas [B, C] is rewritten; prev [B, C] holds the previous step's argmax; state[b] is
// 0 while canvas b runs and its forward count once it has stopped (a stopped canvas is
// left as it is).  bq = min(floor(b 2^48), 2^62); eq = floor(e_stop 2^48) <= 2^52.
template <int NP>
__global__ void __launch_bounds__(NP)
    anneal_sample_kernel(const float* __restrict__ H, const int32_t* __restrict__ amax,
                         const int32_t* __restrict__ sampled, int32_t* __restrict__ canvas,
                         int32_t* __restrict__ prev, int32_t* __restrict__ state,
                         int32_t* __restrict__ nfwd, int32_t* __restrict__ nacc,
                         int32_t* __restrict__ remaining, int C, int V, int k,
                         const int32_t* __restrict__ s_dev, int N, unsigned long long bq,
                         unsigned long long eq, const unsigned long long* __restrict__ seeds) {
  pdl_enter();
  if (s_dev) k = N - *s_dev;
  __shared__ unsigned long long key[NP];
  __shared__ unsigned long long pre[NP];
  __shared__ unsigned long long wsum[NP / 32];
  __shared__ int cnt[NP / 32];
  const int b = blockIdx.x, i = threadIdx.x, lane = i & 31, w = i >> 5;
  const size_t base = (size_t)b * C;
  if (state[b] != 0) {  // stopped at an earlier step
    if (i == 0 && remaining) remaining[b] = 0;
    return;
  }
  // fixed-point entropies, the stop sum (saturating at C eq, the only value compared)
  // and whether the argmax sequence moved
  const unsigned long long lim = (unsigned long long)C * eq;
  unsigned long long kk = ~0ull, q = 0;
  int a = 0, moved = 0;
  if (i < C) {
    const float h = H[base + i];
    q = (unsigned long long)eb_q48(h);
    kk = ((unsigned long long)eb_key_bits(h) << 32) | (unsigned)i;
    a = amax[base + i];
    moved = (k == 0) || a != prev[base + i];
    prev[base + i] = a;
  }
  key[i] = kk;
  unsigned long long ssum = q < lim ? q : lim;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long v = __shfl_xor_sync(0xffffffffu, ssum, o);
    ssum = ssum + v < lim ? ssum + v : lim;  // both <= lim <= 2^62: no wrap
  }
  const unsigned mv = __ballot_sync(0xffffffffu, moved);
  if (lane == 0) {
    wsum[w] = ssum;
    cnt[w] = __popc(mv);
  }
  __syncthreads();
  unsigned long long tot = 0;
  int any_moved = 0;
  for (int j = 0; j < NP / 32; ++j) {
    tot = tot + wsum[j] < lim ? tot + wsum[j] : lim;
    any_moved |= cnt[j];
  }
  const bool stop = tot < lim && !any_moved;
  if (stop || k >= N - 1) {  // the canvas's result: this step's argmax sequence
    if (i < C) canvas[base + i] = a;
    if (i == 0) {
      state[b] = k + 1;
      if (nfwd) nfwd[b] = k + 1;
      if (nacc) nacc[b] = C;
      if (remaining) remaining[b] = 0;
    }
    return;
  }
  __syncthreads();  // cnt is reused below
  // bitonic sort of (entropy bits, position), ascending
  for (int size = 2; size <= NP; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const int j = i ^ stride;
      if (j > i) {
        const unsigned long long x = key[i], y = key[j];
        const bool up = (i & size) == 0;
        if ((x > y) == up) {
          key[i] = y;
          key[j] = x;
        }
      }
      __syncthreads();
    }
  }
  // inclusive prefix sums of the sorted fixed-point entropies, saturating at bq + 1
  // (bq <= 2^62, so two saturated terms never wrap and "<= bq" stays exact)
  const unsigned long long cap = bq + 1;
  unsigned long long qs = 0;
  if (i < C) {
    qs = (unsigned long long)eb_q48(__uint_as_float((unsigned)(key[i] >> 32)));
    if (qs > cap) qs = cap;
  }
  pre[i] = qs;
  __syncthreads();
  for (int off = 1; off < NP; off <<= 1) {
    const unsigned long long add = i >= off ? pre[i - off] : 0;
    __syncthreads();
    const unsigned long long v = pre[i] + add;
    pre[i] = v < cap ? v : cap;
    __syncthreads();
  }
  const int within = (i < C && pre[i] <= bq) ? 1 : 0;
  const unsigned bw = __ballot_sync(0xffffffffu, within);
  if (lane == 0) cnt[w] = __popc(bw);
  __syncthreads();
  int lead = 0;
  for (int j = 0; j < NP / 32; ++j) lead += cnt[j];
  const int n = min(C, lead + 1);
  if (i < C) {  // thread i handles the i-th position in the order
    const int pos = (int)(key[i] & 0xffffffffu);
    canvas[base + pos] =
        i < n ? sampled[base + pos]
              : sm64_token(sm64_draw(sm64_key(seeds[b], SM64_RENOISE),
                                     (unsigned long long)k * C + pos),
                           V);
  }
  if (i == 0) {
    if (nacc) nacc[b] = n;
    if (remaining) remaining[b] = 1;
  }
}

}  // namespace dg
