// a9: the Entropy-Bound sampler step, one CTA per canvas.
//
// "DiffusionGemma 技术报告" (full translation page), §3.3 "DiffusionGemma 采样器",
// paragraph on entropy-bounded refinement: positions are accepted in ascending
// order of entropy until a bound is reached; explainer page "DiffusionGemma
// 深度解析", section "Entropy Bound (EB) 采样器": low-entropy positions first.
// Rule of this path: among the m masked positions sorted by (entropy, position),
// commit n = min(m, max(k_gamma, ceil(m / steps_left))) where k_gamma is the
// longest prefix whose entropies sum to <= gamma.  Sums are exact integers: each
// entropy h (NaN -> +inf, negative -> 0) contributes min(floor(h 2^48), 2^54);
// the bound is min(floor(gamma 2^48), 2^62) (computed on the host).
#pragma once

#include "k_common.cuh"

namespace dg {

__device__ __forceinline__ long long eb_q48(float h) {
  if (h != h) h = INFINITY;
  if (!(h > 0.0f)) h = 0.0f;
  const double v = (double)h * 281474976710656.0;  // 2^48, exact
  if (v >= 18014398509481984.0) return 1LL << 54;  // 2^54
  return (long long)floor(v);
}

__device__ __forceinline__ unsigned eb_key_bits(float h) {
  if (h != h) h = INFINITY;
  if (!(h > 0.0f)) h = 0.0f;
  return __float_as_uint(h);  // non-negative floats order like their bits
}

// blockDim.x = NP, a power of two >= max(C, 32), NP <= 1024.
template <int NP>
__global__ void __launch_bounds__(NP)
    eb_sample_kernel(const float* __restrict__ H, const int32_t* __restrict__ amax,
                     int32_t* __restrict__ canvas, uint8_t* __restrict__ mask, int C,
                     int steps_left, long long gamma_q, int32_t* __restrict__ n_commit,
                     int32_t* __restrict__ n_fwd, int step_no, const int32_t* __restrict__ s_dev,
                     int T, int32_t* __restrict__ remaining) {
  pdl_enter();
  if (s_dev) {  // steps left read from device memory (captured block loop)
    steps_left = *s_dev;
    step_no = T - steps_left + 1;
  }
  __shared__ unsigned long long key[NP];
  __shared__ unsigned long long pre[NP];
  __shared__ int cnt[NP / 32];
  const int b = blockIdx.x, i = threadIdx.x;
  const size_t base = (size_t)b * C;
  bool masked = false;
  unsigned long long k = ~0ull;
  if (i < C) {
    masked = mask[base + i] != 0;
    if (masked) k = ((unsigned long long)eb_key_bits(H[base + i]) << 32) | (unsigned)i;
  }
  key[i] = k;
  const unsigned bal = __ballot_sync(0xffffffffu, masked);
  if ((i & 31) == 0) cnt[i >> 5] = __popc(bal);
  __syncthreads();
  int m = 0;
  for (int w = 0; w < NP / 32; ++w) m += cnt[w];
  // bitonic sort, ascending
  for (int size = 2; size <= NP; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const int j = i ^ stride;
      if (j > i) {
        const unsigned long long a = key[i], c = key[j];
        const bool up = (i & size) == 0;
        if ((a > c) == up) {
          key[i] = c;
          key[j] = a;
        }
      }
      __syncthreads();
    }
  }
  // inclusive prefix sum of the fixed-point entropies of the first m entries, saturating
  // at gamma_q + 1 (gamma_q <= 2^62: two saturated terms never wrap, and "<= gamma_q"
  // is decided exactly however many capped entropies the canvas holds)
  const unsigned long long cap = (unsigned long long)gamma_q + 1;
  unsigned long long q = 0;
  if (i < m) q = (unsigned long long)eb_q48(__uint_as_float((unsigned)(key[i] >> 32)));
  pre[i] = q < cap ? q : cap;
  __syncthreads();
  for (int off = 1; off < NP; off <<= 1) {
    const unsigned long long add = i >= off ? pre[i - off] : 0;
    __syncthreads();
    const unsigned long long v = pre[i] + add;
    pre[i] = v < cap ? v : cap;
    __syncthreads();
  }
  // k_gamma = number of prefixes within the bound (prefix sums are non-decreasing)
  const int within = (i < m && pre[i] <= (unsigned long long)gamma_q) ? 1 : 0;
  const unsigned bw = __ballot_sync(0xffffffffu, within);
  __syncthreads();
  if ((i & 31) == 0) cnt[i >> 5] = __popc(bw);
  __syncthreads();
  int kg = 0;
  for (int w = 0; w < NP / 32; ++w) kg += cnt[w];
  const int floor_n = (m + steps_left - 1) / steps_left;
  const int n = min(m, max(kg, floor_n));
  if (i < n) {
    const int pos = (int)(key[i] & 0xffffffffu);
    canvas[base + pos] = amax[base + pos];
    mask[base + pos] = 0;
  }
  if (i == 0 && n_commit) n_commit[b] = n;
  if (i == 0 && remaining) remaining[b] = m - n;
  // the forward after which this canvas has no [MASK] left
  if (i == 0 && n_fwd && m > 0 && n == m) n_fwd[b] = step_no;
}

}  // namespace dg
