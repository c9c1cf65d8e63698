// Self-conditioning of the denoiser ("DiffusionGemma 技术报告" (full translation
// page), §3.2 "解码器前向传播" and "去噪迭代"; §6 on the cost of the embedding product
// over the whole vocabulary): after a forward, z = FFW(p0 E) with p0 = softmax(l) at
// temperature 1 over the V real tokens and E the token embedding rows of those tokens;
// z is added to the canvas rows' input of the next forward (0 at a block's first).
//
// Device plan: the LM-head epilogue stores, per vocabulary tile t of a row, the values
// exp(l - ref_t) (ref_t = the tile's largest logit at temperature 1) and records
// (ref_t, s_t = sum of those values); the merge kernel turns them into p0 by the factor
// exp(ref_t - M) / S (M = max ref_t, S = sum s_t exp(ref_t - M)); p0 E^T is a split-K
// GEMM (tensor cores on the bf16 path) whose partial sums are added in a fixed order;
// the FFW is the model's SwiGLU GEMM pair.
#pragma once

#include "k_common.cuh"

namespace dg {

constexpr int SC_MAX_PARTS = 16;  // K slices of the p0 E^T GEMM (tensor-core path)

// Where the LM head leaves p0.  P == nullptr: no self-conditioning.
struct ScDev {
  void* P = nullptr;    // [rows, ldp] in the activation type: tile values, then p0
  void* ref = nullptr;  // [tiles, rows, 2] (ref_t, s_t) in the accumulate type
  int ldp = 0;          // V
};

// y[r, c] = sum over z of part[z][r, c] in z order, stored in the activation type.
template <class TA>
__global__ void selfcond_reduce_kernel(const float* __restrict__ part, int nparts, int n, int d,
                                       TA* __restrict__ y) {
  pdl_enter();
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t total = (size_t)n * d;
  if (i >= total) return;
  float s = 0.f;
  for (int z = 0; z < nparts; ++z) s += part[(size_t)z * total + i];
  y[i] = narrow<TA>(s);
}

// embT[c, v] = emb[v, c] for the V real tokens (32 x 32 tiles through shared memory).
template <class TW>
__global__ void transpose_emb_kernel(const TW* __restrict__ emb, TW* __restrict__ embT, int V,
                                     int d) {
  __shared__ TW t[32][33];
  const int v0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int v = v0 + r, c = c0 + threadIdx.x;
    if (v < V && c < d) t[r][threadIdx.x] = emb[(size_t)v * d + c];
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int c = c0 + r, v = v0 + threadIdx.x;
    if (c < d && v < V) embT[(size_t)c * V + v] = t[threadIdx.x][r];
  }
}

}  // namespace dg
