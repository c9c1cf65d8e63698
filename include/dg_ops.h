/*
 * dg_ops.h — single-step entry points of libdg, for testing one kernel group at
 * a time against the oracle.  Same conventions as dg.h (device pointers,
 * dg_status returns, `stream` = cudaStream_t as void*).
 */
#ifndef DG_OPS_H
#define DG_OPS_H

#include "dg.h"

#ifdef __cplusplus
extern "C" {
#endif

/* One dense projection as the path computes it (a2/a4/a7 of the forward):
 * out[M, N] = A[M, K] W[N, K]^T in fp32 (bf16 models: A, W bf16 on the tcgen05
 * kernel; DG_F32 models: A, W fp32 on CUDA cores with fp64 sums).
 * Requires M >= 1, N % 64 == 0, K % 64 == 0 for bf16 models. */
dg_status dg_op_gemm(dg_model* m, const void* A, const void* W, float* out, int32_t M,
                     int32_t N, int32_t K, void* stream);

/* The MoE block of layer `layer` on n residual rows (a5 + a6 + a7):
 * out[n, d] = x + sum_{e in top-k} g_e Expert_e(u) + Shared(u), u = RMSNorm(x),
 * routing as in the forward (softmax over all experts, top-k, renormalised).
 * x, out: [n, d] fp32 (1 <= n <= the model's token capacity). */
dg_status dg_op_moe(dg_model* m, int32_t layer, const float* x, float* out, int32_t n,
                    void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DG_OPS_H */
