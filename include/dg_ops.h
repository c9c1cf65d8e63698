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

/* Test hook for the device-side timeout path (no counterpart on the pages): the next
 * routed-expert launch of this bf16 model makes its down units wait for one more
 * gate/up unit than their token chunk has, and limits every wait of that launch to
 * limit_ns nanoseconds (1e5 .. 1e9).  Each such wait runs out: the launch records
 * DG_ERR_TIMEOUT in the model's device error word and unwinds (every role of the kernel
 * keeps its waits bounded, so it ends within a few multiples of limit_ns), the next
 * dg_sync_status returns DG_ERR_TIMEOUT, and later launches run normally.  Applies to
 * one launch.  DG_ERR_UNSUPPORTED for models whose experts do not use that kernel
 * (fp32, FP8 experts). */
dg_status dg_debug_stall_experts(dg_model* m, int64_t limit_ns);

#ifdef __cplusplus
}
#endif
#endif /* DG_OPS_H */
