// tcgen05 (5th-generation tensor core) kernels for the bf16 dense contractions.
#pragma once

#include "dg_internal.h"

namespace dg {

inline dg_status tc_prepare(dg_model*) { return DG_OK; }
inline void tc_release(dg_model*) {}
inline int tc_group_rows() { return 64; }
inline dg_status tc_unsupported() {
  set_error("tensor-core kernels are not built");
  return DG_ERR_UNSUPPORTED;
}
inline dg_status tc_gemm_store_f32(dg_model*, const bf16*, const void*, float*, int, int, int,
                                   cudaStream_t) { return tc_unsupported(); }
inline dg_status tc_gemm_add_residual(dg_model*, const bf16*, const void*, float*, int, int, int,
                                      cudaStream_t) { return tc_unsupported(); }
inline dg_status tc_gemm_swiglu(dg_model*, const bf16*, const void*, const void*, bf16*, int, int,
                                int, cudaStream_t) { return tc_unsupported(); }
inline dg_status tc_moe_gate_up(dg_model*, int, const bf16*, bf16*, int, cudaStream_t) {
  return tc_unsupported();
}
inline dg_status tc_moe_down(dg_model*, int, const bf16*, float*, int, cudaStream_t) {
  return tc_unsupported();
}
inline dg_status tc_lmhead_stats(dg_model*, const bf16*, int, float*, int32_t*, cudaStream_t) {
  return tc_unsupported();
}

}  // namespace dg
