// dg_lmhead_entropy_noalloc: the LM-head entropy step for callers that cannot
// allocate device memory.
//
// The regular path keeps its scratch (the normalised rows and the per-tile
// softmax statistics) in the model's workspace, which dg_model_create obtains
// with cudaMalloc.  This variant needs no model and no allocation: its scratch
// is the file-scope device array below, a fixed 6 MiB that every GPU loading
// the library holds until the process exits.  All calls on a device share that
// array, so calls whose kernels overlap on the GPU (different streams, or
// several host threads) race with one another and must be serialised by the
// caller.  Nothing in the array needs to start at zero: each call overwrites
// every element it reads.
#include <cudaTypedefs.h>

#include <mutex>

#include "dg_internal.h"
#include "k_simt.cuh"
#include "k_tc_gemm.cuh"

namespace dg {
namespace {

constexpr int NA_MAX_ROWS = 256;        // M
constexpr int NA_MAX_D = 4096;          // d
constexpr int NA_MAX_VOCAB = 262144;    // V
constexpr int NA_BN = 256, NA_ST = 3;   // vocabulary tile and pipeline depth
constexpr size_t NA_XN_BYTES = (size_t)NA_MAX_ROWS * NA_MAX_D * 2;
constexpr size_t NA_PART_BYTES = (size_t)(NA_MAX_VOCAB / NA_BN) * NA_MAX_ROWS * 16;
constexpr size_t NA_SCRATCH_BYTES = NA_XN_BYTES + NA_PART_BYTES + 256;

// Scratch of every dg_lmhead_entropy_noalloc call on a device: bf16 normalised
// rows [M, d], then fp32 (max, sum, weighted sum, argmax) per (tile, row), then an
// error word set by a device-side wait that gave up.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NA_SCRATCH_BYTES];

struct DeviceState {
  bool ready = false;
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch
};
std::mutex g_mu;
DeviceState g_dev[64];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Once per device, with that device current: the scratch array's device address
// (the host-side symbol is only a stand-in and must never reach a kernel), the
// tensor-map encoder and the kernel's shared-memory limit.
dg_status setup(int dev, unsigned char** scratch) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (dev < 0 || dev >= 64) {
    set_error("device ordinal %d out of range", dev);
    return DG_ERR_UNSUPPORTED;
  }
  DeviceState& s = g_dev[dev];
  if (!s.ready) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      set_error("cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
      return DG_ERR_CUDA;
    }
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
        set_error("cuTensorMapEncodeTiled entry point unavailable");
        return DG_ERR_CUDA;
      }
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    typedef DenseCfg<NA_BN, 2, false, NA_ST> Cfg;
    e = cudaFuncSetAttribute(tc_dense_kernel<NA_BN, 2, false, NA_ST, EpiLmStats>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM);
    if (e != cudaSuccess) {
      set_error("cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      return DG_ERR_CUDA;
    }
    s.scratch = static_cast<unsigned char*>(p);
    s.ready = true;
  }
  *scratch = s.scratch;
  return DG_OK;
}

dg_status encode(const void* p, uint64_t rows, uint64_t cols, uint32_t box_rows, CUtensorMap* m) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(p), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (%d)", (int)r);
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

// A wait inside the GEMM that gave up leaves statistics unwritten: mark every row
// (entropy NaN, argmax -1) so the caller sees the failure in the outputs.
__global__ void noalloc_flag_kernel(const int32_t* err, int M, float* entropy, int32_t* argmax) {
  pdl_enter();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < M && *err) {
    entropy[i] = __int_as_float(0x7fc00000);
    argmax[i] = -1;
  }
}

}  // namespace
}  // namespace dg

using namespace dg;

extern "C" dg_status dg_lmhead_entropy_noalloc(const float* hidden, const void* lm_head,
                                               int32_t M, int32_t V, int32_t d, float rms_eps,
                                               float logit_scale, float* entropy,
                                               int32_t* argmax, void* stream) {
  DG_REQUIRE(hidden && lm_head && entropy && argmax, "null argument");
  DG_REQUIRE(M >= 1 && M <= NA_MAX_ROWS, "M=%d outside [1, %d]", M, NA_MAX_ROWS);
  DG_REQUIRE(V >= 1 && V <= NA_MAX_VOCAB, "V=%d outside [1, %d]", V, NA_MAX_VOCAB);
  DG_REQUIRE(d >= 64 && d <= NA_MAX_D && d % 64 == 0, "d=%d must be a multiple of 64 in [64, %d]",
             d, NA_MAX_D);
  DG_REQUIRE((reinterpret_cast<uintptr_t>(lm_head) & 15) == 0, "lm_head must be 16-byte aligned");
  DG_REQUIRE(rms_eps >= 0.0f && std::isfinite(logit_scale), "bad rms_eps / logit_scale");
  int dev = 0;
  DG_TRY_CUDA(cudaGetDevice(&dev));
  unsigned char* scratch = nullptr;
  DG_TRY(setup(dev, &scratch));
  bf16* xn = reinterpret_cast<bf16*>(scratch);
  float* part = reinterpret_cast<float*>(scratch + NA_XN_BYTES);
  int32_t* err = reinterpret_cast<int32_t*>(scratch + NA_XN_BYTES + NA_PART_BYTES);
  cudaStream_t st = (cudaStream_t)stream;
  DG_TRY_CUDA(cudaMemsetAsync(err, 0, sizeof(int32_t), st));

  rmsnorm_kernel<float, bf16, float><<<M, 256, 0, st>>>(hidden, xn, M, d, rms_eps, nullptr);
  CUtensorMap ma, mb;
  DG_TRY(encode(xn, (uint64_t)M, (uint64_t)d, 128, &ma));
  DG_TRY(encode(lm_head, (uint64_t)V, (uint64_t)d, NA_BN, &mb));
  typedef DenseCfg<NA_BN, 2, false, NA_ST> Cfg;
  dim3 grid((M + 255) / 256, (V + NA_BN - 1) / NA_BN, 1);
  tc_dense_kernel<NA_BN, 2, false, NA_ST, EpiLmStats><<<grid, TC_DENSE_THREADS, Cfg::SMEM, st>>>(
      ma, mb, mb, M, d, 1, EpiLmStats{part, M, V, logit_scale}, err, 0, 0);
  lm_merge_kernel<float, bf16><<<M, 128, 0, st>>>(part, (V + NA_BN - 1) / NA_BN, M, entropy,
                                                 argmax, nullptr, nullptr, ScDev{});
  noalloc_flag_kernel<<<(M + 127) / 128, 128, 0, st>>>(err, M, entropy, argmax);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("dg_lmhead_entropy_noalloc launch: %s", cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  return DG_OK;
}
