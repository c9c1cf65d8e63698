// Host side of the tcgen05 kernels: TMA tensor maps (cached per buffer) and
// launch configuration of the dense, grouped-expert and LM-head GEMMs.
#include <cudaTypedefs.h>

#include <mutex>

#include "dg_internal.h"
#include "k_simt.cuh"
#include "k_tc_attn.cuh"
#include "k_tc_expert_fp8.cuh"
#include "k_tc_gemm.cuh"

namespace dg {

namespace {

struct MapKey {
  const void* p;
  uint64_t rows, cols;
  uint32_t box_rows;
  bool bytes = false;  // uint8 elements, no swizzle (FP8 weights, packed NVFP4 weights)
  uint32_t box_cols = 64;  // inner box extent in elements (bytes for uint8 maps)
  bool operator==(const MapKey& o) const {
    return p == o.p && rows == o.rows && cols == o.cols && box_rows == o.box_rows &&
           bytes == o.bytes && box_cols == o.box_cols;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    size_t h = std::hash<const void*>()(k.p);
    h ^= std::hash<uint64_t>()(k.rows * 1315423911ull + k.cols) + 0x9e3779b9 + (h << 6) + (h >> 2);
    return h ^ (k.box_rows * 2654435761u);
  }
};

struct TcState {
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  int n_sm = 148;
  std::unordered_map<MapKey, CUtensorMap, MapKeyHash> maps;
};

std::mutex g_tc_mu;
std::unordered_map<const dg_model*, TcState*> g_tc;

TcState* state(const dg_model* m) {
  std::lock_guard<std::mutex> lk(g_tc_mu);
  auto it = g_tc.find(m);
  return it == g_tc.end() ? nullptr : it->second;
}

int ceil_div_i(long a, long b) { return (int)((a + b - 1) / b); }

// 2-D bf16 tensor [rows, cols] (row-major), box = 64 columns x box_rows rows,
// 128-byte swizzle, out-of-range elements read as zero.
dg_status tmap(const dg_model* m, const void* p, uint64_t rows, uint64_t cols, uint32_t box_rows,
               CUtensorMap* out, bool bytes = false, uint32_t box_cols = 64) {
  TcState* s = state(m);
  if (!s) {
    set_error("tensor-core state missing");
    return DG_ERR_INTERNAL;
  }
  MapKey key{p, rows, cols, box_rows, bytes, box_cols};
  auto it = s->maps.find(key);
  if (it != s->maps.end()) {
    *out = it->second;
    return DG_OK;
  }
  const uint64_t esz = bytes ? 1 : 2;
  if ((reinterpret_cast<uintptr_t>(p) & 15) || (cols * esz) % 16 || box_rows > 256) {
    set_error("tensor map: base %p / row pitch %llu bytes not 16-byte aligned", p,
              (unsigned long long)(cols * esz));
    return DG_ERR_UNSUPPORTED;
  }
  CUtensorMap map;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esz};
  if (box_cols * esz % 16 || box_cols > 256) {
    set_error("tensor map: inner box of %u elements is not a multiple of 16 bytes", box_cols);
    return DG_ERR_UNSUPPORTED;
  }
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = s->encode(&map, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                         2, const_cast<void*>(p), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE,
                         bytes ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (%d) for %p [%llu x %llu] box %u", (int)r, p,
              (unsigned long long)rows, (unsigned long long)cols, box_rows);
    return DG_ERR_CUDA;
  }
  s->maps.emplace(key, map);
  *out = map;
  return DG_OK;
}

template <class K> dg_status set_smem(K kern, size_t bytes) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) {
    set_error("cudaFuncSetAttribute(%zu bytes): %s", bytes, cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

// Split K over a cluster when the (M, N) tiles alone would leave most SMs idle.
template <int BN, int MT, bool DUAL, int ST, class Epi>
dg_status launch_dense(dg_model* m, const CUtensorMap& a, const CUtensorMap& b,
                       const CUtensorMap& b2, int M, int N, int K, Epi epi, cudaStream_t st,
                       bool allow_split = true, int kwrap = 0, bool b_weight = true) {
  typedef DenseCfg<BN, MT, DUAL, ST> Cfg;
  auto kern = tc_dense_kernel<BN, MT, DUAL, ST, Epi>;
  dim3 grid(ceil_div_i(M, 128 * MT), ceil_div_i(N, BN), 1);
  const int tiles = grid.x * grid.y;
  const int nk = ceil_div_i(K, TC_KB);
  int ks = 1;
  if (allow_split)
    while (ks < 8 && tiles * ks * 2 <= state(m)->n_sm && nk >= ks * 2 * 2) ks *= 2;
  cudaError_t e;
  if (ks == 1) {
    e = launch_pdl(kern, grid, TC_DENSE_THREADS, Cfg::SMEM + Epi::kExtraSmem, st, 1, a, b, b2, M, K, 1, epi,
                   m->ws.err, kwrap, b_weight ? 1 : 0);
  } else {
    grid.z = ks;
    e = launch_pdl(kern, grid, TC_DENSE_THREADS, Cfg::SMEM + Epi::kExtraSmem, st, ks, a, b, b2, M, K, ks, epi,
                   m->ws.err, kwrap, b_weight ? 1 : 0);
  }
  ++m->launches;
  if (e != cudaSuccess) {
    set_error("tc_dense launch: %s", cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

constexpr int DENSE_BN = 64, DENSE_MT = 2, DENSE_ST = 5, DUAL_ST = 4;
constexpr int QKV_ST = 4, RT_ST = 4;
constexpr int LM_BN = 256, LM_ST = 3;
constexpr int MOE_ST = 4;
constexpr int MOE8_ST = 3;
constexpr int SC_ST = 3;  // p0 E^T GEMM stages

}  // namespace

dg_status tc_prepare(dg_model* m) {
  const dg_config& c = m->cfg;
  const int qkv_n = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim;
  if (c.d_model % 256 || c.expert_inter % 128 || c.shared_inter % 64 || qkv_n % 64 ||
      (c.n_q_heads * c.head_dim) % 64) {
    set_error("tensor-core tiling needs d %% 256, I %% 128, Is %% 64, (Hq+2Hkv)h %% 64 and Hq h %% 64");
    return DG_ERR_UNSUPPORTED;
  }
  if (c.dtype == DG_BF16_FP8EXP && (c.d_model > 4096 || c.expert_inter > 4096)) {
    set_error("FP8 expert kernel keeps a unit's scales in shared memory: d and I <= 4096");
    return DG_ERR_UNSUPPORTED;
  }
  TcState* s = new TcState();
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
    delete s;
    set_error("cuTensorMapEncodeTiled entry point unavailable");
    return DG_ERR_CUDA;
  }
  s->encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  {
    std::lock_guard<std::mutex> lk(g_tc_mu);
    g_tc[m] = s;
  }
  // dynamic shared-memory limits, set once here so that no attribute call happens
  // while a launch sequence is being captured into a graph
  typedef DenseCfg<DENSE_BN, DENSE_MT, false, DENSE_ST> Dn;
  typedef DenseCfg<DENSE_BN, DENSE_MT, true, DUAL_ST> Du;
  typedef DenseCfg<LM_BN, 2, false, LM_ST> Lm;
  DG_TRY(set_smem(tc_dense_kernel<DENSE_BN, DENSE_MT, false, DENSE_ST, EpiStoreF32>, Dn::SMEM));
  DG_TRY(set_smem(tc_dense_kernel<DENSE_BN, DENSE_MT, false, DENSE_ST, EpiAddF32>,
                  Dn::SMEM + EpiAddF32::kExtraSmem));
  DG_TRY(set_smem(tc_dense_kernel<DENSE_BN, DENSE_MT, true, DUAL_ST, EpiSwigluBf16>, Du::SMEM));
  DG_TRY(set_smem(tc_dense_kernel<LM_BN, 2, false, LM_ST, EpiLmStats>, Lm::SMEM));
  DG_TRY(set_smem(tc_dense_kernel<256, 2, false, SC_ST, EpiPartialRows>,
                  DenseCfg<256, 2, false, SC_ST>::SMEM));
  DG_TRY(set_smem(tc_moe_kernel<MOE_ST>, MoeCfg<MOE_ST>::SMEM));
  DG_TRY(set_smem(tc_attn_kernel, AT_SMEM));
  DG_TRY(set_smem(tc_dense_kernel<128, 1, false, RT_ST, EpiRouterTopk>,
                  DenseCfg<128, 1, false, RT_ST>::SMEM));
  DG_TRY(set_smem(tc_dense_kernel<128, DENSE_MT, false, QKV_ST, EpiQkvRope>,
                  DenseCfg<128, DENSE_MT, false, QKV_ST>::SMEM + EpiQkvRope::kExtraSmem));
  DG_TRY(set_smem(tc_moe_f8_kernel<MOE8_ST>, MoeF8Cfg<MOE8_ST>::smem_bytes(4096, 4096)));
  DG_TRY(set_smem(tc_moe_f4_kernel<MOE8_ST>, MoeLowpCfg<MOE8_ST, true>::smem_bytes(2048, 2048)));
  cudaDeviceGetAttribute(&s->n_sm, cudaDevAttrMultiProcessorCount, m->device);
  return DG_OK;
}

void tc_release(dg_model* m) {
  std::lock_guard<std::mutex> lk(g_tc_mu);
  auto it = g_tc.find(m);
  if (it != g_tc.end()) {
    delete it->second;
    g_tc.erase(it);
  }
}

dg_status tc_gemm_store_f32(dg_model* m, const bf16* A, const void* W, float* out, int M, int N,
                            int K, cudaStream_t st) {
  CUtensorMap a, b;
  DG_TRY(tmap(m, A, m->ws.max_tok, K, 128, &a));
  DG_TRY(tmap(m, W, N, K, DENSE_BN, &b));
  return launch_dense<DENSE_BN, DENSE_MT, false, DENSE_ST>(m, a, b, b, M, N, K,
                                                           EpiStoreF32{out, N, N}, st);
}

dg_status tc_gemm_qkv_rope(dg_model* m, const bf16* A, const void* W, int M, int n_seq, int np,
                           int pos0, bf16* q, bf16* kc, bf16* vc, cudaStream_t st) {
  const dg_config& c = m->cfg;
  const int N = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim, K = c.d_model;
  CUtensorMap a, b;
  DG_TRY(tmap(m, A, m->ws.max_tok, K, 128, &a));
  DG_TRY(tmap(m, W, N, K, 128, &b));
  EpiQkvRope epi;
  epi.q = q;
  epi.kc = kc;
  epi.vc = vc;
  epi.rope = (const float*)m->ws.rope;
  epi.max_pos = m->ws.max_pos;
  epi.n_seq = n_seq;
  epi.np = np;
  epi.pos0 = pos0;
  epi.Hq = c.n_q_heads;
  epi.Hkv = c.n_kv_heads;
  return launch_dense<128, DENSE_MT, false, QKV_ST>(m, a, b, b, M, N, K, epi, st);
}

// Router logits u . w on tensor cores as [u_hi | u_lo] . [w | w] (K = 2 d), top-k
// in the epilogue.  One N-tile holds all experts (E <= 128).
dg_status tc_router_topk(dg_model* m, const bf16* u2, const void* Wr, int M, int32_t* idx,
                         float* gate, cudaStream_t st) {
  const dg_config& c = m->cfg;
  const int d = c.d_model;
  CUtensorMap a, b;
  DG_TRY(tmap(m, u2, m->ws.max_tok, 2 * d, 128, &a));
  DG_TRY(tmap(m, Wr, c.n_experts, d, 128, &b));
  EpiRouterTopk epi;
  epi.idx = idx;
  epi.gate = gate;
  epi.E = c.n_experts;
  epi.top_k = c.top_k;
  return launch_dense<128, 1, false, RT_ST>(m, a, b, b, M, 128, 2 * d, epi, st, true, d);
}

dg_status tc_gemm_f32_rows(dg_model* m, const bf16* A, int a_rows, const void* W, float* out,
                           int M, int N, int K, cudaStream_t st) {
  CUtensorMap a, b;
  DG_TRY(tmap(m, A, a_rows, K, 128, &a));
  DG_TRY(tmap(m, W, N, K, DENSE_BN, &b));
  // W is the caller's tensor, not a model weight: read only after the dependency wait
  return launch_dense<DENSE_BN, DENSE_MT, false, DENSE_ST>(m, a, b, b, M, N, K,
                                                           EpiStoreF32{out, N, N}, st, true, 0,
                                                           false);
}

dg_status tc_gemm_add_residual(dg_model* m, const bf16* A, const void* W, float* x, int M, int N,
                               int K, cudaStream_t st) {
  CUtensorMap a, b;
  DG_TRY(tmap(m, A, m->ws.max_tok, K, 128, &a));
  DG_TRY(tmap(m, W, N, K, DENSE_BN, &b));
  return launch_dense<DENSE_BN, DENSE_MT, false, DENSE_ST>(m, a, b, b, M, N, K,
                                                           EpiAddF32{x, N, N}, st);
}

dg_status tc_gemm_swiglu(dg_model* m, const bf16* A, const void* Wg, const void* Wu, bf16* out,
                         int M, int N, int K, cudaStream_t st) {
  CUtensorMap a, b, b2;
  DG_TRY(tmap(m, A, m->ws.max_tok, K, 128, &a));
  DG_TRY(tmap(m, Wg, N, K, DENSE_BN, &b));
  DG_TRY(tmap(m, Wu, N, K, DENSE_BN, &b2));
  return launch_dense<DENSE_BN, DENSE_MT, true, DUAL_ST>(m, a, b, b2, M, N, K,
                                                         EpiSwigluBf16{out, N, N}, st);
}

dg_status tc_lmhead_stats(dg_model* m, const bf16* xn, int M, float* ent, int32_t* amax,
                          cudaStream_t st, const AnnealDev& an, int32_t* sampled,
                          const ScDev& sc) {
  const dg_config& c = m->cfg;
  CUtensorMap a, b;
  DG_TRY(tmap(m, xn, m->ws.max_tok, c.d_model, 128, &a));
  DG_TRY(tmap(m, m->w.lm_head, c.vocab, c.d_model, LM_BN, &b));
  float* part = (float*)m->ws.lm_part;
  EpiLmStats epi{part, M, c.vocab, c.logit_scale};
  epi.an = an;
  epi.sc = sc;
  DG_TRY((launch_dense<LM_BN, 2, false, LM_ST>(m, a, b, b, M, c.vocab, c.d_model, epi, st,
                                               false)));
  const int n_vt = ceil_div_i(c.vocab, LM_BN);
  launch_pdl((lm_merge_kernel<float, bf16>), M, 128, 0, st, 1, part, n_vt, M, ent, amax,
             (const float*)(an.seeds ? an.gpart : nullptr), an.seeds ? sampled : nullptr, sc);
  ++m->launches;
  if (sc.P) {  // the tile values become p0
    static_assert(LM_BN == 256, "tile shift");
    const long groups = (long)M * (c.vocab / 8);
    launch_pdl((selfcond_scale_kernel<bf16, float>), (int)((groups + 255) / 256), 256, 0, st, 1,
               (bf16*)sc.P, (const float*)sc.ref, M, c.vocab, 8);
    ++m->launches;
  }
  return DG_OK;
}

dg_status tc_selfcond_mix(dg_model* m, int n, cudaStream_t st) {
  const dg_config& c = m->cfg;
  const int V = c.vocab, d = c.d_model;
  const size_t lm_rows = (size_t)c.max_batch * c.canvas;
  CUtensorMap a, b;
  DG_TRY(tmap(m, m->ws.scP, lm_rows, V, 128, &a));
  DG_TRY(tmap(m, m->ws.embT, d, V, 256, &b));
  typedef DenseCfg<256, 2, false, SC_ST> Cfg;
  const int tiles = ceil_div_i(n, 256) * ceil_div_i(d, 256);
  const int nk = ceil_div_i(V, TC_KB);
  const int S = std::max(1, std::min(std::min(SC_MAX_PARTS, state(m)->n_sm / tiles), nk));
  dim3 grid(ceil_div_i(n, 256), ceil_div_i(d, 256), S);
  EpiPartialRows epi{(float*)m->ws.scpart, n, d, (size_t)n * d};
  cudaError_t e = launch_pdl(tc_dense_kernel<256, 2, false, SC_ST, EpiPartialRows>, grid,
                             TC_DENSE_THREADS, Cfg::SMEM, st, 1, a, b, b, n, V, -S, epi,
                             m->ws.err, 0, 1);
  ++m->launches;
  if (e != cudaSuccess) {
    set_error("self-conditioning GEMM launch: %s", cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  const long total = (long)n * d;
  launch_pdl((selfcond_reduce_kernel<bf16>), (int)((total + 255) / 256), 256, 0, st, 1,
             (const float*)m->ws.scpart, S, n, d, (bf16*)m->ws.scy);
  ++m->launches;
  return DG_OK;
}

// FP8 expert weights: both phases in one persistent launch (tc_moe_f8_kernel)
dg_status tc_moe_experts_f8(dg_model* m, int l, const bf16* X, bf16* hb, float* yb,
                            cudaStream_t st) {
  const dg_config& c = m->cfg;
  const dg_layer_weights& L = m->layers[l];
  const int E = c.n_experts, I = c.expert_inter, d = c.d_model;
  const Workspace& ws = m->ws;
  CUtensorMap wg, wu, x, wd, h;
  DG_TRY(tmap(m, L.gate, (uint64_t)E * I, d, 128, &wg, true));
  DG_TRY(tmap(m, L.up, (uint64_t)E * I, d, 128, &wu, true));
  DG_TRY(tmap(m, X, ws.max_rows, d, 32, &x));
  DG_TRY(tmap(m, L.down, (uint64_t)E * d, I, 128, &wd, true));
  DG_TRY(tmap(m, hb, ws.max_rows, I, 32, &h));
  cudaError_t e = launch_pdl((tc_moe_f8_kernel<MOE8_ST>), state(m)->n_sm, TC_F8_THREADS,
                             MoeF8Cfg<MOE8_ST>::smem_bytes(d, I), st, 1, wg, wu, x, wd, h,
                             (const float*)L.gate_scale, (const float*)L.up_scale,
                             (const float*)L.down_scale, ws.tile_e, ws.tile_m0, ws.n_tiles,
                             ws.offsets, I, d, hb, yb, (const float*)ws.gate_of, ws.ready,
                             ws.ready + ws.max_tiles, ws.err);
  ++m->launches;
  if (e != cudaSuccess) {
    set_error("tc_moe_f8 launch: %s", cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

// NVFP4 expert weights (packed E2M1 codes [rows, K / 2] bytes, E4M3 block scales
// [rows, K / 16], one fp32 tensor scale per matrix): the same persistent launch with the
// NVFP4 converter
dg_status tc_moe_experts_f4(dg_model* m, int l, const bf16* X, bf16* hb, float* yb,
                            cudaStream_t st) {
  const dg_config& c = m->cfg;
  const dg_layer_weights& L = m->layers[l];
  const int E = c.n_experts, I = c.expert_inter, d = c.d_model;
  const Workspace& ws = m->ws;
  CUtensorMap wg, wu, x, wd, h;
  DG_TRY(tmap(m, L.gate, (uint64_t)E * I, d / 2, 128, &wg, true, 32));
  DG_TRY(tmap(m, L.up, (uint64_t)E * I, d / 2, 128, &wu, true, 32));
  DG_TRY(tmap(m, X, ws.max_rows, d, 32, &x));
  DG_TRY(tmap(m, L.down, (uint64_t)E * d, I / 2, 128, &wd, true, 32));
  DG_TRY(tmap(m, hb, ws.max_rows, I, 32, &h));
  F4Scales sc{(const uint8_t*)L.gate_scale, (const uint8_t*)L.up_scale,
              (const uint8_t*)L.down_scale, L.gate_tscale, L.up_tscale, L.down_tscale};
  cudaError_t e = launch_pdl((tc_moe_f4_kernel<MOE8_ST>), state(m)->n_sm, TC_F8_THREADS,
                             MoeLowpCfg<MOE8_ST, true>::smem_bytes(d, I), st, 1, wg, wu, x, wd,
                             h, sc, ws.tile_e, ws.tile_m0, ws.n_tiles, ws.offsets, I, d, hb, yb,
                             (const float*)ws.gate_of, ws.ready, ws.ready + ws.max_tiles, ws.err);
  ++m->launches;
  if (e != cudaSuccess) {
    set_error("tc_moe_f4 launch: %s", cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

// bf16 expert weights: both phases in one persistent launch (tc_moe_kernel)
dg_status tc_moe_experts(dg_model* m, int l, const bf16* X, bf16* hb, float* yb,
                         cudaStream_t st) {
  const dg_config& c = m->cfg;
  const dg_layer_weights& L = m->layers[l];
  const int E = c.n_experts, I = c.expert_inter, d = c.d_model;
  const Workspace& ws = m->ws;
  CUtensorMap wg, wu, x, wd, h;
  DG_TRY(tmap(m, L.gate, (uint64_t)E * I, d, 128, &wg));
  DG_TRY(tmap(m, L.up, (uint64_t)E * I, d, 128, &wu));
  DG_TRY(tmap(m, X, ws.max_rows, d, 32, &x));
  DG_TRY(tmap(m, L.down, (uint64_t)E * d, I, 128, &wd));
  DG_TRY(tmap(m, hb, ws.max_rows, I, 32, &h));
  cudaError_t e = launch_pdl((tc_moe_kernel<MOE_ST>), state(m)->n_sm, TC_MOE_THREADS,
                             MoeCfg<MOE_ST>::SMEM, st, 1, wg, wu, x, wd, h, ws.tile_e,
                             ws.tile_m0, ws.n_tiles, ws.offsets, I, d, hb, yb,
                             (const float*)ws.gate_of, ws.ready, ws.ready + ws.max_tiles,
                             ws.err, (uint64_t)(m->stall_limit_ns > 0 ? m->stall_limit_ns
                                                                      : 2000000000ll),
                             m->stall_limit_ns > 0 ? 1 : 0);
  m->stall_limit_ns = 0;  // one launch only
  ++m->launches;
  if (e != cudaSuccess) {
    set_error("tc_moe launch: %s", cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

dg_status tc_attention(dg_model* m, const bf16* q, int B, int nq, int qpos0, const dg_kv* kv,
                       int l, const bf16* kB, const bf16* vB, int nB, int kposB, int npB,
                       bool causal, bf16* out, cudaStream_t st) {
  const dg_config& c = m->cfg;
  const int Hq = c.n_q_heads, Hkv = c.n_kv_heads, h = c.head_dim;
  if (h != 128) {
    set_error("tensor-core attention needs head_dim 128");
    return DG_ERR_UNSUPPORTED;
  }
  CUtensorMap mQ, mKA, mVA, mKB, mVB;
  DG_TRY(tmap(m, q, m->ws.max_tok, (uint64_t)Hq * h, 128, &mQ));
  DG_TRY(tmap(m, kB, (uint64_t)B * Hkv * npB, h, 128, &mKB));
  DG_TRY(tmap(m, vB, (uint64_t)B * Hkv * h, npB, 128, &mVB));
  AttnParams p{};
  if (kv) {
    DG_TRY(tmap(m, kv->k, (uint64_t)c.n_layers * kv->B * Hkv * kv->Wp, h, 128, &mKA));
    DG_TRY(tmap(m, kv->v, (uint64_t)c.n_layers * kv->B * Hkv * h, kv->Wp, 128, &mVA));
    p.nA = kv->W;
    p.kposA = kv->P - kv->W;
    p.rowsA = kv->Wp;
    p.layer_rowA = l * kv->B * Hkv * kv->Wp;
    p.layer_vrowA = l * kv->B * Hkv * h;
  } else {
    mKA = mKB;
    mVA = mVB;
  }
  p.nq = nq;
  p.qpos0 = qpos0;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.nB = nB;
  p.kposB = kposB;
  p.rowsB = npB;
  p.causal = causal ? 1 : 0;
  p.window = c.window;
  p.B = B;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)h));
  p.out = out;
  const int TA = ceil_div_i(p.nA, AT_KT), TB = ceil_div_i(nB, AT_KT);
  // causal: a query tile reaches window + 127 key positions, which meet at most that
  // many tiles of each segment's grid plus one where the grids change
  const int total = causal ? std::min(TA + TB, ceil_div_i(c.window + 127, AT_KT) + 2) : TA + TB;
  const int qtiles = ceil_div_i(nq, 128);
  const int base = qtiles * Hq * B;
  const int n_sm = state(m)->n_sm;
  // one wave: CTAs (one per SM, ~196 KB of shared memory each) never exceed the SM
  // count; the key splits of a query tile form a cluster (a power of two <= 8, so
  // that each owns 128 / splits rows of the merge)
  const int cap = std::min(std::max(1, n_sm / base), std::min((int)ATT_MAX_SPLITS, total));
  int splits = 1;
  while (splits * 2 <= cap) splits *= 2;
  p.tiles_per_split = ceil_div_i(total, splits);
  dim3 grid(qtiles * Hq, B, splits);
  launch_pdl((tc_attn_kernel), grid, AT_THREADS, AT_SMEM, st, splits, mQ, mKA, mVA, mKB, mVB, p,
             m->ws.err);
  ++m->launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("tc_attention launch: %s", cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

}  // namespace dg
