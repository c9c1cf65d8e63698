// libdg: host side of the C-ABI (include/dg.h) — validation, workspace, and
// the launch sequence of the causal prompt pass and the canvas denoise forward.
//
// Launch sequence of one canvas forward (batch B, canvas C, prompt window W):
//   embed + timestep  ->  per layer { RMSNorm -> QKV GEMM -> RoPE/scatter ->
//   attention over [window | canvas] -> O GEMM (+residual) -> RMSNorm ->
//   router -> permute -> grouped gate/up GEMM (SwiGLU) -> grouped down GEMM
//   (x gate) -> shared expert -> combine (+residual) }  ->  RMSNorm -> LM-head
//   statistics -> merge  ->  EB sampler.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "dg_internal.h"
#include "../../include/dg_ops.h"
#include "k_sampler.cuh"
#include "k_simt.cuh"
#include "k_tc_gemm.cuh"

namespace dg {

static thread_local std::string g_err;

void set_error(const char* fmt, ...) {
  char buf[1024];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
}

static dg_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("%s: %s", what, cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

// ---------------------------------------------------------------------------
// precision paths
// ---------------------------------------------------------------------------
struct PathTiny {  // fp32 weights, fp64 activations and sums
  typedef float TW;
  typedef double TA, Acc, TR, TKV;
  static constexpr bool kTensorCores = false;
};
struct PathBF16 {  // bf16 weights/activations, fp32 residual and sums
  typedef bf16 TW, TA, TKV;
  typedef float Acc, TR;
  static constexpr bool kTensorCores = true;
};

static int ceil_div(long a, long b) { return (int)((a + b - 1) / b); }

template <class T> static dg_status ws_alloc(Workspace& ws, T** p, size_t n) {
  void* q = nullptr;
  const size_t bytes = std::max<size_t>(n, 1) * sizeof(T);
  cudaError_t e = cudaMalloc(&q, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    set_error("workspace allocation of %zu bytes failed: %s", bytes, cudaGetErrorString(e));
    return DG_ERR_OOM;
  }
  ws.bufs.push_back({q, bytes});
  *p = static_cast<T*>(q);
  return DG_OK;
}
template <class T> static dg_status ws_alloc_v(Workspace& ws, void** p, size_t n) {
  T* q = nullptr;
  DG_TRY(ws_alloc(ws, &q, n));
  *p = q;
  return DG_OK;
}

static void ws_free(Workspace& ws) {
  for (auto& b : ws.bufs) cudaFree(b.p);
  ws.bufs.clear();
}

__global__ void rope_table_kernel(double base, int h, int max_pos, void* out, int as_double) {
  pdl_enter();
  const int half = h / 2;
  const long n = (long)max_pos * half;
  for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < n;
       e += (long)gridDim.x * blockDim.x) {
    const int pos = (int)(e / half), j = (int)(e % half);
    const double theta = pow(base, -2.0 * (double)j / (double)h);
    const double a = (double)pos * theta;
    const double c = cos(a), s = sin(a);
    if (as_double) {
      ((double*)out)[e] = c;
      ((double*)out)[n + e] = s;
    } else {
      ((float*)out)[e] = (float)c;
      ((float*)out)[n + e] = (float)s;
    }
  }
}

template <class Path> static dg_status alloc_workspace(dg_model* m) {
  typedef typename Path::TW TW;
  typedef typename Path::TA TA;
  typedef typename Path::Acc Acc;
  typedef typename Path::TR TR;
  typedef typename Path::TKV TKV;
  const dg_config& c = m->cfg;
  Workspace& ws = m->ws;
  const size_t d = c.d_model, h = c.head_dim;
  const size_t T = std::max<size_t>((size_t)c.max_batch * c.canvas, (size_t)c.max_prompt);
  const size_t R = T * c.top_k;
  ws.max_tok = T;
  ws.max_rows = R;
  ws.max_tiles = ceil_div((long)R, SG_BM) + c.n_experts + 1;
  ws.n_vtiles = ceil_div(c.vocab, SG_BN);
  ws.max_pos = c.max_prompt + c.canvas;
  const size_t qkv = (size_t)(c.n_q_heads + 2 * c.n_kv_heads) * h;
  DG_TRY(ws_alloc_v<TR>(ws, &ws.x, T * d));
  DG_TRY(ws_alloc_v<TA>(ws, &ws.xn, T * d));
  DG_TRY(ws_alloc_v<Acc>(ws, &ws.qkv, T * qkv));
  DG_TRY(ws_alloc_v<TA>(ws, &ws.q, T * c.n_q_heads * h));
  DG_TRY(ws_alloc_v<TA>(ws, &ws.o, T * c.n_q_heads * h));
  // own keys [B, Hkv, np, h] and transposed values [B, Hkv, h, np], np = n rounded up to 64
  const size_t T_pad = T + 64 * (size_t)c.max_batch;
  DG_TRY(ws_alloc_v<TKV>(ws, &ws.kc, T_pad * c.n_kv_heads * h));
  DG_TRY(ws_alloc_v<TKV>(ws, &ws.vc, T_pad * c.n_kv_heads * h));
  ws.kc_elems = T_pad * c.n_kv_heads * h;
  DG_TRY(ws_alloc_v<Acc>(ws, &ws.ys, T * d));
  DG_TRY(ws_alloc_v<TA>(ws, &ws.sh, T * c.shared_inter));
  DG_TRY(ws_alloc(ws, &ws.ridx, R));
  DG_TRY(ws_alloc(ws, &ws.rank, R));
  DG_TRY(ws_alloc(ws, &ws.row_of, R));
  DG_TRY(ws_alloc(ws, &ws.tok_of, R));
  DG_TRY(ws_alloc_v<Acc>(ws, &ws.rgate, R));
  DG_TRY(ws_alloc_v<Acc>(ws, &ws.gate_of, R));
  DG_TRY(ws_alloc_v<Acc>(ws, &ws.inv_rms, T));
  if constexpr (Path::kTensorCores) DG_TRY(ws_alloc_v<TA>(ws, &ws.u2, T * 2 * d));
  DG_TRY(ws_alloc_v<Acc>(ws, &ws.rlog, std::max<size_t>(4096, T) * c.n_experts));
  DG_TRY(ws_alloc(ws, &ws.counts, c.n_experts));
  DG_TRY(ws_alloc(ws, &ws.offsets, c.n_experts + 1));
  DG_TRY(ws_alloc(ws, &ws.tile_e, ws.max_tiles));
  DG_TRY(ws_alloc(ws, &ws.ready, ws.max_tiles + 1));  // + the expert kernel's unit counter
  DG_TRY_CUDA(cudaMemset(ws.ready, 0, (ws.max_tiles + 1) * sizeof(int32_t)));
  DG_TRY(ws_alloc(ws, &ws.tile_m0, ws.max_tiles));
  DG_TRY(ws_alloc(ws, &ws.n_tiles, 1));
  DG_TRY(ws_alloc_v<TA>(ws, &ws.up, R * d));
  DG_TRY(ws_alloc_v<TA>(ws, &ws.hb, R * c.expert_inter));
  DG_TRY(ws_alloc_v<Acc>(ws, &ws.yb, R * d));
  const size_t lm_rows = (size_t)c.max_batch * c.canvas;
  DG_TRY(ws_alloc_v<Acc>(ws, &ws.lm_part, (size_t)ws.n_vtiles * lm_rows * 4));
  DG_TRY(ws_alloc(ws, &ws.err, 4));
  DG_TRY(ws_alloc(ws, &ws.units, 1));
  DG_TRY_CUDA(cudaMemset(ws.units, 0, sizeof(unsigned long long)));
  DG_TRY(ws_alloc(ws, &ws.ids, T));
  DG_TRY(ws_alloc_v<Acc>(ws, &ws.rope, (size_t)2 * ws.max_pos * (h / 2)));
  DG_TRY(ws_alloc(ws, &ws.mask, lm_rows));
  DG_TRY(ws_alloc(ws, &ws.ent, lm_rows));
  DG_TRY(ws_alloc(ws, &ws.amax, lm_rows));
  DG_TRY(ws_alloc(ws, &ws.ncommit, c.max_batch));
  DG_TRY(ws_alloc(ws, &ws.remaining, c.max_batch));
  DG_TRY(ws_alloc(ws, &ws.loop_s, 1));
  DG_TRY(ws_alloc(ws, &ws.blk, lm_rows));
  DG_TRY(ws_alloc(ws, &ws.sampled, lm_rows));
  DG_TRY(ws_alloc(ws, &ws.prev, lm_rows));
  DG_TRY(ws_alloc(ws, &ws.astate, c.max_batch));
  DG_TRY(ws_alloc_v<Acc>(ws, &ws.gpart, (size_t)ws.n_vtiles * lm_rows * 2));
  if (c.sc_inter > 0) {
    DG_TRY(ws_alloc_v<TW>(ws, &ws.embT, d * c.vocab));
    DG_TRY(ws_alloc_v<TA>(ws, &ws.scP, lm_rows * c.vocab));
    DG_TRY(ws_alloc_v<Acc>(ws, &ws.scref, (size_t)ws.n_vtiles * lm_rows * 2));
    DG_TRY(ws_alloc_v<TA>(ws, &ws.scy, T * d));  // max_tok rows: the GEMMs' A extent
    DG_TRY(ws_alloc_v<TA>(ws, &ws.sch, T * c.sc_inter));
    if constexpr (Path::kTensorCores)
      DG_TRY(ws_alloc(ws, &ws.scpart, (size_t)SC_MAX_PARTS * lm_rows * d));
    DG_TRY(ws_alloc_v<Acc>(ws, &ws.z, lm_rows * d));
    dim3 tg(ceil_div(c.vocab, 32), ceil_div((long)d, 32));
    transpose_emb_kernel<TW><<<tg, dim3(32, 8)>>>((const TW*)m->w.tok_emb, (TW*)ws.embT,
                                                  c.vocab, (int)d);
    DG_TRY(check_launch("embedding transpose"));
  }
  DG_TRY_CUDA(cudaMemset(ws.err, 0, 4 * sizeof(int32_t)));
  launch_pdl((rope_table_kernel), 256, 256, 0, cudaStream_t(0), 1, (double)c.rope_base, (int)h, ws.max_pos, ws.rope,
                                  sizeof(Acc) == 8 ? 1 : 0);
  DG_TRY(check_launch("rope table"));
  if constexpr (Path::kTensorCores) {
    DG_TRY(tc_prepare(m));
    DG_TRY_CUDA(cudaStreamCreateWithFlags(&m->side_stream, cudaStreamNonBlocking));
    DG_TRY_CUDA(cudaEventCreateWithFlags(&m->fork_ev, cudaEventDisableTiming));
    DG_TRY_CUDA(cudaEventCreateWithFlags(&m->join_ev, cudaEventDisableTiming));
  }
  DG_REQUIRE(permute_smem_bytes(c.n_experts, 1024, 0) <= PERMUTE_FUSED_SMEM,
             "n_experts too large for the permutation");
  DG_TRY_CUDA(cudaFuncSetAttribute(moe_permute_gather_kernel<Acc, TA>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)PERMUTE_FUSED_SMEM));
  DG_TRY_CUDA(cudaFuncSetAttribute(moe_permute_kernel<Acc>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)PERMUTE_FUSED_SMEM));
  {
    int dev = 0, n_sm = 0;
    DG_TRY_CUDA(cudaGetDevice(&dev));
    DG_TRY_CUDA(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
    m->n_sm_cache = n_sm;
  }
  DG_TRY_CUDA(cudaDeviceSynchronize());
  return DG_OK;
}

// ---------------------------------------------------------------------------
// GEMM dispatch: tcgen05 for bf16 dense contractions, CUDA cores otherwise
// ---------------------------------------------------------------------------
template <class TA, class TW, class Acc, bool G, bool D, class Epi>
static void gemm_simt(const TA* A, int lda, const TW* W, const TW* W2, int ldw, int M, int N,
                      int K, GroupInfo g, int grid_y, Epi epi, cudaStream_t st,
                      long long* count) {
  dim3 grid(ceil_div(N, SG_BN), G ? grid_y : ceil_div(M, SG_BM));
  launch_pdl((gemm_simt_kernel<TA, TW, Acc, G, D, Epi>), grid, 256, 0, st, 1, A, lda, W, W2, ldw, M, N, K, g, epi);
  ++*count;
}

template <class Path> struct Runner {
  typedef typename Path::TW TW;
  typedef typename Path::TA TA;
  typedef typename Path::Acc Acc;
  typedef typename Path::TR TR;
  typedef typename Path::TKV TKV;

  dg_model* m;
  const dg_config& c;
  Workspace& ws;
  cudaStream_t st;
  const int32_t* s_dev = nullptr;  // steps left in device memory (captured block loop)
  Runner(dg_model* m_, cudaStream_t st_, const int32_t* s_dev_ = nullptr)
      : m(m_), c(m_->cfg), ws(m_->ws), st(st_), s_dev(s_dev_) {}

  TR* x() { return (TR*)ws.x; }
  TA* xn() { return (TA*)ws.xn; }

  void rmsnorm(int n) {
    launch_pdl((rmsnorm_kernel<TR, TA, Acc>), n, 256, 0, st, 1, x(), xn(), n, c.d_model, c.rms_eps,
               (Acc*)nullptr, (TA*)nullptr);
    ++m->launches;
  }

  // y[n, N] (+)= xn W^T  with W [N, K]
  template <class Epi> void dense(const TA* A, int lda, const void* W, int N, int K, int n,
                                  Epi epi) {
    gemm_simt<TA, TW, Acc, false, false>(A, lda, (const TW*)W, nullptr, K, n, N, K, GroupInfo(),
                                         0, epi, st, &m->launches);
  }

  // One decoder layer on n tokens = B_ * n_seq rows at positions pos0 + i.
  // Segment A (the cached window, denoise only): keys [L, B, Hkv, WpA, h] and transposed
  // values [L, B, Hkv, h, WpA] of `kv`, nA valid keys at positions kposA...
  // xn holds RMSNorm(x) on entry for l > 0 (the previous layer's combine writes it).
  dg_status layer(int l, int n, int B_, int n_seq, int pos0, const dg_kv* kv, bool causal,
                  int32_t* load) {
    const int nA = kv ? kv->W : 0, kposA = kv ? kv->P - kv->W : 0, WpA = kv ? kv->Wp : 0;
    const int np = (n_seq + 63) / 64 * 64;
    const dg_layer_weights& L = m->layers[l];
    const int d = c.d_model, h = c.head_dim, Hq = c.n_q_heads, Hkv = c.n_kv_heads;
    const int qkv_n = (Hq + 2 * Hkv) * h;
    if (l == 0) {
      ProfScope ps(m, DG_KIND_GLUE, st);
      rmsnorm(n);
    }
    bool fused_rope = false;
    {
      ProfScope ps(m, DG_KIND_DENSE, st);
      if constexpr (Path::kTensorCores) {
        if (h == 128) {  // RoPE and the q / k / v scatter in the GEMM epilogue
          DG_TRY(tc_gemm_qkv_rope(m, xn(), L.wqkv, n, n_seq, np, pos0, (bf16*)ws.q,
                                  (bf16*)ws.kc, (bf16*)ws.vc, st));
          fused_rope = true;
        } else {
          DG_TRY(tc_gemm_store_f32(m, xn(), L.wqkv, (float*)ws.qkv, n, qkv_n, d, st));
        }
      } else {
        dense(xn(), d, L.wqkv, qkv_n, d, n, EpiStore<Acc, Acc>{(Acc*)ws.qkv, qkv_n});
      }
    }
    if (!fused_rope) {
      launch_pdl((rope_scatter_kernel<Acc, TA, TKV>), n, 128, 0, st, 1,
          (const Acc*)ws.qkv, (TA*)ws.q, (TKV*)ws.kc, (TKV*)ws.vc, n, n_seq, np, pos0, Hq, Hkv, h,
          (const Acc*)ws.rope, ws.max_pos);
      ++m->launches;
    }
    {
      ProfScope ps(m, DG_KIND_ATTENTION, st);
      bool done = false;
      if constexpr (Path::kTensorCores) {
        if (h == 128) {
          DG_TRY(tc_attention(m, (const bf16*)ws.q, B_, n_seq, pos0, kv, l, (const bf16*)ws.kc,
                              (const bf16*)ws.vc, n_seq, pos0, np, causal, (bf16*)ws.o, st));
          done = true;
        }
      }
      if (!done) {
        const long warps = (long)n * Hq;
        const int blocks = ceil_div(warps, 4);
        const size_t lstride = kv ? (size_t)kv->B * Hkv * kv->Wp * h : 0;
        const TKV* kA = kv ? (const TKV*)kv->k + l * lstride : nullptr;
        const TKV* vA = kv ? (const TKV*)kv->v + l * lstride : nullptr;
        const TKV* kB = (const TKV*)ws.kc;
        const TKV* vB = (const TKV*)ws.vc;
#define DG_ATTN(DPL)                                                                            \
  launch_pdl((attention_simt_kernel<TA, TKV, Acc, DPL>), blocks, 128, 0, st, 1,                              \
      (const TA*)ws.q, (TA*)ws.o, kA, vA, nA, WpA, kposA, kB, vB, n_seq, np, pos0, B_, n_seq,  \
      pos0, Hq, Hkv, h, causal ? 1 : 0, c.window)
        if (h <= 32) DG_ATTN(1);
        else if (h <= 64) DG_ATTN(2);
        else if (h <= 96) DG_ATTN(3);
        else DG_ATTN(4);
        ++m->launches;
#undef DG_ATTN
      }
    }
    {
      ProfScope ps(m, DG_KIND_DENSE, st);
      if constexpr (Path::kTensorCores)
        DG_TRY(tc_gemm_add_residual(m, (const TA*)ws.o, L.wo, (float*)x(), n, d, Hq * h, st));
      else
        dense((const TA*)ws.o, Hq * h, L.wo, d, Hq * h, n, EpiAddResidual<TR, Acc>{x(), d});
    }
    DG_TRY(moe(l, n, load));
    return check_launch("decoder layer");
  }

  dg_status moe(int l, int n, int32_t* load) {
    const dg_layer_weights& L = m->layers[l];
    const int d = c.d_model, E = c.n_experts, k = c.top_k, I = c.expert_inter;
    const int Is = c.shared_inter;
    const int n_ent = n * k;
    // u = RMSNorm(x) after attention (bf16 copy for the expert GEMMs, 1/rms for the
    // CUDA-core router, the two-term split for the tensor-core router)
    bool tc_router = false;
    if constexpr (Path::kTensorCores) tc_router = E <= 128 && k <= 8 && d % 64 == 0;
    int bm = SG_BM;
    if constexpr (Path::kTensorCores) bm = tc_group_rows();
    PermuteArgs pa{(const int32_t*)ws.ridx, n_ent, k, E, bm, ws.rank, ws.offsets, ws.tile_e,
                   ws.tile_m0, ws.n_tiles, ws.max_tiles, ws.units, load, ws.row_of, ws.tok_of,
                   ws.ready};
    {
      ProfScope ps(m, DG_KIND_ROUTING, st);
      launch_pdl((rmsnorm_kernel<TR, TA, Acc>), n, 256, 0, st, 1, x(), xn(), n, d, c.rms_eps,
                 (Acc*)ws.inv_rms, tc_router ? (TA*)ws.u2 : (TA*)nullptr);
      ++m->launches;
    }
    if constexpr (Path::kTensorCores) {
      // shared expert on the side stream, concurrent with routing and the routed experts
      cudaStream_t side = m->side_stream;
      DG_TRY_CUDA(cudaEventRecord(m->fork_ev, st));
      DG_TRY_CUDA(cudaStreamWaitEvent(side, m->fork_ev, 0));
      {
        ProfScope ps(m, DG_KIND_SHARED, side);
        DG_TRY(tc_gemm_swiglu(m, xn(), L.sgate, L.sup, (TA*)ws.sh, n, Is, d, side));
        DG_TRY(tc_gemm_store_f32(m, (const TA*)ws.sh, L.sdown, (float*)ws.ys, n, d, Is, side));
      }
      DG_TRY_CUDA(cudaEventRecord(m->join_ev, side));
      if (tc_router) {
        ProfScope ps(m, DG_KIND_ROUTING, st);
        DG_TRY(tc_router_topk(m, (const bf16*)ws.u2, L.router, n, ws.ridx, (float*)ws.rgate, st));
      }
    }
    if (!tc_router) {
      const int splits = std::max(1, std::min(16, 4096 / n));
      const int kps = ceil_div(ceil_div(d, splits), 32) * 32;
      const int ks = ceil_div(d, kps);
      dim3 grid(ceil_div(n, 32), ks, ceil_div(E, 128));
      launch_pdl((router_logits_kernel<TR, TW, Acc>), grid, 256, 0, st, 1, x(), (const TW*)L.router, n, d, E,
                                                              kps, (Acc*)ws.rlog);
      ++m->launches;
      if (E <= 32)
        launch_pdl((router_topk_kernel<Acc, 1>), ceil_div(n, 4), 128, 0, st, 1,
            (const Acc*)ws.rlog, ks, (const Acc*)ws.inv_rms, n, E, k, ws.ridx, (Acc*)ws.rgate,
            (int32_t*)nullptr);
      else if (E <= 128)
        launch_pdl((router_topk_kernel<Acc, 4>), ceil_div(n, 4), 128, 0, st, 1,
            (const Acc*)ws.rlog, ks, (const Acc*)ws.inv_rms, n, E, k, ws.ridx, (Acc*)ws.rgate,
            (int32_t*)nullptr);
      else
        launch_pdl((router_topk_kernel<Acc, 32>), ceil_div(n, 4), 128, 0, st, 1,
            (const Acc*)ws.rlog, ks, (const Acc*)ws.inv_rms, n, E, k, ws.ridx, (Acc*)ws.rgate,
            (int32_t*)nullptr);
      ++m->launches;
    }
    ProfScope pperm(m, DG_KIND_ROUTING, st);
    if (permute_smem_bytes(E, 1024, n_ent) <= PERMUTE_FUSED_SMEM) {
      // every block derives the permutation in shared memory and gathers its rows
      const int blocks = std::max(1, std::min(n_ent, m->n_sm_cache));
      launch_pdl((moe_permute_gather_kernel<Acc, TA>), blocks, 1024,
                 permute_smem_bytes(E, 1024, n_ent), st, 1, pa, (const Acc*)ws.rgate,
                 (Acc*)ws.gate_of, (const TA*)xn(), d, (TA*)ws.up);
      ++m->launches;
    } else {
      launch_pdl((moe_permute_kernel<Acc>), 1, 1024, permute_smem_bytes(E, 1024, 0), st, 1, pa,
                 (const Acc*)ws.rgate, (Acc*)ws.gate_of);
      ++m->launches;
      launch_pdl((gather_rows_kernel<TA>), n_ent, 256, 0, st, 1, xn(), ws.tok_of,
                 ws.offsets + E, d, (TA*)ws.up);
      ++m->launches;
    }
    pperm.end();
    const int grid_y = ceil_div(n_ent, bm) + E;
    if constexpr (Path::kTensorCores) {
      {
        ProfScope ps(m, DG_KIND_EXPERTS, st);
        if (c.dtype == DG_BF16_FP4EXP) {
          DG_TRY(tc_moe_experts_f4(m, l, (const TA*)ws.up, (TA*)ws.hb, (float*)ws.yb, st));
        } else if (c.dtype == DG_BF16_FP8EXP) {
          DG_TRY(tc_moe_experts_f8(m, l, (const TA*)ws.up, (TA*)ws.hb, (float*)ws.yb, st));
        } else {
          DG_TRY(tc_moe_experts(m, l, (const TA*)ws.up, (TA*)ws.hb, (float*)ws.yb, st));
        }
      }
      DG_TRY_CUDA(cudaStreamWaitEvent(st, m->join_ev, 0));  // shared expert done
    } else {
      GroupInfo g;
      g.tile_e = ws.tile_e;
      g.tile_m0 = ws.tile_m0;
      g.n_tiles = ws.n_tiles;
      g.offsets = ws.offsets;
      g.w_slab = (size_t)I * d;
      ProfScope pe(m, DG_KIND_EXPERTS, st);
      gemm_simt<TA, TW, Acc, true, true>((const TA*)ws.up, d, (const TW*)L.gate,
                                         (const TW*)L.up, d, n_ent, I, d, g, grid_y,
                                         EpiSwiglu<TA, Acc>{(TA*)ws.hb, I}, st, &m->launches);
      gemm_simt<TA, TW, Acc, true, false>(
          (const TA*)ws.hb, I, (const TW*)L.down, nullptr, I, n_ent, d, I, g, grid_y,
          EpiRowScale<Acc, Acc>{(Acc*)ws.yb, d, (const Acc*)ws.gate_of}, st, &m->launches);
      pe.end();
      ProfScope pd(m, DG_KIND_DENSE, st);
      gemm_simt<TA, TW, Acc, false, true>(xn(), d, (const TW*)L.sgate, (const TW*)L.sup, d, n,
                                          Is, d, GroupInfo(), 0,
                                          EpiSwiglu<TA, Acc>{(TA*)ws.sh, Is}, st, &m->launches);
      dense((const TA*)ws.sh, Is, L.sdown, d, Is, n, EpiStore<Acc, Acc>{(Acc*)ws.ys, d});
    }
    // residual update fused with the next RMSNorm (next layer's input or the LM head's)
    ProfScope pg(m, DG_KIND_GLUE, st);
    launch_pdl((moe_combine_norm_kernel<TR, TA, Acc, Acc>), n, 256, 0, st, 1, x(),
               (const Acc*)ws.ys, (const Acc*)ws.yb, (const int32_t*)ws.row_of, n, d, k,
               c.rms_eps, xn());
    ++m->launches;
    return check_launch("moe");
  }

  dg_status moe_op(int l, const float* x_in, float* out, int n) {
    const size_t d = c.d_model;
    if constexpr (sizeof(TR) == sizeof(float)) {
      DG_TRY_CUDA(cudaMemcpyAsync(x(), x_in, n * d * sizeof(float), cudaMemcpyDeviceToDevice, st));
    } else {
      launch_pdl((widen_f32_kernel<TR>), ceil_div((long)n * d, 256), 256, 0, st, 1, x_in, x(), (long)n * d);
      ++m->launches;
    }
    DG_TRY(moe(l, n, nullptr));
    launch_pdl((to_f32_kernel<TR>), ceil_div((long)n * d, 256), 256, 0, st, 1, x(), out, (long)n * d);
    ++m->launches;
    return check_launch("moe op");
  }

  // Prompt pass for each batch element, keeping the last W keys/values per layer.
  dg_status prefill(const int32_t* prompt, int B, int P, dg_kv* kv) {
    const int d = c.d_model, h = c.head_dim, Hkv = c.n_kv_heads;
    const int W = kv->W, Wp = kv->Wp;
    const int Pp = (P + 63) / 64 * 64;
    const size_t es = sizeof(TKV);
    for (int b = 0; b < B; ++b) {
      launch_pdl((embed_kernel<TW, TR, Acc>), P, 256, 0, st, 1, prompt + (size_t)b * P, (const TW*)m->w.tok_emb,
                                             x(), P, d, c.vocab - 1, -1.0, ws.err,
                                             (const int32_t*)nullptr, 1, (const Acc*)nullptr);
      ++m->launches;
      // padding columns of the transposed values must read as zero
      DG_TRY_CUDA(cudaMemsetAsync(ws.vc, 0, (size_t)Hkv * h * Pp * es, st));
      for (int l = 0; l < c.n_layers; ++l) {
        DG_TRY(layer(l, P, 1, P, 0, nullptr, true, nullptr));
        // keys [hkv, P-W .. P-1, :] -> cache K [l, b, hkv, 0 .. W-1, :]
        char* kdst = (char*)kv->k + (((size_t)l * kv->B + b) * Hkv) * (size_t)Wp * h * es;
        DG_TRY_CUDA(cudaMemcpy2DAsync(kdst, (size_t)Wp * h * es,
                                      (const char*)ws.kc + (size_t)(P - W) * h * es,
                                      (size_t)Pp * h * es, (size_t)W * h * es, Hkv,
                                      cudaMemcpyDeviceToDevice, st));
        // transposed values [hkv, :, P-W .. P-1] -> cache V^T [l, b, hkv, :, 0 .. W-1]
        char* vdst = (char*)kv->v + (((size_t)l * kv->B + b) * Hkv) * (size_t)h * Wp * es;
        DG_TRY_CUDA(cudaMemcpy2DAsync(vdst, (size_t)Wp * es,
                                      (const char*)ws.vc + (size_t)(P - W) * es, (size_t)Pp * es,
                                      (size_t)W * es, (size_t)Hkv * h, cudaMemcpyDeviceToDevice,
                                      st));
      }
    }
    return check_launch("prefill");
  }

  // Causal pass of B finished blocks (tokens [B, C], positions P .. P + C - 1) over the
  // cached window: per layer the block's rows attend to the cached keys and to their
  // own earlier rows within the sliding window (the same computation the prompt pass
  // would have made had the block been part of the prompt); then each layer's window
  // becomes the last min(W + C, window) positions of (window, block).  No LM head.
  dg_status append(const int32_t* tokens, dg_kv* kv) {
    const int B = kv->B, C = c.canvas, n = B * C, d = c.d_model, h = c.head_dim;
    const int Hkv = c.n_kv_heads;
    const int np = (C + 63) / 64 * 64;
    const size_t es = sizeof(TKV);
    launch_pdl((embed_kernel<TW, TR, Acc>), n, 256, 0, st, 1, tokens, (const TW*)m->w.tok_emb, x(), n,
               d, c.vocab - 1, -1.0, ws.err, (const int32_t*)nullptr, 1, (const Acc*)nullptr);
    ++m->launches;
    // padding columns of the block's transposed values must read as zero
    if (np != C) DG_TRY_CUDA(cudaMemsetAsync(ws.vc, 0, (size_t)B * Hkv * h * np * es, st));
    const int W = kv->W, Wn = std::min(W + C, c.window);
    const int keep = std::max(0, Wn - C);          // cached positions that stay
    const int take = std::min(C, Wn);              // block positions that enter
    const size_t slabK = (size_t)kv->Wp * h * es;  // one (b, g) slab of keys
    const size_t rowV = (size_t)kv->Wp * es;       // one (b, g, dim) row of values^T
    TKV* tmp = (TKV*)ws.up;                        // scratch: the kept part of a layer
    for (int l = 0; l < c.n_layers; ++l) {
      DG_TRY(layer(l, n, B, C, kv->P, kv, true, nullptr));
      char* K = (char*)kv->k + (size_t)l * B * Hkv * slabK;
      char* V = (char*)kv->v + (size_t)l * B * Hkv * h * rowV;
      if (keep > 0 && W - keep > 0) {  // shift the kept positions to the front (via scratch)
        DG_TRY_CUDA(cudaMemcpy2DAsync(tmp, (size_t)keep * h * es, K + (size_t)(W - keep) * h * es,
                                      slabK, (size_t)keep * h * es, (size_t)B * Hkv,
                                      cudaMemcpyDeviceToDevice, st));
        DG_TRY_CUDA(cudaMemcpy2DAsync(K, slabK, tmp, (size_t)keep * h * es,
                                      (size_t)keep * h * es, (size_t)B * Hkv,
                                      cudaMemcpyDeviceToDevice, st));
        DG_TRY_CUDA(cudaMemcpy2DAsync(tmp, (size_t)keep * es, V + (size_t)(W - keep) * es, rowV,
                                      (size_t)keep * es, (size_t)B * Hkv * h,
                                      cudaMemcpyDeviceToDevice, st));
        DG_TRY_CUDA(cudaMemcpy2DAsync(V, rowV, tmp, (size_t)keep * es, (size_t)keep * es,
                                      (size_t)B * Hkv * h, cudaMemcpyDeviceToDevice, st));
      }
      // the block's last `take` keys [B, Hkv, np, h] and values^T [B, Hkv, h, np] after them
      DG_TRY_CUDA(cudaMemcpy2DAsync(K + (size_t)keep * h * es, slabK,
                                    (const char*)ws.kc + (size_t)(C - take) * h * es,
                                    (size_t)np * h * es, (size_t)take * h * es, (size_t)B * Hkv,
                                    cudaMemcpyDeviceToDevice, st));
      DG_TRY_CUDA(cudaMemcpy2DAsync(V + (size_t)keep * es, rowV,
                                    (const char*)ws.vc + (size_t)(C - take) * es, (size_t)np * es,
                                    (size_t)take * es, (size_t)B * Hkv * h,
                                    cudaMemcpyDeviceToDevice, st));
    }
    kv->P += C;
    kv->W = Wn;
    return check_launch("append");
  }

  // Canvas forward: statistics into ent/amax; optional logits/hidden (test hook).
  // With an.N > 0: tempered statistics and (an.seeds) the Gumbel-max draw into sampled.
  // With z_in: the self-conditioning signal added to the canvas rows' input; with z_out
  // (self-conditioned models): z = FFW(p0 E) of this forward's logits written there.
  dg_status forward(const dg_kv* kv, const int32_t* canvas, int s, int T, float* ent,
                    int32_t* amax, float* logits, float* hidden, int32_t* load,
                    const AnnealDev& an = AnnealDev{}, int32_t* sampled = nullptr,
                    const Acc* z_in = nullptr, Acc* z_out = nullptr) {
    const int B = kv->B, C = c.canvas, n = B * C, d = c.d_model;
    const double tau = (double)s / (double)T;
    {
      ProfScope ps(m, DG_KIND_GLUE, st);
      launch_pdl((embed_kernel<TW, TR, Acc>), n, 256, 0, st, 1, canvas, (const TW*)m->w.tok_emb, x(), n,
                 d, c.vocab, tau, ws.err, (const int32_t*)s_dev, T, z_in);
      ++m->launches;
    }
    const int Cp = (C + 63) / 64 * 64;
    if (Cp != C)
      DG_TRY_CUDA(cudaMemsetAsync(ws.vc, 0, (size_t)B * c.n_kv_heads * c.head_dim * Cp * sizeof(TKV), st));
    for (int l = 0; l < c.n_layers; ++l)
      DG_TRY(layer(l, n, B, C, kv->P, kv, false, load ? load + (size_t)l * c.n_experts : nullptr));
    if (hidden) {
      launch_pdl((to_f32_kernel<TR>), ceil_div((long)n * d, 256), 256, 0, st, 1, x(), hidden,
                 (long)n * d);
      ++m->launches;
    }
    // xn = RMSNorm(x): written by the last layer's combine
    ProfScope ps(m, DG_KIND_LMHEAD, st);
    ScDev sc;
    if (z_out) {
      sc.P = ws.scP;
      sc.ref = ws.scref;
      sc.ldp = c.vocab;
    }
    bool done = false;
    if constexpr (Path::kTensorCores) {
      if (logits == nullptr) {
        DG_TRY(tc_lmhead_stats(m, xn(), n, ent, amax, st, an, sampled, sc));
        done = true;
      }
    }
    if (!done) {
      dim3 grid(ws.n_vtiles, ceil_div(n, SG_BM));
      launch_pdl((lmhead_simt_kernel<TA, TW, Acc>), grid, 256, 0, st, 1, xn(), (const TW*)m->w.lm_head, n,
                                                           c.vocab, d, c.logit_scale,
                                                           (Acc*)ws.lm_part, logits, an, sc);
      ++m->launches;
      launch_pdl((lm_merge_kernel<Acc, TA>), n, 128, 0, st, 1, (const Acc*)ws.lm_part, ws.n_vtiles,
                                                          n, ent, amax,
                                                          (const Acc*)(an.seeds ? an.gpart : nullptr),
                                                          an.seeds ? sampled : nullptr, sc);
      ++m->launches;
      if (sc.P) {  // the tile values become p0
        static_assert(SG_BN == 64, "tile shift");
        const long groups = (long)n * (c.vocab / (16 / (int)sizeof(TA)));
        launch_pdl((selfcond_scale_kernel<TA, Acc>), ceil_div(groups, 256), 256, 0, st, 1,
                   (TA*)sc.P, (const Acc*)sc.ref, n, c.vocab, 6);
        ++m->launches;
      }
    }
    if (z_out) DG_TRY(selfcond(n, z_out));
    return check_launch("forward");
  }

  // z = W_down (silu(W_gate y) * W_up y) for y = p0 E, p0 left by the LM head
  dg_status selfcond(int n, Acc* z_out) {
    const int d = c.d_model, V = c.vocab, I = c.sc_inter;
    if constexpr (Path::kTensorCores) {
      DG_TRY(tc_selfcond_mix(m, n, st));
      DG_TRY(tc_gemm_swiglu(m, (const TA*)ws.scy, m->w.sc_gate, m->w.sc_up, (TA*)ws.sch, n, I, d,
                            st));
      DG_TRY(tc_gemm_store_f32(m, (const TA*)ws.sch, m->w.sc_down, (float*)z_out, n, d, I, st));
    } else {
      dense((const TA*)ws.scP, V, ws.embT, d, V, n, EpiStore<TA, Acc>{(TA*)ws.scy, d});
      gemm_simt<TA, TW, Acc, false, true>((const TA*)ws.scy, d, (const TW*)m->w.sc_gate,
                                          (const TW*)m->w.sc_up, d, n, I, d, GroupInfo(), 0,
                                          EpiSwiglu<TA, Acc>{(TA*)ws.sch, I}, st, &m->launches);
      dense((const TA*)ws.sch, I, m->w.sc_down, d, I, n, EpiStore<Acc, Acc>{z_out, d});
    }
    return check_launch("self-conditioning");
  }
};

}  // namespace dg

using namespace dg;

// ---------------------------------------------------------------------------
// sampler launch (shared by dg_eb_sample, dg_denoise_step, dg_generate_block)
// ---------------------------------------------------------------------------
static dg_status gamma_fixed(float gamma, long long* out) {
  DG_REQUIRE(!std::isnan(gamma) && gamma >= 0.0f, "gamma must be >= 0 and not NaN (got %g)",
             (double)gamma);
  const long long cap = 1LL << 62;
  if (std::isinf(gamma)) {
    *out = cap;
    return DG_OK;
  }
  const double v = (double)gamma * 281474976710656.0;
  *out = v >= (double)cap ? cap : (long long)std::floor(v);
  return DG_OK;
}

static dg_status launch_sampler(const float* H, const int32_t* am, int32_t* canvas,
                                uint8_t* mask, int B, int C, int s, long long gq,
                                int32_t* ncommit, int32_t* nfwd, int step_no,
                                cudaStream_t st, long long* counter_,
                                const int32_t* s_dev = nullptr, int T = 0,
                                int32_t* remaining = nullptr) {
#define DG_SAMP(NP)                                                                       \
  launch_pdl((eb_sample_kernel<NP>), B, NP, 0, st, 1, H, am, canvas, mask, C, s, gq, ncommit, nfwd, \
                                         step_no, s_dev, T, remaining)
  if (C <= 32) DG_SAMP(32);
  else if (C <= 64) DG_SAMP(64);
  else if (C <= 128) DG_SAMP(128);
  else if (C <= 256) DG_SAMP(256);
  else if (C <= 512) DG_SAMP(512);
  else DG_SAMP(1024);
  if (counter_) ++*counter_;
#undef DG_SAMP
  return check_launch("eb sampler");
}

static void graph_free(dg::BlockGraph* g) {
  if (g->exec) cudaGraphExecDestroy(g->exec);
  for (int k = 0; k < DG_KIND_COUNT; ++k)
    for (auto& e : g->ev[k]) {
      cudaEventDestroy(e.first);
      cudaEventDestroy(e.second);
    }
  delete g;
}

namespace dg {
void release_graphs(dg_model* m) {
  for (auto* g : m->graphs) graph_free(g);
  m->graphs.clear();
}
}  // namespace dg

extern "C" {

const char* dg_status_str(dg_status s) {
  switch (s) {
    case DG_OK: return "DG_OK";
    case DG_ERR_INVALID_ARG: return "DG_ERR_INVALID_ARG";
    case DG_ERR_UNSUPPORTED: return "DG_ERR_UNSUPPORTED";
    case DG_ERR_OOM: return "DG_ERR_OOM";
    case DG_ERR_CUDA: return "DG_ERR_CUDA";
    case DG_ERR_TIMEOUT: return "DG_ERR_TIMEOUT";
    case DG_ERR_INTERNAL: return "DG_ERR_INTERNAL";
  }
  return "DG_ERR_UNKNOWN";
}

const char* dg_last_error(void) { return g_err.c_str(); }

dg_status dg_model_create(const dg_config* cfg, const dg_weights* w, dg_model** out) {
  g_err.clear();
  DG_REQUIRE(cfg && w && out, "null argument");
  *out = nullptr;
  const dg_config& c = *cfg;
  DG_REQUIRE(c.n_layers >= 1 && c.d_model >= 8 && c.d_model % 8 == 0, "bad n_layers/d_model (d_model: a multiple of 8)");
  DG_REQUIRE(c.n_q_heads >= 1 && c.n_kv_heads >= 1 && c.n_q_heads % c.n_kv_heads == 0,
             "n_q_heads must be a positive multiple of n_kv_heads");
  DG_REQUIRE(c.head_dim >= 2 && c.head_dim % 2 == 0 && c.head_dim <= 128,
             "head_dim must be even and <= 128");
  DG_REQUIRE(c.n_experts >= 1 && c.n_experts <= 1024, "n_experts must be in [1, 1024]");
  DG_REQUIRE(c.top_k >= 1 && c.top_k <= c.n_experts && c.top_k <= 64, "bad top_k");
  DG_REQUIRE(c.expert_inter >= 1 && c.shared_inter >= 1, "bad intermediate sizes");
  DG_REQUIRE(c.vocab >= 2 && c.window >= 1, "bad vocab/window");
  DG_REQUIRE(c.canvas >= 1 && c.canvas <= 1024, "canvas must be in [1, 1024]");
  DG_REQUIRE(c.max_batch >= 1 && c.max_prompt >= 1, "bad max_batch/max_prompt");
  DG_REQUIRE(c.rms_eps >= 0.0f && std::isfinite(c.logit_scale) && c.rope_base > 0.0f,
             "bad eps/logit_scale/rope_base");
  DG_REQUIRE(c.dtype == DG_F32 || c.dtype == DG_BF16 || c.dtype == DG_BF16_FP8EXP ||
                 c.dtype == DG_BF16_FP4EXP,
             "unknown dtype %d", c.dtype);
  if (c.dtype == DG_BF16_FP4EXP)
    DG_REQUIRE(c.d_model % 32 == 0 && c.expert_inter % 32 == 0 && c.d_model <= 2048 &&
                   c.expert_inter <= 2048,
               "NVFP4 experts need d and I multiples of 32 and at most 2048 (a unit's block "
               "scales are staged in shared memory)");
  if (c.dtype == DG_BF16_FP8EXP)
    DG_REQUIRE(c.d_model % 128 == 0 && c.expert_inter % 128 == 0,
               "FP8 experts need d and I multiples of 128 (one scale per 128 columns)");
  DG_REQUIRE(w->tok_emb && w->lm_head && w->layers, "null weight pointer");
  DG_REQUIRE(c.sc_inter >= 0, "sc_inter must be >= 0");
  if (c.sc_inter > 0) {
    DG_REQUIRE(w->sc_gate && w->sc_up && w->sc_down, "null self-conditioning weight pointer");
    DG_REQUIRE(c.vocab % (c.dtype == DG_F32 ? 2 : 8) == 0,
               "self-conditioning needs V a multiple of 16 bytes of activations");
    if (c.dtype != DG_F32)
      DG_REQUIRE(c.sc_inter % 64 == 0 && c.vocab % 8 == 0,
                 "self-conditioning on tensor cores needs sc_inter %% 64 == 0 and V %% 8 == 0");
  }
  for (int l = 0; l < c.n_layers; ++l) {
    const dg_layer_weights& L = w->layers[l];
    DG_REQUIRE(L.wqkv && L.wo && L.router && L.gate && L.up && L.down && L.sgate && L.sup &&
                   L.sdown,
               "null weight pointer in layer %d", l);
    if (c.dtype == DG_BF16_FP4EXP && L.gate_tscale && L.up_tscale && L.down_tscale) {
      // the widened weights are exact only with power-of-two tensor scales (read once here)
      const float* ts[3] = {L.gate_tscale, L.up_tscale, L.down_tscale};
      for (int i = 0; i < 3; ++i) {
        float v = 0.f;
        DG_TRY_CUDA(cudaMemcpy(&v, ts[i], sizeof(float), cudaMemcpyDeviceToHost));
        int ex = 0;
        DG_REQUIRE(std::isfinite(v) && v > 0.f && std::frexp(v, &ex) == 0.5f,
                   "NVFP4 tensor scale %g of layer %d is not a positive power of two", v, l);
      }
    }
    if (c.dtype == DG_BF16_FP8EXP)
      DG_REQUIRE(L.gate_scale && L.up_scale && L.down_scale, "null FP8 scale pointer in layer %d", l);
    if (c.dtype == DG_BF16_FP4EXP)
      DG_REQUIRE(L.gate_scale && L.up_scale && L.down_scale && L.gate_tscale && L.up_tscale &&
                     L.down_tscale,
                 "null NVFP4 scale pointer in layer %d", l);
  }
  dg_model* m = new dg_model();
  m->cfg = c;
  m->w = *w;
  m->layers.assign(w->layers, w->layers + c.n_layers);
  m->w.layers = nullptr;
  cudaGetDevice(&m->device);
  m->selfcond = c.sc_inter > 0;
  {
    const char* env = getenv("DG_NO_GRAPHS");
    m->use_graphs = !(env && env[0] && env[0] != '0');
  }
  dg_status s = c.dtype == DG_F32 ? alloc_workspace<PathTiny>(m) : alloc_workspace<PathBF16>(m);
  if (s != DG_OK) {
    std::string keep = g_err;
    ws_free(m->ws);
    delete m;
    g_err = keep;
    return s;
  }
  *out = m;
  return DG_OK;
}

dg_status dg_model_destroy(dg_model* m) {
  if (!m) return DG_OK;
  cudaDeviceSynchronize();
  release_graphs(m);
  for (dg_kv* kv : m->kvs) kv->m = nullptr;  // caches outlive the model only to be destroyed
  m->kvs.clear();
  if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
  if (m->side_stream) cudaStreamDestroy(m->side_stream);
  if (m->fork_ev) cudaEventDestroy(m->fork_ev);
  if (m->join_ev) cudaEventDestroy(m->join_ev);
  for (int k = 0; k < DG_KIND_COUNT; ++k)
    for (auto& e : m->prof[k]) {
      cudaEventDestroy(e.first);
      cudaEventDestroy(e.second);
    }
  tc_release(m);
  ws_free(m->ws);
  delete m;
  return DG_OK;
}

dg_status dg_sync_status(dg_model* m, void* stream) {
  DG_REQUIRE(m, "null model");
  cudaStream_t st = (cudaStream_t)stream;
  DG_TRY_CUDA(cudaStreamSynchronize(st));
  int32_t err[4] = {0, 0, 0, 0};
  DG_TRY_CUDA(cudaMemcpy(err, m->ws.err, sizeof(err), cudaMemcpyDeviceToHost));
  DG_TRY_CUDA(cudaMemset(m->ws.err, 0, sizeof(err)));
  if (err[0] & ERR_TIMEOUT) {
    set_error("a device-side bounded wait gave up (error bits 0x%x)", err[0]);
    return DG_ERR_TIMEOUT;
  }
  if (err[0] & ERR_BAD_TOKEN) {
    set_error("a token id outside the vocabulary reached the embedding");
    return DG_ERR_INVALID_ARG;
  }
  if (err[0]) {
    set_error("device error bits 0x%x", err[0]);
    return DG_ERR_INTERNAL;
  }
  return DG_OK;
}

dg_status dg_prefill(dg_model* m, const int32_t* prompt, int32_t B, int32_t P, dg_kv** out,
                     void* stream) {
  g_err.clear();
  DG_REQUIRE(m && prompt && out, "null argument");
  *out = nullptr;
  const dg_config& c = m->cfg;
  DG_REQUIRE(B >= 1 && B <= c.max_batch, "B=%d outside [1, max_batch=%d]", B, c.max_batch);
  DG_REQUIRE(P >= 1 && P <= c.max_prompt, "P=%d outside [1, max_prompt=%d]", P, c.max_prompt);
  dg_kv* kv = new dg_kv();
  kv->m = m;
  kv->B = B;
  kv->P = P;
  kv->W = std::min(P, c.window);
  // room for the window the cache can grow to by appended blocks (dg_append_block):
  // the whole context stays within max_prompt positions
  kv->Wp = (std::min(c.max_prompt, c.window) + 63) / 64 * 64;
  kv->elem = c.dtype == DG_F32 ? sizeof(double) : sizeof(bf16);
  const size_t n = (size_t)c.n_layers * B * c.n_kv_heads * kv->Wp * c.head_dim * kv->elem;
  if (cudaMalloc(&kv->k, n) != cudaSuccess || cudaMalloc(&kv->v, n) != cudaSuccess ||
      cudaMemsetAsync(kv->k, 0, n, (cudaStream_t)stream) != cudaSuccess ||
      cudaMemsetAsync(kv->v, 0, n, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    cudaFree(kv->k);
    cudaFree(kv->v);
    delete kv;
    set_error("KV cache allocation of 2 x %zu bytes failed", n);
    return DG_ERR_OOM;
  }
  cudaStream_t st = (cudaStream_t)stream;
  dg_status s = c.dtype == DG_F32 ? Runner<PathTiny>(m, st).prefill(prompt, B, P, kv)
                                  : Runner<PathBF16>(m, st).prefill(prompt, B, P, kv);
  if (s != DG_OK) {
    cudaStreamSynchronize(st);
    cudaFree(kv->k);
    cudaFree(kv->v);
    delete kv;
    return s;
  }
  m->kvs.push_back(kv);
  *out = kv;
  return DG_OK;
}

dg_status dg_prefill_into(dg_model* m, const int32_t* prompt, int32_t B, int32_t P,
                          dg_kv* kv, void* stream) {
  g_err.clear();
  DG_REQUIRE(m && prompt && kv, "null argument");
  DG_REQUIRE(kv->m == m, "the KV handle belongs to another model (or its model is gone)");
  DG_REQUIRE(B == kv->B, "B=%d differs from the handle's B=%d", B, kv->B);
  DG_REQUIRE(P >= 1 && P <= m->cfg.max_prompt, "P=%d outside [1, max_prompt=%d]", P,
             m->cfg.max_prompt);
  kv->P = P;  // a handle grown by appended blocks returns to a prompt of P tokens
  kv->W = std::min(P, m->cfg.window);
  cudaStream_t st = (cudaStream_t)stream;
  return m->cfg.dtype == DG_F32 ? Runner<PathTiny>(m, st).prefill(prompt, B, P, kv)
                                : Runner<PathBF16>(m, st).prefill(prompt, B, P, kv);
}

dg_status dg_kv_destroy(dg_kv* kv) {
  if (!kv) return DG_OK;
  cudaDeviceSynchronize();
  if (kv->m) {  // the model is still alive: forget this cache and its captured graphs
    dg_model* m = kv->m;
    auto& gs = m->graphs;
    for (size_t i = 0; i < gs.size();) {
      if (gs[i]->kv == kv) {
        graph_free(gs[i]);
        gs.erase(gs.begin() + i);
      } else {
        ++i;
      }
    }
    m->kvs.erase(std::remove(m->kvs.begin(), m->kvs.end(), kv), m->kvs.end());
  }
  cudaFree(kv->k);
  cudaFree(kv->v);
  delete kv;
  return DG_OK;
}

dg_status dg_kv_info(const dg_kv* kv, int32_t* B, int32_t* P, int32_t* W) {
  DG_REQUIRE(kv, "null kv");
  if (B) *B = kv->B;
  if (P) *P = kv->P;
  if (W) *W = kv->W;
  return DG_OK;
}

dg_status dg_kv_read(const dg_kv* kv, void* k, void* v, void* stream) {
  DG_REQUIRE(kv && k && v, "null argument");
  DG_REQUIRE(kv->m, "kv handle's model was destroyed");
  const dg_config& c = kv->m->cfg;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t blocks = (size_t)c.n_layers * kv->B * c.n_kv_heads;
  const size_t total = blocks * kv->W * c.head_dim;
  if (kv->elem == sizeof(double))
    launch_pdl((kv_unpack_kernel<double>), ceil_div(total, 256), 256, 0, st, 1, 
        (const double*)kv->k, (const double*)kv->v, (double*)k, (double*)v, blocks, kv->W, kv->Wp,
        c.head_dim);
  else
    launch_pdl((kv_unpack_kernel<bf16>), ceil_div(total, 256), 256, 0, st, 1, 
        (const bf16*)kv->k, (const bf16*)kv->v, (bf16*)k, (bf16*)v, blocks, kv->W, kv->Wp,
        c.head_dim);
  return check_launch("kv read");
}

static dg_status check_step_args(dg_model* m, const dg_kv* kv, int s, int T) {
  DG_REQUIRE(m && kv, "null model/kv");
  DG_REQUIRE(kv->m, "kv handle's model was destroyed");
  DG_REQUIRE(kv->m == m, "kv handle belongs to another model");
  DG_REQUIRE(T >= 1 && s >= 1 && s <= T, "steps_left=%d must be in [1, T=%d]", s, T);
  return DG_OK;
}

// z_in / z_out: the self-conditioning signal in the path's accumulate type (fp64 for
// the fp32 model, fp32 otherwise); nullptr: none in / none computed.
static dg_status run_forward(dg_model* m, const dg_kv* kv, const int32_t* canvas, int s, int T,
                             float* ent, int32_t* am, float* logits, float* hidden,
                             int32_t* load, cudaStream_t st, const int32_t* s_dev = nullptr,
                             const AnnealDev& an = AnnealDev{}, int32_t* sampled = nullptr,
                             const void* z_in = nullptr, void* z_out = nullptr) {
  return m->cfg.dtype == DG_F32
             ? Runner<PathTiny>(m, st, s_dev).forward(kv, canvas, s, T, ent, am, logits, hidden,
                                                      load, an, sampled, (const double*)z_in,
                                                      (double*)z_out)
             : Runner<PathBF16>(m, st, s_dev).forward(kv, canvas, s, T, ent, am, logits, hidden,
                                                      load, an, sampled, (const float*)z_in,
                                                      (float*)z_out);
}

// The block loops' z buffer (nullptr when the model runs without self-conditioning).
static void* loop_z(dg_model* m) { return m->selfcond ? m->ws.z : nullptr; }

static dg_status zero_loop_z(dg_model* m, int B, cudaStream_t st) {
  if (!m->selfcond) return DG_OK;
  const size_t es = m->cfg.dtype == DG_F32 ? sizeof(double) : sizeof(float);
  DG_TRY_CUDA(cudaMemsetAsync(m->ws.z, 0, (size_t)B * m->cfg.canvas * m->cfg.d_model * es, st));
  return DG_OK;
}

dg_status dg_denoise_step(dg_model* m, const dg_kv* kv, int32_t* canvas, uint8_t* mask,
                          int32_t steps_left, int32_t T, float gamma, float* entropy,
                          int32_t* argmax, int32_t* n_committed, void* stream) {
  g_err.clear();
  DG_TRY(check_step_args(m, kv, steps_left, T));
  DG_REQUIRE(canvas && mask && entropy && argmax && n_committed, "null argument");
  long long gq;
  DG_TRY(gamma_fixed(gamma, &gq));
  cudaStream_t st = (cudaStream_t)stream;
  DG_TRY(run_forward(m, kv, canvas, steps_left, T, entropy, argmax, nullptr, nullptr, nullptr, st));
  return launch_sampler(entropy, argmax, canvas, mask, kv->B, m->cfg.canvas, steps_left, gq,
                        n_committed, nullptr, 0, st, &m->launches);
}

// The launch sequence of one block (T forwards + sampler steps), enqueued on st.
static dg_status generate_impl(dg_model* m, const dg_kv* kv, int32_t T, long long gq,
                               int32_t* canvas_out, int32_t* n_forwards, int32_t* router_load,
                               cudaStream_t st, int fcap = 0) {
  const dg_config& c = m->cfg;
  const int B = kv->B, C = c.canvas;
  Workspace& ws = m->ws;
  launch_pdl((fill_i32_kernel), ceil_div((long)B * C, 256), 256, 0, st, 1, canvas_out, B * C, c.vocab);
  ++m->launches;
  DG_TRY_CUDA(cudaMemsetAsync(ws.mask, 1, (size_t)B * C, st));
  DG_TRY(zero_loop_z(m, B, st));
  if (n_forwards) DG_TRY_CUDA(cudaMemsetAsync(n_forwards, 0, B * sizeof(int32_t), st));
  if (router_load)
    DG_TRY_CUDA(cudaMemsetAsync(router_load, 0,
                                (size_t)c.n_layers * c.n_experts * sizeof(int32_t), st));
  const int nfw = fcap > 0 ? std::min(fcap, (int)T) : (int)T;
  for (int k = 0; k < nfw; ++k) {
    const int s = T - k;
    DG_TRY(run_forward(m, kv, canvas_out, s, T, ws.ent, ws.amax, nullptr, nullptr, router_load,
                       st, nullptr, AnnealDev{}, nullptr, loop_z(m), loop_z(m)));
    ProfScope ps(m, DG_KIND_GLUE, st);
    DG_TRY(launch_sampler(ws.ent, ws.amax, canvas_out, ws.mask, B, C, s, gq, ws.ncommit,
                          n_forwards, k + 1, st, &m->launches));
  }
  return DG_OK;
}

static dg_status replay(dg_model* m, dg::BlockGraph* g, cudaStream_t st);

// Builds a block as a graph with a device-controlled loop: init(stream) captured first,
// then a WHILE node whose body is body(stream) (one forward + sampler step) followed by
// a control kernel that decrements the device-side steps-left counter and stops the
// loop once it reaches 0 or no canvas of the batch is still running (remaining[b] > 0
// marks a running canvas).  Returns false (nothing built) if this CUDA build refuses a
// step.
extern "C++" {
template <class Init, class Body>
static bool build_while_graph(dg_model* m, int B, dg::BlockGraph* g, Init&& init, Body&& body) {
  Workspace& ws = m->ws;
  cudaStream_t cap = m->cap_stream;
  cudaGraph_t graph = nullptr;
  if (cudaGraphCreate(&graph, 0) != cudaSuccess) return false;
  bool ok = false;
  do {
    cudaGraphConditionalHandle handle;
    if (cudaGraphConditionalHandleCreate(&handle, graph, 1, cudaGraphCondAssignDefault) !=
        cudaSuccess)
      break;
    if (cudaStreamBeginCaptureToGraph(cap, graph, nullptr, nullptr, 0,
                                      cudaStreamCaptureModeThreadLocal) != cudaSuccess)
      break;
    init(cap);
    cudaGraph_t g1 = nullptr;
    if (cudaStreamEndCapture(cap, &g1) != cudaSuccess) break;
    size_t nn = 0;
    cudaGraphGetNodes(graph, nullptr, &nn);
    std::vector<cudaGraphNode_t> nodes(nn);
    cudaGraphGetNodes(graph, nodes.data(), &nn);
    cudaGraphNodeParams cp = {};
    cp.type = cudaGraphNodeTypeConditional;
    cp.conditional.handle = handle;
    cp.conditional.type = cudaGraphCondTypeWhile;
    cp.conditional.size = 1;
    cudaGraphNode_t cnode;
    if (cudaGraphAddNode(&cnode, graph, nodes.data(), nn, &cp) != cudaSuccess) break;
    cudaGraph_t bodyg = cp.conditional.phGraph_out[0];
    if (cudaStreamBeginCaptureToGraph(cap, bodyg, nullptr, nullptr, 0,
                                      cudaStreamCaptureModeThreadLocal) != cudaSuccess)
      break;
    const long long l0 = m->launches;
    const dg_status s = body(cap);
    launch_pdl((block_step_kernel), 1, 32, 0, cap, 1, handle, ws.loop_s,
               (const int32_t*)ws.remaining, B);
    g->body_launches = m->launches - l0 + 1;
    m->launches = l0;
    cudaGraph_t g2 = nullptr;
    const cudaError_t e = cudaStreamEndCapture(cap, &g2);
    if (s != DG_OK || e != cudaSuccess) break;
    if (cudaGraphInstantiate(&g->exec, graph, 0) != cudaSuccess) break;
    g->launches = 1;
    g->loop = true;
    ok = true;
  } while (false);
  cudaGraphDestroy(graph);
  if (!ok) {
    cudaGetLastError();
    if (g->exec) cudaGraphExecDestroy(g->exec);
    g->exec = nullptr;
  }
  return ok;
}
}  // extern "C++"

// The Entropy-Bound block: init kernel (all [MASK], steps left T), body = forward at
// the device's steps-left + EB sampler step (remaining[b] = masked positions left).
static bool build_loop_graph(dg_model* m, const dg_kv* kv, int32_t T, long long gq,
                             int32_t* canvas_out, int32_t* n_forwards, int32_t* router_load,
                             dg::BlockGraph* g) {
  const dg_config& c = m->cfg;
  Workspace& ws = m->ws;
  const int B = kv->B, C = c.canvas;
  const int n = B * C, n_load = router_load ? c.n_layers * c.n_experts : 0;
  return build_while_graph(
      m, B, g,
      [&](cudaStream_t cap) {
        launch_pdl((block_init_kernel), ceil_div(std::max(n, n_load), 256), 256, 0, cap, 1,
                   canvas_out, ws.mask, n, (int32_t)c.vocab, n_forwards, B, router_load, n_load,
                   ws.loop_s, T);
        zero_loop_z(m, B, cap);
      },
      [&](cudaStream_t cap) {
        dg_status s = run_forward(m, kv, canvas_out, T, T, ws.ent, ws.amax, nullptr, nullptr,
                                  router_load, cap, ws.loop_s, AnnealDev{}, nullptr, loop_z(m),
                                  loop_z(m));
        if (s == DG_OK)
          s = launch_sampler(ws.ent, ws.amax, canvas_out, ws.mask, B, C, T, gq, ws.ncommit,
                             n_forwards, 1, cap, &m->launches, ws.loop_s, T, ws.remaining);
        return s;
      });
}

// Captures the block's launch sequence once per (kv, T, gamma, output buffers,
// profiling) and replays it: one host call per block instead of ~500 launches per
// forward.  With profiling on, the graph also records an event pair around every
// launch group, read back after each replay.
static dg_status generate_graphed(dg_model* m, const dg_kv* kv, int32_t T, long long gq,
                                  int32_t* canvas_out, int32_t* n_forwards,
                                  int32_t* router_load, cudaStream_t st) {
  dg::BlockGraph* g = nullptr;
  for (auto* x : m->graphs)
    if (!x->anneal && x->sc == m->selfcond && x->kv == kv && x->kv_P == kv->P &&
        x->kv_W == kv->W && x->T == T && x->gq == gq &&
        x->canvas == canvas_out &&
        x->nfwd == n_forwards && x->load == router_load && x->prof == m->profiling &&
        (!x->prof || x->fcap == m->prof_forwards)) {
      g = x;
      break;
    }
  if (!g) {
    if (m->graphs.size() >= 8) {
      graph_free(m->graphs.front());
      m->graphs.erase(m->graphs.begin());
    }
    g = new dg::BlockGraph();
    g->kv = kv;
    g->kv_P = kv->P;
    g->kv_W = kv->W;
    g->T = T;
    g->gq = gq;
    g->canvas = canvas_out;
    g->nfwd = n_forwards;
    g->load = router_load;
    g->prof = m->profiling;
    g->fcap = m->profiling ? m->prof_forwards : 0;
    g->sc = m->selfcond;
    // capture on a library-owned stream (the caller's may be the legacy default
    // stream, which cannot be captured); nothing executes during capture
    if (!m->cap_stream) DG_TRY_CUDA(cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking));
    if (!g->prof && build_loop_graph(m, kv, T, gq, canvas_out, n_forwards, router_load, g)) {
      m->graphs.push_back(g);
      return replay(m, g, st);
    }
    const long long l0 = m->launches;
    m->capture = g;
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal);
    dg_status s = DG_OK;
    if (e == cudaSuccess) {
      s = generate_impl(m, kv, T, gq, canvas_out, n_forwards, router_load, m->cap_stream,
                        g->fcap);
      e = cudaStreamEndCapture(m->cap_stream, &graph);
    }
    m->capture = nullptr;
    g->launches = m->launches - l0;
    m->launches = l0;
    if (s == DG_OK && e == cudaSuccess) e = cudaGraphInstantiate(&g->exec, graph, 0);
    if (graph) cudaGraphDestroy(graph);
    if (s != DG_OK || e != cudaSuccess) {
      graph_free(g);
      if (s == DG_OK) {
        set_error("block graph capture failed: %s", cudaGetErrorString(e));
        s = DG_ERR_CUDA;
      }
      cudaGetLastError();
      return s;
    }
    m->graphs.push_back(g);
  }
  return replay(m, g, st);
}

static dg_status replay(dg_model* m, dg::BlockGraph* g, cudaStream_t st) {
  DG_TRY_CUDA(cudaGraphLaunch(g->exec, st));
  m->launches += g->launches;
  m->last_body_launches = g->loop ? g->body_launches : 0;
  if (g->prof) {
    DG_TRY_CUDA(cudaStreamSynchronize(st));
    for (int k = 0; k < DG_KIND_COUNT; ++k)
      for (auto& ev : g->ev[k]) {
        float t = 0.f;
        DG_TRY_CUDA(cudaEventElapsedTime(&t, ev.first, ev.second));
        m->prof_acc_ms[k] += t;
        m->prof_acc_n[k] += 1;
      }
  }
  return DG_OK;
}

dg_status dg_generate_block(dg_model* m, const dg_kv* kv, int32_t T, float gamma,
                            int32_t* canvas_out, int32_t* n_forwards, int32_t* router_load,
                            void* stream) {
  g_err.clear();
  DG_TRY(check_step_args(m, kv, T, T));
  DG_REQUIRE(canvas_out, "null canvas_out");
  long long gq;
  DG_TRY(gamma_fixed(gamma, &gq));
  cudaStream_t st = (cudaStream_t)stream;
  if (m->use_graphs)
    return generate_graphed(m, kv, T, gq, canvas_out, n_forwards, router_load, st);
  return generate_impl(m, kv, T, gq, canvas_out, n_forwards, router_load, st);
}

dg_status dg_append_block(dg_model* m, dg_kv* kv, const int32_t* tokens, void* stream) {
  g_err.clear();
  DG_REQUIRE(m && kv && tokens, "null argument");
  DG_REQUIRE(kv->m == m, "the KV handle belongs to another model (or its model is gone)");
  const dg_config& c = m->cfg;
  DG_REQUIRE(kv->P + c.canvas <= c.max_prompt,
             "P + C = %d exceeds max_prompt = %d (the context the model was created for)",
             kv->P + c.canvas, c.max_prompt);
  // the kept part of a layer's window passes through the gathered-rows buffer
  const size_t need = (size_t)kv->B * c.n_kv_heads * c.head_dim * std::min(kv->W, c.window) *
                      kv->elem;
  DG_REQUIRE(need <= m->ws.max_rows * (size_t)c.d_model * kv->elem,
             "append scratch too small for this cache");
  cudaStream_t st = (cudaStream_t)stream;
  return c.dtype == DG_F32 ? Runner<PathTiny>(m, st).append(tokens, kv)
                           : Runner<PathBF16>(m, st).append(tokens, kv);
}

dg_status dg_generate_blocks(dg_model* m, dg_kv* kv, int32_t n_blocks, int32_t T, float gamma,
                             int32_t* out, int32_t* n_forwards, void* stream) {
  g_err.clear();
  DG_REQUIRE(m && kv && out, "null argument");
  DG_REQUIRE(kv->m == m, "the KV handle belongs to another model (or its model is gone)");
  DG_REQUIRE(n_blocks >= 1, "n_blocks must be >= 1");
  const dg_config& c = m->cfg;
  DG_REQUIRE(kv->P + (long long)(n_blocks - 1) * c.canvas <= c.max_prompt,
             "P + (n_blocks - 1) C exceeds max_prompt = %d", c.max_prompt);
  const int B = kv->B, C = c.canvas;
  cudaStream_t st = (cudaStream_t)stream;
  for (int k = 0; k < n_blocks; ++k) {
    DG_TRY(dg_generate_block(m, kv, T, gamma, m->ws.blk, n_forwards ? n_forwards + k * B : nullptr,
                             nullptr, stream));
    DG_TRY_CUDA(cudaMemcpy2DAsync(out + (size_t)k * C, (size_t)n_blocks * C * sizeof(int32_t),
                                  m->ws.blk, (size_t)C * sizeof(int32_t), C * sizeof(int32_t), B,
                                  cudaMemcpyDeviceToDevice, st));
    if (k + 1 < n_blocks) DG_TRY(dg_append_block(m, kv, m->ws.blk, stream));
  }
  return DG_OK;
}

// ---------------------------------------------------------------------------
// The Report's default sampler: annealed entropy-bounded refinement over a
// uniform-noise canvas (k_anneal.cuh states the rule and the readings).
// ---------------------------------------------------------------------------
struct AnnealQ {
  unsigned long long bq = 0, eq = 0;  // min(floor(b 2^48), 2^62), floor(e_stop 2^48)
};

static dg_status anneal_check(const dg_anneal_params* p, int V, AnnealQ* q) {
  DG_REQUIRE(p, "null params");
  DG_REQUIRE(p->N >= 1 && p->N <= 65536, "N=%d outside [1, 65536]", p->N);
  DG_REQUIRE(!std::isnan(p->b) && p->b >= 0.0f, "b must be >= 0 and not NaN (got %g)",
             (double)p->b);
  DG_REQUIRE(std::isfinite(p->tau_max) && p->tau_max > 0.0f && std::isfinite(p->tau_min) &&
                 p->tau_min > 0.0f,
             "temperatures must be finite and > 0 (got %g, %g)", (double)p->tau_max,
             (double)p->tau_min);
  DG_REQUIRE(p->e_stop >= 0.0f && p->e_stop <= 16.0f, "e_stop outside [0, 16] (got %g)",
             (double)p->e_stop);
  DG_REQUIRE(V >= 1 && V <= (1 << 24), "V=%d outside [1, 2^24]", V);
  const double two48 = 281474976710656.0, cap = 4611686018427387904.0;  // 2^48, 2^62
  const double bv = std::isinf(p->b) ? cap : std::floor((double)p->b * two48);
  q->bq = bv >= cap ? (1ull << 62) : (unsigned long long)bv;
  q->eq = (unsigned long long)std::floor((double)p->e_stop * two48);
  return DG_OK;
}

static AnnealDev anneal_dev(dg_model* m, const dg_anneal_params* p, const uint64_t* seeds,
                            int s, const int32_t* s_dev) {
  AnnealDev a;
  a.seeds = (const unsigned long long*)seeds;
  a.s_dev = s_dev;
  a.s = s;
  a.N = p->N;
  a.C = m->cfg.canvas;
  a.tau_max = p->tau_max;
  a.tau_min = p->tau_min;
  a.gpart = m->ws.gpart;
  return a;
}

static dg_status launch_anneal(const float* H, const int32_t* am, const int32_t* sampled,
                               int32_t* canvas, int32_t* prev, int32_t* state, int32_t* nfwd,
                               int32_t* nacc, int32_t* remaining, int B, int C, int V, int k,
                               const int32_t* s_dev, int N, const AnnealQ& q,
                               const uint64_t* seeds, cudaStream_t st, long long* counter) {
  const unsigned long long* sd = (const unsigned long long*)seeds;
#define DG_ANN(NP)                                                                          \
  launch_pdl((anneal_sample_kernel<NP>), B, NP, 0, st, 1, H, am, sampled, canvas, prev, state, \
             nfwd, nacc, remaining, C, V, k, s_dev, N, q.bq, q.eq, sd)
  if (C <= 32) DG_ANN(32);
  else if (C <= 64) DG_ANN(64);
  else if (C <= 128) DG_ANN(128);
  else if (C <= 256) DG_ANN(256);
  else if (C <= 512) DG_ANN(512);
  else DG_ANN(1024);
#undef DG_ANN
  if (counter) ++*counter;
  return check_launch("annealed sampler");
}

// The annealed block as plain launches: N forwards (min(fcap, N) when profiling); a
// canvas that has stopped is left alone by the later sampler steps.
static dg_status anneal_impl(dg_model* m, const dg_kv* kv, const dg_anneal_params* p,
                             const AnnealQ& q, const uint64_t* seeds, int32_t* canvas_out,
                             int32_t* n_forwards, cudaStream_t st, int fcap) {
  const dg_config& c = m->cfg;
  Workspace& ws = m->ws;
  const int B = kv->B, C = c.canvas, V = c.vocab;
  {
    ProfScope ps(m, DG_KIND_GLUE, st);
    launch_pdl((anneal_init_kernel), ceil_div((long)B * C, 256), 256, 0, st, 1, canvas_out,
               ws.prev, ws.astate, n_forwards, B, C, V, (const unsigned long long*)seeds,
               (int32_t*)nullptr, p->N);
    ++m->launches;
    DG_TRY(zero_loop_z(m, B, st));
  }
  const int nfw = fcap > 0 ? std::min(fcap, (int)p->N) : (int)p->N;
  for (int k = 0; k < nfw; ++k) {
    const int s = p->N - k;
    DG_TRY(run_forward(m, kv, canvas_out, s, p->N, ws.ent, ws.amax, nullptr, nullptr, nullptr,
                       st, nullptr, anneal_dev(m, p, seeds, s, nullptr), ws.sampled, loop_z(m),
                       loop_z(m)));
    ProfScope ps(m, DG_KIND_GLUE, st);
    DG_TRY(launch_anneal(ws.ent, ws.amax, ws.sampled, canvas_out, ws.prev, ws.astate, n_forwards,
                         ws.ncommit, (int32_t*)nullptr, B, C, V, k, (const int32_t*)nullptr,
                         p->N, q, seeds, st, &m->launches));
  }
  return DG_OK;
}

// The annealed block as a device-controlled loop (see build_while_graph).
static bool build_anneal_graph(dg_model* m, const dg_kv* kv, const dg_anneal_params* p,
                               const AnnealQ& q, const uint64_t* seeds, int32_t* canvas_out,
                               int32_t* n_forwards, dg::BlockGraph* g) {
  const dg_config& c = m->cfg;
  Workspace& ws = m->ws;
  const int B = kv->B, C = c.canvas, V = c.vocab, N = p->N;
  return build_while_graph(
      m, B, g,
      [&](cudaStream_t cap) {
        launch_pdl((anneal_init_kernel), ceil_div((long)B * C, 256), 256, 0, cap, 1, canvas_out,
                   ws.prev, ws.astate, n_forwards, B, C, V, (const unsigned long long*)seeds,
                   ws.loop_s, N);
        zero_loop_z(m, B, cap);
      },
      [&](cudaStream_t cap) {
        dg_status s = run_forward(m, kv, canvas_out, N, N, ws.ent, ws.amax, nullptr, nullptr,
                                  nullptr, cap, ws.loop_s, anneal_dev(m, p, seeds, N, ws.loop_s),
                                  ws.sampled, loop_z(m), loop_z(m));
        if (s == DG_OK)
          s = launch_anneal(ws.ent, ws.amax, ws.sampled, canvas_out, ws.prev, ws.astate,
                            n_forwards, ws.ncommit, ws.remaining, B, C, V, 0, ws.loop_s, N, q,
                            seeds, cap, &m->launches);
        return s;
      });
}

dg_status dg_generate_block_annealed(dg_model* m, const dg_kv* kv, const dg_anneal_params* p,
                                     const uint64_t* seeds, int32_t* canvas_out,
                                     int32_t* n_forwards, void* stream) {
  g_err.clear();
  DG_TRY(check_step_args(m, kv, 1, 1));
  DG_REQUIRE(seeds && canvas_out, "null argument");
  AnnealQ q;
  DG_TRY(anneal_check(p, m->cfg.vocab, &q));
  DG_REQUIRE(m->cfg.canvas <= 1024, "canvas %d > 1024", m->cfg.canvas);
  cudaStream_t st = (cudaStream_t)stream;
  if (!m->use_graphs)
    return anneal_impl(m, kv, p, q, seeds, canvas_out, n_forwards, st,
                       m->profiling ? m->prof_forwards : 0);
  dg::BlockGraph* g = nullptr;
  for (auto* x : m->graphs)
    if (x->anneal && x->sc == m->selfcond && x->kv == kv && x->kv_P == kv->P &&
        x->kv_W == kv->W && x->aN == p->N &&
        x->ab == p->b && x->atmax == p->tau_max && x->atmin == p->tau_min &&
        x->aestop == p->e_stop && x->seeds == seeds && x->canvas == canvas_out &&
        x->nfwd == n_forwards && x->prof == m->profiling &&
        (!x->prof || x->fcap == m->prof_forwards)) {
      g = x;
      break;
    }
  if (!g) {
    if (m->graphs.size() >= 8) {
      graph_free(m->graphs.front());
      m->graphs.erase(m->graphs.begin());
    }
    g = new dg::BlockGraph();
    g->anneal = true;
    g->kv = kv;
    g->kv_P = kv->P;
    g->kv_W = kv->W;
    g->aN = p->N;
    g->ab = p->b;
    g->atmax = p->tau_max;
    g->atmin = p->tau_min;
    g->aestop = p->e_stop;
    g->seeds = seeds;
    g->canvas = canvas_out;
    g->nfwd = n_forwards;
    g->prof = m->profiling;
    g->fcap = m->profiling ? m->prof_forwards : 0;
    g->sc = m->selfcond;
    if (!m->cap_stream) DG_TRY_CUDA(cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking));
    if (g->prof) {
      // profiling: the first fcap forwards unrolled, with an event pair around every
      // launch group recorded by the graph (read back after each replay)
      const long long l0 = m->launches;
      m->capture = g;
      cudaGraph_t graph = nullptr;
      cudaError_t e = cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal);
      dg_status s = DG_OK;
      if (e == cudaSuccess) {
        s = anneal_impl(m, kv, p, q, seeds, canvas_out, n_forwards, m->cap_stream, g->fcap);
        e = cudaStreamEndCapture(m->cap_stream, &graph);
      }
      m->capture = nullptr;
      g->launches = m->launches - l0;
      m->launches = l0;
      if (s == DG_OK && e == cudaSuccess) e = cudaGraphInstantiate(&g->exec, graph, 0);
      if (graph) cudaGraphDestroy(graph);
      if (s != DG_OK || e != cudaSuccess) {
        graph_free(g);
        if (s == DG_OK) {
          set_error("annealed block capture failed: %s", cudaGetErrorString(e));
          s = DG_ERR_CUDA;
        }
        cudaGetLastError();
        return s;
      }
    } else if (!build_anneal_graph(m, kv, p, q, seeds, canvas_out, n_forwards, g)) {
      graph_free(g);
      return anneal_impl(m, kv, p, q, seeds, canvas_out, n_forwards, st, 0);
    }
    m->graphs.push_back(g);
  }
  return replay(m, g, st);
}

dg_status dg_anneal_forward(dg_model* m, const dg_kv* kv, const int32_t* canvas, int32_t k,
                            const dg_anneal_params* p, const uint64_t* seeds, float* entropy,
                            int32_t* argmax, int32_t* sampled, const void* z_in, void* z_out,
                            void* stream) {
  g_err.clear();
  DG_REQUIRE(canvas && seeds && entropy && argmax && sampled, "null argument");
  AnnealQ q;
  DG_REQUIRE(m, "null model");
  DG_TRY(anneal_check(p, m->cfg.vocab, &q));
  DG_REQUIRE(k >= 0 && k < p->N, "k=%d outside [0, N=%d)", k, p->N);
  DG_TRY(check_step_args(m, kv, p->N - k, p->N));
  DG_REQUIRE(!z_out || m->cfg.sc_inter > 0, "the model has no self-conditioning FFW");
  return run_forward(m, kv, canvas, p->N - k, p->N, entropy, argmax, nullptr, nullptr, nullptr,
                     (cudaStream_t)stream, nullptr, anneal_dev(m, p, seeds, p->N - k, nullptr),
                     sampled, z_in, z_out);
}

dg_status dg_anneal_sample(const float* entropy, const int32_t* argmax, const int32_t* sampled,
                           int32_t* canvas, int32_t* prev_argmax, int32_t* state,
                           int32_t* n_accepted, int32_t B, int32_t C, int32_t V, int32_t k,
                           const dg_anneal_params* p, const uint64_t* seeds, void* stream) {
  g_err.clear();
  DG_REQUIRE(entropy && argmax && sampled && canvas && prev_argmax && state && seeds,
             "null argument");
  DG_REQUIRE(B >= 1 && C >= 1 && C <= 1024, "need B >= 1 and 1 <= C <= 1024");
  AnnealQ q;
  DG_TRY(anneal_check(p, V, &q));
  DG_REQUIRE(k >= 0 && k < p->N, "k=%d outside [0, N=%d)", k, p->N);
  return launch_anneal(entropy, argmax, sampled, canvas, prev_argmax, state, (int32_t*)nullptr,
                       n_accepted, (int32_t*)nullptr, B, C, V, k, (const int32_t*)nullptr, p->N,
                       q, seeds, (cudaStream_t)stream, nullptr);
}

dg_status dg_anneal_init(int32_t* canvas, int32_t* prev_argmax, int32_t* state, int32_t B,
                         int32_t C, int32_t V, const uint64_t* seeds, void* stream) {
  g_err.clear();
  DG_REQUIRE(canvas && seeds, "null argument");
  DG_REQUIRE(B >= 1 && C >= 1 && (long long)B * C <= (1LL << 30), "bad B=%d, C=%d", B, C);
  DG_REQUIRE(V >= 1 && V <= (1 << 24), "V=%d outside [1, 2^24]", V);
  launch_pdl((anneal_init_kernel), ceil_div((long)B * C, 256), 256, 0, (cudaStream_t)stream, 1,
             canvas, prev_argmax, state, (int32_t*)nullptr, B, C, V,
             (const unsigned long long*)seeds, (int32_t*)nullptr, 1);
  return check_launch("anneal init");
}

dg_status dg_set_selfcond(dg_model* m, int32_t on) {
  g_err.clear();
  DG_REQUIRE(m, "null model");
  DG_REQUIRE(on == 0 || m->cfg.sc_inter > 0, "the model has no self-conditioning FFW");
  m->selfcond = on != 0;
  return DG_OK;
}

dg_status dg_selfcond_forward(dg_model* m, const dg_kv* kv, const int32_t* canvas,
                              int32_t steps_left, int32_t T, const void* z_in, float* entropy,
                              int32_t* argmax, void* z_out, void* stream) {
  g_err.clear();
  DG_TRY(check_step_args(m, kv, steps_left, T));
  DG_REQUIRE(canvas && entropy && argmax && z_out, "null argument");
  DG_REQUIRE(m->cfg.sc_inter > 0, "the model has no self-conditioning FFW");
  return run_forward(m, kv, canvas, steps_left, T, entropy, argmax, nullptr, nullptr, nullptr,
                     (cudaStream_t)stream, nullptr, AnnealDev{}, nullptr, z_in, z_out);
}

dg_status dg_eb_sample(const float* entropy, const int32_t* argmax, int32_t* canvas,
                       uint8_t* mask, int32_t B, int32_t C, int32_t steps_left, float gamma,
                       int32_t* n_committed, void* stream) {
  g_err.clear();
  DG_REQUIRE(entropy && argmax && canvas && mask, "null argument");
  DG_REQUIRE(B >= 1 && C >= 1 && C <= 1024, "need B >= 1 and 1 <= C <= 1024");
  DG_REQUIRE(steps_left >= 1, "steps_left must be >= 1");
  long long gq;
  DG_TRY(gamma_fixed(gamma, &gq));
  return launch_sampler(entropy, argmax, canvas, mask, B, C, steps_left, gq, n_committed,
                        nullptr, 0, (cudaStream_t)stream, nullptr);
}

dg_status dg_op_gemm(dg_model* m, const void* A, const void* W, float* out, int32_t M, int32_t N,
                     int32_t K, void* stream) {
  g_err.clear();
  DG_REQUIRE(m && A && W && out, "null argument");
  DG_REQUIRE(M >= 1 && N >= 1 && K >= 1, "bad sizes");
  cudaStream_t st = (cudaStream_t)stream;
  if (m->cfg.dtype == DG_F32) {
    gemm_simt<float, float, double, false, false>((const float*)A, K, (const float*)W, nullptr, K,
                                                  M, N, K, GroupInfo(), 0,
                                                  EpiStore<float, double>{out, N}, st,
                                                  &m->launches);
    return check_launch("op gemm");
  }
  DG_REQUIRE(N % 64 == 0 && K % 64 == 0, "bf16 GEMM needs N %% 64 == 0 and K %% 64 == 0");
  return tc_gemm_f32_rows(m, (const bf16*)A, M, W, out, M, N, K, st);
}

dg_status dg_op_moe(dg_model* m, int32_t layer, const float* x, float* out, int32_t n,
                    void* stream) {
  g_err.clear();
  DG_REQUIRE(m && x && out, "null argument");
  DG_REQUIRE(layer >= 0 && layer < m->cfg.n_layers, "layer out of range");
  DG_REQUIRE(n >= 1 && (size_t)n <= m->ws.max_tok, "n=%d outside [1, %zu]", n, m->ws.max_tok);
  cudaStream_t st = (cudaStream_t)stream;
  return m->cfg.dtype == DG_F32 ? Runner<PathTiny>(m, st).moe_op(layer, x, out, n)
                                : Runner<PathBF16>(m, st).moe_op(layer, x, out, n);
}

dg_status dg_debug_stall_experts(dg_model* m, int64_t limit_ns) {
  g_err.clear();
  DG_REQUIRE(m, "null model");
  DG_REQUIRE(limit_ns >= 100000 && limit_ns <= 1000000000, "limit_ns outside [1e5, 1e9]");
  if (m->cfg.dtype != DG_BF16) {
    set_error("only the bf16 routed-expert kernel has this test path");
    return DG_ERR_UNSUPPORTED;
  }
  m->stall_limit_ns = limit_ns;
  return DG_OK;
}

dg_status dg_profile_start(dg_model* m, int32_t max_forwards) {
  DG_REQUIRE(m, "null model");
  DG_REQUIRE(max_forwards >= 0, "max_forwards must be >= 0");
  m->prof_forwards = max_forwards;
  for (int k = 0; k < DG_KIND_COUNT; ++k) {
    m->prof_used[k] = 0;
    m->prof_acc_ms[k] = 0.0;
    m->prof_acc_n[k] = 0;
  }
  DG_TRY_CUDA(cudaDeviceSynchronize());
  DG_TRY_CUDA(cudaMemset(m->ws.units, 0, sizeof(unsigned long long)));
  m->profiling = true;
  return DG_OK;
}

dg_status dg_expert_units(dg_model* m, int64_t* units) {
  DG_REQUIRE(m && units, "null argument");
  unsigned long long u = 0;
  DG_TRY_CUDA(cudaDeviceSynchronize());
  DG_TRY_CUDA(cudaMemcpy(&u, m->ws.units, sizeof(u), cudaMemcpyDeviceToHost));
  *units = (int64_t)u;
  return DG_OK;
}

dg_status dg_profile_stop(dg_model* m, float* ms, int64_t* groups) {
  DG_REQUIRE(m, "null model");
  m->profiling = false;
  DG_TRY_CUDA(cudaDeviceSynchronize());
  for (int k = 0; k < DG_KIND_COUNT; ++k) {
    double tot = 0.0;
    for (size_t i = 0; i < m->prof_used[k]; ++i) {
      float t = 0.0f;
      DG_TRY_CUDA(cudaEventElapsedTime(&t, m->prof[k][i].first, m->prof[k][i].second));
      tot += t;
    }
    if (ms) ms[k] = (float)(tot + m->prof_acc_ms[k]);
    if (groups) groups[k] = (int64_t)m->prof_used[k] + m->prof_acc_n[k];
    m->prof_used[k] = 0;
  }
  return DG_OK;
}

dg_status dg_launch_count(const dg_model* m, int64_t* out) {
  DG_REQUIRE(m && out, "null argument");
  *out = m->launches;
  return DG_OK;
}

dg_status dg_block_loop_launches(const dg_model* m, int64_t* per_forward) {
  DG_REQUIRE(m && per_forward, "null argument");
  *per_forward = m->last_body_launches;
  return DG_OK;
}

dg_status dg_debug_forward(dg_model* m, const dg_kv* kv, const int32_t* canvas,
                           int32_t steps_left, int32_t T, float* entropy, int32_t* argmax,
                           float* logits, float* hidden, void* stream) {
  g_err.clear();
  DG_TRY(check_step_args(m, kv, steps_left, T));
  DG_REQUIRE(canvas && entropy && argmax, "null argument");
  return run_forward(m, kv, canvas, steps_left, T, entropy, argmax, logits, hidden, nullptr,
                     (cudaStream_t)stream);
}

}  // extern "C"
