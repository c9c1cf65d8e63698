// Internal declarations of libdg: model/KV structs, workspace, error helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <string>
#include <utility>
#include <vector>

#include "../../include/dg.h"

namespace dg {

void set_error(const char* fmt, ...);

// Launches `kern` with programmatic dependent launch allowed: the kernel may be
// scheduled while its predecessor on the stream is still running; every kernel
// of the library calls griddepcontrol.wait before touching global memory the
// predecessor writes or reads, so only launch latency and prologues overlap.
// cluster_z > 1 additionally groups CTAs into clusters of that size along z.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, int cluster_z, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  int n = 0;
  at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_z > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = 1;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = cluster_z;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

#define DG_TRY_CUDA(call)                                                            \
  do {                                                                               \
    cudaError_t e_ = (call);                                                         \
    if (e_ != cudaSuccess) {                                                         \
      ::dg::set_error("%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), __FILE__, \
                      __LINE__);                                                     \
      return e_ == cudaErrorMemoryAllocation ? DG_ERR_OOM : DG_ERR_CUDA;             \
    }                                                                                \
  } while (0)

#define DG_REQUIRE(cond, ...)        \
  do {                               \
    if (!(cond)) {                   \
      ::dg::set_error(__VA_ARGS__);  \
      return DG_ERR_INVALID_ARG;     \
    }                                \
  } while (0)

#define DG_TRY(expr)                 \
  do {                               \
    dg_status s_ = (expr);           \
    if (s_ != DG_OK) return s_;      \
  } while (0)

// Device error bits (set by kernels, read and cleared by dg_sync_status).
enum : int { ERR_BAD_TOKEN = 1, ERR_TIMEOUT = 2, ERR_BAD_SHAPE = 4 };
constexpr int ATT_MAX_SPLITS = 8;
// shared memory of the fused permutation + gather (ranks and row tokens of all
// (token, slot) entries kept on chip); above it the two steps run separately
constexpr size_t PERMUTE_FUSED_SMEM = 200 * 1024;

// A typed device allocation owned by the workspace.
struct DevBuf {
  void* p = nullptr;
  size_t bytes = 0;
};

struct Workspace {
  size_t max_tok = 0;       // rows of every per-token buffer
  size_t max_rows = 0;      // max_tok * top_k routed rows
  std::vector<DevBuf> bufs; // for release
  // per-token buffers (element types depend on the precision path)
  void *x = nullptr, *xn = nullptr, *qkv = nullptr, *q = nullptr, *o = nullptr;
  void *kc = nullptr, *vc = nullptr;          // current layer's own keys/values
  void *ys = nullptr, *sh = nullptr;          // shared expert output / hidden
  // routing
  int32_t *ridx = nullptr, *rank = nullptr, *row_of = nullptr, *tok_of = nullptr;
  void *rgate = nullptr, *gate_of = nullptr;
  void *inv_rms = nullptr, *rlog = nullptr;  // per-row 1/rms; split-K router partials
  void* u2 = nullptr;  // [rows, 2 d] two-term split of the normalised rows (tensor-core router)
  int32_t* ready = nullptr;  // [max_tiles] phase-1 units finished per token chunk (routed experts)
  int32_t *counts = nullptr, *offsets = nullptr, *tile_e = nullptr, *tile_m0 = nullptr,
          *n_tiles = nullptr;
  void *up = nullptr, *hb = nullptr, *yb = nullptr; // routed rows
  void* lm_part = nullptr;                          // [n_vtiles, max_tok, 4]
  int32_t* load = nullptr;                          // [L, E] routing counts
  int32_t* err = nullptr;                           // device error bits
  unsigned long long* units = nullptr;              // (layer pass, expert) pairs with rows
  int32_t* ids = nullptr;                           // [max_tok] token ids of the pass
  void* rope = nullptr;                             // [max_pos, h/2] cos then sin
  uint8_t* mask = nullptr;                          // [max_batch, C] block-loop mask
  float* ent = nullptr;                             // [max_batch, C] entropies
  int32_t *amax = nullptr, *ncommit = nullptr;      // [max_batch, C], [max_batch]
  int32_t *remaining = nullptr, *loop_s = nullptr;  // [max_batch] masked left; steps left
  int32_t* blk = nullptr;                           // [max_batch, C] a finished block
  // annealed sampler: Gumbel-max draws [max_batch, C], previous argmax [max_batch, C],
  // per-canvas stop state [max_batch], per-tile race winners [n_vtiles, max_batch C, 2]
  int32_t *sampled = nullptr, *prev = nullptr, *astate = nullptr;
  void* gpart = nullptr;
  // self-conditioning (models with sc_inter > 0): the transposed embedding [d, V],
  // p0 [max_batch C, V], per-tile (ref, sum) [n_vtiles, max_batch C, 2], y = p0 E
  // [max_tok, d], the FFW hidden [max_tok, sc_inter], the K-sliced partials
  // [parts, max_batch C, d] (tensor-core path) and z [max_batch C, d]
  void *embT = nullptr, *scP = nullptr, *scref = nullptr, *scy = nullptr, *sch = nullptr;
  float* scpart = nullptr;
  void* z = nullptr;
  int max_pos = 0;
  size_t kc_elems = 0;
  int max_tiles = 0;
  int n_vtiles = 0;
};

}  // namespace dg

namespace dg {
// A captured block (T forwards + sampler steps) and what it was captured for.
struct BlockGraph {
  cudaGraphExec_t exec = nullptr;
  const dg_kv* kv = nullptr;
  int kv_P = 0, kv_W = 0;  // the handle's context when captured (positions, window)
  int T = 0;
  long long gq = 0;
  int32_t *canvas = nullptr, *nfwd = nullptr, *load = nullptr;
  bool prof = false;
  int fcap = 0;            // forwards of a profiled (unrolled) block, 0: T
  // annealed block: its constants and seeds (anneal false: the Entropy-Bound block)
  bool anneal = false;
  bool sc = false;  // captured with the self-conditioning signal carried
  int aN = 0;
  float ab = 0.f, atmax = 0.f, atmin = 0.f, aestop = 0.f;
  const void* seeds = nullptr;
  long long launches = 0;  // kernel launches the graph replays (1 for a loop graph: the init)
  bool loop = false;       // device-controlled WHILE loop over forwards
  long long body_launches = 0;  // kernels per loop iteration (forward + sampler + control)
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> ev[DG_KIND_COUNT];
};
}  // namespace dg

struct dg_model {
  dg_config cfg;
  dg_weights w;
  std::vector<dg_layer_weights> layers;
  int device = 0;
  dg::Workspace ws;
  long long launches = 0;  // kernels launched (host count)
  // event recording around launch groups, per dg_kernel_kind
  bool profiling = false;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> prof[DG_KIND_COUNT];
  size_t prof_used[DG_KIND_COUNT] = {};
  double prof_acc_ms[DG_KIND_COUNT] = {};  // from graph replays
  int64_t prof_acc_n[DG_KIND_COUNT] = {};
  int prof_forwards = 0;  // forwards of a profiled block (0: T)
  // captured blocks
  bool use_graphs = true;
  std::vector<dg::BlockGraph*> graphs;
  dg::BlockGraph* capture = nullptr;  // graph being captured (events go there)
  cudaStream_t cap_stream = nullptr;  // private stream used only for capturing
  // second stream for the shared expert, forked after the MoE RMSNorm and joined
  // before the combine (concurrent graph branches when captured)
  cudaStream_t side_stream = nullptr;
  int n_sm_cache = 148;  // multiprocessors of the model's device
  cudaEvent_t fork_ev = nullptr, join_ev = nullptr;
  long long last_body_launches = 0;   // kernels per forward of the last replayed loop graph
  std::vector<dg_kv*> kvs;            // live KV caches created from this model
  // > 0: the next routed-expert launch stalls its down units on purpose, with every
  // wait limited to this many ns (dg_debug_stall_experts; tests of the timeout path)
  long long stall_limit_ns = 0;
  bool selfcond = false;  // block loops carry the self-conditioning signal (sc_inter > 0)
};

namespace dg {
void release_graphs(dg_model* m);
}

namespace dg {
// RAII bracket recording a start/stop event pair around a launch group.
struct ProfScope {
  dg_model* m;
  int kind;
  cudaStream_t st;
  cudaEvent_t stop = nullptr;
  bool external = false;
  ProfScope(dg_model* m_, int kind_, cudaStream_t st_) : m(m_), kind(kind_), st(st_) {
    if (!m->profiling) return;
    if (m->capture) {  // events owned by the graph being captured
      cudaEvent_t a, b;
      cudaEventCreate(&a);
      cudaEventCreate(&b);
      m->capture->ev[kind].push_back({a, b});
      // "external" records become event-record nodes that fire on every replay
      cudaEventRecordWithFlags(a, st, cudaEventRecordExternal);
      stop = b;
      external = true;
      return;
    }
    auto& pool = m->prof[kind];
    size_t& used = m->prof_used[kind];
    if (used == pool.size()) {
      cudaEvent_t a, b;
      cudaEventCreate(&a);
      cudaEventCreate(&b);
      pool.push_back({a, b});
    }
    cudaEventRecord(pool[used].first, st);
    stop = pool[used].second;
    ++used;
  }
  void end() {
    if (stop) {
      if (external)
        cudaEventRecordWithFlags(stop, st, cudaEventRecordExternal);
      else
        cudaEventRecord(stop, st);
    }
    stop = nullptr;
  }
  ~ProfScope() { end(); }
};
}  // namespace dg

struct dg_kv {
  dg_model* m = nullptr;
  int B = 0, P = 0, W = 0;
  int Wp = 0;         // W rounded up to 64 (padding reads as zero)
  void* k = nullptr;  // keys [L, B, Hkv, Wp, h]
  void* v = nullptr;  // values, transposed: [L, B, Hkv, h, Wp]
  size_t elem = 0;    // bytes per element
};
