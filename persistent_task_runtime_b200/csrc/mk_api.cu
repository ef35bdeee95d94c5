// Host side of the decode megakernel: the C ABI of mk.h.  A plan binds the
// layout of mk_layout.cu (task graph, shared-memory carve-up, workspace,
// counters, RoPE table) to device allocations it owns.
//
// Event counters grow monotonically; in step e a task waits for
// e * required completions, so no counter is reset between steps.

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "mk_internal.h"

using mk::Params;
using mk::Task;

namespace {

thread_local std::string g_err;

int fail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

#define MK_CUDA(call)                                                                  \
  do {                                                                                 \
    cudaError_t e_ = (call);                                                           \
    if (e_ != cudaSuccess)                                                             \
      return fail(MK_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));        \
  } while (0)

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace mk {
void set_last_error(const char *msg) { g_err = msg; }
}  // namespace mk

// A per-operator step recorded as a CUDA graph (MK_MODE_PER_OP_GRAPH): the
// launches of one set of step arguments on one stream.  A replay patches the
// step counter into every kernel node.
struct OpGraph {
  Params key{};                  // the step's parameters, step counter zeroed
  cudaStream_t stream = nullptr;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  std::vector<cudaGraphNode_t> nodes;       // kernel nodes
  std::vector<cudaKernelNodeParams> kp;     // their launch configurations
  std::vector<Params> params;               // their parameters
  uint64_t used = 0;                        // last use (least recently used is replaced)
};

struct mk_plan {
  mk_model_config cfg;
  Params base;  // static part of the kernel parameters
  int dev = 0;
  int grid = 0;
  int smem = 0;
  int max_batch = 1;
  uint32_t epoch = 0;
  mk::Layout lay;           // tasks, per-operator ranges, workspace layout
  void *d_tasks = nullptr, *d_rope = nullptr, *d_ws = nullptr, *d_maps = nullptr;
  void *d_sched = nullptr;   // solidified schedule: offsets [grid + 1], then task indices
  void *d_kvmaps = nullptr;  // tensor maps of the KV cache (2 per layer) for the attention
  std::vector<const void *> kv_key;        // the KV cache those maps describe
  std::vector<unsigned char> kv_maps_host;
  uint32_t *d_sync = nullptr;
  size_t sync_words = 0;
  int32_t *d_host_ids = nullptr, *d_host_pos = nullptr, *d_host_out = nullptr;
  float *d_host_logits = nullptr;
  mk_plan_info_t info{};
  OpGraph graphs[2];   // two argument sets: a caller may alternate input/output buffers
  uint64_t graph_clock = 0;
};

namespace {

int validate_weights(const mk_model_config *c, const mk_weights *w) {
  if (w == nullptr || w->layers == nullptr)
    return fail(MK_ERR_INVALID_ARG, "weights or weights->layers is NULL");
  const void *top[] = {w->embed, w->final_norm, w->lm_head};
  for (const void *p : top) {
    if (p == nullptr) return fail(MK_ERR_INVALID_ARG, "a top-level weight pointer is NULL");
    if (!aligned16(p)) return fail(MK_ERR_INVALID_ARG, "weight pointers must be 16-byte aligned");
  }
  for (int l = 0; l < c->n_layers; ++l) {
    const mk_layer_weights &L = w->layers[l];
    const void *ps[] = {L.attn_norm, L.mlp_norm, L.wq, L.wk, L.wv, L.wo, L.w_gate, L.w_up, L.w_down};
    // (4-bit plans take the projections from w4_layers: only the norms here)
    const int np = w->w4_layers != nullptr ? 2 : 9;
    for (int i = 0; i < np; ++i) {
      const void *p = ps[i];
      if (p == nullptr) return fail(MK_ERR_INVALID_ARG, "layer %d: a weight pointer is NULL", l);
      if (!aligned16(p)) return fail(MK_ERR_INVALID_ARG, "layer %d: weight not 16-byte aligned", l);
    }
    if (w->w4_layers != nullptr)
      for (int j = 0; j < 7; ++j) {
        const void *p = w->w4_layers[l].q[j];
        if (p == nullptr || !aligned16(p))
          return fail(MK_ERR_INVALID_ARG, "layer %d: a 4-bit matrix is NULL or not 16-byte aligned", l);
      }
    if (c->qk_norm && (L.q_norm == nullptr || L.k_norm == nullptr))
      return fail(MK_ERR_INVALID_ARG, "layer %d: q_norm/k_norm NULL with qk_norm on", l);
  }
  return MK_OK;
}

// Plan options -> layout options (defaults filled in).  `w` (NULL when
// describing a plan) says whether the weights are 4-bit.
int layout_options(const mk_plan_options *opts, mk::LayoutOptions &lo, const mk_weights *w = nullptr) {
  mk_plan_options o{};
  if (opts) o = *opts;
  if (o.weight_bits != 0 && o.weight_bits != 4 && o.weight_bits != 16)
    return fail(MK_ERR_INVALID_ARG, "weight_bits %d: 0, 4 or 16", o.weight_bits);
  const bool have4 = w != nullptr && w->w4_layers != nullptr;
  if (w != nullptr && o.weight_bits != 0 && (o.weight_bits == 4) != have4)
    return fail(MK_ERR_INVALID_ARG, "weight_bits %d does not match the weights (w4_layers %s)",
                o.weight_bits, have4 ? "set" : "NULL");
  lo.w4 = have4 || (w == nullptr && o.weight_bits == 4);
  if (o.wait_limit_ns < 0) return fail(MK_ERR_INVALID_ARG, "wait_limit_ns < 0");
  lo.max_batch = o.max_batch == 0 ? 1 : o.max_batch;
  lo.page_size = o.kv_page_size == 0 ? 16 : o.kv_page_size;
  lo.num_ctas = o.num_ctas;
  lo.max_page_cols = o.max_page_cols;
  lo.o_split = o.o_split != 0;
  lo.gemv_path = o.gemv_path;
  lo.schedule = o.schedule;
  lo.prefill = o.prefill != 0;
  lo.attn_path = o.attn_path;
  for (int i = 0; i < 5; ++i) lo.rows_per_task[i] = o.rows_per_task[i];
  lo.wait_limit_ns = o.wait_limit_ns == 0 ? 2000000000LL : o.wait_limit_ns;
  lo.debug_unsatisfiable_dep = o.debug_unsatisfiable_dep != 0;
  return MK_OK;
}

void fill_info(const mk::Layout &lay, const mk_model_config &c, mk_plan_info_t &I) {
  const Params &p = lay.p;
  const int L = c.n_layers, H = c.hidden, d = c.head_dim, F = c.ffn, V = c.vocab;
  I = mk_plan_info_t{};
  I.num_ctas = lay.grid;
  I.threads_per_cta = mk::kThreads;
  I.smem_bytes = lay.smem;
  I.n_pages = p.n_pages;
  I.page_bytes = p.page_bytes;
  I.n_tasks = p.n_tasks;
  I.n_events = lay.n_events;
  I.attn_slots = p.attn_slots;
  I.tokens_per_smem_page = p.tpp;
  for (int i = 0; i < 5; ++i) I.rows_per_task[i] = lay.rows[i];
  for (int i = 0; i < 4; ++i) I.page_cols[i] = p.kp[i];
  I.weight_bytes = 2LL * L *
                       (static_cast<long long>(p.NQKV) * H + static_cast<long long>(H) * c.n_q_heads * d +
                        3LL * F * H) +
                   2LL * V * H;
  if (p.w4) {   // packed 4-bit projections (codes and scales) + the bf16 LM head
    const long long per_layer = mk_w4_packed_bytes(p.NQKV - 2 * c.n_kv_heads * d, H) +
                                2 * mk_w4_packed_bytes(c.n_kv_heads * d, H) +
                                mk_w4_packed_bytes(H, c.n_q_heads * d) +
                                2 * mk_w4_packed_bytes(F, H) + mk_w4_packed_bytes(H, F);
    I.weight_bytes = L * per_layer + 2LL * V * H;
  }
  I.weight_bits = p.w4 ? 4 : 16;
  I.events_per_layer = p.ev_per_layer;
  I.attn_slots_per_group = p.attn_spg;
  I.qkv_tasks_per_group = p.qkv_tasks_per_group;
  I.ffn_parts = p.n_ffn_parts;
  I.ffn_part_cols = p.kchunk[mk::K_FFN] > 0 ? p.kchunk[mk::K_FFN] : F;
  I.o_parts = p.n_o_parts;
  I.o_part_cols = p.kchunk[mk::K_ATT] > 0 ? p.kchunk[mk::K_ATT] : c.n_q_heads * d;
  if (p.tc) {
    I.o_part_cols = p.tc_kt[mk::T_OPROJ] > 0 ? p.tc_kt[mk::T_OPROJ] : c.n_q_heads * d;
    I.ffn_part_cols = p.tc_kt[mk::T_DOWN] > 0 ? p.tc_kt[mk::T_DOWN] : F;
  }
  I.gemv_path = p.tc ? 2 : (p.tm ? 3 : 1);
  I.schedule = lay.sched.empty() ? 0 : 1;
  I.prefill = lay.p.kv_tasks;
  I.qkv_parts = lay.splits[0];
  I.gateup_parts = lay.splits[2];
  I.attn_path = p.attn_mma ? 2 : 1;
}

}  // namespace

extern "C" {

const char *mk_last_error(void) { return g_err.c_str(); }

int mk_plan_create(const mk_model_config *cfg, const mk_weights *weights, int max_batch,
                   int kv_page_size, mk_plan **out) {
  mk_plan_options o{};
  o.max_batch = max_batch;
  o.kv_page_size = kv_page_size;
  return mk_plan_create_ex(cfg, weights, &o, out);
}

int mk_plan_create_ex(const mk_model_config *cfg, const mk_weights *w, const mk_plan_options *opts,
                      mk_plan **out) {
  g_err.clear();
  if (out == nullptr) return fail(MK_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (cfg == nullptr) return fail(MK_ERR_INVALID_ARG, "cfg is NULL");
  int rc = mk::validate_config(*cfg, g_err);
  if (rc) return rc;
  rc = validate_weights(cfg, w);
  if (rc) return rc;
  mk::LayoutOptions lo;
  rc = layout_options(opts, lo, w);
  if (rc) return rc;

  int dev = 0, nsm = 0, smem_optin = 0, coop = 0;
  MK_CUDA(cudaGetDevice(&dev));
  MK_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
  MK_CUDA(cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
  MK_CUDA(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev));
  if (!coop) return fail(MK_ERR_UNSUPPORTED, "device lacks cooperative launch");

  auto plan = new mk_plan();
  mk::Layout &lay = plan->lay;
  rc = mk::build_layout(*cfg, lo, nsm, smem_optin, lay, g_err);
  if (rc) {
    delete plan;
    return rc;
  }
  plan->cfg = *cfg;
  plan->dev = dev;
  plan->grid = lay.grid;
  plan->smem = lay.smem;
  plan->max_batch = lo.max_batch;
  Params &p = plan->base;
  p = lay.p;

  // ---- device allocations ---------------------------------------------------------
  auto cleanup_fail = [&](int code) {
    mk_plan_destroy(plan);
    return code;
  };
  auto upload = [&](void **dst, const void *src, size_t bytes, const char *what) {
    cudaError_t e = cudaMalloc(dst, bytes);
    if (e == cudaSuccess) e = cudaMemcpy(*dst, src, bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return fail(MK_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return MK_OK;
  };
  mk::bind_task_operands(*cfg, *w, lay.tasks);
  if ((rc = upload(&plan->d_tasks, lay.tasks.data(), lay.tasks.size() * sizeof(Task), "task array")) ||
      (rc = upload(&plan->d_rope, lay.rope.data(), lay.rope.size() * sizeof(float2), "RoPE table")))
    return cleanup_fail(rc);
  if (!lay.sched.empty()) {
    std::vector<int> both(lay.sched_off);
    both.insert(both.end(), lay.sched.begin(), lay.sched.end());
    if ((rc = upload(&plan->d_sched, both.data(), both.size() * sizeof(int), "schedule")))
      return cleanup_fail(rc);
  }
  cudaError_t e = cudaMalloc(&plan->d_ws, lay.ws_bytes);
  if (e == cudaSuccess) e = cudaMemset(plan->d_ws, 0, lay.ws_bytes);
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "workspace: %s", cudaGetErrorString(e)));
  e = cudaMalloc(&plan->d_sync, lay.sync_words * sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(plan->d_sync, 0, lay.sync_words * sizeof(uint32_t));
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "counters: %s", cudaGetErrorString(e)));
  plan->sync_words = lay.sync_words;
  if (lay.n_maps > 0) {   // (the staged-input maps point into the workspace)
    std::vector<unsigned char> maps;
    rc = mk::encode_weight_maps(*cfg, *w, lay, static_cast<const char *>(plan->d_ws), maps, g_err);
    if (rc) return cleanup_fail(rc);
    if ((rc = upload(&plan->d_maps, maps.data(), maps.size(), "tensor maps"))) return cleanup_fail(rc);
  }
  mk::bind_workspace(lay, static_cast<char *>(plan->d_ws), plan->d_sync, p);
  p.tasks = static_cast<const Task *>(plan->d_tasks);
  p.embed = static_cast<const __nv_bfloat16 *>(w->embed);
  p.rope_cs = static_cast<const float2 *>(plan->d_rope);
  p.tmaps = plan->d_maps;
  if (p.attn_mma) {
    e = cudaMalloc(&plan->d_kvmaps, static_cast<size_t>(2 * cfg->n_layers) * 128);
    if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "KV maps: %s", cudaGetErrorString(e)));
    p.kvmaps = plan->d_kvmaps;
  }
  if (plan->d_sched != nullptr) {
    p.sched_off = static_cast<const int *>(plan->d_sched);
    p.sched = p.sched_off + lay.sched_off.size();
  }

  e = cudaMalloc(&plan->d_host_ids, 3 * sizeof(int32_t) * MK_MAX_BATCH);
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "cudaMalloc staging: %s", cudaGetErrorString(e)));
  plan->d_host_pos = plan->d_host_ids + MK_MAX_BATCH;
  plan->d_host_out = plan->d_host_pos + MK_MAX_BATCH;

  e = mk::configure_kernel(smem_optin);
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "kernel attribute: %s", cudaGetErrorString(e)));

  fill_info(lay, *cfg, plan->info);
  *out = plan;
  return MK_OK;
}

static int validate_kv(const mk_plan *plan, const mk_kv_cache *kv) {
  if (kv == nullptr || kv->k_pages == nullptr || kv->v_pages == nullptr ||
      kv->block_table == nullptr)
    return fail(MK_ERR_INVALID_ARG, "kv cache or one of its arrays is NULL");
  if (kv->num_pages < 1 || kv->max_pages_per_seq < 1)
    return fail(MK_ERR_INVALID_ARG, "kv num_pages and max_pages_per_seq must be >= 1");
  if (!aligned16(kv->block_table)) return fail(MK_ERR_INVALID_ARG, "block_table not 16-byte aligned");
  for (int l = 0; l < plan->cfg.n_layers; ++l) {
    if (kv->k_pages[l] == nullptr || kv->v_pages[l] == nullptr)
      return fail(MK_ERR_INVALID_ARG, "kv pages of layer %d are NULL", l);
    if (!aligned16(kv->k_pages[l]) || !aligned16(kv->v_pages[l]))
      return fail(MK_ERR_INVALID_ARG, "kv pages of layer %d not 16-byte aligned", l);
  }
  return MK_OK;
}

namespace {

// The attention copies K/V pages with TMA tensor copies: the tensor maps of
// the step's KV cache, encoded when the cache (its pointers or page count)
// differs from the previous step's and copied to the device on the step's
// stream ahead of the launch.
int ensure_kv_maps(mk_plan *plan, const mk_kv_cache *kv, cudaStream_t s) {
  if (!plan->base.attn_mma) return MK_OK;
  std::vector<const void *> key;
  key.reserve(2 * plan->cfg.n_layers + 1);
  key.push_back(reinterpret_cast<const void *>(static_cast<intptr_t>(kv->num_pages)));
  for (int l = 0; l < plan->cfg.n_layers; ++l) {
    key.push_back(kv->k_pages[l]);
    key.push_back(kv->v_pages[l]);
  }
  if (key == plan->kv_key) return MK_OK;
  std::string err;
  const int rc = mk::encode_kv_maps(plan->cfg, *kv, plan->base.page_size, plan->kv_maps_host, err);
  if (rc) return fail(rc, "%s", err.c_str());
  MK_CUDA(cudaMemcpyAsync(plan->d_kvmaps, plan->kv_maps_host.data(), plan->kv_maps_host.size(),
                          cudaMemcpyHostToDevice, s));
  plan->kv_key = std::move(key);
  return MK_OK;
}

void release_graph(OpGraph &g) {
  if (g.exec != nullptr) cudaGraphExecDestroy(g.exec);
  if (g.graph != nullptr) cudaGraphDestroy(g.graph);
  g = OpGraph{};
}

// Record the per-operator launches of `p` on `s` into `g`.
int record_graph(mk_plan *plan, const Params &p, cudaStream_t s, OpGraph &g) {
  release_graph(g);
  MK_CUDA(cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal));
  Params q = p;
  for (const mk::OpRange &r : plan->lay.ops) {
    q.task_begin = r.begin;
    q.task_end = r.end;
    const cudaError_t e = mk::launch_step(q, std::min(plan->grid, r.end - r.begin), plan->smem,
                                          false, s);
    if (e != cudaSuccess) {
      cudaGraph_t partial = nullptr;
      cudaStreamEndCapture(s, &partial);
      if (partial != nullptr) cudaGraphDestroy(partial);
      return fail(MK_ERR_CUDA, "per-op graph capture: %s", cudaGetErrorString(e));
    }
  }
  MK_CUDA(cudaStreamEndCapture(s, &g.graph));
  MK_CUDA(cudaGraphInstantiate(&g.exec, g.graph, 0));
  size_t n = 0;
  MK_CUDA(cudaGraphGetNodes(g.graph, nullptr, &n));
  std::vector<cudaGraphNode_t> all(n);
  MK_CUDA(cudaGraphGetNodes(g.graph, all.data(), &n));
  for (cudaGraphNode_t node : all) {
    cudaGraphNodeType type;
    MK_CUDA(cudaGraphNodeGetType(node, &type));
    if (type != cudaGraphNodeTypeKernel) continue;
    cudaKernelNodeParams kp{};
    MK_CUDA(cudaGraphKernelNodeGetParams(node, &kp));
    g.nodes.push_back(node);
    g.params.push_back(*static_cast<const Params *>(kp.kernelParams[0]));
    kp.kernelParams = nullptr;
    kp.extra = nullptr;
    g.kp.push_back(kp);
  }
  if (g.nodes.size() != plan->lay.ops.size()) {
    release_graph(g);
    return fail(MK_ERR_CUDA, "per-op graph holds an unexpected number of kernels");
  }
  g.key = p;
  g.key.epoch = 0;
  g.stream = s;
  return MK_OK;
}

// Replay the per-operator graph for `p` on `s`, recording it first if no
// recorded graph matches the step's arguments and stream.
int replay_graph(mk_plan *plan, const Params &p, cudaStream_t s) {
  Params key = p;
  key.epoch = 0;
  OpGraph *g = nullptr;
  for (OpGraph &c : plan->graphs)
    if (c.exec != nullptr && c.stream == s && std::memcmp(&c.key, &key, sizeof(Params)) == 0) g = &c;
  if (g == nullptr) {
    g = &plan->graphs[0];
    for (OpGraph &c : plan->graphs)
      if (c.used < g->used) g = &c;
    const int rc = record_graph(plan, p, s, *g);
    if (rc) return rc;
  }
  g->used = ++plan->graph_clock;
  for (size_t i = 0; i < g->nodes.size(); ++i) {
    g->params[i].epoch = p.epoch;
    void *args[] = {&g->params[i]};
    cudaKernelNodeParams kp = g->kp[i];
    kp.kernelParams = args;
    MK_CUDA(cudaGraphExecKernelNodeSetParams(g->exec, g->nodes[i], &kp));
  }
  MK_CUDA(cudaGraphLaunch(g->exec, s));
  return MK_OK;
}

}  // namespace

int mk_decode_step_ex(mk_plan *plan, const mk_step_args *a, void *stream) {
  g_err.clear();
  if (plan == nullptr || a == nullptr) return fail(MK_ERR_INVALID_ARG, "plan or args is NULL");
  if (a->batch < 1 || a->batch > plan->max_batch)
    return fail(MK_ERR_INVALID_ARG, "batch %d outside 1..max_batch %d", a->batch, plan->max_batch);
  if (a->d_ids == nullptr || a->d_pos == nullptr || a->d_out_ids == nullptr)
    return fail(MK_ERR_INVALID_ARG, "d_ids, d_pos and d_out_ids must not be NULL");
  if (a->mode != MK_MODE_MEGAKERNEL && a->mode != MK_MODE_PER_OP && a->mode != MK_MODE_PER_OP_GRAPH)
    return fail(MK_ERR_INVALID_ARG, "unknown mode %d", a->mode);
  if (a->mode == MK_MODE_PER_OP_GRAPH && stream == nullptr)
    return fail(MK_ERR_INVALID_ARG, "graph mode needs a created stream, not the legacy default stream");
  int rc = validate_kv(plan, a->kv);
  if (rc) return rc;
  rc = ensure_kv_maps(plan, a->kv, static_cast<cudaStream_t>(stream));
  if (rc) return rc;

  Params p = plan->base;
  plan->epoch += 1;
  p.epoch = plan->epoch;
  p.batch = a->batch;
  p.chunk_seq = -1;
  p.mode = a->mode;
  p.ids = a->d_ids;
  p.pos = a->d_pos;
  p.out_ids = a->d_out_ids;
  p.out_pos = a->d_out_pos;
  p.out_logits = a->d_out_logits;
  p.hidden_dump = a->d_hidden;
  p.trace = reinterpret_cast<unsigned long long *>(a->d_trace);
  p.block_table = a->kv->block_table;
  p.num_kv_pages = a->kv->num_pages;
  p.max_pages_per_seq = a->kv->max_pages_per_seq;
  const long long cap = static_cast<long long>(a->kv->max_pages_per_seq) * p.page_size;
  p.max_pos = static_cast<int>(std::min<long long>(plan->cfg.max_seq_len, cap));
  for (int l = 0; l < plan->cfg.n_layers; ++l) {
    p.k_pages[l] = static_cast<__nv_bfloat16 *>(a->kv->k_pages[l]);
    p.v_pages[l] = static_cast<__nv_bfloat16 *>(a->kv->v_pages[l]);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a->mode != MK_MODE_MEGAKERNEL) {
    // per-operator launches take their operator's tasks from the queue
    p.sched = nullptr;
    p.sched_off = nullptr;
  }
  if (a->mode == MK_MODE_MEGAKERNEL) {
    p.task_begin = 0;
    p.task_end = p.n_tasks;
    cudaError_t e = mk::launch_step(p, plan->grid, plan->smem, true, s);
    if (e != cudaSuccess) {
      plan->epoch -= 1;
      return fail(MK_ERR_CUDA, "megakernel launch: %s", cudaGetErrorString(e));
    }
  } else if (a->mode == MK_MODE_PER_OP_GRAPH) {
    const int rc2 = replay_graph(plan, p, s);
    if (rc2) {
      plan->epoch -= 1;
      return rc2;
    }
  } else {
    for (const mk::OpRange &r : plan->lay.ops) {
      p.task_begin = r.begin;
      p.task_end = r.end;
      const int grid = std::min(plan->grid, r.end - r.begin);
      cudaError_t e = mk::launch_step(p, grid, plan->smem, false, s);
      if (e != cudaSuccess) return fail(MK_ERR_CUDA, "per-op launch: %s", cudaGetErrorString(e));
    }
  }
  return MK_OK;
}

int mk_prefill_chunk(mk_plan *plan, const mk_prefill_args *a, void *stream) {
  g_err.clear();
  if (plan == nullptr || a == nullptr) return fail(MK_ERR_INVALID_ARG, "plan or args is NULL");
  if (!plan->base.kv_tasks)
    return fail(MK_ERR_INVALID_ARG, "the plan was not created with the prefill option");
  if (a->n_tokens < 1 || a->n_tokens > plan->max_batch)
    return fail(MK_ERR_INVALID_ARG, "n_tokens %d outside 1..max_batch %d", a->n_tokens,
                plan->max_batch);
  if (a->seq < 0 || a->seq >= plan->max_batch)
    return fail(MK_ERR_INVALID_ARG, "seq %d outside 0..max_batch-1", a->seq);
  if (a->pos0 < 0 || a->pos0 + a->n_tokens > plan->cfg.max_seq_len)
    return fail(MK_ERR_INVALID_ARG, "positions %d..%d outside 0..max_seq_len-1", a->pos0,
                a->pos0 + a->n_tokens - 1);
  if (a->d_ids == nullptr || (a->with_lm_head && a->d_out_ids == nullptr))
    return fail(MK_ERR_INVALID_ARG, "d_ids (and, with the LM head, d_out_ids) must not be NULL");
  if (!a->with_lm_head && a->d_out_logits != nullptr)
    return fail(MK_ERR_INVALID_ARG, "d_out_logits needs with_lm_head");
  int rc = validate_kv(plan, a->kv);
  if (rc) return rc;
  rc = ensure_kv_maps(plan, a->kv, static_cast<cudaStream_t>(stream));
  if (rc) return rc;
  Params p = plan->base;
  plan->epoch += 1;
  p.epoch = plan->epoch;
  p.batch = a->n_tokens;
  p.chunk_seq = a->seq;
  p.chunk_pos0 = a->pos0;
  p.mode = MK_MODE_MEGAKERNEL;
  p.ids = a->d_ids;
  p.pos = nullptr;
  p.out_ids = a->d_out_ids;
  p.out_pos = nullptr;
  p.out_logits = a->d_out_logits;
  p.hidden_dump = a->d_hidden;
  p.trace = nullptr;
  p.block_table = a->kv->block_table;
  p.num_kv_pages = a->kv->num_pages;
  p.max_pages_per_seq = a->kv->max_pages_per_seq;
  const long long cap = static_cast<long long>(a->kv->max_pages_per_seq) * p.page_size;
  p.max_pos = static_cast<int>(std::min<long long>(plan->cfg.max_seq_len, cap));
  for (int l = 0; l < plan->cfg.n_layers; ++l) {
    p.k_pages[l] = static_cast<__nv_bfloat16 *>(a->kv->k_pages[l]);
    p.v_pages[l] = static_cast<__nv_bfloat16 *>(a->kv->v_pages[l]);
  }
  p.task_begin = 0;
  // without the LM head the launch ends with the last layer (the queue and a
  // solidified schedule both skip the LM-head tasks)
  p.task_end = a->with_lm_head ? p.n_tasks : plan->lay.first_lm_task;
  if (!a->with_lm_head && p.sched != nullptr) {
    p.sched = nullptr;   // the per-CTA lists include LM-head tasks: use the queue
    p.sched_off = nullptr;
  }
  const cudaError_t e = mk::launch_step(p, plan->grid, plan->smem, true,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    plan->epoch -= 1;
    return fail(MK_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
  }
  return MK_OK;
}

int mk_decode_step(mk_plan *plan, const int32_t *d_ids, const int32_t *d_pos, const mk_kv_cache *kv,
                   int batch, int32_t *d_out_ids, float *d_out_logits, void *stream) {
  mk_step_args a{};
  a.d_ids = d_ids;
  a.d_pos = d_pos;
  a.kv = kv;
  a.batch = batch;
  a.d_out_ids = d_out_ids;
  a.d_out_logits = d_out_logits;
  a.mode = MK_MODE_MEGAKERNEL;
  return mk_decode_step_ex(plan, &a, stream);
}

int mk_decode_step_host(mk_plan *plan, const int32_t *h_ids, const int32_t *h_pos,
                        const mk_kv_cache *kv, int batch, int32_t *h_out_ids, float *h_out_logits,
                        void *stream) {
  g_err.clear();
  if (plan == nullptr || h_ids == nullptr || h_pos == nullptr || h_out_ids == nullptr)
    return fail(MK_ERR_INVALID_ARG, "plan, h_ids, h_pos and h_out_ids must not be NULL");
  if (batch < 1 || batch > plan->max_batch)
    return fail(MK_ERR_INVALID_ARG, "batch %d outside 1..max_batch %d", batch, plan->max_batch);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (h_out_logits != nullptr && plan->d_host_logits == nullptr) {
    MK_CUDA(cudaMalloc(&plan->d_host_logits,
                       sizeof(float) * static_cast<size_t>(plan->max_batch) * plan->cfg.vocab));
  }
  MK_CUDA(cudaMemcpyAsync(plan->d_host_ids, h_ids, sizeof(int32_t) * batch, cudaMemcpyHostToDevice, s));
  MK_CUDA(cudaMemcpyAsync(plan->d_host_pos, h_pos, sizeof(int32_t) * batch, cudaMemcpyHostToDevice, s));
  mk_step_args a{};
  a.d_ids = plan->d_host_ids;
  a.d_pos = plan->d_host_pos;
  a.kv = kv;
  a.batch = batch;
  a.d_out_ids = plan->d_host_out;
  a.d_out_logits = h_out_logits ? plan->d_host_logits : nullptr;
  a.mode = MK_MODE_MEGAKERNEL;
  int rc = mk_decode_step_ex(plan, &a, stream);
  if (rc) return rc;
  uint32_t status = 0;
  MK_CUDA(cudaMemcpyAsync(h_out_ids, plan->d_host_out, sizeof(int32_t) * batch, cudaMemcpyDeviceToHost, s));
  if (h_out_logits)
    MK_CUDA(cudaMemcpyAsync(h_out_logits, plan->d_host_logits,
                            sizeof(float) * static_cast<size_t>(batch) * plan->cfg.vocab,
                            cudaMemcpyDeviceToHost, s));
  MK_CUDA(cudaMemcpyAsync(&status, plan->d_sync + mk::S_STATUS, sizeof(uint32_t),
                          cudaMemcpyDeviceToHost, s));
  MK_CUDA(cudaStreamSynchronize(s));
  return static_cast<int32_t>(status);
}

int mk_plan_status(mk_plan *plan) {
  g_err.clear();
  if (plan == nullptr) return fail(MK_ERR_INVALID_ARG, "plan is NULL");
  MK_CUDA(cudaDeviceSynchronize());
  uint32_t st = 0;
  MK_CUDA(cudaMemcpy(&st, plan->d_sync + mk::S_STATUS, sizeof(st), cudaMemcpyDeviceToHost));
  return static_cast<int32_t>(st);
}

int mk_plan_error_info(mk_plan *plan, int32_t *info) {
  g_err.clear();
  if (plan == nullptr || info == nullptr) return fail(MK_ERR_INVALID_ARG, "plan or info is NULL");
  MK_CUDA(cudaDeviceSynchronize());
  MK_CUDA(cudaMemcpy(info, plan->d_sync + mk::S_INFO, 4 * sizeof(int32_t), cudaMemcpyDeviceToHost));
  return MK_OK;
}

int mk_plan_reset(mk_plan *plan) {
  g_err.clear();
  if (plan == nullptr) return fail(MK_ERR_INVALID_ARG, "plan is NULL");
  MK_CUDA(cudaDeviceSynchronize());
  MK_CUDA(cudaMemset(plan->d_sync, 0, plan->sync_words * sizeof(uint32_t)));
  MK_CUDA(cudaMemset(plan->base.argmax, 0, sizeof(unsigned long long) * plan->max_batch));
  MK_CUDA(cudaDeviceSynchronize());
  plan->epoch = 0;
  return MK_OK;
}

int mk_plan_info(const mk_plan *plan, mk_plan_info_t *info) {
  if (plan == nullptr || info == nullptr) return fail(MK_ERR_INVALID_ARG, "plan or info is NULL");
  *info = plan->info;
  return MK_OK;
}

int mk_plan_describe(const mk_model_config *cfg, const mk_plan_options *opts, int num_sms,
                     int smem_optin, mk_plan_info_t *info, void *tasks, int64_t max_tasks) {
  g_err.clear();
  if (cfg == nullptr || info == nullptr) return fail(MK_ERR_INVALID_ARG, "cfg or info is NULL");
  if (num_sms < 1 || smem_optin < 1)
    return fail(MK_ERR_INVALID_ARG, "num_sms and smem_optin must be positive");
  int rc = mk::validate_config(*cfg, g_err);
  if (rc) return rc;
  mk::LayoutOptions lo;
  rc = layout_options(opts, lo);
  if (rc) return rc;
  mk::Layout lay;
  rc = mk::build_layout(*cfg, lo, num_sms, smem_optin, lay, g_err);
  if (rc) return rc;
  fill_info(lay, *cfg, *info);
  static_assert(sizeof(Task) == MK_TASK_RECORD_BYTES, "task record size");
  if (tasks != nullptr && max_tasks >= static_cast<int64_t>(lay.tasks.size()))
    std::memcpy(tasks, lay.tasks.data(), lay.tasks.size() * sizeof(Task));
  return MK_OK;
}

int mk_plan_describe_schedule(const mk_model_config *cfg, const mk_plan_options *opts,
                              int num_sms, int smem_optin, int32_t *cta_of_task,
                              int64_t max_tasks) {
  g_err.clear();
  if (cfg == nullptr || cta_of_task == nullptr)
    return fail(MK_ERR_INVALID_ARG, "cfg or cta_of_task is NULL");
  if (num_sms < 1 || smem_optin < 1)
    return fail(MK_ERR_INVALID_ARG, "num_sms and smem_optin must be positive");
  int rc = mk::validate_config(*cfg, g_err);
  if (rc) return rc;
  mk::LayoutOptions lo;
  rc = layout_options(opts, lo);
  if (rc) return rc;
  mk::Layout lay;
  rc = mk::build_layout(*cfg, lo, num_sms, smem_optin, lay, g_err);
  if (rc) return rc;
  if (max_tasks < static_cast<int64_t>(lay.tasks.size()))
    return fail(MK_ERR_INVALID_ARG, "cta_of_task holds %lld entries; the plan has %zu tasks",
                static_cast<long long>(max_tasks), lay.tasks.size());
  for (size_t i = 0; i < lay.tasks.size(); ++i) cta_of_task[i] = -1;
  for (size_t c = 0; c + 1 < lay.sched_off.size(); ++c)
    for (int k = lay.sched_off[c]; k < lay.sched_off[c + 1]; ++k)
      cta_of_task[lay.sched[static_cast<size_t>(k)]] = static_cast<int32_t>(c);
  return MK_OK;
}

void mk_plan_destroy(mk_plan *plan) {
  if (plan == nullptr) return;
  cudaDeviceSynchronize();
  for (OpGraph &g : plan->graphs) release_graph(g);
  cudaFree(plan->d_tasks);
  cudaFree(plan->d_rope);
  cudaFree(plan->d_maps);
  cudaFree(plan->d_sched);
  cudaFree(plan->d_kvmaps);
  cudaFree(plan->d_ws);
  cudaFree(plan->d_sync);
  cudaFree(plan->d_host_ids);
  cudaFree(plan->d_host_logits);
  delete plan;
}

}  // extern "C"
