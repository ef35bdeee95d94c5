// Host side of the decode megakernel: plan building (task graph, counters,
// shared-memory carve-up, RoPE table, workspace) and the C ABI of mk.h.
//
// The plan tiles every operator of every layer into tasks and gives each task
// the event it waits on and the number of completions that event needs per
// step -- the TaskDesc / Event{trigger_count, required_count} pair of the MPK
// write-up, "2.1 Mega-Kernel执行模型", re-laid out as a 32-byte descriptor.
// Counters grow monotonically; in step e a task waits for e * required, so no
// counter is ever reset between steps.

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
inline int align_up(int x, int a) { return (x + a - 1) / a * a; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Range {
  int begin, end;
};

}  // namespace

namespace mk {
void set_last_error(const char *msg) { g_err = msg; }
}  // namespace mk

struct mk_plan {
  mk_model_config cfg;
  Params base;  // static part of the kernel parameters
  int dev = 0;
  int grid = 0;
  int smem = 0;
  int max_batch = 1;
  uint32_t epoch = 0;
  std::vector<Task> tasks;
  std::vector<Range> ops;   // per-operator launch ranges (MK_MODE_PER_OP)
  void *d_tasks = nullptr, *d_layers = nullptr, *d_rope = nullptr, *d_ws = nullptr;
  uint32_t *d_sync = nullptr;
  size_t sync_words = 0;
  int32_t *d_host_ids = nullptr, *d_host_pos = nullptr, *d_host_out = nullptr;
  float *d_host_logits = nullptr;
  mk_plan_info_t info{};
};

namespace {

// Rows per task: small enough that every CTA gets ~16 tasks of an operator,
// so the dynamic queue evens out the operator's tail across SMs.
int choose_mtiles(int tiles, int nsm, int cap) {
  int nm = tiles / (16 * nsm);
  return std::max(1, std::min(cap, nm));
}

int validate_cfg(const mk_model_config *c) {
  if (c == nullptr) return fail(MK_ERR_INVALID_ARG, "cfg is NULL");
  if (c->n_layers < 1 || c->n_layers > MK_MAX_LAYERS)
    return fail(MK_ERR_UNSUPPORTED, "n_layers %d outside 1..%d", c->n_layers, MK_MAX_LAYERS);
  if (c->hidden <= 0 || c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 ||
      c->ffn <= 0 || c->vocab <= 0 || c->max_seq_len <= 0)
    return fail(MK_ERR_INVALID_ARG, "model dimensions must be positive");
  if (!(c->rms_eps >= 0.f) || !(c->rope_theta > 0.f))
    return fail(MK_ERR_INVALID_ARG, "rms_eps must be >= 0 and rope_theta > 0");
  const int d = c->head_dim;
  if (d != 32 && d != 64 && d != 128)
    return fail(MK_ERR_UNSUPPORTED, "head_dim %d: supported 32, 64, 128", d);
  if (c->n_q_heads % c->n_kv_heads != 0)
    return fail(MK_ERR_INVALID_ARG, "n_q_heads %d not a multiple of n_kv_heads %d",
                c->n_q_heads, c->n_kv_heads);
  if (c->n_q_heads / c->n_kv_heads > mk::kMaxGroup)
    return fail(MK_ERR_UNSUPPORTED, "more than %d query heads per KV head", mk::kMaxGroup);
  if (c->hidden % 8 || c->ffn % 8 || (c->n_q_heads * d) % 8)
    return fail(MK_ERR_UNSUPPORTED, "hidden, ffn and n_q_heads*head_dim must be multiples of 8");
  if (c->n_q_heads + 2 * c->n_kv_heads > 0xffff)
    return fail(MK_ERR_UNSUPPORTED, "too many heads");
  return MK_OK;
}

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
    const void *ps[] = {L.attn_norm, L.wq, L.wk, L.wv, L.wo, L.mlp_norm, L.w_gate, L.w_up, L.w_down};
    for (const void *p : ps) {
      if (p == nullptr) return fail(MK_ERR_INVALID_ARG, "layer %d: a weight pointer is NULL", l);
      if (!aligned16(p)) return fail(MK_ERR_INVALID_ARG, "layer %d: weight not 16-byte aligned", l);
    }
    if (c->qk_norm && (L.q_norm == nullptr || L.k_norm == nullptr))
      return fail(MK_ERR_INVALID_ARG, "layer %d: q_norm/k_norm NULL with qk_norm on", l);
  }
  return MK_OK;
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
  int rc = validate_cfg(cfg);
  if (rc) return rc;
  rc = validate_weights(cfg, w);
  if (rc) return rc;
  mk_plan_options o{};
  if (opts) o = *opts;
  if (o.max_batch == 0) o.max_batch = 1;
  if (o.kv_page_size == 0) o.kv_page_size = 16;
  if (o.wait_limit_ns == 0) o.wait_limit_ns = 2000000000LL;
  if (o.max_batch < 1 || o.max_batch > MK_MAX_BATCH)
    return fail(MK_ERR_INVALID_ARG, "max_batch %d outside 1..%d", o.max_batch, MK_MAX_BATCH);
  if (o.kv_page_size < 16 || o.kv_page_size % 16)
    return fail(MK_ERR_INVALID_ARG, "kv_page_size %d must be a positive multiple of 16",
                o.kv_page_size);
  if (o.wait_limit_ns < 0) return fail(MK_ERR_INVALID_ARG, "wait_limit_ns < 0");

  const mk_model_config &c = *cfg;
  const int L = c.n_layers, H = c.hidden, Hq = c.n_q_heads, Hkv = c.n_kv_heads, d = c.head_dim;
  const int F = c.ffn, V = c.vocab, G = Hq / Hkv, P = o.kv_page_size;
  const int NQKV = (Hq + 2 * Hkv) * d;
  const int maxB = o.max_batch;

  int dev = 0, nsm = 0, smem_optin = 0, coop = 0;
  MK_CUDA(cudaGetDevice(&dev));
  MK_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
  MK_CUDA(cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
  MK_CUDA(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev));
  if (!coop) return fail(MK_ERR_UNSUPPORTED, "device lacks cooperative launch");
  const int smem_max = std::min(smem_optin, mk::kMaxSmem);
  int grid = o.num_ctas > 0 ? std::min(o.num_ctas, nsm) : nsm;

  // ---- shared-memory carve-up ------------------------------------------------
  const int Kmax = std::max(H, std::max(Hq * d, F));
  // attention scratch in the staging area: q [G][d] plus either the page's
  // scores [G][tokens per page] and per-head statistics, or the combine's
  // per-chunk (m, l) pairs
  const int max_chunks = (c.max_seq_len + P - 1) / P;
  const int tpp_bound = std::min(16 * P, 16 * mk::row_pitch_bytes(1024) / (4 * d));
  const int att_need = G * d * 4 + std::max(G * tpp_bound + 3 * mk::kMaxGroup,
                                            2 * max_chunks * G + 2 * G) * 4;
  // activation staging: the whole widest input of one sequence, or a
  // 1024-column chunk of every sequence, whichever is larger (<= 64 KB)
  const int chunk_need = 2 * maxB * mk::row_pitch_bytes(std::min(1024, align_up(Kmax, 32)));
  int x_cap = std::min(std::max(2 * mk::row_pitch_bytes(Kmax), chunk_need), 64 * 1024);
  x_cap = std::max(x_cap, att_need);
  int kpmax = 0;
  for (int cand : {1024, 512, 256, 128, 64, 32}) {
    if (2 * maxB * mk::row_pitch_bytes(cand) <= x_cap) {
      kpmax = cand;
      break;
    }
  }
  if (kpmax == 0) x_cap = 2 * maxB * mk::row_pitch_bytes(kpmax = 32);
  auto page_cols = [&](int K) {
    if (K <= kpmax) return K;
    const int n = (K + kpmax - 1) / kpmax;
    return align_up((K + n - 1) / n, 32);
  };
  int kp[4] = {page_cols(H), page_cols(Hq * d), page_cols(F), page_cols(H)};
  int kp_big = std::max(std::max(kp[0], kp[1]), kp[2]);
  int page_bytes = 16 * mk::row_pitch_bytes(kp_big);
  int tpp = (page_bytes / (4 * d)) / P * P;
  if (tpp < P) {
    tpp = P;
    page_bytes = align_up(4 * d * P, 128);
  }
  tpp = std::min(tpp, 16 * P);

  const int off_look = 1024;   // loader lookahead (8 x 48 B)
  const int off_slots = off_look + 512;
  const int off_red = align_up(off_slots + mk::kTaskSlots * 64, 128);
  const int red_bytes = mk::kComputeWarps * 16 * (maxB > 8 ? 16 : 8) * 4;
  const int off_out = align_up(off_red + red_bytes, 128);
  const int out_bytes = align_up(maxB * 16 * mk::kMaxMTiles * 4, 128);
  const int off_x = align_up(off_out + mk::kOutSlots * out_bytes, 128);
  const int off_pages = align_up(off_x + x_cap, 128);
  const int n_pages = std::min(mk::kMaxPages, (smem_max - off_pages) / page_bytes);
  if (n_pages < 2)
    return fail(MK_ERR_UNSUPPORTED, "shape leaves room for %d shared-memory pages (need 2)",
                n_pages);
  const int smem = off_pages + n_pages * page_bytes;

  // ---- task graph ---------------------------------------------------------------
  auto plan = new mk_plan();
  plan->cfg = c;
  plan->dev = dev;
  plan->grid = grid;
  plan->smem = smem;
  plan->max_batch = maxB;
  Params &p = plan->base;
  std::memset(&p, 0, sizeof(p));
  p.L = L; p.H = H; p.Hq = Hq; p.Hkv = Hkv; p.d = d; p.F = F; p.V = V; p.G = G; p.NQKV = NQKV;
  p.eps = c.rms_eps;
  p.qk_norm = c.qk_norm ? 1 : 0;
  p.max_batch = maxB;
  p.page_size = P;
  p.tpp = tpp;
  for (int i = 0; i < 4; ++i) p.kp[i] = kp[i];
  p.x_cap = x_cap;
  p.page_bytes = page_bytes;
  p.n_pages = n_pages;
  p.off_look = off_look;
  p.off_slots = off_slots;
  p.off_red = off_red;
  p.off_out = off_out;
  p.out_bytes = out_bytes;
  p.off_x = off_x;
  p.off_pages = off_pages;
  p.attn_target = grid;
  p.attn_slots = grid + maxB * Hkv;
  p.wait_limit_ns = o.wait_limit_ns;
  p.pf_bytes = o.l2_prefetch_kb > 0 ? 1024u * static_cast<uint32_t>(o.l2_prefetch_kb) : 0u;
  p.pf_distance = o.prefetch_distance > 0 ? o.prefetch_distance : 0;
  p.pf_task_bytes = 1024u * static_cast<uint32_t>(o.prefetch_task_kb > 0 ? o.prefetch_task_kb : 256);
  p.ev_embed = 0;
  p.ev_layer0 = 1;
  p.ev_per_layer = Hkv + 4;
  const int n_events = 1 + L * (Hkv + 4);

  auto rows_opt = [&](int i, int dflt) {
    const int r = o.rows_per_task[i];
    return r > 0 ? std::max(16, r / 16 * 16) : dflt;
  };
  // QKV: tasks never straddle heads (the last task of a head runs its RoPE)
  int nm_qkv = choose_mtiles(NQKV / 16, grid, mk::kMaxMTiles);
  while ((d / 16) % nm_qkv) --nm_qkv;
  int R_qkv = rows_opt(0, 16 * nm_qkv);
  if (R_qkv > d || d % R_qkv) R_qkv = 16;
  const int R_o = std::min(rows_opt(1, 16 * choose_mtiles(H / 16, grid, mk::kMaxMTiles)), 16 * mk::kMaxMTiles);
  const int R_gu = std::min(rows_opt(2, 16 * choose_mtiles(F / 16, grid, mk::kMaxMTiles / 2)),
                            16 * (mk::kMaxMTiles / 2));
  const int R_d = std::min(rows_opt(3, 16 * choose_mtiles(H / 16, grid, mk::kMaxMTiles)), 16 * mk::kMaxMTiles);
  const int R_lm = std::min(rows_opt(4, 16 * choose_mtiles(V / 16, grid, mk::kMaxMTiles)), 16 * mk::kMaxMTiles);

  auto ceil_div = [](int a, int b) { return (a + b - 1) / b; };
  const int n_o = ceil_div(H, R_o), n_gu = ceil_div(F, R_gu), n_down = ceil_div(H, R_d);
  const int n_lm = ceil_div(V, R_lm);
  std::vector<Task> &T = plan->tasks;
  auto push = [&](Task t) { T.push_back(t); };
  auto gemv = [&](uint8_t type, int layer, int row0, int nrows, int nm, uint32_t dep, uint32_t cnt,
                  uint32_t outev) {
    Task t{};
    t.type = type;
    t.n_m = static_cast<uint8_t>(nm);
    t.layer = static_cast<uint16_t>(layer);
    t.row0 = row0;
    t.nrows = nrows;
    t.dep_event = dep;
    t.dep_count = cnt;
    t.out_event = outev;
    return t;
  };

  {
    Task t{};
    t.type = mk::T_EMBED;
    t.dep_event = mk::kNoEvent;
    t.out_event = p.ev_embed;
    push(t);
    plan->ops.push_back({0, 1});
  }
  for (int l = 0; l < L; ++l) {
    const uint32_t dep = l == 0 ? p.ev_embed : mk::ev_down(p, l - 1);
    const uint32_t cnt = l == 0 ? 1 : n_down;
    int b0 = static_cast<int>(T.size());
    const int per_head = d / R_qkv;
    for (int mat = 0; mat < 3; ++mat) {
      const int nh = mat == 0 ? Hq : Hkv;
      for (int hh = 0; hh < nh; ++hh) {
        const int head = mat == 0 ? hh : (mat == 1 ? Hq + hh : Hq + Hkv + hh);
        for (int r0 = 0; r0 < d; r0 += R_qkv) {
          Task t = gemv(mk::T_QKV, l, hh * d + r0, R_qkv, R_qkv / 16, dep, cnt, mk::kNoEvent);
          t.aux = mat;
          t.aux2 = static_cast<uint32_t>(head) | (static_cast<uint32_t>(per_head) << 16);
          push(t);
        }
      }
    }
    plan->ops.push_back({b0, static_cast<int>(T.size())});
    b0 = static_cast<int>(T.size());
    for (int s = 0; s < p.attn_slots; ++s) {
      Task t{};
      t.type = mk::T_ATTN;
      t.layer = static_cast<uint16_t>(l);
      t.dep_event = mk::kNoEvent;  // resolved at run time: attn_ready(l, g)
      t.out_event = mk::ev_o_ready(p, l);
      t.aux = s;
      push(t);
    }
    plan->ops.push_back({b0, static_cast<int>(T.size())});
    b0 = static_cast<int>(T.size());
    for (int r0 = 0; r0 < H; r0 += R_o) {
      const int nr = std::min(R_o, H - r0);
      push(gemv(mk::T_OPROJ, l, r0, nr, ceil_div(nr, 16), mk::ev_o_ready(p, l), p.attn_slots,
                mk::ev_oproj(p, l)));
    }
    plan->ops.push_back({b0, static_cast<int>(T.size())});
    b0 = static_cast<int>(T.size());
    for (int r0 = 0; r0 < F; r0 += R_gu) {
      const int nr = std::min(R_gu, F - r0);
      push(gemv(mk::T_GATEUP, l, r0, nr, 2 * ceil_div(nr, 16), mk::ev_oproj(p, l), n_o,
                mk::ev_gateup(p, l)));
    }
    plan->ops.push_back({b0, static_cast<int>(T.size())});
    b0 = static_cast<int>(T.size());
    for (int r0 = 0; r0 < H; r0 += R_d) {
      const int nr = std::min(R_d, H - r0);
      push(gemv(mk::T_DOWN, l, r0, nr, ceil_div(nr, 16), mk::ev_gateup(p, l), n_gu,
                mk::ev_down(p, l)));
    }
    plan->ops.push_back({b0, static_cast<int>(T.size())});
  }
  {
    const int b0 = static_cast<int>(T.size());
    for (int r0 = 0; r0 < V; r0 += R_lm) {
      const int nr = std::min(R_lm, V - r0);
      push(gemv(mk::T_LMHEAD, L - 1, r0, nr, ceil_div(nr, 16), mk::ev_down(p, L - 1), n_down,
                mk::kNoEvent));
    }
    plan->ops.push_back({b0, static_cast<int>(T.size())});
  }
  p.n_lm_tasks = n_lm;
  p.n_tasks = static_cast<int>(T.size());
  if (o.debug_unsatisfiable_dep) T[1].dep_count += 1;  // first QKV task

  // ---- device allocations ---------------------------------------------------------
  auto cleanup_fail = [&](int code) {
    mk_plan_destroy(plan);
    return code;
  };
  cudaError_t e;
  e = cudaMalloc(&plan->d_tasks, T.size() * sizeof(Task));
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "cudaMalloc tasks: %s", cudaGetErrorString(e)));
  e = cudaMemcpy(plan->d_tasks, T.data(), T.size() * sizeof(Task), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "upload tasks: %s", cudaGetErrorString(e)));

  std::vector<mk::LayerW> lw(L);
  for (int l = 0; l < L; ++l) {
    const mk_layer_weights &s = w->layers[l];
    auto bf = [](const void *q) { return static_cast<const __nv_bfloat16 *>(q); };
    lw[l] = {bf(s.attn_norm), bf(s.wq), bf(s.wk), bf(s.wv), bf(s.q_norm), bf(s.k_norm),
             bf(s.wo), bf(s.mlp_norm), bf(s.w_gate), bf(s.w_up), bf(s.w_down)};
  }
  e = cudaMalloc(&plan->d_layers, L * sizeof(mk::LayerW));
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "cudaMalloc layers: %s", cudaGetErrorString(e)));
  e = cudaMemcpy(plan->d_layers, lw.data(), L * sizeof(mk::LayerW), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "upload layers: %s", cudaGetErrorString(e)));

  // RoPE: pair i at position t turns by t * theta^(-2i/d), computed in double
  const int half = d / 2;
  std::vector<float2> cs(static_cast<size_t>(c.max_seq_len) * half);
  for (int t = 0; t < c.max_seq_len; ++t)
    for (int i = 0; i < half; ++i) {
      const double ang = static_cast<double>(t) *
                         std::pow(static_cast<double>(c.rope_theta), -2.0 * i / d);
      cs[static_cast<size_t>(t) * half + i] = make_float2(static_cast<float>(std::cos(ang)),
                                                          static_cast<float>(std::sin(ang)));
    }
  e = cudaMalloc(&plan->d_rope, cs.size() * sizeof(float2));
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "cudaMalloc rope: %s", cudaGetErrorString(e)));
  e = cudaMemcpy(plan->d_rope, cs.data(), cs.size() * sizeof(float2), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "upload rope: %s", cudaGetErrorString(e)));

  // workspace: activations and partials, 256-byte aligned pieces
  size_t off = 0;
  auto carve = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, static_cast<size_t>(256));
    return at;
  };
  const size_t o_h = carve(sizeof(float) * maxB * H);
  const size_t o_qkv = carve(sizeof(float) * maxB * NQKV);
  const size_t o_qrot = carve(sizeof(float) * maxB * Hq * d);
  const size_t o_part = carve(sizeof(float) * static_cast<size_t>(p.attn_slots) * G * (d + 4));
  const size_t o_o = carve(sizeof(float) * maxB * Hq * d);
  const size_t o_u = carve(sizeof(float) * maxB * F);
  const size_t o_arg = carve(sizeof(unsigned long long) * maxB);
  const size_t ws_bytes = off;
  e = cudaMalloc(&plan->d_ws, ws_bytes);
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "cudaMalloc workspace: %s", cudaGetErrorString(e)));
  e = cudaMemset(plan->d_ws, 0, ws_bytes);
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "memset workspace: %s", cudaGetErrorString(e)));
  char *ws = static_cast<char *>(plan->d_ws);
  p.h = reinterpret_cast<float *>(ws + o_h);
  p.qkv = reinterpret_cast<float *>(ws + o_qkv);
  p.qrot = reinterpret_cast<float *>(ws + o_qrot);
  p.attn_part = reinterpret_cast<float *>(ws + o_part);
  p.o = reinterpret_cast<float *>(ws + o_o);
  p.u = reinterpret_cast<float *>(ws + o_u);
  p.argmax = reinterpret_cast<unsigned long long *>(ws + o_arg);

  // counters: fixed words, events, per-head QKV counters, per-(b, g) chunk counters
  const size_t head_words = static_cast<size_t>(L) * (Hq + 2 * Hkv);
  const size_t comb_words = static_cast<size_t>(maxB) * Hkv;
  plan->sync_words = mk::S_EVENTS + n_events + head_words + comb_words;
  e = cudaMalloc(&plan->d_sync, plan->sync_words * sizeof(uint32_t));
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "cudaMalloc counters: %s", cudaGetErrorString(e)));
  e = cudaMemset(plan->d_sync, 0, plan->sync_words * sizeof(uint32_t));
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "memset counters: %s", cudaGetErrorString(e)));
  p.sync = plan->d_sync;
  p.head_ctr = plan->d_sync + mk::S_EVENTS + n_events;
  p.comb_ctr = p.head_ctr + head_words;

  p.tasks = static_cast<const Task *>(plan->d_tasks);
  p.layers = static_cast<const mk::LayerW *>(plan->d_layers);
  p.embed = static_cast<const __nv_bfloat16 *>(w->embed);
  p.final_norm = static_cast<const __nv_bfloat16 *>(w->final_norm);
  p.lm_head = static_cast<const __nv_bfloat16 *>(w->lm_head);
  p.rope_cs = static_cast<const float2 *>(plan->d_rope);

  e = cudaMalloc(&plan->d_host_ids, 3 * sizeof(int32_t) * MK_MAX_BATCH);
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "cudaMalloc staging: %s", cudaGetErrorString(e)));
  plan->d_host_pos = plan->d_host_ids + MK_MAX_BATCH;
  plan->d_host_out = plan->d_host_pos + MK_MAX_BATCH;

  e = mk::configure_kernel(smem);
  if (e != cudaSuccess) return cleanup_fail(fail(MK_ERR_CUDA, "kernel attribute: %s", cudaGetErrorString(e)));

  // ---- facts ------------------------------------------------------------------
  mk_plan_info_t &I = plan->info;
  I.num_ctas = grid;
  I.threads_per_cta = mk::kThreads;
  I.smem_bytes = smem;
  I.n_pages = n_pages;
  I.page_bytes = page_bytes;
  I.n_tasks = p.n_tasks;
  I.n_events = n_events;
  I.attn_slots = p.attn_slots;
  I.tokens_per_smem_page = tpp;
  I.rows_per_task[0] = R_qkv;
  I.rows_per_task[1] = R_o;
  I.rows_per_task[2] = R_gu;
  I.rows_per_task[3] = R_d;
  I.rows_per_task[4] = R_lm;
  for (int i = 0; i < 4; ++i) I.page_cols[i] = kp[i];
  I.weight_bytes = 2LL * L *
                       (static_cast<long long>(NQKV) * H + static_cast<long long>(H) * Hq * d +
                        3LL * F * H) +
                   2LL * V * H;
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

int mk_decode_step_ex(mk_plan *plan, const mk_step_args *a, void *stream) {
  g_err.clear();
  if (plan == nullptr || a == nullptr) return fail(MK_ERR_INVALID_ARG, "plan or args is NULL");
  if (a->batch < 1 || a->batch > plan->max_batch)
    return fail(MK_ERR_INVALID_ARG, "batch %d outside 1..max_batch %d", a->batch, plan->max_batch);
  if (a->d_ids == nullptr || a->d_pos == nullptr || a->d_out_ids == nullptr)
    return fail(MK_ERR_INVALID_ARG, "d_ids, d_pos and d_out_ids must not be NULL");
  if (a->mode != MK_MODE_MEGAKERNEL && a->mode != MK_MODE_PER_OP)
    return fail(MK_ERR_INVALID_ARG, "unknown mode %d", a->mode);
  int rc = validate_kv(plan, a->kv);
  if (rc) return rc;

  Params p = plan->base;
  plan->epoch += 1;
  p.epoch = plan->epoch;
  p.batch = a->batch;
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
  if (a->mode == MK_MODE_MEGAKERNEL) {
    p.task_begin = 0;
    p.task_end = p.n_tasks;
    cudaError_t e = mk::launch_step(p, plan->grid, plan->smem, true, s);
    if (e != cudaSuccess) {
      plan->epoch -= 1;
      return fail(MK_ERR_CUDA, "megakernel launch: %s", cudaGetErrorString(e));
    }
  } else {
    for (const Range &r : plan->ops) {
      p.task_begin = r.begin;
      p.task_end = r.end;
      const int grid = std::min(plan->grid, r.end - r.begin);
      cudaError_t e = mk::launch_step(p, grid, plan->smem, false, s);
      if (e != cudaSuccess) return fail(MK_ERR_CUDA, "per-op launch: %s", cudaGetErrorString(e));
    }
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

void mk_plan_destroy(mk_plan *plan) {
  if (plan == nullptr) return;
  cudaDeviceSynchronize();
  cudaFree(plan->d_tasks);
  cudaFree(plan->d_layers);
  cudaFree(plan->d_rope);
  cudaFree(plan->d_ws);
  cudaFree(plan->d_sync);
  cudaFree(plan->d_host_ids);
  cudaFree(plan->d_host_logits);
  delete plan;
}

}  // extern "C"
