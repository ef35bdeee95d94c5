// A decode step that allocates no device memory.
//
// Who needs it: callers that must not call cudaMalloc -- code running where
// the device allocator is off limits (inside a host that owns every device
// allocation through its own pool, a memory-capped sandbox, or a callback
// that may not allocate).  They still own and pass the weights, the KV cache
// and the step's inputs and outputs; everything the step needs besides those
// (task array, weight-pointer table, RoPE table, activations, counters) lives
// in one file-scope __device__ array of MK_NOALLOC_SCRATCH_BYTES that every
// GPU which loads this library keeps until the process exits.
//
// The step runs the same persistent kernel as mk_decode_step(); only the
// place its scratch comes from differs.  Each call rebuilds the task array on
// the host, uploads it and the tables into the array, zeroes the counters and
// the argmax slots, launches, synchronizes and returns the device status.
// Calls share the one array, so calls that overlap on the GPU (two streams,
// two threads) race and must not be issued.  The first call on a device looks
// up the array's device address (cudaGetSymbolAddress) and sets the kernel's
// shared-memory limit; make that first call before any stream capture.

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "mk_internal.h"

namespace {

// The scratch.  In host code `g_noalloc_scratch` is only a host-side stand-in
// for the symbol: its device address comes from cudaGetSymbolAddress.
__device__ __align__(256) unsigned char g_noalloc_scratch[MK_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};
int g_scratch_smem[kMaxDevices] = {};

int nfail(int code, const char *msg) {
  mk::set_last_error(msg);
  return code;
}

inline int align_up_i(int x, int a) { return (x + a - 1) / a * a; }
inline size_t align_up_z(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int pick_mtiles(int tiles, int nsm, int cap) {
  return std::max(1, std::min(cap, tiles / (16 * nsm)));
}

}  // namespace

extern "C" MK_API int mk_decode_step_noalloc(const mk_model_config *cfg, const mk_weights *w,
                                             int kv_page_size, const mk_step_args *a,
                                             void *stream) {
  using mk::Params;
  using mk::Task;
  mk::set_last_error("");
  if (cfg == nullptr || w == nullptr || w->layers == nullptr || a == nullptr || a->kv == nullptr)
    return nfail(MK_ERR_INVALID_ARG, "cfg, weights, weights->layers, args and args->kv must be set");
  const mk_model_config &c = *cfg;
  const int L = c.n_layers, H = c.hidden, Hq = c.n_q_heads, Hkv = c.n_kv_heads, d = c.head_dim;
  const int F = c.ffn, V = c.vocab, P = kv_page_size, B = a->batch;
  if (L < 1 || L > MK_MAX_LAYERS || H <= 0 || Hq <= 0 || Hkv <= 0 || F <= 0 || V <= 0 ||
      c.max_seq_len <= 0 || Hq % Hkv || Hq / Hkv > mk::kMaxGroup ||
      (d != 32 && d != 64 && d != 128) || H % 8 || F % 8 || (Hq * d) % 8)
    return nfail(MK_ERR_UNSUPPORTED, "model shape not supported (see mk_model_config)");
  if (P < 16 || P % 16) return nfail(MK_ERR_INVALID_ARG, "kv_page_size must be a multiple of 16");
  if (B < 1 || B > MK_MAX_BATCH) return nfail(MK_ERR_INVALID_ARG, "batch outside 1..16");
  if (a->mode != MK_MODE_MEGAKERNEL)
    return nfail(MK_ERR_INVALID_ARG, "only MK_MODE_MEGAKERNEL is available without allocation");
  if (a->d_ids == nullptr || a->d_pos == nullptr || a->d_out_ids == nullptr ||
      a->kv->k_pages == nullptr || a->kv->v_pages == nullptr || a->kv->block_table == nullptr ||
      a->kv->num_pages < 1 || a->kv->max_pages_per_seq < 1)
    return nfail(MK_ERR_INVALID_ARG, "a step input, output or KV-cache pointer is NULL");
  const void *top[] = {w->embed, w->final_norm, w->lm_head, a->kv->block_table};
  for (const void *q : top)
    if (q == nullptr || !aligned16(q)) return nfail(MK_ERR_INVALID_ARG, "NULL or unaligned pointer");
  for (int l = 0; l < L; ++l) {
    const mk_layer_weights &s = w->layers[l];
    const void *ps[] = {s.attn_norm, s.wq, s.wk, s.wv, s.wo, s.mlp_norm, s.w_gate, s.w_up,
                        s.w_down, a->kv->k_pages[l], a->kv->v_pages[l]};
    for (const void *q : ps)
      if (q == nullptr || !aligned16(q))
        return nfail(MK_ERR_INVALID_ARG, "NULL or unaligned weight / KV pointer");
    if (c.qk_norm && (s.q_norm == nullptr || s.k_norm == nullptr))
      return nfail(MK_ERR_INVALID_ARG, "q_norm/k_norm NULL with qk_norm on");
  }

  int dev = 0, nsm = 0, smem_optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return nfail(MK_ERR_CUDA, "cudaGetDevice failed");
  if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
          cudaSuccess)
    return nfail(MK_ERR_CUDA, "device attribute query failed");
  const int grid = nsm, G = Hq / Hkv, NQKV = (Hq + 2 * Hkv) * d, maxB = B;

  // ---- shared-memory carve-up (same rules as a plan built for max_batch = B)
  const int Kmax = std::max(H, std::max(Hq * d, F));
  // attention scratch in the staging area: q [G][d] plus either the page's
  // scores [G][tokens per page] and per-head statistics, or the combine's
  // per-chunk (m, l) pairs
  const int max_chunks = (c.max_seq_len + P - 1) / P;
  const int tpp_bound = std::min(16 * P, 16 * mk::row_pitch_bytes(1024) / (4 * d));
  const int att_need = G * d * 4 + std::max(G * tpp_bound + 3 * mk::kMaxGroup,
                                            2 * max_chunks * G + 2 * G) * 4;
  const int chunk_need = 2 * maxB * mk::row_pitch_bytes(std::min(1024, align_up_i(Kmax, 32)));
  int x_cap = std::min(std::max(2 * mk::row_pitch_bytes(Kmax), chunk_need), 64 * 1024);
  x_cap = std::max(x_cap, att_need);
  int kpmax = 0;
  for (int cand : {1024, 512, 256, 128, 64, 32})
    if (2 * maxB * mk::row_pitch_bytes(cand) <= x_cap) {
      kpmax = cand;
      break;
    }
  if (kpmax == 0) x_cap = 2 * maxB * mk::row_pitch_bytes(kpmax = 32);
  auto page_cols = [&](int K) {
    if (K <= kpmax) return K;
    const int n = (K + kpmax - 1) / kpmax;
    return align_up_i((K + n - 1) / n, 32);
  };
  const int kp[4] = {page_cols(H), page_cols(Hq * d), page_cols(F), page_cols(H)};
  int page_bytes = 16 * mk::row_pitch_bytes(std::max(std::max(kp[0], kp[1]), kp[2]));
  int tpp = (page_bytes / (4 * d)) / P * P;
  if (tpp < P) {
    tpp = P;
    page_bytes = align_up_i(4 * d * P, 128);
  }
  tpp = std::min(tpp, 16 * P);
  const int smem_max = std::min(smem_optin, mk::kMaxSmem);
  const int off_look = 1024;   // loader lookahead (8 x 48 B)
  const int off_slots = off_look + 512;
  const int off_red = align_up_i(off_slots + mk::kTaskSlots * 64, 128);
  const int off_out = align_up_i(off_red + mk::kComputeWarps * 16 * (maxB > 8 ? 16 : 8) * 4, 128);
  const int out_bytes = align_up_i(maxB * 16 * mk::kMaxMTiles * 4, 128);
  const int off_x = align_up_i(off_out + mk::kOutSlots * out_bytes, 128);
  const int off_pages = align_up_i(off_x + x_cap, 128);
  const int n_pages = std::min(mk::kMaxPages, (smem_max - off_pages) / page_bytes);
  if (n_pages < 2) return nfail(MK_ERR_UNSUPPORTED, "shape leaves no room for the page ring");
  const int smem = off_pages + n_pages * page_bytes;

  Params p;
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
  p.wait_limit_ns = 2000000000LL;
  p.pf_bytes = 0u;
  p.pf_distance = 0;
  p.pf_task_bytes = 256u * 1024u;
  p.ev_embed = 0;
  p.ev_layer0 = 1;
  p.ev_per_layer = Hkv + 4;
  const int n_events = 1 + L * (Hkv + 4);

  // ---- task graph (the default tiling of a plan) --------------------------
  int nm_qkv = pick_mtiles(NQKV / 16, grid, mk::kMaxMTiles);
  while ((d / 16) % nm_qkv) --nm_qkv;
  const int R_qkv = 16 * nm_qkv;
  const int R_o = 16 * pick_mtiles(H / 16, grid, mk::kMaxMTiles);
  const int R_gu = 16 * pick_mtiles(F / 16, grid, mk::kMaxMTiles / 2);
  const int R_d = 16 * pick_mtiles(H / 16, grid, mk::kMaxMTiles);
  const int R_lm = 16 * pick_mtiles(V / 16, grid, mk::kMaxMTiles);
  auto cdiv = [](int x, int y) { return (x + y - 1) / y; };
  const int n_o = cdiv(H, R_o), n_gu = cdiv(F, R_gu), n_down = cdiv(H, R_d), n_lm = cdiv(V, R_lm);
  std::vector<Task> T;
  auto gemv = [&](uint8_t type, int layer, int row0, int nrows, int nm, uint32_t dep,
                  uint32_t cnt, uint32_t outev) {
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
    T.push_back(t);
  }
  for (int l = 0; l < L; ++l) {
    const uint32_t dep = l == 0 ? p.ev_embed : mk::ev_down(p, l - 1);
    const uint32_t cnt = l == 0 ? 1 : n_down;
    for (int mat = 0; mat < 3; ++mat) {
      const int nh = mat == 0 ? Hq : Hkv;
      for (int hh = 0; hh < nh; ++hh) {
        const int head = mat == 0 ? hh : (mat == 1 ? Hq + hh : Hq + Hkv + hh);
        for (int r0 = 0; r0 < d; r0 += R_qkv) {
          Task t = gemv(mk::T_QKV, l, hh * d + r0, R_qkv, R_qkv / 16, dep, cnt, mk::kNoEvent);
          t.aux = mat;
          t.aux2 = static_cast<uint32_t>(head) | (static_cast<uint32_t>(d / R_qkv) << 16);
          T.push_back(t);
        }
      }
    }
    for (int s = 0; s < p.attn_slots; ++s) {
      Task t{};
      t.type = mk::T_ATTN;
      t.layer = static_cast<uint16_t>(l);
      t.dep_event = mk::kNoEvent;
      t.out_event = mk::ev_o_ready(p, l);
      t.aux = s;
      T.push_back(t);
    }
    for (int r0 = 0; r0 < H; r0 += R_o) {
      const int nr = std::min(R_o, H - r0);
      T.push_back(gemv(mk::T_OPROJ, l, r0, nr, cdiv(nr, 16), mk::ev_o_ready(p, l), p.attn_slots,
                       mk::ev_oproj(p, l)));
    }
    for (int r0 = 0; r0 < F; r0 += R_gu) {
      const int nr = std::min(R_gu, F - r0);
      T.push_back(gemv(mk::T_GATEUP, l, r0, nr, 2 * cdiv(nr, 16), mk::ev_oproj(p, l), n_o,
                       mk::ev_gateup(p, l)));
    }
    for (int r0 = 0; r0 < H; r0 += R_d) {
      const int nr = std::min(R_d, H - r0);
      T.push_back(gemv(mk::T_DOWN, l, r0, nr, cdiv(nr, 16), mk::ev_gateup(p, l), n_gu,
                       mk::ev_down(p, l)));
    }
  }
  for (int r0 = 0; r0 < V; r0 += R_lm) {
    const int nr = std::min(R_lm, V - r0);
    T.push_back(gemv(mk::T_LMHEAD, L - 1, r0, nr, cdiv(nr, 16), mk::ev_down(p, L - 1), n_down,
                     mk::kNoEvent));
  }
  p.n_lm_tasks = n_lm;
  p.n_tasks = static_cast<int>(T.size());

  std::vector<mk::LayerW> lw(L);
  for (int l = 0; l < L; ++l) {
    const mk_layer_weights &s = w->layers[l];
    auto bf = [](const void *q) { return static_cast<const __nv_bfloat16 *>(q); };
    lw[l] = {bf(s.attn_norm), bf(s.wq), bf(s.wk), bf(s.wv), bf(s.q_norm), bf(s.k_norm),
             bf(s.wo), bf(s.mlp_norm), bf(s.w_gate), bf(s.w_up), bf(s.w_down)};
  }
  const int half = d / 2;
  std::vector<float2> cs(static_cast<size_t>(c.max_seq_len) * half);
  for (int t = 0; t < c.max_seq_len; ++t)
    for (int i = 0; i < half; ++i) {
      const double ang =
          static_cast<double>(t) * std::pow(static_cast<double>(c.rope_theta), -2.0 * i / d);
      cs[static_cast<size_t>(t) * half + i] =
          make_float2(static_cast<float>(std::cos(ang)), static_cast<float>(std::sin(ang)));
    }

  // ---- layout inside the static array -------------------------------------
  size_t off = 0;
  auto carve = [&](size_t bytes) {
    const size_t at = off;
    off = align_up_z(off + bytes, 256);
    return at;
  };
  const size_t o_tasks = carve(T.size() * sizeof(Task));
  const size_t o_layers = carve(L * sizeof(mk::LayerW));
  const size_t o_rope = carve(cs.size() * sizeof(float2));
  const size_t o_h = carve(sizeof(float) * maxB * H);
  const size_t o_qkv = carve(sizeof(float) * maxB * NQKV);
  const size_t o_qrot = carve(sizeof(float) * maxB * Hq * d);
  const size_t o_part = carve(sizeof(float) * static_cast<size_t>(p.attn_slots) * G * (d + 4));
  const size_t o_o = carve(sizeof(float) * maxB * Hq * d);
  const size_t o_u = carve(sizeof(float) * maxB * F);
  const size_t o_arg = carve(sizeof(unsigned long long) * maxB);
  const size_t head_words = static_cast<size_t>(L) * (Hq + 2 * Hkv);
  const size_t sync_words = mk::S_EVENTS + n_events + head_words + static_cast<size_t>(maxB) * Hkv;
  const size_t o_sync = carve(sync_words * sizeof(uint32_t));
  if (off > MK_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "this model/batch/max_seq_len needs %zu bytes of scratch; the no-allocation entry "
             "point has %u (MK_NOALLOC_SCRATCH_BYTES)",
             off, static_cast<unsigned>(MK_NOALLOC_SCRATCH_BYTES));
    return nfail(MK_ERR_UNSUPPORTED, msg);
  }

  // ---- once per device: the array's device address, the kernel's smem cap
  char *base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
      void *ptr = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
      if (e != cudaSuccess || ptr == nullptr)
        return nfail(MK_ERR_CUDA, "cudaGetSymbolAddress of the scratch array failed");
      g_scratch_addr[dev] = ptr;
    }
    if (g_scratch_smem[dev] < smem) {
      if (mk::configure_kernel(smem) != cudaSuccess)
        return nfail(MK_ERR_CUDA, "setting the kernel's shared-memory limit failed");
      g_scratch_smem[dev] = smem;
    }
    base = static_cast<char *>(g_scratch_addr[dev]);
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(base + o_tasks, T.data(), T.size() * sizeof(Task), cudaMemcpyHostToDevice,
                      s) != cudaSuccess ||
      cudaMemcpyAsync(base + o_layers, lw.data(), L * sizeof(mk::LayerW), cudaMemcpyHostToDevice,
                      s) != cudaSuccess ||
      cudaMemcpyAsync(base + o_rope, cs.data(), cs.size() * sizeof(float2),
                      cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemsetAsync(base + o_arg, 0, sizeof(unsigned long long) * maxB, s) != cudaSuccess ||
      cudaMemsetAsync(base + o_sync, 0, sync_words * sizeof(uint32_t), s) != cudaSuccess)
    return nfail(MK_ERR_CUDA, "uploading the step's tables into the scratch array failed");

  p.tasks = reinterpret_cast<const Task *>(base + o_tasks);
  p.layers = reinterpret_cast<const mk::LayerW *>(base + o_layers);
  p.rope_cs = reinterpret_cast<const float2 *>(base + o_rope);
  p.h = reinterpret_cast<float *>(base + o_h);
  p.qkv = reinterpret_cast<float *>(base + o_qkv);
  p.qrot = reinterpret_cast<float *>(base + o_qrot);
  p.attn_part = reinterpret_cast<float *>(base + o_part);
  p.o = reinterpret_cast<float *>(base + o_o);
  p.u = reinterpret_cast<float *>(base + o_u);
  p.argmax = reinterpret_cast<unsigned long long *>(base + o_arg);
  p.sync = reinterpret_cast<uint32_t *>(base + o_sync);
  p.head_ctr = p.sync + mk::S_EVENTS + n_events;
  p.comb_ctr = p.head_ctr + head_words;
  p.embed = static_cast<const __nv_bfloat16 *>(w->embed);
  p.final_norm = static_cast<const __nv_bfloat16 *>(w->final_norm);
  p.lm_head = static_cast<const __nv_bfloat16 *>(w->lm_head);

  p.epoch = 1;  // counters were just zeroed
  p.batch = B;
  p.mode = MK_MODE_MEGAKERNEL;
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
  p.max_pos = static_cast<int>(
      std::min<long long>(c.max_seq_len, static_cast<long long>(a->kv->max_pages_per_seq) * P));
  for (int l = 0; l < L; ++l) {
    p.k_pages[l] = static_cast<__nv_bfloat16 *>(a->kv->k_pages[l]);
    p.v_pages[l] = static_cast<__nv_bfloat16 *>(a->kv->v_pages[l]);
  }
  p.task_begin = 0;
  p.task_end = p.n_tasks;
  if (mk::launch_step(p, grid, smem, true, s) != cudaSuccess)
    return nfail(MK_ERR_CUDA, "megakernel launch failed");
  uint32_t status = 0;
  if (cudaMemcpyAsync(&status, p.sync + mk::S_STATUS, sizeof(status), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return nfail(MK_ERR_CUDA, "reading the step's status failed");
  return static_cast<int32_t>(status);
}
