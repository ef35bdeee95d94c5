// Plan layout: the host-side half of a decode plan that does not depend on
// where its memory comes from.  Both entry points (mk_plan_create_ex, which
// allocates, and mk_decode_step_noalloc, which uses a static array) build the
// same layout here and only bind it to different addresses.
//
// The layout fixes
//   - the shared-memory carve-up of the persistent kernel (task slots,
//     reduction scratch, output buffers, activation staging, weight-page ring);
//   - the task graph: every operator of every layer tiled into 32-byte task
//     descriptors, each naming the event it waits on and how many
//     completions that event needs per step (the TaskDesc /
//     Event{trigger_count, required_count} pair of the MPK write-up, "2.1
//     Mega-Kernel执行模型");
//   - the byte layout of the fp32 workspace and of the counter words;
//   - the RoPE cos/sin table.

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>

#include "mk_internal.h"

namespace mk {

namespace {

int lfail(std::string &err, int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  err = buf;
  return code;
}

inline int align_up_i(int x, int a) { return (x + a - 1) / a * a; }
inline size_t align_up_z(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// Row tiles per task: small enough that every CTA gets ~16 tasks of an
// operator, so the dynamic queue evens out the operator's tail across SMs.
int choose_mtiles(int tiles, int nsm, int cap) { return std::max(1, std::min(cap, tiles / (16 * nsm))); }

}  // namespace

int validate_config(const mk_model_config &c, std::string &err) {
  if (c.n_layers < 1 || c.n_layers > MK_MAX_LAYERS)
    return lfail(err, MK_ERR_UNSUPPORTED, "n_layers %d outside 1..%d", c.n_layers, MK_MAX_LAYERS);
  if (c.hidden <= 0 || c.n_q_heads <= 0 || c.n_kv_heads <= 0 || c.head_dim <= 0 || c.ffn <= 0 ||
      c.vocab <= 0 || c.max_seq_len <= 0)
    return lfail(err, MK_ERR_INVALID_ARG, "model dimensions must be positive");
  if (!(c.rms_eps >= 0.f) || !(c.rope_theta > 0.f))
    return lfail(err, MK_ERR_INVALID_ARG, "rms_eps must be >= 0 and rope_theta > 0");
  const int d = c.head_dim;
  if (d != 32 && d != 64 && d != 128)
    return lfail(err, MK_ERR_UNSUPPORTED, "head_dim %d: supported 32, 64, 128", d);
  if (c.n_q_heads % c.n_kv_heads != 0)
    return lfail(err, MK_ERR_INVALID_ARG, "n_q_heads %d not a multiple of n_kv_heads %d",
                 c.n_q_heads, c.n_kv_heads);
  if (c.n_q_heads / c.n_kv_heads > kMaxGroup)
    return lfail(err, MK_ERR_UNSUPPORTED, "more than %d query heads per KV head", kMaxGroup);
  if (c.hidden % 8 || c.ffn % 8 || (c.n_q_heads * d) % 8)
    return lfail(err, MK_ERR_UNSUPPORTED, "hidden, ffn and n_q_heads*head_dim must be multiples of 8");
  if (c.n_q_heads + 2 * c.n_kv_heads > 0xffff) return lfail(err, MK_ERR_UNSUPPORTED, "too many heads");
  return MK_OK;
}

int build_layout(const mk_model_config &c, const LayoutOptions &o, int nsm, int smem_optin,
                 Layout &out, std::string &err) {
  const int L = c.n_layers, H = c.hidden, Hq = c.n_q_heads, Hkv = c.n_kv_heads, d = c.head_dim;
  const int F = c.ffn, V = c.vocab, G = Hq / Hkv, P = o.page_size;
  const int NQKV = (Hq + 2 * Hkv) * d;
  const int maxB = o.max_batch;
  if (maxB < 1 || maxB > MK_MAX_BATCH)
    return lfail(err, MK_ERR_INVALID_ARG, "max_batch %d outside 1..%d", maxB, MK_MAX_BATCH);
  if (P < 16 || P % 16)
    return lfail(err, MK_ERR_INVALID_ARG, "kv_page_size %d must be a positive multiple of 16", P);
  const int colcap = o.max_page_cols > 0 ? o.max_page_cols : kMaxPageCols;
  if (colcap < 32 || colcap > kMaxPageCols || colcap % 32)
    return lfail(err, MK_ERR_INVALID_ARG, "max_page_cols %d: 32..%d, a multiple of 32", colcap,
                 kMaxPageCols);
  const int grid = o.num_ctas > 0 ? std::min(o.num_ctas, nsm) : nsm;
  const int smem_max = std::min(smem_optin, kMaxSmem);
  const int mt_cap = max_mtiles_for(maxB);

  // ---- rows per task ----------------------------------------------------------
  auto rows_opt = [&](int i, int dflt) {
    const int r = o.rows_per_task[i];
    return r > 0 ? std::max(16, r / 16 * 16) : dflt;
  };
  // When the inputs of every sequence do not fit the staging area whole, each
  // task restages its input chunk by chunk: then every task takes as many
  // row tiles as its accumulators allow, so a staged chunk serves more rows.
  const int kx_limit = std::max(H, Hq * d);
  const bool chunked = maxB * x_row_bytes(kx_limit) > kXWholeMax;
  auto pick = [&](int tiles, int cap) { return chunked ? cap : choose_mtiles(tiles, grid, cap); };
  // QKV tasks never straddle heads (a head's rows belong to one KV group)
  int nm_qkv = pick(NQKV / 16, mt_cap);
  while ((d / 16) % nm_qkv) --nm_qkv;
  int R_qkv = rows_opt(0, 16 * nm_qkv);
  if (R_qkv > d || d % R_qkv || R_qkv > 16 * mt_cap) R_qkv = 16;
  const int R_o = std::min(rows_opt(1, 16 * pick(H / 16, mt_cap)), 16 * mt_cap);
  const int gu_cap = std::max(1, mt_cap / 2);   // gate and up tiles share a task
  const int R_gu = std::min(rows_opt(2, 16 * pick(F / 16, gu_cap)), 16 * gu_cap);
  // a split down projection has a third or less of the columns per task:
  // two row tiles per task keep its per-task costs (dependency check,
  // restaging at each part) small against its pages
  const bool ffn_split = F > kx_limit;
  const int nm_d = std::max(pick(H / 16, mt_cap), ffn_split ? std::min(2, mt_cap) : 1);
  const int R_d = std::min(rows_opt(3, 16 * nm_d), 16 * mt_cap);
  const int R_lm = std::min(rows_opt(4, 16 * pick(V / 16, mt_cap)), 16 * mt_cap);

  // ---- split-K of the down projection --------------------------------------------
  // Parts of at most kx_limit columns (the widest other input), so the down
  // projection's input stages like every other operator's.  A part's columns
  // are whole gate/up tasks' rows, so each part waits only on the gate/up
  // tasks that produce its slice of u.
  int n_ksplit = F > kx_limit ? cdiv(F, kx_limit) : 1;
  int kchunk_ffn = F;
  if (n_ksplit > 1) {
    const int unit = (R_gu % 32 == 0) ? R_gu : 2 * R_gu;   // multiple of 32 and of R_gu
    kchunk_ffn = align_up_i(cdiv(F, n_ksplit), unit);
    n_ksplit = cdiv(F, kchunk_ffn);
    if (n_ksplit < 2) {
      n_ksplit = 1;
      kchunk_ffn = F;
    }
  }
  if (n_ksplit > 255) return lfail(err, MK_ERR_UNSUPPORTED, "ffn too wide for the split-K layout");

  // ---- split-K of the O projection (option) ---------------------------------------------
  // Two parts of whole KV groups: a part waits only for the attention of its
  // groups, so the first part can stream while later groups still attend.
  // Only where a part is at least 1024 columns wide (narrower parts make
  // tasks too small to pay for their staging).  Off by default: on the 8B
  // shape every group's attention ends within a few microseconds of the
  // others, so the overlap does not pay for the extra tasks.
  int o_groups = (o.o_split && Hkv >= 2) ? cdiv(Hkv, 2) : Hkv;
  if (o_groups * G * d < 1024) o_groups = Hkv;
  const int n_o_parts = cdiv(Hkv, o_groups);

  // ---- shared memory: activation staging and the weight-page ring ------------------
  // Activation staging holds fp32 rows of every sequence: a whole input when
  // the widest input other than the FFN's fits in kXWholeMax (staged once,
  // reused by the operator's later tasks on this SM), else one page-wide
  // chunk (<= 64 KB).
  const int max_chunks = cdiv(c.max_seq_len, P);
  const int x_whole = maxB * x_row_bytes(kx_limit);
  const int red_bytes = kComputeWarps * 16 * 8 * n_tiles_for(maxB) * 4;
  const int out_stride = 16 * mt_cap;
  const int out_bytes = align_up_i(maxB * out_stride * 4, 128);
  const int off_look = 1024;   // loader lookahead
  const int off_slots = off_look + kLookBytes;
  const int off_red = align_up_i(off_slots + kTaskSlots * kSlotBytes, 128);
  const int off_out = align_up_i(off_red + red_bytes, 128);
  const int off_x = align_up_i(off_out + kOutSlots * out_bytes, 128);

  struct Geom {
    int kp[4], page_bytes, tpp, x_cap, off_pages, n_pages, ring;
  };
  // Geometry for pages of at most `kpmax` columns; false if the staging
  // area cannot hold one page-wide chunk within 64 KB.
  auto geometry = [&](int kpmax, Geom &g) {
    auto page_cols = [&](int K) {
      if (K <= kpmax) return K;
      return align_up_i(cdiv(K, cdiv(K, kpmax)), 32);
    };
    g.kp[K_HID] = page_cols(H);
    g.kp[K_ATT] = page_cols(n_o_parts > 1 ? o_groups * G * d : Hq * d);
    g.kp[K_FFN] = page_cols(kchunk_ffn);
    g.kp[K_LM] = page_cols(H);
    const int kp_big = std::max(std::max(g.kp[0], g.kp[1]), g.kp[2]);
    const int x_chunk = maxB * x_row_bytes(kp_big);
    if (x_chunk > kXWholeMax) return false;
    int x_cap = x_whole <= kXWholeMax ? std::max(x_whole, x_chunk) : x_chunk;
    g.page_bytes = 16 * row_pitch_bytes(kp_big);
    // attention pages hold tpp tokens of K and V (4 d bytes per token)
    int tpp = (g.page_bytes / (4 * d)) / P * P;
    if (tpp < P) {
      tpp = P;
      g.page_bytes = align_up_i(4 * d * P, 128);
    }
    g.tpp = std::min(tpp, 16 * P);
    // attention scratch in the staging area: q [G][d] plus either the page's
    // scores [G][tpp], per-head statistics and the current token's K and V
    // (bf16), or the combine's per-chunk (m, l) pairs
    const int att_need = G * d * 4 + std::max((G * g.tpp + 3 * kMaxGroup) * 4 + 2 * d * 2,
                                              (2 * max_chunks * G + 2 * G) * 4);
    g.x_cap = std::max(x_cap, att_need);
    g.off_pages = align_up_i(off_x + g.x_cap, 1024);
    g.n_pages = std::min(kMaxPages, (smem_max - g.off_pages) / g.page_bytes);
    g.ring = g.n_pages * g.page_bytes;
    return true;
  };
  // The widest pages whose ring (bytes in flight) is within 10% of the
  // largest ring any width gives with at least 3 pages; wider pages mean
  // fewer hand-offs per byte.  Failing 3 pages, the most pages.
  std::vector<Geom> cands;
  for (int cand = colcap; cand >= 32; cand -= (cand > 256 ? 256 : 32)) {
    Geom g{};
    if (geometry(cand, g)) cands.push_back(g);
  }
  int best_ring = 0;
  for (const Geom &g : cands)
    if (g.n_pages >= 3) best_ring = std::max(best_ring, g.ring);
  // (with chunked staging every chunk is restaged per task: the widest pages
  // that leave 3 in flight, whatever the ring size)
  Geom geo{};
  bool have = false;
  for (const Geom &g : cands)
    if (g.n_pages >= 3 && (chunked || 10LL * g.ring >= 9LL * best_ring)) {
      geo = g;
      have = true;
      break;
    }
  if (!have)
    for (const Geom &g : cands)
      if (!have || g.n_pages > geo.n_pages) {
        geo = g;
        have = true;
      }
  if (!have || geo.n_pages < 2)
    return lfail(err, MK_ERR_UNSUPPORTED, "shape leaves room for fewer than 2 shared-memory pages");
  const int smem = geo.off_pages + geo.n_pages * geo.page_bytes;

  // ---- static kernel parameters -----------------------------------------------------
  Params &p = out.p;
  std::memset(&p, 0, sizeof(p));
  p.L = L; p.H = H; p.Hq = Hq; p.Hkv = Hkv; p.d = d; p.F = F; p.V = V; p.G = G; p.NQKV = NQKV;
  p.eps = c.rms_eps;
  p.qk_norm = c.qk_norm ? 1 : 0;
  p.max_batch = maxB;
  p.page_size = P;
  p.tpp = geo.tpp;
  for (int i = 0; i < 4; ++i) p.kp[i] = geo.kp[i];
  p.kchunk[K_FFN] = n_ksplit > 1 ? kchunk_ffn : 0;
  p.x_cap = geo.x_cap;
  p.page_bytes = geo.page_bytes;
  p.n_pages = geo.n_pages;
  p.off_look = off_look;
  p.off_slots = off_slots;
  p.off_red = off_red;
  p.off_out = off_out;
  p.out_bytes = out_bytes;
  p.out_stride = out_stride;
  p.off_x = off_x;
  p.off_pages = geo.off_pages;
  // attention slots: a fixed block per KV group (so each group's completion
  // is a static count), enough for about one chunk per CTA in all plus one
  // partial chunk per sequence
  p.attn_spg = cdiv(grid, Hkv) + maxB;
  p.attn_slots = Hkv * p.attn_spg;
  p.n_o_parts = n_o_parts;
  p.o_groups = o_groups;
  p.kchunk[K_ATT] = n_o_parts > 1 ? o_groups * G * d : 0;
  p.wait_limit_ns = o.wait_limit_ns;
  p.n_ffn_parts = n_ksplit;
  p.ev_embed = 0;
  p.ev_layer0 = 1;
  // attn_ready[Hkv], o_ready[O parts], oproj, gateup[down parts], down
  p.ev_per_layer = Hkv + n_o_parts + 2 + n_ksplit;
  const int n_events = 1 + L * p.ev_per_layer;

  // ---- task graph -----------------------------------------------------------------------
  std::vector<Task> &T = out.tasks;
  T.clear();
  out.ops.clear();
  auto gemv = [&](uint8_t type, int layer, int row0, int nrows, int nm, uint32_t dep, uint32_t cnt,
                  uint32_t outev) {
    Task t{};
    t.type = type;
    t.n_m = static_cast<uint8_t>(nm);
    t.layer = static_cast<uint16_t>(layer);
    t.row0 = row0;
    t.nrows = static_cast<uint16_t>(nrows);
    t.dep_event = dep;
    t.dep_count = cnt;
    t.out_event = outev;
    return t;
  };
  const int n_o = cdiv(H, R_o), n_down = cdiv(H, R_d), n_lm = cdiv(V, R_lm);
  p.qkv_tasks_per_group = (G + 2) * (d / R_qkv);
  // gate/up tasks per split-K part of the down projection
  std::vector<uint32_t> gu_per_part(n_ksplit, 0);
  for (int r0 = 0; r0 < F; r0 += R_gu) gu_per_part[n_ksplit > 1 ? r0 / kchunk_ffn : 0] += 1;
  {
    Task t{};
    t.type = T_EMBED;
    t.dep_event = kNoEvent;
    t.out_event = p.ev_embed;
    T.push_back(t);
    out.ops.push_back({0, 1});
  }
  for (int l = 0; l < L; ++l) {
    const uint32_t dep = l == 0 ? p.ev_embed : ev_down(p, l - 1);
    const uint32_t cnt = l == 0 ? 1 : n_down;
    int b0 = static_cast<int>(T.size());
    // in KV-group order (the G query heads, then the K and V heads of group
    // 0, then group 1, ...), so each group's attention can start while the
    // later groups are still being projected
    for (int kvg = 0; kvg < Hkv; ++kvg)
      for (int j = 0; j < G + 2; ++j) {
        const int mat = j < G ? 0 : j - G + 1;          // 0 q, 1 k, 2 v
        const int hh = mat == 0 ? kvg * G + j : kvg;     // head within its matrix
        const int head = mat == 0 ? hh : (mat == 1 ? Hq + hh : Hq + Hkv + hh);
        for (int r0 = 0; r0 < d; r0 += R_qkv) {
          Task t = gemv(T_QKV, l, hh * d + r0, R_qkv, R_qkv / 16, dep, cnt, kNoEvent);
          t.aux = mat;
          t.aux2 = static_cast<uint32_t>(head);
          T.push_back(t);
        }
      }
    out.ops.push_back({b0, static_cast<int>(T.size())});
    b0 = static_cast<int>(T.size());
    for (int s = 0; s < p.attn_slots; ++s) {
      Task t{};
      t.type = T_ATTN;
      t.layer = static_cast<uint16_t>(l);
      t.dep_event = kNoEvent;  // resolved at run time: attn_ready(l, g)
      t.out_event = ev_o_ready(p, l, (s / p.attn_spg) / o_groups);
      t.aux = s;
      T.push_back(t);
    }
    out.ops.push_back({b0, static_cast<int>(T.size())});
    b0 = static_cast<int>(T.size());
    for (int k = 0; k < n_o_parts; ++k) {
      const int groups = std::min(o_groups, Hkv - k * o_groups);
      for (int r0 = 0; r0 < H; r0 += R_o) {
        const int nr = std::min(R_o, H - r0);
        Task t = gemv(T_OPROJ, l, r0, nr, cdiv(nr, 16), ev_o_ready(p, l, k),
                      static_cast<uint32_t>(groups * p.attn_spg), ev_oproj(p, l));
        t.ksplit = static_cast<uint8_t>(k);
        t.nsplit = static_cast<uint8_t>(n_o_parts);
        T.push_back(t);
      }
    }
    out.ops.push_back({b0, static_cast<int>(T.size())});
    b0 = static_cast<int>(T.size());
    for (int r0 = 0; r0 < F; r0 += R_gu) {
      const int nr = std::min(R_gu, F - r0);
      const int part = n_ksplit > 1 ? r0 / kchunk_ffn : 0;
      T.push_back(gemv(T_GATEUP, l, r0, nr, 2 * cdiv(nr, 16), ev_oproj(p, l), n_o, ev_gateup(p, l, part)));
    }
    out.ops.push_back({b0, static_cast<int>(T.size())});
    b0 = static_cast<int>(T.size());
    for (int ks = 0; ks < n_ksplit; ++ks)
      for (int r0 = 0; r0 < H; r0 += R_d) {
        const int nr = std::min(R_d, H - r0);
        Task t = gemv(T_DOWN, l, r0, nr, cdiv(nr, 16), ev_gateup(p, l, ks), gu_per_part[ks], ev_down(p, l));
        t.ksplit = static_cast<uint8_t>(ks);
        t.nsplit = static_cast<uint8_t>(n_ksplit);
        T.push_back(t);
      }
    out.ops.push_back({b0, static_cast<int>(T.size())});
  }
  {
    const int b0 = static_cast<int>(T.size());
    for (int r0 = 0; r0 < V; r0 += R_lm) {
      const int nr = std::min(R_lm, V - r0);
      T.push_back(gemv(T_LMHEAD, L - 1, r0, nr, cdiv(nr, 16), ev_down(p, L - 1), n_down, kNoEvent));
    }
    out.ops.push_back({b0, static_cast<int>(T.size())});
  }
  p.n_lm_tasks = n_lm;
  p.n_tasks = static_cast<int>(T.size());
  if (o.debug_unsatisfiable_dep) T[1].dep_count += 1;  // first QKV task

  // ---- RoPE: pair i at position t turns by t * theta^(-2i/d), in double ----------------
  const int half = d / 2;
  out.rope.assign(static_cast<size_t>(c.max_seq_len) * half, make_float2(0.f, 0.f));
  for (int t = 0; t < c.max_seq_len; ++t)
    for (int i = 0; i < half; ++i) {
      const double ang = static_cast<double>(t) * std::pow(static_cast<double>(c.rope_theta), -2.0 * i / d);
      out.rope[static_cast<size_t>(t) * half + i] =
          make_float2(static_cast<float>(std::cos(ang)), static_cast<float>(std::sin(ang)));
    }

  // ---- workspace (256-byte aligned pieces) and counter words ----------------------------
  size_t off = 0;
  auto carve = [&](size_t bytes) {
    const size_t at = off;
    off = align_up_z(off + bytes, 256);
    return at;
  };
  out.o_h = carve(sizeof(float) * maxB * H);
  out.o_qkv = carve(sizeof(float) * maxB * NQKV);
  out.o_part = carve(sizeof(float) * static_cast<size_t>(p.attn_slots) * G * (d + 4));
  out.o_o = carve(sizeof(float) * maxB * Hq * d);
  out.o_u = carve(sizeof(float) * maxB * F);
  out.o_arg = carve(sizeof(unsigned long long) * maxB);
  const int kparts = std::max(n_ksplit > 1 ? n_ksplit : 0, n_o_parts > 1 ? n_o_parts : 0);
  out.o_kpart = carve(sizeof(float) * static_cast<size_t>(kparts) * maxB * H);
  out.ws_bytes = off;
  out.n_events = n_events;
  out.comb_words = static_cast<size_t>(maxB) * Hkv;
  out.tile_words = static_cast<size_t>(H) / 16 + 1;
  out.sync_words = S_EVENTS + n_events + out.comb_words + out.tile_words;

  out.grid = grid;
  out.smem = smem;
  out.rows[0] = R_qkv;
  out.rows[1] = R_o;
  out.rows[2] = R_gu;
  out.rows[3] = R_d;
  out.rows[4] = R_lm;
  return MK_OK;
}

void bind_workspace(const Layout &lay, char *ws, uint32_t *sync, Params &p) {
  p.h = reinterpret_cast<float *>(ws + lay.o_h);
  p.qkv = reinterpret_cast<float *>(ws + lay.o_qkv);
  p.attn_part = reinterpret_cast<float *>(ws + lay.o_part);
  p.o = reinterpret_cast<float *>(ws + lay.o_o);
  p.u = reinterpret_cast<float *>(ws + lay.o_u);
  p.argmax = reinterpret_cast<unsigned long long *>(ws + lay.o_arg);
  p.kpart = reinterpret_cast<float *>(ws + lay.o_kpart);
  p.sync = sync;
  p.comb_ctr = sync + S_EVENTS + lay.n_events;
  p.tile_ctr = p.comb_ctr + lay.comb_words;
}

void bind_task_operands(const mk_model_config &c, const mk_weights &w, std::vector<Task> &tasks) {
  auto bf = [](const void *q) { return static_cast<const __nv_bfloat16 *>(q); };
  for (Task &t : tasks) {
    t.w0 = t.w1 = t.gain = nullptr;
    if (t.type == T_EMBED || t.type == T_END) continue;
    if (t.type == T_LMHEAD) {
      t.w0 = bf(w.lm_head);
      t.gain = bf(w.final_norm);
      continue;
    }
    const mk_layer_weights &lw = w.layers[t.layer < c.n_layers ? t.layer : 0];
    switch (t.type) {
      case T_QKV:
        t.w0 = bf(t.aux == 0 ? lw.wq : (t.aux == 1 ? lw.wk : lw.wv));
        t.gain = bf(lw.attn_norm);
        break;
      case T_ATTN:
        t.w0 = bf(lw.q_norm);
        t.w1 = bf(lw.k_norm);
        break;
      case T_OPROJ: t.w0 = bf(lw.wo); break;
      case T_GATEUP:
        t.w0 = bf(lw.w_gate);
        t.w1 = bf(lw.w_up);
        t.gain = bf(lw.mlp_norm);
        break;
      case T_DOWN: t.w0 = bf(lw.w_down); break;
      default: break;
    }
  }
}

}  // namespace mk
