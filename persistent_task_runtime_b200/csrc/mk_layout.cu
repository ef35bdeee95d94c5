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

// Solidified schedule (the Ada-MK summary's "Offline-Suche und
// Pfad-Solidifizierung": the execution order is fixed offline instead of by
// run-time dispatch).  List scheduling over the task array in queue order:
// each task goes to the CTA on which a cost model says it would start first,
// after that CTA's previous task and after the event it waits on is complete
// (the latest finish among the event's producers).  Costs: a projection task
// streams its weight bytes at an SM's share of the HBM bandwidth, plus a
// fixed per-task cost; an attention slot and the embedding task a fixed cost.
// Each CTA then runs its tasks in ascending index order.  That order cannot
// deadlock: the unfinished task with the smallest index has all of its
// producers (smaller indices) finished, and every earlier task of its own CTA
// too.
void solidify_schedule(const Params &p, const std::vector<Task> &T, int grid,
                       std::vector<int> &sched, std::vector<int> &off) {
  const double per_sm_bytes_per_us = 6.5e6 / 148.0;   // ~6.5 TB/s over 148 SMs
  // (an attention slot: 5 us measured best of 2.5, 5, 8 and 12 over batch 1-16)
  const double task_us = 0.8, attn_us = 5.0;
  const int n = static_cast<int>(T.size());
  std::vector<double> ev_ready(static_cast<size_t>(1 + p.L * p.ev_per_layer), 0.0);
  std::vector<double> cta_free(static_cast<size_t>(grid), 0.0);
  std::vector<int> owner(static_cast<size_t>(n), 0);
  for (int i = 0; i < n; ++i) {
    const Task &t = T[static_cast<size_t>(i)];
    double ready = 0.0, cost = attn_us;
    uint32_t sig = t.out_event;
    if (t.type == T_ATTN) {
      const int g = static_cast<int>(t.aux) / p.attn_spg;
      ready = ev_ready[static_cast<size_t>(ev_attn_input(p, t.layer, g))];
    } else if (t.dep_event != kNoEvent) {
      ready = ev_ready[t.dep_event];
    }
    if (t.type != T_ATTN && t.type != T_EMBED && t.type != T_KVAPP) {
      int K = t.type == T_OPROJ ? p.Hq * p.d : (t.type == T_DOWN ? p.F : p.H);
      const int kt = p.tc ? p.tc_kt[t.type] : (t.type == T_DOWN ? p.kchunk[K_FFN]
                                                : (t.type == T_OPROJ ? p.kchunk[K_ATT] : 0));
      if (t.nsplit > 1 && kt > 0) K = std::min(K - t.ksplit * kt, kt);
      const double rows = static_cast<double>(t.nrows) * (t.type == T_GATEUP ? 2 : 1);
      cost = task_us + rows * K * 2.0 / per_sm_bytes_per_us;
    }
    if (t.type == T_QKV) {
      const int head = static_cast<int>(t.aux2);
      const int g = t.aux == 0 ? head / p.G
                               : (t.aux == 1 ? head - p.Hq : head - p.Hq - p.Hkv);
      sig = static_cast<uint32_t>(ev_attn_ready(p, t.layer, g));
    }
    int best = 0;
    double best_start = 1e300;
    for (int c = 0; c < grid; ++c) {
      const double st = std::max(cta_free[static_cast<size_t>(c)], ready);
      if (st < best_start) {
        best_start = st;
        best = c;
      }
    }
    const double fin = best_start + cost;
    cta_free[static_cast<size_t>(best)] = fin;
    owner[static_cast<size_t>(i)] = best;
    if (sig != kNoEvent) ev_ready[sig] = std::max(ev_ready[sig], fin);
  }
  off.assign(static_cast<size_t>(grid) + 1, 0);
  for (int i = 0; i < n; ++i) off[static_cast<size_t>(owner[static_cast<size_t>(i)]) + 1] += 1;
  for (int c = 0; c < grid; ++c) off[static_cast<size_t>(c) + 1] += off[static_cast<size_t>(c)];
  sched.assign(static_cast<size_t>(n), 0);
  std::vector<int> fill(off.begin(), off.end() - 1);
  for (int i = 0; i < n; ++i) sched[static_cast<size_t>(fill[static_cast<size_t>(owner[static_cast<size_t>(i)])]++)] = i;
}

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
  if (o.attn_path < 0 || o.attn_path > 2)
    return lfail(err, MK_ERR_INVALID_ARG, "attn_path %d: 0 automatic, 1 CUDA cores, 2 mma.sync",
                 o.attn_path);
  if (o.attn_path == 2 && d != 64 && d != 128)
    return lfail(err, MK_ERR_UNSUPPORTED, "the mma.sync attention path needs head_dim 64 or 128");
  // attention on mma.sync tiles on request, and by default from batch 2 up
  // (measured on the 8B shape: as fast as the CUDA-core path at batch 1,
  // 4-17% faster steps from batch 2 to 16)
  const bool attn_mma = o.attn_path == 2 ||
                        (o.attn_path == 0 && (d == 64 || d == 128) && maxB >= kAttnMmaAutoBatch);
  const int smem_max = std::min(smem_optin, kMaxSmem);
  const int mt_cap = max_mtiles_for(maxB);

  // ---- GEMV path: warp-level mma.sync pages, or tcgen05 tiles of 128 rows -------------
  // The tensor-core path needs one 128-row tile per head (head_dim 128) and
  // inputs whose width is a whole number of 64-column swizzle atoms.
  const bool tc_ok = d == kTcRows && H % 64 == 0 && F % 64 == 0 && (Hq * d) % 64 == 0;
  if (o.gemv_path < 0 || o.gemv_path > 3)
    return lfail(err, MK_ERR_INVALID_ARG,
                 "gemv_path %d: 0 automatic, 1 mma.sync, 2 tcgen05, 3 mma.sync from tensor memory",
                 o.gemv_path);
  // mma.sync pages staged in tensor memory: weight pages arrive in boxes of
  // kTmBoxCols columns, so every input width is a whole number of boxes
  const bool tm = o.gemv_path == 3;
  if (tm) {
    if (o.w4) return lfail(err, MK_ERR_UNSUPPORTED, "4-bit weights run on the mma.sync GEMV path");
    if (H % kTmBoxCols || F % kTmBoxCols || (Hq * d) % kTmBoxCols)
      return lfail(err, MK_ERR_UNSUPPORTED,
                   "the tensor-memory GEMV path needs hidden, ffn and n_q_heads*head_dim "
                   "multiples of %d", kTmBoxCols);
    if (o.max_page_cols % kTmBoxCols)
      return lfail(err, MK_ERR_INVALID_ARG, "max_page_cols must be a multiple of %d on this path",
                   kTmBoxCols);
    if (o.o_split) return lfail(err, MK_ERR_INVALID_ARG, "o_split is not available on this path");
  }
  if (o.gemv_path == 2 && !tc_ok)
    return lfail(err, MK_ERR_UNSUPPORTED,
                 "the tensor-core GEMV path needs head_dim 128 and hidden, ffn and "
                 "n_q_heads*head_dim multiples of 64");
  if (o.gemv_path == 2 && o.o_split)
    return lfail(err, MK_ERR_INVALID_ARG, "o_split is an option of the mma.sync path");
  if (o.w4) {
    if (H % MK_W4_BLOCK_COLS || F % MK_W4_BLOCK_COLS || (Hq * d) % MK_W4_BLOCK_COLS)
      return lfail(err, MK_ERR_UNSUPPORTED,
                   "4-bit weights need hidden, ffn and n_q_heads*head_dim multiples of %d",
                   MK_W4_BLOCK_COLS);
    if (o.gemv_path == 2)
      return lfail(err, MK_ERR_UNSUPPORTED, "4-bit weights run on the mma.sync GEMV path");
    if (o.o_split) return lfail(err, MK_ERR_INVALID_ARG, "o_split is not available with 4-bit weights");
  }
  const bool tc = !o.w4 && !tm && (o.gemv_path == 2 || (o.gemv_path == 0 && tc_ok && !o.o_split &&
                                                         maxB >= kTcAutoBatch));
  if (tc) {
    for (int i = 0; i < 5; ++i)
      if (o.rows_per_task[i] != 0)
        return lfail(err, MK_ERR_INVALID_ARG, "rows_per_task is an option of the mma.sync path");
    if (o.max_page_cols != 0)
      return lfail(err, MK_ERR_INVALID_ARG, "max_page_cols is an option of the mma.sync path");
  }

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
  int R_o = std::min(rows_opt(1, 16 * pick(H / 16, mt_cap)), 16 * mt_cap);
  const int gu_cap = std::max(1, mt_cap / 2);   // gate and up tiles share a task
  // (under the solidified lists, which balance the SMs themselves, gate/up
  // tasks of two row tiles each: measured 2.5% faster steps at 8B batch 1 and
  // 7% at 1.5B than one tile)
  const int gu_dflt = o.schedule != 2 && !chunked ? std::min(2, gu_cap) : pick(F / 16, gu_cap);
  int R_gu = std::min(rows_opt(2, 16 * gu_dflt), 16 * gu_cap);
  // a split down projection has a third or less of the columns per task:
  // two row tiles per task keep its per-task costs (dependency check,
  // restaging at each part) small against its pages
  const bool ffn_split = F > kx_limit;
  const int nm_d = std::max(pick(H / 16, mt_cap), ffn_split ? std::min(2, mt_cap) : 1);
  int R_d = std::min(rows_opt(3, 16 * nm_d), 16 * mt_cap);
  int R_lm = std::min(rows_opt(4, 16 * pick(V / 16, mt_cap)), 16 * mt_cap);

  // ---- split-K of the down projection --------------------------------------------
  // Parts of at most kx_limit columns (the widest other input), so the down
  // projection's input stages like every other operator's.  A part's columns
  // are whole gate/up tasks' rows, so each part waits only on the gate/up
  // tasks that produce its slice of u.
  int n_ksplit = F > kx_limit ? cdiv(F, kx_limit) : 1;
  int kchunk_ffn = F;
  if (n_ksplit > 1) {
    // multiple of 32 and of R_gu (4-bit: of the 1024-column packed blocks)
    int unit = o.w4 ? MK_W4_BLOCK_COLS : ((R_gu % 32 == 0) ? R_gu : 2 * R_gu);
    if (tm) {   // ... and of the tensor-memory boxes
      int u = unit;
      while (u % kTmBoxCols) u += unit;
      unit = u;
    }
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
  int n_o_parts = cdiv(Hkv, o_groups);

  // ---- tensor-core path: 128-row tiles, split along K for load balance ----------------
  // A task is one 128-row tile (gate/up: the gate tile and the up tile of the
  // same rows) over a K range.  An operator with few tiles is split along K
  // into parts of whole weight pages so that it has enough tasks to spread;
  // the part that completes a tile sums the parts in a fixed order.  The O
  // projection is split into one part per KV group, each waiting only for the
  // attention of its group.  The down projection's parts are whole gate/up
  // tiles' rows, as on the other path.
  int tc_bpad = 0, tc_kx = 0, tc_kc = 0;
  int split[5] = {1, 1, 1, 1, 1};      // QKV, O, gate/up, down, LM head
  int kt[5] = {0, 0, 0, 0, 0};          // columns per part (0: unsplit)
  if (tc) {
    tc_bpad = align_up_i(maxB, 8);
    tc_kx = kTcXBytes / (2 * tc_bpad * 2);   // bf16 hi + lo rows of tc_bpad sequences
    tc_kc = 128;                             // 32 KB pages (128 rows x 128 columns)
    R_qkv = R_o = R_gu = R_d = R_lm = kTcRows;
    // Split-K parts of an operator of `tiles` tasks' worth of n_m 128-row
    // tiles over K columns: the count that minimises the operator's makespan
    // on `grid` CTAs in a simple model, rounds of tasks (ceil(tasks / grid))
    // times a task's weight columns (per tile) plus a fixed cost per task
    // (epilogue, split-K sum and hand-offs, about 4 us: the time one SM's
    // share of HBM streams 640 columns of a 128-row tile).  Ties go to fewer
    // parts.
    constexpr long long kTaskCostCols = 640;
    auto parts_for = [&](int tiles, int nm, int K, int i) {
      const int nmax = std::max(1, K / tc_kc);
      long long best = -1;
      int bn = 1, bw = K;
      for (int n = 1; n <= nmax; ++n) {
        const int w = align_up_i(cdiv(K, n), tc_kc);
        if (cdiv(K, w) != n) continue;   // the same split as a smaller count
        const long long rounds = cdiv(tiles * n, grid);
        const long long cost = rounds * (static_cast<long long>(nm) * w + kTaskCostCols);
        if (best < 0 || cost < best) {
          best = cost;
          bn = n;
          bw = w;
        }
      }
      split[i] = bn;
      kt[i] = bn > 1 ? bw : 0;
    };
    parts_for(NQKV / kTcRows, 1, H, 0);
    parts_for(cdiv(F, kTcRows), 2, H, 2);
    parts_for(cdiv(H, kTcRows), 1, F, 3);
    // the O projection in parts of whole KV groups (each part waits only for
    // its groups' attention), as many groups per part as the same model says
    {
      long long best = -1;
      for (int og = 1; og <= Hkv; ++og) {
        if (Hkv % og != 0) continue;
        const long long rounds = cdiv(cdiv(H, kTcRows) * (Hkv / og), grid);
        const long long cost = rounds * (static_cast<long long>(og) * G * d + kTaskCostCols);
        if (best < 0 || cost < best) {
          best = cost;
          o_groups = og;
        }
      }
    }
    n_o_parts = Hkv / o_groups;
    split[1] = n_o_parts;
    kt[1] = n_o_parts > 1 ? o_groups * G * d : 0;
    n_ksplit = split[3];
    kchunk_ffn = kt[3] > 0 ? kt[3] : F;
    if (n_ksplit > 255 || split[0] > 255 || split[2] > 255)
      return lfail(err, MK_ERR_UNSUPPORTED, "too many split-K parts");
  } else {
    split[1] = n_o_parts;
    split[3] = n_ksplit;
  }

  // ---- shared memory: activation staging and the weight-page ring ------------------
  // Activation staging holds fp32 rows of every sequence: a whole input when
  // the widest input other than the FFN's fits in kXWholeMax (staged once,
  // reused by the operator's later tasks on this SM), else one page-wide
  // chunk (<= 64 KB).
  const int max_chunks = cdiv(c.max_seq_len, P);
  const int x_whole = maxB * x_row_bytes(kx_limit);
  // (the tensor-core path reduces in tensor memory: no cross-warp scratch;
  // its output buffers hold two 128-row tiles, two of them in flight)
  const int red_bytes = tc ? 0 : kComputeWarps * 16 * 8 * n_tiles_for(maxB) * 4;
  const int out_stride = tc ? 2 * kTcRows : 16 * mt_cap;
  const int out_bytes = align_up_i(maxB * out_stride * 4, 128);
  const int n_out = tc ? 2 : kOutSlots;
  const int off_look = 1024;   // loader lookahead
  const int off_slots = off_look + kLookBytes;
  const int off_red = align_up_i(off_slots + kTaskSlots * kSlotBytes, 128);
  const int off_out = align_up_i(off_red + red_bytes, 128);
  const int off_x = align_up_i(off_out + n_out * out_bytes, tc ? 1024 : 128);

  struct Geom {
    int kp[4], page_bytes, tpp, x_cap, off_pages, n_pages, ring;
  };
  // attention scratch in the staging area: q [G][d] plus either the page's
  // scores [G][tpp], per-head statistics, the current token's K and V (bf16)
  // and (mma.sync attention) the per-page warp counters and the warps'
  // (O, m, l) before their merge, or the combine's per-chunk (m, l) pairs
  auto attn_need = [&](int tpp) {
    const int pages = (G * tpp + 3 * kMaxGroup) * 4 + 2 * d * 2 +
                      (attn_mma ? kMaxPages * 4 + kComputeWarps * G * (d + 2) * 4 : 0);
    return G * d * 4 + std::max(pages, (2 * max_chunks * G + 2 * G) * 4);
  };
  // Geometry for pages of at most `kpmax` columns; false if the staging
  // area cannot hold one page-wide chunk within 64 KB.
  auto geometry = [&](int kpmax, Geom &g) {
    // (tensor-memory staging: whole boxes of kTmBoxCols columns)
    const int pc_unit = tm ? kTmBoxCols : 32;
    auto page_cols = [&](int K) {
      if (K <= kpmax) return K;
      return align_up_i(cdiv(K, cdiv(K, kpmax)), pc_unit);
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
    const int att_need = attn_need(g.tpp);
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
  for (int cand = tm ? colcap / kTmBoxCols * kTmBoxCols : colcap; cand >= (tm ? kTmBoxCols : 32) && !tc && !o.w4;
       cand -= tm ? kTmBoxCols : (cand > 256 ? 256 : 32)) {
    Geom g{};
    if (geometry(cand, g)) cands.push_back(g);
  }
  // 4-bit projections: a page is one packed row tile over up to 4096 columns
  // (4 blocks, 33 KB; fewer blocks when a page-wide activation chunk of every
  // sequence would not fit the staging area); the bf16 LM head streams in
  // pages of 16 rows that fit the same size
  for (int nb = kW4PageBlocks; nb >= 1 && o.w4 && cands.empty(); nb /= 2) {
    Geom g{};
    const int kw = nb * MK_W4_BLOCK_COLS;
    g.kp[K_HID] = std::min(H, kw);
    g.kp[K_ATT] = std::min(Hq * d, kw);
    g.kp[K_FFN] = std::min(kchunk_ffn, kw);
    // (pages start on 1024-byte boundaries: the attention's swizzled K/V copies)
    g.page_bytes = align_up_i(nb * MK_W4_BLOCK_BYTES, 1024);
    g.kp[K_LM] = 32;
    while (16 * row_pitch_bytes(g.kp[K_LM] + 32) <= g.page_bytes && g.kp[K_LM] + 32 <= kMaxPageCols)
      g.kp[K_LM] += 32;
    const int kp_big = std::max(std::max(g.kp[0], g.kp[1]), g.kp[2]);
    const int x_chunk = maxB * x_row_bytes(kp_big);
    if (x_chunk <= kXWholeMax) {
      const int x_cap = x_whole <= kXWholeMax ? std::max(x_whole, x_chunk) : x_chunk;
      g.tpp = std::min((g.page_bytes / (4 * d)) / P * P, 16 * P);
      const int att_need = attn_need(g.tpp);
      g.x_cap = std::max(x_cap, att_need);
      g.off_pages = align_up_i(off_x + g.x_cap, 1024);
      g.n_pages = std::min(kMaxPages, (smem_max - g.off_pages) / g.page_bytes);
      g.ring = g.n_pages * g.page_bytes;
      if (g.tpp >= P && g.n_pages >= 2) cands.push_back(g);
    }
  }
  if (tc) {
    // two activation chunk buffers (also the attention scratch), then the
    // ring of 128-row weight pages
    Geom g{};
    for (int i = 0; i < 4; ++i) g.kp[i] = tc_kc;
    g.page_bytes = kTcRows * tc_kc * 2;
    g.tpp = std::min((g.page_bytes / (4 * d)) / P * P, 16 * P);
    const int att_need = attn_need(g.tpp);
    g.x_cap = std::max(2 * kTcXBytes, align_up_i(att_need, 1024));
    g.off_pages = align_up_i(off_x + g.x_cap, 1024);
    g.n_pages = std::min(kMaxPages, (smem_max - g.off_pages) / g.page_bytes);
    g.ring = g.n_pages * g.page_bytes;
    if (g.tpp >= P) cands.push_back(g);
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
  // partial chunk per sequence -- at larger batches about maxB / 4 chunks per
  // CTA, so that many sequences' long contexts split into chunks small enough
  // to spread evenly over the CTAs (16 sequences at context 1024: chunks of
  // 224 tokens instead of 864)
  p.attn_spg = cdiv(grid * std::max(1, maxB / 4), Hkv) + maxB;
  p.attn_slots = Hkv * p.attn_spg;
  p.n_o_parts = n_o_parts;
  p.o_groups = o_groups;
  p.kchunk[K_ATT] = n_o_parts > 1 ? o_groups * G * d : 0;
  p.wait_limit_ns = o.wait_limit_ns;
  p.n_ffn_parts = n_ksplit;
  p.chunk_seq = -1;   // decode steps (a prompt chunk sets its sequence)
  p.attn_mma = attn_mma ? 1 : 0;
  p.w4 = o.w4 ? 1 : 0;
  p.n_out = n_out;
  p.tile_rows = tc ? kTcRows : 16;
  p.tc = tc ? 1 : 0;
  p.tm = tm ? 1 : 0;
  p.tc_bpad = tc_bpad;
  p.tc_n = 2 * tc_bpad;
  p.tc_kc = tc_kc;
  p.tc_kx = tc_kx;
  p.tc_kt[T_QKV] = kt[0];
  p.tc_kt[T_OPROJ] = kt[1];
  p.tc_kt[T_GATEUP] = kt[2];
  p.tc_kt[T_DOWN] = kt[3];
  p.tc_kt[T_LMHEAD] = kt[4];
  p.ev_embed = 0;
  p.ev_layer0 = 1;
  // attn_ready[Hkv], o_ready[O parts], oproj, gateup[down parts], down
  // (prefill plans: then kv_ready[Hkv])
  p.kv_tasks = o.prefill ? 1 : 0;
  p.ev_per_layer = Hkv + n_o_parts + 2 + n_ksplit + (o.prefill ? Hkv : 0);
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
  // row tiles of `nr` rows: 16-row mma tiles, or 128-row tensor-core tiles
  auto mtiles = [&](int nr) { return tc ? cdiv(nr, kTcRows) : cdiv(nr, 16); };
  // (with split-K parts, only the part that completes a tile signals)
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
        for (int r0 = 0; r0 < d; r0 += R_qkv)
          for (int ks = 0; ks < split[0]; ++ks) {
            Task t = gemv(T_QKV, l, hh * d + r0, R_qkv, mtiles(R_qkv), dep, cnt, kNoEvent);
            t.aux = mat;
            t.aux2 = static_cast<uint32_t>(head);
            t.ksplit = static_cast<uint8_t>(ks);
            t.nsplit = static_cast<uint8_t>(split[0]);
            t.map0 = static_cast<uint32_t>(tc_map_index(l, mat));
            T.push_back(t);
          }
      }
    out.ops.push_back({b0, static_cast<int>(T.size())});
    b0 = static_cast<int>(T.size());
    if (o.prefill)
      // one task per KV group appends every row's K/V before the group's
      // attention reads the cache
      for (int kvg = 0; kvg < Hkv; ++kvg) {
        Task t{};
        t.type = T_KVAPP;
        t.layer = static_cast<uint16_t>(l);
        t.dep_event = static_cast<uint32_t>(ev_attn_ready(p, l, kvg));
        t.dep_count = static_cast<uint32_t>(p.qkv_tasks_per_group);
        t.out_event = static_cast<uint32_t>(ev_kv_ready(p, l, kvg));
        t.aux = static_cast<uint32_t>(kvg);
        T.push_back(t);
      }
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
        Task t = gemv(T_OPROJ, l, r0, nr, mtiles(nr), ev_o_ready(p, l, k),
                      static_cast<uint32_t>(groups * p.attn_spg), ev_oproj(p, l));
        t.ksplit = static_cast<uint8_t>(k);
        t.nsplit = static_cast<uint8_t>(n_o_parts);
        t.map0 = static_cast<uint32_t>(tc_map_index(l, 3));
        T.push_back(t);
      }
    }
    out.ops.push_back({b0, static_cast<int>(T.size())});
    b0 = static_cast<int>(T.size());
    for (int r0 = 0; r0 < F; r0 += R_gu) {
      const int nr = std::min(R_gu, F - r0);
      const int part = n_ksplit > 1 ? r0 / kchunk_ffn : 0;
      for (int ks = 0; ks < split[2]; ++ks) {
        Task t = gemv(T_GATEUP, l, r0, nr, 2 * mtiles(nr), ev_oproj(p, l), n_o,
                      ev_gateup(p, l, part));
        t.ksplit = static_cast<uint8_t>(ks);
        t.nsplit = static_cast<uint8_t>(split[2]);
        t.map0 = static_cast<uint32_t>(tc_map_index(l, 4));
        t.map1 = static_cast<uint32_t>(tc_map_index(l, 5));
        T.push_back(t);
      }
    }
    out.ops.push_back({b0, static_cast<int>(T.size())});
    b0 = static_cast<int>(T.size());
    for (int ks = 0; ks < n_ksplit; ++ks)
      for (int r0 = 0; r0 < H; r0 += R_d) {
        const int nr = std::min(R_d, H - r0);
        Task t = gemv(T_DOWN, l, r0, nr, mtiles(nr), ev_gateup(p, l, ks), gu_per_part[ks],
                      ev_down(p, l));
        t.ksplit = static_cast<uint8_t>(ks);
        t.nsplit = static_cast<uint8_t>(n_ksplit);
        t.map0 = static_cast<uint32_t>(tc_map_index(l, 6));
        T.push_back(t);
      }
    out.ops.push_back({b0, static_cast<int>(T.size())});
  }
  {
    const int b0 = static_cast<int>(T.size());
    out.first_lm_task = b0;
    for (int r0 = 0; r0 < V; r0 += R_lm) {
      const int nr = std::min(R_lm, V - r0);
      Task t = gemv(T_LMHEAD, L - 1, r0, nr, mtiles(nr), ev_down(p, L - 1), n_down, kNoEvent);
      t.map0 = static_cast<uint32_t>(tc_map_index(L, 0));
      T.push_back(t);
    }
    out.ops.push_back({b0, static_cast<int>(T.size())});
  }
  p.n_lm_tasks = n_lm;
  p.n_tasks = static_cast<int>(T.size());
  if (o.schedule < 0 || o.schedule > 2)
    return lfail(err, MK_ERR_INVALID_ARG,
                 "schedule %d: 0 automatic (solidified), 1 solidified, 2 dynamic queue", o.schedule);
  // the solidified lists by default: measured no slower than the queue at 8B
  // batch 1 and 0.5-8% faster at batch 2-16 and at 1.5B batch 1
  if (o.schedule != 2) solidify_schedule(p, T, grid, out.sched, out.sched_off);
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
  // split-K partials: QKV and down share one area (a layer's QKV starts only
  // after the previous layer's down projection is complete, and the down
  // projection only after every QKV tile); the O projection (whose first
  // part may start while later QKV tiles are still summed) and gate/up
  // (which overlaps the down projection) have their own
  size_t kpart_floats = 0;
  if (split[0] > 1) kpart_floats = std::max(kpart_floats, static_cast<size_t>(split[0]) * NQKV);
  if (split[3] > 1) kpart_floats = std::max(kpart_floats, static_cast<size_t>(split[3]) * H);
  out.o_kpart = carve(sizeof(float) * kpart_floats * maxB);
  out.o_kpart_o = carve(sizeof(float) * (split[1] > 1 ? static_cast<size_t>(split[1]) * H : 0) * maxB);
  out.o_kpart2 = carve(sizeof(float) * (split[2] > 1 ? static_cast<size_t>(split[2]) * 2 * F : 0) *
                       maxB);
  // per-128-row sums of h^2, written by the producers of h (tensor-core path)
  const size_t ssq_floats = tc ? static_cast<size_t>(cdiv(H, kTcRows)) * maxB : 0;
  out.o_ssq_attn = carve(sizeof(float) * ssq_floats);
  out.o_ssq_mlp = carve(sizeof(float) * ssq_floats);
  // the staged GEMV inputs, bf16 [2 * bpad][K] (tensor-core path)
  {
    const int xk[4] = {H, H, Hq * d, F};
    for (int i = 0; i < 4; ++i)
      out.o_xs[i] = carve(tc ? sizeof(__nv_bfloat16) * 2 * tc_bpad * static_cast<size_t>(xk[i]) : 0);
  }
  out.ws_bytes = off;
  out.n_events = n_events;
  out.comb_words = static_cast<size_t>(maxB) * Hkv;
  out.tile_words = static_cast<size_t>(std::max(H, tc ? NQKV : 0)) / 16 + 1;
  out.tile2_words = static_cast<size_t>(F) / 16 + 1;
  out.tile_o_words = static_cast<size_t>(H) / 16 + 1;
  out.sync_words = S_EVENTS + n_events + out.comb_words + out.tile_words + out.tile2_words +
                   out.tile_o_words;
  out.n_maps = tc ? L * kTcMatsPerLayer + 1 + 4 : (tm ? L * kTcMatsPerLayer + 1 : 0);
  p.xs_map0 = L * kTcMatsPerLayer + 1;
  for (int i = 0; i < 5; ++i) out.splits[i] = split[i];

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
  p.kpart2 = reinterpret_cast<float *>(ws + lay.o_kpart2);
  p.ssq_attn = reinterpret_cast<float *>(ws + lay.o_ssq_attn);
  p.ssq_mlp = reinterpret_cast<float *>(ws + lay.o_ssq_mlp);
  for (int i = 0; i < 4; ++i) p.xs[i] = reinterpret_cast<__nv_bfloat16 *>(ws + lay.o_xs[i]);
  p.sync = sync;
  p.comb_ctr = sync + S_EVENTS + lay.n_events;
  p.tile_ctr = p.comb_ctr + lay.comb_words;
  p.tile_ctr2 = p.tile_ctr + lay.tile_words;
  p.kpart_o = reinterpret_cast<float *>(ws + lay.o_kpart_o);
  p.tile_ctr_o = p.tile_ctr2 + lay.tile2_words;
}

void bind_task_operands(const mk_model_config &c, const mk_weights &w, std::vector<Task> &tasks) {
  auto bf = [](const void *q) { return static_cast<const __nv_bfloat16 *>(q); };
  for (Task &t : tasks) {
    t.w0 = t.w1 = t.gain = nullptr;
    if (t.type == T_END) continue;
    if (t.type == T_EMBED) {
      t.w1 = bf(w.layers[0].attn_norm);   // the first QKV input's gain (staged input)
      continue;
    }
    if (t.type == T_LMHEAD) {
      t.w0 = bf(w.lm_head);
      t.gain = bf(w.final_norm);
      continue;
    }
    const int li = t.layer < c.n_layers ? t.layer : 0;
    const mk_layer_weights &lw = w.layers[li];
    // 4-bit plans: the projections' packed matrices instead of the bf16 ones
    const mk_w4_layer_weights *q4 = w.w4_layers != nullptr ? &w.w4_layers[li] : nullptr;
    auto mat = [&](int j, const void *bf16_ptr) { return bf(q4 != nullptr ? q4->q[j] : bf16_ptr); };
    switch (t.type) {
      case T_QKV:
        t.w0 = t.aux == 0 ? mat(0, lw.wq) : (t.aux == 1 ? mat(1, lw.wk) : mat(2, lw.wv));
        t.gain = bf(lw.attn_norm);
        break;
      case T_ATTN:
      case T_KVAPP:
        t.w0 = bf(lw.q_norm);
        t.w1 = bf(lw.k_norm);
        break;
      case T_OPROJ:
        t.w0 = mat(3, lw.wo);
        t.w1 = bf(lw.mlp_norm);   // the gain of the input it produces (gate/up's)
        break;
      case T_GATEUP:
        t.w0 = mat(4, lw.w_gate);
        t.w1 = mat(5, lw.w_up);
        t.gain = bf(lw.mlp_norm);
        break;
      case T_DOWN:
        t.w0 = mat(6, lw.w_down);
        // the gain of the input it produces: the next layer's QKV, or the LM head
        t.w1 = bf(t.layer + 1 < c.n_layers ? w.layers[t.layer + 1].attn_norm : w.final_norm);
        break;
      default: break;
    }
  }
}

}  // namespace mk

// ---- tensor maps of the weight matrices (tensor-core path) -------------------------
// One 2-D map per matrix [rows][K] (bf16, row-major): a box is 64 columns
// (128 bytes, one swizzle atom) by 128 rows, copied with the 128-byte swizzle
// that the tensor core's K-major operand layout expects.  Rows past the end
// of a matrix (a ragged last tile) arrive as zeros.

#include <cuda.h>
#include <cudaTypedefs.h>

namespace mk {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder(std::string &err) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (encode == nullptr) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr) {
      lfail(err, MK_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
      return nullptr;
    }
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return encode;
}
}  // namespace

int encode_kv_maps(const mk_model_config &c, const mk_kv_cache &kv, int page_size,
                   std::vector<unsigned char> &out, std::string &err) {
  auto encode = tensor_map_encoder(err);
  if (encode == nullptr) return MK_ERR_CUDA;
  const int L = c.n_layers, d = c.head_dim;
  out.assign(static_cast<size_t>(2 * L) * sizeof(CUtensorMap), 0);
  const cuuint64_t rows = static_cast<cuuint64_t>(kv.num_pages) * c.n_kv_heads * page_size;
  for (int l = 0; l < L; ++l)
    for (int kvi = 0; kvi < 2; ++kvi) {
      CUtensorMap m;
      cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), rows};
      cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
      cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(page_size)};
      cuuint32_t estr[2] = {1, 1};
      void *base = kvi == 0 ? kv.k_pages[l] : kv.v_pages[l];
      const CUresult r = encode(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return lfail(err, MK_ERR_CUDA, "KV tensor map: cuTensorMapEncodeTiled failed (%d)", r);
      std::memcpy(out.data() + static_cast<size_t>(2 * l + kvi) * sizeof(CUtensorMap), &m, sizeof(m));
    }
  return MK_OK;
}

int encode_weight_maps(const mk_model_config &c, const mk_weights &w, const Layout &lay,
                       const char *ws, std::vector<unsigned char> &out, std::string &err) {
  out.clear();
  if (lay.n_maps == 0) return MK_OK;
  auto encode = tensor_map_encoder(err);
  if (encode == nullptr) return MK_ERR_CUDA;
  const int L = c.n_layers, H = c.hidden, F = c.ffn, d = c.head_dim;
  const int Hq = c.n_q_heads, Hkv = c.n_kv_heads;
  out.assign(static_cast<size_t>(lay.n_maps) * sizeof(CUtensorMap), 0);
  auto one = [&](int idx, const void *ptr, int rows, int K, int box_rows = kTcRows) {
    CUtensorMap m;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcAtomCols), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return lfail(err, MK_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", r);
    std::memcpy(out.data() + static_cast<size_t>(idx) * sizeof(CUtensorMap), &m, sizeof(m));
    return MK_OK;
  };
  // tensor-memory staging (mma.sync pages): a 3-D view of each matrix,
  // x = 64 columns (128 bytes), y = rows, z = 64-column blocks, so that a box
  // of 64 x 16 x 8 lands as 128 rows of 128 bytes (row 16 b + r = block b of
  // weight row r), 128-byte swizzled: four tcgen05.cp sources
  auto one_tm = [&](int idx, const void *ptr, int rows, int K) {
    CUtensorMap m;
    cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(K / 64)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2, 128};
    cuuint32_t box[3] = {64, 16, static_cast<cuuint32_t>(kTmBoxCols / 64)};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = encode(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return lfail(err, MK_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", r);
    std::memcpy(out.data() + static_cast<size_t>(idx) * sizeof(CUtensorMap), &m, sizeof(m));
    return MK_OK;
  };
  int rc = MK_OK;
  if (lay.p.tm) {
    for (int l = 0; l < L && rc == MK_OK; ++l) {
      const mk_layer_weights &s = w.layers[l];
      if ((rc = one_tm(tc_map_index(l, 0), s.wq, Hq * d, H)) ||
          (rc = one_tm(tc_map_index(l, 1), s.wk, Hkv * d, H)) ||
          (rc = one_tm(tc_map_index(l, 2), s.wv, Hkv * d, H)) ||
          (rc = one_tm(tc_map_index(l, 3), s.wo, H, Hq * d)) ||
          (rc = one_tm(tc_map_index(l, 4), s.w_gate, F, H)) ||
          (rc = one_tm(tc_map_index(l, 5), s.w_up, F, H)) ||
          (rc = one_tm(tc_map_index(l, 6), s.w_down, H, F)))
        break;
    }
    if (rc == MK_OK) rc = one_tm(tc_map_index(L, 0), w.lm_head, c.vocab, H);
    return rc;
  }
  for (int l = 0; l < L && rc == MK_OK; ++l) {
    const mk_layer_weights &s = w.layers[l];
    if ((rc = one(tc_map_index(l, 0), s.wq, Hq * d, H)) ||
        (rc = one(tc_map_index(l, 1), s.wk, Hkv * d, H)) ||
        (rc = one(tc_map_index(l, 2), s.wv, Hkv * d, H)) ||
        (rc = one(tc_map_index(l, 3), s.wo, H, Hq * d)) ||
        (rc = one(tc_map_index(l, 4), s.w_gate, F, H)) ||
        (rc = one(tc_map_index(l, 5), s.w_up, F, H)) ||
        (rc = one(tc_map_index(l, 6), s.w_down, H, F)))
      break;
  }
  if (rc == MK_OK) rc = one(tc_map_index(L, 0), w.lm_head, c.vocab, H);
  // the staged inputs: one box is every row (2 * bpad) of 64 columns
  const int xk[4] = {H, H, c.n_q_heads * d, F};
  for (int i = 0; i < 4 && rc == MK_OK; ++i)
    rc = one(lay.p.xs_map0 + i, ws + lay.o_xs[i], lay.p.tc_n, xk[i], lay.p.tc_n);
  return rc;
}

}  // namespace mk
