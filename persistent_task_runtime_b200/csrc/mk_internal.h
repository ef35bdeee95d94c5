// Internal layout shared by the host plan builder (mk_api.cu) and the
// persistent kernel (mk_kernel.cu).  Not part of the public ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstring>
#include <string>
#include <vector>

#include "../../include/mk.h"

namespace mk {

// ---- CTA shape -------------------------------------------------------------
// 8 warps per CTA: registers are granted per group of four warps, so 8 warps
// (not 10) leave 255 registers per thread and the consumers run spill-free.
constexpr int kComputeWarps = 6;                  // consumers
constexpr int kLoaderWarp = 0;                    // producer (TMA issue, queue)
constexpr int kStorerWarp = 1 + kComputeWarps;    // epilogues + signalling
constexpr int kThreads = 32 * (kComputeWarps + 2);
constexpr int kComputeThreads = 32 * kComputeWarps;
constexpr int kTaskSlots = 4;                     // tasks in flight per CTA
constexpr int kSlotBytes = 96;                    // one task slot in shared memory
constexpr int kLookBytes = 512;                   // loader lookahead area
constexpr int kOutSlots = 4;                      // compute -> storer buffers (upper bound)
constexpr int kMaxPages = 16;                     // ring entries (upper bound)
constexpr int kMaxMTiles = 8;                     // 16-row tiles per GEMV task (B <= 4)
constexpr int kMaxPageCols = 2048;                // widest weight page (16 rows)
constexpr int kXWholeMax = 72 * 1024;             // largest activation staged whole (all sequences)
constexpr int kMaxGroup = 8;                      // query heads per KV head
constexpr int kMaxSmem = 232448;                  // opt-in smem per CTA (B200)

// ---- tensor-core GEMV path (tcgen05) -------------------------------------------
// A task is one or two 128-row tiles of a weight matrix over a K range; the
// weights arrive by TMA tensor copies in the 128-byte-swizzled K-major layout
// the tensor core reads, the activation is staged as bf16 hi/lo rows in the
// same layout, and the fp32 accumulators live in tensor memory.
constexpr int kTcRows = 128;                      // MMA M: weight rows per tile
constexpr int kTcAtomCols = 64;                   // columns of one 128-byte swizzle atom
constexpr int kTcAtomBytes = kTcRows * 128;       // one weight atom: 128 rows x 128 B
constexpr int kTcXBytes = 32 * 1024;              // one staged activation chunk buffer
constexpr int kTcTmemCols = 128;                  // tensor-memory columns allocated per CTA
constexpr int kTcAutoBatch = 4;                   // smallest max_batch that takes it by default
constexpr int kAttnMmaAutoBatch = 2;              // smallest max_batch that takes the mma.sync attention

// ---- mma.sync GEMV over weights staged in tensor memory -------------------------
// 16-row weight pages arrive by TMA in 512-column boxes (128-byte swizzle, as
// 128 "virtual rows" of 64 columns: 64-column block b of weight row r at row
// 16 b + r), are copied into tensor memory (tcgen05.cp, four 128 x 256-bit
// copies per box, one per 16 columns of the blocks) and read back as mma.sync
// A fragments (tcgen05.ld.16x256b), so a page leaves shared memory as soon as
// it is copied and tensor memory adds kTmSlots pages of bytes in flight per SM.
constexpr int kTmSlots = 4;                       // tensor-memory page slots
constexpr int kTmSlotCols = 128;                  // columns per slot (a 2048-column page)
constexpr int kTmBoxCols = 512;                   // weight columns per TMA box (16 KB)
constexpr int kTmBoxBytes = 16 * kTmBoxCols * 2;
constexpr int kTcMatsPerLayer = 7;                // tensor maps: wq wk wv wo w_gate w_up w_down

// ---- kernel variants (template argument of the step kernel) -------------------
constexpr int kVarTc = 1;        // projections on tcgen05 tiles (else mma.sync pages)
constexpr int kVarW4 = 2;        // 4-bit weight consumer
constexpr int kVarAttnMma = 4;   // attention on mma.sync tiles over swizzled K/V pages
constexpr int kVarTm = 8;        // mma.sync GEMV reading its weight pages from tensor memory

// ---- task descriptor (64 bytes, four 16-byte loads) ---------------------------
enum TaskType : uint8_t {
  T_EMBED = 1,
  T_QKV = 2,
  T_ATTN = 3,
  T_OPROJ = 4,
  T_GATEUP = 5,
  T_DOWN = 6,
  T_LMHEAD = 7,
  T_KVAPP = 8,     // prefill plans: QK-norm + RoPE + KV append of one KV group, every row
  T_END = 255,
};

struct alignas(16) Task {
  uint8_t type;
  uint8_t n_m;        // 16-row tiles (GEMV); gate/up: gate tiles + up tiles
  uint16_t layer;
  uint32_t row0;      // first output row within its matrix
  uint16_t nrows;     // valid output rows (<= 16 * n_m; gate/up: per matrix)
  uint8_t ksplit;     // split-K part of this task (O / down projections)
  uint8_t nsplit;     // number of split-K parts of its row tile (0 or 1: none)
  uint32_t dep_event; // event this task waits on (kNoEvent = none)
  uint32_t dep_count; // completions of dep_event per step
  uint32_t out_event; // event incremented once the task's output is visible
  uint32_t aux;       // QKV: matrix (0 q, 1 k, 2 v); ATTN: slot index
  uint32_t aux2;      // QKV: global head index (q heads, then k, then v)
  // operands, filled in by the plan so that no task looks up a layer table:
  const __nv_bfloat16 *w0;    // GEMV: the weight matrix (gate/up: gate); ATTN: q-norm gain
  const __nv_bfloat16 *w1;    // gate/up: the up matrix; ATTN: k-norm gain
  const __nv_bfloat16 *gain;  // RMSNorm gain of the task's input (QKV, gate/up, LM head)
  uint32_t map0, map1;        // tensor-core path: tensor maps of w0 / w1 (index into Params::tmaps)
};
static_assert(sizeof(Task) == 64, "task descriptor must be 64 bytes");
constexpr uint32_t kNoEvent = 0xffffffffu;

// ---- counters region (uint32 words) ----------------------------------------
enum SyncWord : int {
  S_QUEUE = 0,     // next ticket
  S_EXIT = 1,      // CTAs that finished the launch
  S_STATUS = 2,    // first device error (0 = none)
  S_ABORT = 3,     // nonzero: every CTA leaves as soon as it sees it
  S_INFO = 4,      // 4 words: task index, event, value seen, code detail
  S_LMCTR = 8,     // LM-head tasks finished this step (reset by the last)
  S_EVENTS = 16,   // events start here
};

// ---- op classes for page geometry --------------------------------------------
enum OpK : int { K_HID = 0, K_ATT = 1, K_FFN = 2, K_LM = 3 };

// ---- kernel parameters (passed by value, < 4 KB) ----------------------------
struct Params {
  // plan (static)
  const Task *tasks;
  const __nv_bfloat16 *embed;   // token embedding [V][H]
  const float2 *rope_cs;        // [max_seq_len][d/2] (cos, sin)
  float *h;                     // [maxB][H]      residual stream
  float *qkv;                   // [maxB][NQKV]   raw projections
  float *attn_part;             // [slots][G][d+4] chunk partials (acc, m, l, pad)
  float *o;                     // [maxB][Hq*d]   attention output
  float *u;                     // [maxB][F]      SwiGLU output
  unsigned long long *argmax;   // [maxB]         packed (value, ~index)
  uint32_t *sync;               // counters
  uint32_t *comb_ctr;           // [maxB][Hkv]    attention chunks done

  int L, H, Hq, Hkv, d, F, V, G, NQKV;
  float eps;
  int qk_norm;
  int max_batch, page_size, max_pos, num_kv_pages, max_pages_per_seq;
  int attn_slots, attn_spg, tpp;      // slots per layer, slots per KV group, tokens per smem page
  int qkv_tasks_per_group;            // QKV tasks of one KV group's heads (G q + k + v)
  int kp[4];                          // page columns per op class
  int kchunk[4];                      // split-K columns per op class (0 = unsplit)
  float *kpart;                       // [parts][maxB][rows] split-K partials: QKV, down
  uint32_t *tile_ctr;                 // split-K parts done per 16-row tile: QKV, down
  int x_cap;                          // bytes of the activation staging area
  int page_bytes, n_pages;
  int off_look, off_slots, off_red, off_out, out_bytes, off_x, off_pages;  // smem carve-up
  int out_stride;                     // floats per sequence in an output buffer (16 x row tiles)
  int n_tasks;
  int ev_embed, ev_layer0, ev_per_layer;   // event numbering
  int n_ffn_parts;                         // gate/up events per layer (split-K parts of down)
  int n_o_parts, o_groups;                 // split-K parts of the O projection, KV groups per part
  int n_lm_tasks;
  long long wait_limit_ns;
  int n_out;                          // compute -> storer output buffers in use (<= kOutSlots)
  int attn_mma;                       // 1: attention on mma.sync tiles over swizzled K/V pages
                                      //    copied by TMA tensor copies (head_dim 64 or 128)
  const void *kvmaps;                 // CUtensorMap[2 L]: K then V of each layer (attn_mma)
  int w4;                             // 1: the projections (not the LM head) are packed 4-bit
  int kv_tasks;                       // 1: K/V of the step are appended by T_KVAPP tasks
                                      //    before any attention reads the cache (prefill plans)
  int tile_rows;                      // rows per row tile: 16 (mma.sync) or kTcRows (tcgen05)

  // tensor-core GEMV path (tc = 1): every GEMV task runs on tcgen05 tiles
  int tm;                             // 1: mma.sync GEMV pages staged in tensor memory
  int tc;
  int tc_bpad;                        // sequences per half of the MMA's N (max_batch rounded to 8)
  int tc_n;                           // MMA N = 2 * tc_bpad: bf16 hi rows, then lo rows
  int tc_kc;                          // weight page columns (a multiple of 64)
  int tc_kx;                          // staged activation chunk columns (a multiple of tc_kc)
  int tc_kt[8];                       // split-K part columns per task type (0: unsplit)
  const void *tmaps;                  // CUtensorMap[L * 7 + 1], 128 B each (LM head last)
  float *ssq_attn;                    // [H/128][maxB] sums of h^2 per 128 rows: QKV / LM head input
  float *ssq_mlp;                     // [H/128][maxB] the same for the gate/up input
  // the GEMV inputs as the tensor cores read them, written once by their
  // producers: bf16 [2 * tc_bpad][K] (rows 0..bpad-1: high halves of x * g,
  // rows bpad..: low halves), copied per chunk by a TMA tensor copy
  __nv_bfloat16 *xs[4];               // XS_ATTN (h * g_attn / g_final), XS_MLP (h * g_mlp), XS_O, XS_U
  int xs_map0;                        // tensor map of xs[0]; xs[i] uses xs_map0 + i
  float *kpart2;                      // [parts][maxB][2F] split-K partials of gate/up
  uint32_t *tile_ctr2;                // [F/16 + 1] split-K parts done per gate/up row tile
  // solidified schedule (NULL: the global ticket queue): CTA c runs tasks
  // sched[sched_off[c] .. sched_off[c + 1]) in that (ascending) order
  const int *sched;
  const int *sched_off;
  float *kpart_o;                     // [parts][maxB][H] split-K partials of the O projection
  uint32_t *tile_ctr_o;               // [H/16 + 1] split-K parts done per O row tile

  // per step
  uint32_t epoch;
  int batch;
  int chunk_seq;              // >= 0: a prompt chunk of one sequence: row b is that sequence's
                              //       token at position chunk_pos0 + b (block-table row chunk_seq)
  int chunk_pos0;
  int task_begin, task_end;   // launch covers tickets mapped onto [begin, end)
  int mode;
  const int32_t *ids, *pos;
  int32_t *out_ids, *out_pos;
  float *out_logits, *hidden_dump;
  unsigned long long *trace;  // optional [n_tasks][8] timeline
  const int32_t *block_table;
  __nv_bfloat16 *k_pages[MK_MAX_LAYERS];
  __nv_bfloat16 *v_pages[MK_MAX_LAYERS];
};

// event numbering helpers (host and device)
__host__ __device__ inline int ev_attn_ready(const Params &p, int l, int g) {
  return p.ev_layer0 + l * p.ev_per_layer + g;
}
// attention of the KV groups of O-projection part `part` is complete (o ready)
__host__ __device__ inline int ev_o_ready(const Params &p, int l, int part) {
  return p.ev_layer0 + l * p.ev_per_layer + p.Hkv + part;
}
__host__ __device__ inline int ev_oproj(const Params &p, int l) {
  return p.ev_layer0 + l * p.ev_per_layer + p.Hkv + p.n_o_parts;
}
// gate/up rows of down-projection part `part` (its K range) are complete
__host__ __device__ inline int ev_gateup(const Params &p, int l, int part) {
  return p.ev_layer0 + l * p.ev_per_layer + p.Hkv + p.n_o_parts + 1 + part;
}
__host__ __device__ inline int ev_down(const Params &p, int l) {
  return p.ev_layer0 + l * p.ev_per_layer + p.Hkv + p.n_o_parts + 1 + p.n_ffn_parts;
}
// prefill plans: the K/V of KV group g of every row are in the cache
__host__ __device__ inline int ev_kv_ready(const Params &p, int l, int g) {
  return p.ev_layer0 + l * p.ev_per_layer + p.Hkv + p.n_o_parts + 2 + p.n_ffn_parts + g;
}
// what an attention chunk of KV group g waits for, and how many completions
__host__ __device__ inline int ev_attn_input(const Params &p, int l, int g) {
  return p.kv_tasks ? ev_kv_ready(p, l, g) : ev_attn_ready(p, l, g);
}
__host__ __device__ inline int attn_input_count(const Params &p) {
  return p.kv_tasks ? 1 : p.qkv_tasks_per_group;
}

// Tensor-core path: the staged-input buffers (Params::xs)
enum XsKind : int { XS_ATTN = 0, XS_MLP = 1, XS_O = 2, XS_U = 3 };

// Tensor map of weight matrix j (0 wq, 1 wk, 2 wv, 3 wo, 4 w_gate, 5 w_up,
// 6 w_down) of layer l; the LM head's is the last.
__host__ __device__ inline int tc_map_index(int l, int j) { return l * kTcMatsPerLayer + j; }

// Batch n-tiles of a GEMV: each mma n-tile carries 4 sequences, the bf16
// high parts of their activations in columns 0..3 and the low parts in
// columns 4..7, so one mma covers both halves.  Row tiles per task shrink as
// n-tiles grow, which keeps the accumulators in registers.
__host__ __device__ inline int n_tiles_for(int batch) { return batch <= 4 ? 1 : (batch <= 8 ? 2 : 4); }
__host__ __device__ inline int max_mtiles_for(int batch) { return kMaxMTiles / n_tiles_for(batch); }

// smem pitch of one row of a 16-row weight page, in bytes: rounded to 128
// and offset by 64 so rows g and g+1 fall in opposite halves of the 32 banks
// (conflict-free 16-byte fragment loads).
__host__ __device__ inline int row_pitch_bytes(int cols) {
  return ((cols * 2 + 127) / 128) * 128 + 64;
}

// 4-bit pages: one packed block per 16 rows x 1024 columns
constexpr int kW4PageBlocks = 4;                   // a page: up to 4096 columns of one row tile
constexpr int kW4PageBytes = kW4PageBlocks * MK_W4_BLOCK_BYTES;
__host__ __device__ inline bool is_w4_task(int w4, uint8_t type) { return w4 && type != T_LMHEAD; }

// Staged activation: fp32 rows, pitch rounded to 128 B and offset by 16 B so
// the fragments of consecutive sequences fall on complementary banks.
__host__ __device__ inline int x_row_bytes(int cols) { return ((cols * 4 + 127) / 128) * 128 + 16; }

// ---- plan layout (mk_layout.cu) --------------------------------------------
struct LayoutOptions {
  int max_batch = 1;
  int page_size = 16;
  int num_ctas = 0;             // 0: one per SM
  int max_page_cols = 0;        // 0: kMaxPageCols
  bool o_split = false;         // O projection in two K parts of whole KV groups
  int gemv_path = 0;            // 0 automatic, 1 mma.sync pages, 2 tcgen05 tiles, 3 mma.sync pages through tensor memory
  int schedule = 0;             // 0 automatic (solidified), 1 solidified per-CTA task lists, 2 dynamic ticket queue
  bool prefill = false;         // K/V appended by their own tasks (prompt chunks of one sequence)
  bool w4 = false;              // 4-bit projections (packed, MK_W4_BLOCK_BYTES blocks)
  int attn_path = 0;            // 0 automatic / 1 CUDA-core FMA, 2 mma.sync tiles (d 64, 128)
  int rows_per_task[5] = {0, 0, 0, 0, 0};
  long long wait_limit_ns = 2000000000LL;
  bool debug_unsatisfiable_dep = false;
};
struct OpRange {
  int begin, end;   // task indices of one operator (per-operator launches)
};
struct Layout {
  Params p;                     // static kernel parameters (no pointers bound)
  int grid = 0, smem = 0, n_events = 0;
  int rows[5] = {0, 0, 0, 0, 0};   // rows per task: QKV, O, gate/up, down, LM head
  std::vector<Task> tasks;
  std::vector<OpRange> ops;
  std::vector<float2> rope;     // [max_seq_len][d/2] (cos, sin)
  // workspace byte offsets and size; counter words
  size_t o_h = 0, o_qkv = 0, o_part = 0, o_o = 0, o_u = 0, o_arg = 0, o_kpart = 0;
  size_t o_kpart2 = 0, o_kpart_o = 0, o_ssq_attn = 0, o_ssq_mlp = 0;
  size_t o_xs[4] = {0, 0, 0, 0};
  size_t ws_bytes = 0;
  size_t comb_words = 0, tile_words = 0, tile2_words = 0, tile_o_words = 0, sync_words = 0;
  int n_maps = 0;                      // tensor maps the tensor-core path needs (0: none)
  int first_lm_task = 0;               // task index of the first LM-head task
  // solidified schedule (empty: dynamic queue): task indices per CTA, and
  // the CTA's first entry (grid + 1 offsets)
  std::vector<int> sched, sched_off;
  int splits[5] = {1, 1, 1, 1, 1};     // split-K parts: QKV, O, gate/up, down, LM head
};
int validate_config(const mk_model_config &c, std::string &err);
int build_layout(const mk_model_config &c, const LayoutOptions &o, int nsm, int smem_optin,
                 Layout &out, std::string &err);
void bind_workspace(const Layout &lay, char *ws, uint32_t *sync, Params &p);
// Fill every task's operand pointers (weights, norm gains) from `w`.
void bind_task_operands(const mk_model_config &c, const mk_weights &w, std::vector<Task> &tasks);
// Encode the tensor maps of every weight matrix and of the staged-input
// buffers (lay.n_maps of them, 128 bytes each) into `out` for the
// tensor-core path; `ws` is the workspace the plan binds.  Needs the CUDA
// driver.
int encode_weight_maps(const mk_model_config &c, const mk_weights &w, const Layout &lay,
                       const char *ws, std::vector<unsigned char> &out, std::string &err);

cudaError_t launch_step(const Params &p, int grid, int smem, bool cooperative,
                        cudaStream_t stream);
// Allow the kernel the device's opt-in shared memory (capped at kMaxSmem).
cudaError_t configure_kernel(int smem_optin);
// The kernel variant (kVar* bits) a plan's parameters select.
int kernel_variant(const Params &p);
void set_last_error(const char *msg);  // message returned by mk_last_error()

// Tensor maps of a KV cache for the mma.sync attention: per layer, K then V,
// each a 2-D map over [num_pages * n_kv_heads * page, head_dim] bf16 with
// boxes of 64 dims x page rows, 128-byte swizzle.  Needs the CUDA driver.
int encode_kv_maps(const mk_model_config &c, const mk_kv_cache &kv, int page_size,
                   std::vector<unsigned char> &out, std::string &err);

}  // namespace mk
