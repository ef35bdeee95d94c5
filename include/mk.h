/*
 * mk.h -- C ABI of the B200 decode megakernel.
 *
 * One call of mk_decode_step() runs one whole greedy decode step of a
 * Qwen3-style transformer decoder (embedding gather, then per layer RMSNorm ->
 * QKV projection -> QK-norm + RoPE + KV append -> paged attention -> O
 * projection + residual -> RMSNorm -> SwiGLU MLP + residual, then final
 * RMSNorm -> LM head -> argmax) as ONE persistent kernel launch: one CTA per
 * SM, tasks taken from an in-GPU queue and released by dependency counters,
 * with no host round trip inside the step.
 *
 * Sources: the mega-kernel execution model and the GPU-internal event-driven
 * task dispatch follow the MPK write-up, "2.1 Mega-Kernel执行模型" (task
 * descriptors, events with trigger/required counts); the paged shared-memory
 * allocation and the overlap of the next task's pre-load with the current
 * task's compute follow its "3.1 分页共享内存管理" and "3.2 任务预取与流水线";
 * warp roles (loader / consumer / storer) follow the Ada-MK summary,
 * "Methodik", Phase II ("Warp-Spezialisierung"); the decoder it runs is the
 * "Transformer-Decoder und LM-Head" of the same summary's Phase I.  None of the
 * pages defines an interface; this one is the library's own.
 *
 * Conventions for every function below:
 *   - Pointers named d_* (and every pointer inside mk_weights / mk_kv_cache)
 *     are CUDA device pointers on the plan's device; h_* are host pointers.
 *   - bf16 = IEEE bfloat16 stored as 2 bytes.  Weight matrices are row-major
 *     [out, in] (nn.Linear convention): y = W x.
 *   - Every device pointer must be 16-byte aligned.
 *   - The caller owns all weights, the KV cache, the block table and all step
 *     inputs/outputs; the plan only reads/writes them during a step.  The plan
 *     owns its task array, counters and workspace and frees them in
 *     mk_plan_destroy().
 *   - Return values: MK_OK (0) or a negative MK_ERR_* code.  Argument errors
 *     are detected on the host before any launch and leave the plan
 *     unchanged; mk_last_error() then describes the problem.
 *   - A plan serves one stream at a time and is not thread-safe.
 */
#ifndef MK_H_
#define MK_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MK_API __attribute__((visibility("default")))
#else
#define MK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MK_OK 0
#define MK_ERR_INVALID_ARG (-1) /* bad pointer / size / alignment (host)      */
#define MK_ERR_UNSUPPORTED (-2) /* valid but not supported shape (host)       */
#define MK_ERR_CUDA (-3)        /* a CUDA runtime call failed (host)          */
#define MK_ERR_RANGE (-4)       /* device: token id >= vocab, position out of
                                   range, or block-table entry out of range  */
#define MK_ERR_TIMEOUT (-5)     /* device: a dependency wait exceeded the
                                   plan's wait limit; the step was abandoned  */
#define MK_ERR_STATE (-6)       /* the plan holds an unread/uncleared device
                                   error; call mk_plan_reset()                */

#define MK_MAX_LAYERS 128
#define MK_MAX_BATCH 16

/* Model shape.  hidden, n_q_heads*head_dim and ffn must be multiples of 8;
 * head_dim one of 32, 64, 128; n_q_heads a multiple of n_kv_heads with
 * at most 8 query heads per KV head.  Other shapes: MK_ERR_UNSUPPORTED. */
typedef struct {
  int n_layers;     /* 1 .. MK_MAX_LAYERS                                   */
  int hidden;       /* H                                                    */
  int n_q_heads;    /* Hq                                                   */
  int n_kv_heads;   /* Hkv                                                  */
  int head_dim;     /* d                                                    */
  int ffn;          /* F (SwiGLU inner width)                               */
  int vocab;        /* V                                                    */
  float rms_eps;    /* epsilon of every RMSNorm                             */
  float rope_theta; /* RoPE base; pair i turns by pos * theta^(-2i/d),
                       pairing element i with i + d/2                       */
  int qk_norm;      /* 1: per-head RMSNorm of q and k before RoPE           */
  int max_seq_len;  /* positions must satisfy 0 <= pos < max_seq_len        */
} mk_model_config;

/* Per-layer weights, all bf16 device pointers:
 *   attn_norm [H], wq [Hq*d, H], wk [Hkv*d, H], wv [Hkv*d, H],
 *   q_norm [d], k_norm [d] (ignored when qk_norm == 0), wo [H, Hq*d],
 *   mlp_norm [H], w_gate [F, H], w_up [F, H], w_down [H, F]. */
typedef struct {
  const void *attn_norm, *wq, *wk, *wv, *q_norm, *k_norm, *wo, *mlp_norm,
      *w_gate, *w_up, *w_down;
} mk_layer_weights;

/* 4-bit weights (W4A16; the Ada-MK summary's GPTQ-W4A16, "Quantisierungs-
 * bewusste Optimierung").  A matrix W [rows, cols] is given as codes
 * c[r][k] in 0..15 and bf16 scales s[r][k / 128]; it stands for the bf16
 * matrix bf16_rn(s[r][k / 128] * (c[r][k] - 8)).  cols must be a multiple of
 * MK_W4_BLOCK_COLS.  The kernel reads it in the layout mk_w4_pack writes:
 * per 16 rows (a row tile; missing rows are code 8, scale 0) and 1024
 * columns, one MK_W4_BLOCK_BYTES block = 8 x 16 scales (group-major) then
 * 32 sub-blocks of 32 columns; a sub-block holds, for each lane (g, q) of an
 * mma.sync warp (lane = 4 g + q), the 8 codes of row g and then of row g + 8
 * at columns 8 q .. 8 q + 7, two codes per 16-bit half so that shifting a
 * word by 4 k and masking 0x000F000F leaves the codes of columns 2 k and
 * 2 k + 1 -- the order in which the tensor-core fragments consume them. */
#define MK_W4_GROUP 128
#define MK_W4_BLOCK_COLS 1024
#define MK_W4_BLOCK_BYTES 8448
typedef struct {
  const void *q[7];       /* packed wq, wk, wv, wo, w_gate, w_up, w_down    */
} mk_w4_layer_weights;

/* embed [V, H], final_norm [H], lm_head [V, H] (bf16 device pointers; embed
 * and lm_head may be the same pointer).  `layers` is a HOST array of
 * n_layers entries.  The plan copies the pointers, not the weights: the
 * weights must stay allocated and unchanged for the plan's lifetime.
 * w4_layers: NULL for bf16 projections; else a HOST array of n_layers
 * packed 4-bit layers, whose matrices replace the bf16 ones of `layers`
 * (which may then be NULL; the norms still come from `layers`). */
typedef struct {
  const void *embed;
  const mk_layer_weights *layers;
  const void *final_norm;
  const void *lm_head;
  const mk_w4_layer_weights *w4_layers;
} mk_weights;

/* Bytes of a packed 4-bit matrix of rows x cols (cols a multiple of 1024),
 * or -1 for an unsupported size. */
MK_API int64_t mk_w4_packed_bytes(int rows, int cols);
/* Pack a 4-bit matrix (HOST memory, no GPU): codes uint8 [rows][cols]
 * (0..15), scales bf16 [rows][cols / 128] -> `packed`
 * (mk_w4_packed_bytes(rows, cols) bytes; copy it to the device yourself).
 * MK_ERR_INVALID_ARG for NULL pointers, a code above 15 or a size
 * mk_w4_packed_bytes rejects. */
MK_API int mk_w4_pack(const uint8_t *codes, const void *scales, int rows, int cols,
                      void *packed);

/* Paged KV cache.  For layer l, k_pages[l] and v_pages[l] point to bf16
 * arrays [num_pages, n_kv_heads, page_size, head_dim] (head-major inside a
 * page, so one head's page is contiguous).  k_pages / v_pages are HOST
 * arrays of n_layers device pointers.  block_table is a device int32 array
 * [max_batch, max_pages_per_seq]: sequence b's position p lives in physical
 * page block_table[b*max_pages_per_seq + p/page_size], slot p%page_size.
 * Every page a step touches must already be mapped. */
typedef struct {
  void *const *k_pages;
  void *const *v_pages;
  const int32_t *block_table;
  int num_pages;
  int max_pages_per_seq;
} mk_kv_cache;

/* Plan options (pass NULL to mk_plan_create_ex for the defaults). */
typedef struct {
  int max_batch;          /* 1 .. MK_MAX_BATCH (default 1)                  */
  int kv_page_size;       /* tokens per KV page, multiple of 16 (default 16) */
  int num_ctas;           /* persistent CTAs; 0 = one per SM                 */
  int64_t wait_limit_ns;  /* bound on every in-kernel wait (default 2 s)    */
  int rows_per_task[5];   /* override rows per task for QKV, O, gate/up (per
                             matrix), down, LM head; 0 = automatic          */
  int debug_unsatisfiable_dep; /* fault-injection for tests: the first QKV
                             task waits for one completion more than can
                             ever happen, so the step must end in
                             MK_ERR_TIMEOUT after wait_limit_ns             */
  int max_page_cols;      /* widest weight page, in columns: 32 .. 2048, a
                             multiple of 32; 0 = 2048.  A page is 16 weight
                             rows; wider pages mean fewer ring hand-offs
                             per byte, narrower ones more pages in flight  */
  int o_split;            /* nonzero: split the O projection along K into two
                             parts of whole KV groups, each waiting only for
                             the attention of its groups (needs >= 2 KV heads
                             and >= 1024 columns per part); 0 = one part.
                             mma.sync path only                             */
  int gemv_path;          /* how the projections run: 0 = automatic (tensor
                             cores when max_batch >= 4 and the shape allows),
                             1 = warp-level mma.sync (the pre-tcgen05 tensor
                             core instruction) over 16-row weight pages,
                             2 = tcgen05 tensor cores over 128-row tiles: the
                             weights arrive by TMA tensor copies in the
                             swizzled layout the MMA reads, the activation is
                             staged as bf16 high/low halves, accumulators sit
                             in tensor memory.  2 needs head_dim 128 and
                             hidden, ffn and n_q_heads*head_dim multiples of
                             64 (else MK_ERR_UNSUPPORTED); rows_per_task,
                             max_page_cols and o_split apply to path 1 only.
                             3 = path 1 with its weight pages staged in
                             tensor memory: TMA copies 16-row pages in
                             512-column boxes, the loader copies each landed
                             page into tensor memory (tcgen05.cp) and frees
                             its shared memory, the compute warps read mma
                             A fragments back (tcgen05.ld), so more bytes
                             stay in flight per SM.  3 needs hidden, ffn and
                             n_q_heads*head_dim multiples of 512, no 4-bit
                             weights and no o_split                         */
  int schedule;           /* 0 = automatic: solidified; 1 = solidified: the
                             plan assigns each CTA its task list offline (list
                             scheduling in queue order under a cost model of
                             weight bytes per task; the Ada-MK summary's
                             offline path solidification) and each CTA runs
                             its list in order; 2 = dynamic: every CTA takes
                             the next task from one in-GPU ticket queue.
                             Per-operator modes and mk_decode_step_noalloc
                             always use the queue                           */
  int weight_bits;        /* 0: as the weights are given (mk_plan_describe:
                             bf16); 16: bf16 projections; 4: 4-bit (the
                             weights must carry w4_layers).  4-bit plans run
                             the mma.sync path (gemv_path 0 or 1); hidden,
                             ffn and n_q_heads*head_dim must be multiples
                             of 1024                                        */
  int prefill;            /* nonzero: the plan can also run prompt chunks
                             (mk_prefill_chunk).  Each layer then appends
                             the step's K/V in tasks of their own, one per
                             KV group, and the group's attention waits for
                             them, so a row may attend to positions that
                             other rows of the same launch write.  Decode
                             steps on such a plan give the same results    */
  int attn_path;          /* how attention runs: 0 = automatic (2 when
                             max_batch >= 2 and head_dim is 64 or 128, else
                             1); 1 = CUDA cores: fp32 FMA over K/V pages
                             bulk-copied into shared memory, three phases
                             per page; 2 = mma.sync tensor-core tiles: K/V
                             pages copied by TMA tensor copies with the
                             128-byte swizzle, each warp an online softmax
                             over its own 16-token slices (q.K and P.V as
                             m16n8k16 MMAs fed by ldmatrix), the warps
                             merged at the chunk's end (head_dim 64 or 128,
                             else MK_ERR_UNSUPPORTED)                       */
} mk_plan_options;

typedef struct mk_plan mk_plan;

/* Build a plan: validate the shape, tile every operator of every layer into
 * tasks with dependency counters, build the RoPE table (angles in double
 * precision), allocate and upload the task array, counters and workspace.
 * No kernel runs.  On success *out receives the plan. */
MK_API int mk_plan_create(const mk_model_config *cfg, const mk_weights *weights,
                   int max_batch, int kv_page_size, mk_plan **out);
MK_API int mk_plan_create_ex(const mk_model_config *cfg, const mk_weights *weights,
                      const mk_plan_options *opts, mk_plan **out);

/* Execution modes of a step. */
#define MK_MODE_MEGAKERNEL 0 /* one persistent cooperative launch            */
#define MK_MODE_PER_OP 1     /* the same task code, one launch per operator
                                (embed, then per layer QKV, attention, O,
                                gate/up, down, then LM head), ordered by the
                                stream instead of by in-GPU counters        */
#define MK_MODE_PER_OP_GRAPH 2 /* MK_MODE_PER_OP recorded once as a CUDA graph
                                and replayed.  The plan keeps the graphs of
                                the two most recent argument sets (pointers,
                                batch) and stream, and records a new one for
                                any other; every replay patches the step
                                counter into its kernel nodes.  Needs a
                                created stream (not the legacy default one);
                                a stream that is being captured is refused
                                by CUDA (MK_ERR_CUDA).                      */

/* Everything one step reads and writes. */
typedef struct {
  const int32_t *d_ids;   /* [batch] token fed by each sequence             */
  const int32_t *d_pos;   /* [batch] its position; K/V are written at pos and
                             attention covers positions 0..pos              */
  const mk_kv_cache *kv;  /* host struct, read during the call              */
  int batch;              /* 1 .. max_batch                                 */
  int32_t *d_out_ids;     /* [batch] argmax token (lowest index on ties);
                             may alias d_ids only if not read afterwards     */
  float *d_out_logits;    /* [batch, V] fp32, or NULL                       */
  int32_t *d_out_pos;     /* [batch] receives pos+1, or NULL                 */
  float *d_hidden;        /* [n_layers, batch, H] fp32 residual stream after
                             each layer (debug/parity), or NULL             */
  int mode;               /* MK_MODE_*                                      */
  uint64_t *d_trace;      /* per-task timeline, or NULL: [n_tasks][8] u64 =
                             {CTA index, loader: slot written, loader: last
                             page issued, compute: slot received, compute:
                             input event satisfied, compute: activation
                             staged, compute: done, storer: output released},
                             times in ns of the GPU global timer           */
} mk_step_args;

/* A chunk of one sequence's prompt: n_tokens consecutive tokens at positions
 * pos0 .. pos0 + n_tokens - 1, run as one launch in which row j is the
 * token at pos0 + j.  The multi-token form of the decode step: every
 * projection streams its weights once for the whole chunk, each row's K/V is
 * appended to the cache, and row j attends causally to positions
 * 0 .. pos0 + j (the MPK write-up, "2.2 混合任务启动机制", on running the
 * same task graph for other input shapes; the Ada-MK summary, "Methodik",
 * on prefill beside decode). */
typedef struct {
  const int32_t *d_ids;   /* [n_tokens] the chunk's token ids               */
  int n_tokens;           /* 1 .. max_batch                                 */
  int pos0;               /* position of the chunk's first token            */
  int seq;                /* the sequence: block-table row (0 .. max_batch-1)*/
  const mk_kv_cache *kv;
  int32_t *d_out_ids;     /* [n_tokens] argmax after each token (the last one
                             is the first generated token); may be NULL
                             without the LM head                            */
  float *d_out_logits;    /* [n_tokens, V] or NULL (needs with_lm_head)     */
  float *d_hidden;        /* [n_layers, n_tokens, H] residual stream after
                             each layer, or NULL                            */
  int with_lm_head;       /* 0: stop after the last layer (a chunk whose
                             logits nobody reads); 1: final norm, LM head and
                             argmax for every row                           */
} mk_prefill_args;

/* Enqueue one prompt chunk on `stream` (asynchronous, like mk_decode_step).
 * The plan must have been created with opts->prefill != 0 (else
 * MK_ERR_INVALID_ARG); other argument errors are MK_ERR_INVALID_ARG, found
 * before the launch.  Device errors go to mk_plan_status().  Chunks of one
 * prompt must run in order (pos0 = 0, T, 2T, ...). */
MK_API int mk_prefill_chunk(mk_plan *plan, const mk_prefill_args *args, void *stream);

/* Enqueue one decode step on `stream` (a cudaStream_t; NULL = legacy default
 * stream).  Asynchronous: device-side errors (MK_ERR_RANGE, MK_ERR_TIMEOUT)
 * are reported by mk_plan_status().  A step enqueued while the plan holds a
 * device error does nothing on the device. */
MK_API int mk_decode_step(mk_plan *plan, const int32_t *d_ids, const int32_t *d_pos,
                   const mk_kv_cache *kv, int batch, int32_t *d_out_ids,
                   float *d_out_logits, void *stream);
MK_API int mk_decode_step_ex(mk_plan *plan, const mk_step_args *args, void *stream);

/* The same step from HOST buffers: copies h_ids/h_pos to the device, runs
 * the step, copies the argmax ids (and logits if h_out_logits != NULL) back
 * and synchronizes `stream`.  Returns MK_OK or the device error code. */
MK_API int mk_decode_step_host(mk_plan *plan, const int32_t *h_ids,
                        const int32_t *h_pos, const mk_kv_cache *kv, int batch,
                        int32_t *h_out_ids, float *h_out_logits, void *stream);

/* Synchronize the device and return the device-side status of the plan:
 * MK_OK, MK_ERR_RANGE or MK_ERR_TIMEOUT.  The status is sticky until
 * mk_plan_reset(). */
MK_API int mk_plan_status(mk_plan *plan);

/* Details of the first device error: which task, which event, the value
 * seen.  `info` receives 4 int32. */
MK_API int mk_plan_error_info(mk_plan *plan, int32_t *info);

/* Synchronize, then clear all counters and the status so the plan can run
 * again (the caller's KV cache is not touched). */
MK_API int mk_plan_reset(mk_plan *plan);

/* Plan facts, for tests and benchmarks. */
typedef struct {
  int num_ctas, threads_per_cta, smem_bytes, n_pages, page_bytes;
  int n_tasks, n_events, attn_slots, tokens_per_smem_page;
  int rows_per_task[5];   /* QKV, O, gate/up, down, LM head                 */
  int page_cols[4];       /* columns per weight page: K=H, K=Hq*d, K=F, LM  */
  int64_t weight_bytes;   /* bytes of weights one step streams (excluding the
                             embedding rows)                                */
  /* task-graph facts (event k of layer l is 1 + l*events_per_layer + k:
     attn_ready[n_kv_heads], o_ready[o_parts], oproj, gateup[ffn_parts],
     down; event 0 is the embedding)                                      */
  int events_per_layer;
  int attn_slots_per_group; /* attention slots of one KV group per layer   */
  int qkv_tasks_per_group;  /* QKV tasks whose rows one KV group attends   */
  int ffn_parts, ffn_part_cols; /* split-K parts of the down projection and
                             columns per part (1 part: ffn_part_cols = ffn) */
  int o_parts, o_part_cols; /* the same for the O projection               */
  int gemv_path;          /* the path the plan uses: 1 mma.sync, 2 tcgen05,
                             3 mma.sync from tensor memory                  */
  int schedule;           /* 0 dynamic queue, 1 solidified per-CTA lists    */
  int prefill;            /* 1: created with the prefill option             */
  int weight_bits;        /* 16 bf16 or 4 (W4A16) projections              */
  int qkv_parts, gateup_parts; /* split-K parts of the QKV and gate/up
                             projections (tensor-core path; 1 otherwise)   */
  int attn_path;          /* 1 CUDA-core attention, 2 mma.sync tiles        */
} mk_plan_info_t;
MK_API int mk_plan_info(const mk_plan *plan, mk_plan_info_t *info);

/* Task records returned by mk_plan_describe (MK_TASK_RECORD_BYTES each;
 * for tests and tools, the layout may change between versions):
 *   byte 0 type (1 embed, 2 QKV, 3 attention, 4 O, 5 gate/up, 6 down,
 *   7 LM head), 1 row tiles, 2-3 layer, 4-7 first output row, 8-9 rows,
 *   10 split-K part, 11 split-K parts (0/1: none), 12-15 input event
 *   (0xffffffff: none; attention: resolved at run time), 16-19 completions
 *   of the input event per step, 20-23 output event (0xffffffff: none; a QKV
 *   task signals attn_ready of its head's KV group), 24-27 aux (QKV: 0 q,
 *   1 k, 2 v; attention: slot), 28-31 aux2 (QKV: head index over q, k, v),
 *   32-55 operand pointers (NULL in a described plan), 56-59 and 60-63
 *   tensor-map indices of the task's matrices (tensor-core path). */
#define MK_TASK_RECORD_BYTES 64

/* Describe, without any GPU, the plan mk_plan_create_ex(cfg, weights, opts)
 * would build on a device with `num_sms` SMs and `smem_optin` bytes of
 * opt-in shared memory per block: fills *info and, when `tasks` is not NULL
 * and `max_tasks` >= info->n_tasks, copies the task records.  Returns MK_OK,
 * or the error mk_plan_create_ex would return for the shape and options. */
MK_API int mk_plan_describe(const mk_model_config *cfg, const mk_plan_options *opts,
                            int num_sms, int smem_optin, mk_plan_info_t *info,
                            void *tasks, int64_t max_tasks);

/* The CTA each task of that plan runs on under a solidified schedule
 * (opts->schedule 0 or 1), without any GPU: cta_of_task[i] for i < n_tasks,
 * or -1 for every task when the plan uses the dynamic queue.  Each CTA runs
 * its tasks in ascending index order.  MK_ERR_INVALID_ARG if max_tasks is
 * below the plan's task count. */
MK_API int mk_plan_describe_schedule(const mk_model_config *cfg,
                                     const mk_plan_options *opts, int num_sms,
                                     int smem_optin, int32_t *cta_of_task,
                                     int64_t max_tasks);

/* Message of the last error on the calling thread ("" if none). */
MK_API const char *mk_last_error(void);

/* Free everything the plan owns (synchronizes first).  NULL is a no-op. */
MK_API void mk_plan_destroy(mk_plan *plan);

/* ---- Decode step without any device allocation ---------------------------
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot call cudaMalloc (a host that routes every device allocation
 * through its own pool, a memory-capped sandbox, a callback that must not
 * allocate).  It runs the same kernel as mk_decode_step() without a plan:
 * the task array, tables, activations and counters live in one file-scope
 * __device__ array of MK_NOALLOC_SCRATCH_BYTES, which every GPU that loads
 * this library holds until the process exits.  No cudaMalloc, cudaFree or
 * other allocating call is made.
 *
 * The caller passes the model, the weights, the KV page size and the step
 * exactly as for a plan built with max_batch = args->batch; args->mode must
 * be MK_MODE_MEGAKERNEL and args->d_trace NULL (MK_ERR_INVALID_ARG
 * otherwise: a trace buffer is sized by a plan's task count).  A call builds
 * the plan layout on the host and uploads its task array and RoPE table into
 * the array, unless the previous call on this device had the same model,
 * weight pointers, batch and page size (then both are reused; building them
 * costs tens of milliseconds of host time for an 8B-shaped model).  Every
 * call zeroes the counters, launches on `stream`, synchronizes it and
 * returns the device status (MK_OK, MK_ERR_RANGE, MK_ERR_TIMEOUT) or a host
 * error code.  A shape, batch or max_seq_len whose scratch would exceed the
 * array is rejected with MK_ERR_UNSUPPORTED and a message in
 * mk_last_error().
 *
 * Every call uses the same array and leaves the previous call's contents
 * behind: calls that overlap on the GPU (several streams or threads) race
 * and must not be issued.  The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress) and sets the kernel's
 * shared-memory limit; make that first call before any stream capture. */
#define MK_NOALLOC_SCRATCH_BYTES (16u << 20)
MK_API int mk_decode_step_noalloc(const mk_model_config *cfg,
                                  const mk_weights *weights, int kv_page_size,
                                  const mk_step_args *args, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* MK_H_ */
