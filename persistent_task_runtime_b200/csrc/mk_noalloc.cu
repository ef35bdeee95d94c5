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
// place its scratch comes from differs.  A call builds the plan layout on the
// host and uploads the task array and the RoPE table into the array unless
// the previous upload on this device was for the same model, weights, batch,
// page size and device (then it reuses them); every call zeroes the counters
// and the argmax slots, launches, synchronizes and returns the device status.
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
bool g_configured[kMaxDevices] = {};

// What the array holds on one device: the layout last uploaded into it and
// the inputs it was built from.  A call with the same key reuses the task
// array and the RoPE table already in the array.
struct Uploaded {
  bool valid = false;
  mk_model_config cfg{};
  int page = 0, batch = 0, nsm = 0, smem_optin = 0;
  std::vector<const void *> ptrs;   // every weight pointer, in a fixed order
  mk::Layout lay;
  size_t o_tasks = 0, o_rope = 0, o_ws = 0, o_sync = 0, o_maps = 0, o_kvmaps = 0;
  std::vector<const void *> kv_key;         // the KV cache whose tensor maps the array holds
  std::vector<unsigned char> kv_maps_host;
};
Uploaded g_up[kMaxDevices];

std::vector<const void *> weight_ptrs(const mk_model_config &c, const mk_weights &w) {
  std::vector<const void *> v = {w.embed, w.final_norm, w.lm_head};
  for (int l = 0; l < c.n_layers; ++l) {
    const mk_layer_weights &s = w.layers[l];
    v.insert(v.end(), {s.attn_norm, s.wq, s.wk, s.wv, s.q_norm, s.k_norm, s.wo, s.mlp_norm,
                       s.w_gate, s.w_up, s.w_down});
    if (w.w4_layers != nullptr)
      for (int j = 0; j < 7; ++j) v.push_back(w.w4_layers[l].q[j]);
  }
  v.push_back(w.w4_layers != nullptr ? w.w4_layers : nullptr);
  return v;
}

int nfail(int code, const char *msg) {
  mk::set_last_error(msg);
  return code;
}

inline size_t align_up_z(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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
  const int L = c.n_layers, P = kv_page_size, B = a->batch;
  {
    std::string verr;
    const int vrc = mk::validate_config(c, verr);
    if (vrc) return nfail(vrc, verr.c_str());
  }
  if (P < 16 || P % 16) return nfail(MK_ERR_INVALID_ARG, "kv_page_size must be a multiple of 16");
  if (B < 1 || B > MK_MAX_BATCH) return nfail(MK_ERR_INVALID_ARG, "batch outside 1..16");
  if (a->mode != MK_MODE_MEGAKERNEL)
    return nfail(MK_ERR_INVALID_ARG, "only MK_MODE_MEGAKERNEL is available without allocation");
  if (a->d_trace != nullptr)
    return nfail(MK_ERR_INVALID_ARG,
                 "d_trace is not available without a plan (its size is the plan's task count)");
  if (a->d_ids == nullptr || a->d_pos == nullptr || a->d_out_ids == nullptr ||
      a->kv->k_pages == nullptr || a->kv->v_pages == nullptr || a->kv->block_table == nullptr ||
      a->kv->num_pages < 1 || a->kv->max_pages_per_seq < 1)
    return nfail(MK_ERR_INVALID_ARG, "a step input, output or KV-cache pointer is NULL");
  const void *top[] = {w->embed, w->final_norm, w->lm_head, a->kv->block_table};
  for (const void *q : top)
    if (q == nullptr || !aligned16(q)) return nfail(MK_ERR_INVALID_ARG, "NULL or unaligned pointer");
  for (int l = 0; l < L; ++l) {
    const mk_layer_weights &s = w->layers[l];
    const void *ps[] = {s.attn_norm, s.mlp_norm, a->kv->k_pages[l], a->kv->v_pages[l], s.wq,
                        s.wk, s.wv, s.wo, s.w_gate, s.w_up, s.w_down};
    // (4-bit weights: the projections come from w4_layers)
    const int np = w->w4_layers != nullptr ? 4 : 11;
    for (int i = 0; i < np; ++i)
      if (ps[i] == nullptr || !aligned16(ps[i]))
        return nfail(MK_ERR_INVALID_ARG, "NULL or unaligned weight / KV pointer");
    if (w->w4_layers != nullptr)
      for (int j = 0; j < 7; ++j)
        if (w->w4_layers[l].q[j] == nullptr || !aligned16(w->w4_layers[l].q[j]))
          return nfail(MK_ERR_INVALID_ARG, "NULL or unaligned 4-bit matrix");
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

  std::lock_guard<std::mutex> lock(g_mu);
  // ---- once per device: the array's device address, the kernel's smem cap
  if (g_scratch_addr[dev] == nullptr) {
    void *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return nfail(MK_ERR_CUDA, "cudaGetSymbolAddress of the scratch array failed");
    g_scratch_addr[dev] = ptr;
  }
  if (!g_configured[dev]) {
    if (mk::configure_kernel(smem_optin) != cudaSuccess)
      return nfail(MK_ERR_CUDA, "setting the kernel's shared-memory limit failed");
    g_configured[dev] = true;
  }
  char *base = static_cast<char *>(g_scratch_addr[dev]);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // ---- the layout of a plan built for max_batch = B with default options:
  // built and uploaded unless the array already holds it
  Uploaded &up = g_up[dev];
  std::vector<const void *> ptrs = weight_ptrs(c, *w);
  const bool same = up.valid && std::memcmp(&up.cfg, &c, sizeof(c)) == 0 && up.page == P &&
                    up.batch == B && up.nsm == nsm && up.smem_optin == smem_optin &&
                    up.ptrs == ptrs;
  if (!same) {
    up.valid = false;
    mk::LayoutOptions lo;
    lo.max_batch = B;
    lo.page_size = P;
    lo.w4 = w->w4_layers != nullptr;
    lo.schedule = 2;   // the dynamic queue: the scratch array holds no per-CTA lists
    std::string err;
    const int rc = mk::build_layout(c, lo, nsm, smem_optin, up.lay, err);
    if (rc) return nfail(rc, err.c_str());
    mk::bind_task_operands(c, *w, up.lay.tasks);
    // ---- layout inside the static array -----------------------------------
    size_t off = 0;
    auto carve = [&](size_t bytes) {
      const size_t at = off;
      off = align_up_z(off + bytes, 256);
      return at;
    };
    up.o_tasks = carve(up.lay.tasks.size() * sizeof(Task));
    up.o_rope = carve(up.lay.rope.size() * sizeof(float2));
    up.o_ws = carve(up.lay.ws_bytes);
    up.o_sync = carve(up.lay.sync_words * sizeof(uint32_t));
    std::vector<unsigned char> maps;   // tensor maps of the tensor-core path (or none)
    {
      std::string merr;
      const int mrc = mk::encode_weight_maps(c, *w, up.lay, base + up.o_ws, maps, merr);
      if (mrc) return nfail(mrc, merr.c_str());
    }
    up.o_maps = carve(maps.size());
    up.o_kvmaps = carve(up.lay.p.attn_mma ? static_cast<size_t>(2 * c.n_layers) * 128 : 0);
    up.kv_key.clear();
    if (off > MK_NOALLOC_SCRATCH_BYTES) {
      char msg[256];
      snprintf(msg, sizeof(msg),
               "this model/batch/max_seq_len needs %zu bytes of scratch; the no-allocation entry "
               "point has %u (MK_NOALLOC_SCRATCH_BYTES)",
               off, static_cast<unsigned>(MK_NOALLOC_SCRATCH_BYTES));
      return nfail(MK_ERR_UNSUPPORTED, msg);
    }
    if (cudaMemcpyAsync(base + up.o_tasks, up.lay.tasks.data(), up.lay.tasks.size() * sizeof(Task),
                        cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(base + up.o_rope, up.lay.rope.data(), up.lay.rope.size() * sizeof(float2),
                        cudaMemcpyHostToDevice, s) != cudaSuccess ||
        (!maps.empty() && cudaMemcpyAsync(base + up.o_maps, maps.data(), maps.size(),
                                          cudaMemcpyHostToDevice, s) != cudaSuccess))
      return nfail(MK_ERR_CUDA, "uploading the step's tables into the scratch array failed");
    up.cfg = c;
    up.page = P;
    up.batch = B;
    up.nsm = nsm;
    up.smem_optin = smem_optin;
    up.ptrs = std::move(ptrs);
    up.valid = true;
  }
  // the attention's tensor maps of this call's KV cache (re-encoded when the
  // cache differs from the previous call's)
  if (up.lay.p.attn_mma) {
    std::vector<const void *> key;
    key.push_back(reinterpret_cast<const void *>(static_cast<intptr_t>(a->kv->num_pages)));
    for (int l = 0; l < L; ++l) {
      key.push_back(a->kv->k_pages[l]);
      key.push_back(a->kv->v_pages[l]);
    }
    if (key != up.kv_key) {
      std::string kerr;
      const int krc = mk::encode_kv_maps(c, *a->kv, P, up.kv_maps_host, kerr);
      if (krc) return nfail(krc, kerr.c_str());
      if (cudaMemcpyAsync(base + up.o_kvmaps, up.kv_maps_host.data(), up.kv_maps_host.size(),
                          cudaMemcpyHostToDevice, s) != cudaSuccess) {
        up.valid = false;
        return nfail(MK_ERR_CUDA, "uploading the KV tensor maps into the scratch array failed");
      }
      up.kv_key = std::move(key);
    }
  }
  const mk::Layout &lay = up.lay;
  Params p = lay.p;
  const int grid = lay.grid, smem = lay.smem;
  const size_t o_tasks = up.o_tasks, o_rope = up.o_rope, o_ws = up.o_ws, o_sync = up.o_sync;
  // the counters and the argmax slots start every call at zero
  if (cudaMemsetAsync(base + o_ws + lay.o_arg, 0, sizeof(unsigned long long) * B, s) != cudaSuccess ||
      cudaMemsetAsync(base + o_sync, 0, lay.sync_words * sizeof(uint32_t), s) != cudaSuccess) {
    up.valid = false;
    return nfail(MK_ERR_CUDA, "clearing the counters in the scratch array failed");
  }

  p.tasks = reinterpret_cast<const Task *>(base + o_tasks);
  p.rope_cs = reinterpret_cast<const float2 *>(base + o_rope);
  p.tmaps = base + up.o_maps;
  p.kvmaps = up.lay.p.attn_mma ? base + up.o_kvmaps : nullptr;
  mk::bind_workspace(lay, base + o_ws, reinterpret_cast<uint32_t *>(base + o_sync), p);
  p.embed = static_cast<const __nv_bfloat16 *>(w->embed);

  p.epoch = 1;  // counters were just zeroed
  p.batch = B;
  p.chunk_seq = -1;
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
