// The persistent decode megakernel for sm_100a.
//
// One launch = one decode step.  Each CTA (one per SM) runs three roles:
//   warp 0      loader : pops task tickets from the global queue, resolves
//                        attention chunks, and streams each task's operands
//                        (weight tiles, KV pages) into a ring of shared-memory
//                        pages with 1-D bulk (TMA) copies.  Weights never
//                        depend on activations, so the loader runs ahead into
//                        the next tasks while the compute warps still wait for
//                        a dependency (MPK write-up, "3.2 任务预取与流水线":
//                        the next task's pre-load overlaps the current task).
//   warps 1..8  compute: wait for the task's input event (in-GPU event
//                        counters, MPK write-up "2.1 Mega-Kernel执行模型":
//                        trigger count vs. required count), stage the
//                        activation, and consume the pages (bf16 mma.sync for
//                        the projections, warp-shuffle online softmax for
//                        attention).
//   warp 9      storer : epilogues (residual add, SwiGLU, QK-norm + RoPE + KV
//                        append, split-attention combine, argmax) and the
//                        release of the task's output event.
// (Loader / consumer / storer roles: Ada-MK summary, "Methodik", Phase II.)
//
// Shared-memory pages are a ring guarded by mbarriers (full: TMA bytes landed;
// empty: all compute warps are done with the page) -- the paged shared memory
// of the MPK write-up, "3.1 分页共享内存管理", with the ring order standing in
// for its atomic page counter.
//
// Every wait is bounded by the plan's wait limit (globaltimer).  On expiry the
// waiting thread records MK_ERR_TIMEOUT and raises the global abort flag;
// every role polls that flag, the loader drains its in-flight bulk copies, and
// all CTAs return.

#include <float.h>
#include <math.h>

#include "mk_internal.h"

namespace mk {

// ============================================================================
// PTX helpers
// ============================================================================

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P1;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, P1;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 1-D bulk copy global -> this CTA's shared memory, completion on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_acq_rel() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t *p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;"
               : "=r"(old)
               : "l"(p), "r"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ void red_add_release(uint32_t *p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void compute_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kComputeThreads) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// fp32 -> (hi, lo) bf16 pair with hi + lo == x to ~2^-16 relative.
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16 &hi, __nv_bfloat16 &lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

__device__ __forceinline__ uint32_t pack2(__nv_bfloat16 a, __nv_bfloat16 b) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(a)) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// optional timeline: record k of task `idx`
__device__ __forceinline__ void trace_mark(const Params &p, int idx, int k) {
  if (p.trace != nullptr) p.trace[static_cast<size_t>(idx) * 8 + k] = gtimer();
}

// ============================================================================
// shared-memory control block
// ============================================================================

struct Ctl {
  uint64_t full[kMaxPages];
  uint64_t empty[kMaxPages];
  uint64_t slot_full[kTaskSlots];
  uint64_t slot_empty[kTaskSlots];
  uint64_t out_full[kOutSlots];
  uint64_t out_empty[kOutSlots];
  volatile int cta_abort;
  int skip;
  int flag[2];
  float rs[MK_MAX_BATCH];
  float red8[kComputeWarps][MK_MAX_BATCH];
};
static_assert(sizeof(Ctl) <= 1024, "control block exceeds its 1 KB slot");

// A popped task as the loader hands it to compute and storer (64 bytes).
struct Slot {
  Task t;
  int b, g, t0, t1;          // attention: sequence, KV head, token range
  int first_slot, n_chunks;  // attention: partial slots of (b, g)
  int idx;                   // task index (for error reports)
  int pad;
};
static_assert(sizeof(Slot) == 64, "slot must be 64 bytes");

// ============================================================================
// errors and bounded waits
// ============================================================================

__device__ void raise_error(const Params &p, int code, uint32_t a, uint32_t b, uint32_t c) {
  uint32_t *s = p.sync;
  if (atomicCAS(&s[S_STATUS], 0u, static_cast<uint32_t>(code)) == 0u) {
    s[S_INFO + 0] = a;
    s[S_INFO + 1] = b;
    s[S_INFO + 2] = c;
  }
  __threadfence();
  atomicExch(&s[S_ABORT], 1u);
}

__device__ __forceinline__ bool aborted(const Params &p, Ctl *ctl) {
  return ctl->cta_abort != 0 || ld_relaxed(p.sync + S_ABORT) != 0u;
}

// One thread: wait until mbarrier phase `parity` completed.  `scale` widens
// the limit for intra-CTA waits so that a stuck inter-CTA dependency is what
// reports the timeout.
__device__ bool wait_mbar(const Params &p, Ctl *ctl, uint64_t *bar, uint32_t parity,
                          uint32_t where, int scale) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 7u) == 7u) {
      if (aborted(p, ctl)) return false;
      const uint64_t now = gtimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > static_cast<uint64_t>(p.wait_limit_ns) * scale) {
        raise_error(p, MK_ERR_TIMEOUT, where, 0xfffffffeu, parity);
        return false;
      }
    }
  }
}

// One thread: wait until event `ev` reached epoch * count (acquire).
__device__ bool wait_event(const Params &p, Ctl *ctl, uint32_t ev, uint32_t count,
                           uint32_t task_idx) {
  if (ev == kNoEvent) return true;
  const uint32_t target = p.epoch * count;
  const uint32_t *ctr = p.sync + S_EVENTS + ev;
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    const uint32_t v = ld_relaxed(ctr);
    if (static_cast<int32_t>(v - target) >= 0) {
      fence_acq_rel();
      return true;
    }
    if ((it & 3u) == 3u) {
      if (aborted(p, ctl)) return false;
      const uint64_t now = gtimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > static_cast<uint64_t>(p.wait_limit_ns)) {
        raise_error(p, MK_ERR_TIMEOUT, task_idx, ev, v);
        return false;
      }
    }
  }
}

// Compute group (256 threads): thread 0 waits, the decision is shared through
// a double-buffered flag so every thread takes the same branch.
struct GroupSync {
  int k = 0;
  __device__ bool share(Ctl *ctl, int ctid, bool ok_leader) {
    if (ctid == 0) ctl->flag[k & 1] = ok_leader ? 1 : 0;
    compute_bar();
    const bool ok = ctl->flag[k & 1] != 0;
    ++k;
    return ok;
  }
};

// ============================================================================
// task geometry (shared by the loader and the compute warps)
// ============================================================================

struct Geo {
  int K;        // input width
  int kp;       // columns per weight page
  int kx;       // columns per staged activation chunk
  int whole;    // kx == K: the staged activation can be reused by later tasks
  int cls;      // OpK
};

__device__ __forceinline__ int x_bytes(int B, int cols) { return 2 * B * row_pitch_bytes(cols); }

__device__ Geo gemv_geo(const Params &p, const Task &t, int B) {
  Geo g;
  switch (t.type) {
    case T_OPROJ: g.K = p.Hq * p.d; g.cls = K_ATT; break;
    case T_DOWN: g.K = p.F; g.cls = K_FFN; break;
    case T_LMHEAD: g.K = p.H; g.cls = K_LM; break;
    default: g.K = p.H; g.cls = K_HID; break;
  }
  g.kp = p.kp[g.cls];
  if (x_bytes(B, g.K) <= p.x_cap) {
    g.kx = g.K;
    g.whole = 1;
  } else {
    int n = g.K / g.kp;
    while (n > 1 && x_bytes(B, n * g.kp) > p.x_cap) --n;
    g.kx = n * g.kp;
    g.whole = 0;
  }
  return g;
}

// Row `m`-tile of a GEMV task: weight matrix base, first row, valid rows.
__device__ __forceinline__ void gemv_tile(const Params &p, const Task &t, int m,
                                          const __nv_bfloat16 *&W, int &row, int &rows_valid) {
  const LayerW &lw = p.layers[t.layer < p.L ? t.layer : 0];
  int mm = m;
  switch (t.type) {
    case T_QKV: W = t.aux == 0 ? lw.wq : (t.aux == 1 ? lw.wk : lw.wv); break;
    case T_OPROJ: W = lw.wo; break;
    case T_DOWN: W = lw.w_down; break;
    case T_LMHEAD: W = p.lm_head; break;
    default: {  // gate/up: first half of the tiles read w_gate, second w_up
      const int nh = t.n_m >> 1;
      if (m < nh) {
        W = lw.w_gate;
      } else {
        W = lw.w_up;
        mm = m - nh;
      }
    }
  }
  row = static_cast<int>(t.row0) + 16 * mm;
  const int left = static_cast<int>(t.nrows) - 16 * mm;
  rows_valid = left < 16 ? (left > 0 ? left : 0) : 16;
}

// Attention split: how many smem pages per chunk so that this step's whole
// KV length, over all (sequence, KV head), fills about `attn_target` chunks.
// Lengths are clamped to [1, max_pos] so bad positions cannot blow it up
// (they are reported by the embedding task).
__device__ __forceinline__ int seq_len(const Params &p, int b) {
  int n = p.pos[b] + 1;
  return n < 1 ? 1 : (n > p.max_pos ? p.max_pos : n);
}

__device__ int attn_chunk_pages(const Params &p, int B) {
  int total = 0;
  for (int b = 0; b < B; ++b) total += (seq_len(p, b) + p.tpp - 1) / p.tpp;
  total *= p.Hkv;
  const int c = (total + p.attn_target - 1) / p.attn_target;
  return c < 1 ? 1 : c;
}

// Slot s -> (b, g, chunk token range, first slot of (b, g), chunks of (b, g)).
__device__ bool attn_resolve(const Params &p, int B, int s, Slot &o) {
  const int cp = attn_chunk_pages(p, B);
  const int span = cp * p.tpp;
  int base = 0;
  for (int b = 0; b < B; ++b) {
    const int len = seq_len(p, b);
    const int nb = (len + span - 1) / span;
    if (s < base + p.Hkv * nb) {
      const int r = s - base;
      o.b = b;
      o.g = r / nb;
      const int c = r % nb;
      o.t0 = c * span;
      o.t1 = min(len, o.t0 + span);
      o.first_slot = base + o.g * nb;
      o.n_chunks = nb;
      return true;
    }
    base += p.Hkv * nb;
  }
  o.b = -1;
  return false;
}

__device__ __forceinline__ int kv_phys_page(const Params &p, int b, int logical) {
  int lp = logical < p.max_pages_per_seq ? logical : p.max_pages_per_seq - 1;
  int ph = p.block_table[b * p.max_pages_per_seq + lp];
  return (ph >= 0 && ph < p.num_kv_pages) ? ph : -1;
}

// ============================================================================
// loader (warp 0)
// ============================================================================

__device__ void loader_main(const Params &p, Ctl *ctl, uint8_t *smem) {
  const int lane = threadIdx.x & 31;
  const uint64_t pol = l2_evict_first_policy();
  Slot *slots = reinterpret_cast<Slot *>(smem + p.off_slots);
  uint8_t *pages = smem + p.off_pages;
  const int B = p.batch;

  int pi = 0;
  uint32_t pe_par = 0;            // ring round parity
  uint32_t issued = 0, last_par = 0;
  int ts = 0;
  uint32_t ts_par = 0;
  bool ok = true;

  const int n_launch = p.task_end - p.task_begin;
  uint32_t next = 0;
  if (lane == 0) next = atomicAdd(p.sync + S_QUEUE, 1u);

  while (true) {
    uint32_t ticket = __shfl_sync(0xffffffffu, next, 0);
    const bool done = static_cast<int>(ticket) >= n_launch;
    if (!done && lane == 0) next = atomicAdd(p.sync + S_QUEUE, 1u);

    int okl = 1;
    if (lane == 0) okl = wait_mbar(p, ctl, &ctl->slot_empty[ts], ts_par ^ 1u, 0xfff00000u, 2);
    ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
    if (!ok) break;

    Slot &S = slots[ts];
    if (done) {
      if (lane == 0) {
        S.t.type = T_END;
        mbar_arrive(&ctl->slot_full[ts]);
      }
      break;
    }
    const int tix = p.task_begin + static_cast<int>(ticket);
    Task t = p.tasks[tix];
    Slot info;
    info.t = t;
    info.idx = tix;
    info.b = -1;
    if (t.type == T_ATTN) attn_resolve(p, B, static_cast<int>(t.aux), info);
    if (lane == 0) {
      S = info;
      mbar_arrive(&ctl->slot_full[ts]);
      if (p.trace != nullptr) {
        p.trace[static_cast<size_t>(tix) * 8] =
            blockIdx.x | (static_cast<unsigned long long>(t.type) << 32) |
            (static_cast<unsigned long long>(t.layer) << 40);
        trace_mark(p, tix, 1);
      }
    }
    if (++ts == kTaskSlots) {
      ts = 0;
      ts_par ^= 1u;
    }

    // ---- stream the task's operands into the page ring ----
    if (t.type == T_QKV || t.type == T_OPROJ || t.type == T_GATEUP || t.type == T_DOWN ||
        t.type == T_LMHEAD) {
      const Geo geo = gemv_geo(p, t, B);
      const int pitch = row_pitch_bytes(geo.kp);
      for (int xc0 = 0; xc0 < geo.K && ok; xc0 += geo.kx) {
        const int xend = min(geo.K, xc0 + geo.kx);
        for (int m = 0; m < t.n_m && ok; ++m) {
          const __nv_bfloat16 *W;
          int row, rv;
          gemv_tile(p, t, m, W, row, rv);
          for (int c0 = xc0; c0 < xend; c0 += geo.kp) {
            const int nc = min(geo.kp, xend - c0);
            if (lane == 0) okl = wait_mbar(p, ctl, &ctl->empty[pi], pe_par ^ 1u, 0xfff10000u, 2);
            ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
            if (!ok) break;
            uint8_t *pg = pages + static_cast<size_t>(pi) * p.page_bytes;
            if (lane == 0) mbar_arrive_expect_tx(&ctl->full[pi], static_cast<uint32_t>(rv * nc * 2));
            __syncwarp();
            if (lane < rv) {
              const __nv_bfloat16 *src = W + (static_cast<size_t>(row + lane) * geo.K + c0);
              bulk_load(pg + lane * pitch, src, static_cast<uint32_t>(nc * 2), &ctl->full[pi], pol);
            }
            issued |= 1u << pi;
            last_par = (last_par & ~(1u << pi)) | (pe_par << pi);
            if (++pi == p.n_pages) {
              pi = 0;
              pe_par ^= 1u;
            }
          }
        }
      }
    } else if (t.type == T_ATTN && info.b >= 0) {
      const int l = t.layer;
      const int P = p.page_size, d = p.d;
      const size_t kvpage_elems = static_cast<size_t>(P) * d;
      const uint32_t kvpage_bytes = static_cast<uint32_t>(kvpage_elems * 2);
      for (int tok0 = info.t0; tok0 < info.t1 && ok; tok0 += p.tpp) {
        const int ntok = min(p.tpp, info.t1 - tok0);
        const int nkv = (ntok + P - 1) / P;
        if (lane == 0) okl = wait_mbar(p, ctl, &ctl->empty[pi], pe_par ^ 1u, 0xfff20000u, 2);
        ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
        if (!ok) break;
        uint8_t *pg = pages + static_cast<size_t>(pi) * p.page_bytes;
        if (lane == 0) mbar_arrive_expect_tx(&ctl->full[pi], 2u * nkv * kvpage_bytes);
        __syncwarp();
        const int j = lane & 15;
        if (j < nkv) {
          int ph = kv_phys_page(p, info.b, tok0 / P + j);
          if (ph < 0) {
            raise_error(p, MK_ERR_RANGE, static_cast<uint32_t>(tix), 0xfffffffdu,
                        static_cast<uint32_t>(info.b));
            ph = 0;  // keep the copy in bounds; the step is being abandoned
          }
          const size_t off = (static_cast<size_t>(ph) * p.Hkv + info.g) * kvpage_elems;
          if (lane < 16) {
            bulk_load(pg + j * kvpage_bytes, p.k_pages[l] + off, kvpage_bytes, &ctl->full[pi], pol);
          } else {
            bulk_load(pg + static_cast<size_t>(p.tpp) * d * 2 + j * kvpage_bytes,
                      p.v_pages[l] + off, kvpage_bytes, &ctl->full[pi], pol);
          }
        }
        issued |= 1u << pi;
        last_par = (last_par & ~(1u << pi)) | (pe_par << pi);
        if (++pi == p.n_pages) {
          pi = 0;
          pe_par ^= 1u;
        }
      }
    }
    if (lane == 0) trace_mark(p, tix, 2);
    if (!ok) break;
  }

  if (!ok) {
    // Abandoning the step: no bulk copy may still be landing in shared
    // memory when this CTA exits.  Wait (bounded) for every page's last copy.
    ctl->cta_abort = 1;
    if (lane == 0) {
      for (int q = 0; q < p.n_pages; ++q) {
        if (!(issued & (1u << q))) continue;
        const uint32_t par = (last_par >> q) & 1u;
        const uint64_t t0 = gtimer();
        while (!mbar_try_wait(&ctl->full[q], par)) {
          if (gtimer() - t0 > static_cast<uint64_t>(p.wait_limit_ns) * 4) break;
        }
      }
    }
  }
  __syncwarp();
}

// ============================================================================
// compute warps: GEMV
// ============================================================================

// One weight page (16 rows x nc columns) against the staged activation.
// Lane (g, q): rows g and g+8, columns c..c+7 of each 32-column group; the
// 8 columns feed both k16 steps of the mma (a fixed permutation of k that the
// activation fragment follows as well).
template <int NN>
__device__ __forceinline__ void page_mma(float (&acc)[NN][4], uint32_t pg, int pitch, int nc,
                                         uint32_t xhi, uint32_t xlo, int xpitch, int xcol0, int B,
                                         int warp, int lane) {
  const int g = lane >> 2, q = lane & 3;
  const int groups = (nc + 31) >> 5;
  for (int grp = warp; grp < groups; grp += kComputeWarps) {
    const int c = grp * 32 + q * 8;
    const bool valid = c < nc;
    uint4 wa = make_uint4(0, 0, 0, 0), wb = make_uint4(0, 0, 0, 0);
    if (valid) {
      wa = lds128(pg + g * pitch + c * 2);
      wb = lds128(pg + (g + 8) * pitch + c * 2);
    }
#pragma unroll
    for (int nt = 0; nt < NN; ++nt) {
      const int b = nt * 8 + g;
      uint4 xh = make_uint4(0, 0, 0, 0), xl = make_uint4(0, 0, 0, 0);
      if (valid && b < B) {
        const uint32_t off = b * xpitch + (xcol0 + c) * 2;
        xh = lds128(xhi + off);
        xl = lds128(xlo + off);
      }
      mma_bf16(acc[nt], wa.x, wb.x, wa.y, wb.y, xh.x, xh.y);
      mma_bf16(acc[nt], wa.z, wb.z, wa.w, wb.w, xh.z, xh.w);
      mma_bf16(acc[nt], wa.x, wb.x, wa.y, wb.y, xl.x, xl.y);
      mma_bf16(acc[nt], wa.z, wb.z, wa.w, wb.w, xl.z, xl.w);
    }
  }
}

// Stage activation columns [xc0, xc0 + xlen) of every sequence as bf16 hi/lo
// pairs.  For normed inputs (QKV, gate/up, LM head) x = h * rs[b] * gain with
// rs computed over the full width at the first chunk of the task.
__device__ void stage_x(const Params &p, Ctl *ctl, uint8_t *smem, const Task &t, const Geo &geo,
                        int xc0, int xlen, int B, int ctid) {
  const float *src;
  const __nv_bfloat16 *gain = nullptr;
  int stride;
  const LayerW &lw = p.layers[t.layer < p.L ? t.layer : 0];
  switch (t.type) {
    case T_QKV: src = p.h; gain = lw.attn_norm; stride = p.H; break;
    case T_GATEUP: src = p.h; gain = lw.mlp_norm; stride = p.H; break;
    case T_LMHEAD: src = p.h; gain = p.final_norm; stride = p.H; break;
    case T_OPROJ: src = p.o; stride = p.Hq * p.d; break;
    default: src = p.u; stride = p.F; break;
  }
  const int warp = ctid >> 5, lane = ctid & 31;
  if (gain != nullptr && xc0 == 0) {
    for (int b = 0; b < B; ++b) {
      float s = 0.f;
      for (int i = ctid * 8; i < geo.K; i += kComputeThreads * 8) {
        const float4 a = __ldcg(reinterpret_cast<const float4 *>(src + b * stride + i));
        const float4 c = __ldcg(reinterpret_cast<const float4 *>(src + b * stride + i + 4));
        s += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
        s += c.x * c.x + c.y * c.y + c.z * c.z + c.w * c.w;
      }
      s = warp_sum(s);
      if (lane == 0) ctl->red8[warp][b] = s;
    }
    compute_bar();
    if (ctid < B) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) s += ctl->red8[w][ctid];
      ctl->rs[ctid] = 1.0f / sqrtf(s / static_cast<float>(geo.K) + p.eps);
    }
    compute_bar();
  }
  const int xpitch = row_pitch_bytes(geo.kx);
  const uint32_t xhi = smem_u32(smem + p.off_x);
  const uint32_t xlo = xhi + B * xpitch;
  for (int b = 0; b < B; ++b) {
    const float r = gain != nullptr ? ctl->rs[b] : 1.f;
    for (int i = ctid * 8; i < xlen; i += kComputeThreads * 8) {
      const float *s = src + b * stride + xc0 + i;
      const float4 a = __ldcg(reinterpret_cast<const float4 *>(s));
      const float4 c = __ldcg(reinterpret_cast<const float4 *>(s + 4));
      float v[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
      if (gain != nullptr) {
        const uint4 gw = __ldg(reinterpret_cast<const uint4 *>(gain + xc0 + i));
        const uint32_t gg[4] = {gw.x, gw.y, gw.z, gw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[2 * e] = v[2 * e] * r * bf_lo(gg[e]);
          v[2 * e + 1] = v[2 * e + 1] * r * bf_hi(gg[e]);
        }
      }
      uint32_t hw[4], lw4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat16 h0, l0, h1, l1;
        split_bf16(v[2 * e], h0, l0);
        split_bf16(v[2 * e + 1], h1, l1);
        hw[e] = pack2(h0, h1);
        lw4[e] = pack2(l0, l1);
      }
      sts128(xhi + b * xpitch + i * 2, make_uint4(hw[0], hw[1], hw[2], hw[3]));
      sts128(xlo + b * xpitch + i * 2, make_uint4(lw4[0], lw4[1], lw4[2], lw4[3]));
    }
  }
  compute_bar();
}

struct ComputeState {
  int pi = 0;
  uint32_t pg_par = 0;
  uint32_t xkey = 0xffffffffu;   // (layer, type) of the staged activation
  uint32_t sat_ev = kNoEvent;    // last (event, count) known satisfied
  uint32_t sat_cnt = 0;
  GroupSync gs;
};

template <int NN>
__device__ bool gemv_task(const Params &p, Ctl *ctl, uint8_t *smem, const Slot &S,
                          ComputeState &st, float *out, int ctid) {
  const Task &t = S.t;
  const int B = p.batch;
  const int warp = ctid >> 5, lane = ctid & 31;
  const Geo geo = gemv_geo(p, t, B);
  const int pitch = row_pitch_bytes(geo.kp);
  const int xpitch = row_pitch_bytes(geo.kx);
  const uint32_t pages = smem_u32(smem + p.off_pages);
  const uint32_t xhi = smem_u32(smem + p.off_x);
  const uint32_t xlo = xhi + B * xpitch;
  const uint32_t key = (static_cast<uint32_t>(t.layer) << 8) | t.type;

  if (t.dep_event != st.sat_ev || t.dep_count != st.sat_cnt) {
    bool okl = true;
    if (ctid == 0) okl = wait_event(p, ctl, t.dep_event, t.dep_count, S.idx);
    if (!st.gs.share(ctl, ctid, okl)) return false;
    st.sat_ev = t.dep_event;
    st.sat_cnt = t.dep_count;
  }
  if (ctid == 0) trace_mark(p, S.idx, 4);

  float acc[kMaxMTiles][NN][4];
#pragma unroll
  for (int m = 0; m < kMaxMTiles; ++m)
#pragma unroll
    for (int n = 0; n < NN; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[m][n][e] = 0.f;

  for (int xc0 = 0; xc0 < geo.K; xc0 += geo.kx) {
    const int xend = min(geo.K, xc0 + geo.kx);
    if (!(geo.whole && st.xkey == key)) {
      stage_x(p, ctl, smem, t, geo, xc0, xend - xc0, B, ctid);
      st.xkey = geo.whole ? key : 0xffffffffu;
    }
    if (ctid == 0 && xc0 == 0) trace_mark(p, S.idx, 5);
    for (int m = 0; m < t.n_m; ++m) {
      for (int c0 = xc0; c0 < xend; c0 += geo.kp) {
        const int nc = min(geo.kp, xend - c0);
        bool okl = true;
        if (ctid == 0) okl = wait_mbar(p, ctl, &ctl->full[st.pi], st.pg_par, 0xfff30000u, 2);
        if (!st.gs.share(ctl, ctid, okl)) return false;
        mbar_try_wait(&ctl->full[st.pi], st.pg_par);  // completed: acquire for this thread
        const uint32_t pg = pages + st.pi * p.page_bytes;
        switch (m) {
#define MK_PAGE_CASE(M)                                                                    \
  case M:                                                                                  \
    page_mma<NN>(acc[M], pg, pitch, nc, xhi, xlo, xpitch, c0 - xc0, B, warp, lane); \
    break;
          MK_PAGE_CASE(0)
          MK_PAGE_CASE(1)
          MK_PAGE_CASE(2)
          MK_PAGE_CASE(3)
          MK_PAGE_CASE(4)
          MK_PAGE_CASE(5)
          MK_PAGE_CASE(6)
          MK_PAGE_CASE(7)
#undef MK_PAGE_CASE
          default: break;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->empty[st.pi]);
        if (++st.pi == p.n_pages) {
          st.pi = 0;
          st.pg_par ^= 1u;
        }
      }
    }
  }

  // cross-warp reduction, one 16-row tile at a time, fixed warp order
  float *red = reinterpret_cast<float *>(smem + p.off_red);
  constexpr int NC = NN * 8;
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int m = 0; m < kMaxMTiles; ++m) {
    if (m >= t.n_m) break;
#pragma unroll
    for (int nt = 0; nt < NN; ++nt) {
      float *r0 = red + (warp * 16 + g) * NC + nt * 8 + 2 * q;
      float *r1 = red + (warp * 16 + g + 8) * NC + nt * 8 + 2 * q;
      r0[0] = acc[m][nt][0];
      r0[1] = acc[m][nt][1];
      r1[0] = acc[m][nt][2];
      r1[1] = acc[m][nt][3];
    }
    compute_bar();
    if (ctid < 16 * NC) {
      const int row = ctid / NC, n = ctid % NC;
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) s += red[(w * 16 + row) * NC + n];
      if (n < B) out[n * (16 * kMaxMTiles) + m * 16 + row] = s;
    }
    compute_bar();
  }
  return true;
}

// ============================================================================
// compute warps: attention over one chunk of one (sequence, KV head)
// ============================================================================

template <int DL>
__device__ bool attn_task(const Params &p, Ctl *ctl, uint8_t *smem, const Slot &S,
                          ComputeState &st, float *out, int ctid) {
  const Task &t = S.t;
  const int warp = ctid >> 5, lane = ctid & 31;
  const int d = p.d, G = p.G, l = t.layer;
  const int b = S.b, g = S.g;
  float *qs = reinterpret_cast<float *>(smem + p.off_x);        // [G][d]
  float *wsc = qs + G * d;                                      // [8][G][d+2]
  st.xkey = 0xffffffffu;                                        // x area reused

  {
    const uint32_t ev = static_cast<uint32_t>(ev_attn_ready(p, l, g));
    bool okl = true;
    if (ctid == 0) okl = wait_event(p, ctl, ev, static_cast<uint32_t>(G + 2), S.idx);
    if (!st.gs.share(ctl, ctid, okl)) return false;
    if (ctid == 0) trace_mark(p, S.idx, 4);
  }
  // q (normed, rotated) for the G query heads of KV head g, pre-scaled so
  // that scores are in log2 units: s = q.k / sqrt(d) * log2(e).
  const float qscale = rsqrtf(static_cast<float>(d)) * 1.4426950408889634f;
  for (int i = ctid; i < G * d; i += kComputeThreads)
    qs[i] = __ldcg(p.qrot + (static_cast<size_t>(b) * p.Hq + g * G) * d + i) * qscale;
  compute_bar();
  if (ctid == 0) trace_mark(p, S.idx, 5);

  float qv[kMaxGroup][DL];
  float mrun[kMaxGroup], lrun[kMaxGroup], acc[kMaxGroup][DL];
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    mrun[h] = -INFINITY;
    lrun[h] = 0.f;
#pragma unroll
    for (int i = 0; i < DL; ++i) {
      acc[h][i] = 0.f;
      qv[h][i] = h < G ? qs[h * d + lane * DL + i] : 0.f;
    }
  }

  const int P = p.page_size;
  const int cur = p.pos[b];
  const uint32_t pages = smem_u32(smem + p.off_pages);
  for (int tok0 = S.t0; tok0 < S.t1; tok0 += p.tpp) {
    const int ntok = min(p.tpp, S.t1 - tok0);
    bool okl = true;
    if (ctid == 0) okl = wait_mbar(p, ctl, &ctl->full[st.pi], st.pg_par, 0xfff40000u, 2);
    if (!st.gs.share(ctl, ctid, okl)) return false;
    mbar_try_wait(&ctl->full[st.pi], st.pg_par);
    uint8_t *pg = smem + p.off_pages + static_cast<size_t>(st.pi) * p.page_bytes;
    const uint32_t kbase = pages + st.pi * p.page_bytes;
    const uint32_t vbase = kbase + p.tpp * d * 2;
    // The current token's K/V were appended by this step's QKV epilogue and
    // may have been copied into the page before they landed: reload them.
    const bool has_cur = cur >= tok0 && cur < tok0 + ntok;
    if (has_cur) {
      const int ph = kv_phys_page(p, b, cur / P);
      const size_t src = ((static_cast<size_t>(ph < 0 ? 0 : ph) * p.Hkv + g) * P + cur % P) * d;
      const int j = cur - tok0;
      const int nvec = d / 8;
      if (ctid < 2 * nvec) {
        const bool isv = ctid >= nvec;
        const int e = (isv ? ctid - nvec : ctid) * 8;
        const __nv_bfloat16 *gsrc = (isv ? p.v_pages[l] : p.k_pages[l]) + src + e;
        const uint4 v = __ldcg(reinterpret_cast<const uint4 *>(gsrc));
        sts128((isv ? vbase : kbase) + (j * d + e) * 2, v);
      }
      compute_bar();
    }
    for (int j = warp; j < ntok; j += kComputeWarps) {
      float kf[DL], vf[DL];
      const __nv_bfloat16 *kr = reinterpret_cast<const __nv_bfloat16 *>(pg) + j * d + lane * DL;
      const __nv_bfloat16 *vr =
          reinterpret_cast<const __nv_bfloat16 *>(pg + static_cast<size_t>(p.tpp) * d * 2) + j * d +
          lane * DL;
#pragma unroll
      for (int i = 0; i < DL; ++i) {
        kf[i] = __bfloat162float(kr[i]);
        vf[i] = __bfloat162float(vr[i]);
      }
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) {
        if (h >= G) break;
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < DL; ++i) s += qv[h][i] * kf[i];
        s = warp_sum(s);
        const float mn = fmaxf(mrun[h], s);
        const float corr = exp2f(mrun[h] - mn);
        const float pr = exp2f(s - mn);
        lrun[h] = lrun[h] * corr + pr;
#pragma unroll
        for (int i = 0; i < DL; ++i) acc[h][i] = acc[h][i] * corr + pr * vf[i];
        mrun[h] = mn;
      }
    }
    if (has_cur) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->empty[st.pi]);
    if (++st.pi == p.n_pages) {
      st.pi = 0;
      st.pg_par ^= 1u;
    }
  }

  // merge the 8 warps' running (max, sum, acc) in fixed order
  const int rw = d + 2;
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    if (h >= G) break;
    float *w = wsc + (warp * G + h) * rw;
#pragma unroll
    for (int i = 0; i < DL; ++i) w[lane * DL + i] = acc[h][i];
    if (lane == 0) {
      w[d] = mrun[h];
      w[d + 1] = lrun[h];
    }
  }
  compute_bar();
  for (int e = ctid; e < G * rw; e += kComputeThreads) {
    const int h = e / rw, i = e % rw;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kComputeWarps; ++w) M = fmaxf(M, wsc[(w * G + h) * rw + d]);
    float s = 0.f;
    if (i < d) {
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) {
        const float mw = wsc[(w * G + h) * rw + d];
        if (mw != -INFINITY) s += exp2f(mw - M) * wsc[(w * G + h) * rw + i];
      }
    } else if (i == d) {
      s = M;
    } else {
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) {
        const float mw = wsc[(w * G + h) * rw + d];
        if (mw != -INFINITY) s += exp2f(mw - M) * wsc[(w * G + h) * rw + d + 1];
      }
    }
    out[e] = s;
  }
  compute_bar();
  return true;
}

// ============================================================================
// compute warps: embedding gather
// ============================================================================

__device__ void embed_task(const Params &p, const Slot &S, int ctid) {
  const int B = p.batch, H = p.H;
  for (int b = 0; b < B; ++b) {
    const int id = p.ids[b];
    const int pos = p.pos[b];
    const bool ok = id >= 0 && id < p.V && pos >= 0 && pos < p.max_pos &&
                    kv_phys_page(p, b, pos / p.page_size) >= 0;
    if (!ok) {
      if (ctid == 0)
        raise_error(p, MK_ERR_RANGE, static_cast<uint32_t>(S.idx), static_cast<uint32_t>(b),
                    static_cast<uint32_t>(id));
      continue;
    }
    const __nv_bfloat16 *e = p.embed + static_cast<size_t>(id) * H;
    for (int i = ctid * 8; i < H; i += kComputeThreads * 8) {
      const uint4 w = __ldg(reinterpret_cast<const uint4 *>(e + i));
      float4 a = make_float4(bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y));
      float4 c = make_float4(bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w));
      __stcg(reinterpret_cast<float4 *>(p.h + b * H + i), a);
      __stcg(reinterpret_cast<float4 *>(p.h + b * H + i + 4), c);
    }
  }
  __threadfence();
}

// ============================================================================
// compute warps: main loop
// ============================================================================

__device__ void compute_main(const Params &p, Ctl *ctl, uint8_t *smem) {
  const int ctid = threadIdx.x - 32;
  Slot *slots = reinterpret_cast<Slot *>(smem + p.off_slots);
  ComputeState st;
  int ts = 0, os = 0;
  uint32_t ts_par = 0, os_par = 0;
  bool ok = true;
  while (true) {
    bool okl = true;
    if (ctid == 0) okl = wait_mbar(p, ctl, &ctl->slot_full[ts], ts_par, 0xfff50000u, 2);
    if (!st.gs.share(ctl, ctid, okl)) {
      ok = false;
      break;
    }
    mbar_try_wait(&ctl->slot_full[ts], ts_par);
    const Slot S = slots[ts];
    if (ctid == 0 && S.t.type != T_END) trace_mark(p, S.idx, 3);
    if (ctid == 0) okl = wait_mbar(p, ctl, &ctl->out_empty[os], os_par ^ 1u, 0xfff60000u, 2);
    if (!st.gs.share(ctl, ctid, okl)) {
      ok = false;
      break;
    }
    float *out = reinterpret_cast<float *>(smem + p.off_out + os * p.out_bytes);
    bool tok = true;
    switch (S.t.type) {
      case T_END: break;
      case T_EMBED: embed_task(p, S, ctid); break;
      case T_ATTN:
        if (S.b >= 0) {
          switch (p.d >> 5) {
            case 1: tok = attn_task<1>(p, ctl, smem, S, st, out, ctid); break;
            case 2: tok = attn_task<2>(p, ctl, smem, S, st, out, ctid); break;
            case 4: tok = attn_task<4>(p, ctl, smem, S, st, out, ctid); break;
            default: tok = attn_task<8>(p, ctl, smem, S, st, out, ctid); break;
          }
        }
        break;
      default:
        tok = p.batch > 8 ? gemv_task<2>(p, ctl, smem, S, st, out, ctid)
                          : gemv_task<1>(p, ctl, smem, S, st, out, ctid);
        break;
    }
    if (!tok) {
      ok = false;
      break;
    }
    compute_bar();
    if (ctid == 0) {
      if (S.t.type != T_END) trace_mark(p, S.idx, 6);
      mbar_arrive(&ctl->out_full[os]);
    }
    if (S.t.type == T_END) break;
    if (++ts == kTaskSlots) {
      ts = 0;
      ts_par ^= 1u;
    }
    if (++os == kOutSlots) {
      os = 0;
      os_par ^= 1u;
    }
  }
  if (!ok) ctl->cta_abort = 1;
}

// ============================================================================
// storer warp: epilogues and event release
// ============================================================================

__device__ __forceinline__ void signal(const Params &p, uint32_t ev) {
  red_add_release(p.sync + S_EVENTS + ev, 1u);
}

// QK-norm + RoPE of one head for every sequence, then K/V append or q store.
__device__ void rope_head(const Params &p, const Task &t, int lane) {
  const int d = p.d, half = d / 2, l = t.layer, B = p.batch;
  const int mat = static_cast<int>(t.aux);
  const int head = static_cast<int>(t.aux2 & 0xffffu);
  const int local = mat == 0 ? head : (mat == 1 ? head - p.Hq : head - p.Hq - p.Hkv);
  const int col0 = head * d;  // rows of q, then k, then v are contiguous in qkv
  const LayerW &lw = p.layers[l];
  for (int b = 0; b < B; ++b) {
    const float *y = p.qkv + static_cast<size_t>(b) * p.NQKV + col0;
    const int pos = p.pos[b];
    if (pos < 0 || pos >= p.max_pos) continue;  // reported by the embedding task
    float rs = 1.f;
    if (mat != 2 && p.qk_norm) {
      float s = 0.f;
      for (int i = lane; i < d; i += 32) {
        const float v = __ldcg(y + i);
        s += v * v;
      }
      s = warp_sum(s);
      rs = 1.0f / sqrtf(s / static_cast<float>(d) + p.eps);
    }
    const __nv_bfloat16 *gain = mat == 0 ? lw.q_norm : lw.k_norm;
    __nv_bfloat16 *dst = nullptr;
    if (mat != 0) {
      const int ph = kv_phys_page(p, b, pos / p.page_size);
      if (ph < 0) continue;
      dst = (mat == 1 ? p.k_pages[l] : p.v_pages[l]) +
            ((static_cast<size_t>(ph) * p.Hkv + local) * p.page_size + pos % p.page_size) * d;
    }
    for (int i = lane; i < half; i += 32) {
      float a = __ldcg(y + i), c = __ldcg(y + i + half);
      if (mat != 2) {
        if (p.qk_norm) {
          a = a * rs * __bfloat162float(gain[i]);
          c = c * rs * __bfloat162float(gain[i + half]);
        }
        const float2 cs = p.rope_cs[static_cast<size_t>(pos) * half + i];
        const float ra = a * cs.x - c * cs.y;
        const float rc = c * cs.x + a * cs.y;
        a = ra;
        c = rc;
      }
      if (mat == 0) {
        float *q = p.qrot + (static_cast<size_t>(b) * p.Hq + local) * d;
        __stcg(q + i, a);
        __stcg(q + i + half, c);
      } else {
        dst[i] = __float2bfloat16_rn(a);
        dst[i + half] = __float2bfloat16_rn(c);
      }
    }
  }
}

// Merge the chunks of (b, g) by log-sum-exp and write o for its G heads.
__device__ void attn_combine(const Params &p, const Slot &S, int lane) {
  const int d = p.d, G = p.G, rw = d + 2;
  for (int e = lane; e < G * d; e += 32) {
    const int h = e / d, i = e % d;
    float M = -INFINITY;
    for (int c = 0; c < S.n_chunks; ++c) {
      const float *pc = p.attn_part + (static_cast<size_t>(S.first_slot + c) * G + h) * rw;
      M = fmaxf(M, __ldcg(pc + d));
    }
    float num = 0.f, den = 0.f;
    for (int c = 0; c < S.n_chunks; ++c) {
      const float *pc = p.attn_part + (static_cast<size_t>(S.first_slot + c) * G + h) * rw;
      const float w = exp2f(__ldcg(pc + d) - M);
      num += w * __ldcg(pc + i);
      den += w * __ldcg(pc + d + 1);
    }
    __stcg(p.o + static_cast<size_t>(S.b) * p.Hq * d + (S.g * G + h) * d + i, num / den);
  }
}

__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<unsigned long long>(u) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(idx));
}

__device__ bool storer_epilogue(const Params &p, Ctl *ctl, const Slot &S, const float *out,
                                int lane) {
  const Task &t = S.t;
  const int B = p.batch;
  constexpr int OS = 16 * kMaxMTiles;
  switch (t.type) {
    case T_EMBED: {
      __syncwarp();
      if (lane == 0) signal(p, t.out_event);
      break;
    }
    case T_QKV: {
      const int base = t.aux == 0 ? 0 : (t.aux == 1 ? p.Hq * p.d : (p.Hq + p.Hkv) * p.d);
      for (int b = 0; b < B; ++b)
        for (int r = lane; r < static_cast<int>(t.nrows); r += 32)
          __stcg(p.qkv + static_cast<size_t>(b) * p.NQKV + base + t.row0 + r, out[b * OS + r]);
      __threadfence();
      __syncwarp();
      const int head = static_cast<int>(t.aux2 & 0xffffu);
      const uint32_t need = t.aux2 >> 16;
      uint32_t old = 0;
      if (lane == 0) old = atom_add_acq_rel(p.head_ctr + t.layer * (p.Hq + 2 * p.Hkv) + head, 1u);
      old = __shfl_sync(0xffffffffu, old, 0);
      if (old + 1u == need) {
        fence_acq_rel();
        rope_head(p, t, lane);
        __threadfence();
        __syncwarp();
        if (lane == 0) {
          p.head_ctr[t.layer * (p.Hq + 2 * p.Hkv) + head] = 0u;
          const int g = t.aux == 0 ? head / p.G : (t.aux == 1 ? head - p.Hq : head - p.Hq - p.Hkv);
          signal(p, static_cast<uint32_t>(ev_attn_ready(p, t.layer, g)));
        }
      }
      break;
    }
    case T_ATTN: {
      if (S.b >= 0) {
        const int n = p.G * (p.d + 2);
        float *dst = p.attn_part + static_cast<size_t>(t.aux) * n;
        for (int e = lane; e < n; e += 32) __stcg(dst + e, out[e]);
        __threadfence();
        __syncwarp();
        uint32_t old = 0;
        uint32_t *ctr = p.comb_ctr + S.b * p.Hkv + S.g;
        if (lane == 0) old = atom_add_acq_rel(ctr, 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old + 1u == static_cast<uint32_t>(S.n_chunks)) {
          fence_acq_rel();
          attn_combine(p, S, lane);
          __threadfence();
          __syncwarp();
          if (lane == 0) *ctr = 0u;
        }
      }
      __syncwarp();
      if (lane == 0) signal(p, t.out_event);
      break;
    }
    case T_OPROJ:
    case T_DOWN: {
      for (int b = 0; b < B; ++b)
        for (int r = lane; r < static_cast<int>(t.nrows); r += 32) {
          float *hp = p.h + static_cast<size_t>(b) * p.H + t.row0 + r;
          const float v = __ldcg(hp) + out[b * OS + r];
          __stcg(hp, v);
          if (t.type == T_DOWN && p.hidden_dump != nullptr)
            p.hidden_dump[(static_cast<size_t>(t.layer) * B + b) * p.H + t.row0 + r] = v;
        }
      __threadfence();
      __syncwarp();
      if (lane == 0) signal(p, t.out_event);
      break;
    }
    case T_GATEUP: {
      const int nh16 = (t.n_m >> 1) * 16;
      for (int b = 0; b < B; ++b)
        for (int r = lane; r < static_cast<int>(t.nrows); r += 32) {
          const float gt = out[b * OS + r];
          const float up = out[b * OS + nh16 + r];
          __stcg(p.u + static_cast<size_t>(b) * p.F + t.row0 + r, gt / (1.0f + __expf(-gt)) * up);
        }
      __threadfence();
      __syncwarp();
      if (lane == 0) signal(p, t.out_event);
      break;
    }
    case T_LMHEAD: {
      for (int b = 0; b < B; ++b) {
        float best = -INFINITY;
        int bi = 0x7fffffff;
        for (int r = lane; r < static_cast<int>(t.nrows); r += 32) {
          const float v = out[b * OS + r];
          if (p.out_logits != nullptr)
            p.out_logits[static_cast<size_t>(b) * p.V + t.row0 + r] = v;
          if (v > best) {  // r increases per lane: first max kept
            best = v;
            bi = static_cast<int>(t.row0) + r;
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ob = __shfl_xor_sync(0xffffffffu, best, o);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
          if (ob > best || (ob == best && oi < bi)) {
            best = ob;
            bi = oi;
          }
        }
        if (lane == 0) atomicMax(p.argmax + b, argmax_key(best, bi));
      }
      __threadfence();
      __syncwarp();
      uint32_t old = 0;
      if (lane == 0) old = atom_add_acq_rel(p.sync + S_LMCTR, 1u);
      old = __shfl_sync(0xffffffffu, old, 0);
      if (old + 1u == static_cast<uint32_t>(p.n_lm_tasks)) {
        fence_acq_rel();
        if (lane < B) {
          const unsigned long long k = ld_relaxed_u64(p.argmax + lane);
          p.out_ids[lane] = static_cast<int32_t>(~static_cast<uint32_t>(k & 0xffffffffull));
          if (p.out_pos != nullptr) p.out_pos[lane] = p.pos[lane] + 1;
          p.argmax[lane] = 0ull;
        }
        __syncwarp();
        if (lane == 0) p.sync[S_LMCTR] = 0u;
      }
      break;
    }
    default: break;
  }
  (void)ctl;
  return true;
}

__device__ void storer_main(const Params &p, Ctl *ctl, uint8_t *smem) {
  const int lane = threadIdx.x & 31;
  Slot *slots = reinterpret_cast<Slot *>(smem + p.off_slots);
  int ts = 0, os = 0;
  uint32_t ts_par = 0, os_par = 0;
  bool ok = true;
  while (true) {
    int okl = 1;
    if (lane == 0) okl = wait_mbar(p, ctl, &ctl->out_full[os], os_par, 0xfff70000u, 2);
    ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
    if (!ok) break;
    mbar_try_wait(&ctl->out_full[os], os_par);
    const Slot S = slots[ts];
    if (S.t.type == T_END) break;
    const float *out = reinterpret_cast<const float *>(smem + p.off_out + os * p.out_bytes);
    storer_epilogue(p, ctl, S, out, lane);
    __syncwarp();
    if (lane == 0) trace_mark(p, S.idx, 7);
    if (lane == 0) {
      mbar_arrive(&ctl->out_empty[os]);
      mbar_arrive(&ctl->slot_empty[ts]);
    }
    if (++ts == kTaskSlots) {
      ts = 0;
      ts_par ^= 1u;
    }
    if (++os == kOutSlots) {
      os = 0;
      os_par ^= 1u;
    }
  }
  if (!ok) ctl->cta_abort = 1;
  (void)ts_par;
}

// ============================================================================
// kernel
// ============================================================================

__global__ void __launch_bounds__(kThreads, 1) mk_step_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Ctl *ctl = reinterpret_cast<Ctl *>(smem);
  if (threadIdx.x == 0) {
    for (int i = 0; i < p.n_pages; ++i) {
      mbar_init(&ctl->full[i], 1);
      mbar_init(&ctl->empty[i], kComputeWarps);
    }
    for (int i = 0; i < kTaskSlots; ++i) {
      mbar_init(&ctl->slot_full[i], 1);
      mbar_init(&ctl->slot_empty[i], 1);
    }
    for (int i = 0; i < kOutSlots; ++i) {
      mbar_init(&ctl->out_full[i], 1);
      mbar_init(&ctl->out_empty[i], 1);
    }
    ctl->cta_abort = 0;
    ctl->flag[0] = ctl->flag[1] = 0;
    // a device error from an earlier step is sticky until the host resets
    ctl->skip = (ld_relaxed(p.sync + S_STATUS) != 0u || ld_relaxed(p.sync + S_ABORT) != 0u);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (!ctl->skip) {
    const int warp = threadIdx.x >> 5;
    if (warp == kLoaderWarp) {
      loader_main(p, ctl, smem);
    } else if (warp == kStorerWarp) {
      storer_main(p, ctl, smem);
    } else {
      compute_main(p, ctl, smem);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(p.sync + S_EXIT, 1u);
    if (old == gridDim.x - 1u) {
      // every CTA has stopped popping: rearm the queue for the next launch
      atomicExch(p.sync + S_QUEUE, 0u);
      atomicExch(p.sync + S_EXIT, 0u);
    }
  }
}

cudaError_t configure_kernel(int smem) {
  return cudaFuncSetAttribute(mk_step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

cudaError_t launch_step(const Params &p, int grid, int smem, bool cooperative, cudaStream_t stream) {
  if (cooperative) {
    void *args[] = {const_cast<Params *>(&p)};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(mk_step_kernel), dim3(grid),
                                       dim3(kThreads), args, static_cast<size_t>(smem), stream);
  }
  mk_step_kernel<<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mk
