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
//   warps 1..6  compute: wait for the task's input event (in-GPU event
//                        counters, MPK write-up "2.1 Mega-Kernel执行模型":
//                        trigger count vs. required count), stage the
//                        activation, and consume the pages (bf16 mma.sync for
//                        the projections; for attention: QK-norm + RoPE of the
//                        step's q and K, the KV append, online softmax over the
//                        chunk's pages and the split-attention combine).
//   warp 7      storer : epilogues (residual add, split-K sums, SwiGLU,
//                        argmax) and the release of the task's output event.
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

// Non-blocking probe of a phase (try_wait may suspend the thread for a while
// before it reports an incomplete phase; test_wait returns at once).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P1;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, P1;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
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

// 1-D bulk copy without a cache hint.
__device__ __forceinline__ void bulk_load_plain(void *dst, const void *src, uint32_t bytes,
                                                uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---- tensor-core path: TMA tensor copies and tcgen05 -------------------------

// 2-D tensor copy of one box (tensor map `tmap`, coordinates {x = column,
// y = row}) into this CTA's shared memory, completion on `bar`.  No cluster
// multicast: the map covers this GPU's own memory only.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int x, int y,
                                            uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 3-D tensor copy (x innermost) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void *dst, const void *tmap, int x, int y, int z,
                                            uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Copy 128 rows x 256 bits from shared memory (descriptor) into tensor memory:
// row i to lane i, its 32 bytes to 8 consecutive columns.  Issued by one
// thread; completion is tracked by tcgen05.commit.
__device__ __forceinline__ void tm_cp(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Warp-wide: 16 lanes x 4 x 256 bits of tensor memory starting at lane
// (taddr >> 16) (a multiple of 16 inside this warp's lane quarter): four
// consecutive 8-column groups.  Of group i, thread (g = lane / 4, q = lane % 4)
// receives the 32-bit words 2q and 2q + 1 of rows g and g + 8:
// r[4i] = (g, 2q), r[4i + 1] = (g, 2q + 1), r[4i + 2] = (g + 8, 2q),
// r[4i + 3] = (g + 8, 2q + 1).  (Completion: tcgen05.wait::ld.)
__device__ __forceinline__ void tm_ld16x256_x4(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tm_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand in the 128-byte
// swizzled layout: 8-row groups 1024 bytes apart, rows 128 bytes apart.
// Fields: start address >> 4 (bits 0-13), leading-dimension offset (unused
// for this layout, 1), stride-dimension offset 1024 >> 4 (bits 32-45),
// descriptor version 1 (bits 46-47), layout type 2 = 128-byte swizzle
// (bits 61-63).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (1ull << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of a dense bf16 x bf16 -> fp32 MMA, both operands
// K-major: D format f32 (bits 4-5 = 1), A and B format bf16 (bits 7-9 and
// 10-12 = 1), N >> 3 (bits 17-22), M >> 4 (bits 24-28).
__device__ __forceinline__ uint32_t mma_idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, M = 128, issued by one thread.
__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far has
// completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Warp-wide: allocate `ncols` tensor-memory columns; the base address is
// written to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Warp-wide: 16 consecutive fp32 accumulator columns of this warp's 32 lanes
// (lane i of the warp reads tensor-memory lane (taddr >> 16) + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
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

// Acquire load.  Re-reading a counter with acquire after a relaxed poll saw it
// complete orders the producers' writes (published by their release
// increments) before this thread's later accesses.  It costs a load round
// trip, where a GPU-scope fence also waits for this thread's outstanding
// memory operations: 4% of an 8B decode step when both dependency paths
// used the fence.
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

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
  asm(  // pure register op: the compiler may schedule it freely
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
  uint64_t xbar;                    // activation bulk copy landed
  uint64_t x_full[2];               // tensor-core path: staged chunk buffer ready for the MMAs
  uint64_t x_free[2];               // ... its MMAs completed (buffer may be restaged)
  uint64_t acc_bar;                 // ... the task's MMAs completed (accumulators final)
  uint32_t tmem;                    // tensor-memory base address of this CTA
  volatile int cta_abort;
  volatile int cbad;                // a compute warp gave up (written by compute only)
  int skip;
  int flag[2];
  float rs[MK_MAX_BATCH];           // RMSNorm scale per sequence
  float ss[MK_MAX_BATCH];           // running sum of squares per sequence
  float red8[kComputeWarps][MK_MAX_BATCH];
};
static_assert(sizeof(Ctl) <= 1024, "control block exceeds its 1 KB slot");

// A popped task as the loader hands it to compute and storer (64 bytes).
struct Slot {
  Task t;
  int b, g, t0, t1;          // attention: sequence, KV head, token range
  int first_slot, n_chunks;  // attention: partial slots of (b, g)
  int idx;                   // task index (for error reports)
  int dep_ok;                // the loader saw the input event complete
};
static_assert(sizeof(Slot) == kSlotBytes, "slot size");

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
      // the CTA flag is a shared-memory read; the global flag is polled rarely
      if (ctl->cta_abort != 0) return false;
      if ((it & 255u) == 255u && ld_relaxed(p.sync + S_ABORT) != 0u) return false;
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
      (void)ld_acquire(ctr);
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
  int K;        // full input width (row length of the weight matrix)
  int k0, Kt;   // the task's columns: [k0, k0 + Kt) (split-K parts cover a range)
  int kp;       // columns per weight page
  int kx;       // columns per staged activation chunk
  int whole;    // kx == Kt: the staged activation can be reused by later tasks
  int cls;      // OpK
};

__device__ __forceinline__ int x_bytes(int B, int cols) { return B * x_row_bytes(cols); }

__device__ Geo gemv_geo(const Params &p, const Task &t, int B) {
  Geo g;
  switch (t.type) {
    case T_OPROJ: g.K = p.Hq * p.d; g.cls = K_ATT; break;
    case T_DOWN: g.K = p.F; g.cls = K_FFN; break;
    case T_LMHEAD: g.K = p.H; g.cls = K_LM; break;
    default: g.K = p.H; g.cls = K_HID; break;
  }
  g.kp = p.kp[g.cls];
  if (t.nsplit > 1) {
    g.k0 = t.ksplit * p.kchunk[g.cls];
    g.Kt = min(g.K, g.k0 + p.kchunk[g.cls]) - g.k0;
  } else {
    g.k0 = 0;
    g.Kt = g.K;
  }
  if (x_bytes(B, g.Kt) <= p.x_cap) {
    g.kx = g.Kt;
    g.whole = 1;
  } else {
    int n = g.Kt / g.kp;
    while (n > 1 && x_bytes(B, n * g.kp) > p.x_cap) --n;
    g.kx = n * g.kp;
    g.whole = 0;
  }
  return g;
}

// Tensor-core path: a task's columns [k0, k0 + Kt) of its K-wide input.
struct TcGeo {
  int K, k0, Kt;
};
__device__ __forceinline__ TcGeo tc_geo(const Params &p, const Task &t) {
  TcGeo g;
  g.K = t.type == T_OPROJ ? p.Hq * p.d : (t.type == T_DOWN ? p.F : p.H);
  const int kt = p.tc_kt[t.type];
  if (t.nsplit > 1 && kt > 0) {
    g.k0 = t.ksplit * kt;
    g.Kt = min(g.K, g.k0 + kt) - g.k0;
  } else {
    g.k0 = 0;
    g.Kt = g.K;
  }
  return g;
}

// Row `m`-tile of a GEMV task: weight matrix base, first row, valid rows.
__device__ __forceinline__ void gemv_tile(const Params &p, const Task &t, int m,
                                          const __nv_bfloat16 *&W, int &row, int &rows_valid) {
  int mm = m;
  W = t.w0;
  if (t.type == T_GATEUP) {  // first half of the tiles read w_gate, second w_up
    const int nh = t.n_m >> 1;
    if (m >= nh) {
      W = t.w1;
      mm = m - nh;
    }
  }
  row = static_cast<int>(t.row0) + 16 * mm;
  const int left = static_cast<int>(t.nrows) - 16 * mm;
  rows_valid = left < 16 ? (left > 0 ? left : 0) : 16;
}

// Position of row b this step: its own, or (a prompt chunk of one sequence)
// the chunk's first position + b.
__device__ __forceinline__ int row_pos(const Params &p, int b) {
  return p.chunk_seq >= 0 ? p.chunk_pos0 + b : p.pos[b];
}
// Block-table row of row b: its own, or the chunk's sequence.
__device__ __forceinline__ int row_seq(const Params &p, int b) {
  return p.chunk_seq >= 0 ? p.chunk_seq : b;
}

// Tokens attended by sequence b this step (positions 0..pos), clamped to
// [1, max_pos] so a bad position cannot blow up the attention split (bad
// positions are reported by the embedding task).
__device__ __forceinline__ int seq_len(const Params &p, int b) {
  int n = row_pos(p, b) + 1;
  return n < 1 ? 1 : (n > p.max_pos ? p.max_pos : n);
}

// The loader's view of the batch for one launch: lane b (< B) holds the
// number of tokens sequence b attends (positions 0..pos, clamped to
// [1, max_pos]); every lane holds the attention chunk span: a whole number
// of KV pages, sized so each KV group's chunks over all sequences fit its
// block of slots (one partial chunk per sequence is allowed for).  Read once
// per launch, one position per lane, so resolving a slot later costs no
// global round trip.
struct SeqView {
  int len, span;
};
__device__ SeqView seq_view(const Params &p, int B, int lane) {
  SeqView v;
  const int P = p.page_size;
  v.len = lane < B ? seq_len(p, lane) : 0;
  const int units = __reduce_add_sync(0xffffffffu, (v.len + P - 1) / P);
  const int target = p.attn_spg - B;
  const int c = (units + target - 1) / target;
  v.span = (c < 1 ? 1 : c) * P;
  return v;
}

// Slot s of a layer -> (sequence, KV head, token range) (warp-uniform, all
// lanes).  Slots come in one block per KV group; inside a block, the chunks
// of sequence 0, then 1, ...
__device__ bool attn_resolve(const Params &p, int B, int s, const SeqView &v, int lane, Slot &o) {
  const int g = s / p.attn_spg;
  const int r = s - g * p.attn_spg;
  const int nb = lane < B ? (v.len + v.span - 1) / v.span : 0;
  int incl = nb;   // inclusive prefix sum of chunks over sequences 0..lane
#pragma unroll
  for (int k = 1; k < 32; k <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, k);
    if (lane >= k) incl += y;
  }
  const int excl = incl - nb;
  const unsigned hit = __ballot_sync(0xffffffffu, lane < B && r >= excl && r < incl);
  if (hit == 0u) {
    o.b = -1;
    return false;
  }
  const int b = __ffs(hit) - 1;
  const int base = __shfl_sync(0xffffffffu, excl, b);
  const int nbb = __shfl_sync(0xffffffffu, nb, b);
  const int len = __shfl_sync(0xffffffffu, v.len, b);
  o.b = b;
  o.g = g;
  o.t0 = (r - base) * v.span;
  o.t1 = min(len, o.t0 + v.span);
  o.first_slot = g * p.attn_spg + base;
  o.n_chunks = nbb;
  return true;
}

__device__ __forceinline__ int kv_phys_page(const Params &p, int b, int logical) {
  int lp = logical < p.max_pages_per_seq ? logical : p.max_pages_per_seq - 1;
  int ph = p.block_table[row_seq(p, b) * p.max_pages_per_seq + lp];
  return (ph >= 0 && ph < p.num_kv_pages) ? ph : -1;
}

// ============================================================================
// loader (warp 0)
// ============================================================================

__device__ __forceinline__ bool is_gemv(uint8_t type) {
  return type == T_QKV || type == T_OPROJ || type == T_GATEUP || type == T_DOWN ||
         type == T_LMHEAD;
}

// Tasks popped from the queue but not yet handed to the compute warps.
struct Look {
  Task t;
  int tix;
  int pad[3];
};
// the end of the lookahead area holds the tensor-memory slot barriers
constexpr int kTmBarBytes = 2 * kTmSlots * 8;
constexpr int kLook = (kLookBytes - kTmBarBytes) / static_cast<int>(sizeof(Look));
// Tensor-memory page slot i: filled by the mover's commit (tm_full), read by
// every compute warp (tm_empty).
__device__ __forceinline__ uint64_t *tm_full_bar(uint8_t *smem, const Params &p, int i) {
  return reinterpret_cast<uint64_t *>(smem + p.off_look + kLookBytes - kTmBarBytes) + i;
}
__device__ __forceinline__ uint64_t *tm_empty_bar(uint8_t *smem, const Params &p, int i) {
  return reinterpret_cast<uint64_t *>(smem + p.off_look + kLookBytes - kTmBarBytes) + kTmSlots + i;
}
static_assert(sizeof(Look) == 80 && kLook >= 2, "lookahead entry size");

template <int V>
__device__ void loader_main(const Params &p, Ctl *ctl, uint8_t *smem) {
  constexpr bool TC = (V & kVarTc) != 0, W4 = (V & kVarW4) != 0, AMMA = (V & kVarAttnMma) != 0;
  constexpr bool TM = (V & kVarTm) != 0;
  const int lane = threadIdx.x & 31;
  const uint64_t pol = l2_evict_first_policy();
  Slot *slots = reinterpret_cast<Slot *>(smem + p.off_slots);
  Look *la = reinterpret_cast<Look *>(smem + p.off_look);
  uint8_t *pages = smem + p.off_pages;
  const int B = p.batch;

  int pi = 0;
  uint32_t pe_par = 0;            // ring round parity
  uint32_t issued = 0, last_par = 0;
  int ts = 0;
  uint32_t ts_par = 0;
  bool ok = true;

  // the dynamic queue hands out tickets from one global counter; a
  // solidified schedule walks this CTA's own list of task indices
  const bool fixed = p.sched != nullptr;
  const int s_begin = fixed ? p.sched_off[blockIdx.x] : 0;
  const int n_launch = fixed ? p.sched_off[blockIdx.x + 1] - s_begin : p.task_end - p.task_begin;
  uint32_t next = 0;
  if (lane == 0 && !fixed) next = atomicAdd(p.sync + S_QUEUE, 1u);
  int la_head = 0, la_count = 0;
  bool exhausted = false;
  uint32_t la_ev = 0;   // lane 0: input-event counter read when the task was popped
  const SeqView sv = seq_view(p, B, lane);

  // ---- tensor-memory staging (lane 0): the mover ----
  // Pages are moved in ring order.  A GEMV page, once landed, is copied into
  // the next free tensor-memory slot (one tcgen05.cp per 128-column box);
  // the copies' completion frees the shared-memory page and fills the slot.
  // An attention page is passed over (the compute warps read it from shared
  // memory and free it).  service() never blocks: every wait of the loader
  // calls it, so pages keep moving while the loader waits.
  const uint32_t tmem = TM ? ctl->tmem : 0u;
  int mv_pm = 0, mv_n = 0;          // next page to move; pages issued and not yet moved
  uint32_t mv_ppar = 0;             // its ring round parity
  uint32_t mv_kind = 0;             // per ring page: 1 = GEMV page for tensor memory
  uint64_t mv_ng = 0;               // per ring page: boxes - 1 (4 bits)
  int tslot = 0;                    // next tensor-memory slot and its round parity
  uint32_t tpar = 0;
  int last_slot = -1;               // the slot of the last commit (drained at exit)
  uint32_t last_tpar = 0;
  auto service = [&]() {
    if constexpr (TM) {
      while (mv_n > 0) {
        const int pm = mv_pm;
        if ((mv_kind >> pm) & 1u) {
          if (!mbar_test_wait(&ctl->full[pm], mv_ppar)) return;
          if (!mbar_test_wait(tm_empty_bar(smem, p, tslot), tpar ^ 1u)) return;
          tc_fence_after();
          const int nb = static_cast<int>((mv_ng >> (4 * pm)) & 15u) + 1;
          const uint32_t src = smem_u32(pages + static_cast<size_t>(pm) * p.page_bytes);
          const uint32_t dst = tmem + static_cast<uint32_t>(tslot * kTmSlotCols);
          // box b, 16-column slice j of its 64-column blocks -> columns 32 b + 8 j
          for (int b = 0; b < nb; ++b)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tm_cp(dst + 32u * b + 8u * j, sw128_desc(src + static_cast<uint32_t>(kTmBoxBytes) * b + 32u * j));
          tc_commit(&ctl->empty[pm]);      // the shared-memory page is free once copied
          tc_commit(tm_full_bar(smem, p, tslot));
          last_slot = tslot;
          last_tpar = tpar;
          if (++tslot == kTmSlots) {
            tslot = 0;
            tpar ^= 1u;
          }
        }
        if (++mv_pm == p.n_pages) {
          mv_pm = 0;
          mv_ppar ^= 1u;
        }
        --mv_n;
      }
    }
  };
  // lane 0: wait for a barrier phase (bounded), moving pages meanwhile.
  // For a ring page (`ring`), also until the mover has passed the page's
  // previous occupant: an attention page is freed by the compute warps, and
  // the mover, behind on a page waiting for a tensor-memory slot, must not
  // read the new occupant's kind in its place.
  auto lwait = [&](uint64_t *bar, uint32_t parity, uint32_t where, bool ring = false) -> bool {
    if constexpr (!TM) {
      return wait_mbar(p, ctl, bar, parity, where, 2);
    } else {
      uint64_t t0 = 0;
      for (uint32_t it = 0;; ++it) {
        service();   // (first: pages that landed meanwhile move without delay)
        if ((!ring || mv_n < p.n_pages) && mbar_test_wait(bar, parity)) return true;
        if ((it & 7u) == 7u) {
          if (ctl->cta_abort != 0) return false;
          if ((it & 255u) == 255u && ld_relaxed(p.sync + S_ABORT) != 0u) return false;
          const uint64_t now = gtimer();
          if (t0 == 0) {
            t0 = now;
          } else if (now - t0 > static_cast<uint64_t>(p.wait_limit_ns) * 2) {
            raise_error(p, MK_ERR_TIMEOUT, where, 0xfffffffeu, parity);
            return false;
          }
        }
      }
    }
  };
  // lane 0: wait for an event (bounded, acquire), moving pages meanwhile
  auto lwait_event = [&](uint32_t ev, uint32_t count, uint32_t task_idx) -> bool {
    if constexpr (!TM) {
      return wait_event(p, ctl, ev, count, task_idx);
    } else {
      const uint32_t target = p.epoch * count;
      const uint32_t *ctr = p.sync + S_EVENTS + ev;
      uint64_t t0 = 0;
      for (uint32_t it = 0;; ++it) {
        const uint32_t v = ld_relaxed(ctr);
        if (static_cast<int32_t>(v - target) >= 0) {
          (void)ld_acquire(ctr);
          return true;
        }
        service();
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
  };

  // The descriptor of the next ticket is read ahead: lanes 0..3 hold its
  // 16-byte quarters (ticket pf_ticket, task pf_tix), requested at a top-up
  // after the ticket arrived, so that a pop finds it in registers.
  uint4 pf_q = make_uint4(0u, 0u, 0u, 0u);
  int pf_tix = 0;
  uint32_t pf_ticket = 0xffffffffu;   // warp-uniform; none in flight
  auto prefetch_desc = [&]() {
    const uint32_t ticket = __shfl_sync(0xffffffffu, next, 0);
    if (ticket == pf_ticket || static_cast<int>(ticket) >= n_launch) return;
    const int tix = fixed ? p.sched[s_begin + static_cast<int>(ticket)]
                          : p.task_begin + static_cast<int>(ticket);
    if (lane < 4) pf_q = reinterpret_cast<const uint4 *>(p.tasks + tix)[lane];
    pf_tix = tix;
    pf_ticket = ticket;
  };
  // Pop one task into the lookahead (warp-uniform).  The next ticket is
  // always requested one pop ahead and its descriptor read ahead.  Lane 0
  // also starts reading the GEMV task's input-event counter; the value is
  // looked at only when the task is handed over, a task later.
  auto pop_one = [&]() {
    const uint32_t ticket = __shfl_sync(0xffffffffu, next, 0);
    if (static_cast<int>(ticket) >= n_launch) {
      exhausted = true;
      return;
    }
    prefetch_desc();   // (a no-op when the descriptor is already in flight)
    if (lane == 0) next = fixed ? ticket + 1u : atomicAdd(p.sync + S_QUEUE, 1u);
    const int e = (la_head + la_count) % kLook;
    if (lane < 4) reinterpret_cast<uint4 *>(&la[e].t)[lane] = pf_q;
    __syncwarp();
    if (lane == 0) {
      la[e].tix = pf_tix;
      const uint8_t type = la[e].t.type;
      const uint32_t dep = la[e].t.dep_event;
      if (is_gemv(type) && dep != kNoEvent) la_ev = ld_relaxed(p.sync + S_EVENTS + dep);
    }
    pf_ticket = 0xffffffffu;
    ++la_count;
  };
  // A handed-over GEMV task whose input was not yet complete, or an
  // attention chunk, blocks further pops until its input completes, so a CTA
  // waiting at an operator boundary does not reserve more of the next
  // operator's tasks.
  bool blocked = false;
  uint32_t blk_ev = kNoEvent, blk_cnt = 0;
  int blk_tix = 0;   // the blocked task (named in a timeout report)
  // The blocking event is polled without waiting for the read: each call
  // looks at the value the previous call requested and requests the next
  // (lane 0), so a poll never stalls the loader for a round trip.
  uint32_t poll_v = 0;
  bool poll_out = false;   // lane 0: a read of the blocking event is in flight
  auto may_pop = [&]() {
    if (!blocked) return true;
    int ok = 0;
    if (lane == 0) {
      if (poll_out) ok = static_cast<int32_t>(poll_v - p.epoch * blk_cnt) >= 0;
      poll_v = ld_relaxed(p.sync + S_EVENTS + blk_ev);
      poll_out = true;
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) blocked = false;
    return ok != 0;
  };
  auto top_up = [&](int max_pops) {
    if (!exhausted && la_count >= 1) prefetch_desc();
    for (int k = 0; k < max_pops; ++k) {
      // one task ahead: every popped task is reserved for this CTA, so
      // popping further ahead would delay the last tasks of an operator
      if (exhausted || la_count >= 1 || !may_pop()) break;
      pop_one();
    }
    __syncwarp();
  };

  while (true) {
    top_up(kLook);
    if (la_count == 0 && !exhausted && blocked) {
      int okw = 1;
      if (lane == 0) okw = lwait_event(blk_ev, blk_cnt, static_cast<uint32_t>(blk_tix));
      if (__shfl_sync(0xffffffffu, okw, 0) == 0) {
        ok = false;
        break;
      }
      blocked = false;
      top_up(kLook);
    }
    int okl = 1;
    if (lane == 0) okl = lwait(&ctl->slot_empty[ts], ts_par ^ 1u, 0xfff00000u);
    ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
    if (!ok) break;

    Slot &S = slots[ts];
    if (la_count == 0) {  // queue drained
      if (lane == 0) {
        S.t.type = T_END;
        mbar_arrive(&ctl->slot_full[ts]);
      }
      break;
    }
    const Task t = la[la_head].t;
    const int tix = la[la_head].tix;
    la_head = (la_head + 1) % kLook;
    --la_count;
    Slot info;
    info.t = t;
    info.idx = tix;
    info.b = -1;
    info.dep_ok = 0;
    // attention: the chunk's KV pages from the block table, one per lane,
    // read now so the lookups overlap the wait for free ring pages
    int ph_pre = -1;
    if (t.type == T_ATTN && attn_resolve(p, B, static_cast<int>(t.aux), sv, lane, info)) {
      const int npg = (info.t1 - info.t0 + p.page_size - 1) / p.page_size;
      if (lane < npg) ph_pre = kv_phys_page(p, info.b, info.t0 / p.page_size + lane);
    }
    __syncwarp();
    if (lane == 0) {
      // an input event already complete when the task was popped: acquire
      // its producers' writes before the hand-over (the slot barrier, a
      // CTA-scope release/acquire pair, carries them on to the compute
      // warps), which then skip their own wait
      if (is_gemv(t.type) && t.dep_event != kNoEvent &&
          static_cast<int32_t>(la_ev - p.epoch * t.dep_count) >= 0) {
        (void)ld_acquire(p.sync + S_EVENTS + t.dep_event);
        info.dep_ok = 1;
      }
      S = info;
      mbar_arrive(&ctl->slot_full[ts]);
      if (p.trace != nullptr) {
        p.trace[static_cast<size_t>(tix) * 8] =
            blockIdx.x | (static_cast<unsigned long long>(t.type) << 32) |
            (static_cast<unsigned long long>(t.layer) << 40);
        trace_mark(p, tix, 1);
      }
    }
    {
      const int dok = __shfl_sync(0xffffffffu, info.dep_ok, 0);
      if (is_gemv(t.type) && t.dep_event != kNoEvent && !dok) {
        blocked = true;
        poll_out = false;
        blk_ev = t.dep_event;
        blk_cnt = t.dep_count;
        blk_tix = tix;
      } else if (t.type == T_ATTN && info.b >= 0) {
        // an attention chunk waits for its KV group's projections: one such
        // chunk per CTA, so a group's chunks run on as many SMs as it has
        blocked = true;
        poll_out = false;
        blk_ev = static_cast<uint32_t>(ev_attn_input(p, t.layer, info.g));
        blk_cnt = static_cast<uint32_t>(attn_input_count(p));
        blk_tix = tix;
      }
    }
    if (++ts == kTaskSlots) {
      ts = 0;
      ts_par ^= 1u;
    }

    // ---- stream the task's operands into the page ring ----
    if (TC && is_gemv(t.type)) {
      // tensor-core path: per activation chunk, per 128-row tile, pages of
      // tc_kc columns, each one TMA box per 64-column swizzle atom
      const TcGeo g = tc_geo(p, t);
      const uint8_t *maps = static_cast<const uint8_t *>(p.tmaps);
      for (int xc0 = g.k0; xc0 < g.k0 + g.Kt && ok; xc0 += p.tc_kx) {
        const int xend = min(g.k0 + g.Kt, xc0 + p.tc_kx);
        for (int m = 0; m < t.n_m && ok; ++m) {
          const void *map = maps + static_cast<size_t>(m == 0 ? t.map0 : t.map1) * 128;
          for (int c0 = xc0; c0 < xend; c0 += p.tc_kc) {
            const int nc = min(p.tc_kc, xend - c0);
            if (lane == 0) okl = wait_mbar(p, ctl, &ctl->empty[pi], pe_par ^ 1u, 0xfff10000u, 2);
            ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
            if (!ok) break;
            uint8_t *pg = pages + static_cast<size_t>(pi) * p.page_bytes;
            if (lane == 0) mbar_arrive_expect_tx(&ctl->full[pi], static_cast<uint32_t>(nc * kTcRows * 2));
            __syncwarp();
            if (lane < nc / kTcAtomCols)
              tma_load_2d(pg + lane * kTcAtomBytes, map, c0 + lane * kTcAtomCols,
                          static_cast<int>(t.row0), &ctl->full[pi], pol);
            issued |= 1u << pi;
            last_par = (last_par & ~(1u << pi)) | (pe_par << pi);
            if (++pi == p.n_pages) {
              pi = 0;
              pe_par ^= 1u;
            }
            top_up(1);
          }
        }
      }
    } else if (!TC && is_gemv(t.type)) {
      const Geo geo = gemv_geo(p, t, B);
      const int pitch = row_pitch_bytes(geo.kp);
      for (int xc0 = geo.k0; xc0 < geo.k0 + geo.Kt && ok; xc0 += geo.kx) {
        const int xend = min(geo.k0 + geo.Kt, xc0 + geo.kx);
        for (int m = 0; m < t.n_m && ok; ++m) {
          const __nv_bfloat16 *W;
          int row, rv;
          gemv_tile(p, t, m, W, row, rv);
          for (int c0 = xc0; c0 < xend; c0 += geo.kp) {
            const int nc = min(geo.kp, xend - c0);
            if (lane == 0) okl = lwait(&ctl->empty[pi], pe_par ^ 1u, 0xfff10000u, true);
            ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
            if (!ok) break;
            uint8_t *pg = pages + static_cast<size_t>(pi) * p.page_bytes;
            if (TM) {
              // 512-column boxes of 16 rows (rows past the matrix arrive as
              // zeros), each landing as four tcgen05.cp sources
              const int nb = nc / kTmBoxCols;
              const bool up = t.type == T_GATEUP && m >= (t.n_m >> 1);
              const void *map = static_cast<const uint8_t *>(p.tmaps) +
                                static_cast<size_t>(up ? t.map1 : t.map0) * 128;
              if (lane == 0) {
                mbar_arrive_expect_tx(&ctl->full[pi], static_cast<uint32_t>(nb * kTmBoxBytes));
                mv_kind |= 1u << pi;
                mv_ng = (mv_ng & ~(15ull << (4 * pi))) | (static_cast<uint64_t>(nb - 1) << (4 * pi));
                ++mv_n;
              }
              __syncwarp();
              if (lane < nb)
                tma_load_3d(pg + lane * kTmBoxBytes, map, 0, row, (c0 + lane * kTmBoxCols) / 64,
                            &ctl->full[pi], pol);
            } else if (W4 && is_w4_task(p.w4, t.type)) {
              // 4-bit: the row tile's packed blocks of these columns are
              // contiguous -- one bulk copy
              const uint32_t bytes = static_cast<uint32_t>(nc / MK_W4_BLOCK_COLS) * MK_W4_BLOCK_BYTES;
              const uint8_t *src = reinterpret_cast<const uint8_t *>(W) +
                                   (static_cast<size_t>(row / 16) * (geo.K / MK_W4_BLOCK_COLS) +
                                    c0 / MK_W4_BLOCK_COLS) * MK_W4_BLOCK_BYTES;
              if (lane == 0) {
                mbar_arrive_expect_tx(&ctl->full[pi], bytes);
                bulk_load(pg, src, bytes, &ctl->full[pi], pol);
              }
              __syncwarp();
            } else {
              if (lane == 0) mbar_arrive_expect_tx(&ctl->full[pi], static_cast<uint32_t>(rv * nc * 2));
              __syncwarp();
              if (lane < rv) {
                const __nv_bfloat16 *src = W + (static_cast<size_t>(row + lane) * geo.K + c0);
                bulk_load(pg + lane * pitch, src, static_cast<uint32_t>(nc * 2), &ctl->full[pi], pol);
              }
            }
            issued |= 1u << pi;
            last_par = (last_par & ~(1u << pi)) | (pe_par << pi);
            if (++pi == p.n_pages) {
              pi = 0;
              pe_par ^= 1u;
            }
            top_up(1);
          }
        }
      }
    } else if (t.type == T_ATTN && info.b >= 0) {
      const int l = t.layer;
      if (p.kv_tasks) {
        // the chunk's pages may hold K/V that this step's K/V tasks write:
        // copy them only once those are complete, and order the copies
        // (async proxy) after the acquired writes
        if (lane == 0)
          okl = lwait_event(static_cast<uint32_t>(ev_attn_input(p, l, info.g)),
                            static_cast<uint32_t>(attn_input_count(p)), static_cast<uint32_t>(tix));
        ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
        if (!ok) break;
        __syncwarp();
        asm volatile("fence.proxy.async.global;" ::: "memory");
      }
      const int P = p.page_size, d = p.d;
      const size_t kvpage_elems = static_cast<size_t>(P) * d;
      const uint32_t kvpage_bytes = static_cast<uint32_t>(kvpage_elems * 2);
      for (int tok0 = info.t0; tok0 < info.t1 && ok; tok0 += p.tpp) {
        const int ntok = min(p.tpp, info.t1 - tok0);
        const int nkv = (ntok + P - 1) / P;
        if (lane == 0) okl = lwait(&ctl->empty[pi], pe_par ^ 1u, 0xfff20000u, true);
        if (TM && lane == 0) {   // an attention page: the mover passes it over
          mv_kind &= ~(1u << pi);
          ++mv_n;
        }
        ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
        if (!ok) break;
        uint8_t *pg = pages + static_cast<size_t>(pi) * p.page_bytes;
        if (lane == 0) mbar_arrive_expect_tx(&ctl->full[pi], 2u * nkv * kvpage_bytes);
        __syncwarp();
        const int j = lane & 15;
        const int lp0 = info.t0 / P, jbase = (tok0 - info.t0) / P;
        if (AMMA) {
          // TMA tensor copies, 64 dims x P tokens per box, 128-byte swizzle:
          // the layout the attention's ldmatrix fragment loads read without
          // bank conflicts
          const int na = d / 64;
          const uint8_t *maps = static_cast<const uint8_t *>(p.kvmaps);
          const int n_copies = nkv * 2 * na;
          for (int i0 = 0; i0 < n_copies; i0 += 32) {
            const int idx = i0 + lane;
            const bool act = idx < n_copies;
            const int jj = act ? idx / (2 * na) : 0, kvi = (idx / na) & 1, a = idx % na;
            const int jg = jbase + jj;   // page of the chunk
            int ph = __shfl_sync(0xffffffffu, ph_pre, jg & 31);
            if (!act) continue;
            if (jg >= 32) ph = kv_phys_page(p, info.b, lp0 + jg);
            if (ph < 0) {
              raise_error(p, MK_ERR_RANGE, static_cast<uint32_t>(tix), 0xfffffffdu,
                          static_cast<uint32_t>(info.b));
              ph = 0;  // keep the copy in bounds; the step is being abandoned
            }
            uint8_t *dst = pg + (kvi ? static_cast<size_t>(p.tpp) * d * 2 : 0) +
                           static_cast<size_t>(jj) * kvpage_bytes + a * (P * 128);
            tma_load_2d(dst, maps + static_cast<size_t>(2 * l + kvi) * 128, a * 64,
                        (ph * p.Hkv + info.g) * P, &ctl->full[pi], pol);
          }
        } else {
          const int jg = jbase + j;   // page of the chunk
          int ph = __shfl_sync(0xffffffffu, ph_pre, jg & 31);
          if (j < nkv) {
            if (jg >= 32) ph = kv_phys_page(p, info.b, lp0 + jg);
            if (ph < 0) {
              raise_error(p, MK_ERR_RANGE, static_cast<uint32_t>(tix), 0xfffffffdu,
                          static_cast<uint32_t>(info.b));
              ph = 0;  // keep the copy in bounds; the step is being abandoned
            }
            const size_t off = (static_cast<size_t>(ph) * p.Hkv + info.g) * kvpage_elems;
            if (lane < 16) {
              bulk_load(pg + j * kvpage_bytes, p.k_pages[l] + off, kvpage_bytes, &ctl->full[pi],
                        pol);
            } else {
              bulk_load(pg + static_cast<size_t>(p.tpp) * d * 2 + j * kvpage_bytes,
                        p.v_pages[l] + off, kvpage_bytes, &ctl->full[pi], pol);
            }
          }
        }
        issued |= 1u << pi;
        last_par = (last_par & ~(1u << pi)) | (pe_par << pi);
        if (++pi == p.n_pages) {
          pi = 0;
          pe_par ^= 1u;
        }
        top_up(1);
      }
    }
    if (lane == 0) trace_mark(p, tix, 2);
    if (!ok) break;
  }

  if constexpr (TM) {
    // the compute warps still need every page issued: move the rest (bounded)
    if (ok && lane == 0) {
      const uint64_t t0 = gtimer();
      while (mv_n > 0) {
        service();
        if (ctl->cta_abort != 0 || gtimer() - t0 > static_cast<uint64_t>(p.wait_limit_ns) * 2) {
          if (ctl->cta_abort == 0) raise_error(p, MK_ERR_TIMEOUT, 0xfffffff1u, 0xfffffffeu, 0u);
          ok = false;
          break;
        }
      }
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
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
  if constexpr (TM) {
    // no copy into tensor memory may still run when the CTA frees it: the
    // last commit tracks every earlier copy (bounded wait)
    if (lane == 0 && last_slot >= 0) {
      const uint64_t t0 = gtimer();
      while (!mbar_try_wait(tm_full_bar(smem, p, last_slot), last_tpar)) {
        if (gtimer() - t0 > static_cast<uint64_t>(p.wait_limit_ns) * 4) break;
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
// activation fragment follows as well).  The staged activation holds, per
// 8-column block, 8 bf16 "hi" values then 8 bf16 "lo" values (hi + lo == x to
// ~2^-16).  n-tile nt serves sequences 4nt..4nt+3: lanes with g < 4 supply
// the hi block of sequence 4nt+g (mma column g), lanes with g >= 4 the lo
// block of sequence 4nt+g-4 (column g), so one mma per k-step covers both
// halves and the epilogue adds column n+4 to column n.
template <int NN>
__device__ __forceinline__ void page_mma(float (&acc)[NN][4], const uint8_t *pg, int pitch, int nc,
                                         const uint8_t *xs, int xpitch, int xcol0, int B, int warp,
                                         int lane) {
  const int g = lane >> 2, q = lane & 3;
  const int groups = (nc + 31) >> 5;
  const int xhalf = (g >> 2) * 16;   // 0: hi block, 16: lo block
  float c1[NN][4];                   // second k-step: an independent chain
#pragma unroll
  for (int nt = 0; nt < NN; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) c1[nt][e] = 0.f;
  const uint8_t *wrow0 = pg + g * pitch + q * 16;
  const uint8_t *wrow1 = wrow0 + 8 * pitch;
#pragma unroll 2
  for (int grp = warp; grp < groups; grp += kComputeWarps) {
    const int c = grp * 32 + q * 8;
    const bool valid = c < nc;
    uint4 wa = make_uint4(0, 0, 0, 0), wb = make_uint4(0, 0, 0, 0);
    if (valid) {
      wa = *reinterpret_cast<const uint4 *>(wrow0 + grp * 64);
      wb = *reinterpret_cast<const uint4 *>(wrow1 + grp * 64);
    }
#pragma unroll
    for (int nt = 0; nt < NN; ++nt) {
      const int b = nt * 4 + (g & 3);
      uint4 xv = make_uint4(0, 0, 0, 0);
      if (valid && b < B)
        xv = *reinterpret_cast<const uint4 *>(xs + b * xpitch + (xcol0 + c) * 4 + xhalf);
      mma_bf16(acc[nt], wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
      mma_bf16(c1[nt], wa.z, wb.z, wa.w, wb.w, xv.z, xv.w);
    }
  }
#pragma unroll
  for (int nt = 0; nt < NN; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] += c1[nt][e];
}

// One 4-bit page (a 16-row tile over nc columns, nc / 1024 packed blocks)
// against the staged activation.  The lane (g, q) reads, per 32-column
// group, 8 bytes: the codes of row g and of row g + 8 at columns 8 q .. 8 q + 7
// (the packed order), and the two rows' scales of the group's 128 columns.
// A code pair becomes a bf16 pair exactly: OR-ing the nibble into the bits of
// 128.0 gives 128 + code, minus 136 gives code - 8 (small integers are exact
// in bf16), and one bf16 multiply by the scale rounds the product once, as
// the 4-bit format defines the weight.  Then the same mma as a bf16 page.
template <int NN>
__device__ __forceinline__ void page_mma_w4(float (&acc)[NN][4], const uint8_t *pg, int nc,
                                            const uint8_t *xs, int xpitch, int xcol0, int B,
                                            int warp, int lane) {
  const int g = lane >> 2, q = lane & 3;
  const int groups = nc >> 5;
  const int xhalf = (g >> 2) * 16;   // 0: hi block, 16: lo block
  const __nv_bfloat162 k136 = __floats2bfloat162_rn(136.f, 136.f);
  float c1[NN][4];
#pragma unroll
  for (int nt = 0; nt < NN; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) c1[nt][e] = 0.f;
#pragma unroll 2
  for (int grp = warp; grp < groups; grp += kComputeWarps) {
    const int blk = grp >> 5, sub = grp & 31;
    const uint8_t *bp = pg + blk * MK_W4_BLOCK_BYTES;
    const uint2 cw = *reinterpret_cast<const uint2 *>(bp + 256 + sub * 256 + lane * 8);
    const __nv_bfloat16 *scl = reinterpret_cast<const __nv_bfloat16 *>(bp) + (sub >> 2) * 16;
    const __nv_bfloat162 s0 = __bfloat162bfloat162(scl[g]);
    const __nv_bfloat162 s1 = __bfloat162bfloat162(scl[g + 8]);
    uint32_t wa[4], wb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t na = ((cw.x >> (4 * k)) & 0x000F000Fu) | 0x43004300u;
      const uint32_t nb = ((cw.y >> (4 * k)) & 0x000F000Fu) | 0x43004300u;
      const __nv_bfloat162 va = __hmul2(__hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&na), k136), s0);
      const __nv_bfloat162 vb = __hmul2(__hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&nb), k136), s1);
      wa[k] = *reinterpret_cast<const uint32_t *>(&va);
      wb[k] = *reinterpret_cast<const uint32_t *>(&vb);
    }
    const int c = grp * 32 + q * 8;
#pragma unroll
    for (int nt = 0; nt < NN; ++nt) {
      const int b = nt * 4 + (g & 3);
      uint4 xv = make_uint4(0, 0, 0, 0);
      if (b < B) xv = *reinterpret_cast<const uint4 *>(xs + b * xpitch + (xcol0 + c) * 4 + xhalf);
      mma_bf16(acc[nt], wa[0], wb[0], wa[1], wb[1], xv.x, xv.y);
      mma_bf16(c1[nt], wa[2], wb[2], wa[3], wb[3], xv.z, xv.w);
    }
  }
#pragma unroll
  for (int nt = 0; nt < NN; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] += c1[nt][e];
}

// One 16-row weight page staged in tensor memory (slot columns at `slot`)
// against the staged activation.  Box bx (512 columns) sits at slot columns
// 32 bx .. 32 bx + 31: 64-column block cb of the box in lanes 16 cb ..
// 16 cb + 15, its 16-column slice j in columns 32 bx + 8 j .. + 7.  A
// 16x256b load there is the slice's mma A fragment for the k order
// (4q, 4q + 1 | 4q + 2, 4q + 3) of lane quarter q, which the activation
// fragment follows (columns 4q .. 4q + 3 of the slice, 8 bytes of the staged
// hi or lo half).  A warp reads only its lane quarter qq of tensor memory:
// blocks 2 qq and 2 qq + 1 of every box, its four slices per load; the two
// warps of quarters 1 and 2 take alternate boxes.
template <int NN>
__device__ __forceinline__ void page_tm(float (&acc)[NN][4], uint32_t slot, int nc,
                                        const uint8_t *xs, int xpitch, int xcol0, int B, int warp,
                                        int lane) {
  const int g = lane >> 2, q = lane & 3;
  const int qq = (warp + 1) & 3;
  const bool pair = qq == 1 || qq == 2;
  const int b0 = (pair && warp >= 4) ? 1 : 0;
  const int bstep = pair ? 2 : 1;
  const int nbox = nc / kTmBoxCols;
  const int xq = (8 * (q >> 1)) * 4 + (q & 1) * 8 + (g >> 2) * 16;   // bytes, within a slice
  float c1[NN][4];
#pragma unroll
  for (int nt = 0; nt < NN; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) c1[nt][e] = 0.f;
  for (int bx = b0; bx < nbox; bx += bstep) {
    uint32_t a[2][16];
#pragma unroll
    for (int h = 0; h < 2; ++h)
      tm_ld16x256_x4(slot + (static_cast<uint32_t>(32 * qq + 16 * h) << 16) + 32u * bx, a[h]);
    tm_wait_ld();
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = kTmBoxCols * bx + 64 * (2 * qq + h) + 16 * j;
#pragma unroll
        for (int nt = 0; nt < NN; ++nt) {
          const int b = nt * 4 + (g & 3);
          uint2 xv = make_uint2(0u, 0u);
          if (b < B) xv = *reinterpret_cast<const uint2 *>(xs + b * xpitch + (xcol0 + col) * 4 + xq);
          if (j & 1)
            mma_bf16(c1[nt], a[h][4 * j], a[h][4 * j + 2], a[h][4 * j + 1], a[h][4 * j + 3], xv.x,
                     xv.y);
          else
            mma_bf16(acc[nt], a[h][4 * j], a[h][4 * j + 2], a[h][4 * j + 1], a[h][4 * j + 3], xv.x,
                     xv.y);
        }
      }
  }
#pragma unroll
  for (int nt = 0; nt < NN; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] += c1[nt][e];
}

// All lanes of a compute warp wait (bounded) for a full ring page; the
// result is warp-uniform.
__device__ __forceinline__ bool warp_wait_page(const Params &p, Ctl *ctl, uint64_t *bar,
                                               uint32_t parity, uint32_t where) {
  const bool done = mbar_try_wait(bar, parity);
  if (__all_sync(0xffffffffu, done)) return true;
  int ok = 1;
  if (!done) ok = wait_mbar(p, ctl, bar, parity, where, 2) ? 1 : 0;
  return __all_sync(0xffffffffu, ok) != 0;
}

struct ComputeState {
  int pi = 0;
  uint32_t pg_par = 0;
  int tslot = 0;                 // tensor-memory staging: next page slot and its round parity
  uint32_t tpar = 0;
  uint32_t xuse = 0;             // tensor-core path: staged chunks so far (buffer = xuse & 1)
  uint32_t accuse = 0;           // tensor-core path: tasks whose accumulators were read
  uint32_t x_par = 0;            // phase of the activation-copy barrier
  uint32_t xkey = 0xffffffffu;   // (layer, type) of the staged activation
  uint32_t sat_ev = kNoEvent;    // last (event, count) known satisfied
  uint32_t sat_cnt = 0;
  GroupSync gs;
};

// Activation source of a GEMV task: row stride, and the RMSNorm gain for the
// normed inputs (QKV, gate/up, LM head read the residual stream h).
__device__ __forceinline__ void gemv_source(const Params &p, const Task &t, const float *&src,
                                            int &stride, const __nv_bfloat16 *&gain) {
  gain = t.gain;
  switch (t.type) {
    case T_QKV:
    case T_GATEUP:
    case T_LMHEAD: src = p.h; stride = p.H; break;
    case T_OPROJ: src = p.o; stride = p.Hq * p.d; break;
    default: src = p.u; stride = p.F; break;
  }
}

// RMSNorm gain blocks (8 bf16 each) a compute thread scales while staging:
// column blocks ctid, ctid + kComputeThreads, ...  Gains are static weights,
// so they are requested before the task waits for its input and arrive
// during the wait.
constexpr int kGainPre = 4;   // covers inputs up to 4 x 192 x 8 = 6144 columns
struct GainPre {
  uint4 g[kGainPre];
};

__device__ __forceinline__ void prefetch_gain(const __nv_bfloat16 *gain, int xc0, int xlen,
                                              int ctid, GainPre &gp) {
  const int nblk = xlen / 8;
#pragma unroll
  for (int j = 0; j < kGainPre; ++j) {
    const int k = ctid + j * kComputeThreads;
    gp.g[j] = (gain != nullptr && k < nblk)
                  ? __ldg(reinterpret_cast<const uint4 *>(gain + xc0 + k * 8))
                  : make_uint4(0, 0, 0, 0);
  }
}

// One staged 8-column block: 8 fp32 values -> [8 x bf16 hi | 8 x bf16 lo] of
// x * g (hi + lo == x * g to ~2^-16), in place.  Returns the sum of squares of
// the raw values (before the gain).
__device__ __forceinline__ float stage_block(uint8_t *blk8, bool has_gain, uint4 gw) {
  float4 *blk = reinterpret_cast<float4 *>(blk8);
  const float4 x0 = blk[0], x1 = blk[1];
  float v[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) s += v[e] * v[e];
  if (has_gain) {
    const uint32_t gg[4] = {gw.x, gw.y, gw.z, gw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] *= bf_lo(gg[e]);
      v[2 * e + 1] *= bf_hi(gg[e]);
    }
  }
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat16 h0, l0, h1, l1;
    split_bf16(v[2 * e], h0, l0);
    split_bf16(v[2 * e + 1], h1, l1);
    hw[e] = pack2(h0, h1);
    lw[e] = pack2(l0, l1);
  }
  uint4 *o = reinterpret_cast<uint4 *>(blk8);
  o[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  o[1] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  return s;
}

// Stage activation columns [xc0, xc0 + xlen) of every sequence in shared
// memory: the leader issues one bulk copy per sequence right after the input
// event (one L2 round trip for the whole operand); then one parallel pass
// turns each 8-column block into bf16 hi/lo of x * g and, for normed inputs,
// adds each sequence's sum of squares over the chunk to ss[b] (per-warp
// partials summed in warp order).  The RMSNorm scale is applied to the
// task's outputs, since W (x * g * r) = r * W (x * g).  `gp`, when given,
// holds this thread's gain blocks for the chunk.
__device__ bool stage_x(const Params &p, Ctl *ctl, uint8_t *smem, const Task &t, int xc0,
                        int xlen, int xpitch, int B, int ctid, ComputeState &st, bool first,
                        const GainPre *gp) {
  const float *src;
  int stride;
  const __nv_bfloat16 *gain;
  gemv_source(p, t, src, stride, gain);
  bool okl = true;
  if (ctid == 0) {
    // the rows were written by other SMs (generic proxy) and acquired by this
    // thread; order them, and this CTA's earlier reads of the area, before
    // the bulk copy (async proxy)
    asm volatile("fence.proxy.async.global;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(&ctl->xbar, static_cast<uint32_t>(B * xlen * 4));
    for (int b = 0; b < B; ++b)
      bulk_load_plain(smem + p.off_x + b * xpitch, src + static_cast<size_t>(b) * stride + xc0,
                      static_cast<uint32_t>(xlen * 4), &ctl->xbar);
    okl = wait_mbar(p, ctl, &ctl->xbar, st.x_par, 0xfff80000u, 2);
    if (!okl) {
      // leaving on an abort: let the copy land before this CTA can exit
      const uint64_t t0 = gtimer();
      while (!mbar_try_wait(&ctl->xbar, st.x_par)) {
        if (gtimer() - t0 > static_cast<uint64_t>(p.wait_limit_ns) * 4) break;
      }
    }
  }
  if (!st.gs.share(ctl, ctid, okl)) return false;
  mbar_try_wait(&ctl->xbar, st.x_par);
  st.x_par ^= 1u;
  const int warp = ctid >> 5, lane = ctid & 31;
  const bool has_gain = gain != nullptr;
  const int nblk = xlen / 8;
  for (int b = 0; b < B; ++b) {
    uint8_t *row = smem + p.off_x + b * xpitch;
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < kGainPre; ++j) {
      const int k = ctid + j * kComputeThreads;
      if (k < nblk) {
        const uint4 gw = !has_gain ? make_uint4(0, 0, 0, 0)
                         : gp != nullptr ? gp->g[j]
                                         : __ldg(reinterpret_cast<const uint4 *>(gain + xc0 + k * 8));
        s += stage_block(row + k * 32, has_gain, gw);
      }
    }
    for (int k = ctid + kGainPre * kComputeThreads; k < nblk; k += kComputeThreads) {
      const uint4 gw = has_gain ? __ldg(reinterpret_cast<const uint4 *>(gain + xc0 + k * 8))
                                : make_uint4(0, 0, 0, 0);
      s += stage_block(row + k * 32, has_gain, gw);
    }
    if (has_gain) {
      s = warp_sum(s);
      if (lane == 0) ctl->red8[warp][b] = s;
    }
  }
  if (has_gain) {
    compute_bar();
    if (ctid < B) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) s += ctl->red8[w][ctid];
      ctl->ss[ctid] = (first ? 0.f : ctl->ss[ctid]) + s;
    }
  }
  compute_bar();
  return true;
}

// NN = batch n-tiles (1: B <= 4, 2: B <= 8, 4: B <= 16).  A task holds at
// most kMaxMTiles / NN row tiles (the plan caps rows per task) so that the
// accumulators stay in registers.
template <int NN, bool W4, bool TM, int MT = kMaxMTiles / NN>
__device__ bool gemv_task(const Params &p, Ctl *ctl, uint8_t *smem, const Slot &S,
                          ComputeState &st, float *out, int ctid) {
  const Task &t = S.t;
  const int B = p.batch;
  const int warp = ctid >> 5, lane = ctid & 31;
  const Geo geo = gemv_geo(p, t, B);
  const int pitch = row_pitch_bytes(geo.kp);
  const int xstride = x_row_bytes(geo.kx) / 4;
  const uint8_t *pages = smem + p.off_pages;
  const uint8_t *xs = smem + p.off_x;
  const uint32_t key = (static_cast<uint32_t>(t.layer) << 16) | (static_cast<uint32_t>(t.type) << 8) |
                       t.ksplit;
  const float *src;
  int stride;
  const __nv_bfloat16 *gain;
  gemv_source(p, t, src, stride, gain);
  const bool restage = !(geo.whole && st.xkey == key);
  GainPre gp;
  if (gain != nullptr && restage) prefetch_gain(gain, geo.k0, min(geo.kx, geo.Kt), ctid, gp);

  if (!S.dep_ok && (t.dep_event != st.sat_ev || t.dep_count != st.sat_cnt)) {
    bool okl = true;
    if (ctid == 0) okl = wait_event(p, ctl, t.dep_event, t.dep_count, S.idx);
    if (!st.gs.share(ctl, ctid, okl)) return false;
  }
  st.sat_ev = t.dep_event;
  st.sat_cnt = t.dep_count;
  if (ctid == 0) trace_mark(p, S.idx, 4);

  float acc[MT][NN][4];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int n = 0; n < NN; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[m][n][e] = 0.f;

  bool bad = false;   // this warp gave up waiting for a page (warp-uniform)
  for (int xc0 = geo.k0; xc0 < geo.k0 + geo.Kt; xc0 += geo.kx) {
    const int xend = min(geo.k0 + geo.Kt, xc0 + geo.kx);
    if (!(geo.whole && st.xkey == key)) {
      // a later chunk overwrites the staging area: every compute warp must be
      // done with the previous chunk's pages (warps move through the pages
      // independently)
      if (xc0 != geo.k0) compute_bar();
      if (!stage_x(p, ctl, smem, t, xc0, xend - xc0, xstride * 4, B, ctid, st, xc0 == geo.k0,
                   (gain != nullptr && xc0 == geo.k0) ? &gp : nullptr))
        return false;
      st.xkey = geo.whole ? key : 0xffffffffu;
    }
    if (ctid == 0 && xc0 == geo.k0) trace_mark(p, S.idx, 5);
    // Each warp waits for a page by itself (bounded) and releases its share
    // of it, so warps are not locked together page by page.  A warp whose
    // wait fails stops computing, flags the CTA, and the warps agree on the
    // outcome once, after the last page.
    for (int m = 0; m < t.n_m; ++m) {
      for (int c0 = xc0; c0 < xend; c0 += geo.kp) {
        const int nc = min(geo.kp, xend - c0);
        if constexpr (TM) {
          // the page waits in a tensor-memory slot (the loader freed its ring
          // page once it was copied there)
          if (!bad && !warp_wait_page(p, ctl, tm_full_bar(smem, p, st.tslot), st.tpar, 0xfff30000u)) {
            bad = true;
            if (lane == 0) {
              ctl->cbad = 1;
              ctl->cta_abort = 1;
            }
          }
          if (!bad) {
            tc_fence_after();
            const uint32_t slot = ctl->tmem + static_cast<uint32_t>(st.tslot * kTmSlotCols);
            switch (m) {
#define MK_TM_CASE(M)                                                                          \
  case M:                                                                                      \
    if (M < MT) page_tm<NN>(acc[M < MT ? M : 0], slot, nc, xs, xstride * 4, c0 - xc0, B, warp, lane); \
    break;
              MK_TM_CASE(0)
              MK_TM_CASE(1)
              MK_TM_CASE(2)
              MK_TM_CASE(3)
              MK_TM_CASE(4)
              MK_TM_CASE(5)
              MK_TM_CASE(6)
              MK_TM_CASE(7)
#undef MK_TM_CASE
              default: break;
            }
            tc_fence_before();
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(tm_empty_bar(smem, p, st.tslot));
          if (++st.tslot == kTmSlots) {
            st.tslot = 0;
            st.tpar ^= 1u;
          }
          if (++st.pi == p.n_pages) {
            st.pi = 0;
            st.pg_par ^= 1u;
          }
          continue;
        }
        if (!bad && !warp_wait_page(p, ctl, &ctl->full[st.pi], st.pg_par, 0xfff30000u)) {
          bad = true;
          if (lane == 0) {
            ctl->cbad = 1;
            ctl->cta_abort = 1;
          }
        }
        if (bad) {
          if (++st.pi == p.n_pages) {
            st.pi = 0;
            st.pg_par ^= 1u;
          }
          continue;
        }
        const uint8_t *pg = pages + static_cast<size_t>(st.pi) * p.page_bytes;
        const bool w4 = W4 && is_w4_task(p.w4, t.type);
        switch (m) {
#define MK_PAGE_CASE(M)                                                                        \
  case M:                                                                                      \
    if (M < MT) {                                                                              \
      if (w4)                                                                                  \
        page_mma_w4<NN>(acc[M < MT ? M : 0], pg, nc, xs, xstride * 4, c0 - xc0, B, warp, lane); \
      else                                                                                     \
        page_mma<NN>(acc[M < MT ? M : 0], pg, pitch, nc, xs, xstride * 4, c0 - xc0, B, warp,   \
                     lane);                                                                    \
    }                                                                                          \
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

  // every warp has passed all pages (or given up): one uniform decision
  compute_bar();
  if (ctl->cbad != 0) return false;
  if (gain != nullptr) {
    if (ctid < B) ctl->rs[ctid] = 1.0f / sqrtf(ctl->ss[ctid] / static_cast<float>(geo.K) + p.eps);
    compute_bar();
  }
  // cross-warp reduction, one 16-row tile at a time, fixed warp order; for
  // sequence b = 4 nt + j a warp contributes its columns j (hi) and j + 4 (lo)
  float *red = reinterpret_cast<float *>(smem + p.off_red);
  constexpr int NC = NN * 8;
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int m = 0; m < MT; ++m) {
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
    for (int e = ctid; e < 16 * 4 * NN; e += kComputeThreads) {
      const int row = e / (4 * NN), b = e % (4 * NN);
      const int col = (b >> 2) * 8 + (b & 3);
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) {
        const float *rr = red + (w * 16 + row) * NC + col;
        s += rr[0] + rr[4];
      }
      if (b < B) out[b * p.out_stride + m * 16 + row] = gain != nullptr ? s * ctl->rs[b] : s;
    }
    compute_bar();
  }
  return true;
}

// ============================================================================
// compute warps: GEMV on the tensor cores (tcgen05)
// ============================================================================
//
// A task is n_m (1, or 2 for gate/up) tiles of 128 weight rows over its K
// range.  Thread 0 issues the MMAs: D[128 x N] += W[128 x 16] * X[N x 16]^T
// per 16 columns, accumulating in tensor memory (one N-column accumulator per
// tile).  X holds the activation as bf16 rows: sequences 0..bpad-1 carry the
// high parts of x * g and rows bpad..2*bpad-1 the low parts (hi + lo == x * g
// to ~2^-16), so D[:, b] + D[:, bpad + b] is the fp32-accurate product.
// Warps 2-6 stage the activation chunk by chunk into two buffers, one chunk
// ahead of the MMAs.  After the last MMA, warps 1-4 (tensor-memory lane
// quarters 1, 2, 3, 0) read the accumulators and hand the task's rows to the
// storer, scaled by the RMSNorm factor for normed inputs.

// Tensor-core path: store v (already times the consumer's gain) as column
// `col` of sequence b in a staged-input buffer [2 * bpad][K]: its bf16 high
// half in row b, the low half (v - high, rounded) in row bpad + b.
__device__ __forceinline__ void put_staged(__nv_bfloat16 *xs, int bpad, int K, int b, int col,
                                           float v) {
  __nv_bfloat16 hi, lo;
  split_bf16(v, hi, lo);
  xs[static_cast<size_t>(b) * K + col] = hi;
  xs[static_cast<size_t>(bpad + b) * K + col] = lo;
}

// Tensor-core path, normed inputs: the sums of h^2 per 128 rows that the
// producers of h wrote -> each sequence's RMSNorm scale in ctl->rs.  One
// warp; every load is issued before the first sum (fixed order: per lane
// over its tiles, then a warp tree).
template <int BP>
__device__ void tc_norm_scales(const Params &p, Ctl *ctl, const float *ssq, int B, int lane) {
  const int n = (p.H + kTcRows - 1) / kTcRows;
  float v[BP];
#pragma unroll
  for (int b = 0; b < BP; ++b) v[b] = 0.f;
  for (int i = lane; i < n; i += 32)
#pragma unroll
    for (int b = 0; b < BP; ++b)
      if (b < B) v[b] += __ldcg(ssq + static_cast<size_t>(i) * p.max_batch + b);
#pragma unroll
  for (int b = 0; b < BP; ++b) {
    const float s = warp_sum(v[b]);
    if (lane == 0 && b < B) ctl->rs[b] = 1.0f / sqrtf(s / static_cast<float>(p.H) + p.eps);
  }
}

// Split-K partials and tile counters of a tensor-core task (QKV and down
// share one area; O and gate/up have their own).
struct TcSplit {
  float *kp;
  int rstride;          // floats per sequence row of the partial area
  size_t pstride;       // floats per part
  uint32_t *ctr;
  int grow0;            // the task's first row in its operator's row space
};
__device__ __forceinline__ TcSplit tc_split(const Params &p, const Task &t) {
  TcSplit s;
  const int qbase = t.aux == 0 ? 0 : (t.aux == 1 ? p.Hq * p.d : (p.Hq + p.Hkv) * p.d);
  s.grow0 = static_cast<int>(t.row0) + (t.type == T_QKV ? qbase : 0);
  s.kp = p.kpart;
  s.rstride = p.H;
  s.ctr = p.tile_ctr;
  if (t.type == T_QKV) {
    s.rstride = p.NQKV;
  } else if (t.type == T_OPROJ) {
    s.kp = p.kpart_o;
    s.ctr = p.tile_ctr_o;
  } else if (t.type == T_GATEUP) {
    s.kp = p.kpart2;
    s.rstride = 2 * p.F;
    s.ctr = p.tile_ctr2;
  }
  s.pstride = static_cast<size_t>(p.max_batch) * s.rstride;
  s.ctr += s.grow0 / 16;
  return s;
}

template <int NT>   // accumulator columns / 16: 1 (N = 16, batch <= 8) or 2 (N = 32)
__device__ bool gemv_task_tc(const Params &p, Ctl *ctl, uint8_t *smem, const Slot &S,
                             ComputeState &st, float *out, int ctid) {
  constexpr int BP = 8 * NT;   // tc_bpad of a plan with this NT
  const Task &t = S.t;
  const int B = p.batch;
  const int warp = ctid >> 5, lane = ctid & 31;
  const TcGeo g = tc_geo(p, t);
  const float *src;
  int stride;
  const __nv_bfloat16 *gain;
  gemv_source(p, t, src, stride, gain);
  const bool normed = gain != nullptr;

  if (!S.dep_ok && (t.dep_event != st.sat_ev || t.dep_count != st.sat_cnt)) {
    bool okl = true;
    if (ctid == 0) okl = wait_event(p, ctl, t.dep_event, t.dep_count, S.idx);
    if (!st.gs.share(ctl, ctid, okl)) return false;
  }
  st.sat_ev = t.dep_event;
  st.sat_cnt = t.dep_count;
  if (ctid == 0) trace_mark(p, S.idx, 4);

  const int nchunks = (g.Kt + p.tc_kx - 1) / p.tc_kx;
  uint8_t *xbase = smem + p.off_x;
  if (ctid >= 32 && ctid < 64) {
    // ---- warp 2: the RMSNorm scales (read by the epilogue) ----
    if (normed) tc_norm_scales<BP>(p, ctl, t.type == T_GATEUP ? p.ssq_mlp : p.ssq_attn, B, lane);
  } else if (ctid == 0) {
    // ---- thread 0: the activation chunks (TMA copies of the staged input,
    // one chunk ahead, two buffers) and the MMAs ----
    const int kind = t.type == T_QKV || t.type == T_LMHEAD ? XS_ATTN
                     : t.type == T_GATEUP                  ? XS_MLP
                     : t.type == T_OPROJ                   ? XS_O
                                                           : XS_U;
    const void *xmap = static_cast<const uint8_t *>(p.tmaps) + static_cast<size_t>(p.xs_map0 + kind) * 128;
    const uint64_t xpol = l2_evict_last_policy();
    const uint32_t idesc = mma_idesc_bf16(kTcRows, p.tc_n);
    const uint32_t tmem = ctl->tmem;
    const uint32_t pages = smem_u32(smem + p.off_pages);
    const uint32_t xs0 = smem_u32(xbase);
    const uint32_t xatom = static_cast<uint32_t>(p.tc_n) * 128u;
    bool bad = false;
    // the producers' writes were acquired (input event) by the generic proxy;
    // the tensor copies read through the async proxy
    asm volatile("fence.proxy.async.global;" ::: "memory");
    auto issue_x = [&](int c) {
      const uint32_t u = st.xuse + c;
      const int buf = static_cast<int>(u & 1u);
      const uint32_t use = u >> 1;
      // the buffer's previous chunk: its MMAs must be complete
      if (!bad && use > 0 && !wait_mbar(p, ctl, &ctl->x_free[buf], (use - 1u) & 1u, 0xfff90000u, 2))
        bad = true;
      if (bad) return;
      const int xc0 = g.k0 + c * p.tc_kx;
      const int nbox = min(p.tc_kx, g.k0 + g.Kt - xc0) / kTcAtomCols;
      mbar_arrive_expect_tx(&ctl->x_full[buf], static_cast<uint32_t>(nbox) * xatom);
      for (int a = 0; a < nbox; ++a)
        tma_load_2d(xbase + buf * kTcXBytes + a * xatom, xmap, xc0 + a * kTcAtomCols, 0,
                    &ctl->x_full[buf], xpol);
    };
    issue_x(0);
    bool started0 = false, started1 = false;   // tile 0 / 1 has its first MMA
    for (int c = 0; c < nchunks; ++c) {
      const uint32_t u = st.xuse + c;
      const int buf = static_cast<int>(u & 1u);
      const int xc0 = g.k0 + c * p.tc_kx;
      const int xlen = min(p.tc_kx, g.k0 + g.Kt - xc0);
      if (c + 1 < nchunks) issue_x(c + 1);
      if (!bad && !wait_mbar(p, ctl, &ctl->x_full[buf], (u >> 1) & 1u, 0xfffa0000u, 2)) bad = true;
      tc_fence_after();
      const uint32_t xb = xs0 + static_cast<uint32_t>(buf) * kTcXBytes;
      for (int m = 0; m < t.n_m; ++m) {
        for (int c0 = xc0; c0 < xc0 + xlen; c0 += p.tc_kc) {
          const int nc = min(p.tc_kc, xc0 + xlen - c0);
          if (!bad && !wait_mbar(p, ctl, &ctl->full[st.pi], st.pg_par, 0xfff30000u, 2)) bad = true;
          if (!bad) {
            tc_fence_after();
            const uint32_t pg = pages + static_cast<uint32_t>(st.pi) * p.page_bytes;
            const uint32_t xa0 = xb + static_cast<uint32_t>((c0 - xc0) / kTcAtomCols) * xatom;
            for (int a = 0; a < nc / kTcAtomCols; ++a)
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint64_t ad = sw128_desc(pg + a * kTcAtomBytes + j * 32);
                const uint64_t bd = sw128_desc(xa0 + a * xatom + j * 32);
                tc_mma(tmem + m * p.tc_n, ad, bd, idesc, m == 0 ? started0 : started1);
                if (m == 0) started0 = true; else started1 = true;
              }
            tc_commit(&ctl->empty[st.pi]);   // the page is free once these MMAs complete
          }
          if (++st.pi == p.n_pages) {
            st.pi = 0;
            st.pg_par ^= 1u;
          }
        }
      }
      tc_commit(&ctl->x_free[buf]);
    }
    tc_commit(&ctl->acc_bar);
    // wait for the accumulators (also after a failed wait: no MMA may still
    // be running when the task returns) and for any activation copy in flight
    if (!wait_mbar(p, ctl, &ctl->acc_bar, st.accuse & 1u, 0xfffb0000u, 4)) bad = true;
    if (bad) {
      ctl->cbad = 1;
      ctl->cta_abort = 1;
      for (int c = 0; c < 2; ++c) {   // copies issued but never waited for
        const uint32_t u = st.xuse + nchunks - 1 + c;
        const uint64_t t0 = gtimer();
        while (!mbar_try_wait(&ctl->x_full[u & 1u], (u >> 1) & 1u))
          if (gtimer() - t0 > static_cast<uint64_t>(p.wait_limit_ns)) break;
      }
    }
  }
  if (ctid != 0) {
    // everyone but the MMA issuer: keep the page-ring position in step with it
    for (int c = 0; c < nchunks; ++c) {
      const int xc0 = g.k0 + c * p.tc_kx;
      const int xlen = min(p.tc_kx, g.k0 + g.Kt - xc0);
      const int np = t.n_m * ((xlen + p.tc_kc - 1) / p.tc_kc);
      for (int k = 0; k < np; ++k)
        if (++st.pi == p.n_pages) {
          st.pi = 0;
          st.pg_par ^= 1u;
        }
    }
  }
  st.xuse += static_cast<uint32_t>(nchunks);
  st.xkey = 0xffffffffu;   // the staging area no longer holds an mma.sync operand
  __syncwarp();            // the MMA warp reconverges (thread 0 waited for the accumulators)
  compute_bar();
  if (ctl->cbad != 0) return false;
  if (ctid == 0) trace_mark(p, S.idx, 5);
  tc_fence_after();
  ++st.accuse;

  // ---- epilogue: warps 1-4 read tensor-memory lane quarters 1, 2, 3, 0 ----
  // thread (warp, lane) holds row 32 q + lane of the tile(s): the sum of the
  // hi and lo columns of each sequence, times the RMSNorm scale
  const bool epi = ctid < 128;
  const int q = (warp + 1) & 3;
  const int row = q * 32 + lane;
  const bool vrow = epi && row < static_cast<int>(t.nrows);
  float acc[2][BP];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int b = 0; b < BP; ++b) acc[m][b] = 0.f;
  if (epi) {
    for (int m = 0; m < t.n_m && m < 2; ++m) {
      const uint32_t ta = ctl->tmem + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(m * p.tc_n);
      float v[NT][16];
      tmem_ld16(ta, v[0]);
      if (NT > 1) tmem_ld16(ta + 16, v[NT - 1]);
#pragma unroll
      for (int b = 0; b < BP; ++b) {
        float r = v[b / 16][b % 16] + v[(BP + b) / 16][(BP + b) % 16];
        if (normed && b < B) r *= ctl->rs[b];
        if (m == 0) acc[0][b] = r; else acc[1][b] = r;
      }
    }
  }
  tc_fence_before();

  if (t.type == T_LMHEAD) {
    // logits and argmax: the storer, from the output buffer
    if (vrow)
#pragma unroll
      for (int b = 0; b < BP; ++b)
        if (b < B) out[b * p.out_stride + row] = acc[0][b];
    compute_bar();
    return true;
  }

  // ---- split-K: publish this part; the part that completes the tile sums ----
  const bool split = t.nsplit > 1;
  TcSplit sp{};
  if (split) {
    sp = tc_split(p, t);
    if (vrow)
#pragma unroll
      for (int b = 0; b < BP; ++b)
        if (b < B) {
          float *dst = sp.kp + t.ksplit * sp.pstride + static_cast<size_t>(b) * sp.rstride + sp.grow0 + row;
          __stcg(dst, acc[0][b]);
          if (t.type == T_GATEUP) __stcg(dst + p.F, acc[1][b]);
        }
    compute_bar();
    bool last = false;
    if (ctid == 0) last = atom_add_acq_rel(sp.ctr, 1u) + 1u == static_cast<uint32_t>(t.nsplit);
    if (!st.gs.share(ctl, ctid, last)) return true;   // not the last part: nothing to release
    if (vrow) {
      // the parts in a fixed order (0, 1, ...); this part's own from registers
      float sum[2][BP];
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int b = 0; b < BP; ++b) sum[m][b] = 0.f;
      for (int k = 0; k < t.nsplit; ++k) {
        const float *srck = sp.kp + k * sp.pstride + sp.grow0 + row;
        float v0[BP], v1[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) {
          v0[b] = v1[b] = 0.f;
          if (b < B && k != t.ksplit) {
            v0[b] = __ldcg(srck + static_cast<size_t>(b) * sp.rstride);
            if (t.type == T_GATEUP) v1[b] = __ldcg(srck + static_cast<size_t>(b) * sp.rstride + p.F);
          }
        }
#pragma unroll
        for (int b = 0; b < BP; ++b) {
          sum[0][b] += k == t.ksplit ? acc[0][b] : v0[b];
          sum[1][b] += k == t.ksplit ? acc[1][b] : v1[b];
        }
      }
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int b = 0; b < BP; ++b) acc[m][b] = sum[m][b];
    }
  }

  // ---- the operator's epilogue, one row per thread ----
  float *red = reinterpret_cast<float *>(out);   // [4 warps][BP] per-warp sums of h^2
  if (t.type == T_QKV) {
    // raw q/k/v rows: QK-norm, RoPE and the KV append happen in the attention
    // (or K/V) tasks of the head's KV group
    const int qbase = t.aux == 0 ? 0 : (t.aux == 1 ? p.Hq * p.d : (p.Hq + p.Hkv) * p.d);
    if (vrow)
#pragma unroll
      for (int b = 0; b < BP; ++b)
        if (b < B)
          __stcg(p.qkv + static_cast<size_t>(b) * p.NQKV + qbase + t.row0 + row, acc[0][b]);
  } else if (t.type == T_GATEUP) {
    if (vrow)
#pragma unroll
      for (int b = 0; b < BP; ++b)
        if (b < B) {
          const float gt = acc[0][b];
          const float uv = gt / (1.0f + __expf(-gt)) * acc[1][b];
          __stcg(p.u + static_cast<size_t>(b) * p.F + t.row0 + row, uv);
          put_staged(p.xs[XS_U], BP, p.F, b, t.row0 + row, uv);   // the down projection's input
        }
  } else {
    // O / down: residual add, per-layer dump, the next normed input (x * its
    // gain, staged) and its sums of h^2
    __nv_bfloat16 *xs_next = p.xs[t.type == T_OPROJ ? XS_MLP : XS_ATTN];
    const float gnext = vrow ? __bfloat162float(t.w1[t.row0 + row]) : 0.f;
    float hv[BP];
#pragma unroll
    for (int b = 0; b < BP; ++b)
      hv[b] = (vrow && b < B) ? __ldcg(p.h + static_cast<size_t>(b) * p.H + t.row0 + row) : 0.f;
#pragma unroll
    for (int b = 0; b < BP; ++b) {
      float v = 0.f;
      if (vrow && b < B) {
        v = hv[b] + acc[0][b];
        __stcg(p.h + static_cast<size_t>(b) * p.H + t.row0 + row, v);
        put_staged(xs_next, BP, p.H, b, t.row0 + row, v * gnext);
        if (t.type == T_DOWN && p.hidden_dump != nullptr)
          p.hidden_dump[(static_cast<size_t>(t.layer) * B + b) * p.H + t.row0 + row] = v;
      }
      const float s = warp_sum(v * v);
      if (epi && lane == 0) red[q * BP + b] = s;
    }
    compute_bar();
    if (ctid < B) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) s += red[w * BP + ctid];   // rows 0-31, 32-63, ...
      float *ssq = t.type == T_OPROJ ? p.ssq_mlp : p.ssq_attn;
      __stcg(ssq + static_cast<size_t>(t.row0 / kTcRows) * p.max_batch + ctid, s);
    }
  }
  compute_bar();
  if (ctid == 0) {
    if (split) *sp.ctr = 0u;   // rearm for the next layer / step
    if (t.type == T_QKV) {
      const int head = static_cast<int>(t.aux2);
      const int gq = t.aux == 0 ? head / p.G : (t.aux == 1 ? head - p.Hq : head - p.Hq - p.Hkv);
      red_add_release(p.sync + S_EVENTS + ev_attn_ready(p, t.layer, gq), 1u);
    } else {
      red_add_release(p.sync + S_EVENTS + t.out_event, 1u);
    }
  }
  return true;
}

// ============================================================================
// compute warps: attention over one chunk of one (sequence, KV head)
// ============================================================================

// One head of raw projection values (fp32, d elements at src): optionally an
// RMSNorm over d times `gain`, then optionally RoPE with the table row `cs`
// (pairs (i, i + d/2)).  Lane l < d/4 returns elements 4l..4l+3; the RoPE
// partner of element i sits d/8 lanes away and is fetched by shuffle.  All
// 32 lanes must call it.
template <int D>
__device__ __forceinline__ void head_norm_rope(const float *src, const __nv_bfloat16 *gain,
                                               bool norm, bool rope, const float2 *cs, float eps,
                                               int lane, float (&v)[4]) {
  constexpr int half = D / 2, xo = D / 8;
  const bool active = lane < D / 4;
  const int e0 = lane * 4;
  float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
  if (active) y = __ldcg(reinterpret_cast<const float4 *>(src + e0));
  v[0] = y.x; v[1] = y.y; v[2] = y.z; v[3] = y.w;
  if (norm) {
    float g4[4] = {1.f, 1.f, 1.f, 1.f};
    if (active) {
      const uint2 gw = *reinterpret_cast<const uint2 *>(gain + e0);
      g4[0] = bf_lo(gw.x); g4[1] = bf_hi(gw.x); g4[2] = bf_lo(gw.y); g4[3] = bf_hi(gw.y);
    }
    const float s = warp_sum(v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3]);
    const float rs = 1.0f / sqrtf(s / static_cast<float>(D) + eps);
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = v[k] * rs * g4[k];
  }
  if (rope) {
    const bool first_half = e0 < half;
    const int pair0 = first_half ? e0 : e0 - half;
    float2 c[4] = {make_float2(1.f, 0.f), make_float2(1.f, 0.f), make_float2(1.f, 0.f),
                   make_float2(1.f, 0.f)};
    if (active) {
#pragma unroll
      for (int k = 0; k < 4; ++k) c[k] = cs[pair0 + k];
    }
    float w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = __shfl_xor_sync(0xffffffffu, v[k], xo);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      // first half: (a, c) = (v, w) -> a cos - c sin; second half: c cos + a sin
      v[k] = first_half ? v[k] * c[k].x - w[k] * c[k].y : v[k] * c[k].x + w[k] * c[k].y;
  }
}

// Split-attention merge, one batch of up to kCombRegs chunk partials for one
// (head, 4 columns): row c of `ph` (stride `cstride` floats) holds the
// chunk's unnormalised sum over d columns, then its max m and sum l (log2
// units).  Folds the batch into the running (M, den, num).
constexpr int kCombRegs = 17;
template <int D>
__device__ __forceinline__ void comb_batch(const float *ph, size_t cstride, int i, int n, float &M,
                                           float &den, float4 &num) {
  float2 ml[kCombRegs];
  float4 a[kCombRegs];
#pragma unroll
  for (int c = 0; c < kCombRegs; ++c) {
    if (c < n) {
      ml[c] = __ldcg(reinterpret_cast<const float2 *>(ph + c * cstride + D));
      a[c] = __ldcg(reinterpret_cast<const float4 *>(ph + c * cstride + i));
    } else {
      ml[c] = make_float2(-INFINITY, 0.f);
      a[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  float Mb = M;
#pragma unroll
  for (int c = 0; c < kCombRegs; ++c) Mb = fmaxf(Mb, ml[c].x);
  const float sc = exp2f(M - Mb);   // 0 before the first batch (M = -inf)
  den *= sc;
  num.x *= sc; num.y *= sc; num.z *= sc; num.w *= sc;
#pragma unroll
  for (int c = 0; c < kCombRegs; ++c) {
    const float wgt = exp2f(ml[c].x - Mb);   // 0 for the padding entries
    den += wgt * ml[c].y;
    num.x += wgt * a[c].x; num.y += wgt * a[c].y; num.z += wgt * a[c].z; num.w += wgt * a[c].w;
  }
  M = Mb;
}

// The attention scratch in the staging area (see attn_task).
struct AttnSmem {
  float *qs, *sc, *mst, *lst, *cor;
  __nv_bfloat16 *kvcur;
  float *wmerge;   // mma.sync path: the warps' (O, m, l) before their merge
  int *pg_cnt;     // mma.sync path, tensor-core plans: warps done per ring page
};

// The chunk's pages on the CUDA cores (head_dim 32, or a plan without the
// tensor-map copies): three parallel phases per page, see attn_task; writes
// the chunk's unnormalised partial sums to `part` ([G][D + 4]).
template <int D>
__device__ bool attn_pages_cuda(const Params &p, Ctl *ctl, uint8_t *smem, const Slot &S,
                                ComputeState &st, const AttnSmem &A, bool own_cur, int cur,
                                float *part, int ctid) {
  const int warp = ctid >> 5, lane = ctid & 31;
  const int G = p.G;
  constexpr int NB = D / 8;
  constexpr int Q4 = D / 4;
  constexpr int MAXP = (kMaxGroup * Q4 + kComputeThreads - 1) / kComputeThreads;
  float *qs = A.qs, *sc = A.sc, *mst = A.mst, *lst = A.lst, *cor = A.cor;
  const __nv_bfloat16 *kvcur = A.kvcur;
  const int rw = D + 4;
  float acc[MAXP][4];
#pragma unroll
  for (int k = 0; k < MAXP; ++k) acc[k][0] = acc[k][1] = acc[k][2] = acc[k][3] = 0.f;

  for (int tok0 = S.t0; tok0 < S.t1; tok0 += p.tpp) {
    const int ntok = min(p.tpp, S.t1 - tok0);
    bool okl = true;
    if (ctid == 0) okl = wait_mbar(p, ctl, &ctl->full[st.pi], st.pg_par, 0xfff40000u, 2);
    if (!st.gs.share(ctl, ctid, okl)) return false;
    mbar_try_wait(&ctl->full[st.pi], st.pg_par);
    uint8_t *kpg = smem + p.off_pages + static_cast<size_t>(st.pi) * p.page_bytes;
    uint8_t *vpg = kpg + static_cast<size_t>(p.tpp) * D * 2;
    // The page was copied from the cache before this step's K/V of the
    // current token were formed: put them into its slot.
    const bool has_cur = own_cur && cur >= tok0 && cur < tok0 + ntok;
    if (has_cur) {
      const int j = cur - tok0;
      if (ctid < 2 * NB) {
        const bool isv = ctid >= NB;
        const int e = (isv ? ctid - NB : ctid) * 8;
        *reinterpret_cast<uint4 *>((isv ? vpg : kpg) + (j * D + e) * 2) =
            *reinterpret_cast<const uint4 *>(kvcur + (isv ? D : 0) + e);
      }
      compute_bar();
    }
    // phase 1: scores
    for (int pp = ctid; pp < ntok * G; pp += kComputeThreads) {
      const int tk = pp % ntok, h = pp / ntok;
      const uint8_t *krow = kpg + tk * D * 2;
      const float *qh = qs + h * D;
      float s = 0.f;
#pragma unroll 4
      for (int c = 0; c < NB; ++c) {
        const int cc = (c + tk) & (NB - 1);
        const uint4 kw = *reinterpret_cast<const uint4 *>(krow + cc * 16);
        const float4 q0 = *reinterpret_cast<const float4 *>(qh + cc * 8);
        const float4 q1 = *reinterpret_cast<const float4 *>(qh + cc * 8 + 4);
        s += q0.x * bf_lo(kw.x) + q0.y * bf_hi(kw.x) + q0.z * bf_lo(kw.y) + q0.w * bf_hi(kw.y);
        s += q1.x * bf_lo(kw.z) + q1.y * bf_hi(kw.z) + q1.z * bf_lo(kw.w) + q1.w * bf_hi(kw.w);
      }
      sc[h * p.tpp + tk] = s;
    }
    compute_bar();
    // phase 2: softmax statistics, one warp per head
    for (int h = warp; h < G; h += kComputeWarps) {
      float *row = sc + h * p.tpp;
      float mx = -INFINITY;
      for (int tk = lane; tk < ntok; tk += 32) mx = fmaxf(mx, row[tk]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mold = mst[h];
      const float mnew = fmaxf(mold, mx);
      float sum = 0.f;
      for (int tk = lane; tk < ntok; tk += 32) {
        const float pr = exp2f(row[tk] - mnew);
        row[tk] = pr;
        sum += pr;
      }
      sum = warp_sum(sum);
      __syncwarp();
      if (lane == 0) {
        const float c = exp2f(mold - mnew);   // 0 on the first page (mold = -inf)
        cor[h] = c;
        lst[h] = lst[h] * c + sum;
        mst[h] = mnew;
      }
    }
    compute_bar();
    // phase 3: acc = acc * rescale + sum_t p_t v_t
#pragma unroll
    for (int k = 0; k < MAXP; ++k) {
      const int pq = ctid + k * kComputeThreads;
      if (pq < G * Q4) {
        const int h = pq / Q4, i4 = pq % Q4;
        const float c = cor[h];
        float a0 = acc[k][0] * c, a1 = acc[k][1] * c, a2 = acc[k][2] * c, a3 = acc[k][3] * c;
        const float *prow = sc + h * p.tpp;
        const uint8_t *vcol = vpg + i4 * 8;
#pragma unroll 4
        for (int tk = 0; tk < ntok; ++tk) {
          const float pr = prow[tk];
          const uint2 vw = *reinterpret_cast<const uint2 *>(vcol + tk * D * 2);
          a0 += pr * bf_lo(vw.x);
          a1 += pr * bf_hi(vw.x);
          a2 += pr * bf_lo(vw.y);
          a3 += pr * bf_hi(vw.y);
        }
        acc[k][0] = a0; acc[k][1] = a1; acc[k][2] = a2; acc[k][3] = a3;
      }
    }
    if (has_cur) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (!(p.tc || p.tm) && lane == 0) mbar_arrive(&ctl->empty[st.pi]);
    compute_bar();   // sc is rewritten by the next page
    // (tensor-core plans release a page once, after every warp is done with it)
    if ((p.tc || p.tm) && ctid == 0) mbar_arrive(&ctl->empty[st.pi]);
    if (++st.pi == p.n_pages) {
      st.pi = 0;
      st.pg_par ^= 1u;
    }
  }

  // the chunk's partial goes straight to global memory: row h = (acc, m, l, pad)
#pragma unroll
  for (int k = 0; k < MAXP; ++k) {
    const int pq = ctid + k * kComputeThreads;
    if (pq < G * Q4) {
      const int h = pq / Q4, i4 = pq % Q4;
      __stcg(reinterpret_cast<float4 *>(part + h * rw + i4 * 4),
             make_float4(acc[k][0], acc[k][1], acc[k][2], acc[k][3]));
    }
  }
  return true;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                              uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// 16-byte chunk `c` (0..7) of the 128-byte row at `row` in a 128-byte-swizzled
// TMA box (box base 1024-byte aligned): the chunk sits at c XOR row bits 7..9.
__device__ __forceinline__ uint32_t sw128(uint32_t row, int c) {
  return row + ((static_cast<uint32_t>(c) ^ ((row >> 7) & 7u)) << 4);
}

// fp32 pair -> (hi, lo) bf16x2 pairs (first value in the low half),
// hi + lo == x to ~2^-16: two paired conversions.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - __low2float(h), x1 - __high2float(h));
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

// The chunk's pages on the tensor cores (mma.sync m16n8k16, bf16 -> fp32),
// K and V pages copied by TMA in the 128-byte-swizzled layout (per KV page,
// 64-dim boxes of P rows x 128 bytes), so every ldmatrix reads conflict-free.
// Flash decoding inside the CTA: the chunk's tokens are cut into 16-token
// slices dealt round-robin to the compute warps, and each warp keeps its own
// online softmax (running max m, sum l) and unnormalised O in registers, so
// warps never wait for one another inside the chunk.  Per slice:
//   S = Q K^T: A = the G query heads as rows, bf16 high halves in rows
//   0..7 and low halves in rows 8..15 (registers, built once per chunk); B =
//   8 tokens x 16 dims by ldmatrix; the score of head g = row g + row g + 8;
//   the slice's max (a quad shuffle), rescale, p = 2^(s - m);
//   O += P V: A = p of the G heads as high/low rows, straight from the score
//   registers; B = 16 tokens x 8 dims by ldmatrix.trans.
// Tokens past the page's end: score -inf and their V rows zeroed (the cache
// may hold anything there).  At the end the warps' (m, l, O) merge through
// shared memory by log-sum-exp into the chunk's partial.  A page goes back
// to the loader when its last warp is done with it.
template <int D>
__device__ bool attn_pages_mma(const Params &p, Ctl *ctl, uint8_t *smem, const Slot &S,
                               ComputeState &st, const AttnSmem &A, bool own_cur, int cur,
                               float *part, int ctid) {
  const int warp = ctid >> 5, lane = ctid & 31;
  const int G = p.G, P = p.page_size, tpp = p.tpp;
  const int g = lane >> 2, q = lane & 3;
  constexpr int NB = D / 8;                  // 16-byte chunks per row
  constexpr int KS = D / 16;                 // k-steps of the scores
  constexpr int DT = D / 8;                  // 8-dim tiles of O
  const bool hrow = g < G;                   // rows g / g + 8 carry head g
  const uint32_t kvbytes = static_cast<uint32_t>(P * D * 2);   // one KV page of K (or V)

  // the query fragments (rows g: high halves of head g, g + 8: low halves)
  uint32_t qa[KS][4];
#pragma unroll
  for (int s = 0; s < KS; ++s) {
    float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
    if (hrow) {
      const float *qh = A.qs + g * D + 16 * s + 2 * q;
      x0 = qh[0]; x1 = qh[1]; x2 = qh[8]; x3 = qh[9];
    }
    split_pair(x0, x1, qa[s][0], qa[s][1]);
    split_pair(x2, x3, qa[s][2], qa[s][3]);
  }
  float m_run = -INFINITY, l_run = 0.f;   // head g; l_run: this lane's tokens only
  float acc[DT][4];
#pragma unroll
  for (int i = 0; i < DT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  bool bad = false;
  int slice0 = 0;   // chunk-relative index of the page's first slice
  for (int tok0 = S.t0; tok0 < S.t1; tok0 += tpp) {
    const int ntok = min(tpp, S.t1 - tok0);
    const int nsl = (ntok + 15) >> 4;
    if (!bad && !warp_wait_page(p, ctl, &ctl->full[st.pi], st.pg_par, 0xfff40000u)) {
      bad = true;
      if (lane == 0) {
        ctl->cbad = 1;
        ctl->cta_abort = 1;
      }
    }
    if (!bad) {
      const uint32_t ks = smem_u32(smem + p.off_pages + static_cast<size_t>(st.pi) * p.page_bytes);
      const uint32_t vs = ks + static_cast<uint32_t>(tpp * D * 2);
      bool wrote = false;
      for (int sl = (warp + kComputeWarps - slice0 % kComputeWarps) % kComputeWarps; sl < nsl;
           sl += kComputeWarps) {
        const int tb = 16 * sl;                       // first token of the slice in the page
        const int jp = tb / P;                        // its KV page
        const uint32_t krow = ks + jp * kvbytes + static_cast<uint32_t>(tb - jp * P) * 128u;
        const uint32_t vrow = vs + jp * kvbytes + static_cast<uint32_t>(tb - jp * P) * 128u;
        const uint32_t atom = static_cast<uint32_t>(P * 128);   // one 64-dim box
        // the current token's K/V into its row (the page was copied before
        // they were formed), and V rows past the page's end zeroed
        const int rc = cur - tok0 - tb;
        if (own_cur && rc >= 0 && rc < 16 && tb + rc < ntok) {
          if (lane < 2 * NB) {
            const bool isv = lane >= NB;
            const int c = isv ? lane - NB : lane;
            sts128(sw128((isv ? vrow : krow) + (c >> 3) * atom + rc * 128u, c & 7),
                   *reinterpret_cast<const uint4 *>(A.kvcur + (isv ? D : 0) + 8 * c));
          }
          wrote = true;
        }
        const int nvalid = min(16, ntok - tb);
        if (nvalid < 16) {
          for (int u = lane; u < (16 - nvalid) * NB; u += 32) {
            const int r = nvalid + u / NB, c = u % NB;
            sts128(sw128(vrow + (c >> 3) * atom + r * 128u, c & 7), make_uint4(0, 0, 0, 0));
          }
          wrote = true;
        }
        __syncwarp();
        // scores: two 8-token tiles
        float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s2 = 0; s2 < KS / 2; ++s2) {
          const int dim = 32 * s2 + 8 * (lane >> 3);
          const uint32_t rb = krow + (dim >> 6) * atom;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sw128(rb + (lane & 7) * 128u, (dim & 63) >> 3), b0, b1, b2, b3);
          mma_bf16(c0, qa[2 * s2][0], qa[2 * s2][1], qa[2 * s2][2], qa[2 * s2][3], b0, b1);
          mma_bf16(c0, qa[2 * s2 + 1][0], qa[2 * s2 + 1][1], qa[2 * s2 + 1][2], qa[2 * s2 + 1][3],
                   b2, b3);
          ldsm_x4(sw128(rb + (8 + (lane & 7)) * 128u, (dim & 63) >> 3), b0, b1, b2, b3);
          mma_bf16(c1, qa[2 * s2][0], qa[2 * s2][1], qa[2 * s2][2], qa[2 * s2][3], b0, b1);
          mma_bf16(c1, qa[2 * s2 + 1][0], qa[2 * s2 + 1][1], qa[2 * s2 + 1][2], qa[2 * s2 + 1][3],
                   b2, b3);
        }
        // this lane's tokens: 2q, 2q + 1, 8 + 2q, 9 + 2q of the slice
        float s0 = c0[0] + c0[2], s1 = c0[1] + c0[3], s2v = c1[0] + c1[2], s3 = c1[1] + c1[3];
        if (2 * q >= nvalid) s0 = -INFINITY;
        if (2 * q + 1 >= nvalid) s1 = -INFINITY;
        if (8 + 2 * q >= nvalid) s2v = -INFINITY;
        if (9 + 2 * q >= nvalid) s3 = -INFINITY;
        float mx = fmaxf(fmaxf(s0, s1), fmaxf(s2v, s3));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        // (token 0 of a slice is always valid: mx is finite for head rows)
        float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
        if (hrow) {
          const float mnew = fmaxf(m_run, mx);
          const float sc = exp2f(m_run - mnew);   // 0 on the first slice (m_run = -inf)
          p0 = exp2f(s0 - mnew);
          p1 = exp2f(s1 - mnew);
          p2 = exp2f(s2v - mnew);
          p3 = exp2f(s3 - mnew);
          l_run = l_run * sc + ((p0 + p1) + (p2 + p3));
          m_run = mnew;
#pragma unroll
          for (int i = 0; i < DT; ++i) {
            acc[i][0] *= sc; acc[i][1] *= sc; acc[i][2] *= sc; acc[i][3] *= sc;
          }
        }
        uint32_t a0, a1, a2, a3;
        split_pair(p0, p1, a0, a1);
        split_pair(p2, p3, a2, a3);
        // O += P V, two 8-dim tiles per ldmatrix
#pragma unroll
        for (int i = 0; i < DT; i += 2) {
          const int dim = 8 * i + 8 * (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_trans(sw128(vrow + (dim >> 6) * atom + (lane & 15) * 128u, (dim & 63) >> 3), b0,
                        b1, b2, b3);
          mma_bf16(acc[i], a0, a1, a2, a3, b0, b1);
          mma_bf16(acc[i + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      if (wrote) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    // the page goes back to the loader once every warp is done with it
    __syncwarp();
    if (lane == 0) {
      if (p.tc || p.tm) {
        __threadfence_block();
        if (atomicAdd(&A.pg_cnt[st.pi], 1) == kComputeWarps - 1) {
          A.pg_cnt[st.pi] = 0;
          mbar_arrive(&ctl->empty[st.pi]);
        }
      } else {
        mbar_arrive(&ctl->empty[st.pi]);
      }
    }
    slice0 += nsl;
    if (++st.pi == p.n_pages) {
      st.pi = 0;
      st.pg_par ^= 1u;
    }
  }

  // merge the warps: (m, l) per head and O per (head, dim) through shared memory
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  float *wO = A.wmerge;                                   // [warp][G][D]
  float *wM = wO + kComputeWarps * G * D;                 // [warp][G]
  float *wL = wM + kComputeWarps * G;                     // [warp][G]
  if (hrow) {
    float *o = wO + (warp * G + g) * D;
#pragma unroll
    for (int i = 0; i < DT; ++i)
      *reinterpret_cast<float2 *>(o + 8 * i + 2 * q) =
          make_float2(acc[i][0] + acc[i][2], acc[i][1] + acc[i][3]);
    if (q == 0) {
      wM[warp * G + g] = m_run;
      wL[warp * G + g] = l_run;
    }
  }
  compute_bar();
  if (ctl->cbad != 0) return false;
  constexpr int Q4 = D / 4;
  for (int e = ctid; e < G * Q4; e += kComputeThreads) {
    const int h = e / Q4, i4 = (e % Q4) * 4;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kComputeWarps; ++w) M = fmaxf(M, wM[w * G + h]);
    float den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kComputeWarps; ++w) {
      const float mw = wM[w * G + h];
      const float wt = mw == -INFINITY ? 0.f : exp2f(mw - M);   // a warp without tokens
      den += wt * wL[w * G + h];
      const float4 o = *reinterpret_cast<const float4 *>(wO + (w * G + h) * D + i4);
      num.x += wt * o.x; num.y += wt * o.y; num.z += wt * o.z; num.w += wt * o.w;
    }
    const int rw = D + 4;
    __stcg(reinterpret_cast<float4 *>(part + h * rw + i4), num);
    if (i4 == 0) {
      A.mst[h] = M;
      A.lst[h] = den;
    }
  }
  compute_bar();
  return true;
}

// Attention for one chunk of one (sequence, KV head): scores for the G query
// heads over the chunk's tokens, softmax statistics, and the unnormalised
// P.V, all in three parallel phases per shared-memory page:
//   1. thread <- (token, head): full dot product q.k over d, reading the
//      8-element column blocks in a rotated order (block (c + t) mod d/8) so
//      the 32 lanes of a warp hit distinct banks;
//   2. warp <- head: running max m, rescale factor, p = 2^(s - m), running sum;
//   3. thread <- (head, 4 columns of d): acc = acc * rescale + sum_t p v.
// Scores are in log2 units (q is pre-scaled by log2(e)/sqrt(d)).
template <int D, bool AMMA>
__device__ bool attn_task(const Params &p, Ctl *ctl, uint8_t *smem, const Slot &S,
                          ComputeState &st, float *out, int ctid) {
  const Task &t = S.t;
  const int warp = ctid >> 5, lane = ctid & 31;
  const int G = p.G, l = t.layer;
  const int b = S.b, g = S.g;
  float *qs = reinterpret_cast<float *>(smem + p.off_x);   // [G][D]
  float *sc = qs + G * D;                                   // [G][tpp] scores, then p
  float *mst = sc + G * p.tpp;                              // [G] running max
  float *lst = mst + kMaxGroup;                             // [G] running sum
  float *cor = lst + kMaxGroup;                             // [G] rescale of this page
  __nv_bfloat16 *kvcur = reinterpret_cast<__nv_bfloat16 *>(cor + kMaxGroup);  // [2][D] K, V at pos
  int *pg_cnt = reinterpret_cast<int *>(kvcur + 2 * D);     // [kMaxPages]
  float *wmerge = reinterpret_cast<float *>(pg_cnt + kMaxPages);   // [warps][G][D + 2]
  st.xkey = 0xffffffffu;                                    // staging area reused

  {
    const uint32_t ev = static_cast<uint32_t>(ev_attn_input(p, l, g));
    bool okl = true;
    if (ctid == 0) okl = wait_event(p, ctl, ev, static_cast<uint32_t>(attn_input_count(p)), S.idx);
    if (!st.gs.share(ctl, ctid, okl)) return false;
    if (ctid == 0) trace_mark(p, S.idx, 4);
  }
  // From this step's raw projections, one warp per head: the G query heads
  // (QK-norm, RoPE, pre-scaled by log2(e)/sqrt(d) for the exp2 softmax) and,
  // in the chunk that holds the current position, K (QK-norm, RoPE) and V of
  // the current token, rounded to bf16 and appended to the cache.
  const int P = p.page_size;
  const int cur = row_pos(p, b);
  // (in a plan whose K/V tasks append every row's K/V first, the cache
  // already holds the current token's)
  const bool own_cur = !p.kv_tasks && cur >= S.t0 && cur < S.t1;
  {
    const float qscale = rsqrtf(static_cast<float>(D)) * 1.4426950408889634f;
    // a position outside 0..max_pos-1 is reported by the embedding task; the
    // table row stays in range regardless
    const int cpos = cur < 0 ? 0 : (cur >= p.max_pos ? p.max_pos - 1 : cur);
    const float2 *cs = p.rope_cs + static_cast<size_t>(cpos) * (D / 2);
    const float *raw = p.qkv + static_cast<size_t>(b) * p.NQKV;
    const int nh = G + (own_cur ? 2 : 0);
    for (int h = warp; h < nh; h += kComputeWarps) {
      const int mat = h < G ? 0 : h - G + 1;   // 0 q, 1 k, 2 v
      const int col = mat == 0 ? (g * G + h) * D
                               : (mat == 1 ? (p.Hq + g) * D : (p.Hq + p.Hkv + g) * D);
      float v[4];
      head_norm_rope<D>(raw + col, mat == 0 ? t.w0 : t.w1, p.qk_norm != 0 && mat != 2,
                        mat != 2, cs, p.eps, lane, v);
      if (lane < D / 4) {
        const int e0 = lane * 4;
        if (mat == 0) {
          *reinterpret_cast<float4 *>(qs + h * D + e0) =
              make_float4(v[0] * qscale, v[1] * qscale, v[2] * qscale, v[3] * qscale);
        } else {
          const uint2 pk = make_uint2(pack2(__float2bfloat16_rn(v[0]), __float2bfloat16_rn(v[1])),
                                      pack2(__float2bfloat16_rn(v[2]), __float2bfloat16_rn(v[3])));
          *reinterpret_cast<uint2 *>(kvcur + (mat - 1) * D + e0) = pk;
          const int ph = kv_phys_page(p, b, cur / P);
          if (ph >= 0) {
            __nv_bfloat16 *dst = (mat == 1 ? p.k_pages[l] : p.v_pages[l]) +
                                 ((static_cast<size_t>(ph) * p.Hkv + g) * P + cur % P) * D + e0;
            *reinterpret_cast<uint2 *>(dst) = pk;
          }
        }
      }
    }
  }
  if (ctid < G) {
    mst[ctid] = -INFINITY;
    lst[ctid] = 0.f;
  }
  if (AMMA && ctid < kMaxPages) pg_cnt[ctid] = 0;
  compute_bar();
  if (ctid == 0) trace_mark(p, S.idx, 5);

  const int rw = D + 4;
  float *part = p.attn_part + static_cast<size_t>(t.aux) * G * rw;
  AttnSmem A{qs, sc, mst, lst, cor, kvcur, wmerge, pg_cnt};
  bool pages_ok;
  if constexpr (AMMA && D >= 64)
    pages_ok = attn_pages_mma<D>(p, ctl, smem, S, st, A, own_cur, cur, part, ctid);
  else
    pages_ok = attn_pages_cuda<D>(p, ctl, smem, S, st, A, own_cur, cur, part, ctid);
  if (!pages_ok) return false;
  if (ctid < G) {
    __stcg(part + ctid * rw + D, mst[ctid]);
    __stcg(part + ctid * rw + D + 1, lst[ctid]);
  }
  compute_bar();
  const int d = D;

  // The chunk that completes (b, g) merges all of its chunks by log-sum-exp
  // and writes o for the G query heads.  The bar above orders every thread's
  // partial before thread 0's release; thread 0's acquire orders the other
  // chunks' partials before the reads below.
  uint32_t *ctr = p.comb_ctr + b * p.Hkv + g;
  bool last_l = false;
  if (ctid == 0) last_l = atom_add_acq_rel(ctr, 1u) + 1u == static_cast<uint32_t>(S.n_chunks);
  if (!st.gs.share(ctl, ctid, last_l)) return true;
  // Each (head, 4 columns) thread merges the chunks in batches of kCombRegs:
  // a batch's (m, l) pairs and 4-column partial sums are loaded into
  // registers with all loads in flight together, so a batch costs one L2
  // round trip; the running maximum rescales the earlier batches.  17 is the
  // largest batch that measured no slower elsewhere in the kernel (register
  // pressure); decode at one sequence per 148 SMs splits a head's context
  // into at most about 20 chunks.  The first batch is straight-line code.
  const int nch = S.n_chunks;
  const size_t cstride = static_cast<size_t>(G) * rw;
  const float *p0 = p.attn_part + static_cast<size_t>(S.first_slot) * cstride;
  const int q4 = d / 4;
  for (int e = ctid; e < G * q4; e += kComputeThreads) {
    const int h = e / q4, i = (e % q4) * 4;
    float M = -INFINITY, den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    comb_batch<D>(p0 + h * rw, cstride, i, nch, M, den, num);
    for (int c0 = kCombRegs; c0 < nch; c0 += kCombRegs)
      comb_batch<D>(p0 + c0 * cstride + h * rw, cstride, i, nch - c0, M, den, num);
    const float r = 1.0f / den;
    const float4 ov = make_float4(num.x * r, num.y * r, num.z * r, num.w * r);
    const int col = (g * G + h) * d + i;
    __stcg(reinterpret_cast<float4 *>(p.o + static_cast<size_t>(b) * p.Hq * d + col), ov);
    if (p.tc) {
      // the O projection's input, staged for the tensor cores
      const int K = p.Hq * d;
      put_staged(p.xs[XS_O], p.tc_bpad, K, b, col, ov.x);
      put_staged(p.xs[XS_O], p.tc_bpad, K, b, col + 1, ov.y);
      put_staged(p.xs[XS_O], p.tc_bpad, K, b, col + 2, ov.z);
      put_staged(p.xs[XS_O], p.tc_bpad, K, b, col + 3, ov.w);
    }
  }
  compute_bar();
  if (ctid == 0) *ctr = 0u;   // rearm for the next layer / step
  (void)out;
  return true;
}

// ============================================================================
// compute warps: K/V append of one KV group for every row (prefill plans)
// ============================================================================

// From this step's raw projections: K (QK-norm, RoPE at the row's position)
// and V of KV group t.aux for every row, rounded to bf16 and written to the
// cache, one warp per (row, K or V).  Attention chunks of the group wait for
// this task, so a row may attend to positions that other rows of the same
// step (earlier tokens of the same prompt chunk) write.
template <int D>
__device__ bool kv_append_task(const Params &p, Ctl *ctl, const Slot &S, ComputeState &st,
                               int ctid) {
  const Task &t = S.t;
  const int warp = ctid >> 5, lane = ctid & 31;
  const int g = static_cast<int>(t.aux), l = t.layer, P = p.page_size;
  {
    bool okl = true;
    if (ctid == 0) okl = wait_event(p, ctl, t.dep_event, t.dep_count, S.idx);
    if (!st.gs.share(ctl, ctid, okl)) return false;
    if (ctid == 0) trace_mark(p, S.idx, 4);
  }
  for (int w = warp; w < 2 * p.batch; w += kComputeWarps) {
    const int b = w >> 1, mat = 1 + (w & 1);   // 1 k, 2 v
    const int cur = row_pos(p, b);
    const int cpos = cur < 0 ? 0 : (cur >= p.max_pos ? p.max_pos - 1 : cur);
    const float2 *cs = p.rope_cs + static_cast<size_t>(cpos) * (D / 2);
    const float *raw = p.qkv + static_cast<size_t>(b) * p.NQKV +
                       (mat == 1 ? (p.Hq + g) * D : (p.Hq + p.Hkv + g) * D);
    float v[4];
    head_norm_rope<D>(raw, t.w1, p.qk_norm != 0 && mat == 1, mat == 1, cs, p.eps, lane, v);
    const int ph = kv_phys_page(p, b, cur / P);
    if (lane < D / 4 && ph >= 0) {
      const uint2 pk = make_uint2(pack2(__float2bfloat16_rn(v[0]), __float2bfloat16_rn(v[1])),
                                  pack2(__float2bfloat16_rn(v[2]), __float2bfloat16_rn(v[3])));
      __nv_bfloat16 *dst = (mat == 1 ? p.k_pages[l] : p.v_pages[l]) +
                           ((static_cast<size_t>(ph) * p.Hkv + g) * P + cur % P) * D + lane * 4;
      *reinterpret_cast<uint2 *>(dst) = pk;
    }
  }
  return true;
}

// ============================================================================
// compute warps: embedding gather
// ============================================================================

__device__ void embed_task(const Params &p, const Slot &S, int ctid) {
  const int B = p.batch, H = p.H;
  for (int b = 0; b < B; ++b) {
    const int id = p.ids[b];
    const int pos = row_pos(p, b);
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
      if (p.tc) {
        // the first QKV input, times its gain, staged for the tensor cores
        const uint4 gw = __ldg(reinterpret_cast<const uint4 *>(S.t.w1 + i));
        const float v[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
        const float gg[8] = {bf_lo(gw.x), bf_hi(gw.x), bf_lo(gw.y), bf_hi(gw.y),
                             bf_lo(gw.z), bf_hi(gw.z), bf_lo(gw.w), bf_hi(gw.w)};
#pragma unroll
        for (int k = 0; k < 8; ++k) put_staged(p.xs[XS_ATTN], p.tc_bpad, H, b, i + k, v[k] * gg[k]);
      }
    }
  }
  if (p.tc) {
    // sums of h^2 per 128 rows for the first QKV tasks' RMSNorm (tensor-core path)
    const int nt = (H + kTcRows - 1) / kTcRows;
    for (int u = ctid; u < B * nt; u += kComputeThreads) {
      const int b = u / nt, i = u - b * nt;
      const int id = p.ids[b];
      if (id < 0 || id >= p.V) continue;   // reported above
      const __nv_bfloat16 *e = p.embed + static_cast<size_t>(id) * H + i * kTcRows;
      const int n = min(kTcRows, H - i * kTcRows);
      float sq = 0.f;
      for (int k = 0; k < n; k += 8) {
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(e + k));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) sq += bf_lo(ww[j]) * bf_lo(ww[j]) + bf_hi(ww[j]) * bf_hi(ww[j]);
      }
      __stcg(p.ssq_attn + static_cast<size_t>(i) * p.max_batch + b, sq);
    }
  }
  __threadfence();
}

// ============================================================================
// compute warps: main loop
// ============================================================================

template <int V>
__device__ void compute_main(const Params &p, Ctl *ctl, uint8_t *smem) {
  constexpr bool TC = (V & kVarTc) != 0, W4 = (V & kVarW4) != 0, AMMA = (V & kVarAttnMma) != 0;
  constexpr bool TM = (V & kVarTm) != 0;
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
      case T_KVAPP:
        switch (p.d >> 5) {
          case 1: tok = kv_append_task<32>(p, ctl, S, st, ctid); break;
          case 2: tok = kv_append_task<64>(p, ctl, S, st, ctid); break;
          default: tok = kv_append_task<128>(p, ctl, S, st, ctid); break;
        }
        break;
      case T_ATTN:
        if (S.b >= 0) {
          switch (p.d >> 5) {
            case 1: tok = attn_task<32, AMMA>(p, ctl, smem, S, st, out, ctid); break;
            case 2: tok = attn_task<64, AMMA>(p, ctl, smem, S, st, out, ctid); break;
            default: tok = attn_task<128, AMMA>(p, ctl, smem, S, st, out, ctid); break;
          }
        }
        break;
      default:
        if constexpr (TC)
          tok = p.tc_n > 16 ? gemv_task_tc<2>(p, ctl, smem, S, st, out, ctid)
                            : gemv_task_tc<1>(p, ctl, smem, S, st, out, ctid);
        else
          tok = p.batch > 8   ? gemv_task<4, W4, TM>(p, ctl, smem, S, st, out, ctid)
                : p.batch > 4 ? gemv_task<2, W4, TM>(p, ctl, smem, S, st, out, ctid)
                              : gemv_task<1, W4, TM>(p, ctl, smem, S, st, out, ctid);
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
    if (++os == p.n_out) {
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


__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<unsigned long long>(u) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(idx));
}

// Ordering: every lane's global writes are followed by __syncwarp(), after
// which lane 0's release (red.release / atom.acq_rel) publishes them; a last
// arriver's acquire (atom.acq_rel) is followed by __syncwarp() before any lane
// reads what the other arrivers published.  No full fences are needed.
__device__ bool storer_epilogue(const Params &p, Ctl *ctl, const Slot &S, const float *out,
                                int lane) {
  const Task &t = S.t;
  const int B = p.batch;
  const int OS = p.out_stride;
  switch (t.type) {
    case T_EMBED: {
      __syncwarp();
      if (lane == 0) signal(p, t.out_event);
      break;
    }
    case T_QKV:
    case T_OPROJ:
    case T_DOWN:
    case T_GATEUP: {
      const int nr = static_cast<int>(t.nrows);
      // the rows this task's output covers within its operator's row space
      // (QKV: q rows, then k rows, then v rows; gate/up: gate rows then up
      // rows, 2F in all)
      const int qbase = t.aux == 0 ? 0 : (t.aux == 1 ? p.Hq * p.d : (p.Hq + p.Hkv) * p.d);
      const int grow0 = static_cast<int>(t.row0) + (t.type == T_QKV ? qbase : 0);
      const int up_off = (t.n_m >> 1) * p.tile_rows;   // gate/up: the up rows in `out`
      float *kp = p.kpart;
      int rstride = p.H;
      uint32_t *ctr = p.tile_ctr;
      if (t.type == T_QKV) {
        rstride = p.NQKV;
      } else if (t.type == T_OPROJ) {
        kp = p.kpart_o;
        ctr = p.tile_ctr_o;
      } else if (t.type == T_GATEUP) {
        kp = p.kpart2;
        rstride = 2 * p.F;
        ctr = p.tile_ctr2;
      }
      const size_t pstride = static_cast<size_t>(p.max_batch) * rstride;
      const bool split = t.nsplit > 1;
      if (split) {
        // split-K part: publish the partial; the part that completes the row
        // tile sums all parts in a fixed order and runs the epilogue
        for (int b = 0; b < B; ++b)
          for (int r = lane; r < nr; r += 32) {
            float *dst = kp + t.ksplit * pstride + static_cast<size_t>(b) * rstride + grow0 + r;
            __stcg(dst, out[b * OS + r]);
            if (t.type == T_GATEUP) __stcg(dst + p.F, out[b * OS + up_off + r]);
          }
        __syncwarp();
        ctr += grow0 / 16;
        uint32_t old = 0;
        if (lane == 0) old = atom_add_acq_rel(ctr, 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old + 1u != static_cast<uint32_t>(t.nsplit)) break;
        __syncwarp();
      }
      // the task's (summed) output of sequence b, row r (half 1: gate/up's up rows)
      auto value = [&](int b, int r, int half) -> float {
        if (!split) return out[b * OS + half * up_off + r];
        const float *src = kp + static_cast<size_t>(b) * rstride + grow0 + half * p.F + r;
        float sum = 0.f;
        for (int k = 0; k < t.nsplit; ++k) sum += __ldcg(src + k * pstride);
        return sum;
      };
      if (t.type == T_QKV) {
        // raw projection rows; QK-norm, RoPE and the KV append happen in the
        // attention tasks of the head's KV group
        for (int b = 0; b < B; ++b)
          for (int r = lane; r < nr; r += 32)
            __stcg(p.qkv + static_cast<size_t>(b) * p.NQKV + grow0 + r, value(b, r, 0));
      } else if (t.type == T_GATEUP) {
        for (int b = 0; b < B; ++b)
          for (int r = lane; r < nr; r += 32) {
            const float gt = value(b, r, 0);
            const float up = value(b, r, 1);
            __stcg(p.u + static_cast<size_t>(b) * p.F + t.row0 + r, gt / (1.0f + __expf(-gt)) * up);
          }
      } else {
        // residual add; on the tensor-core path also the sums of h^2 per 16
        // rows that the next normed operator's RMSNorm reads
        float *ssq = t.type == T_OPROJ ? p.ssq_mlp : p.ssq_attn;
        for (int b = 0; b < B; ++b)
          for (int r0 = 0; r0 < nr; r0 += 32) {
            const int r = r0 + lane;
            float v = 0.f;
            if (r < nr) {
              float *hp = p.h + static_cast<size_t>(b) * p.H + t.row0 + r;
              v = __ldcg(hp) + value(b, r, 0);
              __stcg(hp, v);
              if (t.type == T_DOWN && p.hidden_dump != nullptr)
                p.hidden_dump[(static_cast<size_t>(t.layer) * B + b) * p.H + t.row0 + r] = v;
            }
            if (p.tc) {
              float sq = v * v;
#pragma unroll
              for (int o = 8; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
              if ((lane & 15) == 0 && r < nr)
                __stcg(ssq + static_cast<size_t>((t.row0 + r) / 16) * p.max_batch + b, sq);
            }
          }
      }
      __syncwarp();
      if (lane == 0) {
        if (split) *ctr = 0u;   // rearm for the next layer / step
        if (t.type == T_QKV) {
          const int head = static_cast<int>(t.aux2);
          const int g = t.aux == 0 ? head / p.G : (t.aux == 1 ? head - p.Hq : head - p.Hq - p.Hkv);
          signal(p, static_cast<uint32_t>(ev_attn_ready(p, t.layer, g)));
        } else {
          signal(p, t.out_event);
        }
      }
      break;
    }
    case T_ATTN:
    case T_KVAPP: {
      // the compute warps wrote the chunk partial (and, for the chunk that
      // completed its (sequence, KV head), the merged o), or the K/V rows,
      // before handing over
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
      __syncwarp();
      uint32_t old = 0;
      if (lane == 0) old = atom_add_acq_rel(p.sync + S_LMCTR, 1u);
      old = __shfl_sync(0xffffffffu, old, 0);
      if (old + 1u == static_cast<uint32_t>(p.n_lm_tasks)) {
        __syncwarp();
        if (lane < B) {
          const unsigned long long k = ld_relaxed_u64(p.argmax + lane);
          p.out_ids[lane] = static_cast<int32_t>(~static_cast<uint32_t>(k & 0xffffffffull));
          if (p.out_pos != nullptr) p.out_pos[lane] = row_pos(p, lane) + 1;
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
    // (tensor-core plans: the compute warps ran the projections' epilogues
    // and released their events; only the LM head's argmax is left here)
    if (!(p.tc && is_gemv(S.t.type) && S.t.type != T_LMHEAD)) storer_epilogue(p, ctl, S, out, lane);
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
    if (++os == p.n_out) {
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

// One instantiation per variant V (kVarTc: tcgen05 tiles, else mma.sync
// pages; kVarW4: the 4-bit weight consumer; kVarAttnMma: attention on
// mma.sync tiles over swizzled K/V pages), so no plan carries code (and
// register pressure) of a path it does not run.
template <int V>
__global__ void __launch_bounds__(kThreads, 1) mk_step_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Ctl *ctl = reinterpret_cast<Ctl *>(smem);
  if (threadIdx.x == 0) {
    for (int i = 0; i < p.n_pages; ++i) {
      mbar_init(&ctl->full[i], 1);
      // a page is released by each compute warp, or (tensor-core path) once:
      // by the MMAs' commit, or by one thread after an attention page
      mbar_init(&ctl->empty[i], (p.tc || p.tm) ? 1 : kComputeWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->x_full[i], 1);
      mbar_init(&ctl->x_free[i], 1);
    }
    mbar_init(&ctl->acc_bar, 1);
    for (int i = 0; i < kTmSlots; ++i) {
      mbar_init(tm_full_bar(smem, p, i), 1);               // the mover's commit
      mbar_init(tm_empty_bar(smem, p, i), kComputeWarps);  // every compute warp, after reading
    }
    for (int i = 0; i < kTaskSlots; ++i) {
      mbar_init(&ctl->slot_full[i], 1);
      mbar_init(&ctl->slot_empty[i], 1);
    }
    for (int i = 0; i < kOutSlots; ++i) {
      mbar_init(&ctl->out_full[i], 1);
      mbar_init(&ctl->out_empty[i], 1);
    }
    mbar_init(&ctl->xbar, 1);
    ctl->cta_abort = 0;
    ctl->cbad = 0;
    ctl->flag[0] = ctl->flag[1] = 0;
    // a device error from an earlier step is sticky until the host resets
    ctl->skip = (ld_relaxed(p.sync + S_STATUS) != 0u || ld_relaxed(p.sync + S_ABORT) != 0u);
    // the swizzled operand layouts assume 1024-byte aligned shared memory
    if ((p.tc || p.tm) && (smem_u32(smem) & 1023u) != 0u) {
      raise_error(p, MK_ERR_UNSUPPORTED, 0xfffffff0u, smem_u32(smem), 0u);
      ctl->skip = 1;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const bool tmem_owner = (p.tc || p.tm) && !ctl->skip && (threadIdx.x >> 5) == 1;
  const uint32_t tmem_cols = p.tm ? static_cast<uint32_t>(kTmSlots * kTmSlotCols) : kTcTmemCols;
  if (tmem_owner) tmem_alloc(&ctl->tmem, tmem_cols);
  if (p.tc || p.tm) tc_fence_before();
  __syncthreads();
  if (p.tc || p.tm) tc_fence_after();
  if (!ctl->skip) {
    const int warp = threadIdx.x >> 5;
    if (warp == kLoaderWarp) {
      loader_main<V>(p, ctl, smem);
    } else if (warp == kStorerWarp) {
      storer_main(p, ctl, smem);
    } else {
      compute_main<V>(p, ctl, smem);
    }
  }
  if (p.tc || p.tm) tc_fence_before();
  __syncthreads();
  if (p.tc || p.tm) tc_fence_after();
  if (tmem_owner) tmem_dealloc(ctl->tmem, tmem_cols);
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

// The kernel's dynamic shared-memory limit on the current device is set to
// the most any layout may use there (every layout stays within
// min(device opt-in, kMaxSmem)), never to one plan's own size: plans of
// different shapes and the no-allocation entry point share the kernel, and a
// later, smaller setting would fail the launches of an earlier, larger one.
namespace {
// the variants plans use: mma.sync or tcgen05 projections, 4-bit weights
// only on mma.sync, each with either attention path
constexpr int kVariants[] = {0,           kVarTc,   kVarW4, kVarAttnMma, kVarTc | kVarAttnMma,
                             kVarW4 | kVarAttnMma, kVarTm, kVarTm | kVarAttnMma};

const void *kernel_for(int v) {
  switch (v) {
    case 0: return reinterpret_cast<const void *>(mk_step_kernel<0>);
    case kVarTc: return reinterpret_cast<const void *>(mk_step_kernel<kVarTc>);
    case kVarW4: return reinterpret_cast<const void *>(mk_step_kernel<kVarW4>);
    case kVarAttnMma: return reinterpret_cast<const void *>(mk_step_kernel<kVarAttnMma>);
    case kVarTc | kVarAttnMma:
      return reinterpret_cast<const void *>(mk_step_kernel<kVarTc | kVarAttnMma>);
    case kVarW4 | kVarAttnMma:
      return reinterpret_cast<const void *>(mk_step_kernel<kVarW4 | kVarAttnMma>);
    case kVarTm: return reinterpret_cast<const void *>(mk_step_kernel<kVarTm>);
    case kVarTm | kVarAttnMma:
      return reinterpret_cast<const void *>(mk_step_kernel<kVarTm | kVarAttnMma>);
    default: return nullptr;
  }
}
}  // namespace

int kernel_variant(const Params &p) {
  return (p.tc ? kVarTc : 0) | (p.w4 ? kVarW4 : 0) | (p.attn_mma ? kVarAttnMma : 0) |
         (p.tm ? kVarTm : 0);
}

cudaError_t configure_kernel(int smem_optin) {
  const int lim = smem_optin < kMaxSmem ? smem_optin : kMaxSmem;
  for (int v : kVariants) {
    const cudaError_t e =
        cudaFuncSetAttribute(kernel_for(v), cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_step(const Params &p, int grid, int smem, bool cooperative, cudaStream_t stream) {
  const void *fn = kernel_for(kernel_variant(p));
  if (fn == nullptr) return cudaErrorInvalidValue;
  void *args[] = {const_cast<Params *>(&p)};
  if (cooperative)
    return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kThreads), args,
                                       static_cast<size_t>(smem), stream);
  return cudaLaunchKernel(fn, dim3(grid), dim3(kThreads), args, static_cast<size_t>(smem),
                          stream);
}

}  // namespace mk
