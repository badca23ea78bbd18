// The decode interpreter: one persistent CTA per SM runs a queue of
// instructions (fetch -> stage the input vector -> stream weight pages ->
// compute -> store -> signal), after the on-GPU interpreter of the "Hazy
// megakernel summary" page (section 四(二)) and the task loop of the
// "Mirage Persistent Kernel" article (Part 2).
//
// Warp roles (this build's design for sm_100a):
//   warps 0, 1 (lane 0 of each)  loaders: walk the same queue ahead of the
//                   compute warps and stream every weight / KV page of every
//                   instruction into a ring of 16 KiB shared-memory pages
//                   with 1-D bulk copies (cp.async.bulk, mbarrier
//                   completion); loader i owns the pages g with g % 2 == i.
//                   Weights never depend on activations, so the next
//                   instructions' pages load while the current one is still
//                   waiting or storing (the paged shared memory of the same
//                   section, whose freed pages go to the next instruction).
//   warps 2..9      compute: CUDA-core fp32 FMA matrix-vector products over
//                   bf16 pages (batch 1 is a matrix-vector product; tensor
//                   cores do not help there, section 五(二)), warp-shuffle
//                   reductions, fused epilogues, and the signalling.
// Synchronisation between instructions: activations are tagged words that
// carry the step number (epoch), so a reader tells this step's value from a
// stale one by itself; completion counters in global memory (section 四(二)
// "同步") are relaxed hints telling a waiting CTA when to look again.
// Counters are never reset: targets are epoch * producers.  Every wait is
// bounded by a global-timer deadline; a timeout records MK_ERR_TIMEOUT and
// makes every CTA leave cleanly.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mk.h"
#include "mk_internal.h"

namespace mk {
// Internal linkage: every translation unit that includes this file (the
// generic build and each shape-specialised build) gets its own copy.
namespace {
typedef unsigned long long llw;

// ============================================================== PTX helpers
namespace px {

__device__ __forceinline__ uint32_t sa(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(sa(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sa(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(sa(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(sa(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// packed fp32 pair FMA (two lanes of fp32 in one 64-bit register pair)
__device__ __forceinline__ unsigned long long f2pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void ffma2(unsigned long long &acc, unsigned long long a, unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ float f2sum(unsigned long long v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return lo + hi;
}
// Bring [src, src + bytes) into L2 (no completion to wait for).
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(sa(dst)),
      "l"(src), "r"(bytes), "r"(sa(bar)), "l"(policy)
      : "memory");
}
// ---- 5th-generation tensor cores (tcgen05): MMA with the accumulator in
// tensor memory.  Shared-memory operands use the K-major layout without
// swizzle: 16-byte rows of 8 bf16, 8-row groups `sbo` bytes apart, the two
// 8-element K chunks of one MMA `lbo` bytes apart.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);  // version 1, no swizzle
}
// D (f32) += A (bf16, M x 16, K-major) * B (bf16, N x 16, K-major)^T; one thread issues.
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}
// arrive on `bar` once every MMA this thread issued so far has completed
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(sa(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// 16 consecutive f32 columns of this warp's 32 tensor-memory lanes
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_add_acq_rel(unsigned *p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ int ld_volatile(const int *p) { return *(const volatile int *)p; }
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ void red_relaxed_add(unsigned *p, unsigned v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_relaxed_add(unsigned *p, unsigned v) {
  unsigned old;
  asm volatile("atom.relaxed.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ unsigned ld_relaxed(const unsigned *p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
// Tagged activation words: (step tag << 32 | value bits), stored and loaded as
// single-copy-atomic 64-bit accesses, so a reader can tell this step's value
// from a stale one without any fence between the writer's data and a flag.
__device__ __forceinline__ void st_ll(llw *a, float v, uint32_t tag) {
  const llw w = ((llw)tag << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(a), "l"(w) : "memory");
}
__device__ __forceinline__ void st_u64(unsigned long long *a, unsigned long long w) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(a), "l"(w) : "memory");
}
__device__ __forceinline__ llw ld_ll(const llw *a) {
  llw w;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(a));
  return w;
}
__device__ __forceinline__ void ld_ll2(const llw *a, llw &x, llw &y) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(x), "=l"(y) : "l"(a));
}
__device__ __forceinline__ bool ll_fresh(llw w, uint32_t tag) { return (uint32_t)(w >> 32) == tag; }
__device__ __forceinline__ float ll_f(llw w) { return __uint_as_float((uint32_t)w); }
// Tagged fp32 activations (the bulk of the exchanged data): the value rounded
// to 22 significant bits (21 stored mantissa bits and the implicit one), its
// two lowest mantissa bits replaced by the step number mod 4.  Every such word is rewritten every step, so the only stale
// value a reader can meet is the previous step's (or zero-filled memory
// before the first step): a 2-bit tag tells them apart, and 4-byte words keep
// the traffic and registers of plain fp32.
__device__ __forceinline__ uint32_t tf_pack(float v, uint32_t tag) {
  return ((__float_as_uint(v) + 2u) & ~3u) | (tag & 3u);
}
__device__ __forceinline__ void st_tf(float *a, float v, uint32_t tag) {
  asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(a), "r"(tf_pack(v, tag)) : "memory");
}
__device__ __forceinline__ uint32_t ld_tf(const float *a) {
  uint32_t u;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(u) : "l"(a));
  return u;
}
__device__ __forceinline__ uint4 ld_tf4(const float *a) {
  uint4 u;
  asm volatile("ld.relaxed.gpu.global.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
               : "l"(a));
  return u;
}
// Named barrier over the 256 compute threads, returning the OR of `pred`
// over them (a uniform decision for every compute thread).
__device__ __forceinline__ bool cbar_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " barrier.cta.red.or.pred q, 2, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "n"(kComputeThreads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void cbar() {
  asm volatile("barrier.cta.sync 1, %0;" ::"n"(kComputeThreads) : "memory");
}
__device__ __forceinline__ float4 ldcg4(const float *p) { return __ldcg(reinterpret_cast<const float4 *>(p)); }
__device__ __forceinline__ float ldcg(const float *p) { return __ldcg(p); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
__device__ __forceinline__ uint16_t f2bf(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

}  // namespace px

// ============================================================== shared state
struct Shared {
  int abort;       // this CTA saw a failed wait
  int flag;        // broadcast slot
  int pad[2];
  float2 rope[64]; // (cos, sin) of sequence 0's position
  int pos[kMaxBatch], tok[kMaxBatch];  // this step's (clamped) positions and token ids
  int stat_cwait;  // trace mode: pages a compute warp found not yet landed (this instruction)
  int stat_llretry;  // tagged-load groups re-issued because a word was stale (this instruction)
  // the current instruction's dependency: its producers' completion counter
  // (kNoCounter: none), the count that means "all done", and who polls it
  uint32_t dep_ctr, dep_target;
  int dep_seq;
  int dep_state;   // 0: not checked, 1: a thread is polling, 2: met, 3: failed
  // tensor-core LM head (batched builds): tensor-memory columns, the MMA
  // completion barrier and how many times it has completed
  uint32_t tmem_base;
  uint32_t mma_phase;
  unsigned long long mma_bar;
  uint32_t slot_last[16];  // 1 + the last page issued into each ring slot (0: never)
  float red[kComputeWarps][kMaxBatch];
  float argv[kComputeWarps][kMaxBatch];
  int argi[kComputeWarps][kMaxBatch];
};

// ============================================================== small helpers

__device__ void record_error(const KParams &p, int code, int a, int b, int c, int d) {
  if (atomicCAS(p.status, 0, code) == 0) {
    p.status[2] = a;
    p.status[3] = b;
    p.status[4] = c;
    p.status[5] = d;
    p.status[6] = blockIdx.x;
  }
  if (code == MK_ERR_TIMEOUT) atomicExch(p.status + 1, 1);
}

__device__ __forceinline__ bool global_abort(const KParams &p) { return px::ld_volatile(p.status + 1) != 0; }

// positions and token ids are read once per launch into shared memory
__device__ __forceinline__ int read_pos(const Shared *sh, int b) { return sh->pos[b]; }
__device__ __forceinline__ int read_tok(const Shared *sh, int b) { return sh->tok[b]; }
// KV-cache sequence of row b: b in decode steps (kv_seq0 = 0), the prompt's
// sequence kv_seq0 for every row of a prompt chunk
__device__ __forceinline__ int kv_seq(const KParams &p, int b) { return p.kv_seq0 + (p.chunk_n > 0 ? 0 : b); }
// rows of a prompt chunk past its last token: computed, never stored
__device__ __forceinline__ bool chunk_pad(const KParams &p, int b) { return p.chunk_n > 0 && b >= p.chunk_n; }

// Tagged loads are consumed in groups: every word of a group is loaded, the
// values are used as loaded, and `ok` collects whether each word carried this
// step's tag.  A group with a stale word is re-issued as a whole (one round
// trip per retry, not one per stale word), bounded like every other wait.
__device__ __forceinline__ float ll_chk(llw w, uint32_t tag, bool &ok) {
  ok &= px::ll_fresh(w, tag);
  return px::ll_f(w);
}
__device__ __forceinline__ float tf_chk(uint32_t u, uint32_t tag, bool &ok) {
  ok &= ((u ^ tag) & 3u) == 0;
  return __uint_as_float(u & ~3u);
}
__device__ __forceinline__ float4 tf_chk4(uint4 u, uint32_t tag, bool &ok) {
  ok &= (((u.x ^ tag) | (u.y ^ tag) | (u.z ^ tag) | (u.w ^ tag)) & 3u) == 0;
  return make_float4(__uint_as_float(u.x & ~3u), __uint_as_float(u.y & ~3u), __uint_as_float(u.z & ~3u),
                     __uint_as_float(u.w & ~3u));
}
__device__ __noinline__ bool ll_give_up(const KParams *p, Shared *sh, uint64_t t0, int where) {
  if (px::ld_volatile(&sh->abort) || global_abort(*p)) return true;
  if (px::gtimer() - t0 > (uint64_t)p->timeout_ns) {
    record_error(*p, MK_ERR_TIMEOUT, -3, where, 0, 0);
    sh->abort = 1;
    return true;
  }
  return false;
}
// Called after a group came back with a stale word: true = re-issue it,
// false = give up (timeout or abort; the CTA is aborting, values are unused).
// The first retry is immediate, later ones back off (the words are on their
// way; re-issuing at once would only add L2 traffic).
struct LLRetry {
  unsigned n = 0;
  uint64_t t0 = 0;
};
__device__ __forceinline__ bool ll_retry(const KParams &p, Shared *sh, LLRetry &r, int where) {
  if (r.n++ == 0) {
    atomicAdd(&sh->stat_llretry, 1);
    r.t0 = px::gtimer();
  } else {
    __nanosleep(128);
    if ((r.n & 7u) == 0 && ll_give_up(&p, sh, r.t0, where)) return false;
  }
  return true;
}

// Wait until counter idx reaches target; one thread.  false on timeout/abort.
__device__ bool wait_counter(const KParams &p, unsigned idx, unsigned target, int seq) {
  const unsigned *c = p.ctr + idx;
  if ((int)(px::ld_relaxed(c) - target) >= 0) return true;
  const uint64_t t0 = px::gtimer();
  for (unsigned it = 1;; ++it) {
    unsigned v = px::ld_relaxed(c);
    if ((int)(v - target) >= 0) return true;
    if ((it & 31u) == 0) {
      if (global_abort(p)) return false;
      if (px::gtimer() - t0 > (uint64_t)p.timeout_ns) {
        record_error(p, MK_ERR_TIMEOUT, seq, (int)idx, (int)v, (int)target);
        return false;
      }
    }
  }
}

// The current instruction's producers (sh->dep_*): thread 0 waits for their
// completion count unless it is already known to be met; then every compute
// thread passes a barrier.  Called by all compute threads together, only
// after some thread found a stale input word.
__device__ __noinline__ void dep_sync_wait(const KParams *p, Shared *sh) {
  if (sh->dep_state != 2 && sh->dep_ctr != kNoCounter) {
    const bool ok = wait_counter(*p, sh->dep_ctr, sh->dep_target, sh->dep_seq);
    if (!ok) sh->abort = 1;
    sh->dep_state = ok ? 2 : 3;
  } else {
    sh->dep_state = 2;
  }
}

// Wait for an mbarrier phase; bounded, abort-aware.  Any thread.
__device__ bool wait_bar(const KParams &p, Shared *sh, uint64_t *bar, uint32_t parity, int what) {
  if (px::mbar_test(bar, parity)) return true;
  const uint64_t t0 = px::gtimer();
  for (unsigned it = 1;; ++it) {
    if (px::mbar_test(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (px::ld_volatile(&sh->abort) || global_abort(p)) return false;
      if (px::gtimer() - t0 > (uint64_t)p.timeout_ns) {
        record_error(p, MK_ERR_TIMEOUT, -1, what, (int)parity, 0);
        return false;
      }
    }
  }
}

// Attention split geometry of sequence b: positions [start, end) of split s
// (of S), the cached prefix [start, pref_end) that the loader streams, and
// whether the current position belongs to this split.
struct SplitRange {
  int pos, start, end, pref_end;
  bool has_cur;
};
__device__ __forceinline__ SplitRange split_range(const KParams &p, const Shared *sh, int b, int s) {
  SplitRange r;
  r.pos = read_pos(sh, b);
  if (p.chunk_n > 1) {
    // a prompt chunk of several tokens: the S splits share the positions
    // cached before the chunk; the last split also takes the chunk's own
    // rows up to this row's position (this step's K/V exchange, not the cache)
    const int n = p.chunk_pos0, chunk = (n + p.S - 1) / p.S;
    r.start = min(n, s * chunk);
    r.end = min(n, r.start + chunk);
    r.pref_end = r.end;
    r.has_cur = s == p.S - 1;
    return r;
  }
  int n = r.pos + 1;
  int chunk = (n + p.S - 1) / p.S;
  r.start = min(n, s * chunk);
  r.end = min(n, r.start + chunk);
  r.pref_end = min(r.end, r.pos);
  r.has_cur = r.start <= r.pos && r.pos < r.end;
  return r;
}
__device__ __forceinline__ int attn_ppp(const KParams &p) { return kPageBytes / (4 * p.d); }  // positions per page

__device__ __forceinline__ bool selected(const KParams &p, const Instr &I) {
  if (p.stage_filter < 0) return true;
  int st = I.op == OP_LMHEAD ? p.L * kStagesPerLayer : I.layer * kStagesPerLayer + (I.op - 1);
  return st == p.stage_filter;
}

// The pages of the packed layout, gathered from the caller's weights in their
// own layout (several smaller bulk copies per page instead of one): the QKV page
// of rotation pairs is two row runs, a gate/up page is a run of gate rows and
// a run of up rows, a down page is Rd row segments of one K piece.  The page
// contents are identical, so the compute side is unchanged.
__device__ __forceinline__ void issue_page_raw(const KParams &p, const Instr &I, int t, uint8_t *dst,
                                               uint64_t *bar, uint64_t pol_w, uint64_t pol_kv, bool prefetch_only) {
  (void)pol_kv;
  if (I.op == OP_OPROJ) {
    const uint16_t *src = p.layers_raw[I.layer].wo + (size_t)(I.a + t) * kPageElems;
    if (prefetch_only) {
      px::bulk_prefetch_l2(src, kPageBytes);
      return;
    }
    px::mbar_expect_tx(bar, kPageBytes);
    px::bulk_g2s(dst, src, kPageBytes, bar, pol_w);
    return;
  }
  const LayerRaw &W = p.layers_raw[I.layer];
  const int j = I.a + t;
  if (!prefetch_only) px::mbar_expect_tx(bar, kPageBytes);
  auto copy = [&](const uint16_t *src, uint32_t off, uint32_t bytes) {
    if (prefetch_only)
      px::bulk_prefetch_l2(src, bytes);
    else
      px::bulk_g2s(dst + off, src, bytes, bar, pol_w);
  };
  if (I.op == OP_QKV) {
    const int half = p.Rh / 2, pph = p.d / p.Rh;
    const int head = j / pph, jj = j % pph;
    const uint16_t *base;
    int hh;
    if (head < p.nq) {
      base = W.wq;
      hh = head;
    } else if (head < p.nq + p.nkv) {
      base = W.wk;
      hh = head - p.nq;
    } else {
      base = W.wv;
      hh = head - p.nq - p.nkv;
    }
    const uint32_t run = (uint32_t)half * p.H * 2;
    copy(base + ((size_t)hh * p.d + jj * half) * p.H, 0, run);
    copy(base + ((size_t)hh * p.d + p.d / 2 + jj * half) * p.H, run, run);
  } else if (I.op == OP_GATEUP) {
    const int half = p.Rh / 2;
    const uint32_t run = (uint32_t)half * p.H * 2;
    copy(W.wg + (size_t)j * half * p.H, 0, run);
    copy(W.wu + (size_t)j * half * p.H, run, run);
  } else {
    const uint32_t seg = (uint32_t)p.KCd * 2;
    for (int r = 0; r < p.Rd; ++r)
      copy(W.wd + (size_t)(j * p.Rd + r) * p.F + (size_t)I.c * p.KCd, r * seg, seg);
  }
}

// Instruction iterator shared by the loader and the compute warps.  Static
// mode: the CTA's own queue.  (The dynamic mode hands instructions from the
// loader to the compute warps through a small shared-memory FIFO.)
struct Queue {
  const Instr *base;
  int len;
};

// ============================================================== loader
// Source of every page of one instruction: page t is one contiguous copy of
// bytes(t) at a + t * stride (and for KV pages a second one at b, into the
// page's second half).  Computed once per instruction.
struct PageSrc {
  const uint16_t *a, *b;
  size_t stride;            // elements between consecutive pages' sources
  uint32_t bytes, last;     // bytes per copy; of the last page's copies
  int npg;
};
__device__ __forceinline__ PageSrc page_src(const KParams &p, const Shared *sh, const Instr &I) {
  PageSrc s;
  s.b = nullptr;
  s.stride = kPageElems;
  s.bytes = s.last = kPageBytes;
  s.npg = (int)I.b;
  switch (I.op) {
    case OP_QKV:
      if (p.layers[I.layer].wqkv_tc) {  // 128-row tiles of [q; k; v], H / 64 pages
        s.a = p.layers[I.layer].wqkv_tc + (size_t)I.a * (p.H / 64) * kPageElems;
        s.npg = (int)I.b * (p.H / 64);
      } else {
        s.a = p.layers[I.layer].wqkv + (size_t)I.a * kPageElems;
      }
      break;
    case OP_OPROJ:
      if (p.layers[I.layer].wo_tc) {  // 128-row tiles, q_dim / 64 pages
        s.a = p.layers[I.layer].wo_tc + (size_t)I.a * (p.qdim / 64) * kPageElems;
        s.npg = (int)I.b * (p.qdim / 64);
      } else {
        s.a = p.layers[I.layer].wo + (size_t)I.a * kPageElems;
      }
      break;
    case OP_GATEUP:
      if (p.layers[I.layer].wgu_tc) {  // 128-row tiles (64 gate + 64 up rows) of H / 64 pages
        s.a = p.layers[I.layer].wgu_tc + (size_t)I.a * (p.H / 64) * kPageElems;
        s.npg = (int)I.b * (p.H / 64);
      } else {
        s.a = p.layers[I.layer].wgu + (size_t)I.a * kPageElems;
      }
      break;
    case OP_DOWN:
      if (p.layers[I.layer].wd_tc) {  // per K piece: 128-row tiles of KCd / 64 pages
        s.a = p.layers[I.layer].wd_tc + ((size_t)I.c * (p.H / 128) + I.a) * (p.KCd / 64) * kPageElems;
        s.npg = (int)I.b * (p.KCd / 64);
      } else {
        s.a = p.layers[I.layer].wd + ((size_t)I.c * (p.H / p.Rd) + I.a) * kPageElems;
      }
      break;
    case OP_LMHEAD: {
      if (p.lm_tc) {  // whole 128-row tiles of H / 64 pages
        s.a = p.lm_tc + (size_t)I.a * (p.H / 64) * kPageElems;
        s.npg = (int)I.b * (p.H / 64);
        break;
      }
      s.a = p.lm_head + (size_t)I.a * p.Rh * p.H;
      const int r_last = (int)(I.a + I.b - 1) * p.Rh;
      const int rows = p.tp_n > 1 ? p.V_lm : p.V;  // a tensor-parallel rank: its vocabulary rows
      s.last = (uint32_t)min(p.Rh, rows - r_last) * p.H * 2;
      break;
    }
    case OP_ATTN: {
      const SplitRange r = split_range(p, sh, I.c, I.b);
      const int ppp = attn_ppp(p), n = r.pref_end - r.start;
      s.npg = n > 0 ? (n + ppp - 1) / ppp : 0;
      const size_t off = (size_t)I.layer * p.kv_ls + (size_t)kv_seq(p, I.c) * p.kv_bs + (size_t)I.a * p.kv_hs +
                         (size_t)r.start * p.d;
      s.a = p.kc + off;
      s.b = p.vc + off;
      s.stride = (size_t)ppp * p.d;
      s.bytes = (uint32_t)ppp * p.d * 2;
      s.last = s.npg > 0 ? (uint32_t)(n - (s.npg - 1) * ppp) * p.d * 2 : 0;
      break;
    }
    default: s.a = nullptr; s.npg = 0; break;
  }
  return s;
}

// L2 prefetch cursor of one loader lane: it walks this loader's future pages
// (the same order as the copies) and, only while the ring is full (the
// compute warps are waiting on a dependency, so HBM would idle), asks L2 for
// pages up to `pf_pages` ahead of the next copy.  The copies of those pages
// then read L2 instead of HBM when their slots free up.
struct PfCursor {
  int qi = -1;         // instruction index in the queue (-1: not started)
  uint32_t g0 = 0;     // its first page number
  uint32_t gp = 0;     // next page number to prefetch (this loader's)
  PageSrc ps;
};
#ifndef MK_PF_GAP_NS
#define MK_PF_GAP_NS 0
#endif
constexpr uint64_t kPfGapNs = MK_PF_GAP_NS;
// Issue one page prefetch; false when the budget is used up or the queue ends.
__device__ __forceinline__ bool pf_step(const KParams &p, const Shared *sh, const Queue &q, PfCursor &c,
                                        uint32_t g_next, int li, int nl) {
  if (c.gp >= g_next + (uint32_t)p.pf_pages) return false;
  while (c.gp >= c.g0 + (uint32_t)c.ps.npg) {
    const uint32_t g_end = c.g0 + (uint32_t)c.ps.npg;
    int k = c.qi + 1;
    while (k < q.len && !selected(p, q.base[k])) ++k;
    if (k >= q.len) return false;
    c.qi = k;
    c.g0 = g_end;
    c.ps = page_src(p, sh, q.base[k]);
    c.gp = g_end + (uint32_t)((li - (int)(g_end % nl) + nl) % nl);
  }
  const int t = (int)(c.gp - c.g0);
  const uint32_t bytes = (t == c.ps.npg - 1) ? c.ps.last : c.ps.bytes;
  px::bulk_prefetch_l2(c.ps.a + (size_t)t * c.ps.stride, bytes);
  if (c.ps.b) px::bulk_prefetch_l2(c.ps.b + (size_t)t * c.ps.stride, bytes);
  c.gp += (uint32_t)nl;
  return true;
}

// One loader lane streams the pages g with g % nl == li of every instruction
// of its CTA's queue into the ring (several loaders overlap the issue
// latency of the bulk copies, which is long for a single thread).
template <bool RAW>
__device__ void run_loader(const KParams &p, Shared *sh, uint8_t *pages, uint64_t *full, uint64_t *empty,
                           Queue q, volatile int *dyn_fifo, volatile int *dyn_tail, volatile int *dyn_head,
                           unsigned epoch, int li, int nl) {
  const uint64_t pol_w = px::policy_evict_first();
  const uint64_t pol_kv = px::policy_evict_last();
  const uint32_t NP = (uint32_t)p.num_pages;
  const uint32_t cap = (uint32_t)p.max_inflight;
  const bool trace = (p.mode & MODE_TRACE) != 0;
  uint32_t g = 0;
  bool ok = true;
  const bool dyn = (p.mode & MODE_DYNAMIC) != 0;
  const bool ev = dyn && (p.mode & MODE_EVENT) != 0;
  // claims per step: every queue entry plus one past the end per CTA
  const unsigned dyn_base = dyn ? (epoch - 1u) * (unsigned)((ev ? p.n_ev : p.n_instr) + gridDim.x) : 0u;
  int claimed = 0;
  const bool use_pf = !RAW && !dyn && p.pf_pages > 0;
  PfCursor pf;
  uint64_t pf_last = 0;
  for (int qi = 0; ok; ++qi) {
    Instr I;
    if (dyn) {
      // claim the next instruction of the global queue; publish it to the compute warps
      unsigned k = atomicAdd(p.ctr + p.dyn_head, 1u) - dyn_base;
      if (ev) {
        // event-driven queue: claim k is ready slot k (the first n_ev_init
        // are the instructions that wait on nothing); a slot past those is
        // filled by the producer that completes a dependency count
        if (k >= (unsigned)p.n_ev) {
          k = (unsigned)p.n_instr;  // past the end: this loader is done
        } else if (k < (unsigned)p.n_ev_init) {
          k = (unsigned)p.ev_init[k];
        } else {
          const uint64_t tw = px::gtimer();
          unsigned long long w;
          for (unsigned it = 1;; ++it) {
            w = px::ld_ll(p.ev_ready + k);
            if ((uint32_t)(w >> 32) == epoch) break;
            if ((it & 31u) == 0 &&
                (px::ld_volatile(&sh->abort) || global_abort(p) || px::gtimer() - tw > (uint64_t)p.timeout_ns)) {
              if (!global_abort(p)) record_error(p, MK_ERR_TIMEOUT, -4, (int)k, (int)(w >> 32), (int)epoch);
              ok = false;
              break;
            }
          }
          if (!ok) break;
          k = (unsigned)(w & 0xffffffffu);
        }
      }
      int slot = claimed & 31;
      const uint64_t t0 = px::gtimer();
      while (claimed - *dyn_head >= 32) {  // FIFO space (bounded)
        if (px::ld_volatile(&sh->abort) || global_abort(p) || px::gtimer() - t0 > (uint64_t)p.timeout_ns) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      dyn_fifo[slot] = k < (unsigned)p.n_instr ? (int)k : -1;
      __threadfence_block();
      *dyn_tail = ++claimed;
      if (k >= (unsigned)p.n_instr) break;
      I = p.instrs[k];
    } else {
      if (qi >= q.len) break;
      I = q.base[qi];
      if (!selected(p, I)) continue;
    }
    unsigned long long *ltr = (trace && li == 0) ? p.trace + (size_t)I.seq * MK_TRACE_WORDS : nullptr;
    if (ltr) ltr[5] = px::gtimer();
    if (li == 0) {
      // the RMSNorm weight the compute warps load with the instruction's
      // input: bring it into L2 now (it is small, and read from HBM it would
      // add a memory round trip to the staging)
      const uint16_t *gamma = I.op == OP_QKV      ? p.layers[I.layer].attn_norm
                              : I.op == OP_GATEUP ? p.layers[I.layer].ffn_norm
                              : I.op == OP_LMHEAD ? p.final_norm
                                                  : nullptr;
      if (gamma && ((uintptr_t)gamma & 15u) == 0 && (p.H * 2) % 16 == 0) px::bulk_prefetch_l2(gamma, (uint32_t)p.H * 2);
    }
    unsigned lwait = 0;
    const PageSrc ps = page_src(p, sh, I);
    const uint32_t g0 = g;
    g += (uint32_t)ps.npg;
    // this loader's pages of the instruction
    for (uint32_t gg = g0 + (uint32_t)((li - (int)(g0 % nl) + nl) % nl); gg < g; gg += nl) {
      const int t = (int)(gg - g0);
      const uint32_t slot = gg % NP;
      const uint32_t ph = (gg / NP) & 1u;
      if (gg >= NP) {
        if (!px::mbar_test(&empty[slot], ph ^ 1u)) {
          if (ltr) ++lwait;
          if (use_pf) {
            // ring full: spend the wait bringing later pages into L2
            if (pf.qi < qi || (pf.qi == qi && pf.gp < gg)) {
              pf.qi = qi;
              pf.g0 = g0;
              pf.gp = gg;
              pf.ps = ps;
            }
            // paced: at most one page per kPfGapNs per loader, so that the
            // look-ahead uses spare HBM bandwidth without queueing ahead of
            // the activation exchanges
            while (!px::mbar_test(&empty[slot], ph ^ 1u)) {
              const uint64_t now = px::gtimer();
              if (now - pf_last < kPfGapNs) continue;
              if (!pf_step(p, sh, q, pf, gg, li, nl)) break;
              pf_last = now;
            }
          }
        }
        if (!wait_bar(p, sh, &empty[slot], ph ^ 1u, 1)) {
          ok = false;
          break;
        }
      }
      // keep at most `cap` pages in flight: more only queues in the memory
      // system and delays every other access of this SM
      if (cap > 0 && gg >= cap) {
        const uint32_t k = gg - cap;
        if (!wait_bar(p, sh, &full[k % NP], (k / NP) & 1u, 3)) {
          ok = false;
          break;
        }
      }
      uint8_t *dst = pages + (size_t)slot * kPageBytes;
      sh->slot_last[slot] = gg + 1;
      if constexpr (RAW) {
        if (I.op == OP_QKV || I.op == OP_GATEUP || I.op == OP_DOWN || I.op == OP_OPROJ) {
          issue_page_raw(p, I, t, dst, &full[slot], pol_w, pol_kv, false);
          continue;
        }
      }
      const uint32_t bytes = (t == ps.npg - 1) ? ps.last : ps.bytes;
      if (ps.b) {
        px::mbar_expect_tx(&full[slot], 2 * bytes);
        px::bulk_g2s(dst, ps.a + (size_t)t * ps.stride, bytes, &full[slot], pol_kv);
        px::bulk_g2s(dst + kPageBytes / 2, ps.b + (size_t)t * ps.stride, bytes, &full[slot], pol_kv);
      } else {
        px::mbar_expect_tx(&full[slot], bytes);
        px::bulk_g2s(dst, ps.a + (size_t)t * ps.stride, bytes, &full[slot], pol_w);
      }
    }
    if (ltr) {
      ltr[6] = px::gtimer();
      ltr[9] = lwait;
    }
    if (!ok) break;  // copies already issued land before the CTA exits: thread 0 waits on
                     // each ring slot's last issued page (slot_last) at the end of the kernel
    if (px::ld_volatile(&sh->abort) || global_abort(p)) ok = false;
  }
  if (dyn && ok == false) {
    // make sure the compute warps see the end of the queue
    dyn_fifo[claimed & 31] = -1;
    __threadfence_block();
    *dyn_tail = claimed + 1;
  }
}

// ============================================================== compute
struct CCtx {
  const KParams &p;
  Shared *sh;
  uint8_t *pages;
  float *act;     // staging region (input vector(s), attention scratch)
  int act_stride; // floats per sequence in the staging region
  uint64_t *full, *empty;
  unsigned epoch;
  int cw, lane, ctid;
  uint32_t g;     // page sequence number (same as the loader's)
  unsigned long long *tr;  // this instruction's trace record (or null)
  float *xch;     // batched builds: tensor-core epilogue exchange [128 rows][16 sequences]
};

// Register-resident view of the page ring (copied out of the context once per
// instruction so that no loop reloads it from memory after a barrier or an
// mbarrier poll).
struct Ring {
  uint8_t *pages;
  uint64_t *full, *empty;
  Shared *sh;
  uint32_t np;
};
__device__ __forceinline__ Ring ring_of(const CCtx &c) {
  return Ring{c.pages, c.full, c.empty, c.sh, (uint32_t)c.p.num_pages};
}
// Wait for ring page g (every compute warp calls this for pages it reads).
// A parity test only tells the last two phases apart, so first make sure the
// slot's previous page (g - np, possibly another warp's) has been released:
// then its full barrier is in page g's phase (pending or complete) and the
// parity test is unambiguous.  (The previous use of the empty barrier, page
// g - 2np, belongs to this same warp because 2np is a multiple of the warp
// count, so that test is unambiguous too.)
__device__ __forceinline__ bool ring_wait(const KParams &p, const Ring &r, uint32_t g) {
  const uint32_t slot = g % r.np;
  const uint32_t ph = (g / r.np) & 1u;
  if (g >= r.np && !px::mbar_test(&r.empty[slot], ph ^ 1u)) {
    if (px::ld_volatile(&r.sh->abort)) return false;
    if (!wait_bar(p, r.sh, &r.empty[slot], ph ^ 1u, 4)) {
      r.sh->abort = 1;
      return false;
    }
  }
  if (px::mbar_test(&r.full[slot], ph)) return true;  // fast path: already landed
  if ((threadIdx.x & 31) == 0) atomicAdd(&r.sh->stat_cwait, 1);
  if (px::ld_volatile(&r.sh->abort)) return false;
  if (!wait_bar(p, r.sh, &r.full[slot], ph, 0)) {
    r.sh->abort = 1;
    return false;
  }
  return true;
}
// Split pages (every compute warp consumes every page of the instruction, in
// order): when a warp waits for page g, page g - np has landed (this warp
// consumed it, or -- in an earlier instruction -- its owner did before the
// instruction's closing barrier), and page g + np cannot have been issued
// (that needs this warp's release of page g).  So the full barrier's parity
// test alone is unambiguous; slot and phase are tracked by the caller.
__device__ __forceinline__ bool ring_wait_full(const KParams &p, const Ring &r, uint32_t slot, uint32_t ph) {
  if (px::mbar_test(&r.full[slot], ph)) return true;
  if ((threadIdx.x & 31) == 0) atomicAdd(&r.sh->stat_cwait, 1);
  if (px::ld_volatile(&r.sh->abort)) return false;
  if (!wait_bar(p, r.sh, &r.full[slot], ph, 0)) {
    r.sh->abort = 1;
    return false;
  }
  return true;
}
__device__ __forceinline__ const uint8_t *ring_page(const Ring &r, uint32_t g) {
  return r.pages + (size_t)(g % r.np) * kPageBytes;
}
__device__ __forceinline__ void ring_release(const Ring &r, uint32_t g, uint32_t count) {
  px::mbar_arrive(&r.empty[g % r.np], count);
}
__device__ __forceinline__ bool page_ready(CCtx &c, uint32_t g) { return ring_wait(c.p, ring_of(c), g); }
__device__ __forceinline__ const uint8_t *page_ptr(CCtx &c, uint32_t g) { return ring_page(ring_of(c), g); }
__device__ __forceinline__ void page_release(CCtx &c, uint32_t g, uint32_t count) {
  ring_release(ring_of(c), g, count);
}

// Load this thread's share of an instruction's tagged inputs: `attempt(ok)`
// issues every load and clears ok if a word was stale.  If any compute
// thread saw a stale word, thread 0 waits for the producers' completion count
// (at most once per instruction) while the others wait at a barrier, and then
// the threads with stale words re-issue their loads until every word is
// fresh.  Called by all compute threads together.
template <class F>
__device__ __forceinline__ void settle(CCtx &c, int where, F &&attempt) {
  LLRetry r;
  for (bool first = true;; first = false) {
    bool ok = true;
    attempt(ok);
    if (first) {
      if (!px::cbar_or(!ok)) break;  // every word fresh: the common case
      if (c.ctid == 0) dep_sync_wait(&c.p, c.sh);
      px::cbar();
      if (ok) break;
      continue;  // the producers are done: re-issue at once
    }
    if (ok || !ll_retry(c.p, c.sh, r, where)) break;
  }
}

// Staging layout of an input vector of length K (fp32): element e of 8-chunk
// ch = e / 8 lives at float4 slot ch (elements 0..3 of the chunk) or at
// K/8 + ch (elements 4..7), so lane-consecutive chunks are bank-conflict free.
__device__ __forceinline__ int stage_slot4(int e4, int K) { return (e4 & 1) * (K / 8) + (e4 >> 1); }

// x_in of layer l (the residual stream entering layer l) for elements
// 4*e4 .. 4*e4+3 of sequence b: the embedding for l == 0, else xres[l-1] +
// the down-projection pieces of layer l-1 (fixed order).  Tagged loads: all
// issued before any is checked.
__device__ __forceinline__ float4 layer_input4(const KParams &p, uint32_t tag, int l, int b, int tok, int e4,
                                               bool &ok) {
  if (l == 0) {
    const uint2 w = __ldg(reinterpret_cast<const uint2 *>(p.embed + (size_t)tok * p.H) + e4);
    return make_float4(px::bf_lo(w.x), px::bf_hi(w.x), px::bf_lo(w.y), px::bf_hi(w.y));
  }
  const size_t BH = (size_t)p.B * p.H;
  float4 x = tf_chk4(px::ld_tf4(p.xres + (size_t)(l - 1) * BH + (size_t)b * p.H + e4 * 4), tag, ok);
  for (int k0 = 0; k0 < p.ndp; k0 += 4) {  // four pieces' loads in flight at a time
    uint4 d[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k0 + k < p.ndp) d[k] = px::ld_tf4(p.dpart + ((size_t)(l - 1) * p.ndp + k0 + k) * BH + (size_t)b * p.H + e4 * 4);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k0 + k < p.ndp) {
        const float4 v = tf_chk4(d[k], tag, ok);
        x.x += v.x;
        x.y += v.y;
        x.z += v.z;
        x.w += v.w;
      }
  }
  return x;
}
__device__ __forceinline__ float layer_input1(const KParams &p, uint32_t tag, int l, int b, int tok, int e,
                                              bool &ok) {
  if (l == 0) return px::bf16f(__ldg(p.embed + (size_t)tok * p.H + e));
  const size_t BH = (size_t)p.B * p.H;
  float x = tf_chk(px::ld_tf(p.xres + (size_t)(l - 1) * BH + (size_t)b * p.H + e), tag, ok);
  for (int k0 = 0; k0 < p.ndp; k0 += 4) {
    uint32_t d[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k0 + k < p.ndp) d[k] = px::ld_tf(p.dpart + ((size_t)(l - 1) * p.ndp + k0 + k) * BH + (size_t)b * p.H + e);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k0 + k < p.ndp) x += tf_chk(d[k], tag, ok);
  }
  return x;
}
__device__ __noinline__ float layer_input1_settled(const KParams &p, Shared *sh, uint32_t tag, int l, int b, int tok,
                                                   int e) {
  float x;
  for (LLRetry r;;) {
    bool ok = true;
    x = layer_input1(p, tag, l, b, tok, e, ok);
    if (ok || !ll_retry(p, sh, r, 1)) break;
  }
  return x;
}

// four consecutive tagged words as a float4
__device__ __forceinline__ float4 ll_load4(uint32_t tag, const float *a, bool &ok) {
  return tf_chk4(px::ld_tf4(a), tag, ok);
}

// Stage x*gamma for every sequence, x = layer_input(l) (l == L: final norm),
// and return inv[b] = 1 / rms(x_b): the consumer scales its dot products,
// since W (x*gamma*inv) == (W (x*gamma)) * inv, so the matrix-vector pages
// need not wait for a second pass over the staged vector.  One compute
// barrier.
// IT = float4 loads per thread (H / 4 / 256, at least 1), fixed by the caller's
// rows-per-page so that every load is issued before the first one is used.
// bf16 pair (hi, lo) with hi + lo == x to about 16 significant bits: the
// tensor-core path multiplies bf16 weights by both halves of each activation
__device__ __forceinline__ void split_bf16x4(float4 x, uint16_t *hi, uint16_t *lo) {
  const uint16_t h0 = px::f2bf(x.x), h1 = px::f2bf(x.y), h2 = px::f2bf(x.z), h3 = px::f2bf(x.w);
  const uint16_t l0 = px::f2bf(x.x - px::bf16f(h0)), l1 = px::f2bf(x.y - px::bf16f(h1)),
                 l2 = px::f2bf(x.z - px::bf16f(h2)), l3 = px::f2bf(x.w - px::bf16f(h3));
  *reinterpret_cast<uint2 *>(hi) = make_uint2((uint32_t)h0 | ((uint32_t)h1 << 16), (uint32_t)h2 | ((uint32_t)h3 << 16));
  *reinterpret_cast<uint2 *>(lo) = make_uint2((uint32_t)l0 | ((uint32_t)l1 << 16), (uint32_t)l2 | ((uint32_t)l3 << 16));
}

// TC: stage x*gamma as bf16 (hi, lo) in the tensor cores' K-major layout
// instead: 8-element chunk ch of sequence b at byte ((ch * 16) + b) * 16 of
// the hi block (H * 32 bytes), the lo block right after it.
template <int NB, int IT, bool TC = false>
__device__ void stage_norm(CCtx &c, int l, const uint16_t *gamma, bool from_xres_only, float (&inv)[NB]) {
  const KParams &p = c.p;
  const int H = p.H, n4 = H / 4;
  float ss[NB];
  uint2 gws[IT];
#pragma unroll
  for (int b = 0; b < NB; ++b) ss[b] = 0.f;
  // sequences in groups of GB: one group's loads are in flight together
  constexpr int GB = NB == 1 ? 1 : 4;
#pragma unroll
  for (int b0 = 0; b0 < NB; b0 += GB) {
    if (b0 >= p.B) break;
    float4 xs[GB][IT];
    settle(c, 2, [&](bool &ok) {
#pragma unroll
      for (int i = 0; i < GB; ++i) {
        const int b = b0 + i;
        if (b >= p.B) break;
        const int tok = (l == 0 && !from_xres_only) ? read_tok(c.sh, b) : 0;
#pragma unroll
        for (int it = 0; it < IT; ++it) {
          const int e4 = c.ctid + it * kComputeThreads;
          if (e4 < n4) {
            if (b == 0) gws[it] = __ldg(reinterpret_cast<const uint2 *>(gamma) + e4);  // with x: one round trip
            if (from_xres_only)
              xs[i][it] = ll_load4(c.epoch, p.xres + ((size_t)l * p.B + b) * H + e4 * 4, ok);
            else if (NB > 1 && p.xin && l > 0)  // summed once by the down tiles
              xs[i][it] = ll_load4(c.epoch, p.xin + ((size_t)(l - 1) * p.B + b) * H + e4 * 4, ok);
            else
              xs[i][it] = layer_input4(p, c.epoch, l, b, tok, e4, ok);
          }
        }
      }
    });
#pragma unroll
    for (int i = 0; i < GB; ++i) {
      const int b = b0 + i;
      if (b >= p.B) break;
      float4 *dst = reinterpret_cast<float4 *>(c.act + (size_t)b * c.act_stride);
#pragma unroll
      for (int it = 0; it < IT; ++it) {
        const int e4 = c.ctid + it * kComputeThreads;
        if (e4 < n4) {
          const float4 x = xs[i][it];
          const uint2 gw = gws[it];
          ss[b] += x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
          const float4 xg =
              make_float4(x.x * px::bf_lo(gw.x), x.y * px::bf_hi(gw.x), x.z * px::bf_lo(gw.y), x.w * px::bf_hi(gw.y));
          if constexpr (TC) {
            uint16_t *hi = reinterpret_cast<uint16_t *>(c.act);
            const size_t o = ((size_t)(e4 >> 1) * 16 + b) * 8 + (e4 & 1) * 4;
            split_bf16x4(xg, hi + o, hi + (size_t)H * 16 + o);
          } else {
            dst[stage_slot4(e4, H)] = xg;
          }
        }
      }
    }
  }
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    float v = px::warp_sum(ss[b]);
    if (c.lane == 0) c.sh->red[c.cw][b] = v;
  }
  px::cbar();
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kComputeWarps; ++w) t += c.sh->red[w][b];
    inv[b] = __frsqrt_rn(t * p.inv_H + p.eps);  // one rounding; t * (1/H) == t / H for H = 2^k
  }
  if (c.tr && c.ctid == 0) c.tr[2] = px::gtimer();
}

// Stage a plain fp32 vector slice src[b*src_stride .. + K) for each sequence.
// With nrows > 0 (O projection, batch 1) also stage x_in(l) for output rows
// row0 .. row0+nrows after the vector, loaded in the same round trip.
template <int NB, int IT>
__device__ void stage_copy(CCtx &c, const float *src, size_t src_stride, int K, int l = 0, int row0 = 0,
                           int nrows = 0) {
  const KParams &p = c.p;
  const int n4 = K / 4;
  float xr = 0.f;
  const bool has_row = c.ctid < nrows;
  const int tok0 = l == 0 ? read_tok(c.sh, 0) : 0;
  constexpr int GB = NB == 1 ? 1 : 4;  // sequences whose loads are in flight together
#pragma unroll
  for (int b0 = 0; b0 < NB; b0 += GB) {
    if (b0 >= p.B) break;
    float4 vs[GB][IT];
    settle(c, 3, [&](bool &ok) {  // the row of x_in rides along with sequence 0's vector
      if (b0 == 0 && has_row) xr = layer_input1(p, c.epoch, l, 0, tok0, row0 + c.ctid, ok);
#pragma unroll
      for (int i = 0; i < GB; ++i) {
        if (b0 + i >= p.B) break;
#pragma unroll
        for (int it = 0; it < IT; ++it) {
          const int e4 = c.ctid + it * kComputeThreads;
          if (e4 < n4) vs[i][it] = ll_load4(c.epoch, src + (size_t)(b0 + i) * src_stride + e4 * 4, ok);
        }
      }
    });
#pragma unroll
    for (int i = 0; i < GB; ++i) {
      if (b0 + i >= p.B) break;
      float4 *dst = reinterpret_cast<float4 *>(c.act + (size_t)(b0 + i) * c.act_stride);
#pragma unroll
      for (int it = 0; it < IT; ++it) {
        const int e4 = c.ctid + it * kComputeThreads;
        if (e4 < n4) dst[stage_slot4(e4, K)] = vs[i][it];
      }
    }
  }
  for (int r = c.ctid; r < nrows; r += kComputeThreads)
    c.act[K + r] = (r == c.ctid) ? xr : layer_input1_settled(p, c.sh, c.epoch, l, 0, tok0, row0 + r);
  px::cbar();
  if (c.tr && c.ctid == 0) c.tr[2] = px::gtimer();
}

// acc[b][r] = dot(page row r, staged vector b) for R rows of KC = 8192/R
// columns; every lane ends with every result (up to 4 sequences; more use
// mv_page_t).
template <int NB, int R>
__device__ __forceinline__ void mv_page(const uint8_t *page, const float *act, int act_stride, int B, int lane,
                                        float (&acc)[NB][R]) {
  static_assert(NB <= 4, "more sequences: mv_page_t");
  constexpr int KC = kPageElems / R;
  constexpr int CH = KC / 8;  // 16-byte chunks per row
  const uint4 *pg = reinterpret_cast<const uint4 *>(page);
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int r = 0; r < R; ++r) acc[b][r] = 0.f;
#pragma unroll(CH / 32 > 2 ? 2 : CH / 32)
  for (int j = 0; j < CH / 32; ++j) {
    const int ch = lane + 32 * j;
    uint4 w[R];
#pragma unroll
    for (int r = 0; r < R; ++r) w[r] = pg[r * CH + ch];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (NB > 1 && b >= B) break;
      const float4 *a = reinterpret_cast<const float4 *>(act + (size_t)b * act_stride);
      const float4 a0 = a[ch], a1 = a[CH + ch];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float s = acc[b][r];
        s = fmaf(px::bf_lo(w[r].x), a0.x, s);
        s = fmaf(px::bf_hi(w[r].x), a0.y, s);
        s = fmaf(px::bf_lo(w[r].y), a0.z, s);
        s = fmaf(px::bf_hi(w[r].y), a0.w, s);
        s = fmaf(px::bf_lo(w[r].z), a1.x, s);
        s = fmaf(px::bf_hi(w[r].z), a1.y, s);
        s = fmaf(px::bf_lo(w[r].w), a1.z, s);
        s = fmaf(px::bf_hi(w[r].w), a1.w, s);
        acc[b][r] = s;
      }
    }
  }
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    if (NB > 1 && b >= B) break;
#pragma unroll
    for (int r = 0; r < R; ++r) acc[b][r] = px::warp_sum(acc[b][r]);
  }
}

// pick acc[idx] with a compile-time-unrolled select (no local memory)
template <int R>
__device__ __forceinline__ float pick(const float (&v)[R], int idx) {
  float out = 0.f;
#pragma unroll
  for (int r = 0; r < R; ++r)
    if (r == idx) out = v[r];
  return out;
}

// Butterfly reduction of NV partial sums per lane over the warp, transposed:
// afterwards v[0] of lane L holds the full sum of value index L >> (5 - log2 NV)
// (each sum in 32 / NV lanes), after NV - 1 + log2(32 / NV) shuffles instead of
// 5 per value.
template <int NV>
__device__ __forceinline__ void warp_sum_transposed(float (&v)[NV], int lane) {
  static_assert(NV >= 1 && NV <= 32 && (NV & (NV - 1)) == 0, "power of two up to 32");
  int n = NV;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      const int hn = n / 2;
      const bool up = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < (NV > 1 ? NV / 2 : 1); ++i) {
        if (i < hn) {
          const float send = up ? v[i] : v[i + hn];
          const float keep = up ? v[i + hn] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      n = hn;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
}
constexpr int log2_pow2(int n) { return n <= 1 ? 0 : 1 + log2_pow2(n / 2); }

// Row sums of a page for more than 4 sequences, kept transposed: v[grp] of
// lane L is the sum of (sequence 4 * grp + i, row r) with i * R + r = L >> SH.
// acc_row() fetches one by a shuffle, so a lane holds NB / 4 sums instead of
// NB * R copies of all of them.
template <int NB, int R>
struct AccT {
  static_assert(NB % 4 == 0 && 4 * R <= 32, "groups of 4 sequences, 4 * R sums per group");
  static constexpr int SH = 5 - log2_pow2(4 * R);
  float v[NB / 4];
};
template <int R, int NB>
__device__ __forceinline__ float acc_row(const float (&acc)[NB][R], int b, int r) {
  return pick<R>(acc[b], r);
}
// every lane of the warp must call this (a shuffle); r is taken modulo R
template <int R, int NB>
__device__ __forceinline__ float acc_row(const AccT<NB, R> &acc, int b, int r) {
  return __shfl_sync(0xffffffffu, acc.v[b >> 2], (((b & 3) * R + (r & (R - 1))) << AccT<NB, R>::SH));
}

// mv_page for more than 4 sequences: one pass over the page per group of 4
// sequences, so that the running sums of a pass stay in registers (the page
// is read from shared memory once per group), then one transposed reduction
// of the group's 4 * R sums
template <int NB, int R>
__device__ __forceinline__ void mv_page_t(const uint8_t *page, const float *act, int act_stride, int B, int lane,
                                          AccT<NB, R> &acc) {
  constexpr int KC = kPageElems / R;
  constexpr int CH = KC / 8;  // 16-byte chunks per row
  const uint4 *pg = reinterpret_cast<const uint4 *>(page);
#pragma unroll
  for (int b0 = 0; b0 < NB; b0 += 4) {
    acc.v[b0 / 4] = 0.f;
    if (b0 >= B) continue;
    float part[4 * R];
#pragma unroll
    for (int i = 0; i < 4 * R; ++i) part[i] = 0.f;
#pragma unroll 1
    for (int j = 0; j < CH / 32; ++j) {
      const int ch = lane + 32 * j;
      uint4 w[R];
#pragma unroll
      for (int r = 0; r < R; ++r) w[r] = pg[r * CH + ch];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (b0 + i >= B) break;
        const float4 *a = reinterpret_cast<const float4 *>(act + (size_t)(b0 + i) * act_stride);
        const float4 a0 = a[ch], a1 = a[CH + ch];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float t = part[i * R + r];
          t = fmaf(px::bf_lo(w[r].x), a0.x, t);
          t = fmaf(px::bf_hi(w[r].x), a0.y, t);
          t = fmaf(px::bf_lo(w[r].y), a0.z, t);
          t = fmaf(px::bf_hi(w[r].y), a0.w, t);
          t = fmaf(px::bf_lo(w[r].z), a1.x, t);
          t = fmaf(px::bf_hi(w[r].z), a1.y, t);
          t = fmaf(px::bf_lo(w[r].w), a1.z, t);
          t = fmaf(px::bf_hi(w[r].w), a1.w, t);
          part[i * R + r] = t;
        }
      }
    }
    warp_sum_transposed<4 * R>(part, lane);
    acc.v[b0 / 4] = part[0];
  }
}


// float4 loads per compute thread to stage a K = 8192 / R vector
template <int R>
struct StageIt {
  static constexpr int v = (8 / R) > 0 ? (8 / R) : 1;
};

// ---------------------------------------------------------------- matvec ops
// Loop over the instruction's pages owned by this warp (page g -> warp g % 8).
template <int NB, int R, class Epi>
__device__ __forceinline__ void matvec_pages(CCtx &c, const Instr &I, Epi epi) {
  const KParams &p = c.p;
  const Ring rg = ring_of(c);
  const uint32_t g0 = c.g;
  const int np = (int)I.b, first = (int)I.a, cw = c.cw, lane = c.lane, B = p.B, stride = c.act_stride;
  const float *act = c.act;
  // this warp's pages: g = g0 + t with g % 8 == cw
  int t = (int)((uint32_t)(cw - (int)(g0 % kComputeWarps) + kComputeWarps) % kComputeWarps);
  for (; t < np; t += kComputeWarps) {
    const uint32_t g = g0 + (uint32_t)t;
    if (!ring_wait(p, rg, g)) break;
    if constexpr (NB > 4) {
      AccT<NB, R> acc;
      mv_page_t<NB, R>(ring_page(rg, g), act, stride, B, lane, acc);
      __syncwarp();
      if (lane == 0) ring_release(rg, g, kComputeWarps);
      epi(first + t, acc);
    } else {
      float acc[NB][R];
      mv_page<NB, R>(ring_page(rg, g), act, stride, B, lane, acc);
      __syncwarp();
      if (lane == 0) ring_release(rg, g, kComputeWarps);
      epi(first + t, acc);
    }
  }
  c.g = g0 + (uint32_t)np;
}

// ---------------------------------------------------------------- split pages
// Batch-1 matrix-vector instructions whose page rows are 2048 or 4096 columns
// long (R = 4 or 2 rows per page: hidden, q_dim and the down-projection K
// piece of 2048 or more) are computed with every page SPLIT across the eight
// compute warps: warp w takes columns [w * KC / 8, (w + 1) * KC / 8) of all R
// rows, lane l the 16-byte chunks w * 32 * CPL + 32 * j + l (j < CPL).  So
//  - a page is finished ~8x sooner after it lands than when one warp owns it
//    (the last page of an instruction no longer costs one warp ~1 us: the
//    instruction's tail, which every dependent instruction waits for, shrinks);
//  - the thread's slice of the input vector is the same for every page: it is
//    loaded once into registers (no shared-memory staging of the vector);
//  - each row's sum is the eight warp partials added in a fixed order, so the
//    result stays independent of the plan.
// Row partials go to a double-buffered shared-memory table; after every T
// pages one compute barrier, then the epilogue of those pages' rows.
template <int R>
struct Split {
  static constexpr int KC = kPageElems / R;  // columns per page row
  static constexpr int CPL = KC / 2048;      // 16-byte chunks per lane and row
  static constexpr int NX = 8 * CPL;         // input elements per thread
  static constexpr int T = 16;               // pages per epilogue batch
  static constexpr int LOG2R = R == 4 ? 2 : 1;
  static_assert(R == 2 || R == 4, "split pages: 2 or 4 rows per page");
};
// Page scheme of a batch-1 matrix instruction: 1 = split pages (every warp a
// column slice of every page) in builds that ask for it (SPL: the Llama-8B
// shape, where it measured 3481 against 3942 us per step); 0 = one warp per
// page otherwise (the Llama-1B shape, where split pages measured 716 and two
// warps per page 745 against 673 us per step: with 4-row pages the per-page
// reduction and synchronisation cost more than the shorter tails save).
template <int NB, int R, bool SPL>
struct Scheme {
  static constexpr int v = NB == 1 && SPL && (R == 2 || R == 4) ? 1 : 0;
};
// the partial table occupies the first kSplitRedFloats floats of the staging
// region (two buffers of T * R * 8 floats = 512 floats each at most); the O
// projection's residual rows follow it
static_assert(2 * Split<4>::T * 4 * 8 <= kSplitRedFloats, "partial table");

template <int R>
__device__ __forceinline__ int split_chunk(int cw, int lane, int j) {
  return cw * 32 * Split<R>::CPL + 32 * j + lane;
}

// Sum N per-lane values over the warp's 32 lanes; lane l ends with the total
// of value l / (32 / N) (halving exchanges, then a butterfly).
template <int N>
__device__ __forceinline__ float warp_sum_rows(float (&v)[N], int lane) {
  constexpr int LOG2N = N >= 32 ? 5 : N >= 16 ? 4 : N >= 8 ? 3 : N >= 4 ? 2 : N >= 2 ? 1 : 0;
  static_assert((1 << LOG2N) == N && N <= 32, "power of two, at most 32 values");
#pragma unroll
  for (int st = 0; st < LOG2N; ++st) {
    const int n = N >> st, off = 16 >> st;
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      if (i < n / 2) {
        const float send = up ? v[i] : v[i + n / 2];
        const float keep = up ? v[i + n / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
    }
  }
  float t = v[0];
#pragma unroll
  for (int off = 16 >> LOG2N; off; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
  return t;
}

// Pages a warp takes at once in the split scheme: every warp works on the
// same pages, so one page at a time would leave each warp's loads, FMAs and
// shuffles a serial chain; a group of four keeps four pages' work in flight.
constexpr int kSplitGroup = 4;

// dot products of this thread's slice with the R rows of the group's pages
// (acc[k * R + r]: page k of the group, row r; zero for pages k >= qn)
template <int R>
__device__ __forceinline__ void split_group_dots(const uint8_t *const (&pages)[kSplitGroup], int qn, int cw, int lane,
                                                 const float (&xa)[Split<R>::NX], float (&acc)[kSplitGroup * R]) {
  using G = Split<R>;
  uint4 w[kSplitGroup][R][G::CPL];
#pragma unroll
  for (int k = 0; k < kSplitGroup; ++k) {
    const uint4 *pg = reinterpret_cast<const uint4 *>(pages[k]);
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int j = 0; j < G::CPL; ++j)
        w[k][r][j] = k < qn ? pg[r * (G::KC / 8) + split_chunk<R>(cw, lane, j)] : make_uint4(0u, 0u, 0u, 0u);
  }
  // packed pair FMAs: even and odd columns accumulate in the two halves of a
  // 64-bit register pair (12 instead of 16 instructions per 8 weights)
  unsigned long long xp[4 * G::CPL];
#pragma unroll
  for (int j = 0; j < 4 * G::CPL; ++j) xp[j] = px::f2pack(xa[2 * j], xa[2 * j + 1]);
#pragma unroll
  for (int k = 0; k < kSplitGroup; ++k)
#pragma unroll
    for (int r = 0; r < R; ++r) {
      unsigned long long s2 = 0ull;
#pragma unroll
      for (int j = 0; j < G::CPL; ++j) {
        const uint4 q = w[k][r][j];
        px::ffma2(s2, px::f2pack(px::bf_lo(q.x), px::bf_hi(q.x)), xp[4 * j + 0]);
        px::ffma2(s2, px::f2pack(px::bf_lo(q.y), px::bf_hi(q.y)), xp[4 * j + 1]);
        px::ffma2(s2, px::f2pack(px::bf_lo(q.z), px::bf_hi(q.z)), xp[4 * j + 2]);
        px::ffma2(s2, px::f2pack(px::bf_lo(q.w), px::bf_hi(q.w)), xp[4 * j + 3]);
      }
      acc[k * R + r] = px::f2sum(s2);
    }
}

// The instruction's pages, split across the warps.  PAIRED: the epilogue
// takes rows (i, i + R/2) of a page together, epi(page, i, v_i, v_{i+R/2})
// (RoPE pairs, gate/up); else epi(page, r, v_r).  Called by every compute
// thread; every thread passes the same barriers even after an abort.
template <int R, bool PAIRED, class Epi>
__device__ __forceinline__ void matvec_split(CCtx &c, const Instr &I, const float (&xa)[Split<R>::NX], Epi epi) {
  using G = Split<R>;
  constexpr int NV = kSplitGroup * R;  // values reduced per group
  constexpr int LPV = 32 / NV;         // lanes holding each reduced value
  static_assert(G::T % kSplitGroup == 0, "epilogue batches hold whole groups");
  const Ring rg = ring_of(c);
  const uint32_t g0 = c.g;
  const int np = (int)I.b, first = (int)I.a, cw = c.cw, lane = c.lane, ctid = c.ctid;
  float *const red = c.act;  // [2][T][R][8 warps]
  bool dead = false;
  int buf = 0;
  // ring slot and phase of the next page, advanced page by page (no division
  // by the ring size per page)
  uint32_t slot = g0 % rg.np, ph = (g0 / rg.np) & 1u;
  for (int t0 = 0; t0 < np; t0 += G::T, buf ^= 1) {
    const int tn = min(G::T, np - t0);
    float *const rb = red + buf * (G::T * R * 8);
    for (int q0 = 0; q0 < tn; q0 += kSplitGroup) {
      const int qn = min(kSplitGroup, tn - q0);
      const uint8_t *pages[kSplitGroup];
      uint32_t slots[kSplitGroup];
#pragma unroll
      for (int k = 0; k < kSplitGroup; ++k) {
        slots[k] = slot;
        pages[k] = rg.pages + (size_t)slot * kPageBytes;
        if (k < qn) {
          if (!dead && !ring_wait_full(c.p, rg, slot, ph)) dead = true;
          if (++slot == rg.np) {
            slot = 0;
            ph ^= 1u;
          }
        }
      }
      if (dead) continue;
      float acc[NV];
      split_group_dots<R>(pages, qn, cw, lane, xa, acc);
      __syncwarp();
      if (lane == 0)
        for (int k = 0; k < qn; ++k) px::mbar_arrive(&rg.empty[slots[k]], 1);
      const float v = warp_sum_rows<NV>(acc, lane);
      const int idx = lane / LPV;  // k * R + r
      if ((lane & (LPV - 1)) == 0 && idx / R < qn) rb[((q0 + idx / R) * R + idx % R) * 8 + cw] = v;
    }
    px::cbar();  // every warp's partials of this batch are in rb
    constexpr int PER = PAIRED ? R / 2 : R;
    if (ctid < tn * PER) {
      const int tt = ctid / PER, i = ctid % PER;
      const float4 *a = reinterpret_cast<const float4 *>(rb + (tt * R + i) * 8);
      const float4 a0 = a[0], a1 = a[1];
      const float va = ((((((a0.x + a0.y) + a0.z) + a0.w) + a1.x) + a1.y) + a1.z) + a1.w;
      if constexpr (PAIRED) {
        const float4 *b = reinterpret_cast<const float4 *>(rb + (tt * R + i + R / 2) * 8);
        const float4 b0 = b[0], b1 = b[1];
        const float vb = ((((((b0.x + b0.y) + b0.z) + b0.w) + b1.x) + b1.y) + b1.z) + b1.w;
        epi(first + t0 + tt, i, va, vb);
      } else {
        epi(first + t0 + tt, i, va);
      }
    }
    // the other buffer is rewritten by the next batch only after the next
    // barrier, which every epilogue thread reaches after its reads
  }
  c.g = g0 + (uint32_t)np;
}

// This thread's slice of x_in(l) (QKV: the residual stream entering layer l;
// gate/up: x_mid from xres[l]; LM head: l == L) times gamma, and 1 / rms(x):
// the dot products are scaled by it afterwards.  One compute barrier.
template <int R>
__device__ __forceinline__ float stage_split_norm(CCtx &c, int l, const uint16_t *gamma, bool from_xres_only,
                                                  float (&xa)[Split<R>::NX]) {
  using G = Split<R>;
  const KParams &p = c.p;
  float4 xs[2 * G::CPL];
  uint4 gw[G::CPL];
  const int tok = (l == 0 && !from_xres_only) ? read_tok(c.sh, 0) : 0;
  settle(c, 2, [&](bool &ok) {
#pragma unroll
    for (int j = 0; j < G::CPL; ++j) {
      const int ch = split_chunk<R>(c.cw, c.lane, j);
      gw[j] = __ldg(reinterpret_cast<const uint4 *>(gamma) + ch);  // with x: one round trip
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int e4 = 2 * ch + h;
        xs[2 * j + h] = from_xres_only ? ll_load4(c.epoch, p.xres + (size_t)l * p.H + e4 * 4, ok)
                                       : layer_input4(p, c.epoch, l, 0, tok, e4, ok);
      }
    }
  });
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < G::CPL; ++j) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float4 x = xs[2 * j + h];
      const uint32_t g01 = h ? gw[j].z : gw[j].x, g23 = h ? gw[j].w : gw[j].y;
      ss += x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
      float *o = xa + 8 * j + 4 * h;
      o[0] = x.x * px::bf_lo(g01);
      o[1] = x.y * px::bf_hi(g01);
      o[2] = x.z * px::bf_lo(g23);
      o[3] = x.w * px::bf_hi(g23);
    }
  }
  ss = px::warp_sum(ss);
  if (c.lane == 0) c.sh->red[c.cw][0] = ss;
  px::cbar();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kComputeWarps; ++w) t += c.sh->red[w][0];
  if (c.tr && c.ctid == 0) c.tr[2] = px::gtimer();
  return __frsqrt_rn(t * p.inv_H + p.eps);  // one rounding; t * (1/H) == t / H for H = 2^k
}

// This thread's slice of a tagged fp32 vector (attention output, SwiGLU
// activations); with nrows > 0 (O projection) also x_in(l) for output rows
// row0 .. row0 + nrows into the staging region after the partial table,
// loaded in the same round trip.
template <int R>
__device__ __forceinline__ void stage_split_copy(CCtx &c, const float *src, float (&xa)[Split<R>::NX], int l = 0,
                                                 int row0 = 0, int nrows = 0) {
  using G = Split<R>;
  const KParams &p = c.p;
  const bool has_row = c.ctid < nrows;
  const int tok0 = l == 0 ? read_tok(c.sh, 0) : 0;
  float xr = 0.f;
  float4 xs[2 * G::CPL];
  settle(c, 3, [&](bool &ok) {
    if (has_row) xr = layer_input1(p, c.epoch, l, 0, tok0, row0 + c.ctid, ok);
#pragma unroll
    for (int j = 0; j < G::CPL; ++j) {
      const int ch = split_chunk<R>(c.cw, c.lane, j);
#pragma unroll
      for (int h = 0; h < 2; ++h) xs[2 * j + h] = ll_load4(c.epoch, src + (2 * ch + h) * 4, ok);
    }
  });
#pragma unroll
  for (int j = 0; j < G::CPL; ++j)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float4 x = xs[2 * j + h];
      float *o = xa + 8 * j + 4 * h;
      o[0] = x.x;
      o[1] = x.y;
      o[2] = x.z;
      o[3] = x.w;
    }
  float *rows = c.act + kSplitRedFloats;
  for (int r = c.ctid; r < nrows; r += kComputeThreads)
    rows[r] = (r == c.ctid) ? xr : layer_input1_settled(p, c.sh, c.epoch, l, 0, tok0, row0 + r);
  if (c.tr && c.ctid == 0) c.tr[2] = px::gtimer();
}

// Normed input of a split-page instruction: 1 / rms(x), with x * gamma as
// this thread's register slice.
template <int R, int MODE>
__device__ __forceinline__ float stage_rows_norm(CCtx &c, int l, const uint16_t *gamma, bool from_xres_only,
                                                 float (&xa)[Split<R>::NX]) {
  static_assert(MODE == 1, "split pages");
  return stage_split_norm<R>(c, l, gamma, from_xres_only, xa);
}
template <int R, int MODE, bool PAIRED, class Epi>
__device__ __forceinline__ void matvec_rows(CCtx &c, const Instr &I, const float (&xa)[Split<R>::NX], Epi epi) {
  static_assert(MODE == 1, "split pages");
  matvec_split<R, PAIRED>(c, I, xa, epi);
}

template <int R, int MODE>
__device__ __forceinline__ uint32_t qkv_rows(CCtx c, const Instr I) {
  const KParams &p = c.p;
  const int l = I.layer;
  float xa[Split<R>::NX];
  const float inv = stage_rows_norm<R, MODE>(c, l, p.layers[l].attn_norm, false, xa);
  const int half = R / 2, pph = p.d / R, hd = p.d / 2, pos = read_pos(c.sh, 0);
  const int nq = p.nq, nkv = p.nkv, d = p.d, kvdim = p.kvdim;
  const uint32_t tag = c.epoch;
  float *const qrow = p.qbuf + (size_t)l * p.qdim;
  float *const kvc = p.kvcur + (size_t)l * 2 * kvdim;
  uint16_t *const kl = p.kc + (size_t)l * p.kv_ls, *const vl = p.vc + (size_t)l * p.kv_ls;
  const long long kv_hs = p.kv_hs;
  const float2 *rope_s = c.sh->rope;
  matvec_rows<R, MODE, true>(c, I, xa, [&](int j, int pr, float u, float w) {
    const int head = j / pph, jj = j % pph;
    const int i = jj * half + pr;  // rotation pair index inside the head
    u *= inv;
    w *= inv;
    if (head < nq + nkv) {
      const float2 cs = rope_s[i];
      const float u2 = u * cs.x - w * cs.y, w2 = u * cs.y + w * cs.x;
      u = u2;
      w = w2;
    }
    if (head < nq) {
      float *q = qrow + head * d;
      px::st_tf(q + i, u, tag);
      px::st_tf(q + i + hd, w, tag);
    } else {
      const bool isk = head < nq + nkv;
      const int gk = isk ? head - nq : head - nq - nkv;
      uint16_t *dst = (isk ? kl : vl) + (size_t)kv_seq(p, 0) * p.kv_bs + (size_t)gk * kv_hs + (size_t)pos * d;
      const uint16_t bu = px::f2bf(u), bw = px::f2bf(w);
      dst[i] = bu;
      dst[i + hd] = bw;
      float *cur = kvc + (isk ? 0 : kvdim) + gk * d;
      px::st_tf(cur + i, px::bf16f(bu), tag);  // bf16 values: exact in 22 significant bits
      px::st_tf(cur + i + hd, px::bf16f(bw), tag);
    }
  });
  return c.g;
}

template <int R, int MODE>
__device__ __forceinline__ uint32_t oproj_rows(CCtx c, const Instr I) {
  const KParams &p = c.p;
  const int l = I.layer;
  const int row0 = (int)I.a * R, nrows = (int)I.b * R;
  float xa[Split<R>::NX];
  // the residual rows x_in(l)[row0 ..] follow the split partial table
  stage_split_copy<R>(c, p.obuf + (size_t)l * p.qdim, xa, l, row0, nrows);
  const uint32_t tag = c.epoch;
  const float *xrows = c.act + kSplitRedFloats - row0;
  float *const xout = p.xres + (size_t)l * p.H;
  matvec_rows<R, MODE, false>(c, I, xa, [&](int j, int r, float v) {
    const int row = j * R + r;
    px::st_tf(xout + row, xrows[row] + v, tag);
  });
  return c.g;
}

template <int R, int MODE>
__device__ __forceinline__ uint32_t gateup_rows(CCtx c, const Instr I) {
  const KParams &p = c.p;
  const int l = I.layer;
  float xa[Split<R>::NX];
  const float inv = stage_rows_norm<R, MODE>(c, l, p.layers[l].ffn_norm, true, xa);
  const int half = R / 2;
  const uint32_t tag = c.epoch;
  float *const aout = p.actb + (size_t)l * p.F;
  matvec_rows<R, MODE, true>(c, I, xa, [&](int j, int pr, float gt, float up) {
    gt *= inv;
    up *= inv;
    const float silu = gt / (1.0f + expf(-gt));
    px::st_tf(aout + j * half + pr, silu * up, tag);
  });
  return c.g;
}

template <int R, int MODE>
__device__ __forceinline__ uint32_t down_rows(CCtx c, const Instr I) {
  const KParams &p = c.p;
  const int l = I.layer, k = I.c;
  float xa[Split<R>::NX];
  stage_split_copy<R>(c, p.actb + (size_t)l * p.F + (size_t)k * p.KCd, xa);
  const uint32_t tag = c.epoch;
  float *const dout = p.dpart + ((size_t)l * p.ndp + k) * p.H;
  matvec_rows<R, MODE, false>(c, I, xa, [&](int j, int r, float v) { px::st_tf(dout + j * R + r, v, tag); });
  return c.g;
}

// forward declaration: the LM head's argmax merge (defined with the paged bodies)
template <int NB, bool TP = false>
__device__ __forceinline__ void lm_argmax_tail(CCtx &c, const Instr &I, float (&bv)[NB], int (&bi)[NB]);
__device__ __forceinline__ bool arg_better(float v, int i, float bv, int bi);

template <int R, int MODE>
__device__ __forceinline__ uint32_t lmhead_rows(CCtx c, const Instr I) {
  const KParams &p = c.p;
  float xa[Split<R>::NX];
  const float inv = stage_rows_norm<R, MODE>(c, p.L, p.final_norm, false, xa);
  float bv[1] = {-INFINITY};
  int bi[1] = {0x7fffffff};
  const int V = p.V;
  float *const logits = p.logits;
  matvec_rows<R, MODE, false>(c, I, xa, [&](int j, int r, float v) {
    const int row = j * R + r;
    if (row >= V) return;  // the rows past the vocabulary of a partial last page
    v *= inv;
    if (logits) logits[row] = v;
    if (arg_better(v, row, bv[0], bi[0])) {
      bv[0] = v;
      bi[0] = row;
    }
  });
  lm_argmax_tail<1>(c, I, bv, bi);
  return c.g;
}

template <int NB, int R, bool SPL = false>
__device__ __forceinline__ uint32_t qkv_body(CCtx c, const Instr I) {
  if constexpr (Scheme<NB, R, SPL>::v != 0) {
    return qkv_rows<R, Scheme<NB, R, SPL>::v>(c, I);
  } else {
    const KParams &p = c.p;
    const int l = I.layer;
    const int half = R / 2, pph = p.d / R, hd = p.d / 2;
    const int pos0 = read_pos(c.sh, 0);
    float inv[NB];
    stage_norm<NB, StageIt<R>::v>(c, l, p.layers[l].attn_norm, false, inv);
    const int nq = p.nq, nkv = p.nkv, d = p.d, lane = c.lane, Bn = p.B, kvdim = p.kvdim;
    const uint32_t tag = c.epoch;
    float *const qrow = p.qbuf + (size_t)l * Bn * p.qdim;
    float *const kvc = p.kvcur + (size_t)l * Bn * 2 * kvdim;
    uint16_t *const kl = p.kc + (size_t)l * p.kv_ls, *const vl = p.vc + (size_t)l * p.kv_ls;
    const long long kv_bs = p.kv_bs, kv_hs = p.kv_hs;
    const int qdim = p.qdim;
    const float2 *rope_s = c.sh->rope;
    const float2 *rope_g = p.rope;
    matvec_pages<NB, R>(c, I, [&](int j, auto &acc) {
      constexpr bool kT = NB > 4;  // transposed sums: every lane takes part in the shuffles
      const int head = j / pph, jj = j % pph;
      if (!kT && lane >= half) return;
      const int i = jj * half + lane;  // rotation pair index inside the head
  #pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (NB > 1 && b >= Bn) break;
        float u = acc_row<R>(acc, b, lane) * inv[b], w = acc_row<R>(acc, b, lane + half) * inv[b];
        if (kT && lane >= half) continue;
        const int pos = NB == 1 ? pos0 : read_pos(c.sh, b);
        if (head < nq + nkv) {
          const float2 cs = NB == 1 ? rope_s[i] : __ldg(rope_g + (size_t)pos * hd + i);
          const float u2 = u * cs.x - w * cs.y, w2 = u * cs.y + w * cs.x;
          u = u2;
          w = w2;
        }
        if (head < nq) {
          float *q = qrow + (size_t)b * qdim + head * d;
          px::st_tf(q + i, u, tag);
          px::st_tf(q + i + hd, w, tag);
        } else {
          // the cache row (bf16) for later steps, and the rounded values for
          // this step's attention as tagged words
          const bool isk = head < nq + nkv;
          const int gk = isk ? head - nq : head - nq - nkv;
          uint16_t *dst = (isk ? kl : vl) + (size_t)kv_seq(p, b) * kv_bs + (size_t)gk * kv_hs + (size_t)pos * d;
          const uint16_t bu = px::f2bf(u), bw = px::f2bf(w);
          if (!chunk_pad(p, b)) {
            dst[i] = bu;
            dst[i + hd] = bw;
          }
          float *cur = kvc + ((size_t)b * 2 + (isk ? 0 : 1)) * kvdim + gk * d;
          px::st_tf(cur + i, px::bf16f(bu), tag);  // bf16 values: exact in 22 significant bits
          px::st_tf(cur + i + hd, px::bf16f(bw), tag);
        }
      }
    });
    return c.g;
  }
}
template <int NB, int R>
__device__ __noinline__ uint32_t op_qkv(CCtx c, const Instr I) { return qkv_body<NB, R>(c, I); }

template <int NB, int R, bool SPL = false>
__device__ __forceinline__ uint32_t oproj_body(CCtx c, const Instr I) {
  if constexpr (Scheme<NB, R, SPL>::v != 0) {
    return oproj_rows<R, Scheme<NB, R, SPL>::v>(c, I);
  } else {
    const KParams &p = c.p;
    const int l = I.layer;
    const int row0 = (int)I.a * R, nrows = NB == 1 ? (int)I.b * R : 0;
    stage_copy<NB, StageIt<R>::v>(c, p.obuf + (size_t)l * p.B * p.qdim, p.qdim, p.qdim, l, row0, nrows);
    const int lane = c.lane, Bn = p.B, H = p.H;
    const uint32_t tag = c.epoch;
    const float *xrows = c.act + p.qdim - row0;
    float *const xout = p.xres + (size_t)l * Bn * H;
    matvec_pages<NB, R>(c, I, [&](int j, auto &acc) {
      constexpr bool kT = NB > 4;
      if (!kT && lane >= R) return;
      const int row = j * R + lane;
      if constexpr (NB == 1) {
        px::st_tf(xout + row, xrows[row] + acc_row<R>(acc, 0, lane), tag);
      } else {
        float av[NB];
  #pragma unroll
        for (int b = 0; b < NB; ++b) av[b] = (b < Bn) ? acc_row<R>(acc, b, lane) : 0.f;
        if (kT && lane >= R) return;
        // the residual row of every sequence: one group of loads (retried as a whole)
        float xin[NB];
        for (LLRetry r;;) {
          bool ok = true;
  #pragma unroll
          for (int b = 0; b < NB; ++b)
            if (b < Bn)
              xin[b] = (p.xin && l > 0) ? tf_chk(px::ld_tf(p.xin + ((size_t)(l - 1) * Bn + b) * H + row), tag, ok)
                                        : layer_input1(p, tag, l, b, l == 0 ? read_tok(c.sh, b) : 0, row, ok);
          if (ok || !ll_retry(p, c.sh, r, 9)) break;
        }
  #pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b >= Bn) break;
          px::st_tf(xout + (size_t)b * H + row, xin[b] + av[b], tag);
        }
      }
    });
    return c.g;
  }
}
template <int NB, int R>
__device__ __noinline__ uint32_t op_oproj(CCtx c, const Instr I) { return oproj_body<NB, R>(c, I); }

template <int NB, int R, bool SPL = false>
__device__ __forceinline__ uint32_t gateup_body(CCtx c, const Instr I) {
  if constexpr (Scheme<NB, R, SPL>::v != 0) {
    return gateup_rows<R, Scheme<NB, R, SPL>::v>(c, I);
  } else {
    const KParams &p = c.p;
    const int l = I.layer;
    float inv[NB];
    stage_norm<NB, StageIt<R>::v>(c, l, p.layers[l].ffn_norm, true, inv);
    const int half = R / 2, lane = c.lane, Bn = p.B, F = p.F;
    const uint32_t tag = c.epoch;
    float *const aout = p.actb + (size_t)l * Bn * F;
    matvec_pages<NB, R>(c, I, [&](int j, auto &acc) {
      constexpr bool kT = NB > 4;
      if (!kT && lane >= half) return;
      const int row = j * half + lane;
  #pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (NB > 1 && b >= Bn) break;
        const float gt = acc_row<R>(acc, b, lane) * inv[b], up = acc_row<R>(acc, b, lane + half) * inv[b];
        if (kT && lane >= half) continue;
        const float silu = gt / (1.0f + expf(-gt));
        px::st_tf(aout + (size_t)b * F + row, silu * up, tag);
      }
    });
    return c.g;
  }
}
template <int NB, int R>
__device__ __noinline__ uint32_t op_gateup(CCtx c, const Instr I) { return gateup_body<NB, R>(c, I); }

template <int NB, int R, bool SPL = false>
__device__ __forceinline__ uint32_t down_body(CCtx c, const Instr I) {
  if constexpr (Scheme<NB, R, SPL>::v != 0) {
    return down_rows<R, Scheme<NB, R, SPL>::v>(c, I);
  } else {
    const KParams &p = c.p;
    const int l = I.layer, k = I.c;
    stage_copy<NB, StageIt<R>::v>(c, p.actb + (size_t)l * p.B * p.F + (size_t)k * p.KCd, p.F, p.KCd);
    const int lane = c.lane, Bn = p.B, H = p.H;
    const uint32_t tag = c.epoch;
    float *const dout = p.dpart + ((size_t)l * p.ndp + k) * Bn * H;
    matvec_pages<NB, R>(c, I, [&](int j, auto &acc) {
      constexpr bool kT = NB > 4;
      if (!kT && lane >= R) return;
      const int row = j * R + lane;
  #pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (NB > 1 && b >= Bn) break;
        const float v = acc_row<R>(acc, b, lane);
        if (kT && lane >= R) continue;
        px::st_tf(dout + (size_t)b * H + row, v, tag);
      }
    });
    return c.g;
  }
}
template <int NB, int R>
__device__ __noinline__ uint32_t op_down(CCtx c, const Instr I) { return down_body<NB, R>(c, I); }

__device__ __forceinline__ bool arg_better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// The LM-head instruction's argmax: per thread (bv, bi) of each sequence ->
// per warp -> per CTA (the instruction's tagged slot); the last LM instruction
// to finish merges every slot and writes the next tokens.
template <int NB, bool TP>
__device__ __forceinline__ void lm_argmax_tail(CCtx &c, const Instr &I, float (&bv)[NB], int (&bi)[NB]) {
  const KParams &p = c.p;
  // CTA-wide argmax of this instruction
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    if (b >= p.B) break;
    float v = bv[b];
    int i = bi[b];
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      float v2 = __shfl_xor_sync(0xffffffffu, v, o);
      int i2 = __shfl_xor_sync(0xffffffffu, i, o);
      if (arg_better(v2, i2, v, i)) {
        v = v2;
        i = i2;
      }
    }
    if (c.lane == 0) {
      c.sh->argv[c.cw][b] = v;
      c.sh->argi[c.cw][b] = i;
    }
  }
  px::cbar();
  if (c.ctid < p.B) {
    const int b = c.ctid;
    float v = -INFINITY;
    int i = 0x7fffffff;
    for (int w = 0; w < kComputeWarps; ++w)
      if (arg_better(c.sh->argv[w][b], c.sh->argi[w][b], v, i)) {
        v = c.sh->argv[w][b];
        i = c.sh->argi[w][b];
      }
    if constexpr (TP) {
      // this rank's slot in every rank's table
      const size_t slot = (size_t)b * p.n_lm + (size_t)p.tp_rank * p.n_lm_local + I.c;
      for (int rr = 0; rr < p.tp_n; ++rr) {
        px::st_ll(p.tp_peers[rr].arg_val + slot, v, c.epoch);
        px::st_ll(p.tp_peers[rr].arg_idx + slot, __int_as_float(i), c.epoch);
      }
    } else {
      px::st_ll(p.arg_val + (size_t)b * p.n_lm + I.c, v, c.epoch);
      px::st_ll(p.arg_idx + (size_t)b * p.n_lm + I.c, __int_as_float(i), c.epoch);
    }
  }
  px::cbar();
  // the last LM instruction to finish merges every slot (all compute threads
  // load a share of the slots at once, then a tree reduction); the slots are
  // tagged words, so the ticket needs no fence
  if (c.ctid == 0) {
    const unsigned old = px::atom_relaxed_add(p.ctr + p.arg_ticket0, 1u);
    // (tensor parallelism: the rank's own LM instructions; the other ranks'
    // slots are tagged, and the merge below waits for them)
    c.sh->flag = (old == c.epoch * (unsigned)(TP ? p.n_lm_local : p.n_lm) - 1u);
  }
  px::cbar();
  if (c.sh->flag) {  // uniform: every compute thread reads the same flag
    for (int b = 0; b < p.B; ++b) {
      float v = -INFINITY;
      int i = 0x7fffffff;
      for (int s0 = c.ctid; s0 < p.n_lm; s0 += kComputeThreads) {
        const llw *av = p.arg_val + (size_t)b * p.n_lm + s0, *ai = p.arg_idx + (size_t)b * p.n_lm + s0;
        float sv;
        int si;
        for (LLRetry r;;) {
          bool ok = true;
          const llw wv = px::ld_ll(av), wi = px::ld_ll(ai);
          sv = ll_chk(wv, c.epoch, ok);
          si = __float_as_int(ll_chk(wi, c.epoch, ok));
          if (ok || !ll_retry(p, c.sh, r, 4)) break;
        }
        if (arg_better(sv, si, v, i)) {
          v = sv;
          i = si;
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
        if (arg_better(v2, i2, v, i)) {
          v = v2;
          i = i2;
        }
      }
      if (c.lane == 0) {
        c.sh->argv[c.cw][b] = v;
        c.sh->argi[c.cw][b] = i;
      }
    }
    px::cbar();
    if (c.ctid < p.B) {
      const int b = c.ctid;
      float v = -INFINITY;
      int i = 0x7fffffff;
      for (int w = 0; w < kComputeWarps; ++w)
        if (arg_better(c.sh->argv[w][b], c.sh->argi[w][b], v, i)) {
          v = c.sh->argv[w][b];
          i = c.sh->argi[w][b];
        }
      p.next_tokens[b] = (i == 0x7fffffff) ? 0 : i;
    }
  }
}

template <int NB, int R, bool SPL = false>
__device__ __forceinline__ uint32_t lmhead_body(CCtx c, const Instr I) {
  if constexpr (Scheme<NB, R, SPL>::v != 0) {
    return lmhead_rows<R, Scheme<NB, R, SPL>::v>(c, I);
  } else {
    const KParams &p = c.p;
    float inv[NB];
    stage_norm<NB, StageIt<R>::v>(c, p.L, p.final_norm, false, inv);
    float bv[NB];
    int bi[NB];
  #pragma unroll
    for (int b = 0; b < NB; ++b) {
      bv[b] = -INFINITY;
      bi[b] = 0x7fffffff;
    }
    const int lane = c.lane, Bn = p.B, V = p.V;
    float *const logits = p.logits;
    matvec_pages<NB, R>(c, I, [&](int j, auto &acc) {
      const int row = j * R + lane;
      const bool valid = lane < R && row < V;
  #pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (NB > 1 && b >= Bn) break;
        const float v = acc_row<R>(acc, b, lane) * inv[b];
        if (valid) {
          if (logits && !chunk_pad(p, b)) logits[(size_t)b * V + row] = v;
          if (arg_better(v, row, bv[b], bi[b])) {
            bv[b] = v;
            bi[b] = row;
          }
        }
      }
    });
    lm_argmax_tail<NB>(c, I, bv, bi);
    return c.g;
  }
}

// Tensor-core matrix product for batched builds: the matrix is in 128-row
// tiles of 64 columns per 16 KiB page (K-major, no swizzle), an instruction
// covers whole tiles, and every tile accumulates D[128 rows][16 sequences]
// (f32, tensor memory) over the tile's pages with two MMAs per 16 columns
// (the staged activations' bf16 hi and lo halves, staged by stage_norm /
// stage_copy_tc).  One thread issues the MMAs and recycles each page once
// its MMAs completed; then the four warps of the tensor-memory lane quarters
// read the tile (row = 32 * quarter + lane, 16 sequences) and run
// epi(tile, quarter, v).  At 16 sequences the product is a dense contraction
// (about 16 flops per weight byte).
__device__ __forceinline__ bool tc_reader(const CCtx &c) { return c.cw >= 2 && c.cw < 6; }
__device__ __forceinline__ int tc_quarter(const CCtx &c) { return (c.cw + kLoaders) & 3; }
// barrier of the four reader warps only
__device__ __forceinline__ void tc_readers_sync() { asm volatile("barrier.cta.sync 3, 128;" ::: "memory"); }

template <int NB, class Epi>
__device__ __forceinline__ bool tc_tiles(CCtx &c, int ntiles, int ppb, int K, Epi &&epi) {
  static_assert(NB == 16, "the MMA's N is the batch slot count");
  const KParams &p = c.p;
  const uint32_t hi_s = px::sa(c.act), lo_s = hi_s + (uint32_t)K * 32u;  // K staged columns
  // D f32, A and B bf16, both K-major, N = 16, M = 128
  constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);
  const uint32_t tmem = c.sh->tmem_base;
  const Ring rg = ring_of(c);
  for (int blk = 0; blk < ntiles; ++blk) {
    if (c.ctid == 0) {
      for (int kb = 0; kb < ppb; ++kb) {
        const uint32_t g = c.g + (uint32_t)(blk * ppb + kb);
        if (!ring_wait(p, rg, g)) break;
        const uint32_t pg = px::sa(ring_page(rg, g));
        px::tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t a = px::umma_desc(pg + ks * 4096u, 2048u, 128u);
          const uint32_t boff = (uint32_t)(kb * 8 + 2 * ks) * 256u;
          px::umma_bf16(tmem, a, px::umma_desc(hi_s + boff, 256u, 128u), kIdesc, kb > 0 || ks > 0);
          px::umma_bf16(tmem, a, px::umma_desc(lo_s + boff, 256u, 128u), kIdesc, true);
        }
        // the page is free once its MMAs have read it
        px::umma_commit(reinterpret_cast<uint64_t *>(&c.sh->mma_bar));
        const uint32_t ph = c.sh->mma_phase & 1u;
        c.sh->mma_phase += 1u;
        if (!wait_bar(p, c.sh, reinterpret_cast<uint64_t *>(&c.sh->mma_bar), ph, 6)) {
          c.sh->abort = 1;
          break;
        }
        ring_release(rg, g, kComputeWarps);
      }
      px::tc_fence_before();
    }
    // every MMA of the tile has completed (thread 0 waited for each page's)
    if (px::cbar_or(px::ld_volatile(&c.sh->abort) != 0)) return false;
    px::tc_fence_after();
    if (tc_reader(c)) {
      const int q = tc_quarter(c);
      float v[16];
      px::tmem_ld16(tmem + ((uint32_t)(q * 32) << 16), v);
      epi(blk, q, v);
    }
    px::tc_fence_before();
    px::cbar();  // the tile is read before the next tile's MMAs overwrite it
  }
  c.g += (uint32_t)(ntiles * ppb);
  return true;
}

template <int NB, int R>
__device__ __forceinline__ uint32_t lmhead_tc_body(CCtx c, const Instr I) {
  const KParams &p = c.p;
  const int V = p.V, Bn = p.B;
  float inv[NB];
  stage_norm<NB, StageIt<R>::v, true>(c, p.L, p.final_norm, false, inv);
  px::fence_proxy_async_smem();  // the staged operand, written by the generic proxy, is read by the MMAs
  px::cbar();
  float bv[NB];
  int bi[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    bv[b] = -INFINITY;
    bi[b] = 0x7fffffff;
  }
  const bool ok = tc_tiles<NB>(c, (int)I.b, p.H / 64, p.H, [&](int blk, int q, const float (&v)[16]) {
    const int row = ((int)I.a + blk) * 128 + q * 32 + c.lane;
    if (row >= V) return;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b >= Bn) break;
      const float x = v[b] * inv[b];
      if (p.logits && !chunk_pad(p, b)) p.logits[(size_t)b * V + row] = x;
      if (arg_better(x, row, bv[b], bi[b])) {
        bv[b] = x;
        bi[b] = row;
      }
    }
  });
  if (!ok) return c.g;
  lm_argmax_tail<NB>(c, I, bv, bi);
  return c.g;
}

// gate/up on the tensor cores: a tile holds 64 gate rows then the same 64 up
// rows, so quarters 0-1 pair their gate rows with the up rows quarters 2-3 read
template <int NB, int R>
__device__ __forceinline__ uint32_t gateup_tc_body(CCtx c, const Instr I) {
  const KParams &p = c.p;
  const int l = I.layer, Bn = p.B, F = p.F;
  float inv[NB];
  stage_norm<NB, StageIt<R>::v, true>(c, l, p.layers[l].ffn_norm, true, inv);
  px::fence_proxy_async_smem();
  px::cbar();
  const uint32_t tag = c.epoch;
  float *const aout = p.actb + (size_t)l * Bn * F;
  float *xch = c.xch;  // [64 rows][16 sequences]
  tc_tiles<NB>(c, (int)I.b, p.H / 64, p.H, [&](int blk, int q, const float (&v)[16]) {
    const int r = (q & 1) * 32 + c.lane;  // row inside the tile's 64 gate / up rows
    if (q >= 2) {
#pragma unroll
      for (int b = 0; b < 16; ++b) xch[r * 16 + b] = v[b];
    }
    tc_readers_sync();
    if (q < 2) {
      const int row = ((int)I.a + blk) * 64 + r;
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b >= Bn) break;
        const float gt = v[b] * inv[b], up = xch[r * 16 + b] * inv[b];
        const float silu = gt / (1.0f + expf(-gt));
        px::st_tf(aout + (size_t)b * F + row, silu * up, tag);
      }
    }
    tc_readers_sync();  // the exchange buffer is reused by the next tile
  });
  return c.g;
}

// down projection on the tensor cores: K piece I.c (KCd columns of act,
// staged as bf16 hi / lo), tiles of 128 output rows
template <int NB>
__device__ __forceinline__ void stage_copy_tc(CCtx &c, const float *src, size_t src_stride, int K) {
  const KParams &p = c.p;
  uint16_t *hi = reinterpret_cast<uint16_t *>(c.act);
  const int n4 = K / 4;
  for (int b0 = 0; b0 < NB; b0 += 4) {
    if (b0 >= p.B) break;
    constexpr int IT = 2;  // K <= 2048: two float4 per thread and sequence
    float4 x[4][IT];
    settle(c, 8, [&](bool &ok) {
#pragma unroll
      for (int it = 0; it < IT; ++it) {
        const int e4 = c.ctid + it * kComputeThreads;
        if (e4 >= n4) break;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (b0 + i < p.B) x[i][it] = ll_load4(c.epoch, src + (size_t)(b0 + i) * src_stride + e4 * 4, ok);
      }
    });
#pragma unroll
    for (int it = 0; it < IT; ++it) {
      const int e4 = c.ctid + it * kComputeThreads;
      if (e4 >= n4) break;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (b0 + i < p.B) {
          const size_t o = ((size_t)(e4 >> 1) * 16 + b0 + i) * 8 + (e4 & 1) * 4;
          split_bf16x4(x[i][it], hi + o, hi + (size_t)K * 16 + o);
        }
    }
  }
  px::fence_proxy_async_smem();
  px::cbar();
  if (c.tr && c.ctid == 0) c.tr[2] = px::gtimer();
}

template <int NB>
__device__ __forceinline__ uint32_t down_tc_body(CCtx c, const Instr I) {
  const KParams &p = c.p;
  const int l = I.layer, k = I.c, Bn = p.B, H = p.H;
  stage_copy_tc<NB>(c, p.actb + (size_t)l * p.B * p.F + (size_t)k * p.KCd, p.F, p.KCd);
  const uint32_t tag = c.epoch;
  float *const dout = p.dpart + ((size_t)l * p.ndp + k) * Bn * H;
  tc_tiles<NB>(c, (int)I.b, p.KCd / 64, p.KCd, [&](int blk, int q, const float (&v)[16]) {
    const int row = ((int)I.a + blk) * 128 + q * 32 + c.lane;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b >= Bn) break;
      px::st_tf(dout + (size_t)b * H + row, v[b], tag);
    }
  });
  if (!p.xin) return c.g;
  // the last of the tile's K pieces to finish (a ticket; the pieces are
  // tagged words, so no fence) sums the tile's rows once: x_in(l + 1) =
  // x_mid + piece 0 + piece 1 + ... (the order every consumer used), so the
  // next layer's consumers load one word per element instead of 1 + ndp
  px::cbar();
  if (c.ctid == 0) {
    const unsigned t = p.dn_ticket0 + (unsigned)l * (unsigned)(H / 128) + I.a;
    const unsigned old = px::atom_relaxed_add(p.ctr + t, 1u);
    c.sh->flag = (old == c.epoch * (unsigned)p.ndp - 1u);
  }
  px::cbar();
  if (c.sh->flag) {
    const int r0 = (int)I.a * 128;
    // 32 float4 per sequence in the tile's rows
    for (int idx = c.ctid; idx < Bn * 32; idx += kComputeThreads) {
      const int b = idx / 32, e = r0 + (idx % 32) * 4;
      const size_t off = (size_t)b * H + e;
      float4 x;
      for (LLRetry rr;;) {
        bool ok = true;
        uint4 w[1 + kMaxDownPieces];
        w[0] = px::ld_tf4(p.xres + (size_t)l * Bn * H + off);
        for (int kk = 0; kk < p.ndp; ++kk) w[1 + kk] = px::ld_tf4(p.dpart + ((size_t)l * p.ndp + kk) * Bn * H + off);
        x = tf_chk4(w[0], tag, ok);
        for (int kk = 0; kk < p.ndp; ++kk) {
          const float4 v = tf_chk4(w[1 + kk], tag, ok);
          x.x += v.x;
          x.y += v.y;
          x.z += v.z;
          x.w += v.w;
        }
        if (ok || !ll_retry(p, c.sh, rr, 10)) break;
      }
      float *dst = p.xin + (size_t)l * Bn * H + off;
      px::st_tf(dst + 0, x.x, tag);
      px::st_tf(dst + 1, x.y, tag);
      px::st_tf(dst + 2, x.z, tag);
      px::st_tf(dst + 3, x.w, tag);
    }
  }
  return c.g;
}

// fused QKV on the tensor cores: a tile is 128 rows of [q; k; v] (two heads
// of 64 or one of 128); RoPE pairs rows i and i + d/2, which sit in lane
// quarters q and q ^ 1 (d = 64) or q ^ 2 (d = 128), so the quarters swap
// their values through shared memory first
template <int NB, int R>
__device__ __forceinline__ uint32_t qkv_tc_body(CCtx c, const Instr I) {
  const KParams &p = c.p;
  const int l = I.layer, Bn = p.B, d = p.d, hd = d / 2, nq = p.nq, nkv = p.nkv, kvdim = p.kvdim;
  float inv[NB];
  stage_norm<NB, StageIt<R>::v, true>(c, l, p.layers[l].attn_norm, false, inv);
  px::fence_proxy_async_smem();
  px::cbar();
  const uint32_t tag = c.epoch;
  float *const qrow = p.qbuf + (size_t)l * Bn * p.qdim;
  float *const kvc = p.kvcur + (size_t)l * Bn * 2 * kvdim;
  uint16_t *const kl = p.kc + (size_t)l * p.kv_ls, *const vl = p.vc + (size_t)l * p.kv_ls;
  float *xch = c.xch;  // [128 rows][16 sequences]
  tc_tiles<NB>(c, (int)I.b, p.H / 64, p.H, [&](int blk, int q, const float (&v)[16]) {
    const int rr = q * 32 + c.lane, row = ((int)I.a + blk) * 128 + rr;
    const int head = row / d, i = row % d;
#pragma unroll
    for (int b = 0; b < 16; ++b) xch[rr * 16 + b] = v[b];
    tc_readers_sync();
    const int partner = i < hd ? rr + hd : rr - hd;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b >= Bn) break;
      const int pos = read_pos(c.sh, b);
      const float mine = v[b] * inv[b], other = xch[partner * 16 + b] * inv[b];
      float out = mine;
      if (head < nq + nkv) {  // q and k heads are rotated
        const float2 cs = __ldg(p.rope + (size_t)pos * hd + (i < hd ? i : i - hd));
        out = i < hd ? mine * cs.x - other * cs.y : other * cs.y + mine * cs.x;
      }
      if (head < nq) {
        px::st_tf(qrow + (size_t)b * p.qdim + row, out, tag);
      } else {
        const bool isk = head < nq + nkv;
        const int gk = isk ? head - nq : head - nq - nkv;
        const uint16_t bo = px::f2bf(out);
        uint16_t *dst = (isk ? kl : vl) + (size_t)kv_seq(p, b) * p.kv_bs + (size_t)gk * p.kv_hs + (size_t)pos * d;
        if (!chunk_pad(p, b)) dst[i] = bo;
        px::st_tf(kvc + ((size_t)b * 2 + (isk ? 0 : 1)) * kvdim + (size_t)gk * d + i, px::bf16f(bo), tag);
      }
    }
    tc_readers_sync();  // the exchange buffer is reused by the next tile
  });
  return c.g;
}

// output projection + residual on the tensor cores (attention output staged
// as bf16 hi / lo; the residual rows of every sequence in one load group)
template <int NB>
__device__ __forceinline__ uint32_t oproj_tc_body(CCtx c, const Instr I) {
  const KParams &p = c.p;
  const int l = I.layer, Bn = p.B, H = p.H;
  stage_copy_tc<NB>(c, p.obuf + (size_t)l * p.B * p.qdim, p.qdim, p.qdim);
  const uint32_t tag = c.epoch;
  float *const xout = p.xres + (size_t)l * Bn * H;
  tc_tiles<NB>(c, (int)I.b, p.qdim / 64, p.qdim, [&](int blk, int q, const float (&v)[16]) {
    const int row = ((int)I.a + blk) * 128 + q * 32 + c.lane;
    float xin[NB];
    for (LLRetry r;;) {
      bool ok = true;
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if (b < Bn)
          xin[b] = (p.xin && l > 0) ? tf_chk(px::ld_tf(p.xin + ((size_t)(l - 1) * Bn + b) * H + row), tag, ok)
                                    : layer_input1(p, tag, l, b, l == 0 ? read_tok(c.sh, b) : 0, row, ok);
      if (ok || !ll_retry(p, c.sh, r, 9)) break;
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b >= Bn) break;
      px::st_tf(xout + (size_t)b * H + row, xin[b] + v[b], tag);
    }
  });
  return c.g;
}

template <int NB, int R>
__device__ __noinline__ uint32_t op_qkv_tc(CCtx c, const Instr I) { return qkv_tc_body<NB, R>(c, I); }
template <int NB>
__device__ __noinline__ uint32_t op_oproj_tc(CCtx c, const Instr I) { return oproj_tc_body<NB>(c, I); }
template <int NB, int R>
__device__ __noinline__ uint32_t op_gateup_tc(CCtx c, const Instr I) { return gateup_tc_body<NB, R>(c, I); }
template <int NB>
__device__ __noinline__ uint32_t op_down_tc(CCtx c, const Instr I) { return down_tc_body<NB>(c, I); }
template <int NB, int R>
__device__ __noinline__ uint32_t op_lmhead_tc(CCtx c, const Instr I) { return lmhead_tc_body<NB, R>(c, I); }
template <int NB, int R>
__device__ __noinline__ uint32_t op_lmhead(CCtx c, const Instr I) { return lmhead_body<NB, R>(c, I); }

// ---------------------------------------------------------------- tensor parallelism
// One rank of a tensor-parallel group (batch 1, one page per warp; the
// "Mirage Persistent Kernel" article, part 1: a collective split into chunks,
// each depending only on the tile that produces it).  The rank holds the
// heads, FFN columns and vocabulary rows of its shard: the O projection (row
// split: its heads' columns of Wo) and the down projection (its FFN columns)
// produce partial sums of every output row, which each producing page stores
// into every rank's copy of the partial buffers (peer stores; tagged words,
// so a consumer needs no flag beyond the counters it already polls); the
// consumers sum the ranks' partials in rank order -- an all-reduce whose
// chunks are single pages.

// x_mid(l) * gamma staged (x_mid = x_in(l) + the ranks' O partials), 1/rms
// returned; this instruction also stores rows [row_lo, row_hi) of x_mid as the
// rank's residual copy xres[l] (the next layer's input starts from it).
template <int IT>
__device__ float stage_norm_tp_mid(CCtx &c, int l, const uint16_t *gamma, int row_lo, int row_hi) {
  const KParams &p = c.p;
  const int H = p.H, n4 = H / 4;
  const uint32_t tag = c.epoch;
  float4 xs[IT];
  uint2 gws[IT];
  const int tok = l == 0 ? read_tok(c.sh, 0) : 0;
  settle(c, 2, [&](bool &ok) {
#pragma unroll
    for (int it = 0; it < IT; ++it) {
      const int e4 = c.ctid + it * kComputeThreads;
      if (e4 < n4) {
        gws[it] = __ldg(reinterpret_cast<const uint2 *>(gamma) + e4);
        float4 x = layer_input4(p, tag, l, 0, tok, e4, ok);
        for (int r = 0; r < p.tp_n; ++r) {
          const float4 v = tf_chk4(px::ld_tf4(p.opart + ((size_t)l * p.tp_n + r) * p.B * H + e4 * 4), tag, ok);
          x.x += v.x;
          x.y += v.y;
          x.z += v.z;
          x.w += v.w;
        }
        xs[it] = x;
      }
    }
  });
  float ss = 0.f;
  float4 *dst = reinterpret_cast<float4 *>(c.act);
  float *const xres = p.xres + (size_t)l * p.B * H;
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int e4 = c.ctid + it * kComputeThreads;
    if (e4 < n4) {
      const float4 x = xs[it];
      const uint2 gw = gws[it];
      ss += x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
      dst[stage_slot4(e4, H)] =
          make_float4(x.x * px::bf_lo(gw.x), x.y * px::bf_hi(gw.x), x.z * px::bf_lo(gw.y), x.w * px::bf_hi(gw.y));
      if (e4 * 4 >= row_lo && e4 * 4 < row_hi) {
        px::st_tf(xres + e4 * 4 + 0, x.x, tag);
        px::st_tf(xres + e4 * 4 + 1, x.y, tag);
        px::st_tf(xres + e4 * 4 + 2, x.z, tag);
        px::st_tf(xres + e4 * 4 + 3, x.w, tag);
      }
    }
  }
  ss = px::warp_sum(ss);
  if (c.lane == 0) c.sh->red[c.cw][0] = ss;
  px::cbar();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kComputeWarps; ++w) t += c.sh->red[w][0];
  if (c.tr && c.ctid == 0) c.tr[2] = px::gtimer();
  return __frsqrt_rn(t * p.inv_H + p.eps);
}

// O projection, row split: this rank's heads' columns; the partial of every
// output row goes to slot tp_rank of every rank's opart[l]
template <int R>
__device__ __noinline__ uint32_t op_oproj_tp(CCtx c, const Instr I) {
  const KParams &p = c.p;
  const int l = I.layer, lane = c.lane;
  stage_copy<1, StageIt<R>::v>(c, p.obuf + (size_t)l * p.B * p.qdim, p.qdim, p.qdim);
  const uint32_t tag = c.epoch;
  const size_t off = ((size_t)l * p.tp_n + p.tp_rank) * p.B * p.H;
  matvec_pages<1, R>(c, I, [&](int j, float (&acc)[1][R]) {
    if (lane >= R) return;
    const int row = j * R + lane;
    const float v = pick<R>(acc[0], lane);
    for (int rr = 0; rr < p.tp_n; ++rr) px::st_tf(p.tp_peers[rr].opart + off + row, v, tag);
  });
  return c.g;
}

// gate/up + SiLU * up for this rank's FFN columns; the instruction's slice of
// x_mid becomes the rank's residual copy
template <int R>
__device__ __noinline__ uint32_t op_gateup_tp(CCtx c, const Instr I) {
  const KParams &p = c.p;
  const int l = I.layer, half = R / 2, lane = c.lane, F = p.F;
  const int n4 = p.H / 4, per = (n4 + p.n_gu_layer - 1) / p.n_gu_layer;
  const int row_lo = min(n4, (int)I.c * per) * 4, row_hi = min(n4, ((int)I.c + 1) * per) * 4;
  const float inv = stage_norm_tp_mid<StageIt<R>::v>(c, l, p.layers[l].ffn_norm, row_lo, row_hi);
  const uint32_t tag = c.epoch;
  float *const aout = p.actb + (size_t)l * p.B * F;
  matvec_pages<1, R>(c, I, [&](int j, float (&acc)[1][R]) {
    if (lane >= half) return;
    const int row = j * half + lane;
    const float gt = pick<R>(acc[0], lane) * inv, up = pick<R>(acc[0], lane + half) * inv;
    const float silu = gt / (1.0f + expf(-gt));
    px::st_tf(aout + row, silu * up, tag);
  });
  return c.g;
}

// down projection of this rank's FFN columns, K piece I.c: the partial goes
// to piece tp_rank * ndp_local + I.c of every rank's dpart[l]
template <int R>
__device__ __noinline__ uint32_t op_down_tp(CCtx c, const Instr I) {
  const KParams &p = c.p;
  const int l = I.layer, k = I.c, lane = c.lane, H = p.H;
  stage_copy<1, StageIt<R>::v>(c, p.actb + (size_t)l * p.B * p.F + (size_t)k * p.KCd, p.F, p.KCd);
  const uint32_t tag = c.epoch;
  const size_t off = ((size_t)l * p.ndp + (size_t)p.tp_rank * p.ndp_local + k) * p.B * H;
  matvec_pages<1, R>(c, I, [&](int j, float (&acc)[1][R]) {
    if (lane >= R) return;
    const int row = j * R + lane;
    const float v = pick<R>(acc[0], lane);
    for (int rr = 0; rr < p.tp_n; ++rr) px::st_tf(p.tp_peers[rr].dpart + off + row, v, tag);
  });
  return c.g;
}

// LM head of this rank's vocabulary rows: their logits, and the rank's
// argmax candidates in every rank's slots; the rank's last LM instruction
// merges all ranks' slots
template <int R>
__device__ __noinline__ uint32_t op_lmhead_tp(CCtx c, const Instr I) {
  const KParams &p = c.p;
  float inv[1];
  stage_norm<1, StageIt<R>::v>(c, p.L, p.final_norm, false, inv);
  float bv[1] = {-INFINITY};
  int bi[1] = {0x7fffffff};
  const int lane = c.lane;
  float *const logits = p.logits;
  matvec_pages<1, R>(c, I, [&](int j, float (&acc)[1][R]) {
    const int row = j * R + lane;
    if (lane < R && row < p.V_lm) {
      const float v = pick<R>(acc[0], lane) * inv[0];
      const int gi = p.lm_row0 + row;
      if (logits) logits[gi] = v;
      if (arg_better(v, gi, bv[0], bi[0])) {
        bv[0] = v;
        bi[0] = gi;
      }
    }
  });
  lm_argmax_tail<1, true>(c, I, bv, bi);
  return c.g;
}

// ---------------------------------------------------------------- attention
// One (sequence b, kv head g, split s) item: online softmax over the split's
// cached positions (streamed through the ring, all compute warps per page,
// a block of positions per warp), plus the current position (read from the
// cache row this step's QKV instruction wrote).  Unnormalised partials
// (o, max, sum) go to global memory; the last split to finish merges all
// splits of the head group with log-sum-exp weights.
template <int G, int DPL, int PB>
__device__ __forceinline__ void load_row(const uint16_t *rowp, int lane, float (&f)[DPL]) {
  if constexpr (DPL == 2) {
    const uint32_t w = *reinterpret_cast<const uint32_t *>(rowp + lane * 2);
    f[0] = px::bf_lo(w);
    f[1] = px::bf_hi(w);
  } else {
    const uint2 w = *reinterpret_cast<const uint2 *>(rowp + lane * 4);
    f[0] = px::bf_lo(w.x);
    f[1] = px::bf_hi(w.x);
    f[2] = px::bf_lo(w.y);
    f[3] = px::bf_hi(w.y);
  }
}

// PB consecutive positions (rows of kb / vb, row stride D) for one warp, of
// which the first `nvalid` are real.  G*PB <= 32 scores are reduced with a
// transposed butterfly so that one lane ends with one score; the softmax
// update is then one exp per lane.
template <int G, int DPL, int PB>
__device__ void attn_block(const float (&q)[G][DPL], const uint16_t *kb, const uint16_t *vb, int nvalid,
                           int lane, float (&m)[G], float (&l)[G], float (&o)[G][DPL]) {
  constexpr int D = DPL * 32;
  constexpr int NV = G * PB;
  static_assert(NV <= 32 && (NV & (NV - 1)) == 0, "block size");
  float v[NV];
#pragma unroll
  for (int j = 0; j < PB; ++j) {
    float kf[DPL];
    if (j < nvalid) {
      load_row<G, DPL, PB>(kb + j * D, lane, kf);
    } else {
#pragma unroll
      for (int i = 0; i < DPL; ++i) kf[i] = 0.f;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < DPL; ++i) s = fmaf(q[h][i], kf[i], s);
      v[h * PB + j] = s;
    }
  }
  // transposed reduction: afterwards the lane holds the full score of value
  // index (lane >> SH), index = h * PB + j
  int n = NV;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      const int hn = n / 2;
      const bool up = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < (NV > 1 ? NV / 2 : 1); ++i) {
        if (i < hn) {
          const float send = up ? v[i] : v[i + hn];
          const float keep = up ? v[i + hn] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      n = hn;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
  constexpr int LOGNV = (NV >= 32) ? 5 : (NV >= 16) ? 4 : (NV >= 8) ? 3 : (NV >= 4) ? 2 : (NV >= 2) ? 1 : 0;
  constexpr int SH = 5 - LOGNV;
  constexpr int GRP = 32 / G;  // lanes per head after the reduction
  const int idx = lane >> SH;
  const int myh = idx / PB, myj = idx % PB;
  const float s = (myj < nvalid) ? v[0] : -INFINITY;
  float bm = s;
#pragma unroll
  for (int off = GRP / 2; off >= 1; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
  float mh_old = -INFINITY;
#pragma unroll
  for (int h = 0; h < G; ++h)
    if (h == myh) mh_old = m[h];
  const float mnew = fmaxf(mh_old, bm);
  const float pr = (s == -INFINITY) ? 0.f : expf(s - mnew);
  // 2^SH lanes hold each score: count one of them in the sum
  float ps = (lane & ((1 << SH) - 1)) == 0 ? pr : 0.f;
#pragma unroll
  for (int off = GRP / 2; off >= 1; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float mn = __shfl_sync(0xffffffffu, mnew, h * GRP);
    const float bs = __shfl_sync(0xffffffffu, ps, h * GRP);
    const float corr = (m[h] == -INFINITY) ? 0.f : expf(m[h] - mn);
    l[h] = l[h] * corr + bs;
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[h][i] *= corr;
    m[h] = mn;
  }
#pragma unroll
  for (int j = 0; j < PB; ++j) {
    if (j >= nvalid) break;
    float vf[DPL];
    load_row<G, DPL, PB>(vb + j * D, lane, vf);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float ph = __shfl_sync(0xffffffffu, pr, (h * PB + j) << SH);
#pragma unroll
      for (int i = 0; i < DPL; ++i) o[h][i] = fmaf(ph, vf[i], o[h][i]);
    }
  }
}

template <int G, int DPL, bool CHUNK>
__device__ __forceinline__ uint32_t attn_body(CCtx c, const Instr I) {
  const KParams &p = c.p;
  constexpr int D = DPL * 32;
  constexpr int PPP = kPageBytes / (4 * D);
  constexpr int PW = PPP / kComputeWarps;        // positions per warp per page
  constexpr int PB = PW < 32 / G ? PW : 32 / G;  // positions per reduction block
  const int l = I.layer, g = I.a, s = I.b, b = I.c;
  const SplitRange r = split_range(p, c.sh, b, s);
  const int npg = r.pref_end > r.start ? (r.pref_end - r.start + PPP - 1) / PPP : 0;
  // q of the G heads of this group (pre-scaled by 1/sqrt(d)) and, for the
  // split holding the current position, that position's K and V rows (this
  // step's QKV wrote them as tagged words): one group of loads
  const uint32_t tag = c.epoch;
  // the current position's row goes to the first warp with less than a full
  // share of the last cached page (often none), not to an already loaded warp
  const int last_cnt = npg > 0 ? (r.pref_end - r.start) - (npg - 1) * PPP : 0;
  const int cur_warp = min(kComputeWarps - 1, last_cnt / PW);
  // a prompt chunk of several tokens (batched builds): the last split takes
  // the chunk's rows 0 .. cb instead of one current row -- row j is token j's
  // K/V row of this step's exchange; warp w takes rows w and w + 8
  const bool chunk_rows = CHUNK && p.chunk_n > 1 && r.has_cur;
  const int cb = chunk_rows ? r.pos - p.chunk_pos0 : -1;
  const int nmine = chunk_rows ? (c.cw <= cb) + (c.cw + kComputeWarps <= cb) : 0;
  const bool load_cur = !chunk_rows && r.has_cur && c.cw == cur_warp;
  const float *kcur = p.kvcur + (((size_t)l * p.B + b) * 2) * p.kvdim + (size_t)g * D;
  const float *vcur = kcur + p.kvdim;
  const float *qb = p.qbuf + ((size_t)l * p.B + b) * p.qdim + (size_t)g * G * D;
  // scratch in the staging region: [warp][G][D + 2] floats, then the
  // current position's K and V rows (bf16)
  float *scr = c.act;
  uint16_t *cur = reinterpret_cast<uint16_t *>(c.act + kComputeWarps * G * (D + 2));
  // after the merge weights (below): this warp's chunk rows, K [2][D] then V [2][D]
  uint16_t *mine = reinterpret_cast<uint16_t *>(c.act + kComputeWarps * G * (D + 2) + D +
                                                ((G * (kComputeWarps + 2) + 3) & ~3)) +
                   (size_t)c.cw * 4 * D;
  float q[G][DPL], ck[DPL], cv[DPL];
  settle(c, 5, [&](bool &ok) {
    uint32_t wk[DPL], wv[DPL], wq[G][DPL];
    if constexpr (CHUNK) {
      if (nmine > 0) {
        uint32_t rk[2][DPL], rv[2][DPL];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (j >= nmine) break;
          const float *kr = p.kvcur + (((size_t)l * p.B + c.cw + j * kComputeWarps) * 2) * p.kvdim + (size_t)g * D;
#pragma unroll
          for (int i = 0; i < DPL; ++i) {
            rk[j][i] = px::ld_tf(kr + c.lane * DPL + i);
            rv[j][i] = px::ld_tf(kr + p.kvdim + c.lane * DPL + i);
          }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (j >= nmine) break;
#pragma unroll
          for (int i = 0; i < DPL; ++i) {
            mine[j * D + c.lane * DPL + i] = px::f2bf(tf_chk(rk[j][i], tag, ok));
            mine[2 * D + j * D + c.lane * DPL + i] = px::f2bf(tf_chk(rv[j][i], tag, ok));
          }
        }
      }
    }
    if (load_cur) {
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        wk[i] = px::ld_tf(kcur + c.lane * DPL + i);
        wv[i] = px::ld_tf(vcur + c.lane * DPL + i);
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < DPL; ++i) wq[h][i] = px::ld_tf(qb + h * D + c.lane * DPL + i);
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < DPL; ++i) q[h][i] = tf_chk(wq[h][i], tag, ok) * p.attn_scale;
    if (load_cur) {
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        ck[i] = tf_chk(wk[i], tag, ok);
        cv[i] = tf_chk(wv[i], tag, ok);
      }
    }
  });
  if (c.tr && c.ctid == 0) c.tr[2] = px::gtimer();
  float m[G], lsum[G], o[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    lsum[h] = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[h][i] = 0.f;
  }
  if (load_cur) {
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      cur[c.lane * DPL + i] = px::f2bf(ck[i]);
      cur[D + c.lane * DPL + i] = px::f2bf(cv[i]);
    }
  }
  const Ring rg = ring_of(c);
  const int cw = c.cw, lane = c.lane;
  for (int t = 0; t < npg; ++t) {
    const uint32_t gg = c.g + t;
    if (!ring_wait(p, rg, gg)) break;
    const uint8_t *pg = ring_page(rg, gg);
    const int p0 = r.start + t * PPP;
    const int cnt = min(PPP, r.pref_end - p0);
#pragma unroll
    for (int sb = 0; sb < PW / PB; ++sb) {
      const int jb = cw * PW + sb * PB;
      const int nvalid = max(0, min(PB, cnt - jb));
      if (nvalid > 0)
        attn_block<G, DPL, PB>(q, reinterpret_cast<const uint16_t *>(pg) + (size_t)jb * D,
                               reinterpret_cast<const uint16_t *>(pg + kPageBytes / 2) + (size_t)jb * D, nvalid,
                               lane, m, lsum, o);
    }
    __syncwarp();
    if (lane == 0) ring_release(rg, gg, 1);
  }
  c.g += npg;
  __syncwarp();
  if (load_cur && !c.sh->abort) {
    // one valid position; the block reads PW rows, rows past the first are masked
    attn_block<G, DPL, PB>(q, cur, cur + D, 1, c.lane, m, lsum, o);
  }
  if constexpr (CHUNK) {
    if (nmine > 0 && !c.sh->abort) attn_block<G, DPL, PB>(q, mine, mine + 2 * D, nmine, c.lane, m, lsum, o);
  }
  if (c.tr && c.ctid == 0) c.tr[10] = px::gtimer();
  // merge the warps
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float *w = scr + ((size_t)c.cw * G + h) * (D + 2);
#pragma unroll
    for (int i = 0; i < DPL; ++i) w[c.lane * DPL + i] = o[h][i];
    if (c.lane == 0) {
      w[D] = m[h];
      w[D + 1] = lsum[h];
    }
  }
  px::cbar();
  // per head: the warps' weights exp(m_w - M) once (one thread per (head,
  // warp), 8-lane groups of warp 0), then every output element sums the
  // warps' contributions with them
  float *fac = reinterpret_cast<float *>(cur + 2 * D);  // [G][warps] weights, then [G] M and [G] L
  if (c.ctid < G * kComputeWarps) {
    constexpr unsigned fm = (G * kComputeWarps >= 32) ? 0xffffffffu : ((1u << (G * kComputeWarps)) - 1u);
    const int h = c.ctid / kComputeWarps, w = c.ctid % kComputeWarps;
    const float *ws = scr + ((size_t)w * G + h) * (D + 2);
    const float mw = ws[D];
    float M = mw;
#pragma unroll
    for (int off = kComputeWarps / 2; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(fm, M, off));
    const float f = (mw == -INFINITY) ? 0.f : expf(mw - M);
    float L = f * ws[D + 1];
#pragma unroll
    for (int off = kComputeWarps / 2; off; off >>= 1) L += __shfl_xor_sync(fm, L, off);
    fac[h * kComputeWarps + w] = f;
    if (w == 0) {
      fac[G * kComputeWarps + h] = M;
      fac[G * kComputeWarps + G + h] = L;
    }
  }
  px::cbar();
  const size_t hbase = ((size_t)l * p.B + b) * p.nq + (size_t)g * G;  // [l][b][head]
  for (int e = c.ctid; e < G * D; e += kComputeThreads) {
    const int h = e / D, dd = e % D;
    float O = 0.f;
#pragma unroll
    for (int w = 0; w < kComputeWarps; ++w) O += fac[h * kComputeWarps + w] * scr[((size_t)w * G + h) * (D + 2) + dd];
    px::st_tf(p.part_o + ((hbase + h) * p.S + s) * D + dd, O, tag);
    if (dd == 0) {
      llw *ml = p.part_ml + ((hbase + h) * p.S + s) * 2;
      px::st_ll(ml + 0, fac[G * kComputeWarps + h], tag);
      px::st_ll(ml + 1, fac[G * kComputeWarps + G + h], tag);
    }
  }
  px::cbar();
  if (c.ctid == 0) {  // tagged partials: the ticket needs no fence
    const unsigned t = p.attn_ticket0 + ((unsigned)l * p.B + b) * p.nkv + g;
    const unsigned old = px::atom_relaxed_add(p.ctr + t, 1u);
    c.sh->flag = (old == c.epoch * (unsigned)p.S - 1u);
  }
  px::cbar();
  if (c.sh->flag) {  // uniform: the last split of the group merges all S splits
    constexpr int NE = G * D;                            // outputs of the group
    constexpr int EPT = (NE + kComputeThreads - 1) / kComputeThreads;
    constexpr int SB = (64 / EPT) < 32 ? (64 / EPT) : 32;  // splits per load batch
    const int S = p.S;
    float *sml = scr;  // [G][S] (m, l) then (weight, -)
    for (int i = c.ctid; i < G * S; i += kComputeThreads) {
      const int h = i / S, sp = i % S;
      const llw *a = p.part_ml + ((hbase + h) * S + sp) * 2;
      for (LLRetry rr;;) {
        bool ok = true;
        llw w0, w1;
        px::ld_ll2(a, w0, w1);
        sml[2 * i] = ll_chk(w0, tag, ok);
        sml[2 * i + 1] = ll_chk(w1, tag, ok);
        if (ok || !ll_retry(p, c.sh, rr, 6)) break;
      }
    }
    // the first batch of this thread's partial outputs, in flight with the table
    uint32_t ov[EPT][SB];
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const int idx = c.ctid + e * kComputeThreads;
      const int h = idx / D, dd = idx % D;
#pragma unroll
      for (int j = 0; j < SB; ++j) ov[e][j] = (idx < NE && j < S) ? px::ld_tf(p.part_o + ((hbase + h) * S + j) * D + dd) : 0u;
    }
    px::cbar();
    if (c.cw < G) {  // warp h: head h's max, weights exp(m_s - M) and total weight L, lanes over splits
      const int h = c.cw;
      float M = -INFINITY;
      for (int sp = c.lane; sp < S; sp += 32) M = fmaxf(M, sml[2 * (h * S + sp)]);
      M = px::warp_max(M);
      float L = 0.f;
      for (int sp = c.lane; sp < S; sp += 32) {
        const float ms = sml[2 * (h * S + sp)];
        const float wgt = (ms == -INFINITY) ? 0.f : expf(ms - M);
        L += wgt * sml[2 * (h * S + sp) + 1];
        sml[2 * (h * S + sp)] = wgt;
      }
      L = px::warp_sum(L);
      if (c.lane == 0) c.sh->red[h % kComputeWarps][h / kComputeWarps] = L;
    }
    px::cbar();
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const int idx = c.ctid + e * kComputeThreads;
      if (idx >= NE) break;
      const int h = idx / D, dd = idx % D;
      float O = 0.f;
      bool ok = true;
#pragma unroll
      for (int j = 0; j < SB; ++j)
        if (j < S) O += sml[2 * (h * S + j)] * tf_chk(ov[e][j], tag, ok);
      for (int s0 = ok ? SB : 0; s0 < S; s0 += SB) {  // further batches (S > SB), or all again
        float Ob = 0.f;
        for (LLRetry rr;;) {
          bool okb = true;
          uint32_t tmp[SB];
#pragma unroll
          for (int j = 0; j < SB; ++j)
            tmp[j] = (s0 + j < S) ? px::ld_tf(p.part_o + ((hbase + h) * S + s0 + j) * D + dd) : 0u;
          Ob = 0.f;
#pragma unroll
          for (int j = 0; j < SB; ++j)
            if (s0 + j < S) Ob += sml[2 * (h * S + s0 + j)] * tf_chk(tmp[j], tag, okb);
          if (okb || !ll_retry(p, c.sh, rr, 7)) break;
        }
        O = (s0 == 0) ? Ob : O + Ob;
      }
      const float L = c.sh->red[h % kComputeWarps][h / kComputeWarps];
      px::st_tf(p.obuf + ((size_t)l * p.B + b) * p.qdim + (size_t)(g * G + h) * D + dd, O / L, tag);
    }
  }
  return c.g;
}
template <int G, int DPL, bool CHUNK>
__device__ __noinline__ uint32_t op_attn_t(CCtx c, const Instr I) { return attn_body<G, DPL, CHUNK>(c, I); }

template <bool CHUNK>
__device__ __forceinline__ uint32_t op_attn(const CCtx &c, const Instr &I) {
  const int G = c.p.nq / c.p.nkv;
  if (c.p.d == 64) {
    switch (G) {
      case 1: return op_attn_t<1, 2, CHUNK>(c, I);
      case 2: return op_attn_t<2, 2, CHUNK>(c, I);
      case 4: return op_attn_t<4, 2, CHUNK>(c, I);
      default: return op_attn_t<8, 2, CHUNK>(c, I);
    }
  }
  switch (G) {
    case 1: return op_attn_t<1, 4, CHUNK>(c, I);
    case 2: return op_attn_t<2, 4, CHUNK>(c, I);
    case 4: return op_attn_t<4, 4, CHUNK>(c, I);
    default: return op_attn_t<8, 4, CHUNK>(c, I);
  }
}

// dispatch on the rows-per-page of the instruction's matrix
#define MK_DISPATCH_R(fn, NB, R, c, I)            \
  switch (R) {                                    \
    case 2: c.g = fn<NB, 2>(c, I); break;         \
    case 4: c.g = fn<NB, 4>(c, I); break;         \
    case 8: c.g = fn<NB, 8>(c, I); break;         \
    case 16: c.g = fn<NB, 16>(c, I); break;       \
    default: c.g = fn<NB, 32>(c, I); break;       \
  }
#define MK_DISPATCH_R1(fn, R, c, I)               \
  switch (R) {                                    \
    case 2: c.g = fn<2>(c, I); break;             \
    case 4: c.g = fn<4>(c, I); break;             \
    case 8: c.g = fn<8>(c, I); break;             \
    case 16: c.g = fn<16>(c, I); break;           \
    default: c.g = fn<32>(c, I); break;           \
  }

__device__ __forceinline__ int &sh_stat(CCtx &c) { return c.sh->stat_cwait; }

// Shape specialisation of the interpreter: rows per page of the QKV / gate-up /
// LM-head pages (RH), of the output-projection pages (RO) and of the
// down-projection pages (RD), the query heads per KV head (G) and head_dim / 32
// (DPL).  With every value fixed, each op body is inlined into the interpreter
// loop (no call, no spills across a call boundary); the shape-generic build
// (all zero) reaches the bodies through calls selected at run time.  TQO
// (batched builds): QKV and the O projection may run as tensor-core tiles; a
// build of its own, since the extra op bodies raise every body's spills.
template <int RH_, int RO_, int RD_, int G_, int DPL_, bool TQO_ = false, bool SPL_ = false, bool TP_ = false>
struct Spec {
  static constexpr bool fixed = RH_ > 0;
  static constexpr bool TQO = TQO_;
  static constexpr bool SPL = SPL_;  // batch 1: split pages for rows of 2048 / 4096 columns
  static constexpr bool TP = TP_;    // the tensor-parallel rank build (shape-generic, batch 1)
  static constexpr int RH = RH_, RO = RO_, RD = RD_, G = G_, DPL = DPL_;
};
using SpecGeneric = Spec<0, 0, 0, 0, 0>;
using SpecGenericTP = Spec<0, 0, 0, 0, 0, false, false, true>;

// Ops that start before their producers are known to be done (bit op): all
// of them (measured: 682 us/step, against 697 with attention and the output
// projection waiting for their counters first).
#ifndef MK_SPECULATIVE_OPS
#define MK_SPECULATIVE_OPS 0xFEu
#endif
constexpr unsigned kSpeculativeOps = MK_SPECULATIVE_OPS;

// Event-driven queue: signal counter c; the signal that completes the
// step's count appends the instructions waiting on it to the ready queue
// (slot = step << 32 | instruction index).  Thread 0 of the producer.
__device__ __noinline__ void event_signal(const KParams &p, unsigned c, unsigned epoch) {
  const unsigned old = px::atom_relaxed_add(p.ctr + c, 1u);
  const unsigned cnt = p.ev_cnt[c];
  if (cnt == 0 || old + 1u != epoch * cnt) return;
  const int j0 = p.ev_off[c], n = p.ev_off[c + 1] - j0;
  const unsigned per_step = (unsigned)(p.n_ev - p.n_ev_init);
  const unsigned pos = px::atom_relaxed_add(p.ctr + p.ev_tail, (unsigned)n) - (epoch - 1u) * per_step +
                       (unsigned)p.n_ev_init;
  for (int j = 0; j < n; ++j) {
    if (pos + (unsigned)j >= (unsigned)p.n_ev) {
      record_error(p, MK_ERR_TIMEOUT, -5, (int)c, (int)pos, j);
      return;
    }
    px::st_u64(p.ev_ready + pos + j, ((unsigned long long)epoch << 32) | (unsigned)p.ev_list[j0 + j]);
  }
}


template <int NB, class S>
__device__ void run_compute(CCtx &c, Queue q, volatile int *dyn_fifo, volatile int *dyn_tail,
                            volatile int *dyn_head) {
  // op bodies inline in the loop for the batch-1 shape builds; a batched
  // build calls them (each body alone fits the register budget, the loop
  // holding all six would spill)
  constexpr bool kInline = S::fixed && NB == 1;
  const KParams &p = c.p;
  const bool dyn = (p.mode & MODE_DYNAMIC) != 0;
  const bool trace = (p.mode & MODE_TRACE) != 0;
  for (int qi = 0;; ++qi) {
    Instr I;
    if (dyn) {
      // next claimed instruction from the loader (bounded wait, thread 0)
      if (c.ctid == 0) {
        const uint64_t t0 = px::gtimer();
        int k = -1;
        bool okw = true;
        while (*dyn_tail <= qi) {
          if (px::ld_volatile(&c.sh->abort) || global_abort(p) || px::gtimer() - t0 > (uint64_t)p.timeout_ns) {
            okw = false;
            break;
          }
        }
        if (okw) k = dyn_fifo[qi & 31];
        c.sh->flag = k;
      }
      px::cbar();
      const int k = c.sh->flag;
      px::cbar();
      if (c.ctid == 0) *dyn_head = qi + 1;
      if (k < 0) break;
      I = p.instrs[k];
    } else {
      if (qi >= q.len) break;
      I = q.base[qi];
      if (!selected(p, I)) continue;
    }
    if (I.op == OP_NOP) continue;
    unsigned long long *tr = trace ? p.trace + (size_t)I.seq * MK_TRACE_WORDS : nullptr;
    if (tr && c.ctid == 0) tr[0] = px::gtimer();
    if (c.ctid == 0) {
      // every input of the instruction carries this step's tag, so an op in
      // kSpeculativeOps starts at once and polls its producers' completion
      // count only when a load comes back stale; the others wait for the
      // count first
      const bool has_dep = I.wait_ctr != kNoCounter && !(p.mode & MODE_NO_WAIT);
      c.sh->dep_ctr = has_dep ? I.wait_ctr : kNoCounter;
      c.sh->dep_target = c.epoch * I.wait_cnt;
      c.sh->dep_seq = I.seq;
      c.sh->dep_state = 0;
      if (has_dep && !((kSpeculativeOps >> I.op) & 1u)) {
        c.sh->dep_state = 1;
        const bool ok = wait_counter(p, I.wait_ctr, c.epoch * I.wait_cnt, I.seq);
        if (!ok) c.sh->abort = 1;
        c.sh->dep_state = ok ? 2 : 3;
      }
    }
    if (px::cbar_or(px::ld_volatile(&c.sh->abort))) break;
    if (tr && c.ctid == 0) {
      tr[1] = px::gtimer();
      tr[10] = 0;
      tr[11] = c.g;  // pages consumed: replaced by the difference below
    }
    c.tr = tr;
    switch (I.op) {
      case OP_QKV:
        if constexpr (NB > 1 && S::fixed && S::TQO) {
          if (p.layers[I.layer].wqkv_tc) {
            c.g = op_qkv_tc<NB, S::RH>(c, I);
            break;
          }
        }
        if constexpr (kInline) c.g = qkv_body<NB, S::RH, S::SPL>(c, I);
        else if constexpr (S::fixed) c.g = op_qkv<NB, S::RH>(c, I);
        else MK_DISPATCH_R(op_qkv, NB, p.Rh, c, I);
        break;
      case OP_ATTN:
        if constexpr (kInline) c.g = attn_body<S::G, S::DPL, false>(c, I);
        else if constexpr (S::fixed) {
          // the prompt-chunk rows only in prompt launches: decode steps run
          // the instantiation without them (fewer live registers)
          if (NB > 1 && p.chunk_n > 1) c.g = op_attn_t<S::G, S::DPL, (NB > 1)>(c, I);
          else c.g = op_attn_t<S::G, S::DPL, false>(c, I);
        } else {
          c.g = op_attn<(NB > 1)>(c, I);
        }
        break;
      case OP_OPROJ:
        if constexpr (NB > 1 && S::fixed && S::TQO) {
          if (p.layers[I.layer].wo_tc) {
            c.g = op_oproj_tc<NB>(c, I);
            break;
          }
        }
        if constexpr (kInline) c.g = oproj_body<NB, S::RO, S::SPL>(c, I);
        else if constexpr (S::fixed) c.g = op_oproj<NB, S::RO>(c, I);
        else if constexpr (S::TP) {
          MK_DISPATCH_R1(op_oproj_tp, p.Ro, c, I);
        } else {
          MK_DISPATCH_R(op_oproj, NB, p.Ro, c, I);
        }
        break;
      case OP_GATEUP:
        if constexpr (NB > 1 && S::fixed) {
          if (p.layers[I.layer].wgu_tc) {
            c.g = op_gateup_tc<NB, S::RH>(c, I);
            break;
          }
        }
        if constexpr (kInline) c.g = gateup_body<NB, S::RH, S::SPL>(c, I);
        else if constexpr (S::fixed) c.g = op_gateup<NB, S::RH>(c, I);
        else if constexpr (S::TP) {
          MK_DISPATCH_R1(op_gateup_tp, p.Rh, c, I);
        } else {
          MK_DISPATCH_R(op_gateup, NB, p.Rh, c, I);
        }
        break;
      case OP_DOWN:
        if constexpr (NB > 1 && S::fixed) {
          if (p.layers[I.layer].wd_tc) {
            c.g = op_down_tc<NB>(c, I);
            break;
          }
        }
        if constexpr (kInline) c.g = down_body<NB, S::RD, S::SPL>(c, I);
        else if constexpr (S::fixed) c.g = op_down<NB, S::RD>(c, I);
        else if constexpr (S::TP) {
          MK_DISPATCH_R1(op_down_tp, p.Rd, c, I);
        } else {
          MK_DISPATCH_R(op_down, NB, p.Rd, c, I);
        }
        break;
      case OP_LMHEAD:
        if constexpr (NB > 1 && S::fixed) {
          if (p.lm_tc) {
            c.g = op_lmhead_tc<NB, S::RH>(c, I);
            break;
          }
        }
        if constexpr (kInline) c.g = lmhead_body<NB, S::RH, S::SPL>(c, I);
        else if constexpr (S::fixed) c.g = op_lmhead<NB, S::RH>(c, I);
        else if constexpr (S::TP) {
          MK_DISPATCH_R1(op_lmhead_tp, p.Rh, c, I);
        } else {
          MK_DISPATCH_R(op_lmhead, NB, p.Rh, c, I);
        }
        break;
      default: break;
    }
    if (tr && c.ctid == 0) {
      tr[3] = px::gtimer();
      tr[11] = (uint64_t)(c.g - (uint32_t)tr[11]);
    }
    const bool abort_now = px::cbar_or(px::ld_volatile(&c.sh->abort) != 0);
    if (abort_now) break;
    // all of this CTA's outputs of the instruction are written: publish
    // (merging instructions signal only when they merged: the last split of
    // an attention group, the last piece of a tensor-core down tile)
    const bool merging = I.op == OP_ATTN || (NB > 1 && I.op == OP_DOWN && p.xin);
    const bool sig = I.sig_ctr != kNoCounter && (!merging || c.sh->flag);
    if (c.ctid == 0 && sig) {
      // a hint only: the data words carry this step's tag, so no fence
      if (p.mode & MODE_EVENT) {
        for (int k = 0; k < I.sig_n; ++k) event_signal(p, I.sig_ctr + k, c.epoch);
      } else {
        if constexpr (S::TP) {
          // the O and down partials feed every rank: count them on every rank
          const bool all = I.op == OP_OPROJ || I.op == OP_DOWN;
          for (int rr = 0; rr < (all ? p.tp_n : 1); ++rr) {
            unsigned *ctr = all ? p.tp_peers[rr].ctr : p.ctr;
            for (int k = 0; k < I.sig_n; ++k) px::red_relaxed_add(ctr + I.sig_ctr + k, 1u);
          }
        } else {
          for (int k = 0; k < I.sig_n; ++k) px::red_relaxed_add(p.ctr + I.sig_ctr + k, 1u);
        }
      }
    }
    if (tr && c.ctid == 0) {
      tr[4] = px::gtimer();
      tr[7] = (uint64_t)I.op | ((uint64_t)I.layer << 8) | ((uint64_t)blockIdx.x << 16);
      tr[8] = (uint64_t)(unsigned)atomicExch(&sh_stat(c), 0) |
              ((uint64_t)(unsigned)atomicExch(&c.sh->stat_llretry, 0) << 32);
    }
    px::cbar();  // the staging region and the broadcast flag are reused next
  }
}

// ============================================================== kernel
template <int NB, bool RAW, class S>
__global__ void __launch_bounds__(kThreads, 1) interp_kernel(const __grid_constant__ KParams pk) {
  // the tensor-parallel build runs an emulated group in one launch: CTA
  // blocks of tp_ctas each run one rank, with that rank's parameters
  const KParams &p = S::TP ? pk.tp_params[blockIdx.x / pk.tp_ctas] : pk;
  const unsigned cta = S::TP ? blockIdx.x % (unsigned)pk.tp_ctas : blockIdx.x;
  const unsigned ncta = S::TP ? (unsigned)pk.tp_ctas : gridDim.x;
  extern __shared__ __align__(128) uint8_t smem[];
  const int NP = p.num_pages;
  uint8_t *pages = smem;
  // batched builds keep the tensor-core epilogue exchange at the end of the
  // staging region (kTcXchFloats), after the NB staged vectors
  const long long xch_floats = NB > 1 ? kTcXchFloats : 0;
  const int act_stride = (int)((p.act_floats - xch_floats) / NB);
  float *act = reinterpret_cast<float *>(smem + (size_t)NP * kPageBytes);
  uint64_t *full = reinterpret_cast<uint64_t *>(act + p.act_floats);
  uint64_t *empty = full + NP;
  Shared *sh = reinterpret_cast<Shared *>(empty + NP);
  volatile int *dyn_fifo = reinterpret_cast<volatile int *>(sh + 1);
  volatile int *dyn_tail = dyn_fifo + 32;
  volatile int *dyn_head = dyn_tail + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NP; ++i) {
      px::mbar_init(&full[i], 1);
      px::mbar_init(&empty[i], kComputeWarps);
    }
    px::mbar_init(reinterpret_cast<uint64_t *>(&sh->mma_bar), 1);
    sh->mma_phase = 0;
    px::fence_mbar_init();
    sh->abort = 0;
    sh->flag = 0;
    sh->stat_cwait = 0;
    sh->stat_llretry = 0;
    for (int i = 0; i < 16; ++i) sh->slot_last[i] = 0;
    *dyn_tail = 0;
    *dyn_head = 0;
  }
  if (threadIdx.x < (unsigned)p.B) {
    // this step's inputs, clamped once (out-of-range values are reported)
    const int b = threadIdx.x;
    int t, pos;
    if (p.chunk_n > 0) {  // prompt chunk: consecutive tokens of one sequence
      const int j = min(b, p.chunk_n - 1);
      t = __ldcg(p.tokens + j);
      pos = p.chunk_pos0 + j;
    } else {
      t = __ldcg(p.tokens + b);  // tokens may alias next_tokens
      pos = __ldcg(p.positions + b);
    }
    if (t < 0 || t >= p.V || pos < 0 || pos >= p.max_seq) record_error(p, MK_ERR_DEVICE_INPUT, b, t, pos, 0);
    sh->tok[b] = (t < 0 || t >= p.V) ? 0 : t;
    sh->pos[b] = pos < 0 ? 0 : (pos >= p.max_seq ? p.max_seq - 1 : pos);
  }
  __syncthreads();
  if (threadIdx.x < (unsigned)(p.d / 2)) sh->rope[threadIdx.x] = __ldg(p.rope + (size_t)sh->pos[0] * (p.d / 2) + threadIdx.x);
  if constexpr (NB > 1) {
    // tensor memory for the LM head's accumulators (32 columns: 16 used)
    if (warp == kLoaders) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 32;" ::"r"(px::sa(&sh->tmem_base))
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    px::tc_fence_before();
  }
  __syncthreads();
  if constexpr (NB > 1) px::tc_fence_after();
  const unsigned epoch = *reinterpret_cast<volatile unsigned *>(p.epoch);
  Queue q;
  q.base = p.instrs + p.q_off[cta];
  q.len = p.q_len[cta];
  if (warp < kLoaders) {
    // the dynamic queue is claimed by one loader only
    const bool dyn = (p.mode & MODE_DYNAMIC) != 0;
    if (lane == 0 && (!dyn || warp == 0))
      run_loader<RAW>(p, sh, pages, full, empty, q, dyn_fifo, dyn_tail, dyn_head, epoch, warp, dyn ? 1 : kLoaders);
  } else {
    CCtx c{p,     sh,    pages, act, act_stride, full, empty, epoch, warp - kLoaders, lane, (int)threadIdx.x - 32 * kLoaders,
           0u,    nullptr, NB > 1 ? act + (p.act_floats - xch_floats) : nullptr};
    run_compute<NB, S>(c, q, dyn_fifo, dyn_tail, dyn_head);
  }
  if constexpr (NB > 1) px::tc_fence_before();
  __syncthreads();
  if constexpr (NB > 1) {
    px::tc_fence_after();
    if (warp == kLoaders)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 32;" ::"r"(sh->tmem_base) : "memory");
  }
  if (threadIdx.x == 0) {
    // every bulk copy must land before the CTA exits: after an abort the
    // compute warps stop consuming pages, so wait on each slot's latest use
    for (int s = 0; s < NP; ++s) {
      const uint32_t last = sh->slot_last[s];
      if (last == 0) continue;
      const uint32_t ph = ((last - 1) / (uint32_t)NP) & 1u;
      const uint64_t t0 = px::gtimer();
      while (!px::mbar_test(&full[s], ph)) {
        if (px::gtimer() - t0 > (uint64_t)p.timeout_ns) {
          record_error(p, MK_ERR_TIMEOUT, -2, 2, s, (int)last);
          break;
        }
      }
    }
  }
  if (threadIdx.x == 0 && (p.mode & MODE_FINAL_LAUNCH)) {
    __threadfence();
    const unsigned old = px::atom_add_acq_rel(p.ctr + p.exit_ticket, 1u);
    if (old == epoch * ncta - 1u) {
      // every CTA of the step has finished: advance the step number
      atomicExch(p.epoch, epoch + 1u);
    }
  }
}

}  // namespace
}  // namespace mk
