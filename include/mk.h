/*
 * mk -- decode megakernel engine for Llama-style decoders on B200 (sm_100a).
 *
 * One call of mk_decode_step runs one autoregressive decode step of a batch of
 * sequences (RMSNorm, fused QKV projection + RoPE + KV-cache append, GQA
 * attention over the KV cache, O projection + residual, RMSNorm + gate/up +
 * SiLU, down projection + residual, final RMSNorm + LM head + argmax) as ONE
 * persistent kernel: every SM runs an interpreter over an instruction queue
 * that a host planner built once (mk_plan) and that every later step reuses.
 *
 * Sources (web pages on decode megakernels):
 *  - "Hazy megakernel summary" (yaoshibet.com), section 四(二): the on-GPU
 *    interpreter, the per-SM instruction sequences scheduled ahead of time on
 *    the host and reused across forward passes, the fused instruction set,
 *    paged shared memory and the global counter array;
 *  - "MegaKernel 日志" (koas-w.github.io), sections on the on-GPU interpreter
 *    and on static (per-SM queues) versus dynamic (one global queue)
 *    scheduling;
 *  - "Mirage Persistent Kernel" article (m.kljzs.com), Part 2: a runtime
 *    loop of fetch task -> run -> notify event -> repeat.
 *
 * Conventions for every call below:
 *  - Pointers named *device* point to CUDA device memory of the device that
 *    was current at mk_create; everything else is host memory.
 *  - All tensors are row-major.  Weight matrices are [out][in] (bf16), so one
 *    output row is contiguous.  bf16 = IEEE bfloat16 bit pattern (uint16).
 *  - Return value: MK_OK (0) or a negative MK_ERR_* code.  No call throws.
 *  - A handle is not thread-safe: one host thread at a time per handle.
 */
#ifndef MK_H
#define MK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ errors */
enum {
  MK_OK = 0,
  MK_ERR_INVALID_ARG = -1,      /* NULL/negative/inconsistent argument */
  MK_ERR_UNSUPPORTED_SHAPE = -2,/* shape outside what the kernels implement */
  MK_ERR_NOT_PLANNED = -3,      /* mk_decode_step before a successful mk_plan */
  MK_ERR_CUDA = -4,             /* a CUDA runtime call failed */
  MK_ERR_LAUNCH = -5,           /* the persistent launch was refused (co-residency) */
  MK_ERR_TIMEOUT = -6,          /* a device-side wait gave up (reported by mk_get_status) */
  MK_ERR_DEVICE_INPUT = -7,     /* a token id or position was out of range on the device */
  MK_ERR_OUT_OF_MEMORY = -8     /* a device allocation failed */
};

typedef struct mk_handle mk_handle;

/* ------------------------------------------------------------------ model */
typedef struct {
  int32_t n_layers;     /* decoder layers */
  int32_t hidden;       /* H */
  int32_t n_q_heads;    /* query heads */
  int32_t n_kv_heads;   /* key/value heads; n_q_heads % n_kv_heads == 0 */
  int32_t head_dim;     /* d */
  int32_t ffn;          /* F, SwiGLU width */
  int32_t vocab;        /* V */
  float rms_eps;        /* RMSNorm epsilon */
  double rope_theta;    /* RoPE base */
  int32_t tied_lm_head; /* 1: lm_head == embed (the weights pointer may be either) */
  int32_t max_batch;    /* capacity: sequences per step */
  int32_t max_seq;      /* capacity: KV positions per sequence */
} mk_config;

typedef struct {
  const void *attn_norm; /* device bf16 [H] */
  const void *wq;        /* device bf16 [n_q_heads*d][H] */
  const void *wk;        /* device bf16 [n_kv_heads*d][H] */
  const void *wv;        /* device bf16 [n_kv_heads*d][H] */
  const void *wo;        /* device bf16 [H][n_q_heads*d] */
  const void *ffn_norm;  /* device bf16 [H] */
  const void *w_gate;    /* device bf16 [F][H] */
  const void *w_up;      /* device bf16 [F][H] */
  const void *w_down;    /* device bf16 [H][F] */
} mk_layer_weights;

typedef struct {
  const void *embed;      /* device bf16 [V][H] */
  const void *lm_head;    /* device bf16 [V][H]; ignored (embed used) when tied */
  const void *final_norm; /* device bf16 [H] */
  const mk_layer_weights *layers; /* HOST array [n_layers]; read during mk_create only */
} mk_weights;

typedef struct {
  void *k; /* device bf16 [n_layers][max_batch][n_kv_heads][max_seq][head_dim] */
  void *v; /* same layout */
} mk_kv_cache;

/*
 * mk_create: validate the shape, take the weight and KV pointers, and build the
 * device-side state (repacked weight copies, RoPE table, activation buffers).
 * ("Hazy megakernel summary", section 四(二): the model's weights streamed
 * page by page by the interpreter; the repacking makes each page one copy.)
 *  - Ownership: weights and the KV cache are BORROWED; they must stay valid
 *    until mk_destroy and the library never frees them.  The library keeps its
 *    own repacked copy of the fused QKV, gate/up and down-projection weights
 *    (taken at mk_create: later changes to the caller's weights are not seen),
 *    and reads embed / wo / lm_head / norm weights in place.  The KV cache is
 *    written only at row positions[b] of sequence b by mk_decode_step.
 *  - Shapes implemented: head_dim in {64, 128}, hidden and n_q_heads*head_dim
 *    in {256, 512, 1024, 2048, 4096}, n_q_heads a multiple of n_kv_heads with
 *    at most 8 query heads per KV head, ffn in {256, 512, 1024, 2048} or a
 *    multiple of 2048 up to 16384 (the down projection's K pieces divide a
 *    16 KiB page), vocab >= 1, max_batch in [1, 16], max_seq >= 1.  Others
 *    give MK_ERR_UNSUPPORTED_SHAPE.  Batch > 1 is planned only for shapes with
 *    a batched build (the Llama-3.2-1B shape).
 *  - Uses the current CUDA device.  Synchronous (returns when set-up is done).
 *  - Errors: MK_ERR_INVALID_ARG (NULL pointer, non-positive size),
 *    MK_ERR_UNSUPPORTED_SHAPE, MK_ERR_OUT_OF_MEMORY, MK_ERR_CUDA.
 *    On error *out is set to NULL and nothing is leaked.
 */
int mk_create(const mk_config *cfg, const mk_weights *w, const mk_kv_cache *kv,
              mk_handle **out);

/* ------------------------------------------------------------------ plan */
enum { MK_SCHED_STATIC = 0, MK_SCHED_DYNAMIC = 1, MK_SCHED_EVENT = 2 };
enum {
  MK_EXEC_MEGAKERNEL = 0,        /* one persistent launch per step */
  MK_EXEC_PER_OP = 1,            /* comparison path: one launch per instruction class */
  MK_EXEC_PER_OP_GRAPH = 2,      /* the same launches replayed as a CUDA graph */
  MK_EXEC_MEGAKERNEL_GENERIC = 3 /* one persistent launch of the shape-generic
                                    interpreter build (identical results; the
                                    default picks a shape-specialised build when
                                    the model's shape has one) */
};

typedef struct {
  int32_t batch;          /* sequences per step, 1..max_batch */
  int32_t kv_splits;      /* split-KV factor of decode attention; 0 = automatic
                             (one attention item per CTA, at least ~32
                             positions per split); -1 = the count the plan cost
                             model (mk_host.h) estimates fastest at max_seq */
  int32_t sched_mode;     /* MK_SCHED_STATIC (per-SM queues), MK_SCHED_DYNAMIC
                             (one global queue in topological order, claimed
                             with an atomic), or MK_SCHED_EVENT (one global
                             queue of ready instructions: the producer whose
                             signal completes a dependency count appends the
                             instructions waiting on it -- the event-driven
                             scheduling of the "Mirage Persistent Kernel"
                             article, part 2) */
  int32_t exec_mode;      /* MK_EXEC_MEGAKERNEL, or the comparison path:
                             one launch per instruction class (PER_OP), optionally
                             replayed as a CUDA graph (PER_OP_GRAPH), or
                             MK_EXEC_MEGAKERNEL_GENERIC */
  int32_t num_sms;        /* CTAs of the persistent grid; 0 = every SM */
  int32_t trace;          /* 1: record per-instruction timestamps (mk_trace_read) */
  int64_t wait_timeout_ns;/* bound on every device-side wait; 0 = 1 second */
  int32_t l2_prefetch_kb; /* L2 look-ahead per CTA, KiB: while its page ring is
                             full (the compute warps wait on a dependency), the
                             loader asks L2 for up to this many bytes of later
                             weight / KV pages; 0 = automatic, -1 = off */
  int32_t debug_drop_producer; /* TEST HOOK: 1 drops one producer instruction so
                             that a dependency can never be met and the bounded
                             wait must report MK_ERR_TIMEOUT; 0 in normal use */
  int32_t max_inflight_pages; /* 16 KiB weight/KV pages a CTA keeps in flight
                             (the rest of its page ring only buffers landed
                             pages); 0 = automatic (4), -1 = no cap; rounded
                             down to a multiple of the loader count (2) */
  int32_t tensor_qkv_o;   /* batched plans (batch > 1): 1 = QKV and the O
                             projection run on the tensor cores as well, as
                             whole 128-row tiles (fewer, larger instructions:
                             on 148 SMs the Llama-1B shape then has 24 QKV and
                             16 O tiles per layer, and the step is slower);
                             0 = on CUDA cores (default).  Ignored at batch 1;
                             needs the tensor cores (use_tcgen05 not -1) */
  int32_t use_tcgen05;    /* 5th-generation tensor cores (tcgen05.mma with
                             tensor-memory accumulators) for the matrix
                             instructions of batched plans, where a step's
                             matrix-vector products are dense contractions
                             over the batch: 0 = automatic (batch > 1: on
                             when the plan cost model expects them to beat
                             the CUDA cores), 1 = on (MK_ERR_INVALID_ARG at
                             batch 1, where every product is a matrix-vector
                             product and CUDA-core FMAs are used), -1 = off
                             (CUDA cores for every batch) */
} mk_plan_opts;

/*
 * mk_plan ("Hazy megakernel summary", section 四(二): every SM's instruction
 * sequence is scheduled on the host ahead of time and one schedule serves
 * many forward passes; "MegaKernel 日志", section on static and dynamic
 * scheduling): build the instruction DAG for this batch size, partition it into
 * per-SM queues (or one global queue), set the dependency-counter targets,
 * check the plan (every queue follows one global topological order) and upload
 * it.  Call once; the plan is reused by every later mk_decode_step.  Calling it
 * again replaces the plan (and synchronises the device).  Resets the step
 * counters, so it must not overlap a running step of this handle.
 *  - opts may be NULL (defaults: batch = max_batch, everything else automatic).
 *  - Errors: MK_ERR_INVALID_ARG (batch out of range, bad mode),
 *    MK_ERR_UNSUPPORTED_SHAPE, MK_ERR_OUT_OF_MEMORY, MK_ERR_CUDA.
 */
int mk_plan(mk_handle *h, const mk_plan_opts *opts);

/* ------------------------------------------------------------------ step */
/*
 * mk_decode_step ("Hazy megakernel summary", section 四(二): one persistent
 * kernel whose per-SM interpreter fetches, runs and retires the fused
 * instructions; "Mirage Persistent Kernel" article, Part 2: the runtime loop
 * of fetch task -> run -> notify event): one decode step for sequences
 * b = 0..batch-1.
 *  - tokens          device int32 [batch]: the input token of each sequence.
 *  - positions       device int32 [batch]: its position p_b (0 <= p_b < max_seq).
 *                    The step writes the token's K and V at row p_b of the
 *                    cache and attends over rows 0..p_b, so rows 0..p_b-1 must
 *                    hold this sequence's earlier keys (post-RoPE) and values.
 *  - logits_out      device float [batch][vocab], or NULL to skip writing logits.
 *  - next_tokens_out device int32 [batch]: argmax of the logits (lowest index
 *                    among equal maxima).  May alias `tokens` (feeding the next
 *                    step without a host round trip).
 *  - stream          cudaStream_t (as void*); NULL = legacy default stream.
 * Asynchronous and stream-ordered: returns once the work is enqueued, with no
 * host synchronisation.  Device-side problems (a wait timeout, a token id
 * outside [0, vocab) or a position outside [0, max_seq) -- which are clamped)
 * are reported by the next mk_get_status.  Errors returned here:
 * MK_ERR_INVALID_ARG, MK_ERR_NOT_PLANNED, MK_ERR_LAUNCH, MK_ERR_CUDA.
 */
int mk_decode_step(mk_handle *h, const int32_t *tokens, const int32_t *positions,
                   float *logits_out, int32_t *next_tokens_out, void *stream);

/*
 * mk_prefill ("One Megakernel is Not Enough" digest, 首次出现的概念: prefill,
 * which processes a prompt's tokens together, against decode, one token per
 * step; the digest notes that prefill is usually left to conventional
 * execution -- here it runs in the same persistent interpreter): write the K
 * and V rows of prompt tokens pos0 .. pos0+n_tokens-1 of KV sequence `seq`
 * and return the logits and greedy next token of the last one.
 *  - seq             0 <= seq < max_batch: the cache sequence to fill.
 *  - tokens          device int32 [n_tokens]: the prompt tokens, in order.
 *  - n_tokens, pos0  n_tokens >= 1, pos0 >= 0, pos0 + n_tokens <= max_seq;
 *                    rows 0 .. pos0-1 of the sequence must already hold its
 *                    earlier keys and values (e.g. an earlier mk_prefill).
 *  - logits_out      device float [vocab]: the last token's logits, or NULL.
 *  - next_token_out  device int32 [1]: their argmax (lowest index on ties).
 *  - stream          cudaStream_t (as void*).
 * With a batched plan (batch B > 1, a shape with a batched build) the prompt
 * runs in chunks of up to B consecutive tokens, one launch per chunk: the
 * chunk's tokens are the B rows of the tensor-core matrix instructions, and
 * token j of a chunk attends over the cache rows before the chunk and the
 * chunk's rows 0..j (this launch's K/V exchange).  With a batch-1 plan, one
 * token per launch (any shape).  Needs a plan with a one-launch exec_mode;
 * each launch counts as a step of the plan (like mk_decode_step).
 * Asynchronous and stream-ordered.  Errors: MK_ERR_INVALID_ARG,
 * MK_ERR_NOT_PLANNED, MK_ERR_OUT_OF_MEMORY (its scratch, allocated with the
 * plan on first use), MK_ERR_LAUNCH, MK_ERR_CUDA; device-side ones at the
 * next mk_get_status.
 */
int mk_prefill(mk_handle *h, int32_t seq, const int32_t *tokens, int32_t n_tokens, int32_t pos0,
               float *logits_out, int32_t *next_token_out, void *stream);

/*
 * mk_get_status ("Hazy megakernel summary", section 四(二) 同步: the counters
 * in global memory that replace kernel boundaries; every wait on them is
 * bounded here, and a wait that gives up is reported by this call):
 * synchronise `stream` and return the first device-side error
 * recorded since the last call (MK_ERR_TIMEOUT, MK_ERR_DEVICE_INPUT), or a CUDA
 * error (MK_ERR_CUDA), or MK_OK.  Clears the recorded device error.
 */
int mk_get_status(mk_handle *h, void *stream);

/* Static English text for a code (never NULL). */
const char *mk_status_string(int code);

/* Free everything the handle owns (synchronises the device first).  Borrowed
   weights and KV are untouched.  NULL is allowed. */
void mk_destroy(mk_handle *h);

/* ------------------------------------------------------------------ tensor parallelism */
/*
 * A tensor-parallel group ("Mirage Persistent Kernel" article, part 1: the
 * matrix products split across GPUs, with each chunk of the collective that
 * follows depending only on the tile that produces it).  Rank r of n holds
 * query heads [r nq/n, (r+1) nq/n) and their KV heads, FFN columns
 * [r F/n, (r+1) F/n) and vocabulary rows [r V/n, (r+1) V/n): QKV and gate/up
 * are split by output rows (no exchange), the O and down projections by
 * input columns -- each of their pages stores its partial sums into every
 * rank's partial buffers (the all-reduce, chunked by page; consumers sum the
 * ranks' partials in rank order) -- and the LM head by vocabulary rows, with
 * the argmax merged over every rank's candidates.  This build emulates the
 * group on one GPU: one cooperative launch of n * (SMs / n) CTAs runs every
 * rank's plan with its own parameters and buffers (ranks whose kernels wait
 * on one another must share a launch on one GPU); the stores into the other
 * ranks' buffers are the ones a group of GPUs makes over NVLink.
 */
typedef struct mk_tp_group mk_tp_group;

/*
 * mk_tp_create: n_ranks in {2, 4, 8}, dividing n_q_heads, n_kv_heads, ffn and
 * vocab.  Weights and the KV cache as for mk_create (borrowed; each rank
 * reads its heads' rows of the caller's cache in place, and copies its column
 * shards of Wo and W_down).  Errors: MK_ERR_INVALID_ARG,
 * MK_ERR_UNSUPPORTED_SHAPE, MK_ERR_OUT_OF_MEMORY, MK_ERR_CUDA.
 */
int mk_tp_create(const mk_config *cfg, const mk_weights *w, const mk_kv_cache *kv, int32_t n_ranks,
                 mk_tp_group **out);
/* Plan every rank (opts: batch 1, static queues, a one-launch exec_mode; the
   ranks run the shape-generic build on SMs / n CTAs each). */
int mk_tp_plan(mk_tp_group *g, const mk_plan_opts *opts);
/* One decode step of the group (arguments as mk_decode_step, batch 1);
   asynchronous, stream-ordered.  logits_out receives every rank's rows. */
int mk_tp_decode_step(mk_tp_group *g, const int32_t *tokens, const int32_t *positions, float *logits_out,
                      int32_t *next_tokens_out, void *stream);
/* Synchronise and return the first device-side error of any rank (then the
   group must be planned again), or MK_OK. */
int mk_tp_get_status(mk_tp_group *g, void *stream);
void mk_tp_destroy(mk_tp_group *g);

/* ------------------------------------------------------------------ introspection */
typedef struct {
  int32_t num_ctas;        /* persistent grid size */
  int32_t threads_per_cta;
  int32_t smem_bytes;      /* dynamic shared memory per CTA */
  int32_t num_pages;       /* 16 KiB shared-memory pages per CTA */
  int32_t num_instructions;/* per step */
  int32_t num_counters;
  int32_t kv_splits;
  int32_t max_queue_len;   /* longest per-CTA queue (static mode) */
  int64_t weight_bytes_per_step; /* weight bytes the plan streams per step */
  int32_t kernel_variant;  /* 0: the shape-generic interpreter build, 1: a build
                              specialised for this model's shape (every op body
                              inlined into the interpreter loop) */
  int32_t estimated_step_us; /* the plan cost model's estimate of one step with
                              every sequence at max_seq, microseconds (see
                              mk_host_plan_estimate); 0 for the dynamic queue */
} mk_plan_info;

/*
 * mk_get_error_detail: the detail words of the last device-side error that
 * mk_get_status returned (host int32 [6]): instruction sequence number (-1:
 * a shared-memory page wait, -2: the final drain, -3: a group of tagged
 * activation loads that never saw this step's tag, -4: an event-driven
 * ready-queue slot that was never filled, -5: a ready-queue overflow),
 * counter index or wait kind,
 * observed value, target value, CTA, and the abort flag.  All zero if none.
 */
int mk_get_error_detail(const mk_handle *h, int32_t detail[6]);

/* Fill *info for the current plan.  MK_ERR_NOT_PLANNED before mk_plan. */
int mk_get_plan_info(const mk_handle *h, mk_plan_info *info);

/*
 * mk_trace_read: copy the per-instruction timestamps of the last step into
 * `out` (host, uint64 [num_instructions][MK_TRACE_WORDS], nanoseconds of the
 * device global timer).  Requires a plan with trace = 1; synchronises.
 * Word meaning: 0 = instruction fetched by the compute warps, 1 = its
 * dependencies were met, 2 = its input vector was staged, 3 = its pages were
 * consumed and its outputs written, 4 = it signalled completion, 5 / 6 = the
 * loader issued its first / last page (5 == 6 when it has no pages),
 * 7 = (opcode | layer << 8 | cta << 16), 8 = pages the compute warps found
 * not yet landed (low 32 bits) | groups of tagged activation loads re-issued
 * because a word was not yet this step's (high 32 bits), 9 = pages the loader
 * found no free ring slot for, 10 = attention: the first compute warp left
 * the page loop (before the warps' merge and the split merge; 0 for other
 * instructions), 11 = pages the instruction consumed.
 */
#define MK_TRACE_WORDS 12
int mk_trace_read(mk_handle *h, uint64_t *out, size_t n_words);

/* ------------------------------------------------------------------ allocation-free step */
/*
 * mk_decode_step_noalloc: the same decode step as mk_decode_step, for callers
 * that cannot allocate device memory when they run it.  (The pages have no
 * counterpart of this call.)
 *
 * Who needs it: code that may not call cudaMalloc or any allocating routine at
 * this point -- e.g. a host callback or a context where allocation calls are
 * not allowed, a runtime whose device memory is owned and budgeted by another
 * component, or a caller that must avoid the implicit synchronisation an
 * allocation can cause.  mk_create is not available to them because it
 * allocates the repacked weights, activation and counter buffers and the plan.
 *
 * How: no handle.  The step's scratch (plan, RoPE table, activations,
 * attention and argmax partials, counters, status) lives in one file-scope
 * device array of MK_NOALLOC_SCRATCH_BYTES (16 MiB), which every GPU that loads
 * the library holds until the process exits.  The weights are read in the
 * caller's own layout, so no repacked copy is made.  This call makes no
 * cudaMalloc / cudaFree and uses no allocating library routine.
 *  - cfg, w, kv: as for mk_create (host structs; device tensor pointers,
 *    16-byte aligned).  cfg->max_batch must be 1 (the batch of this step).
 *  - tokens, positions, logits_out (may be NULL), next_tokens_out, stream: as
 *    for mk_decode_step.  The kernel plan is the one mk_plan builds with
 *    default options on this device, so results are identical to mk_create +
 *    mk_plan(NULL) + mk_decode_step.
 *  - First call on a device (with that device current): looks up the array's
 *    device address and uploads the plan and tables, synchronising `stream`.
 *    Make that first call before any stream capture.  Later calls re-upload
 *    (and synchronise) only when cfg or the weight pointers change.
 *  - Every call shares the array and leaves its contents behind; each call
 *    clears the counters, status and activation words it needs.  Calls that overlap on the GPU
 *    (other streams, other threads) race on the array: serialise them.
 *  - Errors: MK_ERR_INVALID_ARG (NULL or misaligned pointer, bad cfg),
 *    MK_ERR_UNSUPPORTED_SHAPE (shape not implemented, batch != 1, or the
 *    scratch this shape needs exceeds MK_NOALLOC_SCRATCH_BYTES -- roughly the
 *    Llama-1B shape up to ~8K positions fits, the 8B shape does not),
 *    MK_ERR_LAUNCH, MK_ERR_CUDA.  Device-side errors of the step (timeout,
 *    clamped input) are reported by mk_noalloc_get_status until the next call
 *    clears them.
 */
#define MK_NOALLOC_SCRATCH_BYTES (16u << 20)
int mk_decode_step_noalloc(const mk_config *cfg, const mk_weights *w, const mk_kv_cache *kv,
                           const int32_t *tokens, const int32_t *positions, float *logits_out,
                           int32_t *next_tokens_out, void *stream);

/*
 * mk_noalloc_get_status: synchronise `stream` and return the device-side
 * error of the last mk_decode_step_noalloc on the current device
 * (MK_ERR_TIMEOUT, MK_ERR_DEVICE_INPUT), MK_OK, or MK_ERR_CUDA; `detail`
 * (host int32 [6] or NULL) as for mk_get_error_detail.  The next call clears
 * the status.  MK_OK before any call on the device.
 */
int mk_noalloc_get_status(void *stream, int32_t *detail);

#ifdef __cplusplus
}
#endif
#endif /* MK_H */
