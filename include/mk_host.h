/*
 * mk host-only planner entry points (no GPU needed).
 *
 * The planner of mk_plan is host code: it builds the instruction DAG of one
 * decode step, places it into per-SM queues (or one global queue) and sets the
 * dependency-counter targets, once, for reuse by every step ("Hazy megakernel
 * summary" page, section 四(二): the per-SM instruction sequences are laid out
 * on the host ahead of time and one schedule serves many forward passes).
 * These two calls expose that planner without a device, for inspection and
 * for a host simulation of the counter protocol; they allocate only host
 * memory and never touch CUDA.
 */
#ifndef MK_HOST_H
#define MK_HOST_H

#include <stddef.h>
#include <stdint.h>

#include "mk.h"

#ifdef __cplusplus
extern "C" {
#endif

/* One instruction of a plan (mirrors the 32-byte device record). */
typedef struct {
  uint8_t op;      /* 0 nop, 1 qkv, 2 attention, 3 o-proj, 4 gate/up, 5 down, 6 lm-head */
  uint8_t pad;
  uint16_t layer;  /* n_layers for the LM head */
  uint32_t a;      /* matvec ops: first unit (a 16 KiB weight page; in batched
                      plans a 128-row tensor-core tile for gate/up (64 gate +
                      64 up rows), down, LM head, and QKV / O projection with
                      tensor_qkv_o); attention: kv head */
  uint32_t b;      /* matvec ops: number of units; attention: split index */
  uint32_t c;      /* down: K piece; attention: sequence; lm-head: argmax slot */
  uint32_t wait_ctr, wait_cnt; /* wait until counter[wait_ctr] >= step * wait_cnt
                                  (wait_ctr = 0xFFFFFFFF: no wait) */
  uint32_t sig_ctr;            /* first counter signalled on completion (0xFFFFFFFF: none) */
  uint16_t sig_n;              /* consecutive counters signalled */
  uint16_t seq;                /* position in the global topological order */
} mk_instr_desc;

/*
 * mk_host_plan: build and validate the plan mk_plan would build for `cfg`
 * (mk_create's config) and `opts` on `num_ctas` CTAs, without a device.
 *  - instrs_out: host array of max_instrs entries, or NULL (then only counts).
 *    Static mode: the per-CTA queues back to back; queue_off / queue_len
 *    (host int32 [num_ctas] each, may be NULL) give each CTA's slice.
 *    Dynamic mode: the global order.
 *  - n_instrs: receives the number of instructions.
 *  - info: receives the plan summary (smem fields are 0), may be NULL.
 *  - err: receives a message on failure (may be NULL).
 * Errors: MK_ERR_INVALID_ARG, MK_ERR_UNSUPPORTED_SHAPE (message in err),
 * MK_ERR_INVALID_ARG also when max_instrs is too small.
 */
int mk_host_plan(const mk_config *cfg, const mk_plan_opts *opts, int32_t num_ctas,
                 mk_instr_desc *instrs_out, int32_t max_instrs, int32_t *n_instrs,
                 int32_t *queue_off, int32_t *queue_len, mk_plan_info *info, char *err,
                 size_t err_len);

/*
 * mk_host_plan_simulate: run the plan for `steps` steps with one CPU thread
 * per CTA, real atomic counters with acquire/release ordering, random delays,
 * and a version stamp on every element of every intermediate buffer.  Fails
 * (MK_ERR_INVALID_ARG, message in err) if an instruction reads an element not
 * yet written in the current step, writes one twice, leaves one unwritten, or
 * waits longer than timeout_ms (a deadlock).  MK_OK otherwise.
 */
int mk_host_plan_simulate(const mk_config *cfg, const mk_plan_opts *opts, int32_t num_ctas,
                          int32_t steps, uint64_t seed, int32_t timeout_ms, char *err,
                          size_t err_len);

/*
 * Cost model of a plan (no GPU).  After the "One Megakernel is Not Enough"
 * digest: section 2.2 (a service table of operator times that scale with the
 * CTA waves ceil(g / W) of the CTAs an operator gets) and section 2.3 (a
 * region is worth a persistent kernel when its per-step savings S(b) over
 * conventional launches exceed its fixed cost F).  The plan's instructions
 * are replayed in their global order: each CTA streams its 16 KiB pages at
 * its share of the HBM bandwidth into a ring of ring_pages pages; an
 * instruction starts when its CTA is free and its producers have finished
 * plus one exchange through global memory, consumes its pages at the compute
 * rate and ends after a fixed cost; a ticketed attention merge adds two
 * exchanges and the merge itself to the last split.  The conventional path is
 * one launch per instruction class and layer, each launch as long as its
 * slowest CTA from a cold ring, in ceil(g / W) waves.  The default
 * parameters are this build's measurements on a B200 (see each field).
 */
typedef struct {
  double sm_gbs;          /* bulk-copy bandwidth one SM sustains, GB/s (49) */
  int32_t ring_pages;     /* 16 KiB ring pages per CTA (12) */
  double exchange_us;     /* producer's last store -> consumer's loads fresh, under load (1.6) */
  double page_us;         /* batch 1: compute per 16 KiB weight page (0.13) */
  double attn_page_us;    /* attention compute per K/V page (0.30) */
  double attn_fixed_us;   /* attention item: current row, warp merge, stores (0.8) */
  double merge_us;        /* ticketed merge: the last split's own merge work (0.6) */
  double instr_us;        /* per matrix instruction: barriers, epilogue, signal (0.25) */
  double launch_us;       /* conventional path: one launch from a CUDA graph (1.3) */
  double tc_page_us;      /* batched plans: tensor-core MMAs per weight page (0.20) */
  double cc_page_us_seq;  /* batched plans on CUDA cores: per weight page and sequence (0.12) */
  int32_t conv_ctas;      /* CTAs the conventional path gets, W (0: the plan's) */
  double merge_split_us;  /* ticketed merge: per split whose partial the last split reloads (0) */
} mk_cost_params;

typedef struct {
  double step_us;         /* the megakernel step */
  double per_op_us;       /* the conventional path: one launch per instruction class and layer */
  double hbm_floor_us;    /* the plan's weight and K/V pages at every SM's bandwidth */
  double savings_us;      /* S(b) = per_op_us - step_us */
  double stage_us[7];     /* per opcode (index = mk_instr_desc.op): mean instruction time */
} mk_cost_estimate;

/* The default parameters (host, filled in). */
void mk_cost_params_default(mk_cost_params *params);

/*
 * mk_host_plan_estimate: the plan mk_plan would build for cfg / opts on
 * num_ctas CTAs (static queues only), replayed with the sequences at position
 * `context`.  params NULL = defaults.  Errors: MK_ERR_INVALID_ARG (bad
 * arguments, dynamic queue; message in err), MK_ERR_UNSUPPORTED_SHAPE.
 */
int mk_host_plan_estimate(const mk_config *cfg, const mk_plan_opts *opts, int32_t num_ctas, int32_t context,
                          const mk_cost_params *params, mk_cost_estimate *out, char *err, size_t err_len);

#ifdef __cplusplus
}
#endif
#endif /* MK_HOST_H */
