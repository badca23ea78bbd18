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

#ifdef __cplusplus
}
#endif
#endif /* MK_HOST_H */
