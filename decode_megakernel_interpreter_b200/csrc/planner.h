// Host-side planner: builds the decode-step instruction DAG, splits it into
// per-CTA queues (or one global queue), assigns dependency counters and
// checks the result.  Plain C++ (no CUDA), so it also runs on machines
// without a GPU (tests and the host simulation).
#pragma once
#include <stdint.h>

#include <string>
#include <vector>

#include "mk_internal.h"

namespace mk {

struct Shape {
  int L, H, nq, nkv, d, F, V;
};

struct PlanRequest {
  Shape s;
  int B = 1;          // batch
  int S = 0;          // kv splits (0 = automatic)
  int num_ctas = 148;
  bool dynamic = false;
  int dyn_chunks_per_cta = 2;  // dynamic mode: instructions per CTA per matvec stage
  int assumed_context = 1024;  // for the automatic split count
  bool drop_producer = false;  // test hook (see mk_plan_opts)
  // tensor cores (batched plans): gate/up, down and LM-head instructions
  // cover whole 128-row tiles of tiled weight copies (64 columns per page)
  bool tensor = false;
  // with `tensor`: QKV and O-projection instructions as tensor-core tiles too
  bool tensor_qkv_o = false;
};

struct Plan {
  // geometry
  int Rh = 0, Ro = 0, Rd = 0, KCd = 0, ndp = 0, S = 0;
  bool tensor = false;  // see PlanRequest
  bool tensor_qkv_o = false;
  int gu_rows_unit = 0;  // act rows per gate/up unit (page, or 64 on the tensor cores)
  int dn_rows_unit = 0;  // output rows per down unit (page, or 128 on the tensor cores)
  int qkv_pages_unit = 1;  // batch-1 QKV pages per QKV unit (1, or 128 / Rh for a tile)
  int o_rows_unit = 0;     // output rows per O-projection unit (page, or 128)
  int P_qkv = 0, P_o = 0, P_gu = 0, P_dp = 0, P_lm = 0;  // pages per layer / piece / head
  // instructions: static mode = per-CTA queues back to back; dynamic = global order
  std::vector<Instr> instrs;
  std::vector<int> q_off, q_len;
  int num_ctas = 0;
  bool dynamic = false;
  // counters
  int ctr_per_layer = 0;
  int n_counters = 0;
  unsigned attn_ticket0 = 0, arg_ticket0 = 0, exit_ticket = 0, dyn_head = 0;
  int n_lm = 0;
  int64_t weight_bytes = 0;  // weight bytes streamed per step

  unsigned ctr_qkv(int l) const { return l * ctr_per_layer + 0; }
  unsigned ctr_attn(int l) const { return l * ctr_per_layer + 1; }
  unsigned ctr_o(int l) const { return l * ctr_per_layer + 2; }
  unsigned ctr_gu(int l, int k) const { return l * ctr_per_layer + 3 + k; }
  unsigned ctr_dn(int l) const { return l * ctr_per_layer + 3 + ndp; }
};

// Geometry checks shared by mk_create/mk_plan.  Returns "" when supported,
// else the reason.
std::string check_shape(const Shape &s, int B);

// Build a plan.  Returns "" on success, else an error message.
std::string build_plan(const PlanRequest &req, Plan *out);

// Structural validation: every dependency is produced by instructions that
// come earlier in the global order, every queue is a subsequence of that
// order, counter targets equal producer counts and every output element is
// written exactly once.  Returns "" when the plan is valid.
std::string validate_plan(const PlanRequest &req, const Plan &p);

// Host simulation: `threads` CPU threads play the CTAs and run the queues
// for `steps` steps under random delays, with real atomic counters and
// version stamps on every buffer element; any read of a stale element, any
// double write or a deadlock (no progress for `timeout_ms`) is an error.
std::string simulate_plan(const PlanRequest &req, const Plan &p, int steps, uint64_t seed,
                          int timeout_ms);

}  // namespace mk
