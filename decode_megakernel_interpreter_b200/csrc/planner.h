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

constexpr int kSplitsByCost = -1;

struct PlanRequest {
  Shape s;
  int B = 1;          // batch
  int S = 0;          // kv splits (0: the fixed rule; kSplitsByCost: the cost model's choice)
  int num_ctas = 148;
  bool dynamic = false;
  int dyn_chunks_per_cta = 2;  // dynamic mode: instructions per CTA per matvec stage
  // with `dynamic`: the global queue holds only ready instructions -- an
  // instruction is appended when the last of its producers signals (the
  // event-driven mode); without it the queue is the fixed topological order
  bool events = false;
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
  // event-driven mode: for counter c, the instructions (indices into instrs)
  // that wait on it are ev_list[ev_off[c] .. ev_off[c+1]) and become ready
  // when it reaches epoch * ev_cnt[c]; ev_init lists the instructions that
  // wait on nothing (ready at the start of every step)
  bool events = false;
  std::vector<int> ev_off, ev_list, ev_init;
  std::vector<unsigned> ev_cnt;
  // counters
  int ctr_per_layer = 0;
  int n_counters = 0;
  unsigned attn_ticket0 = 0, arg_ticket0 = 0, exit_ticket = 0, dyn_head = 0, ev_tail = 0;
  unsigned dn_ticket0 = 0;  // tensor cores: [L][H / 128] tickets of the down tiles' merges
  int n_lm = 0;
  int n_gu = 0;  // gate/up instructions per layer
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
// The most down-projection K pieces any plan of this shape uses (buffers of
// per-piece partial sums are sized for it).
int down_pieces_max(const Shape &s);

// Structural validation: every dependency is produced by instructions that
// come earlier in the global order, every queue is a subsequence of that
// order, counter targets equal producer counts and every output element is
// written exactly once.  Returns "" when the plan is valid.
std::string validate_plan(const PlanRequest &req, const Plan &p);

// ------------------------------------------------------------------ cost model
// Time model of a plan on the device, after the "One Megakernel is Not Enough"
// digest (section 2.2: a service table whose operator times scale with the
// CTA waves ceil(g / W) of the CTAs they get; section 2.3: a region is worth a
// persistent kernel when its per-step savings S(b) over conventional launches
// exceed its fixed cost F).  The plan's instructions are replayed in their
// global order: each CTA streams its pages at its share of the HBM bandwidth
// into its ring, an instruction starts once its CTA is free and its
// producers finished plus one exchange through global memory, consumes its
// pages at the compute rate, and finishes after a fixed epilogue/signal
// cost.  Attention items cost a per-KV-page time; the ticketed split merge
// adds two exchanges and the merge to the last split.  The
// conventional path is one launch per instruction class and layer whose CTAs
// run in ceil(items / W) waves with no prefetch across launches.
struct CostParams {
  // Defaults: fitted (least squares on log time) to B200 measurements of this
  // build -- the Llama-1B shape at contexts 1024 and 8192 with 6 to 72 KV
  // splits, the Llama-8B shape with 9 to 18, the 1B shape at batch 16 with 1
  // to 8 splits and with and without tensor cores, and the per-op path
  // replayed as a CUDA graph (absolute times, and the ratios between the
  // split counts of one sweep).
  double sm_gbs = 39.4;         // bulk-copy bandwidth one SM sustains (GB/s)
  int ring_pages = 12;          // 16 KiB pages per CTA ring
  double exchange_us = 1.0;     // a producer's last store -> a consumer's loads see it (under load)
  double page_us = 0.05;        // compute time per 16 KiB weight page per sequence group (batch 1)
  double attn_page_us = 1.45;   // attention compute per K/V page, all warps
  double attn_fixed_us = 8.6;   // attention: q loads, current row, warp merge, partial stores, ticket
  double merge_us = 0.1;        // ticketed merge: the last split's own work besides its two exchanges
  double instr_us = 0.46;       // per instruction: fetch, barriers, epilogue, signal
  double launch_us = 26.6;      // conventional path: one launch (cooperative, from a CUDA graph) and its prologue
  double tc_page_us = 3.56;     // batched plans: tensor-core MMAs of one weight page (16 sequences)
  double cc_page_us_seq = 0.49; // batched plans on CUDA cores: per weight page and sequence
  int conv_ctas = 0;            // CTAs the conventional path gets (0: the plan's); fewer -> more waves
  double merge_split_us = 0.28; // ticketed merge: per split whose partial the last split reloads
};

struct CostEstimate {
  double step_us = 0;          // the megakernel step
  double per_op_us = 0;        // the conventional path (one launch per stage)
  double hbm_floor_us = 0;     // weight + K/V bytes at every SM's share of the bandwidth
  double stage_us[7] = {0};    // per opcode: mean instruction time (start to finish)
};

// Estimate a plan (static queues) for sequences at position `context`.
std::string estimate_plan(const PlanRequest &req, const Plan &p, const CostParams &c, int context,
                          CostEstimate *out);

// Split counts for a request whose S is not fixed: the fixed rule (one
// attention item per CTA), and the cost model's choice among candidate counts
// at the request's assumed context (*best_us: its estimate, may be NULL).
int rule_kv_splits(const PlanRequest &req);
int cost_kv_splits(const PlanRequest &req, const CostParams &c, double *best_us);
// Batched requests: whether the cost model expects the tensor-core matrix
// instructions to beat the CUDA-core ones (false at batch 1).
bool cost_prefers_tensor(const PlanRequest &req, const CostParams &c);

// Host simulation: `threads` CPU threads play the CTAs and run the queues
// for `steps` steps under random delays, with real atomic counters and
// version stamps on every buffer element; any read of a stale element, any
// double write or a deadlock (no progress for `timeout_ms`) is an error.
std::string simulate_plan(const PlanRequest &req, const Plan &p, int steps, uint64_t seed,
                          int timeout_ms);

}  // namespace mk
