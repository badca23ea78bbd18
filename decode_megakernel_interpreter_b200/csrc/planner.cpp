// Host planner for the decode interpreter.
//
// The schedule is built on the host ahead of time and reused for every step
// ("Hazy megakernel summary" page, section 四(二): each SM's instruction
// sequence is laid out in Python ahead of time and one schedule serves
// hundreds of forward passes).  Two placements are offered, after the
// "MegaKernel 日志" page's section on static and dynamic scheduling: static
// per-CTA queues (default), or one global queue in topological order that the
// CTAs claim with an atomic.  Work of a stage is split by bytes into at most
// one chunk per CTA and placed largest-first on the least-loaded CTA (a
// load-balancing refinement of the round-robin placement the "Mirage
// Persistent Kernel" article describes as its current policy).
#include "planner.h"

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdio>
#include <cstring>
#include <memory>
#include <mutex>
#include <numeric>
#include <random>
#include <thread>

namespace mk {

static bool pow2_in(int x, int lo, int hi) {
  return x >= lo && x <= hi && (x & (x - 1)) == 0;
}

static int down_kc(int F) { return F <= 2048 ? F : 2048; }
// Tensor-core plans split the down projection's K into pieces of 1024 when the
// piece count allows: one 128-row tile per instruction, so at hidden 2048 and
// ffn 8192 that is 128 instructions of 16 pages instead of 64 of 32 (64 of
// the 148 SMs busy), at the price of 1 + 8 instead of 1 + 4 loads per element
// in the tile's sum.  The CUDA-core layout (rows per page) keeps down_kc.
static int down_kc_tensor(int F) { return (F % 1024 == 0 && F / 1024 <= kMaxDownPieces) ? 1024 : down_kc(F); }
int down_pieces_max(const Shape &s) { return std::max(s.F / down_kc(s.F), s.F / down_kc_tensor(s.F)); }

std::string check_shape(const Shape &s, int B) {
  char buf[256];
  if (s.L < 1 || s.H < 1 || s.nq < 1 || s.nkv < 1 || s.d < 1 || s.F < 1 || s.V < 1)
    return "non-positive dimension";
  if (s.d != 64 && s.d != 128) return "head_dim must be 64 or 128";
  if (!pow2_in(s.H, 256, 4096)) return "hidden must be a power of two in [256, 4096]";
  if (!pow2_in(s.nq * s.d, 256, 4096)) return "n_q_heads*head_dim must be a power of two in [256, 4096]";
  if (s.nq % s.nkv) return "n_q_heads must be a multiple of n_kv_heads";
  if (s.nq / s.nkv > 8) return "more than 8 query heads per KV head";
  int Rh = kPageElems / s.H;
  if (s.d % Rh) return "head_dim must be a multiple of the rows per page";
  int kc = down_kc(s.F);
  if (s.F % 256 || (s.F > 2048 && s.F % 2048) || kPageElems % kc) {
    snprintf(buf, sizeof buf, "ffn=%d must be a multiple of 256 (and of 2048 above 2048)", s.F);
    return buf;
  }
  if (s.F % (Rh / 2)) return "ffn must be a multiple of half the rows per page";
  if (s.F / kc > kMaxDownPieces) return "ffn above 16384 is not implemented";
  if (B < 1 || B > kMaxBatch) return "batch must be in [1, 16]";
  return "";
}

namespace {

struct Chunk {
  int first, count;
};

std::vector<Chunk> split_even(int n, int parts) {
  std::vector<Chunk> v;
  if (n <= 0) return v;
  parts = std::max(1, std::min(parts, n));
  int base = n / parts, rem = n % parts, at = 0;
  for (int i = 0; i < parts; ++i) {
    int c = base + (i < rem ? 1 : 0);
    v.push_back({at, c});
    at += c;
  }
  return v;
}

struct Pending {
  Instr ins;
  int64_t bytes;
  int stage_key;  // layer * 8 + stage (global order key)
  int order;      // order inside the stage
};

}  // namespace

// The fixed rule: one attention item per CTA, but at least ~32 positions per
// split; when the sequences alone fill the CTAs (batched plans), still split
// long contexts up to ~4 items per CTA with >= 256 positions each, so that the
// longest sequence does not run on one CTA alone.
int rule_kv_splits(const PlanRequest &req) {
  const int items = req.B * req.s.nkv;
  int S = std::max(1, req.num_ctas / items);
  S = std::min(S, std::max(1, req.assumed_context / 32));
  // batched: about 3 splits per CTA's share of the (sequence, KV head) items
  // (batch 16, contexts U[512, 4096]: 3 splits 5383, 2: 5445, 4: 5483 us/step)
  if (req.B > 1) S = std::max(S, std::min(3 * req.num_ctas / items, req.assumed_context / 256));
  return std::max(1, std::min(S, 64));
}

// The cost model's choice: the candidate split count whose plan has the least
// estimated step with every sequence at the assumed context (a dynamic plan is
// estimated through its static twin).  Candidates keep >= ~32 positions per
// split; a tie keeps the smaller count.
int cost_kv_splits(const PlanRequest &req, const CostParams &c, double *best_us) {
  static const int kCand[] = {1, 2, 3, 4, 6, 8, 9, 12, 16, 18, 24, 32, 36, 48, 64};
  PlanRequest r = req;
  r.dynamic = false;
  const int max_s = std::max(1, std::min(64, req.assumed_context / 32));
  const int ctx = std::max(0, req.assumed_context - 1);
  int best = 0;
  double best_t = 0.0;
  for (int S : kCand) {
    if (S > max_s) break;
    r.S = S;
    Plan p;
    CostEstimate e;
    if (!build_plan(r, &p).empty() || !estimate_plan(r, p, c, ctx, &e).empty()) continue;
    if (best == 0 || e.step_us < best_t) {
      best = S;
      best_t = e.step_us;
    }
  }
  if (best == 0) return rule_kv_splits(req);
  if (best_us) *best_us = best_t;
  return best;
}

// The cost model's choice between the tensor-core and the CUDA-core matrix
// instructions of a batched request (each at its own split count when the
// request leaves that open).  A request for tensor-core QKV / O tiles keeps
// the tensor cores.
bool cost_prefers_tensor(const PlanRequest &req, const CostParams &c) {
  if (req.B <= 1) return false;
  if (req.tensor_qkv_o) return true;
  const int ctx = std::max(0, req.assumed_context - 1);
  double t[2] = {0.0, 0.0};
  for (int k = 0; k < 2; ++k) {
    PlanRequest r = req;
    r.dynamic = false;
    r.tensor = k == 0;
    Plan p;
    CostEstimate e;
    if (!build_plan(r, &p).empty() || !estimate_plan(r, p, c, ctx, &e).empty()) return k != 0;
    t[k] = e.step_us;
  }
  return t[0] <= t[1];
}

std::string build_plan(const PlanRequest &req, Plan *out) {
  const Shape &s = req.s;
  std::string err = check_shape(s, req.B);
  if (!err.empty()) return err;
  if (req.num_ctas < 1) return "num_ctas must be >= 1";
  Plan p;
  p.num_ctas = req.num_ctas;
  p.dynamic = req.dynamic;
  p.Rh = kPageElems / s.H;
  p.Ro = kPageElems / (s.nq * s.d);
  p.KCd = down_kc(s.F);
  p.Rd = kPageElems / p.KCd;  // rows per page of the CUDA-core down layout
  if (req.tensor) p.KCd = down_kc_tensor(s.F);
  p.ndp = s.F / p.KCd;
  const int G = s.nq / s.nkv;
  if (req.S > 0) {
    p.S = std::min(req.S, 256);
  } else if (req.S == kSplitsByCost) {
    p.S = cost_kv_splits(req, CostParams(), nullptr);
  } else {
    p.S = rule_kv_splits(req);
  }
  p.P_qkv = (s.nq + 2 * s.nkv) * s.d / p.Rh;
  p.P_o = s.H / p.Ro;
  p.P_gu = s.F / (p.Rh / 2);
  p.P_dp = s.H / p.Rd;
  p.P_lm = (s.V + p.Rh - 1) / p.Rh;
  p.ctr_per_layer = 4 + p.ndp;
  unsigned next = (unsigned)(s.L * p.ctr_per_layer);
  p.attn_ticket0 = next;
  next += (unsigned)(s.L * req.B * s.nkv);
  p.arg_ticket0 = next;
  next += (unsigned)req.B;
  p.exit_ticket = next++;
  p.dyn_head = next++;
  p.ev_tail = next++;
  // tensor cores: one ticket per (layer, 128-row tile) of the down projection
  p.dn_ticket0 = next;
  if (req.tensor) next += (unsigned)(s.L * (s.H / 128));
  p.n_counters = (int)next;

  const int n = req.num_ctas;
  const int parts = req.dynamic ? n * std::max(1, req.dyn_chunks_per_cta) : n;
  std::vector<Pending> all;
  auto mk_instr = [](Op op, int layer) {
    Instr I;
    memset(&I, 0, sizeof I);
    I.op = op;
    I.layer = (uint16_t)layer;
    I.wait_ctr = kNoCounter;
    I.sig_ctr = kNoCounter;
    return I;
  };
  std::vector<int> n_down(s.L, 0), n_qkv(s.L, 0), n_o(s.L, 0);
  p.tensor = req.tensor;
  p.tensor_qkv_o = req.tensor && req.tensor_qkv_o;
  p.gu_rows_unit = p.tensor ? 64 : p.Rh / 2;
  p.dn_rows_unit = p.tensor ? 128 : p.Rd;
  const int gu_units = p.tensor ? s.F / 64 : p.P_gu;
  const int dn_units = p.tensor ? s.H / 128 : p.P_dp;
  const int64_t gu_unit_bytes = p.tensor ? (int64_t)(s.H / 64) * kPageBytes : kPageBytes;
  // QKV: pages, or 128-row tiles of [q; k; v] (128 / Rh pages of the batch-1
  // page numbering each); O projection: pages, or 128-row tiles
  const int qdim = s.nq * s.d, kvdim = s.nkv * s.d;
  const int qkv_units = p.tensor_qkv_o ? (qdim + 2 * kvdim) / 128 : p.P_qkv;
  const int o_units = p.tensor_qkv_o ? s.H / 128 : p.P_o;
  const int64_t qkv_unit_bytes = p.tensor_qkv_o ? (int64_t)(s.H / 64) * kPageBytes : kPageBytes;
  const int64_t o_unit_bytes = p.tensor_qkv_o ? (int64_t)(qdim / 64) * kPageBytes : kPageBytes;
  p.qkv_pages_unit = p.tensor_qkv_o ? 128 / p.Rh : 1;
  p.o_rows_unit = p.tensor_qkv_o ? 128 : p.Ro;
  const int64_t dn_unit_bytes = p.tensor ? (int64_t)(p.KCd / 64) * kPageBytes : kPageBytes;
  for (int l = 0; l < s.L; ++l) {
    // fused RMSNorm + QKV + RoPE
    auto cq = split_even(qkv_units, parts);
    n_qkv[l] = (int)cq.size();
    for (size_t i = 0; i < cq.size(); ++i) {
      Instr I = mk_instr(OP_QKV, l);
      I.a = cq[i].first;
      I.b = cq[i].count;
      if (l > 0) {
        I.wait_ctr = p.ctr_dn(l - 1);
        I.wait_cnt = n_down[l - 1];
      }
      I.sig_ctr = p.ctr_qkv(l);
      I.sig_n = 1;
      all.push_back({I, (int64_t)cq[i].count * qkv_unit_bytes, l * 8 + ST_QKV, (int)i});
    }
    // split-KV attention
    int ord = 0;
    for (int b = 0; b < req.B; ++b)
      for (int g = 0; g < s.nkv; ++g)
        for (int sp = 0; sp < p.S; ++sp) {
          Instr I = mk_instr(OP_ATTN, l);
          I.a = g;
          I.b = sp;
          I.c = b;
          I.wait_ctr = p.ctr_qkv(l);
          I.wait_cnt = n_qkv[l];
          I.sig_ctr = p.ctr_attn(l);  // signalled by the split that merges
          I.sig_n = 1;
          int64_t bytes = (int64_t)req.assumed_context / p.S * s.d * 4 + 4096;
          all.push_back({I, bytes, l * 8 + ST_ATTN, ord++});
        }
    // O projection + residual
    auto co = split_even(o_units, parts);
    n_o[l] = (int)co.size();
    for (size_t i = 0; i < co.size(); ++i) {
      Instr I = mk_instr(OP_OPROJ, l);
      I.a = co[i].first;
      I.b = co[i].count;
      I.wait_ctr = p.ctr_attn(l);
      I.wait_cnt = req.B * s.nkv;
      I.sig_ctr = p.ctr_o(l);
      I.sig_n = 1;
      all.push_back({I, (int64_t)co[i].count * o_unit_bytes, l * 8 + ST_OPROJ, (int)i});
    }
    // RMSNorm + gate/up + SiLU; signals the down-projection K pieces it feeds
    // (units: pages of R/2 gate + R/2 up rows, or 128-row tensor-core tiles
    // of 64 gate + 64 up rows)
    auto cg = split_even(gu_units, parts);
    std::vector<int> gu_per_piece(p.ndp, 0);
    const int half = p.gu_rows_unit;
    for (size_t i = 0; i < cg.size(); ++i) {
      Instr I = mk_instr(OP_GATEUP, l);
      I.a = cg[i].first;
      I.b = cg[i].count;
      I.c = (uint32_t)i;  // its index in the layer (tensor parallelism: its slice of x_mid)
      I.wait_ctr = p.ctr_o(l);
      I.wait_cnt = n_o[l];
      int row0 = cg[i].first * half, row1 = (cg[i].first + cg[i].count) * half;  // act rows
      int k0 = row0 / p.KCd, k1 = (row1 - 1) / p.KCd;
      I.sig_ctr = p.ctr_gu(l, k0);
      I.sig_n = (uint16_t)(k1 - k0 + 1);
      for (int k = k0; k <= k1; ++k) gu_per_piece[k]++;
      all.push_back({I, (int64_t)cg[i].count * gu_unit_bytes, l * 8 + ST_GATEUP, (int)i});
    }
    p.n_gu = (int)cg.size();
    // down projection, K-split into pieces; each piece waits only for the
    // gate/up instructions that produce its K range
    int total = p.ndp * p.P_dp;
    int ord2 = 0;
    for (int k = 0; k < p.ndp; ++k) {
      int ck = (int)((int64_t)parts * (k + 1) / p.ndp - (int64_t)parts * k / p.ndp);
      // tensor cores: one 128-row tile per instruction (the last piece of a
      // tile to finish sums the tile's pieces: one signal per tile)
      auto cd = split_even(dn_units, p.tensor ? dn_units : std::max(1, ck));
      for (auto &c : cd) {
        Instr I = mk_instr(OP_DOWN, l);
        I.a = c.first;
        I.b = c.count;
        I.c = k;
        I.wait_ctr = p.ctr_gu(l, k);
        I.wait_cnt = gu_per_piece[k];
        I.sig_ctr = p.ctr_dn(l);
        I.sig_n = 1;
        if (!p.tensor || k == 0) n_down[l]++;
        all.push_back({I, (int64_t)c.count * dn_unit_bytes, l * 8 + ST_DOWN, ord2++});
      }
    }
    (void)total;
  }
  // final RMSNorm + LM head + argmax (units: pages of R rows, or 128-row
  // blocks of H / 64 pages on the tensor-core path)
  const int lm_units = p.tensor ? (s.V + 127) / 128 : p.P_lm;
  const int64_t lm_unit_bytes = p.tensor ? (int64_t)(s.H / 64) * kPageBytes : kPageBytes;
  auto cl = split_even(lm_units, parts);
  p.n_lm = (int)cl.size();
  for (size_t i = 0; i < cl.size(); ++i) {
    Instr I = mk_instr(OP_LMHEAD, s.L);
    I.a = cl[i].first;
    I.b = cl[i].count;
    I.c = (uint32_t)i;
    I.wait_ctr = p.ctr_dn(s.L - 1);
    I.wait_cnt = n_down[s.L - 1];
    all.push_back({I, (int64_t)cl[i].count * lm_unit_bytes, s.L * 8 + ST_QKV + 0, (int)i});
  }
  // the LM head sorts after every layer
  for (auto &x : all)
    if (x.ins.op == OP_LMHEAD) x.stage_key = s.L * 8;

  std::stable_sort(all.begin(), all.end(), [](const Pending &a, const Pending &b) {
    if (a.stage_key != b.stage_key) return a.stage_key < b.stage_key;
    return a.order < b.order;
  });
  if (all.size() > 65535) return "too many instructions for one step";
  for (size_t i = 0; i < all.size(); ++i) all[i].ins.seq = (uint16_t)i;
  for (auto &x : all) {
    if (x.ins.op >= OP_QKV && x.ins.op <= OP_LMHEAD && x.ins.op != OP_ATTN)
      p.weight_bytes += (int64_t)x.ins.b * (x.ins.op == OP_LMHEAD   ? lm_unit_bytes
                                           : x.ins.op == OP_GATEUP ? gu_unit_bytes
                                           : x.ins.op == OP_DOWN   ? dn_unit_bytes
                                           : x.ins.op == OP_QKV    ? qkv_unit_bytes
                                           : x.ins.op == OP_OPROJ  ? o_unit_bytes
                                                                   : (int64_t)kPageBytes);
  }
  // the last LM page (or block) may be partial
  {
    int64_t full = (int64_t)lm_units * lm_unit_bytes, real = (int64_t)s.V * s.H * 2;
    p.weight_bytes -= full - real;
  }

  if (req.drop_producer) {
    // test hook: remove the first QKV instruction of layer 0 but keep the
    // counter targets, so attention in layer 0 can never start
    for (size_t i = 0; i < all.size(); ++i)
      if (all[i].ins.op == OP_QKV && all[i].ins.layer == 0) {
        all[i].ins.op = OP_NOP;
        all[i].ins.sig_ctr = kNoCounter;
        all[i].ins.sig_n = 0;
        all[i].ins.wait_ctr = kNoCounter;
        break;
      }
  }

  if (req.dynamic) {
    for (auto &x : all) p.instrs.push_back(x.ins);
    p.q_off.assign(n, 0);
    p.q_len.assign(n, 0);
    if (req.events) {
      // event tables: dependents of every counter, grouped by counter in
      // topological order, and the instructions that wait on nothing
      p.events = true;
      p.ev_off.assign(p.n_counters + 1, 0);
      p.ev_cnt.assign(p.n_counters, 0);
      for (const Instr &I : p.instrs) {
        if (I.op == OP_NOP) continue;
        if (I.wait_ctr == kNoCounter) continue;
        if (I.wait_ctr >= (unsigned)p.n_counters) return "event plan: bad counter";
        if (p.ev_cnt[I.wait_ctr] != 0 && p.ev_cnt[I.wait_ctr] != I.wait_cnt)
          return "event plan: dependents of one counter wait for different counts";
        p.ev_cnt[I.wait_ctr] = I.wait_cnt;
        p.ev_off[I.wait_ctr + 1]++;
      }
      for (int c = 0; c < p.n_counters; ++c) p.ev_off[c + 1] += p.ev_off[c];
      p.ev_list.assign(p.ev_off[p.n_counters], 0);
      std::vector<int> fill(p.ev_off.begin(), p.ev_off.end() - 1);
      for (int k = 0; k < (int)p.instrs.size(); ++k) {
        const Instr &I = p.instrs[k];
        if (I.op == OP_NOP) continue;
        if (I.wait_ctr == kNoCounter) p.ev_init.push_back(k);
        else p.ev_list[fill[I.wait_ctr]++] = k;
      }
    }
  } else {
    std::vector<std::vector<Instr>> q(n);
    std::vector<int64_t> load(n, 0);
    std::vector<int> idx(n);
    size_t i = 0;
    while (i < all.size()) {
      size_t j = i;
      while (j < all.size() && all[j].stage_key == all[i].stage_key) ++j;
      // this stage: largest chunk onto the least-loaded CTA, one chunk per CTA per round
      std::vector<size_t> items(j - i);
      std::iota(items.begin(), items.end(), i);
      std::stable_sort(items.begin(), items.end(),
                       [&](size_t a, size_t b) { return all[a].bytes > all[b].bytes; });
      size_t at = 0;
      while (at < items.size()) {
        std::iota(idx.begin(), idx.end(), 0);
        std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return load[a] < load[b]; });
        for (int c = 0; c < n && at < items.size(); ++c, ++at) {
          const Pending &pp = all[items[at]];
          q[idx[c]].push_back(pp.ins);
          load[idx[c]] += pp.bytes;
        }
      }
      i = j;
    }
    for (int c = 0; c < n; ++c) {
      std::sort(q[c].begin(), q[c].end(), [](const Instr &a, const Instr &b) { return a.seq < b.seq; });
      p.q_off.push_back((int)p.instrs.size());
      p.q_len.push_back((int)q[c].size());
      for (auto &I : q[c]) p.instrs.push_back(I);
    }
  }
  *out = std::move(p);
  return "";
}

// ------------------------------------------------------------------ validation

namespace {

// Element sets read and written by one instruction, as (buffer id, begin,
// end) ranges over flattened per-step buffers.
enum Buf { B_QKV, B_PART, B_O, B_XRES, B_ACT, B_DPART, B_ARG, B_XIN, B_NBUF };

struct Range {
  int buf;
  int64_t lo, hi;
};

struct Layout {
  int64_t base[B_NBUF];
  int64_t size[B_NBUF];
};

Layout make_layout(const PlanRequest &req, const Plan &p) {
  const Shape &s = req.s;
  Layout L;
  L.size[B_QKV] = (int64_t)s.L * p.P_qkv;
  L.size[B_PART] = (int64_t)s.L * req.B * s.nkv * p.S;
  L.size[B_O] = (int64_t)s.L * req.B * s.nkv;
  L.size[B_XRES] = (int64_t)s.L * s.H;
  L.size[B_ACT] = (int64_t)s.L * s.F;
  L.size[B_DPART] = (int64_t)s.L * p.ndp * s.H;
  L.size[B_ARG] = p.n_lm;
  L.size[B_XIN] = p.tensor ? (int64_t)s.L * s.H : 0;  // tensor cores: x_in of the next layer, summed once
  int64_t at = 0;
  for (int b = 0; b < B_NBUF; ++b) {
    L.base[b] = at;
    at += L.size[b];
  }
  return L;
}

void layer_input_reads(const PlanRequest &req, const Plan &p, int l, int64_t r0, int64_t r1,
                       std::vector<Range> &rd) {
  if (l <= 0) return;  // embedding rows
  const Shape &s = req.s;
  if (p.tensor) {  // summed once by the down tiles' last pieces
    rd.push_back({B_XIN, (int64_t)(l - 1) * s.H + r0, (int64_t)(l - 1) * s.H + r1});
    return;
  }
  rd.push_back({B_XRES, (int64_t)(l - 1) * s.H + r0, (int64_t)(l - 1) * s.H + r1});
  for (int k = 0; k < p.ndp; ++k)
    rd.push_back({B_DPART, ((int64_t)(l - 1) * p.ndp + k) * s.H + r0,
                  ((int64_t)(l - 1) * p.ndp + k) * s.H + r1});
}

// reads before the instruction's own work, the writes, and (attention/LM)
// the reads of the merging instance
void rw_sets(const PlanRequest &req, const Plan &p, const Instr &I, std::vector<Range> &rd,
             std::vector<Range> &wr, std::vector<Range> &merge_rd, std::vector<Range> &merge_wr) {
  const Shape &s = req.s;
  const int G = s.nq / s.nkv;
  const int l = I.layer;
  switch (I.op) {
    case OP_QKV:
      layer_input_reads(req, p, l, 0, s.H, rd);
      wr.push_back({B_QKV, (int64_t)l * p.P_qkv + (int64_t)I.a * p.qkv_pages_unit,
                    (int64_t)l * p.P_qkv + (int64_t)(I.a + I.b) * p.qkv_pages_unit});
      break;
    case OP_ATTN: {
      const int pph = s.d / p.Rh;  // pages per head
      int g = I.a;
      int64_t q0 = (int64_t)l * p.P_qkv;
      rd.push_back({B_QKV, q0 + (int64_t)g * G * pph, q0 + (int64_t)(g + 1) * G * pph});
      rd.push_back({B_QKV, q0 + (int64_t)(s.nq + g) * pph, q0 + (int64_t)(s.nq + g + 1) * pph});
      rd.push_back({B_QKV, q0 + (int64_t)(s.nq + s.nkv + g) * pph,
                    q0 + (int64_t)(s.nq + s.nkv + g + 1) * pph});
      int64_t part0 = (((int64_t)l * req.B + I.c) * s.nkv + g) * p.S;
      wr.push_back({B_PART, part0 + I.b, part0 + I.b + 1});
      merge_rd.push_back({B_PART, part0, part0 + p.S});
      int64_t o = ((int64_t)l * req.B + I.c) * s.nkv + g;
      merge_wr.push_back({B_O, o, o + 1});
      break;
    }
    case OP_OPROJ: {
      rd.push_back({B_O, (int64_t)l * req.B * s.nkv, (int64_t)(l + 1) * req.B * s.nkv});
      int64_t r0 = (int64_t)I.a * p.o_rows_unit, r1 = (int64_t)(I.a + I.b) * p.o_rows_unit;
      layer_input_reads(req, p, l, r0, r1, rd);
      wr.push_back({B_XRES, (int64_t)l * s.H + r0, (int64_t)l * s.H + r1});
      break;
    }
    case OP_GATEUP: {
      rd.push_back({B_XRES, (int64_t)l * s.H, (int64_t)(l + 1) * s.H});
      int half = p.gu_rows_unit;
      wr.push_back({B_ACT, (int64_t)l * s.F + (int64_t)I.a * half,
                    (int64_t)l * s.F + (int64_t)(I.a + I.b) * half});
      break;
    }
    case OP_DOWN: {
      rd.push_back({B_ACT, (int64_t)l * s.F + (int64_t)I.c * p.KCd,
                    (int64_t)l * s.F + (int64_t)(I.c + 1) * p.KCd});
      int64_t base = ((int64_t)l * p.ndp + I.c) * s.H;
      const int64_t r0 = (int64_t)I.a * p.dn_rows_unit, r1 = (int64_t)(I.a + I.b) * p.dn_rows_unit;
      wr.push_back({B_DPART, base + r0, base + r1});
      if (p.tensor) {
        // the tile's last piece: x_mid + every piece of the tile's rows -> x_in(l + 1)
        merge_rd.push_back({B_XRES, (int64_t)l * s.H + r0, (int64_t)l * s.H + r1});
        for (int k = 0; k < p.ndp; ++k)
          merge_rd.push_back({B_DPART, ((int64_t)l * p.ndp + k) * s.H + r0, ((int64_t)l * p.ndp + k) * s.H + r1});
        merge_wr.push_back({B_XIN, (int64_t)l * s.H + r0, (int64_t)l * s.H + r1});
      }
      break;
    }
    case OP_LMHEAD:
      layer_input_reads(req, p, s.L, 0, s.H, rd);
      wr.push_back({B_ARG, I.c, I.c + 1});
      merge_rd.push_back({B_ARG, 0, p.n_lm});
      break;
    default:
      break;
  }
}

std::vector<const Instr *> global_order(const Plan &p) {
  std::vector<const Instr *> v;
  for (auto &I : p.instrs) v.push_back(&I);
  std::sort(v.begin(), v.end(), [](const Instr *a, const Instr *b) { return a->seq < b->seq; });
  return v;
}

}  // namespace

std::string validate_plan(const PlanRequest &req, const Plan &p) {
  char buf[512];
  const Shape &s = req.s;
  auto order = global_order(p);
  for (size_t i = 0; i < order.size(); ++i)
    if (order[i]->seq != i) return "instruction sequence numbers are not 0..n-1";
  // queues follow the global order
  if (!p.dynamic) {
    if ((int)p.q_off.size() != p.num_ctas) return "queue table size";
    size_t total = 0;
    for (int c = 0; c < p.num_ctas; ++c) {
      for (int i = 1; i < p.q_len[c]; ++i)
        if (p.instrs[p.q_off[c] + i].seq <= p.instrs[p.q_off[c] + i - 1].seq) {
          snprintf(buf, sizeof buf, "queue of CTA %d is not a subsequence of the global order", c);
          return buf;
        }
      total += p.q_len[c];
    }
    if (total != p.instrs.size()) return "queues do not cover every instruction exactly once";
  }
  // producers of every counter
  std::vector<int> n_prod(p.n_counters, 0), last_prod(p.n_counters, -1);
  for (auto *I : order) {
    if (I->sig_ctr == kNoCounter) continue;
    for (int k = 0; k < I->sig_n; ++k) {
      unsigned c = I->sig_ctr + k;
      if (c >= (unsigned)p.n_counters) return "signal counter out of range";
      if (I->op == OP_ATTN) {
        // one signal per (sequence, kv head): counted once, by split 0's slot
        if (I->b == 0) n_prod[c]++;
      } else if (I->op == OP_DOWN && p.tensor) {
        // one signal per tile (the last of its pieces): counted by piece 0's slot
        if (I->c == 0) n_prod[c]++;
      } else {
        n_prod[c]++;
      }
      last_prod[c] = std::max(last_prod[c], (int)I->seq);
    }
  }
  for (auto *I : order) {
    if (I->wait_ctr == kNoCounter) continue;
    unsigned c = I->wait_ctr;
    if (c >= (unsigned)p.n_counters) return "wait counter out of range";
    if (n_prod[c] != (int)I->wait_cnt && !req.drop_producer) {
      snprintf(buf, sizeof buf, "instruction %d (op %d layer %d) waits for %u signals of counter %u but %d producers exist",
               I->seq, I->op, I->layer, I->wait_cnt, c, n_prod[c]);
      return buf;
    }
    if (last_prod[c] >= (int)I->seq) {
      snprintf(buf, sizeof buf, "instruction %d waits on a producer that comes later (%d)", I->seq, last_prod[c]);
      return buf;
    }
  }
  // every element written exactly once per step; every read covered by a
  // producer that the reader (transitively) waits for is checked by the
  // simulation, here we check coverage
  Layout L = make_layout(req, p);
  std::vector<int> wcount(L.base[B_NBUF - 1] + L.size[B_NBUF - 1], 0);
  for (auto *I : order) {
    std::vector<Range> rd, wr, mrd, mwr;
    rw_sets(req, p, *I, rd, wr, mrd, mwr);
    if ((I->op == OP_ATTN && I->b == 0) || (I->op == OP_DOWN && p.tensor && I->c == 0))
      wr.insert(wr.end(), mwr.begin(), mwr.end());
    for (auto &r : wr)
      for (int64_t e = r.lo; e < r.hi; ++e) wcount[L.base[r.buf] + e]++;
  }
  if (!req.drop_producer)
    for (int b = 0; b < B_NBUF; ++b)
      for (int64_t e = 0; e < L.size[b]; ++e)
        if (wcount[L.base[b] + e] != 1) {
          snprintf(buf, sizeof buf, "buffer %d element %lld written %d times per step", b, (long long)e,
                   wcount[L.base[b] + e]);
          return buf;
        }
  (void)s;
  return "";
}

// ------------------------------------------------------------------ simulation

std::string simulate_plan(const PlanRequest &req, const Plan &p, int steps, uint64_t seed,
                          int timeout_ms) {
  Layout L = make_layout(req, p);
  const int64_t n_el = L.base[B_NBUF - 1] + L.size[B_NBUF - 1];
  std::unique_ptr<std::atomic<uint32_t>[]> stamp(new std::atomic<uint32_t>[n_el]);
  for (int64_t i = 0; i < n_el; ++i) stamp[i].store(0);
  std::unique_ptr<std::atomic<uint32_t>[]> ctr(new std::atomic<uint32_t>[p.n_counters]);
  for (int i = 0; i < p.n_counters; ++i) ctr[i].store(0);
  std::atomic<bool> failed{false};
  std::mutex err_mu;
  std::string err;
  auto fail = [&](const std::string &m) {
    std::lock_guard<std::mutex> g(err_mu);
    if (!failed.exchange(true)) err = m;
  };

  // event-driven plans: the ready queue (instruction index and the step
  // that appended it, per slot)
  const int n_init = (int)p.ev_init.size();
  const int n_ev = n_init + (int)p.ev_list.size();
  std::unique_ptr<std::atomic<uint32_t>[]> ready_step(new std::atomic<uint32_t>[n_ev > 0 ? n_ev : 1]);
  std::unique_ptr<std::atomic<int>[]> ready_id(new std::atomic<int>[n_ev > 0 ? n_ev : 1]);
  for (int i = 0; i < n_ev; ++i) {
    ready_step[i].store(0);
    ready_id[i].store(-1);
  }
  for (uint32_t epoch = 1; epoch <= (uint32_t)steps && !failed; ++epoch) {
    std::atomic<uint32_t> dyn_next{0};
    std::atomic<uint32_t> ev_tail{(uint32_t)n_init};
    auto run_cta = [&](int cta) {
      std::mt19937_64 rng(seed * 1000003ull + cta * 7919ull + epoch);
      std::uniform_int_distribution<int> jitter(0, 9);
      auto pause = [&]() {
        int j = jitter(rng);
        if (j < 5) std::this_thread::yield();
        else if (j == 9) std::this_thread::sleep_for(std::chrono::microseconds(50));
      };
      auto check_reads = [&](const std::vector<Range> &rd, const Instr &I) {
        for (auto &r : rd)
          for (int64_t e = r.lo; e < r.hi; ++e)
            if (stamp[L.base[r.buf] + e].load(std::memory_order_relaxed) != epoch) {
              char b[256];
              snprintf(b, sizeof b, "step %u: instruction %d (op %d layer %d) read a stale element of buffer %d",
                       epoch, I.seq, I.op, I.layer, r.buf);
              fail(b);
              return false;
            }
        return true;
      };
      auto do_writes = [&](const std::vector<Range> &wr, const Instr &I) {
        for (auto &r : wr)
          for (int64_t e = r.lo; e < r.hi; ++e) {
            uint32_t old = stamp[L.base[r.buf] + e].exchange(epoch, std::memory_order_relaxed);
            if (old == epoch) {
              char b[256];
              snprintf(b, sizeof b, "step %u: instruction %d wrote buffer %d element twice", epoch, I.seq, r.buf);
              fail(b);
            }
          }
      };
      int qi = 0;
      while (!failed) {
        const Instr *I;
        if (p.events) {
          // the next ready instruction: the initial ones, then the slots the
          // producers' events append (wait until this slot is filled)
          const uint32_t k = dyn_next.fetch_add(1);
          if (k >= (uint32_t)n_ev) break;
          int id;
          if ((int)k < n_init) {
            id = p.ev_init[k];
          } else {
            auto t0 = std::chrono::steady_clock::now();
            while (ready_step[k].load(std::memory_order_acquire) != epoch) {
              if (failed) return;
              std::this_thread::yield();
              if (std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(timeout_ms)) {
                char b[256];
                snprintf(b, sizeof b, "step %u: ready-queue slot %u never filled", epoch, k);
                fail(b);
                return;
              }
            }
            id = ready_id[k].load(std::memory_order_relaxed);
          }
          I = &p.instrs[id];
          if (I->wait_ctr != kNoCounter &&
              ctr[I->wait_ctr].load(std::memory_order_acquire) < (uint64_t)epoch * I->wait_cnt) {
            char b[256];
            snprintf(b, sizeof b, "step %u: instruction %d became ready before its producers finished", epoch, I->seq);
            fail(b);
            return;
          }
        } else if (p.dynamic) {
          uint32_t k = dyn_next.fetch_add(1);
          if (k >= p.instrs.size()) break;
          I = &p.instrs[k];
        } else {
          if (qi >= p.q_len[cta]) break;
          I = &p.instrs[p.q_off[cta] + qi++];
        }
        if (I->op == OP_NOP) continue;
        std::vector<Range> rd, wr, mrd, mwr;
        rw_sets(req, p, *I, rd, wr, mrd, mwr);
        // the kernel starts every instruction at once and loads its inputs
        // before it knows its producers are done, telling this step's words
        // from stale ones by a 2-bit step tag: that is sound only if a word
        // it can meet was written this step or the step before (never two
        // or more steps back, whose tag could alias)
        for (auto &r : rd)
          for (int64_t e = r.lo; e < r.hi; ++e) {
            const uint32_t st = stamp[L.base[r.buf] + e].load(std::memory_order_relaxed);
            if (st != epoch && st + 1 != epoch) {
              char b[256];
              snprintf(b, sizeof b, "step %u: instruction %d (op %d layer %d) could meet an element of buffer %d "
                       "last written at step %u (its tag would alias)", epoch, I->seq, I->op, I->layer, r.buf, st);
              fail(b);
              return;
            }
          }
        if (I->wait_ctr != kNoCounter) {
          uint64_t target = (uint64_t)epoch * I->wait_cnt;
          auto t0 = std::chrono::steady_clock::now();
          while (ctr[I->wait_ctr].load(std::memory_order_acquire) < target) {
            if (failed) return;
            std::this_thread::yield();
            if (std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(timeout_ms)) {
              char b[256];
              snprintf(b, sizeof b, "step %u: instruction %d (op %d layer %d) waited too long on counter %u",
                       epoch, I->seq, I->op, I->layer, I->wait_ctr);
              fail(b);
              return;
            }
          }
        }
        pause();
        if (!check_reads(rd, *I)) return;
        pause();
        do_writes(wr, *I);
        bool signal = true;
        if (I->op == OP_ATTN || I->op == OP_LMHEAD || (I->op == OP_DOWN && p.tensor)) {
          // tickets: the last split (attention), LM-head instruction or piece
          // of a down tile (tensor cores) merges
          unsigned t = I->op == OP_ATTN   ? p.attn_ticket0 + (I->layer * req.B + I->c) * req.s.nkv + I->a
                       : I->op == OP_DOWN ? p.dn_ticket0 + (unsigned)(I->layer * (req.s.H / 128) + I->a)
                                          : p.arg_ticket0;
          uint32_t per = I->op == OP_ATTN ? (uint32_t)p.S : I->op == OP_DOWN ? (uint32_t)p.ndp : (uint32_t)p.n_lm;
          uint32_t old = ctr[t].fetch_add(1, std::memory_order_acq_rel);
          signal = false;
          if (old == epoch * per - 1) {  // the last one merges
            if (!check_reads(mrd, *I)) return;
            do_writes(mwr, *I);
            signal = I->op != OP_LMHEAD;
          }
        }
        if (signal && I->sig_ctr != kNoCounter)
          for (int k = 0; k < I->sig_n; ++k) {
            const unsigned c = I->sig_ctr + k;
            const uint32_t old = ctr[c].fetch_add(1, std::memory_order_acq_rel);
            if (p.events && p.ev_cnt[c] != 0 && old + 1 == epoch * p.ev_cnt[c]) {
              // the last producer: its dependents become ready
              const int n = p.ev_off[c + 1] - p.ev_off[c];
              const uint32_t pos = ev_tail.fetch_add((uint32_t)n);
              for (int j = 0; j < n; ++j) {
                if (pos + j >= (uint32_t)n_ev) {
                  fail("ready queue overflow");
                  return;
                }
                ready_id[pos + j].store(p.ev_list[p.ev_off[c] + j], std::memory_order_relaxed);
                ready_step[pos + j].store(epoch, std::memory_order_release);
              }
            }
          }
      }
    };
    std::vector<std::thread> th;
    for (int c = 0; c < p.num_ctas; ++c) th.emplace_back(run_cta, c);
    for (auto &t : th) t.join();
    if (failed) break;
    for (int b = 0; b < B_NBUF; ++b)
      for (int64_t e = 0; e < L.size[b]; ++e)
        if (stamp[L.base[b] + e].load() != epoch) {
          char bb[256];
          snprintf(bb, sizeof bb, "step %u: buffer %d element %lld never written", epoch, b, (long long)e);
          fail(bb);
          break;
        }
  }
  return failed ? err : "";
}

}  // namespace mk

// ------------------------------------------------------------------ cost model

namespace mk {

namespace {

// weight pages one instruction streams (tensor-core units are whole tiles of
// 64-column pages), and how many of its pages are K/V (attention)
int instr_pages(const PlanRequest &req, const Plan &p, const Instr &I, int context, bool *kv) {
  const Shape &s = req.s;
  *kv = false;
  switch (I.op) {
    case OP_QKV: return (int)I.b * (p.tensor_qkv_o ? s.H / 64 : 1);
    case OP_OPROJ: return (int)I.b * (p.tensor_qkv_o ? s.nq * s.d / 64 : 1);
    case OP_GATEUP: return (int)I.b * (p.tensor ? s.H / 64 : 1);
    case OP_DOWN: return (int)I.b * (p.tensor ? p.KCd / 64 : 1);
    case OP_LMHEAD: return (int)I.b * (p.tensor ? s.H / 64 : 1);
    case OP_ATTN: {
      *kv = true;
      const int n = context + 1, chunk = (n + p.S - 1) / p.S;
      const int start = std::min(n, (int)I.b * chunk), end = std::min(n, start + chunk);
      const int cached = std::max(0, std::min(end, context) - start);
      const int ppp = kPageBytes / (4 * s.d);
      return (cached + ppp - 1) / ppp;
    }
    default: return 0;
  }
}

// compute time of one weight page of an instruction
double page_time(const PlanRequest &req, const Plan &p, const Instr &I, const CostParams &c) {
  if (req.B == 1) return c.page_us;
  const bool tc = (I.op == OP_GATEUP || I.op == OP_DOWN || I.op == OP_LMHEAD) ? p.tensor
                  : (I.op == OP_QKV || I.op == OP_OPROJ)                     ? p.tensor_qkv_o
                                                                             : false;
  return tc ? c.tc_page_us : c.cc_page_us_seq * req.B;
}

}  // namespace

std::string estimate_plan(const PlanRequest &req, const Plan &p, const CostParams &c, int context,
                          CostEstimate *out) {
  if (p.dynamic) return "the cost model replays static queues";
  if (context < 0 || c.sm_gbs <= 0 || c.ring_pages < 1) return "bad cost parameters";
  if ((int)p.q_off.size() != p.num_ctas || (int)p.q_len.size() != p.num_ctas || p.num_ctas < 1) return "not a plan";
  const Shape &s = req.s;
  const int n = p.num_ctas;
  const double t_hbm = kPageBytes / (c.sm_gbs * 1e3);  // us per 16 KiB page at one SM's bandwidth
  std::vector<const Instr *> order(p.instrs.size());
  std::vector<int> cta_of(p.instrs.size());
  for (int q = 0; q < n; ++q)
    for (int i = 0; i < p.q_len[q]; ++i) {
      const Instr &I = p.instrs[p.q_off[q] + i];
      order[I.seq] = &I;
      cta_of[I.seq] = q;
    }
  // per-CTA state: compute warps free at, loader's last arrival, and the
  // consumption times of the last ring_pages pages (their slots free then)
  std::vector<double> t_cta(n, 0.0), arrive(n, 0.0);
  std::vector<std::vector<double>> ring(n);
  std::vector<size_t> ring_head(n, 0);
  std::vector<double> ctr_done(p.n_counters, 0.0);
  // ticketed attention merges: latest split finish per (layer, sequence, kv head)
  std::vector<double> group_max((size_t)s.L * req.B * s.nkv, 0.0);
  double sum_t[7] = {0}, cnt_t[7] = {0}, end = 0.0, hbm_bytes = 0.0;
  for (const Instr *Ip : order) {
    const Instr &I = *Ip;
    const int q = cta_of[I.seq];
    if (I.op == OP_NOP) continue;
    double dep = 0.0;
    if (I.wait_ctr != kNoCounter) dep = ctr_done[I.wait_ctr] + c.exchange_us;
    const double start = std::max(t_cta[q], dep);
    bool kv = false;
    const int np = instr_pages(req, p, I, context, &kv);
    const double pt = kv ? c.attn_page_us : page_time(req, p, I, c);
    double done = start;
    for (int k = 0; k < np; ++k) {
      // the loader issues a page once its ring slot is free, one SM's
      // bandwidth apart
      std::vector<double> &rg = ring[q];
      const double slot_free = rg.size() < (size_t)c.ring_pages ? 0.0 : rg[ring_head[q]];
      arrive[q] = std::max(arrive[q], slot_free) + t_hbm;
      done = std::max(done, arrive[q]) + pt;
      if (rg.size() < (size_t)c.ring_pages) {
        rg.push_back(done);
      } else {
        rg[ring_head[q]] = done;
        ring_head[q] = (ring_head[q] + 1) % rg.size();
      }
    }
    hbm_bytes += (double)np * kPageBytes;
    double finish = done + (I.op == OP_ATTN ? c.attn_fixed_us : c.instr_us);
    t_cta[q] = finish;
    sum_t[I.op] += finish - start;
    cnt_t[I.op] += 1;
    // producers' completion
    if (I.op == OP_ATTN) {
      const size_t gi = ((size_t)I.layer * req.B + I.c) * s.nkv + I.a;
      group_max[gi] = std::max(group_max[gi], finish);
      // the last split of the group merges: the ticket and the reload of the
      // partials are two exchanges
      const double merged = group_max[gi] + 2 * c.exchange_us + c.merge_us + p.S * c.merge_split_us;
      for (int k = 0; k < I.sig_n; ++k) ctr_done[I.sig_ctr + k] = std::max(ctr_done[I.sig_ctr + k], merged);
    } else if (I.sig_ctr != kNoCounter) {
      for (int k = 0; k < I.sig_n; ++k) ctr_done[I.sig_ctr + k] = std::max(ctr_done[I.sig_ctr + k], finish);
    }
    end = std::max(end, finish);
  }
  CostEstimate e;
  e.step_us = end + c.exchange_us;  // the argmax merge of the LM-head instructions (ticket)
  for (int o = 0; o < 7; ++o) e.stage_us[o] = cnt_t[o] > 0 ? sum_t[o] / cnt_t[o] : 0.0;
  e.hbm_floor_us = hbm_bytes / (c.sm_gbs * 1e3 * n);
  // conventional path: one launch per (layer, instruction class); a launch's
  // instructions run on the plan's CTAs (one wave when every CTA holds at most
  // one), each from a cold ring, and the launch ends with its slowest CTA
  const int n_stage = s.L * kStagesPerLayer + 1;
  std::vector<std::vector<double>> per_cta(n_stage, std::vector<double>(n, 0.0));
  std::vector<double> merge_extra(n_stage, 0.0);
  for (const Instr *Ip : order) {
    const Instr &I = *Ip;
    if (I.op == OP_NOP) continue;
    const int st = I.op == OP_LMHEAD ? s.L * kStagesPerLayer : I.layer * kStagesPerLayer + (I.op - 1);
    bool kv = false;
    const int np = instr_pages(req, p, I, context, &kv);
    const double pt = kv ? c.attn_page_us : page_time(req, p, I, c);
    // cold ring: the first page arrives one page-time after the launch, later
    // ones overlap compute
    const double t = np > 0 ? t_hbm + (np - 1) * std::max(t_hbm, pt) + pt : 0.0;
    per_cta[st][cta_of[I.seq]] += t + (kv ? c.attn_fixed_us : c.instr_us);
    if (I.op == OP_ATTN) merge_extra[st] = 2 * c.exchange_us + c.merge_us + p.S * c.merge_split_us;
  }
  // CTA waves: a launch whose work sits on g CTAs runs in ceil(g / W) waves
  // on W available CTAs
  const int W = c.conv_ctas > 0 ? std::min(c.conv_ctas, n) : n;
  double per_op = 0.0;
  for (int st = 0; st < n_stage; ++st) {
    double mx = 0.0;
    int g = 0;
    for (double t : per_cta[st]) {
      mx = std::max(mx, t);
      g += t > 0.0;
    }
    const int waves = g > 0 ? (g + W - 1) / W : 0;
    per_op += c.launch_us + c.exchange_us + waves * mx + merge_extra[st];
  }
  e.per_op_us = per_op;
  *out = e;
  return "";
}

}  // namespace mk
