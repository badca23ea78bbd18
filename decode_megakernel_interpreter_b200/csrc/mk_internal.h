// Internal types shared by the host planner, the C ABI and the interpreter
// kernel.  Not part of the public ABI (include/mk.h is).
#pragma once
#include <stdint.h>
#include <vector_types.h>  // float2

namespace mk {

// ---------------------------------------------------------------- geometry
// Every weight byte the interpreter streams moves in 16 KiB shared-memory
// pages (the paged shared memory of the "Hazy megakernel summary" page,
// section 四(二), re-sized for Blackwell's 227 KB per CTA).  A matrix-vector
// page holds R rows x KC columns of bf16 with R * KC = 8192.
constexpr int kPageBytes = 16384;
constexpr int kPageElems = kPageBytes / 2;
constexpr int kLoaders = 2;                   // loader warps (lane 0 of each issues bulk copies)
constexpr int kComputeWarps = 8;              // warps kLoaders .. kLoaders+7
constexpr int kThreads = 32 * (kLoaders + kComputeWarps);
constexpr int kComputeThreads = 32 * kComputeWarps;
constexpr int kMaxKc = 4096;                  // largest K staged in one page row
constexpr int kMaxBatch = 16;
constexpr int kMaxDownPieces = 8;             // down-projection K pieces at most
constexpr int kDefaultInflight = 4;           // bulk-copy pages in flight per CTA
constexpr int kTcXchFloats = 128 * 16;        // batched builds: tensor-core epilogue exchange (floats)
constexpr int kSplitRedFloats = 1024;         // batch 1: split-page row partials (floats, staging region)

// ---------------------------------------------------------------- opcodes
// The instruction set of the decode step (the fused instructions the
// "Hazy megakernel summary" page lists: RMSNorm + QKV + RoPE, attention, ...).
enum Op : uint8_t {
  OP_NOP = 0,
  OP_QKV = 1,    // rms(x)*g1 -> fused QKV rows -> RoPE -> q (fp32) / K,V cache (bf16)
  OP_ATTN = 2,   // one (sequence, kv head, split) of split-KV GQA decode attention;
                 // the last split to finish merges the splits (log-sum-exp)
  OP_OPROJ = 3,  // x_mid = x_in + Wo * attn
  OP_GATEUP = 4, // rms(x_mid)*g2 -> gate/up rows -> silu(gate)*up
  OP_DOWN = 5,   // partial_k = Wd[:, K-piece k] * act[K-piece k]
  OP_LMHEAD = 6, // rms(x_out)*gf -> logits rows -> per-instruction argmax; last merges
};

// Instruction classes double as the "stage" used by the per-op comparison path
// (one launch per stage per layer).
enum Stage : uint8_t { ST_QKV = 0, ST_ATTN = 1, ST_OPROJ = 2, ST_GATEUP = 3, ST_DOWN = 4, ST_LMHEAD = 5 };
constexpr int kStagesPerLayer = 5;

constexpr uint32_t kNoCounter = 0xFFFFFFFFu;

// One interpreter instruction (32 bytes).
struct Instr {
  uint8_t op;
  uint8_t pad0;
  uint16_t layer;
  uint32_t a;        // matvec: first page | attn: kv head g | lmhead: first page
  uint32_t b;        // matvec: page count | attn: split index s
  uint32_t c;        // down: K piece | attn: sequence | lmhead: argmax slot
  uint32_t wait_ctr; // counter to wait on (kNoCounter: none)
  uint32_t wait_cnt; // producers per step: wait until ctr >= epoch * wait_cnt
  uint32_t sig_ctr;  // first counter to signal (kNoCounter: none)
  uint16_t sig_n;    // number of consecutive counters to signal
  uint16_t seq;      // global position of the instruction in the topological order
};
static_assert(sizeof(Instr) == 32, "Instr must be 32 bytes");

// Per-layer weight pointers the kernel reads.
struct LayerDev {
  const uint16_t *wqkv;     // packed [(nq+2nkv)*d / R pages][R][H]
  const uint16_t *wo;       // caller's [H][q_dim]
  const uint16_t *wgu;      // packed [F/(R/2) pages][R][H] (R/2 gate rows, R/2 up rows)
  const uint16_t *wd;       // packed [F/KCd pieces][H/Rd pages][Rd][KCd]
  const uint16_t *attn_norm;
  const uint16_t *ffn_norm;
  // batched plans: gate/up and down in 128-row tensor-core tiles (64 columns
  // per page, K-major without swizzle); null otherwise
  const uint16_t *wgu_tc;   // [F/64 tiles: 64 gate + 64 up rows][H/64 pages]
  const uint16_t *wd_tc;    // [F/KCd pieces][H/128 tiles][KCd/64 pages]
  const uint16_t *wqkv_tc;  // [(q_dim + 2 kv_dim)/128 tiles of [q; k; v] rows][H/64 pages]
  const uint16_t *wo_tc;    // [H/128 tiles][q_dim/64 pages]
};

// Per-layer pointers to the caller's weights in their own [out][in] layout
// (used by the kernel variant that cannot keep a repacked copy).
struct LayerRaw {
  const uint16_t *wq, *wk, *wv, *wo, *wg, *wu, *wd;
};

// Mode bits.
enum : uint32_t {
  MODE_NO_WAIT = 1u,      // per-op path: kernel boundaries order the stages
  MODE_TRACE = 2u,
  MODE_DYNAMIC = 4u,      // one global queue claimed with an atomic
  MODE_FINAL_LAUNCH = 8u, // this launch ends the step (advances the epoch)
  MODE_EVENT = 16u,       // with MODE_DYNAMIC: the global queue holds ready instructions only
};

// Tensor parallelism: where the outputs of one rank that the other ranks read
// go -- every rank's own copies of these buffers (device pointers; on one GPU
// for an emulated group, peer pointers over NVLink for a group of GPUs).
struct TpPeer {
  float *opart;                  // [L][tp_n][B][H] O-projection partials, by producing rank
  float *dpart;                  // [L][ndp][B][H] down-projection pieces (rank r: pieces r*ndp_local ..)
  unsigned *ctr;                 // counters (the O and down counters count every rank's producers)
  unsigned long long *arg_val;   // [B][n_lm] argmax slots (rank r: slots r*n_lm_local ..)
  unsigned long long *arg_idx;
};

// Status words (device): [0] first error code, [1] abort flag, [2..7] detail.
constexpr int kStatusWords = 8;

struct KParams {
  // shape
  int L, H, nq, nkv, d, F, V, qdim, kvdim, B;
  int Rh;       // rows per page of the H-input matrices (QKV, gate/up, LM head) = 8192 / H
  int Ro;       // rows per page of O projection = 8192 / q_dim
  int Rd, KCd;  // rows per page / K piece width of the down projection
  int ndp;      // number of down K pieces = F / KCd
  int S;        // kv splits
  int max_seq;
  float eps, attn_scale;
  float inv_H;                     // 1 / hidden (exact: hidden is a power of two)
  // batched plans: the LM head in 128-row tensor-core tiles (64 columns per
  // page, K-major without swizzle); null otherwise
  const uint16_t *lm_tc;
  // weights
  const LayerDev *layers;
  const LayerRaw *layers_raw;  // only read by the raw-layout kernel variant
  const uint16_t *embed, *lm_head, *final_norm;
  // kv cache
  uint16_t *kc, *vc;
  long long kv_ls, kv_bs, kv_hs;   // element strides: layer, batch, head (position stride = d)
  const float2 *rope;              // [max_seq][d/2] (cos, sin)
  // activations: tagged fp32 words (value rounded to 22 significant bits, the
  // two low mantissa bits = step number mod 4)
  float *qbuf;                  // [L][B][q_dim]
  float *kvcur;                 // [L][B][2][kv_dim]  this step's K and V rows (bf16-rounded)
  float *part_o;                // [L][B][nq][S][d]
  float *obuf;                  // [L][B][q_dim]
  float *xres;                  // [L][B][H]
  float *actb;                  // [L][B][F]
  float *dpart;                 // [L][ndp][B][H]
  // batched tensor-core plans: x_in of the next layer, [L][B][H], summed once
  // per 128-row tile by the last of the tile's down pieces (ticket
  // dn_ticket0 + l * (H / 128) + tile); null otherwise (consumers then sum
  // the residual and the pieces themselves)
  float *xin;
  unsigned dn_ticket0;
  // tagged 64-bit words (step number << 32 | 32-bit value): values that may
  // be -inf, and indices
  unsigned long long *part_ml;  // [L][B][nq][S][2]
  unsigned long long *arg_val;  // [B][n_lm]
  unsigned long long *arg_idx;  // [B][n_lm] (index bits in the value field)
  int n_lm;        // LM-head instructions (argmax slots) per step
  // sync
  unsigned *ctr;      // counters + tickets
  unsigned *epoch;    // current step number (>= 1), advanced by the last CTA
  int *status;        // kStatusWords
  unsigned attn_ticket0;  // index of the first attention merge ticket [L][B][nkv]
  unsigned arg_ticket0;   // index of the first argmax ticket [B]
  unsigned exit_ticket;   // index of the exit ticket
  unsigned dyn_head;      // index of the dynamic-queue head counter
  // event-driven queue (MODE_EVENT): claims k < n_ev_init take ev_init[k];
  // later claims wait for ready slot k, which the last producer of a counter
  // fills (step << 32 | instruction index) with the counter's dependents
  // ev_list[ev_off[c] .. ev_off[c+1]) once it reaches epoch * ev_cnt[c]
  unsigned ev_tail;       // index of the ready-queue tail counter
  int n_ev, n_ev_init;    // claimable instructions per step, of which ready at the start
  const int *ev_off, *ev_list, *ev_init;
  const unsigned *ev_cnt;
  unsigned long long *ev_ready;  // [n_ev]
  // plan
  const Instr *instrs;    // all instructions; static: per-CTA contiguous queues
  const int *q_off, *q_len;
  int n_instr;
  int num_pages;          // ring pages per CTA
  long long act_floats;   // floats of the staging region (input vectors, attention scratch)
  int pf_pages;           // L2 prefetch distance in pages (0 = off)
  int max_inflight;       // bulk-copy pages in flight per CTA (0 = no cap)
  long long timeout_ns;
  unsigned long long *trace;  // [n_instr][5]
  uint32_t mode;
  int stage_filter;       // per-op path: run only this (layer*5 + stage), -1 = all
  // tensor parallelism (tp_n > 1, the TP interpreter build only): this rank
  // computes the heads, FFN columns and vocabulary rows of its shard; the O
  // projection and the down projection write partial sums into every rank's
  // opart / dpart (summed by the consumers in a fixed order), the gate/up
  // instructions materialise x_mid as this rank's residual copy, and the LM
  // head writes its rows' logits and argmax slots.  Unused otherwise.
  int tp_n, tp_rank, tp_ctas;     // ranks, this rank, CTAs per rank
  const KParams *tp_params;       // emulated group (one launch): every rank's parameters, by CTA
  const TpPeer *tp_peers;         // [tp_n]
  float *opart;                   // this rank's copy [L][tp_n][B][H]
  int ndp_local, n_lm_local;      // this rank's down pieces per layer and LM-head instructions
  int n_gu_layer;                 // gate/up instructions per layer (each stores a slice of x_mid)
  int lm_row0, V_lm;              // this rank's LM-head rows [lm_row0, lm_row0 + V_lm)
  // prompt chunks (chunk_n > 0; see mk_prefill): row b of the step is prompt
  // token j = min(b, chunk_n - 1) at position chunk_pos0 + j, and every row
  // uses KV sequence kv_seq0; rows past chunk_n - 1 repeat the last token and
  // write neither the cache nor logits.  0 for decode steps.
  int chunk_n, chunk_pos0, kv_seq0;
  // io
  const int *tokens, *positions;
  float *logits;
  int *next_tokens;
};

}  // namespace mk
