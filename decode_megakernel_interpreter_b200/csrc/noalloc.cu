// mk_decode_step_noalloc: one decode step that allocates no device memory.
//
// Who needs it: callers that cannot call cudaMalloc (or any allocator) at the
// point where they want to run a step -- for example code running inside a
// host callback or a signal-safe context where allocation calls are not
// allowed, an embedding runtime whose memory is owned and budgeted by another
// component (a serving framework with its own pooling allocator, a process
// whose device memory is fully reserved up front), or a caller that must not
// trigger the implicit synchronisation an allocation can cause.  mk_create
// cannot serve them: it allocates the repacked weights, the activation and
// counter buffers and the plan.
//
// What this file does instead: the step's scratch (plan, RoPE table,
// activations, split-attention partials, argmax partials, counters, status)
// lives in one file-scope __device__ array of fixed size, so the memory is
// reserved once when the module is loaded on a device and held until the
// process exits.  The kernel reads the caller's weights in their own layout
// (the raw-layout variant of the interpreter), so no repacked copy is needed.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "interp_launch.h"
#include "mk_internal.h"
#include "planner.h"

using namespace mk;

// The scratch of every call on a device.  In host code `g_noalloc_scratch` is
// only a host-side stand-in for the symbol, never a device address: the kernel
// gets the address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MK_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;

struct DeviceSlot {
  bool ready = false;
  unsigned char *scratch = nullptr;  // device address of g_noalloc_scratch on this device
  int sm_count = 0, smem_optin = 0;
  // what the scratch currently holds (skip re-uploading an unchanged plan)
  std::vector<unsigned char> key;
};

std::mutex g_mu;
DeviceSlot g_slots[kMaxDevices];

// Set-up, once per device, with that device current.
int device_setup(int dev, DeviceSlot **out) {
  if (dev < 0 || dev >= kMaxDevices) return MK_ERR_INVALID_ARG;
  DeviceSlot &s = g_slots[dev];
  if (!s.ready) {
    void *ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&s.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&s.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return MK_ERR_CUDA;
    }
    s.scratch = static_cast<unsigned char *>(ptr);
    s.ready = true;
  }
  *out = &s;
  return MK_OK;
}

// the status words sit at this offset of the scratch (right after the step
// number), where mk_noalloc_get_status reads them
constexpr size_t kStatusAt = 256;

struct Layout {
  size_t off = 0;
  size_t take(size_t bytes) {
    size_t at = off;
    off += (bytes + 255) / 256 * 256;
    return at;
  }
};

}  // namespace

extern "C" int mk_decode_step_noalloc(const mk_config *cfg, const mk_weights *w, const mk_kv_cache *kv,
                                      const int32_t *tokens, const int32_t *positions, float *logits_out,
                                      int32_t *next_tokens_out, void *stream) {
  if (!cfg || !w || !kv || !tokens || !positions || !next_tokens_out || !w->embed || !w->final_norm ||
      !w->layers || !kv->k || !kv->v || (!cfg->tied_lm_head && !w->lm_head))
    return MK_ERR_INVALID_ARG;
  if (cfg->max_batch < 1 || cfg->max_seq < 1 || cfg->n_layers < 1 || !(cfg->rope_theta > 0.0) ||
      !(cfg->rms_eps >= 0.f))
    return MK_ERR_INVALID_ARG;
  const Shape s{cfg->n_layers, cfg->hidden, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim, cfg->ffn, cfg->vocab};
  if (!check_shape(s, cfg->max_batch).empty()) return MK_ERR_UNSUPPORTED_SHAPE;
  if (cfg->max_batch != 1) return MK_ERR_UNSUPPORTED_SHAPE;  // batched instructions: not in this build
  const void *lm = cfg->tied_lm_head ? w->embed : w->lm_head;
  for (const void *q : {w->embed, lm, w->final_norm, (const void *)kv->k, (const void *)kv->v})
    if (reinterpret_cast<uintptr_t>(q) & 15u) return MK_ERR_INVALID_ARG;
  for (int l = 0; l < cfg->n_layers; ++l) {
    const mk_layer_weights &L = w->layers[l];
    const void *ps[] = {L.attn_norm, L.wq, L.wk, L.wv, L.wo, L.ffn_norm, L.w_gate, L.w_up, L.w_down};
    for (const void *q : ps)
      if (!q || (reinterpret_cast<uintptr_t>(q) & 15u)) return MK_ERR_INVALID_ARG;
  }

  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  DeviceSlot *slot = nullptr;
  int rc = device_setup(dev, &slot);
  if (rc) return rc;

  // the plan mk_plan would build with default options on this device
  PlanRequest req;
  req.s = s;
  req.B = 1;
  req.num_ctas = slot->sm_count;
  req.assumed_context = cfg->max_seq;
  req.S = 0;
  Plan p;
  if (!build_plan(req, &p).empty()) return MK_ERR_UNSUPPORTED_SHAPE;

  // carve the scratch; reject shapes that need more than the array holds
  const int B = 1, hd = s.d / 2;
  Layout lay;
  const size_t o_epoch = lay.take(4), o_status = lay.take(sizeof(int) * kStatusWords);
  if (o_status != kStatusAt) return MK_ERR_CUDA;
  const size_t o_ctr = lay.take(sizeof(unsigned) * (size_t)p.n_counters);
  const size_t sync_end = lay.off;
  const size_t o_instr = lay.take(sizeof(Instr) * p.instrs.size());
  const size_t o_qoff = lay.take(sizeof(int) * p.num_ctas), o_qlen = lay.take(sizeof(int) * p.num_ctas);
  const size_t o_layers = lay.take(sizeof(LayerDev) * s.L), o_raw = lay.take(sizeof(LayerRaw) * s.L);
  const size_t o_rope = lay.take(sizeof(float2) * (size_t)cfg->max_seq * hd);
  const size_t qd = (size_t)s.nq * s.d;
  // activations are tagged words; all of them, with the counters, are cleared
  // by every call (the step number restarts at 1 each call)
  const size_t tagged_begin = lay.off;
  const size_t o_q = lay.take(4 * (size_t)s.L * B * qd), o_o = lay.take(4 * (size_t)s.L * B * qd);
  const size_t o_x = lay.take(4 * (size_t)s.L * B * s.H), o_act = lay.take(4 * (size_t)s.L * B * s.F);
  const size_t o_dp = lay.take(4 * (size_t)s.L * p.ndp * B * s.H);
  const size_t o_kv = lay.take(4 * (size_t)s.L * B * 2 * s.nkv * s.d);
  const size_t o_po = lay.take(4 * (size_t)s.L * B * s.nq * p.S * s.d);
  const size_t o_pml = lay.take(8 * (size_t)s.L * B * s.nq * p.S * 2);
  const size_t o_av = lay.take(8 * (size_t)B * p.n_lm), o_ai = lay.take(8 * (size_t)B * p.n_lm);
  if (lay.off > MK_NOALLOC_SCRATCH_BYTES) return MK_ERR_UNSUPPORTED_SHAPE;

  // shared memory geometry (as mk_plan)
  const size_t act = staging_floats(s.H, (int)qd, p.KCd, s.nq / s.nkv, s.d, 1);
  const int num_pages = ring_pages(slot->smem_optin, act);  // as mk_plan
  if (num_pages == 0) return MK_ERR_UNSUPPORTED_SHAPE;
  const int smem = shared_bytes_fixed(num_pages, act);

  unsigned char *base = slot->scratch;
  cudaStream_t st = (cudaStream_t)stream;
  // (re)upload the plan, the layer tables and the RoPE table when they differ
  // from what the scratch holds
  std::vector<LayerDev> ld(s.L);
  std::vector<LayerRaw> lr(s.L);
  for (int l = 0; l < s.L; ++l) {
    const mk_layer_weights &L = w->layers[l];
    ld[l] = LayerDev{nullptr, (const uint16_t *)L.wo, nullptr, nullptr, (const uint16_t *)L.attn_norm,
                     (const uint16_t *)L.ffn_norm};
    lr[l] = LayerRaw{(const uint16_t *)L.wq, (const uint16_t *)L.wk, (const uint16_t *)L.wv,
                     (const uint16_t *)L.wo, (const uint16_t *)L.w_gate, (const uint16_t *)L.w_up,
                     (const uint16_t *)L.w_down};
  }
  // what the uploaded tables depend on, field by field (a caller's mk_config
  // may carry indeterminate padding bytes, so the struct is not copied whole)
  std::vector<unsigned char> key;
  auto put = [&key](const void *v, size_t n) {
    key.insert(key.end(), static_cast<const unsigned char *>(v), static_cast<const unsigned char *>(v) + n);
  };
  const int32_t ints[] = {cfg->n_layers, cfg->hidden, cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim, cfg->ffn,
                          cfg->vocab, cfg->tied_lm_head, cfg->max_batch, cfg->max_seq, slot->sm_count};
  put(ints, sizeof ints);
  put(&cfg->rms_eps, sizeof cfg->rms_eps);
  put(&cfg->rope_theta, sizeof cfg->rope_theta);
  for (int l = 0; l < s.L; ++l) {
    const void *ptrs[] = {ld[l].wo, ld[l].attn_norm, ld[l].ffn_norm, lr[l].wq, lr[l].wk, lr[l].wv,
                          lr[l].wo, lr[l].wg, lr[l].wu, lr[l].wd};
    put(ptrs, sizeof ptrs);
  }
  cudaError_t e = cudaSuccess;
  if (key != slot->key) {
    std::vector<float2> rope((size_t)cfg->max_seq * hd);
    for (int i = 0; i < hd; ++i) {
      const double fr = std::pow(cfg->rope_theta, -2.0 * i / s.d);
      for (int pos = 0; pos < cfg->max_seq; ++pos) {
        const double a = (double)pos * fr;
        rope[(size_t)pos * hd + i] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
    }
    // pageable host memory: each copy has consumed its source when it returns
    e = cudaMemcpyAsync(base + o_instr, p.instrs.data(), sizeof(Instr) * p.instrs.size(), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(base + o_qoff, p.q_off.data(), sizeof(int) * p.num_ctas, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(base + o_qlen, p.q_len.data(), sizeof(int) * p.num_ctas, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(base + o_layers, ld.data(), sizeof(LayerDev) * s.L, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(base + o_raw, lr.data(), sizeof(LayerRaw) * s.L, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(base + o_rope, rope.data(), sizeof(float2) * rope.size(), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
      cudaGetLastError();
      slot->key.clear();
      return MK_ERR_CUDA;
    }
    slot->key = key;
  }
  // every call starts from zeroed counters, status and tagged activations,
  // step number 1: the epoch word lies in the zeroed range, so setting its
  // lowest byte to 1 makes the little-endian word 1 (no host copy per call)
  static_assert(sizeof(unsigned) == 4, "epoch word");
  e = cudaMemsetAsync(base, 0, sync_end, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(base + tagged_begin, 0, lay.off - tagged_begin, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(base + o_epoch, 1, 1, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }

  KParams k;
  memset(&k, 0, sizeof k);
  k.L = s.L;
  k.H = s.H;
  k.nq = s.nq;
  k.nkv = s.nkv;
  k.d = s.d;
  k.F = s.F;
  k.V = s.V;
  k.qdim = (int)qd;
  k.kvdim = s.nkv * s.d;
  k.B = B;
  k.Rh = p.Rh;
  k.Ro = p.Ro;
  k.Rd = p.Rd;
  k.KCd = p.KCd;
  k.ndp = p.ndp;
  k.S = p.S;
  k.max_seq = cfg->max_seq;
  k.eps = cfg->rms_eps;
  k.inv_H = 1.0f / (float)s.H;
  k.attn_scale = (float)(1.0 / std::sqrt((double)s.d));
  k.layers = reinterpret_cast<const LayerDev *>(base + o_layers);
  k.layers_raw = reinterpret_cast<const LayerRaw *>(base + o_raw);
  k.embed = (const uint16_t *)w->embed;
  k.lm_head = (const uint16_t *)(cfg->tied_lm_head ? w->embed : w->lm_head);
  k.final_norm = (const uint16_t *)w->final_norm;
  k.kc = (uint16_t *)kv->k;
  k.vc = (uint16_t *)kv->v;
  k.kv_hs = (long long)cfg->max_seq * s.d;
  k.kv_bs = k.kv_hs * s.nkv;
  k.kv_ls = k.kv_bs * cfg->max_batch;
  k.rope = reinterpret_cast<const float2 *>(base + o_rope);
  typedef unsigned long long llw;
  k.qbuf = reinterpret_cast<float *>(base + o_q);
  k.kvcur = reinterpret_cast<float *>(base + o_kv);
  k.part_o = reinterpret_cast<float *>(base + o_po);
  k.part_ml = reinterpret_cast<llw *>(base + o_pml);
  k.obuf = reinterpret_cast<float *>(base + o_o);
  k.xres = reinterpret_cast<float *>(base + o_x);
  k.actb = reinterpret_cast<float *>(base + o_act);
  k.dpart = reinterpret_cast<float *>(base + o_dp);
  k.arg_val = reinterpret_cast<llw *>(base + o_av);
  k.arg_idx = reinterpret_cast<llw *>(base + o_ai);
  k.n_lm = p.n_lm;
  k.ctr = reinterpret_cast<unsigned *>(base + o_ctr);
  k.epoch = reinterpret_cast<unsigned *>(base + o_epoch);
  k.status = reinterpret_cast<int *>(base + o_status);
  k.attn_ticket0 = p.attn_ticket0;
  k.arg_ticket0 = p.arg_ticket0;
  k.exit_ticket = p.exit_ticket;
  k.dyn_head = p.dyn_head;
  k.instrs = reinterpret_cast<const Instr *>(base + o_instr);
  k.q_off = reinterpret_cast<const int *>(base + o_qoff);
  k.q_len = reinterpret_cast<const int *>(base + o_qlen);
  k.n_instr = (int)p.instrs.size();
  k.num_pages = num_pages;
  k.act_floats = (long long)act;
  k.pf_pages = 0;
  k.max_inflight = std::max(kLoaders, std::min(kDefaultInflight, num_pages) / kLoaders * kLoaders);
  k.timeout_ns = 1000000000LL;
  k.trace = nullptr;
  k.mode = MODE_FINAL_LAUNCH;
  k.stage_filter = -1;
  k.tokens = tokens;
  k.positions = positions;
  k.logits = logits_out;
  k.next_tokens = next_tokens_out;
  const void *fn = interp_kernel_raw();
  int per_sm = 0;
  e = interp_prepare(fn, smem, &per_sm);
  if (e == cudaSuccess && per_sm < 1) return MK_ERR_LAUNCH;
  if (e == cudaSuccess) e = launch_interp(fn, k, p.num_ctas, smem, st, true);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return (e == cudaErrorCooperativeLaunchTooLarge || e == cudaErrorLaunchOutOfResources) ? MK_ERR_LAUNCH
                                                                                              : MK_ERR_CUDA;
  }
  return MK_OK;
}

extern "C" int mk_noalloc_get_status(void *stream, int32_t *detail) {
  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  const DeviceSlot &slot = g_slots[dev];
  if (!slot.ready) return MK_OK;  // no call on this device yet
  int st[kStatusWords];
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaMemcpy(st, slot.scratch + kStatusAt, sizeof st, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  if (detail)
    for (int i = 0; i < 6; ++i) detail[i] = st[0] ? st[i < 5 ? 2 + i : 1] : 0;
  return st[0];
}
