// C ABI of the decode megakernel engine (declared in include/mk.h and
// include/mk_host.h).  Host code: validation, device buffers, weight
// repacking, the RoPE table, plan upload and launches.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "../../include/mk_host.h"
#include "interp_launch.h"
#include "mk_internal.h"
#include "planner.h"

using namespace mk;

static_assert(sizeof(mk_instr_desc) == sizeof(Instr), "mk_instr_desc mirrors Instr");

struct mk_handle {
  mk_config cfg;
  Shape shape;
  int device = 0, sm_count = 0, smem_optin = 0;
  // borrowed
  const uint16_t *embed = nullptr, *lm_head = nullptr, *final_norm = nullptr;
  uint16_t *kc = nullptr, *vc = nullptr;
  std::vector<mk_layer_weights> lw;
  // owned for the handle's lifetime
  std::vector<void *> allocs;
  uint16_t *wqkv = nullptr, *wgu = nullptr, *wd = nullptr;
  LayerDev *d_layers = nullptr;
  float2 *d_rope = nullptr;
  // tagged fp32 activation words (the step number mod 4 in the two low
  // mantissa bits)
  float *qbuf = nullptr, *obuf = nullptr, *xres = nullptr, *actb = nullptr, *dpart = nullptr, *kvcur = nullptr;
  int dpart_pieces = 0;  // down-projection K pieces dpart holds per layer and sequence
  unsigned *ctr_epoch = nullptr;  // [0] = epoch
  // every tagged buffer (pointer, bytes): zeroed whenever the step number restarts
  std::vector<std::pair<void *, size_t>> tagged;
  int *status = nullptr;
  // owned per plan
  std::vector<void *> plan_allocs;
  bool planned = false;
  Plan plan;
  mk_plan_opts opts;
  KParams kp;
  int smem = 0, grid = 0, nb = 1;
  const void *kernel = nullptr;  // the interpreter build this plan launches
  int kernel_variant = 0;        // 1: specialised for this model's shape
  int est_step_us = 0;           // the plan cost model's step estimate at max_seq (0: dynamic queue)
  // mk_prefill's scratch for the logits and greedy tokens of a chunk's rows
  // (allocated with the plan on first use)
  float *pf_logits = nullptr;
  int *pf_next = nullptr;
  int last_detail[6] = {0, 0, 0, 0, 0, 0};
  // per-op graph mode
  cudaGraphExec_t gexec = nullptr;
  const void *g_tokens = nullptr, *g_pos = nullptr, *g_logits = nullptr, *g_next = nullptr;
};

namespace {

int cuda_code(cudaError_t e) {
  if (e == cudaSuccess) return MK_OK;
  if (e == cudaErrorMemoryAllocation) return MK_ERR_OUT_OF_MEMORY;
  if (e == cudaErrorCooperativeLaunchTooLarge || e == cudaErrorLaunchOutOfResources) return MK_ERR_LAUNCH;
  return MK_ERR_CUDA;
}

#define MK_CUDA(call)                  \
  do {                                 \
    cudaError_t e_ = (call);           \
    if (e_ != cudaSuccess) {           \
      cudaGetLastError();              \
      return cuda_code(e_);            \
    }                                  \
  } while (0)

template <class T>
int dalloc(std::vector<void *> &list, T **out, size_t count, bool zero = true) {
  void *p = nullptr;
  size_t bytes = std::max<size_t>(count * sizeof(T), 16);
  cudaError_t e = cudaMalloc(&p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_OUT_OF_MEMORY;
  }
  list.push_back(p);
  if (zero) {
    e = cudaMemset(p, 0, bytes);
    if (e != cudaSuccess) return MK_ERR_CUDA;
  }
  *out = static_cast<T *>(p);
  return MK_OK;
}

void free_list(std::vector<void *> &list) {
  for (void *p : list) cudaFree(p);
  list.clear();
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

Shape shape_of(const mk_config &c) {
  return Shape{c.n_layers, c.hidden, c.n_q_heads, c.n_kv_heads, c.head_dim, c.ffn, c.vocab};
}

// Copy rows of `row_elems` bf16 from src_ptrs[r] to dst + r * row_elems.
__global__ void gather_rows_kernel(uint16_t *dst, const unsigned long long *src_ptrs, int row_elems,
                                   long long n_rows) {
  const int n16 = row_elems / 8;
  for (long long r = blockIdx.x; r < n_rows; r += gridDim.x) {
    const uint4 *s = reinterpret_cast<const uint4 *>(src_ptrs[r]);
    uint4 *d = reinterpret_cast<uint4 *>(dst + r * (long long)row_elems);
    for (int i = threadIdx.x; i < n16; i += blockDim.x) d[i] = s[i];
  }
}

// The LM head as 128-row tiles for the tensor cores: tile (block, kb) is one
// 16 KiB page of 64 columns, stored as 8 column chunks of 128 rows x 8 bf16
// (16-byte rows); rows past the vocabulary are zero.
__global__ void tile_lm_kernel(uint16_t *dst, const uint16_t *src, int V, int H, long long n16) {
  const int kpb = H / 64;
  const bool aligned = ((reinterpret_cast<uintptr_t>(src) & 15) == 0);
  for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < n16; u += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(u % 128);
    long long t = u / 128;
    const int ch = (int)(t % 8);
    t /= 8;
    const int kb = (int)(t % kpb);
    const long long blk = t / kpb;
    const long long row = blk * 128 + r;
    const long long col = (long long)kb * 64 + ch * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (row < V) {
      const uint16_t *sp = src + row * H + col;
      if (aligned) {
        v = *reinterpret_cast<const uint4 *>(sp);
      } else {
        uint16_t e[8];
        for (int i = 0; i < 8; ++i) e[i] = sp[i];
        v = make_uint4(e[0] | ((uint32_t)e[1] << 16), e[2] | ((uint32_t)e[3] << 16), e[4] | ((uint32_t)e[5] << 16),
                       e[6] | ((uint32_t)e[7] << 16));
      }
    }
    reinterpret_cast<uint4 *>(dst)[u] = v;
  }
}

// One 16-byte unit of a tensor-core tile copy (row `row` of a matrix with
// row stride ld elements, columns col..col+7), zero past `rows`.
__device__ __forceinline__ uint4 tile_unit(const uint16_t *src, long long row, long long rows, long long ld,
                                           long long col) {
  if (row >= rows) return make_uint4(0, 0, 0, 0);
  const uint16_t *sp = src + row * ld + col;
  if ((reinterpret_cast<uintptr_t>(sp) & 15) == 0) return *reinterpret_cast<const uint4 *>(sp);
  uint16_t e[8];
  for (int i = 0; i < 8; ++i) e[i] = sp[i];
  return make_uint4(e[0] | ((uint32_t)e[1] << 16), e[2] | ((uint32_t)e[3] << 16), e[4] | ((uint32_t)e[5] << 16),
                    e[6] | ((uint32_t)e[7] << 16));
}
// gate/up tiles: tile t = gate rows 64t..64t+63 then up rows 64t..64t+63;
// page kb = columns 64kb..64kb+63 as 8 chunks of 128 rows x 8 bf16
__global__ void tile_gu_kernel(uint16_t *dst, const uint16_t *gate, const uint16_t *up, int F, int H, long long n16) {
  const int kpt = H / 64;
  for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < n16; u += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(u % 128);
    long long t = u / 128;
    const int ch = (int)(t % 8);
    t /= 8;
    const int kb = (int)(t % kpt);
    const long long tile = t / kpt;
    const long long col = (long long)kb * 64 + ch * 8;
    reinterpret_cast<uint4 *>(dst)[u] =
        r < 64 ? tile_unit(gate, tile * 64 + r, F, H, col) : tile_unit(up, tile * 64 + r - 64, F, H, col);
  }
}
// fused QKV tiles: rows of [q; k; v] (wq, wk, wv stacked), 128 per tile
__global__ void tile_qkv_kernel(uint16_t *dst, const uint16_t *wq, const uint16_t *wk, const uint16_t *wv, int qdim,
                                int kvdim, int H, long long n16) {
  const int kpt = H / 64;
  for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < n16; u += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(u % 128);
    long long t = u / 128;
    const int ch = (int)(t % 8);
    t /= 8;
    const int kb = (int)(t % kpt);
    const long long row = (t / kpt) * 128 + r;
    const long long col = (long long)kb * 64 + ch * 8;
    uint4 v;
    if (row < qdim) v = tile_unit(wq, row, qdim, H, col);
    else if (row < qdim + kvdim) v = tile_unit(wk, row - qdim, kvdim, H, col);
    else v = tile_unit(wv, row - qdim - kvdim, kvdim, H, col);
    reinterpret_cast<uint4 *>(dst)[u] = v;
  }
}
// down tiles: piece k (columns k*KCd..), row tile rt (rows 128rt..), page kb
__global__ void tile_down_kernel(uint16_t *dst, const uint16_t *wd, int H, int F, int KCd, long long n16) {
  const int kpt = KCd / 64, rts = H / 128;
  for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < n16; u += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(u % 128);
    long long t = u / 128;
    const int ch = (int)(t % 8);
    t /= 8;
    const int kb = (int)(t % kpt);
    t /= kpt;
    const int rt = (int)(t % rts);
    const long long k = t / rts;
    reinterpret_cast<uint4 *>(dst)[u] =
        tile_unit(wd, (long long)rt * 128 + r, H, F, k * KCd + (long long)kb * 64 + ch * 8);
  }
}

int gather_rows(uint16_t *dst, const std::vector<unsigned long long> &src, int row_elems) {
  if (src.empty()) return MK_OK;
  unsigned long long *d_src = nullptr;
  MK_CUDA(cudaMalloc(&d_src, src.size() * sizeof(unsigned long long)));
  cudaError_t e = cudaMemcpy(d_src, src.data(), src.size() * sizeof(unsigned long long), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) {
    int blocks = (int)std::min<size_t>(src.size(), 65535);
    gather_rows_kernel<<<blocks, 256>>>(dst, d_src, row_elems, (long long)src.size());
    e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
  }
  cudaFree(d_src);
  return cuda_code(e);
}

// Repack the weights so that every 16 KiB page an instruction streams is
// contiguous: QKV rows in rotation-pair order, gate/up rows interleaved per
// page, down projection split into K pieces.
int repack(mk_handle *h, const Plan &p) {
  const Shape &s = h->shape;
  const int H = s.H, d = s.d;
  const size_t per_qkv = (size_t)p.P_qkv * kPageElems, per_gu = (size_t)p.P_gu * kPageElems,
               per_dn = (size_t)p.ndp * p.P_dp * kPageElems;
  int rc;
  if ((rc = dalloc(h->allocs, &h->wqkv, per_qkv * s.L, false))) return rc;
  if ((rc = dalloc(h->allocs, &h->wgu, per_gu * s.L, false))) return rc;
  if ((rc = dalloc(h->allocs, &h->wd, per_dn * s.L, false))) return rc;
  const int Rh = p.Rh, half = Rh / 2, pph = d / Rh;
  std::vector<unsigned long long> src;
  for (int l = 0; l < s.L; ++l) {
    const mk_layer_weights &W = h->lw[l];
    const uint16_t *wq = (const uint16_t *)W.wq, *wk = (const uint16_t *)W.wk, *wv = (const uint16_t *)W.wv;
    src.clear();
    for (int j = 0; j < p.P_qkv; ++j) {
      const int head = j / pph, jj = j % pph;
      for (int t = 0; t < Rh; ++t) {
        const int rin = t < half ? jj * half + t : d / 2 + jj * half + (t - half);
        const uint16_t *base;
        int hh;
        if (head < s.nq) {
          base = wq;
          hh = head;
        } else if (head < s.nq + s.nkv) {
          base = wk;
          hh = head - s.nq;
        } else {
          base = wv;
          hh = head - s.nq - s.nkv;
        }
        src.push_back((unsigned long long)(base + ((size_t)hh * d + rin) * H));
      }
    }
    if ((rc = gather_rows(h->wqkv + per_qkv * l, src, H))) return rc;
    src.clear();
    const uint16_t *wg = (const uint16_t *)W.w_gate, *wu = (const uint16_t *)W.w_up;
    for (int j = 0; j < p.P_gu; ++j)
      for (int t = 0; t < Rh; ++t) {
        const uint16_t *base = t < half ? wg : wu;
        const int row = j * half + (t < half ? t : t - half);
        src.push_back((unsigned long long)(base + (size_t)row * H));
      }
    if ((rc = gather_rows(h->wgu + per_gu * l, src, H))) return rc;
    src.clear();
    const uint16_t *wdn = (const uint16_t *)W.w_down;
    for (int k = 0; k < p.ndp; ++k)
      for (int r = 0; r < H; ++r) src.push_back((unsigned long long)(wdn + (size_t)r * s.F + (size_t)k * p.KCd));
    if ((rc = gather_rows(h->wd + per_dn * l, src, p.KCd))) return rc;
  }
  std::vector<LayerDev> ld(s.L);
  for (int l = 0; l < s.L; ++l) {
    ld[l].wqkv = h->wqkv + per_qkv * l;
    ld[l].wo = (const uint16_t *)h->lw[l].wo;
    ld[l].wgu = h->wgu + per_gu * l;
    ld[l].wd = h->wd + per_dn * l;
    ld[l].attn_norm = (const uint16_t *)h->lw[l].attn_norm;
    ld[l].ffn_norm = (const uint16_t *)h->lw[l].ffn_norm;
  }
  if ((rc = dalloc(h->allocs, &h->d_layers, s.L, false))) return rc;
  MK_CUDA(cudaMemcpy(h->d_layers, ld.data(), sizeof(LayerDev) * s.L, cudaMemcpyHostToDevice));
  return MK_OK;
}

// RoPE table: angle pos * theta^(-2i/d) in double, stored as float (cos, sin).
int build_rope(mk_handle *h) {
  const int d = h->cfg.head_dim, hd = d / 2, S = h->cfg.max_seq;
  std::vector<float2> t((size_t)S * hd);
  for (int i = 0; i < hd; ++i) {
    const double w = std::pow(h->cfg.rope_theta, -2.0 * i / d);
    for (int pos = 0; pos < S; ++pos) {
      const double a = (double)pos * w;
      t[(size_t)pos * hd + i] = make_float2((float)std::cos(a), (float)std::sin(a));
    }
  }
  int rc = dalloc(h->allocs, &h->d_rope, t.size(), false);
  if (rc) return rc;
  MK_CUDA(cudaMemcpy(h->d_rope, t.data(), t.size() * sizeof(float2), cudaMemcpyHostToDevice));
  return MK_OK;
}

mk_plan_opts default_opts(const mk_config &c) {
  mk_plan_opts o;
  memset(&o, 0, sizeof o);
  o.batch = c.max_batch;
  return o;
}

PlanRequest make_request(const mk_config &c, const mk_plan_opts &o, int num_ctas) {
  PlanRequest r;
  r.s = shape_of(c);
  r.B = o.batch;
  r.S = o.kv_splits;
  r.num_ctas = num_ctas;
  r.dynamic = o.sched_mode == MK_SCHED_DYNAMIC || o.sched_mode == MK_SCHED_EVENT;
  r.events = o.sched_mode == MK_SCHED_EVENT;
  r.assumed_context = std::max(1, c.max_seq);
  r.drop_producer = o.debug_drop_producer != 0;
  r.tensor_qkv_o = o.tensor_qkv_o != 0;
  // batched plans: gate/up, down and the LM head on the tensor cores when
  // asked (1), or automatically (0) when the plan cost model expects them to
  // beat the CUDA cores at this batch
  r.tensor = o.batch > 1 && (o.use_tcgen05 > 0 || (o.use_tcgen05 == 0 && cost_prefers_tensor(r, CostParams())));
  return r;
}

// use_tcgen05: -1, 0 or 1; 1 only for batched plans; the tensor-core QKV /
// O projection only with the tensor cores on
bool tensor_opts_ok(const mk_plan_opts &o) {
  if (o.use_tcgen05 < -1 || o.use_tcgen05 > 1) return false;
  if (o.use_tcgen05 == 1 && o.batch <= 1) return false;
  if (o.tensor_qkv_o && o.use_tcgen05 < 0) return false;
  return true;
}

void set_err(char *err, size_t n, const std::string &m) {
  if (err && n) {
    snprintf(err, n, "%s", m.c_str());
  }
}

int check_cfg(const mk_config *c, std::string *why) {
  if (!c) return MK_ERR_INVALID_ARG;
  if (c->max_batch < 1 || c->max_seq < 1 || c->n_layers < 1 || !(c->rms_eps >= 0.f) ||
      !(c->rope_theta > 0.0)) {
    *why = "non-positive capacity or parameter";
    return MK_ERR_INVALID_ARG;
  }
  std::string e = check_shape(shape_of(*c), c->max_batch);
  if (!e.empty()) {
    *why = e;
    return MK_ERR_UNSUPPORTED_SHAPE;
  }
  return MK_OK;
}

size_t act_floats_for(const mk_config &c, const Plan &p, int nb) {
  return staging_floats(c.hidden, c.n_q_heads * c.head_dim, p.KCd, c.n_q_heads / c.n_kv_heads, c.head_dim, nb);
}

}  // namespace

// ====================================================================== ABI

extern "C" const char *mk_status_string(int code) {
  switch (code) {
    case MK_OK: return "ok";
    case MK_ERR_INVALID_ARG: return "invalid argument";
    case MK_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MK_ERR_NOT_PLANNED: return "mk_plan has not been called";
    case MK_ERR_CUDA: return "CUDA runtime error";
    case MK_ERR_LAUNCH: return "persistent launch refused (CTAs not co-resident)";
    case MK_ERR_TIMEOUT: return "a device-side wait timed out";
    case MK_ERR_DEVICE_INPUT: return "token id or position out of range on the device";
    case MK_ERR_OUT_OF_MEMORY: return "device allocation failed";
    default: return "unknown status";
  }
}

extern "C" int mk_create(const mk_config *cfg, const mk_weights *w, const mk_kv_cache *kv, mk_handle **out) {
  if (out) *out = nullptr;
  if (!cfg || !w || !kv || !out) return MK_ERR_INVALID_ARG;
  std::string why;
  int rc = check_cfg(cfg, &why);
  if (rc) return rc;
  if (!w->embed || !w->final_norm || !w->layers || (!cfg->tied_lm_head && !w->lm_head) || !kv->k || !kv->v)
    return MK_ERR_INVALID_ARG;
  for (int l = 0; l < cfg->n_layers; ++l) {
    const mk_layer_weights &L = w->layers[l];
    const void *ps[] = {L.attn_norm, L.wq, L.wk, L.wv, L.wo, L.ffn_norm, L.w_gate, L.w_up, L.w_down};
    for (const void *p : ps)
      if (!p || !aligned16(p)) return MK_ERR_INVALID_ARG;
  }
  const void *lm = cfg->tied_lm_head ? w->embed : w->lm_head;
  if (!aligned16(w->embed) || !aligned16(lm) || !aligned16(w->final_norm) || !aligned16(kv->k) ||
      !aligned16(kv->v))
    return MK_ERR_INVALID_ARG;

  mk_handle *h = new (std::nothrow) mk_handle();
  if (!h) return MK_ERR_OUT_OF_MEMORY;
  h->cfg = *cfg;
  h->shape = shape_of(*cfg);
  h->embed = (const uint16_t *)w->embed;
  h->lm_head = (const uint16_t *)lm;
  h->final_norm = (const uint16_t *)w->final_norm;
  h->kc = (uint16_t *)kv->k;
  h->vc = (uint16_t *)kv->v;
  h->lw.assign(w->layers, w->layers + cfg->n_layers);
  auto fail = [&](int code) {
    cudaDeviceSynchronize();
    free_list(h->allocs);
    delete h;
    return code;
  };
  cudaError_t e = cudaGetDevice(&h->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->sm_count, cudaDevAttrMultiProcessorCount, h->device);
  if (e == cudaSuccess)
    e = cudaDeviceGetAttribute(&h->smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, h->device);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MK_ERR_CUDA);
  }
  // geometry of the CUDA-core page layouts (independent of batch and CTA
  // count; a tensor-core plan's down pieces are its own)
  PlanRequest req = make_request(*cfg, default_opts(*cfg), 1);
  req.B = 1;
  req.tensor = false;
  req.tensor_qkv_o = false;
  Plan geo;
  std::string err = build_plan(req, &geo);
  if (!err.empty()) return fail(MK_ERR_UNSUPPORTED_SHAPE);
  if ((rc = repack(h, geo))) return fail(rc);
  if ((rc = build_rope(h))) return fail(rc);
  const Shape &s = h->shape;
  const size_t Bm = cfg->max_batch;
  auto tagged = [&](float **ptr, size_t n) {
    int r = dalloc(h->allocs, ptr, n);
    if (!r) h->tagged.push_back({*ptr, n * sizeof(float)});
    return r;
  };
  if ((rc = tagged(&h->qbuf, (size_t)s.L * Bm * s.nq * s.d))) return fail(rc);
  if ((rc = tagged(&h->obuf, (size_t)s.L * Bm * s.nq * s.d))) return fail(rc);
  if ((rc = tagged(&h->xres, (size_t)s.L * Bm * s.H))) return fail(rc);
  if ((rc = tagged(&h->actb, (size_t)s.L * Bm * s.F))) return fail(rc);
  // the partial sums of every K piece of the down projection, for the plan
  // with the most pieces (tensor-core plans split K finer than the CUDA-core
  // layout)
  h->dpart_pieces = down_pieces_max(s);
  if ((rc = tagged(&h->dpart, (size_t)s.L * h->dpart_pieces * Bm * s.H))) return fail(rc);
  if ((rc = tagged(&h->kvcur, (size_t)s.L * Bm * 2 * s.nkv * s.d))) return fail(rc);
  if ((rc = dalloc(h->allocs, &h->ctr_epoch, 4))) return fail(rc);
  if ((rc = dalloc(h->allocs, &h->status, kStatusWords))) return fail(rc);
  e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MK_ERR_CUDA);
  }
  *out = h;
  return MK_OK;
}

static void drop_plan(mk_handle *h) {
  if (h->gexec) {
    cudaGraphExecDestroy(h->gexec);
    h->gexec = nullptr;
  }
  free_list(h->plan_allocs);
  h->pf_logits = nullptr;
  h->pf_next = nullptr;
  h->planned = false;
}

// The plan cost model's estimate of a step with every sequence at max_seq,
// rounded to whole microseconds (0 for the dynamic queue, which the model
// does not replay).
static int plan_estimate_us(const PlanRequest &req, const Plan &p) {
  if (p.dynamic) return 0;
  CostEstimate e;
  if (!estimate_plan(req, p, CostParams(), std::max(0, req.assumed_context - 1), &e).empty()) return 0;
  return (int)std::lround(e.step_us);
}

extern "C" int mk_plan(mk_handle *h, const mk_plan_opts *opts_in) {
  if (!h) return MK_ERR_INVALID_ARG;
  mk_plan_opts o = opts_in ? *opts_in : default_opts(h->cfg);
  if (o.batch < 1 || o.batch > h->cfg.max_batch) return MK_ERR_INVALID_ARG;
  if (o.sched_mode < MK_SCHED_STATIC || o.sched_mode > MK_SCHED_EVENT) return MK_ERR_INVALID_ARG;
  if (o.exec_mode < MK_EXEC_MEGAKERNEL || o.exec_mode > MK_EXEC_MEGAKERNEL_GENERIC) return MK_ERR_INVALID_ARG;
  const bool one_launch = o.exec_mode == MK_EXEC_MEGAKERNEL || o.exec_mode == MK_EXEC_MEGAKERNEL_GENERIC;
  if (!one_launch && o.sched_mode != MK_SCHED_STATIC) return MK_ERR_INVALID_ARG;
  if (o.kv_splits < kSplitsByCost || o.num_sms < 0 || o.wait_timeout_ns < 0) return MK_ERR_INVALID_ARG;
  if (!tensor_opts_ok(o)) return MK_ERR_INVALID_ARG;
  cudaError_t ce = cudaDeviceSynchronize();
  if (ce != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  drop_plan(h);
  const int num_ctas = o.num_sms > 0 ? std::min(o.num_sms, h->sm_count) : h->sm_count;
  PlanRequest req = make_request(h->cfg, o, num_ctas);
  Plan p;
  std::string err = build_plan(req, &p);
  if (err.empty()) err = validate_plan(req, p);
  if (err.empty() && p.ndp > h->dpart_pieces) err = "more down-projection pieces than the partial-sum buffer holds";
  if (!err.empty()) {
    fprintf(stderr, "mk_plan: %s\n", err.c_str());
    return MK_ERR_UNSUPPORTED_SHAPE;
  }
  // batched plans run the kernel instantiated for up to kMaxBatch sequences
  const int nb = o.batch > 1 ? kMaxBatch : 1;
  const size_t act_floats = act_floats_for(h->cfg, p, nb);
  // a multiple of the loader count (page g and the next user of its slot,
  // g + num_pages, then belong to the same loader) with 2 * num_pages a
  // multiple of the compute-warp count (page g - 2 * num_pages belongs to the
  // same warp as page g): every mbarrier parity test is then unambiguous
  const int num_pages = ring_pages(h->smem_optin, act_floats);
  if (num_pages == 0) return MK_ERR_UNSUPPORTED_SHAPE;
  const int smem = shared_bytes_fixed(num_pages, act_floats);
  // the interpreter build: specialised for this shape unless asked otherwise
  KParams sel;
  memset(&sel, 0, sizeof sel);
  sel.nq = h->shape.nq;
  sel.nkv = h->shape.nkv;
  sel.d = h->shape.d;
  sel.Rh = p.Rh;
  sel.Ro = p.Ro;
  sel.Rd = p.Rd;
  int variant = 0;
  const void *kernel =
      interp_kernel_for(sel, o.exec_mode != MK_EXEC_MEGAKERNEL_GENERIC, nb, p.tensor_qkv_o, &variant);
  if (!kernel) return MK_ERR_UNSUPPORTED_SHAPE;  // batch > 1 without a batched build for this shape
  int per_sm = 0;
  cudaError_t e = interp_prepare(kernel, smem, &per_sm);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  if (per_sm < 1) return MK_ERR_LAUNCH;

  const Shape &s = h->shape;
  const int B = o.batch;
  KParams &k = h->kp;
  memset(&k, 0, sizeof k);
  int rc;
  float *part_o;
  unsigned long long *part_ml, *arg_val, *arg_idx;
  int *q_off, *q_len;
  unsigned *ctr;
  Instr *instrs;
  unsigned long long *trace = nullptr;
  if ((rc = dalloc(h->plan_allocs, &part_o, (size_t)s.L * B * s.nq * p.S * s.d))) return rc;
  if ((rc = dalloc(h->plan_allocs, &part_ml, (size_t)s.L * B * s.nq * p.S * 2))) return rc;
  if ((rc = dalloc(h->plan_allocs, &arg_val, (size_t)B * p.n_lm))) return rc;
  if ((rc = dalloc(h->plan_allocs, &arg_idx, (size_t)B * p.n_lm))) return rc;
  // the handle's tagged buffers may hold tags of earlier steps: the step
  // number restarts at 1, so clear them (the plan's own buffers are new)
  for (auto &tb : h->tagged)
    if ((e = cudaMemset(tb.first, 0, tb.second)) != cudaSuccess) {
      cudaGetLastError();
      return MK_ERR_CUDA;
    }
  if ((rc = dalloc(h->plan_allocs, &ctr, (size_t)p.n_counters))) return rc;
  if ((rc = dalloc(h->plan_allocs, &instrs, p.instrs.size(), false))) return rc;
  if ((rc = dalloc(h->plan_allocs, &q_off, (size_t)num_ctas, false))) return rc;
  if ((rc = dalloc(h->plan_allocs, &q_len, (size_t)num_ctas, false))) return rc;
  if (o.trace && (rc = dalloc(h->plan_allocs, &trace, p.instrs.size() * MK_TRACE_WORDS))) return rc;
  // event-driven plans: the counters' dependent lists and the ready queue
  // (zeroed: no slot carries a step number >= 1 until a producer fills it)
  int *ev_off = nullptr, *ev_list = nullptr, *ev_init = nullptr;
  unsigned *ev_cnt = nullptr;
  unsigned long long *ev_ready = nullptr;
  const int n_ev = (int)(p.ev_init.size() + p.ev_list.size());
  if (p.events) {
    if ((rc = dalloc(h->plan_allocs, &ev_off, p.ev_off.size(), false))) return rc;
    if ((rc = dalloc(h->plan_allocs, &ev_list, std::max<size_t>(1, p.ev_list.size()), false))) return rc;
    if ((rc = dalloc(h->plan_allocs, &ev_init, std::max<size_t>(1, p.ev_init.size()), false))) return rc;
    if ((rc = dalloc(h->plan_allocs, &ev_cnt, p.ev_cnt.size(), false))) return rc;
    if ((rc = dalloc(h->plan_allocs, &ev_ready, (size_t)std::max(1, n_ev)))) return rc;
    e = cudaMemcpy(ev_off, p.ev_off.data(), sizeof(int) * p.ev_off.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !p.ev_list.empty())
      e = cudaMemcpy(ev_list, p.ev_list.data(), sizeof(int) * p.ev_list.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !p.ev_init.empty())
      e = cudaMemcpy(ev_init, p.ev_init.data(), sizeof(int) * p.ev_init.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
      e = cudaMemcpy(ev_cnt, p.ev_cnt.data(), sizeof(unsigned) * p.ev_cnt.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return MK_ERR_CUDA;
    }
  }
  e = cudaMemcpy(instrs, p.instrs.data(), p.instrs.size() * sizeof(Instr), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(q_off, p.q_off.data(), sizeof(int) * num_ctas, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(q_len, p.q_len.data(), sizeof(int) * num_ctas, cudaMemcpyHostToDevice);
  const unsigned one = 1;
  if (e == cudaSuccess) e = cudaMemcpy(h->ctr_epoch, &one, sizeof one, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemset(h->status, 0, sizeof(int) * kStatusWords);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }

  k.L = s.L;
  k.H = s.H;
  k.nq = s.nq;
  k.nkv = s.nkv;
  k.d = s.d;
  k.F = s.F;
  k.V = s.V;
  k.qdim = s.nq * s.d;
  k.kvdim = s.nkv * s.d;
  k.B = B;
  k.Rh = p.Rh;
  k.Ro = p.Ro;
  k.Rd = p.Rd;
  k.KCd = p.KCd;
  k.ndp = p.ndp;
  k.S = p.S;
  k.max_seq = h->cfg.max_seq;
  k.eps = h->cfg.rms_eps;
  k.inv_H = 1.0f / (float)s.H;
  k.attn_scale = (float)(1.0 / std::sqrt((double)s.d));
  k.layers = h->d_layers;
  k.embed = h->embed;
  k.lm_head = h->lm_head;
  k.lm_tc = nullptr;
  if (p.tensor) {
    // the tensor-core instructions read tiled copies (plan-owned): LM head,
    // and per layer gate/up and down, with a plan-owned layer table
    const int grid = 4 * h->sm_count;
    const long long lm16 = (long long)((s.V + 127) / 128) * 128 * (s.H / 8);
    const long long gu16 = (long long)(s.F / 64) * 128 * (s.H / 8);
    const long long dn16 = (long long)s.H * (s.F / 8);
    const int qdim = s.nq * s.d, kvdim = s.nkv * s.d;
    const long long qkv16 = (long long)(qdim + 2 * kvdim) * (s.H / 8), o16 = (long long)s.H * (qdim / 8);
    uint16_t *lm_t = nullptr, *gu_t = nullptr, *dn_t = nullptr, *qkv_t = nullptr, *o_t = nullptr;
    if ((rc = dalloc(h->plan_allocs, &lm_t, (size_t)lm16 * 8, false))) return rc;
    if ((rc = dalloc(h->plan_allocs, &gu_t, (size_t)gu16 * 8 * s.L, false))) return rc;
    if ((rc = dalloc(h->plan_allocs, &dn_t, (size_t)dn16 * 8 * s.L, false))) return rc;
    if (p.tensor_qkv_o) {
      if ((rc = dalloc(h->plan_allocs, &qkv_t, (size_t)qkv16 * 8 * s.L, false))) return rc;
      if ((rc = dalloc(h->plan_allocs, &o_t, (size_t)o16 * 8 * s.L, false))) return rc;
    }
    tile_lm_kernel<<<grid, 256>>>(lm_t, h->lm_head, s.V, s.H, lm16);
    std::vector<LayerDev> ld(s.L);
    MK_CUDA(cudaMemcpy(ld.data(), h->d_layers, sizeof(LayerDev) * s.L, cudaMemcpyDeviceToHost));
    for (int l = 0; l < s.L; ++l) {
      const mk_layer_weights &W = h->lw[l];
      uint16_t *gl = gu_t + (size_t)gu16 * 8 * l, *dl = dn_t + (size_t)dn16 * 8 * l;
      tile_gu_kernel<<<grid, 256>>>(gl, (const uint16_t *)W.w_gate, (const uint16_t *)W.w_up, s.F, s.H, gu16);
      tile_down_kernel<<<grid, 256>>>(dl, (const uint16_t *)W.w_down, s.H, s.F, p.KCd, dn16);
      ld[l].wgu_tc = gl;
      ld[l].wd_tc = dl;
      if (p.tensor_qkv_o) {
        uint16_t *ql = qkv_t + (size_t)qkv16 * 8 * l, *ol = o_t + (size_t)o16 * 8 * l;
        tile_qkv_kernel<<<grid, 256>>>(ql, (const uint16_t *)W.wq, (const uint16_t *)W.wk, (const uint16_t *)W.wv,
                                       qdim, kvdim, s.H, qkv16);
        tile_lm_kernel<<<grid, 256>>>(ol, (const uint16_t *)W.wo, s.H, qdim, o16);  // rows H, K = q_dim
        ld[l].wqkv_tc = ql;
        ld[l].wo_tc = ol;
      }
    }
    if ((e = cudaGetLastError()) != cudaSuccess || (e = cudaDeviceSynchronize()) != cudaSuccess) {
      cudaGetLastError();
      return MK_ERR_CUDA;
    }
    LayerDev *d_ld = nullptr;
    if ((rc = dalloc(h->plan_allocs, &d_ld, s.L, false))) return rc;
    MK_CUDA(cudaMemcpy(d_ld, ld.data(), sizeof(LayerDev) * s.L, cudaMemcpyHostToDevice));
    k.layers = d_ld;
    k.lm_tc = lm_t;
  }
  k.final_norm = h->final_norm;
  k.kc = h->kc;
  k.vc = h->vc;
  k.kv_hs = (long long)h->cfg.max_seq * s.d;
  k.kv_bs = k.kv_hs * s.nkv;
  k.kv_ls = k.kv_bs * h->cfg.max_batch;
  k.rope = h->d_rope;
  k.qbuf = h->qbuf;
  k.kvcur = h->kvcur;
  k.part_o = part_o;
  k.part_ml = part_ml;
  k.obuf = h->obuf;
  k.xres = h->xres;
  // batched tensor-core plans: the next layer's input, summed once per down tile
  if (p.tensor) {
    float *xin = nullptr;
    if ((rc = dalloc(h->plan_allocs, &xin, (size_t)s.L * B * s.H))) return rc;
    k.xin = xin;
    k.dn_ticket0 = p.dn_ticket0;
  }
  k.actb = h->actb;
  k.dpart = h->dpart;
  k.arg_val = arg_val;
  k.arg_idx = arg_idx;
  k.n_lm = p.n_lm;
  k.ctr = ctr;
  k.epoch = h->ctr_epoch;
  k.status = h->status;
  k.attn_ticket0 = p.attn_ticket0;
  k.arg_ticket0 = p.arg_ticket0;
  k.exit_ticket = p.exit_ticket;
  k.dyn_head = p.dyn_head;
  k.instrs = instrs;
  k.q_off = q_off;
  k.q_len = q_len;
  k.n_instr = (int)p.instrs.size();
  k.num_pages = num_pages;
  k.act_floats = (long long)act_floats;
  int pf_kb = o.l2_prefetch_kb;
  if (pf_kb == 0) pf_kb = -1;  // automatic: off until measured otherwise
  k.pf_pages = pf_kb > 0 ? (pf_kb * 1024) / kPageBytes : 0;
  {
    // rounded to a multiple of the loader count (same reason as num_pages)
    const int want = o.max_inflight_pages > 0 ? std::min(o.max_inflight_pages, num_pages)
                                              : (o.max_inflight_pages < 0 ? 0 : kDefaultInflight);
    k.max_inflight = want > 0 ? std::max(kLoaders, want / kLoaders * kLoaders) : 0;
  }
  k.timeout_ns = o.wait_timeout_ns > 0 ? o.wait_timeout_ns : 1000000000LL;
  k.trace = trace;
  k.mode = (o.trace ? MODE_TRACE : 0u) | (p.dynamic ? MODE_DYNAMIC : 0u) | (p.events ? MODE_EVENT : 0u);
  k.ev_tail = p.ev_tail;
  k.n_ev = n_ev;
  k.n_ev_init = (int)p.ev_init.size();
  k.ev_off = ev_off;
  k.ev_list = ev_list;
  k.ev_init = ev_init;
  k.ev_cnt = ev_cnt;
  k.ev_ready = ev_ready;
  k.stage_filter = -1;
  h->plan = std::move(p);
  h->opts = o;
  h->smem = smem;
  h->grid = num_ctas;
  h->nb = nb;
  h->kernel = kernel;
  h->kernel_variant = variant;
  h->est_step_us = plan_estimate_us(req, h->plan);
  h->planned = true;
  return MK_OK;
}

static int launch_per_op(mk_handle *h, KParams k, cudaStream_t st) {
  const int n_stage = h->shape.L * kStagesPerLayer + 1;
  for (int sidx = 0; sidx < n_stage; ++sidx) {
    // skip the empty per-layer stage slot of the LM head
    k.stage_filter = sidx;
    k.mode = (h->kp.mode & MODE_TRACE) | MODE_NO_WAIT | (sidx == n_stage - 1 ? MODE_FINAL_LAUNCH : 0u);
    cudaError_t e = launch_interp(h->kernel, k, h->grid, h->smem, st, false);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_code(e);
    }
  }
  return MK_OK;
}

extern "C" int mk_decode_step(mk_handle *h, const int32_t *tokens, const int32_t *positions, float *logits_out,
                              int32_t *next_tokens_out, void *stream) {
  if (!h || !tokens || !positions || !next_tokens_out) return MK_ERR_INVALID_ARG;
  if (!h->planned) return MK_ERR_NOT_PLANNED;
  cudaStream_t st = (cudaStream_t)stream;
  KParams k = h->kp;
  k.tokens = tokens;
  k.positions = positions;
  k.logits = logits_out;
  k.next_tokens = next_tokens_out;
  if (h->opts.exec_mode == MK_EXEC_MEGAKERNEL || h->opts.exec_mode == MK_EXEC_MEGAKERNEL_GENERIC) {
    k.mode |= MODE_FINAL_LAUNCH;
    cudaError_t e = launch_interp(h->kernel, k, h->grid, h->smem, st, true);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_code(e);
    }
    return MK_OK;
  }
  if (h->opts.exec_mode == MK_EXEC_PER_OP) return launch_per_op(h, k, st);
  // per-op launches replayed as one CUDA graph (re-captured if the I/O pointers change)
  if (!h->gexec || h->g_tokens != tokens || h->g_pos != positions || h->g_logits != logits_out ||
      h->g_next != next_tokens_out) {
    if (h->gexec) {
      cudaGraphExecDestroy(h->gexec);
      h->gexec = nullptr;
    }
    cudaStream_t cap;
    MK_CUDA(cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking));
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal);
    int rc = MK_OK;
    if (e == cudaSuccess) {
      rc = launch_per_op(h, k, cap);
      e = cudaStreamEndCapture(cap, &graph);
    }
    if (e == cudaSuccess && rc == MK_OK) e = cudaGraphInstantiate(&h->gexec, graph, 0);
    if (graph) cudaGraphDestroy(graph);
    cudaStreamDestroy(cap);
    if (rc != MK_OK) return rc;
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_code(e);
    }
    h->g_tokens = tokens;
    h->g_pos = positions;
    h->g_logits = logits_out;
    h->g_next = next_tokens_out;
  }
  MK_CUDA(cudaGraphLaunch(h->gexec, st));
  return MK_OK;
}

extern "C" int mk_prefill(mk_handle *h, int32_t seq, const int32_t *tokens, int32_t n_tokens, int32_t pos0,
                          float *logits_out, int32_t *next_token_out, void *stream) {
  if (!h || !tokens || !next_token_out || n_tokens < 1 || pos0 < 0) return MK_ERR_INVALID_ARG;
  if (!h->planned) return MK_ERR_NOT_PLANNED;
  if (seq < 0 || seq >= h->cfg.max_batch || (int64_t)pos0 + n_tokens > h->cfg.max_seq) return MK_ERR_INVALID_ARG;
  if (h->opts.exec_mode != MK_EXEC_MEGAKERNEL && h->opts.exec_mode != MK_EXEC_MEGAKERNEL_GENERIC)
    return MK_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const int B = h->kp.B, V = h->kp.V;
  if (!h->pf_next) {
    int rc;
    if ((rc = dalloc(h->plan_allocs, &h->pf_logits, (size_t)B * V, false))) return rc;
    if ((rc = dalloc(h->plan_allocs, &h->pf_next, (size_t)B, false))) return rc;
  }
  // chunks of up to B consecutive tokens, one launch each: row b of a chunk
  // is its b-th token (batched plans), or one token per launch (batch 1)
  int last_n = 0;
  for (int c0 = 0; c0 < n_tokens; c0 += B) {
    KParams k = h->kp;
    k.chunk_n = std::min(B, n_tokens - c0);
    k.chunk_pos0 = pos0 + c0;
    k.kv_seq0 = seq;
    k.tokens = tokens + c0;
    k.positions = tokens + c0;  // unused for chunks
    k.logits = (c0 + B >= n_tokens && logits_out) ? h->pf_logits : nullptr;
    k.next_tokens = h->pf_next;
    k.mode |= MODE_FINAL_LAUNCH;
    cudaError_t e = launch_interp(h->kernel, k, h->grid, h->smem, st, true);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_code(e);
    }
    last_n = k.chunk_n;
  }
  // the last token's row: its logits and greedy next token
  if (logits_out)
    MK_CUDA(cudaMemcpyAsync(logits_out, h->pf_logits + (size_t)(last_n - 1) * V, sizeof(float) * V,
                            cudaMemcpyDeviceToDevice, st));
  MK_CUDA(cudaMemcpyAsync(next_token_out, h->pf_next + (last_n - 1), sizeof(int32_t), cudaMemcpyDeviceToDevice, st));
  return MK_OK;
}

extern "C" int mk_get_status(mk_handle *h, void *stream) {
  if (!h) return MK_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  int st[kStatusWords];
  e = cudaMemcpy(st, h->status, sizeof st, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  if (st[0] == 0) return MK_OK;
  const int code = st[0];
  for (int i = 0; i < 6; ++i) h->last_detail[i] = st[i < 5 ? 2 + i : 1];
  // the step that failed left the counters inconsistent: start the step
  // numbering again
  e = cudaMemset(h->status, 0, sizeof(int) * kStatusWords);
  if (e == cudaSuccess && h->planned) {
    // restart the step numbering; every tagged word must then look stale
    const unsigned one = 1;
    e = cudaMemset(h->kp.ctr, 0, sizeof(unsigned) * h->plan.n_counters);
    for (auto &tb : h->tagged)
      if (e == cudaSuccess) e = cudaMemset(tb.first, 0, tb.second);
    const size_t S = (size_t)h->plan.S, L = h->shape.L, B = h->kp.B, nq = h->shape.nq, d = h->shape.d;
    if (e == cudaSuccess) e = cudaMemset(h->kp.part_o, 0, sizeof(float) * L * B * nq * S * d);
    if (e == cudaSuccess) e = cudaMemset(h->kp.part_ml, 0, 8 * L * B * nq * S * 2);
    if (e == cudaSuccess) e = cudaMemset(h->kp.arg_val, 0, 8 * B * h->plan.n_lm);
    if (e == cudaSuccess) e = cudaMemset(h->kp.arg_idx, 0, 8 * B * h->plan.n_lm);
    if (e == cudaSuccess && h->kp.xin) e = cudaMemset(h->kp.xin, 0, sizeof(float) * L * B * h->shape.H);
    if (e == cudaSuccess) e = cudaMemcpy(h->ctr_epoch, &one, sizeof one, cudaMemcpyHostToDevice);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  return code;
}

extern "C" void mk_destroy(mk_handle *h) {
  if (!h) return;
  cudaDeviceSynchronize();
  drop_plan(h);
  free_list(h->allocs);
  delete h;
}

extern "C" int mk_get_error_detail(const mk_handle *h, int32_t detail[6]) {
  if (!h || !detail) return MK_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i) detail[i] = h->last_detail[i];
  return MK_OK;
}

extern "C" int mk_get_plan_info(const mk_handle *h, mk_plan_info *info) {
  if (!h || !info) return MK_ERR_INVALID_ARG;
  if (!h->planned) return MK_ERR_NOT_PLANNED;
  info->num_ctas = h->grid;
  info->threads_per_cta = kThreads;
  info->smem_bytes = h->smem;
  info->num_pages = h->kp.num_pages;
  info->num_instructions = (int)h->plan.instrs.size();
  info->num_counters = h->plan.n_counters;
  info->kv_splits = h->plan.S;
  int mx = 0;
  for (int l : h->plan.q_len) mx = std::max(mx, l);
  info->max_queue_len = mx;
  info->weight_bytes_per_step = h->plan.weight_bytes;
  info->kernel_variant = h->kernel_variant;
  info->estimated_step_us = h->est_step_us;
  return MK_OK;
}

extern "C" int mk_trace_read(mk_handle *h, uint64_t *out, size_t n_words) {
  if (!h || !out) return MK_ERR_INVALID_ARG;
  if (!h->planned) return MK_ERR_NOT_PLANNED;
  if (!h->kp.trace) return MK_ERR_INVALID_ARG;
  const size_t need = h->plan.instrs.size() * MK_TRACE_WORDS;
  if (n_words < need) return MK_ERR_INVALID_ARG;
  MK_CUDA(cudaDeviceSynchronize());
  MK_CUDA(cudaMemcpy(out, h->kp.trace, need * sizeof(uint64_t), cudaMemcpyDeviceToHost));
  return MK_OK;
}

// ====================================================================== host-only planner

extern "C" int mk_host_plan(const mk_config *cfg, const mk_plan_opts *opts, int32_t num_ctas,
                            mk_instr_desc *instrs_out, int32_t max_instrs, int32_t *n_instrs, int32_t *queue_off,
                            int32_t *queue_len, mk_plan_info *info, char *err, size_t err_len) {
  std::string why;
  int rc = check_cfg(cfg, &why);
  if (rc) {
    set_err(err, err_len, why);
    return rc;
  }
  if (num_ctas < 1) return MK_ERR_INVALID_ARG;
  mk_plan_opts o = opts ? *opts : default_opts(*cfg);
  if (o.batch < 1 || o.batch > cfg->max_batch || !tensor_opts_ok(o) || o.kv_splits < kSplitsByCost ||
      o.sched_mode < MK_SCHED_STATIC || o.sched_mode > MK_SCHED_EVENT)
    return MK_ERR_INVALID_ARG;
  PlanRequest req = make_request(*cfg, o, num_ctas);
  Plan p;
  std::string e = build_plan(req, &p);
  if (e.empty()) e = validate_plan(req, p);
  if (!e.empty()) {
    set_err(err, err_len, e);
    return MK_ERR_UNSUPPORTED_SHAPE;
  }
  if (n_instrs) *n_instrs = (int32_t)p.instrs.size();
  if (instrs_out) {
    if (max_instrs < (int32_t)p.instrs.size()) return MK_ERR_INVALID_ARG;
    memcpy(instrs_out, p.instrs.data(), p.instrs.size() * sizeof(Instr));
  }
  if (queue_off)
    for (int c = 0; c < num_ctas; ++c) queue_off[c] = p.q_off[c];
  if (queue_len)
    for (int c = 0; c < num_ctas; ++c) queue_len[c] = p.q_len[c];
  if (info) {
    memset(info, 0, sizeof *info);
    info->num_ctas = num_ctas;
    info->threads_per_cta = kThreads;
    info->num_instructions = (int)p.instrs.size();
    info->num_counters = p.n_counters;
    info->kv_splits = p.S;
    int mx = 0;
    for (int l : p.q_len) mx = std::max(mx, l);
    info->max_queue_len = mx;
    info->weight_bytes_per_step = p.weight_bytes;
    info->estimated_step_us = plan_estimate_us(req, p);
  }
  return MK_OK;
}

extern "C" int mk_host_plan_simulate(const mk_config *cfg, const mk_plan_opts *opts, int32_t num_ctas, int32_t steps,
                                     uint64_t seed, int32_t timeout_ms, char *err, size_t err_len) {
  std::string why;
  int rc = check_cfg(cfg, &why);
  if (rc) {
    set_err(err, err_len, why);
    return rc;
  }
  if (num_ctas < 1 || steps < 1 || timeout_ms < 1) return MK_ERR_INVALID_ARG;
  mk_plan_opts o = opts ? *opts : default_opts(*cfg);
  if (o.batch < 1 || o.batch > cfg->max_batch || !tensor_opts_ok(o) || o.kv_splits < kSplitsByCost ||
      o.sched_mode < MK_SCHED_STATIC || o.sched_mode > MK_SCHED_EVENT)
    return MK_ERR_INVALID_ARG;
  PlanRequest req = make_request(*cfg, o, num_ctas);
  Plan p;
  std::string e = build_plan(req, &p);
  if (e.empty()) e = validate_plan(req, p);
  if (e.empty()) e = simulate_plan(req, p, steps, seed, timeout_ms);
  if (!e.empty()) {
    set_err(err, err_len, e);
    return MK_ERR_INVALID_ARG;
  }
  return MK_OK;
}

// ====================================================================== cost model

static CostParams cost_params_from(const mk_cost_params *q) {
  CostParams c;
  if (!q) return c;
  c.sm_gbs = q->sm_gbs;
  c.ring_pages = q->ring_pages;
  c.exchange_us = q->exchange_us;
  c.page_us = q->page_us;
  c.attn_page_us = q->attn_page_us;
  c.attn_fixed_us = q->attn_fixed_us;
  c.merge_us = q->merge_us;
  c.instr_us = q->instr_us;
  c.launch_us = q->launch_us;
  c.tc_page_us = q->tc_page_us;
  c.cc_page_us_seq = q->cc_page_us_seq;
  c.conv_ctas = q->conv_ctas;
  c.merge_split_us = q->merge_split_us;
  return c;
}

extern "C" void mk_cost_params_default(mk_cost_params *q) {
  if (!q) return;
  const CostParams c;
  q->sm_gbs = c.sm_gbs;
  q->ring_pages = c.ring_pages;
  q->exchange_us = c.exchange_us;
  q->page_us = c.page_us;
  q->attn_page_us = c.attn_page_us;
  q->attn_fixed_us = c.attn_fixed_us;
  q->merge_us = c.merge_us;
  q->instr_us = c.instr_us;
  q->launch_us = c.launch_us;
  q->tc_page_us = c.tc_page_us;
  q->cc_page_us_seq = c.cc_page_us_seq;
  q->conv_ctas = c.conv_ctas;
  q->merge_split_us = c.merge_split_us;
}

extern "C" int mk_host_plan_estimate(const mk_config *cfg, const mk_plan_opts *opts, int32_t num_ctas,
                                     int32_t context, const mk_cost_params *params, mk_cost_estimate *out,
                                     char *err, size_t err_len) {
  std::string why;
  int rc = check_cfg(cfg, &why);
  if (rc) {
    set_err(err, err_len, why);
    return rc;
  }
  if (num_ctas < 1 || context < 0 || context >= cfg->max_seq || !out) return MK_ERR_INVALID_ARG;
  mk_plan_opts o = opts ? *opts : default_opts(*cfg);
  if (o.batch < 1 || o.batch > cfg->max_batch || !tensor_opts_ok(o) || o.kv_splits < kSplitsByCost ||
      o.sched_mode < MK_SCHED_STATIC || o.sched_mode > MK_SCHED_EVENT)
    return MK_ERR_INVALID_ARG;
  PlanRequest req = make_request(*cfg, o, num_ctas);
  Plan p;
  std::string e = build_plan(req, &p);
  if (e.empty()) e = validate_plan(req, p);
  if (!e.empty()) {
    set_err(err, err_len, e);
    return MK_ERR_UNSUPPORTED_SHAPE;
  }
  CostEstimate est;
  e = estimate_plan(req, p, cost_params_from(params), context, &est);
  if (!e.empty()) {
    set_err(err, err_len, e);
    return MK_ERR_INVALID_ARG;
  }
  out->step_us = est.step_us;
  out->per_op_us = est.per_op_us;
  out->hbm_floor_us = est.hbm_floor_us;
  out->savings_us = est.per_op_us - est.step_us;
  for (int i = 0; i < 7; ++i) out->stage_us[i] = est.stage_us[i];
  return MK_OK;
}

// ====================================================================== tensor parallelism

// A tensor-parallel group of n ranks emulated on this GPU: rank r is a handle
// over its shard of the model (heads, FFN columns, vocabulary rows), and one
// cooperative launch of n * (SMs / n) CTAs runs every rank's plan, each block
// of SMs / n CTAs with its rank's parameters (ranks whose kernels wait on one
// another must run in one launch on one GPU).
struct mk_tp_group {
  int n = 0;
  mk_config cfg;                      // the full model's
  std::vector<mk_handle *> ranks;
  std::vector<void *> allocs;         // column shards of Wo and Wd
  std::vector<void *> plan_allocs;    // per plan: partial buffers, tables, I/O
  KParams *d_params = nullptr;        // [n]
  int32_t *d_tok = nullptr, *d_pos = nullptr, *d_next = nullptr;  // [B]
  float *d_logits = nullptr;          // [B][V]
  KParams launch{};                   // rank 0's parameters + the group table
  const void *kernel = nullptr;
  int smem = 0, ctas = 0, B = 1;
  bool planned = false;
};

extern "C" int mk_tp_create(const mk_config *cfg, const mk_weights *w, const mk_kv_cache *kv, int32_t n_ranks,
                            mk_tp_group **out) {
  if (out) *out = nullptr;
  if (!cfg || !w || !kv || !out || !w->layers) return MK_ERR_INVALID_ARG;
  if (n_ranks != 2 && n_ranks != 4 && n_ranks != 8) return MK_ERR_INVALID_ARG;
  std::string why;
  int rc = check_cfg(cfg, &why);
  if (rc) return rc;
  const int n = n_ranks;
  if (cfg->n_q_heads % n || cfg->n_kv_heads % n || cfg->ffn % n || cfg->vocab % n) return MK_ERR_UNSUPPORTED_SHAPE;
  if (!w->embed || !w->final_norm || (!cfg->tied_lm_head && !w->lm_head) || !kv->k || !kv->v)
    return MK_ERR_INVALID_ARG;
  mk_tp_group *g = new (std::nothrow) mk_tp_group();
  if (!g) return MK_ERR_OUT_OF_MEMORY;
  g->n = n;
  g->cfg = *cfg;
  auto fail = [&](int code) {
    cudaDeviceSynchronize();
    for (mk_handle *h : g->ranks) mk_destroy(h);
    free_list(g->allocs);
    delete g;
    return code;
  };
  const int H = cfg->hidden, d = cfg->head_dim, L = cfg->n_layers;
  const int qd_r = cfg->n_q_heads / n * d, kvd_r = cfg->n_kv_heads / n * d, F_r = cfg->ffn / n,
            V_r = cfg->vocab / n;
  const uint16_t *lm = (const uint16_t *)(cfg->tied_lm_head ? w->embed : w->lm_head);
  for (int r = 0; r < n; ++r) {
    mk_config rc_cfg = *cfg;
    rc_cfg.n_q_heads = cfg->n_q_heads / n;
    rc_cfg.n_kv_heads = cfg->n_kv_heads / n;
    rc_cfg.ffn = F_r;
    rc_cfg.vocab = V_r;
    rc_cfg.tied_lm_head = 0;
    std::vector<mk_layer_weights> lw(L);
    for (int l = 0; l < L; ++l) {
      const mk_layer_weights &S = w->layers[l];
      mk_layer_weights &D = lw[l];
      D = S;
      // row shards are views; column shards (Wo, Wd) are copied
      D.wq = (const uint16_t *)S.wq + (size_t)r * qd_r * H;
      D.wk = (const uint16_t *)S.wk + (size_t)r * kvd_r * H;
      D.wv = (const uint16_t *)S.wv + (size_t)r * kvd_r * H;
      D.w_gate = (const uint16_t *)S.w_gate + (size_t)r * F_r * H;
      D.w_up = (const uint16_t *)S.w_up + (size_t)r * F_r * H;
      uint16_t *wo = nullptr, *wd = nullptr;
      if ((rc = dalloc(g->allocs, &wo, (size_t)H * qd_r, false))) return fail(rc);
      if ((rc = dalloc(g->allocs, &wd, (size_t)H * F_r, false))) return fail(rc);
      cudaError_t e = cudaMemcpy2D(wo, (size_t)qd_r * 2, (const uint16_t *)S.wo + (size_t)r * qd_r,
                                   (size_t)cfg->n_q_heads * d * 2, (size_t)qd_r * 2, H, cudaMemcpyDeviceToDevice);
      if (e == cudaSuccess)
        e = cudaMemcpy2D(wd, (size_t)F_r * 2, (const uint16_t *)S.w_down + (size_t)r * F_r, (size_t)cfg->ffn * 2,
                         (size_t)F_r * 2, H, cudaMemcpyDeviceToDevice);
      if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(MK_ERR_CUDA);
      }
      D.wo = wo;
      D.w_down = wd;
    }
    mk_weights rw = *w;
    rw.lm_head = lm + (size_t)r * V_r * H;
    rw.layers = lw.data();
    // this rank's KV heads inside the caller's cache (strides of the full cache
    // are set when planning)
    mk_kv_cache rk;
    rk.k = (uint16_t *)kv->k + (size_t)r * (cfg->n_kv_heads / n) * cfg->max_seq * d;
    rk.v = (uint16_t *)kv->v + (size_t)r * (cfg->n_kv_heads / n) * cfg->max_seq * d;
    mk_handle *h = nullptr;
    if ((rc = mk_create(&rc_cfg, &rw, &rk, &h))) return fail(rc);
    g->ranks.push_back(h);
  }
  *out = g;
  return MK_OK;
}

static void tp_drop_plan(mk_tp_group *g) {
  free_list(g->plan_allocs);
  g->d_params = nullptr;
  g->planned = false;
}

extern "C" int mk_tp_plan(mk_tp_group *g, const mk_plan_opts *opts_in) {
  if (!g) return MK_ERR_INVALID_ARG;
  mk_plan_opts o = opts_in ? *opts_in : default_opts(g->cfg);
  // the rank build: batch 1, static per-SM queues, one launch
  if (o.batch != 1 || o.sched_mode != MK_SCHED_STATIC || o.kv_splits < 0 ||
      (o.exec_mode != MK_EXEC_MEGAKERNEL && o.exec_mode != MK_EXEC_MEGAKERNEL_GENERIC) || o.trace)
    return MK_ERR_INVALID_ARG;
  cudaDeviceSynchronize();
  tp_drop_plan(g);
  const int n = g->n;
  mk_handle *h0 = g->ranks[0];
  const int C = h0->sm_count / n;
  if (C < 1) return MK_ERR_LAUNCH;
  o.exec_mode = MK_EXEC_MEGAKERNEL_GENERIC;
  o.num_sms = C;
  int rc;
  for (mk_handle *h : g->ranks)
    if ((rc = mk_plan(h, &o))) return rc;
  const mk_config &c = g->cfg;
  const int B = 1, H = c.hidden, L = c.n_layers, V = c.vocab;
  const int ndp_r = h0->plan.ndp, n_lm_r = h0->plan.n_lm;
  for (mk_handle *h : g->ranks)
    if (h->plan.ndp != ndp_r || h->plan.n_lm != n_lm_r || h->smem != h0->smem) return MK_ERR_UNSUPPORTED_SHAPE;
  if (n * ndp_r > kMaxDownPieces) return MK_ERR_UNSUPPORTED_SHAPE;
  TpPeer *d_peers = nullptr;
  std::vector<TpPeer> peers(n);
  if ((rc = dalloc(g->plan_allocs, &d_peers, (size_t)n, false))) return rc;
  if ((rc = dalloc(g->plan_allocs, &g->d_params, (size_t)n, false))) return rc;
  if ((rc = dalloc(g->plan_allocs, &g->d_tok, (size_t)B))) return rc;
  if ((rc = dalloc(g->plan_allocs, &g->d_pos, (size_t)B))) return rc;
  if ((rc = dalloc(g->plan_allocs, &g->d_next, (size_t)B))) return rc;
  if ((rc = dalloc(g->plan_allocs, &g->d_logits, (size_t)B * V))) return rc;
  std::vector<KParams> kp(n);
  for (int r = 0; r < n; ++r) {
    mk_handle *h = g->ranks[r];
    KParams &k = kp[r];
    k = h->kp;
    // every rank's copies of the cross-rank buffers (zeroed: no step tag yet)
    if ((rc = dalloc(g->plan_allocs, &k.opart, (size_t)L * n * B * H))) return rc;
    if ((rc = dalloc(g->plan_allocs, &k.dpart, (size_t)L * n * ndp_r * B * H))) return rc;
    if ((rc = dalloc(g->plan_allocs, &k.arg_val, (size_t)B * n * n_lm_r))) return rc;
    if ((rc = dalloc(g->plan_allocs, &k.arg_idx, (size_t)B * n * n_lm_r))) return rc;
    peers[r] = TpPeer{k.opart, k.dpart, k.ctr, k.arg_val, k.arg_idx};
    k.tp_n = n;
    k.tp_rank = r;
    k.tp_ctas = C;
    k.tp_peers = d_peers;
    k.ndp_local = ndp_r;
    k.ndp = n * ndp_r;
    k.n_lm_local = n_lm_r;
    k.n_lm = n * n_lm_r;
    k.n_gu_layer = h->plan.n_gu;
    k.V = V;
    k.V_lm = V / n;
    k.lm_row0 = r * (V / n);
    // the caller's full cache: this rank's heads, full strides
    k.kv_hs = (long long)c.max_seq * c.head_dim;
    k.kv_bs = k.kv_hs * c.n_kv_heads;
    k.kv_ls = k.kv_bs * c.max_batch;
    k.tokens = g->d_tok;
    k.positions = g->d_pos;
    k.logits = g->d_logits;
    k.next_tokens = g->d_next;
    k.mode = MODE_FINAL_LAUNCH;
    // the O and down counters count every rank's producers
    std::vector<Instr> ins = h->plan.instrs;
    for (Instr &I : ins)
      if ((I.op == OP_GATEUP) || (I.op == OP_QKV && I.layer > 0) || I.op == OP_LMHEAD) I.wait_cnt *= (uint32_t)n;
    cudaError_t e = cudaMemcpy(const_cast<Instr *>(k.instrs), ins.data(), ins.size() * sizeof(Instr),
                               cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return MK_ERR_CUDA;
    }
  }
  cudaError_t e = cudaMemcpy(d_peers, peers.data(), sizeof(TpPeer) * n, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(g->d_params, kp.data(), sizeof(KParams) * n, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  g->kernel = interp_kernel_tp();
  g->smem = h0->smem;
  g->ctas = C;
  g->B = B;
  int per_sm = 0;
  e = interp_prepare(g->kernel, g->smem, &per_sm);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MK_ERR_CUDA;
  }
  if (per_sm < 1) return MK_ERR_LAUNCH;
  g->launch = kp[0];
  g->launch.tp_params = g->d_params;
  g->planned = true;
  return MK_OK;
}

extern "C" int mk_tp_decode_step(mk_tp_group *g, const int32_t *tokens, const int32_t *positions, float *logits_out,
                                 int32_t *next_tokens_out, void *stream) {
  if (!g || !tokens || !positions || !next_tokens_out) return MK_ERR_INVALID_ARG;
  if (!g->planned) return MK_ERR_NOT_PLANNED;
  cudaStream_t st = (cudaStream_t)stream;
  MK_CUDA(cudaMemcpyAsync(g->d_tok, tokens, sizeof(int32_t) * g->B, cudaMemcpyDeviceToDevice, st));
  MK_CUDA(cudaMemcpyAsync(g->d_pos, positions, sizeof(int32_t) * g->B, cudaMemcpyDeviceToDevice, st));
  cudaError_t e = launch_interp(g->kernel, g->launch, g->n * g->ctas, g->smem, st, true);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_code(e);
  }
  if (logits_out)
    MK_CUDA(cudaMemcpyAsync(logits_out, g->d_logits, sizeof(float) * g->B * g->cfg.vocab, cudaMemcpyDeviceToDevice,
                            st));
  MK_CUDA(cudaMemcpyAsync(next_tokens_out, g->d_next, sizeof(int32_t) * g->B, cudaMemcpyDeviceToDevice, st));
  return MK_OK;
}

extern "C" int mk_tp_get_status(mk_tp_group *g, void *stream) {
  if (!g) return MK_ERR_INVALID_ARG;
  int first = MK_OK;
  for (mk_handle *h : g->ranks) {
    const int rc = mk_get_status(h, stream);
    if (rc != MK_OK && first == MK_OK) first = rc;
  }
  // a failed step leaves the ranks' counters and step numbers apart: plan again
  if (first != MK_OK) tp_drop_plan(g);
  return first;
}

extern "C" void mk_tp_destroy(mk_tp_group *g) {
  if (!g) return;
  cudaDeviceSynchronize();
  tp_drop_plan(g);
  for (mk_handle *h : g->ranks) mk_destroy(h);
  free_list(g->allocs);
  delete g;
}
