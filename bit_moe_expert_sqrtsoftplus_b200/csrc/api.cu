// api.cu -- the extern "C" boundary declared in include/moe.h.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <new>
#include <string>

#include "../../include/moe.h"
#include "gemm.cuh"
#include "layer.cuh"
#include "prefill.cuh"
#include "q4k.cuh"
#include "quant.cuh"

static_assert(MOE_SMALL_T_MAX == moe::kDecodeMaxT, "header and kernels disagree on the small-T limit");
// q2 layers with up to this many tokens run the small-token kernels twice
constexpr int kChunkedMaxT = MOE_CHUNKED_T_MAX;
static_assert(kChunkedMaxT == 2 * moe::kDecodeMaxT, "two small-token chunks");

constexpr int kGemmMaps = 3;  // tensor maps of gate, up and down for the batched path

struct moe_handle {
  moe_config cfg;
  moe_weights w;
  moe::LayerDims d;
  moe::LayerWeights wt;
  int *err;          // device error word inside persist
  float *row_norms;  // [E] 2-norms of the router rows (fp32), inside persist
  int num_sms;
  int device;
  cudaEvent_t ev_begin, ev_end;  // optional timing of the dominant kernel
  moe::NextLayerPrefetch next;   // the next layer's first-read weights (stack decode)
  moe::TensorMap gemm_tm_host[kGemmMaps];  // host copies of wt.gemm_tm's maps
};

namespace {

thread_local std::string g_last_error;

moe_status fail(moe_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
moe_status fail(moe_status s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

moe_status cuda_fail(cudaError_t e, const char *where) {
  return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kPersistHeader = 256;

size_t persist_bytes_for(const moe_config &c) {
  // header, row norms, then (64-byte aligned) the batched path's tensor maps
  return kPersistHeader + sizeof(float) * (size_t)(c.n_experts > 0 ? c.n_experts : 0) + 64 +
         kGemmMaps * sizeof(moe::TensorMap) + 256;
}

// MOE_GEMM_TMA=0 in the environment turns the TMA staging of the batched
// path's packed weight tiles off for handles created afterwards (the
// producers then load the packed bytes themselves; results are identical).
bool gemm_tma_wanted() {
  const char *v = getenv("MOE_GEMM_TMA");
  return !(v && v[0] == '0' && v[1] == 0);
}

moe_status check_config(const moe_config *c) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "config is NULL");
  if (c->hidden <= 0 || c->hidden % 256)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "hidden=%d must be a positive multiple of 256", c->hidden);
  if (c->inter <= 0 || c->inter % 256)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "inter=%d must be a positive multiple of 256", c->inter);
  if (c->shared_inter <= 0 || c->shared_inter % 256)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "shared_inter=%d must be a positive multiple of 256", c->shared_inter);
  if (c->top_k < 1 || c->top_k > moe::kMaxK)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "top_k=%d must be in 1..%d", c->top_k, moe::kMaxK);
  if (c->n_experts < c->top_k || c->n_experts > moe::kMaxE)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n_experts=%d must be in top_k..%d", c->n_experts, moe::kMaxE);
  if (c->mode != MOE_ROUTE_ROUTER && c->mode != MOE_ROUTE_HASH)
    return fail(MOE_ERR_INVALID_ARG, "mode=%d is not a moe_route_mode", c->mode);
  if (c->mode == MOE_ROUTE_HASH && c->vocab <= 0)
    return fail(MOE_ERR_INVALID_ARG, "hash mode needs vocab > 0 (got %d)", c->vocab);
  if (!isfinite(c->routed_scaling)) return fail(MOE_ERR_INVALID_ARG, "routed_scaling is not finite");
  if ((c->flags & MOE_FLAG_PRENORM_RESIDUAL) && !(c->rms_eps >= 0.f && isfinite(c->rms_eps)))
    return fail(MOE_ERR_INVALID_ARG, "rms_eps must be finite and >= 0");
  if (c->flags & ~(MOE_FLAG_PRENORM_RESIDUAL | MOE_FLAG_EXPERTS_ONLY | MOE_FLAG_NO_ROUTED | MOE_FLAG_DETERMINISTIC))
    return fail(MOE_ERR_INVALID_ARG, "unknown flags 0x%x", c->flags);
  if ((c->flags & MOE_FLAG_EXPERTS_ONLY) && (c->flags & MOE_FLAG_NO_ROUTED))
    return fail(MOE_ERR_INVALID_ARG, "MOE_FLAG_EXPERTS_ONLY and MOE_FLAG_NO_ROUTED exclude each other");
  if (c->routed_format != MOE_ROUTED_Q2 && c->routed_format != MOE_ROUTED_Q4K)
    return fail(MOE_ERR_INVALID_ARG, "routed_format=%d is not a MOE_ROUTED_* format", c->routed_format);
  return MOE_OK;
}

moe::LayerDims dims_of(const moe_config &c) {
  moe::LayerDims d;
  d.H = c.hidden;
  d.I = c.inter;
  d.Is = c.shared_inter;
  d.E = c.n_experts;
  d.k = c.top_k;
  d.mode = c.mode;
  d.flags = c.flags;
  d.vocab = c.vocab;
  d.scaling = c.routed_scaling;
  d.eps = c.rms_eps;
  d.wait_cycles = moe::kDefaultWaitCycles;
  // MOE_SHARED_DENSE=0 in the environment keeps the batched path's shared
  // expert on per-tile Q8_0 decoding (results are identical)
  const char *sd = getenv("MOE_SHARED_DENSE");
  d.shared_dense = (sd && sd[0] == '0' && sd[1] == 0) ? 0 : 1;
  return d;
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

size_t scratch_bytes_for(const moe::LayerDims &d, int max_tokens) {
  size_t dec = moe::decode_scratch_bytes(d, max_tokens < moe::kDecodeMaxT ? max_tokens : moe::kDecodeMaxT);
  size_t pre = max_tokens > moe::kDecodeMaxT ? moe::prefill_scratch_bytes(d, max_tokens) : 0;
  return dec > pre ? dec : pre;
}

// Q4_K forward (T <= kDecodeMaxT): the routing scratch, then idx and w, then
// the expert kernels' buffers.
size_t q4k_scratch_bytes(const moe::LayerDims &d, int T) {
  return align256(moe::decode_scratch_bytes(d, T)) + 2 * align256(sizeof(int32_t) * (size_t)T * d.k) +
         moe::q4k_expert_bytes(d, T);
}

size_t scratch_bytes_for(const moe_config &c, int max_tokens) {
  const moe::LayerDims d = dims_of(c);
  size_t s = scratch_bytes_for(d, max_tokens);
  if (c.routed_format == MOE_ROUTED_Q4K) {
    const size_t q = q4k_scratch_bytes(d, max_tokens < moe::kDecodeMaxT ? max_tokens : moe::kDecodeMaxT);
    s = q > s ? q : s;
  }
  return s;
}

// The kernels run on the current device with the handle's pointers, which
// belong to the device that was current at moe_init.
moe_status check_device(const moe_handle *h) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != h->device)
    return fail(MOE_ERR_INVALID_ARG, "the current device (%d) is not the handle's device (%d)", dev, h->device);
  return MOE_OK;
}

moe_status check_whole_layer(const moe_handle *h) {
  if (h->d.flags & (MOE_FLAG_EXPERTS_ONLY | MOE_FLAG_NO_ROUTED))
    return fail(MOE_ERR_INVALID_ARG, "a handle made with MOE_FLAG_EXPERTS_ONLY or MOE_FLAG_NO_ROUTED serves the "
                                     "moe_ep_* calls only");
  return MOE_OK;
}

moe_status check_call(moe_handle *h, const float *x, const int32_t *token_ids, int T, void *scratch,
                      size_t scratch_bytes) {
  if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d is negative", T);
  if (T == 0) return MOE_OK;
  if (!x) return fail(MOE_ERR_INVALID_ARG, "x is NULL");
  if (!aligned16(x)) return fail(MOE_ERR_MISALIGNED, "x is not 16-byte aligned");
  if (h->d.mode == MOE_ROUTE_HASH && !token_ids) return fail(MOE_ERR_INVALID_ARG, "hash mode needs token_ids");
  if (!scratch) return fail(MOE_ERR_INVALID_ARG, "scratch is NULL");
  if (!aligned16(scratch)) return fail(MOE_ERR_MISALIGNED, "scratch is not 16-byte aligned");
  const size_t need = scratch_bytes_for(h->cfg, T);
  if (scratch_bytes < need)
    return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "scratch has %zu bytes, %zu needed for T=%d", scratch_bytes, need, T);
  return check_device(h);
}

}  // namespace

extern "C" {

const char *moe_last_error(void) { return g_last_error.c_str(); }

moe_status moe_workspace_size(const moe_config *cfg, int max_tokens, size_t *persist_bytes, size_t *scratch_bytes) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (max_tokens < 0) return fail(MOE_ERR_INVALID_ARG, "max_tokens=%d is negative", max_tokens);
  if (persist_bytes) *persist_bytes = persist_bytes_for(*cfg);
  if (scratch_bytes) *scratch_bytes = max_tokens > 0 ? scratch_bytes_for(*cfg, max_tokens) : 0;
  g_last_error.clear();
  return MOE_OK;
}

moe_status moe_init(const moe_config *cfg, const moe_weights *w, void *persist, size_t persist_bytes,
                    moe_stream_t stream, moe_handle **out) {
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!w) return fail(MOE_ERR_INVALID_ARG, "weights is NULL");
  const bool experts_only = (cfg->flags & MOE_FLAG_EXPERTS_ONLY) != 0;
  const bool no_routed = (cfg->flags & MOE_FLAG_NO_ROUTED) != 0;
  const void *need[] = {w->gate_iq2xxs, w->up_iq2xxs, w->down_q2k, w->iq2_grid, w->sh_gate_q80, w->sh_up_q80,
                        w->sh_down_q80};
  const char *names[] = {"gate_iq2xxs", "up_iq2xxs", "down_q2k", "iq2_grid", "sh_gate_q80", "sh_up_q80",
                         "sh_down_q80"};
  for (int i = 0; i < 7; ++i) {
    const bool routed = i < 4;
    if (routed && no_routed) continue;                                   // router and shared expert only
    if (!routed && experts_only) continue;                               // routed experts only
    if (i == 3 && cfg->routed_format == MOE_ROUTED_Q4K) continue;        // Q4_K layers read no codebook
    if (!need[i]) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned16(need[i])) return fail(MOE_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
  }
  if (experts_only) {
    // no routing
  } else if (cfg->mode == MOE_ROUTE_ROUTER) {
    if (!w->router_w_f16 || !w->router_bias) return fail(MOE_ERR_INVALID_ARG, "router mode needs router_w_f16 and router_bias");
    if (!aligned16(w->router_w_f16) || !aligned16(w->router_bias))
      return fail(MOE_ERR_MISALIGNED, "router weights are not 16-byte aligned");
  } else {
    if (!w->tid2eid) return fail(MOE_ERR_INVALID_ARG, "hash mode needs tid2eid");
    if (!aligned16(w->tid2eid)) return fail(MOE_ERR_MISALIGNED, "tid2eid is not 16-byte aligned");
  }
  if (!persist) return fail(MOE_ERR_INVALID_ARG, "persist is NULL");
  if (!aligned16(persist)) return fail(MOE_ERR_MISALIGNED, "persist is not 16-byte aligned");
  if (persist_bytes < persist_bytes_for(*cfg))
    return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "persist has %zu bytes, %zu needed", persist_bytes,
                persist_bytes_for(*cfg));

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");

  moe_handle *h = new (std::nothrow) moe_handle;
  if (!h) return fail(MOE_ERR_INVALID_ARG, "out of host memory");
  h->cfg = *cfg;
  h->w = *w;
  h->d = dims_of(*cfg);
  h->wt.Wr = static_cast<const uint16_t *>(w->router_w_f16);
  h->wt.bias = w->router_bias;
  h->wt.tid2eid = w->tid2eid;
  h->wt.gate = static_cast<const uint8_t *>(w->gate_iq2xxs);
  h->wt.up = static_cast<const uint8_t *>(w->up_iq2xxs);
  h->wt.down = static_cast<const uint8_t *>(w->down_q2k);
  h->wt.sh_gate = static_cast<const uint8_t *>(w->sh_gate_q80);
  h->wt.sh_up = static_cast<const uint8_t *>(w->sh_up_q80);
  h->wt.sh_down = static_cast<const uint8_t *>(w->sh_down_q80);
  h->wt.grid = w->iq2_grid;
  h->wt.tma = 0;
  if (cfg->routed_format == MOE_ROUTED_Q2 && !no_routed && !experts_only) moe::build_chunk_tensor_maps(h->wt, h->d);
  h->err = static_cast<int *>(persist);
  h->row_norms = reinterpret_cast<float *>(static_cast<uint8_t *>(persist) + kPersistHeader);
  h->wt.gemm_tm = nullptr;
  h->num_sms = sms;
  h->device = dev;
  h->ev_begin = nullptr;
  h->ev_end = nullptr;
  h->next = moe::NextLayerPrefetch{};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  e = cudaMemsetAsync(persist, 0, kPersistHeader, s);
  if (e != cudaSuccess) {
    delete h;
    return cuda_fail(e, "cudaMemsetAsync(persist)");
  }
  if (cfg->routed_format == MOE_ROUTED_Q2 && !no_routed && gemm_tma_wanted()) {
    // tensor maps of the routed matrices, all experts' rows stacked
    const size_t rbI = (size_t)(cfg->hidden / 256) * 66, rbD = (size_t)(cfg->inter / 256) * 84;
    const size_t E = (size_t)cfg->n_experts;
    const uintptr_t at = reinterpret_cast<uintptr_t>(h->row_norms + E);
    void *maps = reinterpret_cast<void *>((at + 63) & ~uintptr_t(63));
    if (moe::gemm_tensor_map(&h->gemm_tm_host[0], h->wt.gate, rbI, E * cfg->inter, moe::kFmtIQ2) &&
        moe::gemm_tensor_map(&h->gemm_tm_host[1], h->wt.up, rbI, E * cfg->inter, moe::kFmtIQ2) &&
        moe::gemm_tensor_map(&h->gemm_tm_host[2], h->wt.down, rbD, E * cfg->hidden, moe::kFmtQ2K)) {
      e = cudaMemcpyAsync(maps, h->gemm_tm_host, kGemmMaps * sizeof(moe::TensorMap), cudaMemcpyHostToDevice, s);
      if (e != cudaSuccess) {
        delete h;
        return cuda_fail(e, "copying tensor maps");
      }
      h->wt.gemm_tm = maps;
    }
  }
  if (!experts_only) e = moe::prefill_init(h->d, h->wt, h->row_norms, h->err, s);
  if (e != cudaSuccess) {
    delete h;
    return cuda_fail(e, "init kernels");
  }
  if (cfg->mode == MOE_ROUTE_HASH && !experts_only) {
    // the kernels index the weights with the table's ids and assume a token
    // selects an expert once: check every row before the handle is used
    int bad = -1;
    e = moe::check_tid2eid(h->d, w->tid2eid, h->err + 1, &bad, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(h->err + 1, 0, sizeof(int), s);
    if (e != cudaSuccess) {
      delete h;
      return cuda_fail(e, "checking tid2eid");
    }
    if (bad >= 0) {
      delete h;
      return fail(MOE_ERR_INVALID_ARG, "tid2eid row %d does not hold %d distinct expert ids in [0, %d)", bad,
                  cfg->top_k, cfg->n_experts);
    }
  }
  *out = h;
  g_last_error.clear();
  return MOE_OK;
}

static moe::DecodeArgs decode_args(moe_handle *h, const float *x, const int32_t *token_ids, int T, float *y,
                                   void *scratch) {
  moe::DecodeArgs a;
  a.d = h->d;
  a.wt = h->wt;
  a.pf = h->next;
  a.T = T;
  a.x = x;
  a.token_ids = token_ids;
  a.y = y;
  moe::decode_carve(a.s, h->d, T, scratch);
  a.err = h->err;
  a.ev_begin = h->ev_begin;
  a.ev_end = h->ev_end;
  return a;
}

// Routing as the small-token path does it, then the Q4_K expert kernels.
static cudaError_t q4k_forward(moe_handle *h, const float *x, const int32_t *token_ids, int T, float *y, void *scratch,
                               cudaStream_t s) {
  uint8_t *base = static_cast<uint8_t *>(scratch);
  size_t off = align256(moe::decode_scratch_bytes(h->d, T));
  int32_t *idx = reinterpret_cast<int32_t *>(base + off);
  off += align256(sizeof(int32_t) * (size_t)T * h->d.k);
  float *w = reinterpret_cast<float *>(base + off);
  off += align256(sizeof(float) * (size_t)T * h->d.k);
  moe::DecodeArgs a = decode_args(h, x, token_ids, T, nullptr, scratch);
  a.ev_begin = a.ev_end = nullptr;
  cudaError_t e = moe::decode_route(a, idx, w, s);
  if (e != cudaSuccess) return e;
  moe::Q4kArgs q;
  q.d = h->d;
  q.gate = h->wt.gate;
  q.up = h->wt.up;
  q.down = h->wt.down;
  q.sh_gate = h->wt.sh_gate;
  q.sh_up = h->wt.sh_up;
  q.sh_down = h->wt.sh_down;
  q.T = T;
  q.x = x;
  q.y = y;
  q.idx = idx;
  q.w = w;
  q.h = reinterpret_cast<float *>(base + off);
  off += align256(sizeof(float) * (size_t)T * h->d.k * h->d.I);
  q.hs = reinterpret_cast<float *>(base + off);
  off += align256(sizeof(float) * (size_t)T * h->d.Is);
  q.xsum = reinterpret_cast<float *>(base + off);
  off += align256(sizeof(float) * (size_t)T * (h->d.H / 32));
  const size_t nh = (size_t)T * h->d.k * h->d.I + (size_t)T * h->d.Is;
  q.hq = reinterpret_cast<int8_t *>(base + off);
  off += align256(3 * nh);
  q.hqs = reinterpret_cast<float *>(base + off);
  off += align256(sizeof(float) * 4 * ((size_t)T * h->d.k + T));
  q.hsum = reinterpret_cast<float *>(base + off);
  q.xq = a.s.xq;
  q.xs = a.s.xs;
  if (h->ev_begin) cudaEventRecord(h->ev_begin, s);
  e = moe::q4k_experts(q, s);
  if (h->ev_end) cudaEventRecord(h->ev_end, s);
  return e;
}

moe_status moe_route(moe_handle *h, const float *x, const int32_t *token_ids, int T, int32_t *idx, float *w,
                     int32_t *expert_offsets, int32_t *perm, void *scratch, size_t scratch_bytes,
                     moe_stream_t stream) {
  moe_status st = check_call(h, x, token_ids, T, scratch, scratch_bytes);
  if (st != MOE_OK) return st;
  if (h->d.flags & MOE_FLAG_EXPERTS_ONLY)
    return fail(MOE_ERR_INVALID_ARG, "a MOE_FLAG_EXPERTS_ONLY handle has no router");
  if (T == 0) return MOE_OK;
  if (!idx || !w) return fail(MOE_ERR_INVALID_ARG, "idx and w must not be NULL");
  if ((expert_offsets == nullptr) != (perm == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "expert_offsets and perm must both be set or both be NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (T <= moe::kDecodeMaxT) {
    moe::DecodeArgs a = decode_args(h, x, token_ids, T, nullptr, scratch);
    e = moe::decode_route(a, idx, w, s);
  } else {
    moe::PrefillArgs p = moe::prefill_args(h->d, h->wt, T, x, token_ids, nullptr, scratch, h->row_norms, h->err);
    e = moe::prefill_route(p, idx, w, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "moe_route launch");
  if (perm) {
    e = moe::permute(idx, T, h->d.k, h->d.E, expert_offsets, perm, s);
    if (e != cudaSuccess) return cuda_fail(e, "moe_route permutation");
  }
  g_last_error.clear();
  return MOE_OK;
}

moe_status moe_ffn_forward(moe_handle *h, const float *x, const int32_t *token_ids, int T, float *y, void *scratch,
                           size_t scratch_bytes, moe_stream_t stream) {
  if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  moe_status st = check_whole_layer(h);
  if (st != MOE_OK) return st;
  if ((st = check_call(h, x, token_ids, T, scratch, scratch_bytes)) != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!y) return fail(MOE_ERR_INVALID_ARG, "y is NULL");
  if (!aligned16(y)) return fail(MOE_ERR_MISALIGNED, "y is not 16-byte aligned");
  if (y == x && !(h->d.flags & MOE_FLAG_PRENORM_RESIDUAL))
    return fail(MOE_ERR_INVALID_ARG, "y may alias x only with MOE_FLAG_PRENORM_RESIDUAL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (h->cfg.routed_format == MOE_ROUTED_Q4K && T <= moe::kDecodeMaxT) {
    e = q4k_forward(h, x, token_ids, T, y, scratch, s);
  } else if (T <= moe::kDecodeMaxT) {
    moe::DecodeArgs a = decode_args(h, x, token_ids, T, y, scratch);
    e = moe::decode_forward(a, s, h->num_sms);
  } else if (T <= kChunkedMaxT && h->cfg.routed_format == MOE_ROUTED_Q2) {
    // two small-token calls, the first 32 tokens and the rest, one after the
    // other on the stream (a token's result depends on its own row only, so
    // the split changes no bit of it): each chunk reads the union of its own
    // tokens' experts, which up to 64 tokens costs less than the batched
    // path's fixed work (measured on B200 at 64 tokens: 1.54 against 1.88 ms)
    moe::DecodeArgs a0 = decode_args(h, x, token_ids, moe::kDecodeMaxT, y, scratch);
    e = moe::decode_forward(a0, s, h->num_sms);
    if (e == cudaSuccess) {
      const size_t off = (size_t)moe::kDecodeMaxT * h->d.H;
      moe::DecodeArgs a1 = decode_args(h, x + off, token_ids ? token_ids + moe::kDecodeMaxT : nullptr,
                                       T - moe::kDecodeMaxT, y + off, scratch);
      e = moe::decode_forward(a1, s, h->num_sms);
    }
  } else {
    moe::PrefillArgs p = moe::prefill_args(h->d, h->wt, T, x, token_ids, y, scratch, h->row_norms, h->err);
    p.ev_begin = h->ev_begin;
    p.ev_end = h->ev_end;
    p.q4k = h->cfg.routed_format == MOE_ROUTED_Q4K;
    e = moe::prefill_forward(p, s, h->num_sms);
  }
  if (e != cudaSuccess) return cuda_fail(e, "moe_ffn_forward launch");
  g_last_error.clear();
  return MOE_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ no-allocation forward
//
// Scratch for moe_ffn_forward_noalloc: one buffer per device that loads this
// library, held until the process exits.  Host code must not take the
// array's address directly (its name stands for a host-side shadow); the
// device address comes from cudaGetSymbolAddress with the device current.
// It is looked up again on every call made outside stream capture (after a
// cudaDeviceReset the module is loaded anew and the array may move) and the
// last address is kept per device for calls made during a capture.
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kNoAllocMaxT = 8;                            // tokens per call of the no-alloc forward
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 128;
void *g_static_scratch_addr[kMaxDevices] = {};
std::mutex g_static_scratch_mutex;

moe_status static_scratch_for(int dev, cudaStream_t stream, void **out) {
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_INVALID_ARG, "device ordinal %d out of range", dev);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t ce = cudaStreamIsCapturing(stream, &cap);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaStreamIsCapturing");
  std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
  if (!g_static_scratch_addr[dev] || cap == cudaStreamCaptureStatusNone) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    g_static_scratch_addr[dev] = p;
  }
  *out = g_static_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_ffn_forward_noalloc(moe_handle *h, const float *x, const int32_t *token_ids, int T, float *y,
                                   moe_stream_t stream) {
  if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d is negative", T);
  moe_status wl = check_whole_layer(h);
  if (wl != MOE_OK) return wl;
  if (T == 0) return MOE_OK;
  if (h->cfg.routed_format != MOE_ROUTED_Q2)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_ffn_forward_noalloc runs the q2 routed formats only");
  if (T > kNoAllocMaxT)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_ffn_forward_noalloc handles at most %d tokens per call (got %d)",
                kNoAllocMaxT, T);
  const size_t need = moe::decode_scratch_bytes(h->d, T);
  if (need > kStaticScratchBytes)
    return fail(MOE_ERR_WORKSPACE_TOO_SMALL,
                "this layer needs %zu bytes of scratch for T=%d; the built-in buffer holds %zu bytes", need, T,
                kStaticScratchBytes);
  if (!x || !y) return fail(MOE_ERR_INVALID_ARG, "x and y must not be NULL");
  if (!aligned16(x) || !aligned16(y)) return fail(MOE_ERR_MISALIGNED, "x and y must be 16-byte aligned");
  if (h->d.mode == MOE_ROUTE_HASH && !token_ids) return fail(MOE_ERR_INVALID_ARG, "hash mode needs token_ids");
  if (y == x && !(h->d.flags & MOE_FLAG_PRENORM_RESIDUAL))
    return fail(MOE_ERR_INVALID_ARG, "y may alias x only with MOE_FLAG_PRENORM_RESIDUAL");
  moe_status st = check_device(h);
  if (st != MOE_OK) return st;
  void *scratch = nullptr;
  st = static_scratch_for(h->device, reinterpret_cast<cudaStream_t>(stream), &scratch);
  if (st != MOE_OK) return st;
  moe::DecodeArgs a = decode_args(h, x, token_ids, T, y, scratch);
  const cudaError_t e = moe::decode_forward(a, reinterpret_cast<cudaStream_t>(stream), h->num_sms);
  if (e != cudaSuccess) return cuda_fail(e, "moe_ffn_forward_noalloc launch");
  g_last_error.clear();
  return MOE_OK;
}

moe_status moe_poll_device_error(moe_handle *h, moe_stream_t stream) {
  if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int code = 0;
  e = cudaMemcpy(&code, h->err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (code != 0) {
    const int zero = 0;
    e = cudaMemcpy(h->err, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    switch (code) {
      case MOE_ERR_TIMEOUT:
        return fail(MOE_ERR_TIMEOUT, "a bounded device wait ran out");
      case MOE_ERR_UNSUPPORTED_SHAPE:
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "an IQ2_XXS codebook entry exceeds 127");
      case MOE_ERR_INVALID_ARG:
        return fail(MOE_ERR_INVALID_ARG, "a token id was outside [0, vocab)");
      default:
        return fail(MOE_ERR_DEVICE_FAULT, "device error code %d", code);
    }
  }
  g_last_error.clear();
  return MOE_OK;
}

moe_status moe_set_wait_limit(moe_handle *h, long long cycles) {
  if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (cycles < 0) return fail(MOE_ERR_INVALID_ARG, "cycles=%lld is negative", cycles);
  h->d.wait_cycles = cycles > 0 ? cycles : moe::kDefaultWaitCycles;
  g_last_error.clear();
  return MOE_OK;
}

moe_status moe_set_next_layer(moe_handle *h, const moe_handle *next) {
  if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  h->next = moe::NextLayerPrefetch{};
  if (next) {
    if (next->device != h->device) return fail(MOE_ERR_INVALID_ARG, "the next layer's handle is on another device");
    const moe::LayerDims &d = next->d;
    if (next->wt.Wr) {
      h->next.ptr[0] = next->wt.Wr;
      h->next.bytes[0] = (size_t)d.E * d.H * 2;
    }
    if (next->wt.sh_gate && next->wt.sh_up) {
      h->next.ptr[1] = next->wt.sh_gate;
      h->next.ptr[2] = next->wt.sh_up;
      h->next.bytes[1] = h->next.bytes[2] = (size_t)d.Is * (d.H / 32) * 34;
    }
  }
  g_last_error.clear();
  return MOE_OK;
}

moe_status moe_set_timing_events(moe_handle *h, void *ev_begin, void *ev_end) {
  if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if ((ev_begin == nullptr) != (ev_end == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "ev_begin and ev_end must both be set or both be NULL");
  h->ev_begin = static_cast<cudaEvent_t>(ev_begin);
  h->ev_end = static_cast<cudaEvent_t>(ev_end);
  g_last_error.clear();
  return MOE_OK;
}

moe_status moe_quantize(int format, const float *x, int64_t n, void *out, int32_t *nonfinite_blocks,
                        moe_stream_t stream) {
  if (format != MOE_QUANT_Q8_0 && format != MOE_QUANT_Q2_K && format != MOE_QUANT_Q4_K)
    return fail(MOE_ERR_INVALID_ARG, "format=%d is not a MOE_QUANT_* format", format);
  if (n < 0) return fail(MOE_ERR_INVALID_ARG, "n=%lld is negative", (long long)n);
  const int per = format == MOE_QUANT_Q8_0 ? 32 : 256;
  if (n % per)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "n=%lld is not a multiple of the block size %d", (long long)n, per);
  if (n == 0) {
    g_last_error.clear();
    return MOE_OK;
  }
  if (!x || !out) return fail(MOE_ERR_INVALID_ARG, "x and out must not be NULL");
  if (!aligned16(x) || !aligned16(out)) return fail(MOE_ERR_MISALIGNED, "x and out must be 16-byte aligned");
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  e = moe::quantize_blocks(format, x, n / per, out, nonfinite_blocks, reinterpret_cast<cudaStream_t>(stream), sms);
  if (e != cudaSuccess) return cuda_fail(e, "moe_quantize launch");
  g_last_error.clear();
  return MOE_OK;
}

// ------------------------------------------------------------------ expert parallelism

moe_status moe_ep_workspace_size(const moe_config *cfg, int max_tokens, int max_recv_rows, size_t *dispatch_bytes,
                                 size_t *experts_bytes, size_t *combine_bytes) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (max_tokens < 0 || max_recv_rows < 0) return fail(MOE_ERR_INVALID_ARG, "negative sizes");
  const moe::LayerDims d = dims_of(*cfg);
  if (dispatch_bytes) *dispatch_bytes = max_tokens > 0 ? moe::ep_dispatch_scratch_bytes(d, max_tokens) : 0;
  if (experts_bytes) *experts_bytes = max_recv_rows > 0 ? moe::ep_experts_scratch_bytes(d, max_recv_rows) : 0;
  if (combine_bytes) *combine_bytes = max_tokens > 0 ? moe::ep_combine_scratch_bytes(d, max_tokens) : 0;
  g_last_error.clear();
  return MOE_OK;
}

moe_status moe_ep_dispatch(moe_handle *h, const float *x, const int32_t *token_ids, int T, int32_t *expert_offsets,
                           int32_t *perm, void *x_send, int32_t *e_send, float *w_send, void *scratch,
                           size_t scratch_bytes, moe_stream_t stream) {
  if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (h->d.flags & MOE_FLAG_EXPERTS_ONLY) return fail(MOE_ERR_INVALID_ARG, "an experts-only handle has no router");
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d is negative", T);
  if (T == 0) return MOE_OK;
  if (!x || !expert_offsets || !perm || !x_send || !e_send || !w_send || !scratch)
    return fail(MOE_ERR_INVALID_ARG, "a pointer argument is NULL");
  if (!aligned16(x) || !aligned16(x_send) || !aligned16(scratch))
    return fail(MOE_ERR_MISALIGNED, "x, x_send and scratch must be 16-byte aligned");
  if (h->d.mode == MOE_ROUTE_HASH && !token_ids) return fail(MOE_ERR_INVALID_ARG, "hash mode needs token_ids");
  const size_t need = moe::ep_dispatch_scratch_bytes(h->d, T);
  if (scratch_bytes < need)
    return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "scratch has %zu bytes, %zu needed for T=%d", scratch_bytes, need, T);
  moe_status st = check_device(h);
  if (st != MOE_OK) return st;
  moe::PrefillArgs p = moe::prefill_args(h->d, h->wt, T, x, token_ids, nullptr, scratch, h->row_norms, h->err);
  const cudaError_t e = moe::ep_dispatch(p, expert_offsets, perm, static_cast<__half *>(x_send), e_send, w_send,
                                         reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "moe_ep_dispatch launch");
  g_last_error.clear();
  return MOE_OK;
}

moe_status moe_ep_experts(moe_handle *shard, const void *x_recv, const int32_t *e_recv, const float *w_recv, int N,
                          int first_expert, float *out, void *scratch, size_t scratch_bytes, moe_stream_t stream) {
  if (!shard) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (shard->d.flags & MOE_FLAG_NO_ROUTED) return fail(MOE_ERR_INVALID_ARG, "this handle holds no routed experts");
  if (N < 0 || first_expert < 0) return fail(MOE_ERR_INVALID_ARG, "negative N or first_expert");
  if (N == 0) return MOE_OK;
  if (!x_recv || !e_recv || !w_recv || !out || !scratch) return fail(MOE_ERR_INVALID_ARG, "a pointer argument is NULL");
  if (!aligned16(x_recv) || !aligned16(out) || !aligned16(scratch))
    return fail(MOE_ERR_MISALIGNED, "x_recv, out and scratch must be 16-byte aligned");
  const size_t need = moe::ep_experts_scratch_bytes(shard->d, N);
  if (scratch_bytes < need)
    return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "scratch has %zu bytes, %zu needed for %d rows", scratch_bytes, need, N);
  moe_status st = check_device(shard);
  if (st != MOE_OK) return st;
  const cudaError_t e =
      moe::ep_experts(shard->d, shard->wt, shard->cfg.routed_format == MOE_ROUTED_Q4K, static_cast<const __half *>(x_recv),
                      e_recv, w_recv, N, first_expert, out, scratch, shard->err, reinterpret_cast<cudaStream_t>(stream),
                      shard->num_sms);
  if (e != cudaSuccess) return cuda_fail(e, "moe_ep_experts launch");
  g_last_error.clear();
  return MOE_OK;
}

moe_status moe_ep_combine(moe_handle *h, const float *x, int T, const int32_t *perm, const float *out_back, float *y,
                          void *scratch, size_t scratch_bytes, moe_stream_t stream) {
  if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
  if (h->d.flags & MOE_FLAG_EXPERTS_ONLY) return fail(MOE_ERR_INVALID_ARG, "an experts-only handle has no shared expert");
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d is negative", T);
  if (T == 0) return MOE_OK;
  if (!x || !perm || !out_back || !y || !scratch) return fail(MOE_ERR_INVALID_ARG, "a pointer argument is NULL");
  if (!aligned16(x) || !aligned16(out_back) || !aligned16(y) || !aligned16(scratch))
    return fail(MOE_ERR_MISALIGNED, "x, out_back, y and scratch must be 16-byte aligned");
  if (y == x && !(h->d.flags & MOE_FLAG_PRENORM_RESIDUAL))
    return fail(MOE_ERR_INVALID_ARG, "y may alias x only with MOE_FLAG_PRENORM_RESIDUAL");
  const size_t need = moe::ep_combine_scratch_bytes(h->d, T);
  if (scratch_bytes < need)
    return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "scratch has %zu bytes, %zu needed for T=%d", scratch_bytes, need, T);
  moe_status st = check_device(h);
  if (st != MOE_OK) return st;
  const cudaError_t e = moe::ep_combine(h->d, h->wt, x, T, perm, out_back, y, scratch, h->err,
                                        reinterpret_cast<cudaStream_t>(stream), h->num_sms);
  if (e != cudaSuccess) return cuda_fail(e, "moe_ep_combine launch");
  g_last_error.clear();
  return MOE_OK;
}

void moe_destroy(moe_handle *h) { delete h; }

}  // extern "C"
