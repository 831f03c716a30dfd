// prefill.cuh -- the layer for larger token counts (T > 32): certified router,
// token permutation and grouped tensor-core GEMMs.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "layer.cuh"

namespace moe {

struct PrefillScratch {
  float *z;          // [T][E] fp32 router logits
  int32_t *idx;      // [T][k]
  float *w;          // [T][k]
  int32_t *counts;   // [E]
  int32_t *offsets;  // [E+1]
  int32_t *perm;     // [T*k]
  int32_t *fix;      // [1 + 2T] count, tokens that need the fp64 router, per-token block arrivals
  void *big;         // remaining scratch for the expert GEMMs
  size_t big_bytes;
};

struct PrefillArgs {
  LayerDims d;
  LayerWeights wt;
  int T;
  const float *x;
  const int32_t *token_ids;
  float *y;
  PrefillScratch s;
  const float *row_norms;  // [E] 2-norms of the router rows
  int *err;
  cudaEvent_t ev_begin, ev_end;  // recorded around the routed gate/up GEMM when set
  int q4k;                       // routed gate/up/down in Q4_K (else IQ2_XXS gate/up, Q2_K down)
};

size_t prefill_scratch_bytes(const LayerDims &d, int T);
PrefillArgs prefill_args(const LayerDims &d, const LayerWeights &wt, int T, const float *x,
                         const int32_t *token_ids, float *y, void *scratch, const float *row_norms, int *err);
cudaError_t prefill_init(const LayerDims &d, const LayerWeights &wt, float *row_norms, int *err, cudaStream_t s);
// Hash mode: checks that every row of the token-id table holds k distinct
// expert ids in [0, E).  Uses one device int (dev_word) as a temporary, waits
// for the stream, and sets *first_bad to the first failing row (-1 if none).
cudaError_t check_tid2eid(const LayerDims &d, const int32_t *tab, int *dev_word, int *first_bad, cudaStream_t s);
cudaError_t prefill_route(const PrefillArgs &p, int32_t *idx, float *w, cudaStream_t s);
cudaError_t prefill_forward(const PrefillArgs &p, cudaStream_t s, int num_sms);
// Expert parallelism (experts split over ranks in contiguous blocks).
//   ep_dispatch: routing, grouping of the T*k pairs by expert (offsets,
//     perm), and per pair in that order the f16 expert input row, the
//     expert id and the routing weight.
//   ep_experts: on a shard of E = d.E experts starting at global id e0, the
//     rows received for them: out[i] = w[i] * E_{e[i]}(x[i]).
//   ep_combine: y = shared expert (+ the residual input with the pre-norm
//     flag) + the returned rows of each token's pairs, in ascending slot order.
size_t ep_dispatch_scratch_bytes(const LayerDims &d, int T);
cudaError_t ep_dispatch(const PrefillArgs &p, int32_t *offsets, int32_t *perm, __half *x_send, int32_t *e_send,
                        float *w_send, cudaStream_t s);
size_t ep_experts_scratch_bytes(const LayerDims &d, int N);
cudaError_t ep_experts(const LayerDims &d, const LayerWeights &wt, bool q4k, const __half *x_recv,
                       const int32_t *e_recv, const float *w_recv, int N, int e0, float *out, void *scratch,
                       int *err, cudaStream_t s, int num_sms);
size_t ep_combine_scratch_bytes(const LayerDims &d, int T);
cudaError_t ep_combine(const LayerDims &d, const LayerWeights &wt, const float *x, int T, const int32_t *perm,
                       const float *out_back, float *y, void *scratch, int *err, cudaStream_t s, int num_sms);

// Stable grouping of the T*k (token, slot) pairs by expert.
cudaError_t permute(const int32_t *idx, int T, int k, int E, int32_t *offsets, int32_t *perm, cudaStream_t s);

}  // namespace moe
