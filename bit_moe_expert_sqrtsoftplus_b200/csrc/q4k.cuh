// q4k.cuh -- the layer with Q4_K routed experts (the q2-q4 build's upgraded
// layers) for small token counts: host interface.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "layer.cuh"

namespace moe {

struct Q4kArgs {
  LayerDims d;
  const uint8_t *gate, *up, *down;           // Q4_K [E][I][H/256] / [E][H][I/256] 144-byte blocks
  const uint8_t *sh_gate, *sh_up, *sh_down;  // Q8_0 [Is][H/32] / [H][Is/32] 34-byte blocks
  int T;
  const float *x;  // [T][H]
  float *y;        // [T][H]; may alias x with MOE_FLAG_PRENORM_RESIDUAL
  const int32_t *idx;  // [T][k] ascending expert ids
  const float *w;      // [T][k]
  float *h;            // [T*k][I] scratch: routed SwiGLU outputs
  float *hs;           // [T][Is] scratch: shared SwiGLU outputs
  float *xsum;         // [T][H/32] scratch: sums of the expert input over each 32-value sub-block
  const int8_t *xq;    // [T][3][H] int8 limbs of the expert input (the small-token router kernel's)
  const float *xs;     // [T][4] limb scales
  int8_t *hq;          // scratch: int8 limbs of the down inputs, [T*k][3][I] (h) then [T][3][Is] (hs)
  float *hqs;          // [T*k + T][4] their limb scales
  float *hsum;         // their sums over each 32-value sub-block, [T*k][I/32] then [T][Is/32]
};

// Scratch the expert kernels take beside the routing scratch (h, hs, xsum and
// the down inputs' limbs, scales and sums).
size_t q4k_expert_bytes(const LayerDims &d, int T);

// The expert work of one call, after the routing (idx, w) is in place: four
// launches on `stream` (input sums, gate/up with SwiGLU, the down inputs'
// limbs, down with the weighted combine).
cudaError_t q4k_experts(const Q4kArgs &a, cudaStream_t stream);

}  // namespace moe
