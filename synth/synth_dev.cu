// synth_dev.cu -- device fills built on synth.h, byte-identical to the host
// fills in synth_host.c (same source, integer fields, explicitly rounded fp32).
// Used to materialise multi-gigabyte weight sets directly in device memory.
#include <cuda_runtime.h>
#include "synth.h"

namespace {

template <int KIND>
__global__ void fill_kernel(uint64_t key, uint64_t first, uint64_t n, uint8_t *__restrict__ out) {
  constexpr int BYTES = KIND == 0   ? SYNTH_IQ2XXS_BYTES
                        : KIND == 1 ? SYNTH_Q2K_BYTES
                        : KIND == 3 ? SYNTH_Q4K_BYTES
                                    : SYNTH_Q80_BYTES;
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t b = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; b < n; b += stride) {
    uint8_t tmp[BYTES];
    if (KIND == 0)
      synth_iq2xxs_block(key, first + b, tmp);
    else if (KIND == 1)
      synth_q2k_block(key, first + b, tmp);
    else if (KIND == 3)
      synth_q4k_block(key, first + b, tmp);
    else
      synth_q80_block(key, first + b, tmp);
    uint8_t *dst = out + b * BYTES;
#pragma unroll
    for (int i = 0; i < BYTES; i += 2) {
      // every block size is even and every block starts on a 2-byte boundary
      *reinterpret_cast<uint16_t *>(dst + i) = (uint16_t)(tmp[i] | (tmp[i + 1] << 8));
    }
  }
}

}  // namespace

extern "C" int synth_dev_fill_routed(uint64_t seed, uint32_t layer, uint32_t tensor, int kind, int e0, int ne,
                                     int rows, int cols, void *out, void *stream) {
  if (kind < 0 || kind > 3 || ne < 0 || rows <= 0 || cols <= 0 || out == nullptr) return -1;
  if ((reinterpret_cast<uintptr_t>(out) & 1u) != 0) return -1;
  uint64_t bpr = (uint64_t)cols / (kind == 2 ? 32u : 256u);
  uint64_t per_expert = (uint64_t)rows * bpr;
  uint64_t n = (uint64_t)ne * per_expert;
  if (n == 0) return 0;
  uint64_t key = synth_key(seed, layer, tensor);
  uint64_t first = (uint64_t)e0 * per_expert;
  int threads = 256;
  uint64_t want = (n + threads - 1) / threads;
  int blocks = (int)(want < 148ull * 64ull ? want : 148ull * 64ull);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t *o = static_cast<uint8_t *>(out);
  if (kind == 0)
    fill_kernel<0><<<blocks, threads, 0, s>>>(key, first, n, o);
  else if (kind == 1)
    fill_kernel<1><<<blocks, threads, 0, s>>>(key, first, n, o);
  else if (kind == 3)
    fill_kernel<3><<<blocks, threads, 0, s>>>(key, first, n, o);
  else
    fill_kernel<2><<<blocks, threads, 0, s>>>(key, first, n, o);
  return cudaGetLastError() == cudaSuccess ? 0 : -2;
}
