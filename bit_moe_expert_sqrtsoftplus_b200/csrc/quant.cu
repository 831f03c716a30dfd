// quant.cu -- offline encoders: fp32 values -> Q8_0 / Q2_K / Q4_K blocks (sm_100a).
//
// The Q2_K writer's steps ("2bit 量子化はなぜ「冗談ではない」のか", section 3
// "Q2_K: 256 要素を 84 バイトにする K-quant"): a scale and a min for every
// 16-element sub-block, each value rounded to a 2-bit code 0..3, four codes
// per byte by the page's packing expression (element e in byte
// 32*(e/128) + e%32 of qs, shift 2*((e%128)/32)), the f16 bases d and dmin at
// bytes 80 and 82.  Q8_0 ("DeepSeek-V4-Flash one-token computation flow",
// section "Dwarf Star の量子化の工夫"): one symmetric scale per 32 values.
// The pages give no estimator and no precision; this encoder estimates by
// min/max and takes every decision in IEEE binary32 with round-to-nearest-
// even (explicit _rn operations, so nothing is contracted into an FMA), in
// this order:
//   Q8_0  d = f16(max|x| / 127);  q = clamp(rint(x / d), -127, 127)
//   Q2_K  per sub-block lo = min(0, min x), hi = max x, scale = (hi - lo) / 3,
//         min = 0 - lo;  d = f16(max scale / 15), dmin = f16(max min / 15);
//         sc = clamp(rint(scale / d), 0, 15), m = clamp(rint(min / dmin), 0, 15);
//         q = clamp(rint((x + dmin*m) / (d*sc)), 0, 3)
//   Q4_K  the same as Q2_K one level up: 32-value sub-blocks, scale =
//         (hi - lo) / 15, bases max / 63, 6-bit scales and mins, codes 0..15,
//         in the Q4_K layout (see k_quantize_q4k)
// where a zero base gives zero nibbles and a zero step zero codes.  The
// decoded value is d*q (Q8_0) and d*sc*q - dmin*m (Q2_K, Q4_K).
//
// One warp encodes one block per loop trip.  Q2_K: lane l holds elements
// 32i + l (i = 0..7), so element 32i + l lies in sub-block 2i + l/16 (a
// half-warp reduces its range) and its code goes to qs byte 32*(i/4) + l at
// shift 2*(i%4): each lane assembles two whole qs bytes.  The block is put
// together in shared memory and stored as whole 32-bit (Q2_K) or 16-bit
// (Q8_0) words.  A block holding a non-finite value is written as zeros and
// counted.

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "quant.cuh"

namespace moe {
namespace {

constexpr int kQuantWarps = 8;  // blocks in flight per CTA

__device__ __forceinline__ uint16_t f16_rn_bits(float v) { return __half_as_ushort(__float2half_rn(v)); }
__device__ __forceinline__ float f16_value(uint16_t b) { return __half2float(__ushort_as_half(b)); }
__device__ __forceinline__ float clamp_rint(float v, float lo, float hi) { return fminf(fmaxf(rintf(v), lo), hi); }

__global__ void __launch_bounds__(kQuantWarps * kWarp) k_quantize_q80(const float *__restrict__ x, int64_t nblocks,
                                                                     uint8_t *__restrict__ out, int32_t *nonfinite) {
  __shared__ __align__(16) uint8_t stage[kQuantWarps][48];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint8_t *st = stage[w];
  for (int64_t b = (int64_t)blockIdx.x * kQuantWarps + w; b < nblocks; b += (int64_t)gridDim.x * kQuantWarps) {
    const float v = x[b * 32 + lane];
    const bool bad = __any_sync(0xffffffffu, !isfinite(v));
    float amax = fabsf(v);
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const uint16_t dh = bad ? 0 : f16_rn_bits(__fdiv_rn(amax, 127.0f));
    const float dq = f16_value(dh);
    float q = 0.0f;
    if (dq > 0.0f) q = clamp_rint(__fdiv_rn(v, dq), -127.0f, 127.0f);
    st[2 + lane] = (uint8_t)(int8_t)(int)q;
    if (lane == 0) {
      st[0] = (uint8_t)(dh & 0xff);
      st[1] = (uint8_t)(dh >> 8);
      if (bad && nonfinite) atomicAdd(nonfinite, 1);
    }
    __syncwarp();
    if (lane < 17) reinterpret_cast<uint16_t *>(out + b * 34)[lane] = reinterpret_cast<const uint16_t *>(st)[lane];
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kQuantWarps * kWarp) k_quantize_q2k(const float *__restrict__ x, int64_t nblocks,
                                                                     uint8_t *__restrict__ out, int32_t *nonfinite) {
  __shared__ __align__(16) uint8_t stage[kQuantWarps][96];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, half = lane >> 4;
  uint8_t *st = stage[w];
  for (int64_t b = (int64_t)blockIdx.x * kQuantWarps + w; b < nblocks; b += (int64_t)gridDim.x * kQuantWarps) {
    const float *xb = x + b * 256;
    float v[8];
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = xb[32 * i + lane];
      bad |= !isfinite(v[i]);
    }
    bad = __any_sync(0xffffffffu, bad);
    // range of sub-block 2i + half over its 16 lanes
    float scale[8], mn[8], maxs = 0.0f, maxm = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float lo = fminf(v[i], 0.0f), hi = v[i];
#pragma unroll
      for (int o = 8; o; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      }
      scale[i] = __fdiv_rn(__fsub_rn(hi, lo), 3.0f);
      mn[i] = __fsub_rn(0.0f, lo);
      maxs = fmaxf(maxs, scale[i]);
      maxm = fmaxf(maxm, mn[i]);
    }
    maxs = fmaxf(maxs, __shfl_xor_sync(0xffffffffu, maxs, 16));
    maxm = fmaxf(maxm, __shfl_xor_sync(0xffffffffu, maxm, 16));
    const uint16_t dh = bad ? 0 : f16_rn_bits(__fdiv_rn(maxs, 15.0f));
    const uint16_t mh = bad ? 0 : f16_rn_bits(__fdiv_rn(maxm, 15.0f));
    const float dq = f16_value(dh), mq = f16_value(mh);
    uint32_t byte_lo = 0, byte_hi = 0;  // qs bytes lane and 32 + lane
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float sc = dq > 0.0f ? clamp_rint(__fdiv_rn(scale[i], dq), 0.0f, 15.0f) : 0.0f;
      const float m = mq > 0.0f ? clamp_rint(__fdiv_rn(mn[i], mq), 0.0f, 15.0f) : 0.0f;
      const float step = __fmul_rn(dq, sc), off = __fmul_rn(mq, m);
      float q = 0.0f;
      if (step > 0.0f) q = clamp_rint(__fdiv_rn(__fadd_rn(v[i], off), step), 0.0f, 3.0f);
      const uint32_t code = (uint32_t)(int)q << (2 * (i & 3));
      if (i < 4)
        byte_lo |= code;
      else
        byte_hi |= code;
      if ((lane & 15) == 0) st[2 * i + half] = (uint8_t)((int)sc | ((int)m << 4));
    }
    st[16 + lane] = (uint8_t)byte_lo;
    st[48 + lane] = (uint8_t)byte_hi;
    if (lane == 0) {
      st[80] = (uint8_t)(dh & 0xff);
      st[81] = (uint8_t)(dh >> 8);
      st[82] = (uint8_t)(mh & 0xff);
      st[83] = (uint8_t)(mh >> 8);
      if (bad && nonfinite) atomicAdd(nonfinite, 1);
    }
    __syncwarp();
    if (lane < 21) reinterpret_cast<uint32_t *>(out + b * 84)[lane] = reinterpret_cast<const uint32_t *>(st)[lane];
    __syncwarp();
  }
}

// Q4_K (the same estimator one level up, 32-value sub-blocks, sixteen codes,
// 6-bit scales and mins under f16 bases of max/63, the Q4_K layout: d, dmin,
// 12 bytes of scales and mins, 128 bytes of codes).  Lane l holds values
// 8l .. 8l+7: sub-block l/4 (four lanes reduce its range), code bytes
// 32*(l/8) + 8*(l%4) .. +7, nibble (l%8)/4, so lanes l and l+4 fill the same
// eight bytes and one shuffle joins them.
__global__ void __launch_bounds__(kQuantWarps * kWarp) k_quantize_q4k(const float *__restrict__ x, int64_t nblocks,
                                                                     uint8_t *__restrict__ out, int32_t *nonfinite) {
  __shared__ __align__(16) uint8_t stage[kQuantWarps][144];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint8_t *st = stage[w];
  for (int64_t b = (int64_t)blockIdx.x * kQuantWarps + w; b < nblocks; b += (int64_t)gridDim.x * kQuantWarps) {
    const float4 *xb = reinterpret_cast<const float4 *>(x + b * 256 + 8 * lane);
    const float4 a0 = xb[0], a1 = xb[1];
    const float v[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    bool bad = false;
    float lo = 0.0f, hi = v[0];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      bad |= !isfinite(v[k]);
      lo = fminf(lo, v[k]);
      hi = fmaxf(hi, v[k]);
    }
    bad = __any_sync(0xffffffffu, bad);
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const float scale = __fdiv_rn(__fsub_rn(hi, lo), 15.0f), mn = __fsub_rn(0.0f, lo);
    float maxs = scale, maxm = mn;
#pragma unroll
    for (int o = 4; o <= 16; o <<= 1) {
      maxs = fmaxf(maxs, __shfl_xor_sync(0xffffffffu, maxs, o));
      maxm = fmaxf(maxm, __shfl_xor_sync(0xffffffffu, maxm, o));
    }
    maxs = fmaxf(maxs, 0.0f);
    const uint16_t dh = bad ? 0 : f16_rn_bits(__fdiv_rn(maxs, 63.0f));
    const uint16_t mh = bad ? 0 : f16_rn_bits(__fdiv_rn(maxm, 63.0f));
    const float dq = f16_value(dh), mq = f16_value(mh);
    const float sc = dq > 0.0f ? clamp_rint(__fdiv_rn(scale, dq), 0.0f, 63.0f) : 0.0f;
    const float m = mq > 0.0f ? clamp_rint(__fdiv_rn(mn, mq), 0.0f, 63.0f) : 0.0f;
    const float step = __fmul_rn(dq, sc), off = __fmul_rn(mq, m);
    uint32_t codes = 0;  // eight 4-bit codes, value 8l+k in bits 4k..4k+3
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float q = 0.0f;
      if (step > 0.0f) q = clamp_rint(__fdiv_rn(__fadd_rn(v[k], off), step), 0.0f, 15.0f);
      codes |= (uint32_t)(int)q << (4 * k);
    }
    const uint32_t upper = __shfl_down_sync(0xffffffffu, codes, 4);  // lane l+4: the high nibbles
    if ((lane & 7) < 4) {
      uint8_t *dst = st + 16 + 32 * (lane >> 3) + 8 * (lane & 3);
#pragma unroll
      for (int k = 0; k < 8; ++k) dst[k] = (uint8_t)(((codes >> (4 * k)) & 15u) | (((upper >> (4 * k)) & 15u) << 4));
    }
    // the eight (scale, min) pairs, from lanes 0, 4, ..., 28
    int scj[8], mj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      scj[j] = __shfl_sync(0xffffffffu, (int)sc, 4 * j);
      mj[j] = __shfl_sync(0xffffffffu, (int)m, 4 * j);
    }
    if (lane == 0) {
      st[0] = (uint8_t)(dh & 0xff);
      st[1] = (uint8_t)(dh >> 8);
      st[2] = (uint8_t)(mh & 0xff);
      st[3] = (uint8_t)(mh >> 8);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        st[4 + j] = (uint8_t)(scj[j] | ((scj[j + 4] >> 4) << 6));
        st[8 + j] = (uint8_t)(mj[j] | ((mj[j + 4] >> 4) << 6));
        st[12 + j] = (uint8_t)((scj[j + 4] & 15) | ((mj[j + 4] & 15) << 4));
      }
      if (bad && nonfinite) atomicAdd(nonfinite, 1);
    }
    __syncwarp();
    if (lane < 9) reinterpret_cast<uint4 *>(out + b * 144)[lane] = reinterpret_cast<const uint4 *>(st)[lane];
    __syncwarp();
  }
}

}  // namespace

cudaError_t quantize_blocks(int format, const float *x, int64_t nblocks, void *out, int32_t *nonfinite,
                            cudaStream_t stream, int num_sms) {
  if (nblocks <= 0) return cudaSuccess;
  const int64_t ctas = (nblocks + kQuantWarps - 1) / kQuantWarps;
  const int64_t cap = (int64_t)num_sms * 8;  // 8 CTAs of 256 threads fill an SM
  const int grid = (int)(ctas < cap ? ctas : cap);
  uint8_t *o = static_cast<uint8_t *>(out);
  if (format == kQuantQ80)
    k_quantize_q80<<<grid, kQuantWarps * kWarp, 0, stream>>>(x, nblocks, o, nonfinite);
  else if (format == kQuantQ2K)
    k_quantize_q2k<<<grid, kQuantWarps * kWarp, 0, stream>>>(x, nblocks, o, nonfinite);
  else
    k_quantize_q4k<<<grid, kQuantWarps * kWarp, 0, stream>>>(x, nblocks, o, nonfinite);
  return cudaGetLastError();
}

}  // namespace moe
