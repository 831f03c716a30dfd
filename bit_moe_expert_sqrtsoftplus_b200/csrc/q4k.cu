// q4k.cu -- expert work of a layer whose routed experts are Q4_K (the q2-q4
// build: "DeepSeek-V4-Flash one-token computation flow", section "128GB に
// どう収めるか: Q4 層数の試算", where the last six layers keep their routed
// experts in Q4_K), for calls of up to 32 tokens.  The routing is the
// layer's own (it does not depend on the expert format); this file takes
// (idx, w) and computes
//   y[t] = shared(x̂[t]) + sum_i w[t][i] * E_idx[t][i](x̂[t])   (+ x[t] with the
//   pre-norm residual), E(v) = W_down (SiLU(W_gate v) * (W_up v))
// with fp32 dot products over blocks decoded in registers: one warp per
// output row.  It is the plain first form of this path (three launches, no
// tensor cores); its arithmetic is exact decoding and fp32 accumulation.
//
// Q4_K block (144 bytes, 256 values; "2bit 量子化はなぜ「冗談ではない」のか",
// section 3 type table; layout read as the public GGUF block): f16 d at 0,
// f16 dmin at 2, 12 bytes of 6-bit scales and mins at 4, 128 bytes of 4-bit
// codes at 16.  Sub-block j (32 values): j < 4: scale = low 6 bits of scale
// byte j, min = low 6 bits of scale byte j+4; j >= 4: scale = low nibble of
// scale byte j+4 plus the top two bits of scale byte j-4 as bits 4-5, min =
// high nibble of scale byte j+4 plus the top two bits of scale byte j.  The
// code of value e is nibble (e%64)/32 of code byte 32*(e/64) + e%32.  Value =
// d*scale*q - dmin*min.  Lane l of a warp takes values 8l .. 8l+7 of each
// block: sub-block l/4, eight consecutive code bytes at 32*(l/8) + 8*(l%4),
// nibble (l%8)/4.

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "q4k.cuh"

namespace moe {
namespace {

constexpr int kRowsPerCta = 8;  // one warp per output row

__device__ __forceinline__ float f16_at(const uint8_t *p) {
  return __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t *>(p)));
}

// sum_k W[row][k] v[k] over K values of Q4_K blocks (K a multiple of 256);
// every lane returns the sum.
__device__ float dot_q4k(const uint8_t *row, const float *v, int K, int lane) {
  const float4 *v4 = reinterpret_cast<const float4 *>(v);
  const int j = lane >> 2, jj = j & 3;
  const int code_off = 16 + 32 * (lane >> 3) + 8 * (lane & 3);
  const int shift = 4 * ((lane & 7) >> 2);
  float part = 0.0f;
#pragma unroll 4
  for (int b = 0; b < K / 256; ++b) {  // unrolled so several blocks' loads are in flight
    const uint8_t *blk = row + (size_t)b * 144;
    const uint4 hd = *reinterpret_cast<const uint4 *>(blk);  // d, dmin, scale bytes 0..11
    const float d = __half2float(__ushort_as_half((uint16_t)(hd.x & 0xffffu)));
    const float dmin = __half2float(__ushort_as_half((uint16_t)(hd.x >> 16)));
    const uint32_t b03 = hd.y, b47 = hd.z, b811 = hd.w;  // scale bytes 0-3, 4-7, 8-11
    int sc, mn;
    if (j < 4) {
      sc = (int)((b03 >> (8 * jj)) & 63u);
      mn = (int)((b47 >> (8 * jj)) & 63u);
    } else {
      const uint32_t lowb = (b811 >> (8 * jj)) & 255u;
      sc = (int)((lowb & 15u) | (((b03 >> (8 * jj + 6)) & 3u) << 4));
      mn = (int)((lowb >> 4) | (((b47 >> (8 * jj + 6)) & 3u) << 4));
    }
    const uint2 cw = *reinterpret_cast<const uint2 *>(blk + code_off);
    const float4 x0 = v4[64 * b + 2 * lane], x1 = v4[64 * b + 2 * lane + 1];
    const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    float sqx = 0.0f, sx = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t byte = ((k < 4 ? cw.x : cw.y) >> (8 * (k & 3))) & 255u;
      const float q = (float)((byte >> shift) & 15u);
      sqx = fmaf(q, xs[k], sqx);
      sx += xs[k];
    }
    part += d * (float)sc * sqx - dmin * (float)mn * sx;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  return part;
}

// The same over Q8_0 blocks (K a multiple of 32): lane l takes value l of
// every block.
__device__ float dot_q80(const uint8_t *row, const float *v, int K, int lane) {
  float part = 0.0f;
#pragma unroll 8
  for (int b = 0; b < K / 32; ++b) {
    const uint8_t *blk = row + (size_t)b * 34;
    part = fmaf(f16_at(blk) * (float)(int8_t)blk[2 + lane], v[32 * b + lane], part);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  return part;
}

// xn[t] = x[t], or x[t] / sqrt(mean(x[t]^2) + eps) with the pre-norm residual.
__global__ void __launch_bounds__(256) k_q4k_input(const float *__restrict__ x, int H, int flags, float eps,
                                                   float *__restrict__ xn) {
  __shared__ double red[8];
  __shared__ float inv_s;
  const int t = blockIdx.x, tid = threadIdx.x;
  const float *xt = x + (size_t)t * H;
  float inv = 1.0f;
  if (flags & MOE_FLAG_PRENORM_RESIDUAL) {
    double ss = 0.0;
    for (int c = tid; c < H; c += 256) ss += (double)xt[c] * (double)xt[c];
    ss = warp_sum_d(ss);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    if (tid == 0) {
      double tot = 0.0;
      for (int w = 0; w < 8; ++w) tot += red[w];
      inv_s = (float)(1.0 / sqrt(tot / (double)H + (double)eps));
    }
    __syncthreads();
    inv = inv_s;
  }
  for (int c = tid; c < H; c += 256) xn[(size_t)t * H + c] = xt[c] * inv;
}

// Blocks (row tile, p): p < T*k is the routed pair p (Q4_K gate/up rows of
// I), p >= T*k the shared expert for token p - T*k (Q8_0 rows of Is).
__global__ void __launch_bounds__(kRowsPerCta * 32) k_q4k_gate_up(const Q4kArgs a) {
  const LayerDims &d = a.d;
  const int lane = threadIdx.x & 31, row = blockIdx.x * kRowsPerCta + (threadIdx.x >> 5);
  const int p = blockIdx.y, npairs = a.T * d.k;
  if (p < npairs) {
    if (row >= d.I) return;
    const int t = p / d.k, e = a.idx[p];
    float hv = 0.0f;
    if (e >= 0 && e < d.E) {
      const size_t rb = (size_t)(d.H / 256) * 144;
      const size_t off = ((size_t)e * d.I + row) * rb;
      const float *xt = a.xn + (size_t)t * d.H;
      const float g = dot_q4k(a.gate + off, xt, d.H, lane);
      const float u = dot_q4k(a.up + off, xt, d.H, lane);
      hv = silu(g) * u;
    }
    if (lane == 0) a.h[(size_t)p * d.I + row] = hv;
  } else {
    if (row >= d.Is) return;
    const int t = p - npairs;
    const size_t rb = (size_t)(d.H / 32) * 34;
    const float *xt = a.xn + (size_t)t * d.H;
    const float g = dot_q80(a.sh_gate + (size_t)row * rb, xt, d.H, lane);
    const float u = dot_q80(a.sh_up + (size_t)row * rb, xt, d.H, lane);
    if (lane == 0) a.hs[(size_t)t * d.Is + row] = silu(g) * u;
  }
}

// y[t][r] = (x[t][r]) + shared_down[r] . hs[t] + sum_i w[t][i] down_e[r] . h[t,i],
// the routed terms in the routing's ascending expert order.
__global__ void __launch_bounds__(kRowsPerCta * 32) k_q4k_down(const Q4kArgs a) {
  const LayerDims &d = a.d;
  const int lane = threadIdx.x & 31, r = blockIdx.x * kRowsPerCta + (threadIdx.x >> 5), t = blockIdx.y;
  if (r >= d.H) return;
  const size_t rbs = (size_t)(d.Is / 32) * 34, rbd = (size_t)(d.I / 256) * 144;
  float acc = dot_q80(a.sh_down + (size_t)r * rbs, a.hs + (size_t)t * d.Is, d.Is, lane);
  for (int i = 0; i < d.k; ++i) {
    const int p = t * d.k + i, e = a.idx[p];
    if (e < 0 || e >= d.E) continue;
    const float o = dot_q4k(a.down + ((size_t)e * d.H + r) * rbd, a.h + (size_t)p * d.I, d.I, lane);
    acc = fmaf(a.w[p], o, acc);
  }
  if (lane == 0) {
    const size_t at = (size_t)t * d.H + r;
    a.y[at] = (d.flags & MOE_FLAG_PRENORM_RESIDUAL) ? a.x[at] + acc : acc;
  }
}

}  // namespace

size_t q4k_expert_bytes(const LayerDims &d, int T) {
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  return al(sizeof(float) * (size_t)T * d.H) + al(sizeof(float) * (size_t)T * d.k * d.I) +
         al(sizeof(float) * (size_t)T * d.Is);
}

cudaError_t q4k_experts(const Q4kArgs &a, cudaStream_t stream) {
  const LayerDims &d = a.d;
  if (a.T <= 0) return cudaSuccess;
  k_q4k_input<<<a.T, 256, 0, stream>>>(a.x, d.H, d.flags, d.eps, a.xn);
  const int rmax = d.I > d.Is ? d.I : d.Is;
  k_q4k_gate_up<<<dim3((rmax + kRowsPerCta - 1) / kRowsPerCta, a.T * d.k + a.T), kRowsPerCta * 32, 0, stream>>>(a);
  k_q4k_down<<<dim3((d.H + kRowsPerCta - 1) / kRowsPerCta, a.T), kRowsPerCta * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
