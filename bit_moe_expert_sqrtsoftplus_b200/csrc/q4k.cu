// q4k.cu -- expert work of a layer whose routed experts are Q4_K (the q2-q4
// build: "DeepSeek-V4-Flash one-token computation flow", section "128GB に
// どう収めるか: Q4 層数の試算", where the last six layers keep their routed
// experts in Q4_K), for calls of up to 32 tokens.  The routing is the
// layer's own (it does not depend on the expert format); this file takes
// (idx, w) and computes
//   y[t] = shared(x̂[t]) + sum_i w[t][i] * E_idx[t][i](x̂[t])   (+ x[t] with the
//   pre-norm residual), E(v) = W_down (SiLU(W_gate v) * (W_up v))
// with fp32 dot products over blocks decoded in registers: one warp per
// output row (gate and up rows of a pair read together), three launches, no
// tensor cores; its arithmetic is exact decoding and fp32 accumulation.
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

// Lane l's share of a Q4_K block: values 8l .. 8l+7, i.e. sub-block l/4,
// code bytes 32*(l/8) + 8*(l%4) .. +7, nibble (l%8)/4.
struct Q4kLane {
  int j, jj, code_off, shift;
  __device__ explicit Q4kLane(int lane)
      : j(lane >> 2), jj((lane >> 2) & 3), code_off(16 + 32 * (lane >> 3) + 8 * (lane & 3)),
        shift(4 * ((lane & 7) >> 2)) {}
};

// Lane l's part of one block's dot product with its 8 values xs of v:
// d*scale*sum(q*x) - dmin*min*sum(x), sx = sum(x) given.
__device__ __forceinline__ float q4k_part(const uint4 hd, const uint2 cw, const Q4kLane &L, const float (&xs)[8],
                                          float sx) {
  const float d = __half2float(__ushort_as_half((uint16_t)(hd.x & 0xffffu)));
  const float dmin = __half2float(__ushort_as_half((uint16_t)(hd.x >> 16)));
  const uint32_t b03 = hd.y, b47 = hd.z, b811 = hd.w;  // scale bytes 0-3, 4-7, 8-11
  int sc, mn;
  if (L.j < 4) {
    sc = (int)((b03 >> (8 * L.jj)) & 63u);
    mn = (int)((b47 >> (8 * L.jj)) & 63u);
  } else {
    const uint32_t lowb = (b811 >> (8 * L.jj)) & 255u;
    sc = (int)((lowb & 15u) | (((b03 >> (8 * L.jj + 6)) & 3u) << 4));
    mn = (int)((lowb >> 4) | (((b47 >> (8 * L.jj + 6)) & 3u) << 4));
  }
  float sqx = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t byte = ((k < 4 ? cw.x : cw.y) >> (8 * (k & 3))) & 255u;
    sqx = fmaf((float)((byte >> L.shift) & 15u), xs[k], sqx);
  }
  return d * (float)sc * sqx - dmin * (float)mn * sx;
}

__device__ __forceinline__ void load8(const float *v, float (&xs)[8], float &sx) {
  const float4 a = reinterpret_cast<const float4 *>(v)[0], b = reinterpret_cast<const float4 *>(v)[1];
  xs[0] = a.x, xs[1] = a.y, xs[2] = a.z, xs[3] = a.w, xs[4] = b.x, xs[5] = b.y, xs[6] = b.z, xs[7] = b.w;
  sx = ((a.x + a.y) + (a.z + a.w)) + ((b.x + b.y) + (b.z + b.w));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Lane l's part of sum_k W[row][k] v[k] over Q8_0 blocks (K a multiple of
// 128): per iteration the warp takes four blocks, lane l the values
// 4*(l%8) .. +3 of block l/8 of them (two 16-bit loads: blocks are 34 bytes,
// so their quants are 2-byte aligned).
__device__ __forceinline__ float q80_part(const uint8_t *row, const float *v, int K, int lane) {
  const int sub = lane >> 3, q4 = 4 * (lane & 7);
  float part = 0.0f;
#pragma unroll 4
  for (int b = sub; b < K / 32; b += 4) {
    const uint8_t *blk = row + (size_t)b * 34;
    const float d = f16_at(blk);
    const uint32_t lo = *reinterpret_cast<const uint16_t *>(blk + 2 + q4);
    const uint32_t hi = *reinterpret_cast<const uint16_t *>(blk + 4 + q4);
    const float4 x = *reinterpret_cast<const float4 *>(v + 32 * b + q4);
    const float s = (float)(int8_t)(lo & 255u) * x.x + (float)(int8_t)(lo >> 8) * x.y +
                    (float)(int8_t)(hi & 255u) * x.z + (float)(int8_t)(hi >> 8) * x.w;
    part = fmaf(d, s, part);
  }
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
      // gate and up rows of the pair together: both rows' loads of a block
      // are in flight at once, and the x values and their sum serve both
      const size_t rb = (size_t)(d.H / 256) * 144;
      const uint8_t *gr = a.gate + ((size_t)e * d.I + row) * rb, *ur = a.up + ((size_t)e * d.I + row) * rb;
      const float *xt = a.xn + (size_t)t * d.H;
      const Q4kLane L(lane);
      float pg = 0.0f, pu = 0.0f;
#pragma unroll 4
      for (int b = 0; b < d.H / 256; ++b) {
        const uint4 hg = *reinterpret_cast<const uint4 *>(gr + (size_t)b * 144);
        const uint4 hu = *reinterpret_cast<const uint4 *>(ur + (size_t)b * 144);
        const uint2 cg = *reinterpret_cast<const uint2 *>(gr + (size_t)b * 144 + L.code_off);
        const uint2 cu = *reinterpret_cast<const uint2 *>(ur + (size_t)b * 144 + L.code_off);
        float xs[8], sx;
        load8(xt + 256 * b + 8 * lane, xs, sx);
        pg += q4k_part(hg, cg, L, xs, sx);
        pu += q4k_part(hu, cu, L, xs, sx);
      }
      hv = silu(warp_sum(pg)) * warp_sum(pu);
    }
    if (lane == 0) a.h[(size_t)p * d.I + row] = hv;
  } else {
    if (row >= d.Is) return;
    const int t = p - npairs;
    const size_t rb = (size_t)(d.H / 32) * 34;
    const float *xt = a.xn + (size_t)t * d.H;
    const float g = warp_sum(q80_part(a.sh_gate + (size_t)row * rb, xt, d.H, lane));
    const float u = warp_sum(q80_part(a.sh_up + (size_t)row * rb, xt, d.H, lane));
    if (lane == 0) a.hs[(size_t)t * d.Is + row] = silu(g) * u;
  }
}

// Lane l's part of sum_k W[row][k] v[k] over Q4_K blocks (K a multiple of
// 256), several blocks' loads in flight.
__device__ __forceinline__ float q4k_row_part(const uint8_t *row, const float *v, int K, const Q4kLane &L, int lane) {
  float part = 0.0f;
#pragma unroll 4
  for (int b = 0; b < K / 256; ++b) {
    const uint4 hd = *reinterpret_cast<const uint4 *>(row + (size_t)b * 144);
    const uint2 cw = *reinterpret_cast<const uint2 *>(row + (size_t)b * 144 + L.code_off);
    float xs[8], sx;
    load8(v + 256 * b + 8 * lane, xs, sx);
    part += q4k_part(hd, cw, L, xs, sx);
  }
  return part;
}

// y[t][r] = (x[t][r]) + shared_down[r] . hs[t] + sum_i w[t][i] down_e[r] . h[t,i],
// the routed terms in the routing's ascending expert order; one warp per
// output row, one dot product after the other.  (Reading the k routed rows
// block by block together measured slower: 68 against 44 us per launch at
// one token.)
__global__ void __launch_bounds__(kRowsPerCta * 32) k_q4k_down(const Q4kArgs a) {
  const LayerDims &d = a.d;
  const int lane = threadIdx.x & 31, r = blockIdx.x * kRowsPerCta + (threadIdx.x >> 5), t = blockIdx.y;
  if (r >= d.H) return;
  const size_t rbs = (size_t)(d.Is / 32) * 34, rbd = (size_t)(d.I / 256) * 144;
  const Q4kLane L(lane);
  float acc = warp_sum(q80_part(a.sh_down + (size_t)r * rbs, a.hs + (size_t)t * d.Is, d.Is, lane));
  for (int i = 0; i < d.k; ++i) {
    const int p = t * d.k + i, e = a.idx[p];
    if (e < 0 || e >= d.E) continue;
    const float o = warp_sum(q4k_row_part(a.down + ((size_t)e * d.H + r) * rbd, a.h + (size_t)p * d.I, d.I, L, lane));
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
