// q4k.cu -- expert work of a layer whose routed experts are Q4_K (the q2-q4
// build: "DeepSeek-V4-Flash one-token computation flow", section "128GB に
// どう収めるか: Q4 層数の試算", where the last six layers keep their routed
// experts in Q4_K), for calls of up to 32 tokens.  The routing is the
// layer's own (it does not depend on the expert format); this file takes
// (idx, w) and computes
//   y[t] = shared(x̂[t]) + sum_i w[t][i] * E_idx[t][i](x̂[t])   (+ x[t] with the
//   pre-norm residual), E(v) = W_down (SiLU(W_gate v) * (W_up v))
// with one warp per output row (gate and up rows of a pair read together),
// four launches, no tensor cores.  Every product takes its input vector as
// three int8 limbs (within 6e-8 of its max |value|: the expert input's from
// the small-token router kernel, h's and hs's from a kernel of their own):
// sum q * v per 32-value block is exact in int32 (dp4a), and the Q4_K min
// term uses the fp32 sum of v over the sub-block.  Decoding is exact and the
// sums over blocks are fp32.
//
// Q4_K block (144 bytes, 256 values; "2bit 量子化はなぜ「冗談ではない」のか",
// section 3 type table; layout read as the public GGUF block): f16 d at 0,
// f16 dmin at 2, 12 bytes of 6-bit scales and mins at 4, 128 bytes of 4-bit
// codes at 16.  Sub-block j (32 values): j < 4: scale = low 6 bits of scale
// byte j, min = low 6 bits of scale byte j+4; j >= 4: scale = low nibble of
// scale byte j+4 plus the top two bits of scale byte j-4 as bits 4-5, min =
// high nibble of scale byte j+4 plus the top two bits of scale byte j.  The
// code of value e is nibble (e%64)/32 of code byte 32*(e/64) + e%32.  Value =
// d*scale*q - dmin*min.

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

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Scale step d*scale and offset dmin*min of sub-block j (0..7) of a Q4_K
// block whose first 16 bytes are hd.
__device__ __forceinline__ void q4k_sc_mn(const uint4 hd, int j, float &dsc, float &dmn) {
  const float d = __half2float(__ushort_as_half((uint16_t)(hd.x & 0xffffu)));
  const float dmin = __half2float(__ushort_as_half((uint16_t)(hd.x >> 16)));
  const int jj = j & 3;
  int sc, mn;
  if (j < 4) {
    sc = (int)((hd.y >> (8 * jj)) & 63u);
    mn = (int)((hd.z >> (8 * jj)) & 63u);
  } else {
    const uint32_t lowb = (hd.w >> (8 * jj)) & 255u;
    sc = (int)((lowb & 15u) | (((hd.y >> (8 * jj + 6)) & 3u) << 4));
    mn = (int)((lowb >> 4) | (((hd.z >> (8 * jj + 6)) & 3u) << 4));
  }
  dsc = d * (float)sc;
  dmn = dmin * (float)mn;
}

// Sub-block j of a Q4_K block holds values 32j .. 32j+31: the low (j even) or
// high (j odd) nibbles of the 32 code bytes at 16 + 32 * (j/2).  In the
// routines below lane l takes sub-block l%8 of the blocks l/8, l/8 + 4, ...
// of a row.
__device__ __forceinline__ void q4k_codes(const uint8_t *blk, int j, uint32_t (&qn)[8]) {
  const uint4 c0 = *reinterpret_cast<const uint4 *>(blk + 16 + 32 * (j >> 1));
  const uint4 c1 = *reinterpret_cast<const uint4 *>(blk + 32 + 32 * (j >> 1));
  const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const int shift = 4 * (j & 1);
#pragma unroll
  for (int w = 0; w < 8; ++w) qn[w] = (cw[w] >> shift) & 0x0F0F0F0Fu;  // four codes 0..15 as bytes
}

// A vector v as three int8 limbs (v = s1 q1 + s2 q2 + s3 q3 per value, the
// small-token path's representation, within 6e-8 of max|v|): lane l's part of
// the dot products of NR Q4_K rows with v, sum q * v exact in int32 by dp4a
// per limb, the min term from the fp32 sum S of v over the sub-block.
template <int NR>
__device__ __forceinline__ void q4k_rows_part_limbs(const uint8_t *const (&rows)[NR], const int8_t *vq, int K,
                                                    const float (&s)[3], const float *S, int lane, float (&part)[NR]) {
  const int j = lane & 7;
  for (int b = lane >> 3; b < K / 256; b += 4) {
    const int sb = 8 * b + j;  // sub-block of the row
    uint32_t x[3][8];
#pragma unroll
    for (int l = 0; l < 3; ++l) {
      const uint4 *xl = reinterpret_cast<const uint4 *>(vq + (size_t)l * K + 32 * sb);
      const uint4 a = xl[0], c = xl[1];
      x[l][0] = a.x, x[l][1] = a.y, x[l][2] = a.z, x[l][3] = a.w;
      x[l][4] = c.x, x[l][5] = c.y, x[l][6] = c.z, x[l][7] = c.w;
    }
    const float sx = S[sb];
#pragma unroll
    for (int m = 0; m < NR; ++m) {
      const uint8_t *blk = rows[m] + (size_t)b * 144;
      const uint4 hd = *reinterpret_cast<const uint4 *>(blk);
      uint32_t qn[8];
      q4k_codes(blk, j, qn);
      int acc[3] = {0, 0, 0};
#pragma unroll
      for (int w = 0; w < 8; ++w)
#pragma unroll
        for (int l = 0; l < 3; ++l) acc[l] = __dp4a((int)qn[w], (int)x[l][w], acc[l]);
      float dsc, dmn;
      q4k_sc_mn(hd, j, dsc, dmn);
      const float f = fmaf(s[0], (float)acc[0], fmaf(s[1], (float)acc[1], s[2] * (float)acc[2]));
      part[m] = fmaf(dsc, f, fmaf(-dmn, sx, part[m]));
    }
  }
}

// Lane l's part of a Q8_0 row's dot product with the expert input's int8
// limbs: lane l takes the 32-value blocks l, l + 32, ...; sum q * x per block
// exact in int32 (dp4a per limb).  A block's codes start 2 bytes into it, so
// they are 4-byte aligned when its index is odd and otherwise read as the
// aligned words around them (the last as 16 bits, to stay in the block).
__device__ __forceinline__ float q80_row_part_limbs(const uint8_t *row, const int8_t *xq, int H,
                                                    const float (&s)[3], int lane) {
  float part = 0.0f;
  for (int b = lane; b < H / 32; b += 32) {
    const uint8_t *blk = row + (size_t)b * 34;
    const float d = f16_at(blk);
    uint32_t q[8];
    if ((reinterpret_cast<uintptr_t>(blk + 2) & 3u) == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = *reinterpret_cast<const uint32_t *>(blk + 2 + 4 * i);
    } else {
      uint32_t u[9];
#pragma unroll
      for (int i = 0; i < 8; ++i) u[i] = *reinterpret_cast<const uint32_t *>(blk + 4 * i);
      u[8] = *reinterpret_cast<const uint16_t *>(blk + 32);
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = __byte_perm(u[i], u[i + 1], 0x5432);
    }
    int acc[3] = {0, 0, 0};
#pragma unroll
    for (int l = 0; l < 3; ++l) {
      const uint4 *xl = reinterpret_cast<const uint4 *>(xq + (size_t)l * H + 32 * b);
      const uint4 a = xl[0], c = xl[1];
      const uint32_t xw[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
      for (int w = 0; w < 8; ++w) acc[l] = __dp4a((int)q[w], (int)xw[w], acc[l]);
    }
    part = fmaf(d, fmaf(s[0], (float)acc[0], fmaf(s[1], (float)acc[1], s[2] * (float)acc[2])), part);
  }
  return part;
}

// Per token: the sums of the expert input xhat = x (or x / sqrt(mean(x^2) + eps)
// with the pre-norm residual) over each 32-value sub-block, for the min
// terms of the Q4_K gate/up rows.
__global__ void __launch_bounds__(256) k_q4k_input(const float *__restrict__ x, int H, int flags, float eps,
                                                   float *__restrict__ xsum) {
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
  // two threads per sub-block, 16 values each
  for (int base = 0; base < H / 16; base += 256) {  // the same trip count in every thread
    const int h2 = base + tid;
    float acc = 0.0f;
    if (h2 < H / 16) {
      const float4 *x4 = reinterpret_cast<const float4 *>(xt + 16 * h2);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = x4[i];
        acc += ((v.x * inv + v.y * inv) + (v.z * inv + v.w * inv));
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (h2 < H / 16 && (h2 & 1) == 0) xsum[(size_t)t * (H / 32) + (h2 >> 1)] = acc;
  }
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
      // gate and up rows of the pair together, on the input's int8 limbs
      const size_t rb = (size_t)(d.H / 256) * 144;
      const uint8_t *gr = a.gate + ((size_t)e * d.I + row) * rb, *ur = a.up + ((size_t)e * d.I + row) * rb;
      const float sc[3] = {a.xs[4 * t], a.xs[4 * t + 1], a.xs[4 * t + 2]};
      const uint8_t *const rows[2] = {gr, ur};
      float pp[2] = {0.0f, 0.0f};
      q4k_rows_part_limbs<2>(rows, a.xq + (size_t)t * 3 * d.H, d.H, sc, a.xsum + (size_t)t * (d.H / 32), lane, pp);
      hv = silu(warp_sum(pp[0])) * warp_sum(pp[1]);
    }
    if (lane == 0) a.h[(size_t)p * d.I + row] = hv;
  } else {
    if (row >= d.Is) return;
    const int t = p - npairs;
    const size_t rb = (size_t)(d.H / 32) * 34;
    const int8_t *xq = a.xq + (size_t)t * 3 * d.H;
    const float sc[3] = {a.xs[4 * t], a.xs[4 * t + 1], a.xs[4 * t + 2]};
    const float g = warp_sum(q80_row_part_limbs(a.sh_gate + (size_t)row * rb, xq, d.H, sc, lane));
    const float u = warp_sum(q80_row_part_limbs(a.sh_up + (size_t)row * rb, xq, d.H, sc, lane));
    if (lane == 0) a.hs[(size_t)t * d.Is + row] = silu(g) * u;
  }
}

// The down projection's inputs as int8 limbs: block v < T*k takes the routed
// SwiGLU output h[v] (I values), block T*k + t the shared one hs[t] (Is
// values): the vector's max |value| sets the limb scales (as for the expert
// input), each value becomes three int8 limbs, and the fp32 sums over each
// 32-value sub-block serve the min terms.
__global__ void __launch_bounds__(256) k_q4k_hlimbs(const Q4kArgs a) {
  const LayerDims &d = a.d;
  const int v = blockIdx.x, npairs = a.T * d.k, tid = threadIdx.x;
  const bool routed = v < npairs;
  const int len = routed ? d.I : d.Is;
  const float *src = routed ? a.h + (size_t)v * d.I : a.hs + (size_t)(v - npairs) * d.Is;
  int8_t *q = a.hq + (routed ? (size_t)v * 3 * d.I : (size_t)npairs * 3 * d.I + (size_t)(v - npairs) * 3 * d.Is);
  float *sum = a.hsum + (routed ? (size_t)v * (d.I / 32) : (size_t)npairs * (d.I / 32) + (size_t)(v - npairs) * (d.Is / 32));
  __shared__ float red[8];
  float amax = 0.0f;
  for (int i = tid; i < len; i += 256) amax = fmaxf(amax, fabsf(src[i]));
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  amax = 0.0f;
  for (int w = 0; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float s1 = amax > 0.f ? amax / 127.f : 1.f;
  const float s2 = s1 / 254.f, s3 = s2 / 254.f;
  const float r1 = 1.f / s1, r2 = 1.f / s2, r3 = 1.f / s3;
  uint32_t *q32 = reinterpret_cast<uint32_t *>(q);
  const int n4 = len / 4;
  for (int j = tid; j < n4; j += 256) {
    const float4 x4 = reinterpret_cast<const float4 *>(src)[j];
    const float e[4] = {x4.x, x4.y, x4.z, x4.w};
    uint32_t w1 = 0u, w2 = 0u, w3 = 0u;
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
      const float x = e[k4];
      const float q1 = fminf(fmaxf(rintf(x * r1), -127.f), 127.f);
      const float e1 = fmaf(-q1, s1, x);
      const float q2 = fminf(fmaxf(rintf(e1 * r2), -127.f), 127.f);
      const float e2 = fmaf(-q2, s2, e1);
      const float q3 = fminf(fmaxf(rintf(e2 * r3), -127.f), 127.f);
      w1 |= ((uint32_t)(int)q1 & 255u) << (8 * k4);
      w2 |= ((uint32_t)(int)q2 & 255u) << (8 * k4);
      w3 |= ((uint32_t)(int)q3 & 255u) << (8 * k4);
    }
    q32[j] = w1;
    q32[n4 + j] = w2;
    q32[2 * n4 + j] = w3;
  }
  for (int g = tid; g < len / 32; g += 256) {
    const float4 *x4 = reinterpret_cast<const float4 *>(src + 32 * g);
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 x = x4[i];
      acc += (x.x + x.y) + (x.z + x.w);
    }
    sum[g] = acc;
  }
  if (tid == 0) {
    a.hqs[4 * v] = s1;
    a.hqs[4 * v + 1] = s2;
    a.hqs[4 * v + 2] = s3;
    a.hqs[4 * v + 3] = 0.f;
  }
}

// y[t][r] = (x[t][r]) + shared_down[r] . hs[t] + sum_i w[t][i] down_e[r] . h[t,i],
// the routed terms in the routing's ascending expert order; one warp per
// output row, one dot product after the other, on the int8 limbs of h and hs
// by dp4a.  (Measured slower at one token with fp32 h: reading the k routed
// rows block by block together, 68 against 43 us per launch; one block per
// output row with a warp per dot product, 48 us.)
__global__ void __launch_bounds__(kRowsPerCta * 32) k_q4k_down(const Q4kArgs a) {
  const LayerDims &d = a.d;
  const int lane = threadIdx.x & 31, r = blockIdx.x * kRowsPerCta + (threadIdx.x >> 5), t = blockIdx.y;
  if (r >= d.H) return;
  const int npairs = a.T * d.k, vs = npairs + t;
  const size_t rbs = (size_t)(d.Is / 32) * 34, rbd = (size_t)(d.I / 256) * 144;
  const float ss[3] = {a.hqs[4 * vs], a.hqs[4 * vs + 1], a.hqs[4 * vs + 2]};
  float acc = warp_sum(q80_row_part_limbs(a.sh_down + (size_t)r * rbs,
                                          a.hq + (size_t)npairs * 3 * d.I + (size_t)t * 3 * d.Is, d.Is, ss, lane));
  for (int i = 0; i < d.k; ++i) {
    const int p = t * d.k + i, e = a.idx[p];
    if (e < 0 || e >= d.E) continue;
    const uint8_t *const rows[1] = {a.down + ((size_t)e * d.H + r) * rbd};
    const float sp[3] = {a.hqs[4 * p], a.hqs[4 * p + 1], a.hqs[4 * p + 2]};
    float o[1] = {0.0f};
    q4k_rows_part_limbs<1>(rows, a.hq + (size_t)p * 3 * d.I, d.I, sp, a.hsum + (size_t)p * (d.I / 32), lane, o);
    acc = fmaf(a.w[p], warp_sum(o[0]), acc);
  }
  if (lane == 0) {
    const size_t at = (size_t)t * d.H + r;
    a.y[at] = (d.flags & MOE_FLAG_PRENORM_RESIDUAL) ? a.x[at] + acc : acc;
  }
}

}  // namespace

size_t q4k_expert_bytes(const LayerDims &d, int T) {
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  const size_t nh = (size_t)T * d.k * d.I + (size_t)T * d.Is;  // down inputs: routed h, then shared hs
  return al(sizeof(float) * (size_t)T * d.k * d.I) + al(sizeof(float) * (size_t)T * d.Is) +
         al(sizeof(float) * (size_t)T * (d.H / 32)) + al(3 * nh) + al(sizeof(float) * 4 * ((size_t)T * d.k + T)) +
         al(sizeof(float) * (nh / 32));
}

cudaError_t q4k_experts(const Q4kArgs &a, cudaStream_t stream) {
  const LayerDims &d = a.d;
  if (a.T <= 0) return cudaSuccess;
  k_q4k_input<<<a.T, 256, 0, stream>>>(a.x, d.H, d.flags, d.eps, a.xsum);
  const int rmax = d.I > d.Is ? d.I : d.Is;
  k_q4k_gate_up<<<dim3((rmax + kRowsPerCta - 1) / kRowsPerCta, a.T * d.k + a.T), kRowsPerCta * 32, 0, stream>>>(a);
  k_q4k_hlimbs<<<a.T * d.k + a.T, 256, 0, stream>>>(a);
  k_q4k_down<<<dim3((d.H + kRowsPerCta - 1) / kRowsPerCta, a.T), kRowsPerCta * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
