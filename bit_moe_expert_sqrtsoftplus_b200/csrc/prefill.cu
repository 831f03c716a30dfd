// prefill.cu -- routing and token permutation for larger token counts.
//
// Router: z = W_r x for all tokens as a tiled fp32 GEMM on the CUDA cores,
// each 32-element K chunk summed with fp32 FMAs and the chunk sums added in
// fp64.  A chunk of n FMAs has error at most gamma_n * sum|w x| (Higham,
// "Accuracy and Stability of Numerical Algorithms", Thm 3.1 with
// gamma_n = n u / (1 - n u), u = 2^-24), and sum|w x| <= |w_e|_2 |x_t|_2
// (Cauchy-Schwarz), so each logit comes with a rigorous interval.  The
// sqrtsoftplus score is increasing in z, so the selection is certified when
// every selected key's lower end beats every other key's upper end; tokens
// that fail the test are recomputed in fp64 (exactly the oracle's reduction
// up to fp64 rounding order).
#include <float.h>
#include <math.h>

#include <cuda_fp16.h>

#include "common.cuh"
#include "gemm.cuh"
#include "launch.cuh"
#include "prefill.cuh"

namespace moe {

namespace {

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__device__ __forceinline__ double sqrtsoftplus(double z) { return sqrt(fmax(z, 0.0) + log1p(exp(-fabs(z)))); }

// ---------------------------------------------------------------- init

// 2-norm of every router row, rounded up to fp32.
__global__ void k_row_norms(const uint16_t *Wr, int E, int H, float *out) {
  const int e = blockIdx.x;
  double ss = 0.0;
  for (int j = threadIdx.x; j < H; j += blockDim.x) {
    double v = (double)half_bits_to_float(Wr[(size_t)e * H + j]);
    ss += v * v;
  }
  ss = warp_sum_d(ss);
  __shared__ double red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    out[e] = __double2float_ru(sqrt(t) * (1.0 + 1e-15));
  }
}

// ---------------------------------------------------------------- router

// Per token: inverse RMS (1 without the pre-norm flag) and the 2-norm of the
// router input, both in fp64.
__global__ void k_token_norms(const float *x, int T, int H, int flags, float eps, double *inv, double *nrm) {
  const int t = blockIdx.x;
  double ss = 0.0;
  // 16-byte loads (H is a multiple of 256 and rows are 16-byte aligned), four in flight per thread
  const float4 *x4 = reinterpret_cast<const float4 *>(x + (size_t)t * H);
#pragma unroll 4
  for (int j = threadIdx.x; j < H / 4; j += blockDim.x) {
    const float4 v = x4[j];
    ss += (double)v.x * (double)v.x + (double)v.y * (double)v.y + (double)v.z * (double)v.z +
          (double)v.w * (double)v.w;
  }
  ss = warp_sum_d(ss);
  __shared__ double red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
    double iv = (flags & MOE_FLAG_PRENORM_RESIDUAL) ? 1.0 / sqrt(tot / (double)H + (double)eps) : 1.0;
    inv[t] = iv;
    nrm[t] = sqrt(tot) * iv;
  }
}

// z[t][e] for a 64-token x 64-expert tile (T = 4096 and E = 256 give 256
// blocks, so every SM has work); 256 threads, each 4 tokens x 4 experts.  Per
// 32-element K chunk every output is a sum of 32 fp32 FMAs (the chunk the
// error bound below assumes), added to an fp64 accumulator; the tile shape
// does not change any output's arithmetic.  Rows are staged with 16-byte
// loads (x scaled by the token's fp32 inverse RMS, W_r converted from f16),
// transposed into K-major shared tiles; the next chunk's loads are in flight
// while the current one is multiplied.
constexpr int RE = 64, RK = 32;
// Router GEMM tiles: 128 tokens per block (8 per thread: 32 accumulators, one
// block per SM) once there are enough tokens to give every SM a block at E =
// 256, 64 below.
#ifndef MOE_ROUTER_WIDE_MIN_T
#define MOE_ROUTER_WIDE_MIN_T 2048
#endif
template <int RTT>
__global__ void __launch_bounds__(256) k_router_f32(const float *x, const double *inv, const uint16_t *Wr, int T,
                                                    int E, int H, double *z) {
  // RTT tokens x RE experts per block; thread (tx, ty) owns tokens ty*TPT ..
  // and experts tx*4 ..
  constexpr int TPT = RTT / 16, XP = RTT / 32;
  __shared__ __align__(16) float xs[RK][RTT + 4];
  __shared__ __align__(16) float ws[RK][RE + 4];
  const int t0 = blockIdx.x * RTT, e0 = blockIdx.y * RE;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  // staging roles: x float4 pieces (token i>>3, K quad i&7) for i = tid,
  // tid + 256, ..., and one W uint4 piece (expert tid>>2, K octet tid&3);
  // the pieces of chunk k0 + RK are loaded into registers while chunk k0 is
  // multiplied
  float invf[XP];
  const float *xrow[XP];
#pragma unroll
  for (int r = 0; r < XP; ++r) {
    const int i = tid + 256 * r;
    const int t = t0 + (i >> 3);
    invf[r] = t < T ? (float)inv[t] : 0.f;
    xrow[r] = t < T ? x + (size_t)t * H + 4 * (i & 7) : nullptr;
  }
  const int we = e0 + (tid >> 2);
  const uint16_t *wrow = we < E ? Wr + (size_t)we * H + 8 * (tid & 3) : nullptr;
  float4 xv_next[XP];
  uint4 wv_next;
  auto fetch = [&](int k0) {
#pragma unroll
    for (int r = 0; r < XP; ++r)
      xv_next[r] = xrow[r] ? *reinterpret_cast<const float4 *>(xrow[r] + k0) : make_float4(0.f, 0.f, 0.f, 0.f);
    wv_next = wrow ? *reinterpret_cast<const uint4 *>(wrow + k0) : make_uint4(0u, 0u, 0u, 0u);
  };
  double acc[TPT][4];
#pragma unroll
  for (int i = 0; i < TPT; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
  fetch(0);
  for (int k0 = 0; k0 < H; k0 += RK) {
#pragma unroll
    for (int r = 0; r < XP; ++r) {
      const int i = tid + 256 * r;
      const int tt = i >> 3, kq = i & 7;
      const float4 v = xv_next[r];
      xs[4 * kq + 0][tt] = v.x * invf[r];
      xs[4 * kq + 1][tt] = v.y * invf[r];
      xs[4 * kq + 2][tt] = v.z * invf[r];
      xs[4 * kq + 3][tt] = v.w * invf[r];
    }
    {
      const int ee = tid >> 2, ko = tid & 3;
      const uint32_t w4[4] = {wv_next.x, wv_next.y, wv_next.z, wv_next.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        ws[8 * ko + 2 * q][ee] = half_bits_to_float((uint16_t)(w4[q] & 0xFFFFu));
        ws[8 * ko + 2 * q + 1][ee] = half_bits_to_float((uint16_t)(w4[q] >> 16));
      }
    }
    __syncthreads();
    if (k0 + RK < H) fetch(k0 + RK);
    // each logit: a 32-term fp32 FMA chain from zero in K order, then added
    // into its fp64 accumulator (the same arithmetic whatever the tile)
    float part[TPT][4];
#pragma unroll
    for (int i = 0; i < TPT; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) part[i][j] = 0.f;
#pragma unroll 8
    for (int kk = 0; kk < RK; ++kk) {
      float xa[TPT];
#pragma unroll
      for (int q = 0; q < TPT / 4; ++q) {
        const float4 xv = *reinterpret_cast<const float4 *>(&xs[kk][ty * TPT + 4 * q]);
        xa[4 * q] = xv.x;
        xa[4 * q + 1] = xv.y;
        xa[4 * q + 2] = xv.z;
        xa[4 * q + 3] = xv.w;
      }
      const float4 wv = *reinterpret_cast<const float4 *>(&ws[kk][tx * 4]);
      const float wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int i = 0; i < TPT; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = fmaf(xa[i], wa[j], part[i][j]);
    }
#pragma unroll
    for (int i = 0; i < TPT; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] += (double)part[i][j];
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TPT; ++i) {
    const int t = t0 + ty * TPT + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) z[(size_t)t * E + e] = acc[i][j];
    }
  }
}

// Error bound of one logit.  The staged fp32 input fl(x * fl(inv)) is within
// 2u of x*inv per element; a 32-term FMA chunk adds at most gamma_33; the
// fp64 chunk additions and the oracle's own fp64 reduction are covered by
// the 1e-12 term; everything is proportional to sum|w x| <= |w|_2 |x|_2.
__device__ __forceinline__ double logit_bound(float wn, double xn) {
  const double u = 5.9604644775390625e-8;  // 2^-24
  const double g = 33.0 * u / (1.0 - 33.0 * u);
  return (g + 2.0 * u + 1e-12) * (double)wn * xn * (1.0 + 1e-6) + 1e-300;
}

// One warp per token: top-k from the fp32-GEMM logits; certified tokens get
// idx/w, the others are queued for the fp64 router.
__global__ void k_topk_cert(const double *z, const float *bias, const float *wn, const double *xn, int T, int E,
                            int k, float scaling, int32_t *idx, float *w, int32_t *fix) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const double *zt = z + (size_t)t * E;
  double key[8], dzs[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      dzs[i] = logit_bound(wn[e], xn[t]);
      key[i] = sqrtsoftplus(zt[e]) + (double)bias[e];
    } else {
      key[i] = -DBL_MAX;
      dzs[i] = 0.0;
    }
  }
  unsigned taken = 0;
  int sel[kMaxK];
#pragma unroll
  for (int r = 0; r < kMaxK; ++r) {
    sel[r] = INT_MAX;
    if (r < k) {
      double bk = -INFINITY;
      int be = INT_MAX;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !((taken >> i) & 1u) && key[i] > bk) {
          bk = key[i];
          be = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ok = __shfl_xor_sync(0xffffffffu, bk, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (ok > bk || (ok == bk && oe < be)) {
          bk = ok;
          be = oe;
        }
      }
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      sel[r] = be;
    }
  }
  // certificate: min lower end of the selected vs max upper end of the rest.
  // sqrt(softplus) has slope below 0.71 everywhere, so key -/+ dz (plus the
  // fp64 slack) bound an expert's interval; the exact ends
  // sqrtsoftplus(z -/+ dz) are evaluated only for experts whose coarse
  // bound does not settle the comparison, which certifies the same tokens.
  double sel_lo = DBL_MAX, rest_hi = -DBL_MAX;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    if (e >= E) continue;
    if ((taken >> i) & 1u)
      sel_lo = fmin(sel_lo, key[i] - dzs[i] - 2e-12);
    else
      rest_hi = fmax(rest_hi, key[i] + dzs[i] + 2e-12);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sel_lo = fmin(sel_lo, __shfl_xor_sync(0xffffffffu, sel_lo, o));
    rest_hi = fmax(rest_hi, __shfl_xor_sync(0xffffffffu, rest_hi, o));
  }
  if (!(sel_lo > rest_hi)) {
    const double coarse_lo = sel_lo, coarse_hi = rest_hi;
    sel_lo = DBL_MAX;
    rest_hi = -DBL_MAX;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e >= E) continue;
      const double b = (double)bias[e];
      if ((taken >> i) & 1u) {
        const double c = key[i] - dzs[i] - 2e-12;
        sel_lo = fmin(sel_lo, c > coarse_hi ? c : sqrtsoftplus(zt[e] - dzs[i]) + b - 1e-12);
      } else {
        const double c = key[i] + dzs[i] + 2e-12;
        rest_hi = fmax(rest_hi, c < coarse_lo ? c : sqrtsoftplus(zt[e] + dzs[i]) + b + 1e-12);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sel_lo = fmin(sel_lo, __shfl_xor_sync(0xffffffffu, sel_lo, o));
      rest_hi = fmax(rest_hi, __shfl_xor_sync(0xffffffffu, rest_hi, o));
    }
  }
  const bool certified = (k == E) || sel_lo > rest_hi;
  if (lane != 0) return;
  if (!certified) {
    const int slot = atomicAdd(fix, 1);
    fix[1 + slot] = t;
    fix[1 + T + slot] = 0;  // arrivals of the fix-up blocks of this slot
    return;
  }
  // ascending ids
  for (int i = 1; i < k; ++i)
    for (int j = i; j > 0 && sel[j - 1] > sel[j]; --j) {
      const int tmp = sel[j - 1];
      sel[j - 1] = sel[j];
      sel[j] = tmp;
    }
  double sv[kMaxK], tot = 0.0;
  for (int i = 0; i < k; ++i) {
    sv[i] = sqrtsoftplus(zt[sel[i]]);
    tot += sv[i];
  }
  for (int i = 0; i < k; ++i) {
    idx[(size_t)t * k + i] = sel[i];
    w[(size_t)t * k + i] = (float)((double)scaling * sv[i] / tot);
  }
}

// fp64 router for the queued tokens.  A work item is (queued token, group of
// kFixGroup experts); blocks stride over the items.  The token's x * inv is
// staged in shared memory as fp64; each warp takes experts of the group with
// 8 consecutive weights per 16-byte load per lane and four independent partial
// sums, and the logits go to z.  The block that completes a token's last group
// (an acquire/release count per queued token) selects its experts and weights.
constexpr int kFixGroup = 16;

__global__ void __launch_bounds__(256) k_router_fix(const float *x, const double *inv, const uint16_t *Wr,
                                                    const float *bias, int T, int E, int H, int k, float scaling,
                                                    int32_t *fix, double *z, int32_t *idx, float *w) {
  const int nfix = fix[0];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ngroups = (E + kFixGroup - 1) / kFixGroup;
  extern __shared__ double xsd[];  // [H]
  __shared__ int last_s;
  for (int item = blockIdx.x; item < nfix * ngroups; item += gridDim.x) {
    const int f = item / ngroups, grp = item % ngroups;
    const int t = fix[1 + f];
    const float *xt = x + (size_t)t * H;
    const double iv = inv[t];
    for (int j = threadIdx.x; j < H; j += blockDim.x) xsd[j] = (double)xt[j] * iv;
    __syncthreads();
    const int e1 = min(E, (grp + 1) * kFixGroup);
    for (int e = grp * kFixGroup + warp; e < e1; e += 8) {
      const uint16_t *we = Wr + (size_t)e * H;
      double acc[4] = {0.0, 0.0, 0.0, 0.0};
      for (int j0 = 8 * lane; j0 < H; j0 += 256) {
        const uint4 wv = __ldg(reinterpret_cast<const uint4 *>(we + j0));
        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[q] = fma((double)half_bits_to_float((uint16_t)(ww[q] & 0xFFFFu)), xsd[j0 + 2 * q], acc[q]);
          acc[q] = fma((double)half_bits_to_float((uint16_t)(ww[q] >> 16)), xsd[j0 + 2 * q + 1], acc[q]);
        }
      }
      const double sum = warp_sum_d((acc[0] + acc[1]) + (acc[2] + acc[3]));
      if (lane == 0) z[(size_t)t * E + e] = sum;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int old;
      asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;\n" : "=r"(old) : "l"(fix + 1 + T + f) : "memory");
      last_s = old == ngroups - 1;
    }
    __syncthreads();
    if (last_s && warp == 0) {
      const double *zt = z + (size_t)t * E;
      double key[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        key[i] = e < E ? sqrtsoftplus(__ldcg(zt + e)) + (double)bias[e] : -DBL_MAX;
      }
      unsigned taken = 0;
      int sel[kMaxK];
#pragma unroll
      for (int r = 0; r < kMaxK; ++r) {
        sel[r] = INT_MAX;
        if (r < k) {
          double bk = -INFINITY;
          int be = INT_MAX;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u) && key[i] > bk) {
              bk = key[i];
              be = e;
            }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const double ok = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (ok > bk || (ok == bk && oe < be)) {
              bk = ok;
              be = oe;
            }
          }
          if ((be & 31) == lane) taken |= 1u << (be >> 5);
          sel[r] = be;
        }
      }
      if (lane == 0) {
        for (int i = 1; i < k; ++i)
          for (int j = i; j > 0 && sel[j - 1] > sel[j]; --j) {
            const int tmp = sel[j - 1];
            sel[j - 1] = sel[j];
            sel[j] = tmp;
          }
        double sv[kMaxK], tot = 0.0;
        for (int i = 0; i < k; ++i) {
          sv[i] = sqrtsoftplus(__ldcg(zt + sel[i]));
          tot += sv[i];
        }
        for (int i = 0; i < k; ++i) {
          idx[(size_t)t * k + i] = sel[i];
          w[(size_t)t * k + i] = (float)((double)scaling * sv[i] / tot);
        }
      }
    }
    __syncthreads();
  }
}

// Hash routing: ids from the table (ascending), weights scaling / k.
__global__ void k_hash_route(const int32_t *token_ids, const int32_t *tid2eid, int vocab, int T, int k,
                             float scaling, int32_t *idx, float *w, int *err) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  int tid = token_ids[t];
  if (tid < 0 || tid >= vocab) {
    set_error(err, kErrTokenId);
    tid = 0;
  }
  int sel[kMaxK];
  for (int i = 0; i < k; ++i) sel[i] = tid2eid[(size_t)tid * k + i];
  for (int i = 1; i < k; ++i)
    for (int j = i; j > 0 && sel[j - 1] > sel[j]; --j) {
      const int tmp = sel[j - 1];
      sel[j - 1] = sel[j];
      sel[j] = tmp;
    }
  for (int i = 0; i < k; ++i) {
    idx[(size_t)t * k + i] = sel[i];
    w[(size_t)t * k + i] = scaling / (float)k;
  }
}

// ---------------------------------------------------------------- permutation

// counts[e] = number of pairs routed to e (one block per expert).
// The 8 expert ids of pairs i .. i+7 (-1 past n): two 16-byte loads when
// all 8 exist and idx is 16-byte aligned (i is a multiple of 8; a caller's
// idx from moe_route may be only 4-byte aligned).
__device__ __forceinline__ void load8_ids(const int32_t *idx, int n, int i, int (&v)[8]) {
  if (i + 8 <= n && (reinterpret_cast<uintptr_t>(idx) & 15u) == 0) {
    const int4 a = *reinterpret_cast<const int4 *>(idx + i), b = *reinterpret_cast<const int4 *>(idx + i + 4);
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = i + j < n ? idx[i + j] : -1;
  }
}

// counts[e] = pairs with expert e; one block per expert, 8 pairs per thread
// per pass.
__global__ void __launch_bounds__(256) k_perm_count(const int32_t *idx, int n, int32_t *counts) {
  const int e = blockIdx.x;
  int c = 0;
#pragma unroll 2
  for (int i = 8 * threadIdx.x; i < n; i += 8 * blockDim.x) {
    int v[8];
    load8_ids(idx, n, i, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) c += v[j] == e;
  }
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  __shared__ int red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    counts[e] = t;
  }
}

// Exclusive prefix sum of E <= kMaxE counts (one block of kMaxE threads):
// every count is read before any offset is written (counts may alias
// offsets), then a scan of warp sums.
__global__ void __launch_bounds__(kMaxE) k_perm_scan(const int32_t *counts, int E, int32_t *offsets) {
  __shared__ int wsum[kMaxE / 32];
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  const int c = e < E ? counts[e] : 0;
  int incl = c;  // inclusive scan within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();  // every count has been read
  int before = 0;
  for (int q = 0; q < warp; ++q) before += wsum[q];
  if (e < E) offsets[e] = before + incl - c;
  if (e == kMaxE - 1) {
    int total = 0;
    for (int q = 0; q < kMaxE / 32; ++q) total += wsum[q];
    offsets[E] = total;
  }
}

// perm[offsets[e] + rank] = pair id, ranks in ascending pair order (stable).
// One block per expert; per pass each thread takes 8 consecutive pairs, so
// the block's hits of a pass are ranked by a scan over threads (thread order
// is pair order).
__global__ void __launch_bounds__(256) k_perm_scatter(const int32_t *idx, int n, const int32_t *offsets, int32_t *perm) {
  const int e = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __shared__ int wcount[32];
  int base = offsets[e];
  for (int i0 = 0; i0 < n; i0 += 8 * blockDim.x) {
    const int i = i0 + 8 * threadIdx.x;
    int v[8];
    load8_ids(idx, n, i, v);
    int mine = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) mine += v[j] == e;
    int incl = mine;  // inclusive scan of the hit counts over the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) wcount[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
    for (int q = 0; q < nw; ++q) {
      if (q < warp) before += wcount[q];
      total += wcount[q];
    }
    int at = base + before + incl - mine;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (v[j] == e) perm[at++] = i + j;
    base += total;
    __syncthreads();
  }
}

}  // namespace

size_t prefill_big_bytes(const LayerDims &d, int T);

size_t prefill_scratch_bytes(const LayerDims &d, int T) {
  PrefillArgs p = prefill_args(d, LayerWeights{}, T, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
  return reinterpret_cast<size_t>(p.s.big) + prefill_big_bytes(d, T) + 256;
}

PrefillArgs prefill_args(const LayerDims &d, const LayerWeights &wt, int T, const float *x,
                         const int32_t *token_ids, float *y, void *scratch, const float *row_norms, int *err) {
  PrefillArgs p;
  p.d = d;
  p.wt = wt;
  p.T = T;
  p.x = x;
  p.token_ids = token_ids;
  p.y = y;
  p.row_norms = row_norms;
  p.ev_begin = nullptr;
  p.ev_end = nullptr;
  p.err = err;
  p.q4k = 0;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    off = align_up(off, 256);
    uint8_t *q = static_cast<uint8_t *>(scratch) + off;
    off += bytes;
    return q;
  };
  p.s.z = reinterpret_cast<float *>(take(sizeof(double) * (size_t)T * d.E));
  p.s.idx = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)T * d.k));
  p.s.w = reinterpret_cast<float *>(take(sizeof(float) * (size_t)T * d.k));
  p.s.counts = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * d.E));
  p.s.offsets = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (d.E + 1)));
  p.s.perm = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)T * d.k));
  p.s.fix = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)(2 * T + 1)));
  // token norms (2 x fp64 per token)
  take(2 * sizeof(double) * (size_t)T);
  p.s.big = static_cast<uint8_t *>(scratch) + align_up(off, 256);
  p.s.big_bytes = 0;
  return p;
}

cudaError_t prefill_init(const LayerDims &d, const LayerWeights &wt, float *row_norms, int *err, cudaStream_t s) {
  (void)err;
  if (d.mode != MOE_ROUTE_ROUTER) return cudaSuccess;
  k_row_norms<<<d.E, 256, 0, s>>>(wt.Wr, d.E, d.H, row_norms);
  return cudaGetLastError();
}

namespace {
// One thread per table row: the row must hold k distinct ids in [0, E);
// the smallest failing row index is kept in *first_bad.
__global__ void k_check_tid2eid(const int32_t *tab, int vocab, int k, int E, int *first_bad) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= vocab) return;
  const int32_t *r = tab + (size_t)row * k;
  int v[kMaxK];
  bool ok = true;
  for (int i = 0; i < k; ++i) {
    v[i] = r[i];
    if (v[i] < 0 || v[i] >= E) ok = false;
    for (int j = 0; j < i; ++j)
      if (v[j] == v[i]) ok = false;
  }
  if (!ok) atomicMin(first_bad, row);
}
}  // namespace

cudaError_t check_tid2eid(const LayerDims &d, const int32_t *tab, int *dev_word, int *first_bad, cudaStream_t s) {
  *first_bad = -1;
  cudaError_t e = cudaMemsetAsync(dev_word, 0x7F, sizeof(int), s);  // 0x7F7F7F7F > any row index
  if (e != cudaSuccess) return e;
  k_check_tid2eid<<<(d.vocab + 255) / 256, 256, 0, s>>>(tab, d.vocab, d.k, d.E, dev_word);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int v = 0;
  e = cudaMemcpyAsync(&v, dev_word, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  if (v < d.vocab) *first_bad = v;
  return cudaSuccess;
}

static double *token_norm_ptr(const PrefillArgs &p) {
  uint8_t *fixp = reinterpret_cast<uint8_t *>(p.s.fix);
  return reinterpret_cast<double *>(fixp + align_up(sizeof(int32_t) * (size_t)(2 * p.T + 1), 256));
}

cudaError_t prefill_route(const PrefillArgs &p, int32_t *idx, float *w, cudaStream_t s) {
  const LayerDims &d = p.d;
  const int T = p.T;
  if (d.mode == MOE_ROUTE_HASH) {
    k_hash_route<<<(T + 255) / 256, 256, 0, s>>>(p.token_ids, p.wt.tid2eid, d.vocab, T, d.k, d.scaling, idx, w,
                                                 p.err);
    return cudaGetLastError();
  }
  double *inv = token_norm_ptr(p);
  double *xn = inv + T;
  double *z = reinterpret_cast<double *>(p.s.z);
  cudaError_t e = cudaMemsetAsync(p.s.fix, 0, sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  k_token_norms<<<T, 256, 0, s>>>(p.x, T, d.H, d.flags, d.eps, inv, xn);
  if (T >= MOE_ROUTER_WIDE_MIN_T) {
    const dim3 g((T + 127) / 128, (d.E + RE - 1) / RE);
    k_router_f32<128><<<g, 256, 0, s>>>(p.x, inv, p.wt.Wr, T, d.E, d.H, z);
  } else {
    const dim3 g((T + 63) / 64, (d.E + RE - 1) / RE);
    k_router_f32<64><<<g, 256, 0, s>>>(p.x, inv, p.wt.Wr, T, d.E, d.H, z);
  }
  k_topk_cert<<<(T + 7) / 8, 256, 0, s>>>(z, p.wt.bias, p.row_norms, xn, T, d.E, d.k, d.scaling, idx, w, p.s.fix);
  // enough blocks for the usual handful of queued tokens; more stride
  const int nfix_items = T * ((d.E + kFixGroup - 1) / kFixGroup);
  const int nfix_blocks = nfix_items < 296 ? nfix_items : 296;
  const size_t fix_smem = sizeof(double) * (size_t)d.H;
  if (fix_smem > 48 * 1024) {  // the x row in fp64 for H > 6144; opt in to the most any H may need
    static SmemOptIn opt;
    if ((e = opt_in_smem(k_router_fix, kSmemOptInMax, opt)) != cudaSuccess) return e;
  }
  k_router_fix<<<nfix_blocks, 256, fix_smem, s>>>(p.x, inv, p.wt.Wr, p.wt.bias, T, d.E, d.H, d.k, d.scaling,
                                                  p.s.fix, z, idx, w);
  return cudaGetLastError();
}

namespace {

// x (optionally RMS-normalised) -> f16 [T][H], the B operand of the gate/up GEMMs.
__global__ void k_prep_x16(const float *x, int T, int H, int flags, float eps, __half *out) {
  const int t = blockIdx.x;
  const float *xt = x + (size_t)t * H;
  float inv = 1.f;
  if (flags & MOE_FLAG_PRENORM_RESIDUAL) {
    double ss = 0.0;
    for (int j = threadIdx.x; j < H; j += blockDim.x) ss += (double)xt[j] * (double)xt[j];
    ss = warp_sum_d(ss);
    __shared__ double red[32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    double tot = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
    inv = (float)(1.0 / sqrt(tot / (double)H + (double)eps));
  }
  for (int j = threadIdx.x * 4; j < H; j += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4 *>(xt + j);
    __half2 a = __floats2half2_rn(v.x * inv, v.y * inv);
    __half2 b = __floats2half2_rn(v.z * inv, v.w * inv);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t *>(&a);
    o.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(out + (size_t)t * H + j) = o;
  }
}

// y[t] += slots[t*k] + slots[t*k + 1] + ... (ascending slot = ascending expert id)
__global__ void k_sum_slots(int H, int k, const float *slots, float *y) {
  const int t = blockIdx.x;
  for (int j = threadIdx.x * 4; j < H; j += blockDim.x * 4) {
    float4 acc = *reinterpret_cast<const float4 *>(y + (size_t)t * H + j);
    for (int q = 0; q < k; ++q) {
      const float4 v = *reinterpret_cast<const float4 *>(slots + ((size_t)t * k + q) * H + j);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    *reinterpret_cast<float4 *>(y + (size_t)t * H + j) = acc;
  }
}

struct BigScratch {
  __half *x16;      // [T][H]
  uint16_t *hperm;  // [T*k][I] bf16, rows in permuted order
  uint16_t *hs;     // [T][Is] bf16
  float *slots;     // [T*k][H] weighted expert outputs per pair (deterministic combine only)
  uint16_t *sh16;   // shared expert rows expanded to 16 bits (T >= kSharedDenseMinT only): gate, up [Is][H], down [H][Is]
  size_t bytes;
};

BigScratch carve_big(const LayerDims &d, int T, void *base) {
  BigScratch b;
  size_t off = 0;
  auto take = [&](size_t n) {
    off = align_up(off, 256);
    uint8_t *q = static_cast<uint8_t *>(base) + off;
    off += n;
    return q;
  };
  b.x16 = reinterpret_cast<__half *>(take(2 * (size_t)T * d.H));
  b.hperm = reinterpret_cast<uint16_t *>(take(2 * (size_t)T * d.k * d.I));
  b.hs = reinterpret_cast<uint16_t *>(take(2 * (size_t)T * d.Is));
  b.slots = (d.flags & MOE_FLAG_DETERMINISTIC) ? reinterpret_cast<float *>(take(sizeof(float) * (size_t)T * d.k * d.H))
                                                : nullptr;
  b.sh16 = T >= kSharedDenseMinT ? reinterpret_cast<uint16_t *>(take(2 * 3 * (size_t)d.Is * d.H)) : nullptr;
  b.bytes = off;
  return b;
}

}  // namespace

size_t prefill_big_bytes(const LayerDims &d, int T) { return carve_big(d, T, nullptr).bytes; }

namespace {

// Routed gate/up GEMM over (token, slot) pairs grouped by expert: column c
// (offsets[g] <= c < offsets[g+1] for group g) reads activation row
// perm[c] / b_div of x16; SwiGLU outputs h (bf16) in grouped order.
GemmArgs routed_gateup_args(const LayerDims &d, const LayerWeights &wt, bool q4k, int n_groups,
                            const int32_t *offsets, const int32_t *perm, int b_div, const __half *x16,
                            uint16_t *hperm, int *err) {
  const size_t rbIQ = (size_t)(d.H / 256) * (q4k ? 144 : 66);
  GemmArgs g{};
  g.fmt = q4k ? kFmtQ4K : kFmtIQ2;
  g.bf16 = 0;
  g.epi = kEpiSwiGLU;
  g.M = d.I;
  g.K = d.H;
  g.n_groups = n_groups;
  g.offsets = offsets;
  g.A0 = wt.gate;
  g.A1 = wt.up;
  g.a_group_stride = (size_t)d.I * rbIQ;
  g.a_row_bytes = rbIQ;
  g.grid = wt.grid;
  g.b_base = reinterpret_cast<const uint16_t *>(x16);
  g.b_ld = d.H;
  g.b_perm = perm;
  g.b_div = b_div;
  g.h_out = hperm;
  g.h_ld = d.I;
  g.h_bf16 = 1;
  g.err = err;
  g.wait_cycles = d.wait_cycles;
  g.tmA = q4k ? nullptr : wt.gemm_tm;  // gate's map, then up's
  return g;
}

// Routed down GEMM: y[(perm[c] / k) * H + m] += w[perm[c]] * (W_down h)[m].
GemmArgs routed_down_args(const LayerDims &d, const LayerWeights &wt, bool q4k, int n_groups, const int32_t *offsets,
                          const int32_t *perm, int k, const uint16_t *hperm, const float *w, float *y, int *err) {
  const size_t rbQ2 = (size_t)(d.I / 256) * (q4k ? 144 : 84);
  GemmArgs rd{};
  rd.fmt = q4k ? kFmtQ4K : kFmtQ2K;
  rd.bf16 = 1;
  rd.epi = kEpiScatterAdd;
  rd.M = d.H;
  rd.K = d.I;
  rd.n_groups = n_groups;
  rd.offsets = offsets;
  rd.A0 = wt.down;
  rd.A1 = nullptr;
  rd.a_group_stride = (size_t)d.H * rbQ2;
  rd.a_row_bytes = rbQ2;
  rd.b_base = hperm;
  rd.b_ld = d.I;
  rd.b_perm = nullptr;
  rd.b_div = 1;
  rd.y = y;
  rd.y_ld = d.H;
  rd.w = w;
  rd.perm = perm;
  rd.k = k;
  rd.err = err;
  rd.wait_cycles = d.wait_cycles;
  rd.tmA = q4k || !wt.gemm_tm ? nullptr : static_cast<const uint8_t *>(wt.gemm_tm) + 2 * sizeof(TensorMap);
  return rd;
}

// The shared expert over T activation rows: SwiGLU into hs, then the down
// projection stored into y (plus res, the residual input, when given).
GemmArgs shared_gateup_args(const LayerDims &d, const LayerWeights &wt, int T, const __half *x16, uint16_t *hs,
                            int *err) {
  GemmArgs sg{};
  sg.fmt = kFmtQ80;
  sg.bf16 = 0;
  sg.epi = kEpiSwiGLU;
  sg.M = d.Is;
  sg.K = d.H;
  sg.n_groups = 1;
  sg.offsets = nullptr;
  sg.cols = T;
  sg.A0 = wt.sh_gate;
  sg.A1 = wt.sh_up;
  sg.a_group_stride = 0;
  sg.a_row_bytes = (size_t)(d.H / 32) * 34;
  sg.grid = wt.grid;
  sg.b_base = reinterpret_cast<const uint16_t *>(x16);
  sg.b_ld = d.H;
  sg.b_perm = nullptr;
  sg.b_div = 1;
  sg.h_out = hs;
  sg.h_ld = d.Is;
  sg.h_bf16 = 1;
  sg.err = err;
  sg.wait_cycles = d.wait_cycles;
  return sg;
}

GemmArgs shared_down_args(const LayerDims &d, const LayerWeights &wt, int T, const uint16_t *hs, const float *res,
                          float *y, int *err) {
  GemmArgs sd{};
  sd.fmt = kFmtQ80;
  sd.bf16 = 1;
  sd.epi = kEpiStore;
  sd.M = d.H;
  sd.K = d.Is;
  sd.n_groups = 1;
  sd.offsets = nullptr;
  sd.cols = T;
  sd.A0 = wt.sh_down;
  sd.A1 = nullptr;
  sd.a_row_bytes = (size_t)(d.Is / 32) * 34;
  sd.b_base = hs;
  sd.b_ld = d.Is;
  sd.b_div = 1;
  sd.y = y;
  sd.y_ld = d.H;
  sd.res = res;
  sd.err = err;
  sd.wait_cycles = d.wait_cycles;
  return sd;
}

cudaError_t shared_gemms(const LayerDims &d, const LayerWeights &wt, int T, const __half *x16, uint16_t *hs,
                         const float *res, float *y, int *err, cudaStream_t s, int num_sms) {
  cudaError_t e = grouped_gemm(shared_gateup_args(d, wt, T, x16, hs, err), s, num_sms);
  if (e != cudaSuccess) return e;
  return grouped_gemm(shared_down_args(d, wt, T, hs, res, y, err), s, num_sms);
}

// The same with the shared expert's rows expanded to 16 bits first (sh16:
// gate and up [Is][H] f16, then down [H][Is] bf16) and TMA-fed GEMMs: at
// large T every weight tile would otherwise be decoded once per 256 tokens.
cudaError_t shared_gemms_dense(const LayerDims &d, const LayerWeights &wt, int T, const __half *x16, uint16_t *hs,
                               uint16_t *sh16, const float *res, float *y, int *err, cudaStream_t s, int num_sms) {
  uint16_t *g16 = sh16, *u16 = g16 + (size_t)d.Is * d.H, *dn16 = u16 + (size_t)d.Is * d.H;
  cudaError_t e = expand_q80(wt.sh_gate, d.Is, d.H, 0, g16, s);
  if (e == cudaSuccess) e = expand_q80(wt.sh_up, d.Is, d.H, 0, u16, s);
  if (e == cudaSuccess) e = expand_q80(wt.sh_down, d.H, d.Is, 1, dn16, s);
  if (e != cudaSuccess) return e;
  e = dense_gemm(shared_gateup_args(d, wt, T, x16, hs, err), g16, u16, reinterpret_cast<const uint16_t *>(x16), s,
                 num_sms);
  if (e != cudaSuccess) return e;
  return dense_gemm(shared_down_args(d, wt, T, hs, res, y, err), dn16, nullptr, hs, s, num_sms);
}

}  // namespace

cudaError_t prefill_forward(const PrefillArgs &p, cudaStream_t s, int num_sms) {
  const LayerDims &d = p.d;
  const int T = p.T;
  cudaError_t e = prefill_route(p, p.s.idx, p.s.w, s);
  if (e != cudaSuccess) return e;
  e = permute(p.s.idx, T, d.k, d.E, p.s.offsets, p.s.perm, s);
  if (e != cudaSuccess) return e;
  BigScratch b = carve_big(d, T, p.s.big);
  k_prep_x16<<<T, 256, 0, s>>>(p.x, T, d.H, d.flags, d.eps, b.x16);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // routed gate/up: IQ2_XXS (or Q4_K) x f16 activations, SwiGLU -> h (bf16) in permuted order
  const GemmArgs g = routed_gateup_args(d, p.wt, p.q4k, d.E, p.s.offsets, p.s.perm, d.k, b.x16, b.hperm, p.err);
  if (p.ev_begin) cudaEventRecord(p.ev_begin, s);
  if ((e = grouped_gemm(g, s, num_sms)) != cudaSuccess) return e;
  if (p.ev_end) cudaEventRecord(p.ev_end, s);
  // shared expert: Q8_0 gate/up over all tokens, down stored into y (plus the residual input when pre-norm)
  const float *res = (d.flags & MOE_FLAG_PRENORM_RESIDUAL) ? p.x : nullptr;
  e = b.sh16 && d.shared_dense ? shared_gemms_dense(d, p.wt, T, b.x16, b.hs, b.sh16, res, p.y, p.err, s, num_sms)
                               : shared_gemms(d, p.wt, T, b.x16, b.hs, res, p.y, p.err, s, num_sms);
  if (e != cudaSuccess) return e;
  // routed down: Q2_K (or Q4_K) x bf16 h, y[token] += w * (W_down h)
  if (!(d.flags & MOE_FLAG_DETERMINISTIC))
    return grouped_gemm(routed_down_args(d, p.wt, p.q4k, d.E, p.s.offsets, p.s.perm, d.k, b.hperm, p.s.w, p.y, p.err),
                        s, num_sms);
  // deterministic: each pair's weighted output stored into its own slot row
  // (every pair is in exactly one expert's columns and every row of H is in
  // one tile, so each slot element is written once), then every token's
  // slots summed in ascending slot order
  GemmArgs rd = routed_down_args(d, p.wt, p.q4k, d.E, p.s.offsets, p.s.perm, 1, b.hperm, p.s.w, b.slots, p.err);
  rd.epi = kEpiSlotStore;
  if ((e = grouped_gemm(rd, s, num_sms)) != cudaSuccess) return e;
  k_sum_slots<<<T, 256, 0, s>>>(d.H, d.k, b.slots, p.y);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- expert parallelism

namespace {

// 1 / RMS of each token row in fp64 (1 without the pre-norm flag), as the
// single-GPU path scales the expert input.
__global__ void k_ep_inv(const float *x, int T, int H, int flags, float eps, float *inv) {
  const int t = blockIdx.x;
  if (!(flags & MOE_FLAG_PRENORM_RESIDUAL)) {
    if (threadIdx.x == 0) inv[t] = 1.f;
    return;
  }
  double ss = 0.0;
  for (int j = threadIdx.x; j < H; j += blockDim.x) ss += (double)x[(size_t)t * H + j] * (double)x[(size_t)t * H + j];
  ss = warp_sum_d(ss);
  __shared__ double red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
    inv[t] = (float)(1.0 / sqrt(tot / (double)H + (double)eps));
  }
}

// Dispatch row i (pairs in grouped order): the f16 expert input of token
// perm[i] / k, its expert id and routing weight.
__global__ void k_ep_pack(const float *x, const float *inv, int H, int k, const int32_t *idx, const float *w,
                          const int32_t *perm, __half *x_send, int32_t *e_send, float *w_send) {
  const int i = blockIdx.x;
  const int pr = perm[i], t = pr / k;
  const float sc = inv[t];
  const float *xt = x + (size_t)t * H;
  for (int j = threadIdx.x * 4; j < H; j += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4 *>(xt + j);
    __half2 a = __floats2half2_rn(v.x * sc, v.y * sc);
    __half2 b = __floats2half2_rn(v.z * sc, v.w * sc);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t *>(&a);
    o.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(x_send + (size_t)i * H + j) = o;
  }
  if (threadIdx.x == 0) {
    e_send[i] = idx[pr];
    w_send[i] = w[pr];
  }
}

// Received rows: global expert ids -> ids local to the shard; an id outside
// the shard is reported and its row gets no expert (local id -1).
__global__ void k_ep_local_ids(const int32_t *e_recv, int N, int e0, int E_local, int32_t *local, int *err) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const int e = e_recv[i] - e0;
  if (e < 0 || e >= E_local) {
    set_error(err, kErrTokenId);
    local[i] = -1;
  } else {
    local[i] = e;
  }
}

// y[t] += sum over the token's k pairs, in ascending slot order, of the
// returned expert rows; pos[t*k + slot] is the pair's row in the dispatch order.
__global__ void k_ep_combine(int H, int k, const int32_t *pos, const float *out, float *y) {
  const int t = blockIdx.x;
  for (int j = threadIdx.x * 4; j < H; j += blockDim.x * 4) {
    float4 acc = *reinterpret_cast<const float4 *>(y + (size_t)t * H + j);
    for (int q = 0; q < k; ++q) {
      const float4 v = *reinterpret_cast<const float4 *>(out + (size_t)pos[t * k + q] * H + j);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    *reinterpret_cast<float4 *>(y + (size_t)t * H + j) = acc;
  }
}

__global__ void k_inverse_perm(const int32_t *perm, int n, int32_t *pos) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) pos[perm[i]] = i;
}

}  // namespace

size_t ep_dispatch_scratch_bytes(const LayerDims &d, int T) {
  // the router's scratch (as the batched path carves it), then 1/RMS per token
  PrefillArgs p = prefill_args(d, LayerWeights{}, T, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
  return reinterpret_cast<size_t>(p.s.big) + align_up(sizeof(float) * (size_t)T, 256) + 256;
}

cudaError_t ep_dispatch(const PrefillArgs &p, int32_t *offsets, int32_t *perm, __half *x_send, int32_t *e_send,
                        float *w_send, cudaStream_t s) {
  const LayerDims &d = p.d;
  const int T = p.T;
  cudaError_t e = prefill_route(p, p.s.idx, p.s.w, s);
  if (e != cudaSuccess) return e;
  e = permute(p.s.idx, T, d.k, d.E, offsets, perm, s);
  if (e != cudaSuccess) return e;
  float *inv = reinterpret_cast<float *>(p.s.big);
  k_ep_inv<<<T, 256, 0, s>>>(p.x, T, d.H, d.flags, d.eps, inv);
  k_ep_pack<<<T * d.k, 256, 0, s>>>(p.x, inv, d.H, d.k, p.s.idx, p.s.w, perm, x_send, e_send, w_send);
  return cudaGetLastError();
}

size_t ep_experts_scratch_bytes(const LayerDims &d, int N) {
  size_t off = 0;
  auto take = [&](size_t n) { off = align_up(off, 256) + n; };
  take(sizeof(int32_t) * (size_t)N);        // local ids
  take(sizeof(int32_t) * (size_t)(d.E + 1));  // offsets
  take(sizeof(int32_t) * (size_t)N);        // perm
  take(2 * (size_t)N * d.I);                // h (bf16), grouped order
  return off + 256;
}

cudaError_t ep_experts(const LayerDims &d, const LayerWeights &wt, bool q4k, const __half *x_recv,
                       const int32_t *e_recv, const float *w_recv, int N, int e0, float *out, void *scratch,
                       int *err, cudaStream_t s, int num_sms) {
  uint8_t *base = static_cast<uint8_t *>(scratch);
  size_t off = 0;
  auto take = [&](size_t n) {
    off = align_up(off, 256);
    uint8_t *q = base + off;
    off += n;
    return q;
  };
  int32_t *local = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)N));
  int32_t *offsets = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)(d.E + 1)));
  int32_t *perm = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)N));
  uint16_t *h = reinterpret_cast<uint16_t *>(take(2 * (size_t)N * d.I));
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)N * d.H, s);
  if (e != cudaSuccess) return e;
  k_ep_local_ids<<<(N + 255) / 256, 256, 0, s>>>(e_recv, N, e0, d.E, local, err);
  if ((e = permute(local, N, 1, d.E, offsets, perm, s)) != cudaSuccess) return e;
  e = grouped_gemm(routed_gateup_args(d, wt, q4k, d.E, offsets, perm, 1, x_recv, h, err), s, num_sms);
  if (e != cudaSuccess) return e;
  // each received row is in one expert's columns at most: a plain store of
  // w * E(x) into its row (rows outside the shard stay zero)
  GemmArgs rd = routed_down_args(d, wt, q4k, d.E, offsets, perm, 1, h, w_recv, out, err);
  rd.epi = kEpiSlotStore;
  return grouped_gemm(rd, s, num_sms);
}

size_t ep_combine_scratch_bytes(const LayerDims &d, int T) {
  return align_up(sizeof(float) * (size_t)T, 256) + align_up(sizeof(int32_t) * (size_t)T * d.k, 256) +
         align_up(2 * (size_t)T * d.H, 256) + align_up(2 * (size_t)T * d.Is, 256) + 256;
}

cudaError_t ep_combine(const LayerDims &d, const LayerWeights &wt, const float *x, int T, const int32_t *perm,
                       const float *out_back, float *y, void *scratch, int *err, cudaStream_t s, int num_sms) {
  uint8_t *base = static_cast<uint8_t *>(scratch);
  size_t off = 0;
  auto take = [&](size_t n) {
    off = align_up(off, 256);
    uint8_t *q = base + off;
    off += n;
    return q;
  };
  (void)take(sizeof(float) * (size_t)T);
  int32_t *pos = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)T * d.k));
  __half *x16 = reinterpret_cast<__half *>(take(2 * (size_t)T * d.H));
  uint16_t *hs = reinterpret_cast<uint16_t *>(take(2 * (size_t)T * d.Is));
  k_prep_x16<<<T, 256, 0, s>>>(x, T, d.H, d.flags, d.eps, x16);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = shared_gemms(d, wt, T, x16, hs, (d.flags & MOE_FLAG_PRENORM_RESIDUAL) ? x : nullptr, y, err, s, num_sms);
  if (e != cudaSuccess) return e;
  const int n = T * d.k;
  k_inverse_perm<<<(n + 255) / 256, 256, 0, s>>>(perm, n, pos);
  k_ep_combine<<<T, 256, 0, s>>>(d.H, d.k, pos, out_back, y);
  return cudaGetLastError();
}

cudaError_t permute(const int32_t *idx, int T, int k, int E, int32_t *offsets, int32_t *perm, cudaStream_t s) {
  // the counts are written into offsets[0..E) and scanned in place
  const int n = T * k;
  k_perm_count<<<E, 256, 0, s>>>(idx, n, offsets);
  k_perm_scan<<<1, kMaxE, 0, s>>>(offsets, E, offsets);
  k_perm_scatter<<<E, 256, 0, s>>>(idx, n, offsets, perm);
  return cudaGetLastError();
}

}  // namespace moe
