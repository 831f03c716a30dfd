// decode.cu -- the layer for small token counts (T <= 32): two kernels.
//
//   k1_prep_router  x -> int8 limbs (optionally RMSNorm first); fp64 router
//                   logits, scores s = sqrtsoftplus(z) and selection keys
//                   s + bias, one block per pair of experts.
//   k2_experts      top-k routing from the keys (comparisons only, per CTA),
//                   then all the expert work as warp-sized units on one
//                   counter: every (16-row tile, 1024-element K part) of the
//                   shared and the routed gate/up matrices, then every
//                   (K part, 16-row output tile) of the shared and the routed
//                   down matrices, for the tokens of one job (2 per unit by
//                   default: one MMA column pair).  Packed rows are staged
//                   into shared memory by TMA tensor copies (cp.async where
//                   the row stride rules TMA out), decoded in registers into
//                   int8 A fragments and multiplied with mma.sync m16n8k32
//                   against the int8 limbs of the activations.  The warp that
//                   completes a gate/up tile applies the SwiGLU; the warp that
//                   completes a 1024-element slice of h quantises it into
//                   limbs and flags it, and down units wait for the slices
//                   they read.  The warp that completes an output tile sums
//                   its parts in a fixed order (deterministic) into y.
// k2 is launched as a programmatic dependent of k1: its set-up (tables,
// shared memory, the x limbs, the shared expert's first units) overlaps k1
// and the routing, and griddepcontrol.wait guards every read of k1's results.
//
// Activations enter the tensor cores as three int8 limbs with one scale per
// vector (per slice for h): x ~= s1*q1 + s2*q2 + s3*q3, s2 = s1/254,
// s3 = s2/254, which keeps x to 6e-8 of max|x|; the weight side is exact in
// int8 (IQ2_XXS grid values with signs, Q2_K code*scale <= 45, Q8_0 values),
// so the products are exact integers and only the fp32 block scaling rounds.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <float.h>
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "launch.cuh"
#include "layer.cuh"

namespace moe {

namespace {

constexpr int kWarps2 = 16;  // warps per CTA in k2 / k3 (at most)
#ifndef MOE_DECODE_CLAIM
#define MOE_DECODE_CLAIM 1
#endif
constexpr int kClaim = MOE_DECODE_CLAIM;  // consecutive units a warp claims at a time
#ifndef MOE_DECODE_AHEAD
#define MOE_DECODE_AHEAD 0
#endif
// 1: a unit is claimed and its first chunk staged while the previous unit's
// last chunk is computed; 0: only after it
constexpr bool kAheadClaim = MOE_DECODE_AHEAD != 0;
#ifndef MOE_DECODE_GUNROLL
#define MOE_DECODE_GUNROLL 2
#endif
constexpr int kGUnroll = MOE_DECODE_GUNROLL;  // unrolling of the IQ2_XXS group loop
#ifndef MOE_DECODE_BUNROLL
#define MOE_DECODE_BUNROLL 4
#endif
constexpr int kBUnroll = MOE_DECODE_BUNROLL;  // unrolling of the IQ2_XXS block loop (code size)
constexpr int kThreads2 = kWarps2 * kWarp;
// k2 threads: 12 warps for four token pairs, whose accumulators need more
// than the 128 registers a thread has at 16 warps
__host__ __device__ constexpr int k2_threads(int maxp) { return maxp >= 4 ? 12 * kWarp : kThreads2; }
constexpr int kStage2 = 16 * 272;      // chunk: 16 rows of <= 272 bytes
constexpr int kGpmBytes = 256 * 128;   // +/- codebook, 8 replicas
constexpr int kSelBytes = 128 * 128;   // byte-permute selectors per sign mask, 16 replicas

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// sqrt(softplus(z)) in fp64, softplus computed as max(z,0) + log1p(exp(-|z|)).
__device__ __forceinline__ double sqrtsoftplus(double z) { return sqrt(fmax(z, 0.0) + log1p(exp(-fabs(z)))); }

// ------------------------------------------------------------------ k1

constexpr int kRouterThreads = 256;

template <int MAXT>
__global__ void __launch_bounds__(kRouterThreads) k1_prep_router(DecodeArgs a) {
  pdl_launch_dependents();
  const LayerDims &d = a.d;
  const int T = a.T;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = kRouterThreads / 32;
  __shared__ double red[NW][3 * MAXT];
  __shared__ float redf[NW];

  {
    // per-call counters and flags of the expert kernel, spread over the grid
    const int V = T * d.k + T;
    const int nv = V * a.s.NSL, nh = (a.s.G + a.s.Jmax) * a.s.TM, ny = d.H / 16;
    for (int i = blockIdx.x * blockDim.x + tid; i < nv + nh + ny + 4; i += gridDim.x * blockDim.x) {
      if (i < nv) {
        a.s.hmax[i] = 0u;
        a.s.Xmax[i] = 0u;
        a.s.scount[i] = 0;
        a.s.ready[i] = 0;
      } else if (i < nv + nh) {
        a.s.hcount[i - nv] = 0;
      } else if (i < nv + nh + ny) {
        a.s.ycount[i - nv - nh] = 0;
      } else {
        a.s.work[i - nv - nh - ny] = 0;
      }
    }
  }

  if ((int)blockIdx.x < T) {
    // ---- activation limbs for token t; every thread takes float4 words
    // tid, tid + 256, ... and loads a batch of them before using any
    const int t = blockIdx.x;
    const float4 *xt = reinterpret_cast<const float4 *>(a.x + (size_t)t * d.H);
    const int n4 = d.H / 4;
    constexpr int kB = 4;
    double ss = 0.0;
    float amax = 0.f;
    for (int j0 = tid; j0 < n4; j0 += kB * kRouterThreads) {
      float4 v[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int j = j0 + u * kRouterThreads;
        v[u] = j < n4 ? xt[j] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          ss += (double)e[q] * (double)e[q];
          amax = fmaxf(amax, fabsf(e[q]));
        }
      }
    }
    ss = warp_sum_d(ss);
    amax = warp_max(amax);
    if (lane == 0) {
      red[warp][0] = ss;
      redf[warp] = amax;
    }
    __syncthreads();
    ss = 0.0;
    amax = 0.f;
    for (int w = 0; w < NW; ++w) {
      ss += red[w][0];
      amax = fmaxf(amax, redf[w]);
    }
    float inv = 1.f;
    if (d.flags & MOE_FLAG_PRENORM_RESIDUAL) {
      inv = (float)(1.0 / sqrt(ss / (double)d.H + (double)d.eps));
      amax = amax * inv;
    }
    const float s1 = amax > 0.f ? amax / 127.f : 1.f;
    const float s2 = s1 / 254.f, s3 = s2 / 254.f;
    const float r1 = 1.f / s1, r2 = 1.f / s2, r3 = 1.f / s3;
    uint32_t *q = reinterpret_cast<uint32_t *>(a.s.xq + (size_t)t * 3 * d.H);
    for (int j0 = tid; j0 < n4; j0 += kB * kRouterThreads) {
      float4 v[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int j = j0 + u * kRouterThreads;
        v[u] = j < n4 ? xt[j] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int j = j0 + u * kRouterThreads;
        if (j < n4) {
          const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
          uint32_t w1 = 0u, w2 = 0u, w3 = 0u;
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const float x = e[k4] * inv;
            const float q1 = fminf(fmaxf(rintf(x * r1), -127.f), 127.f);
            const float e1 = fmaf(-q1, s1, x);
            const float q2 = fminf(fmaxf(rintf(e1 * r2), -127.f), 127.f);
            const float e2 = fmaf(-q2, s2, e1);
            const float q3 = fminf(fmaxf(rintf(e2 * r3), -127.f), 127.f);
            w1 |= ((uint32_t)(int)q1 & 255u) << (8 * k4);
            w2 |= ((uint32_t)(int)q2 & 255u) << (8 * k4);
            w3 |= ((uint32_t)(int)q3 & 255u) << (8 * k4);
          }
          q[j] = w1;
          q[n4 + j] = w2;
          q[2 * n4 + j] = w3;
        }
      }
    }
    if (tid == 0) {
      float *sx = a.s.xs + 4 * t;
      sx[0] = s1;
      sx[1] = s2;
      sx[2] = s3;
      sx[3] = 0.f;
    }
    return;
  }

  if (d.mode != MOE_ROUTE_ROUTER) return;
  // ---- router logits, scores and keys for experts e0, e0 + 1 (fp64)
  const int e0 = 2 * ((int)blockIdx.x - T);
  if (e0 >= d.E) return;
  const bool two = e0 + 1 < d.E;
  const uint16_t *w0 = a.wt.Wr + (size_t)e0 * d.H;
  const uint16_t *w1 = a.wt.Wr + (size_t)(two ? e0 + 1 : e0) * d.H;
  // tokens in groups of MAXT (the two weight rows are re-read from L1/L2)
  for (int t0 = 0; t0 < T; t0 += MAXT) {
    const int nt = min(MAXT, T - t0);
    double acc0[MAXT], acc1[MAXT], ssq[MAXT];
#pragma unroll
    for (int t = 0; t < MAXT; ++t) acc0[t] = acc1[t] = ssq[t] = 0.0;
    // every thread covers 8 consecutive elements per pass; all loads of a pass are independent
    for (int j = tid * 8; j < d.H; j += kRouterThreads * 8) {
      const uint4 hv0 = *reinterpret_cast<const uint4 *>(w0 + j);
      const uint4 hv1 = *reinterpret_cast<const uint4 *>(w1 + j);
      float4 xv[MAXT][2];
#pragma unroll
      for (int t = 0; t < MAXT; ++t) {
        if (t < nt) {
          const float4 *xp = reinterpret_cast<const float4 *>(a.x + (size_t)(t0 + t) * d.H + j);
          xv[t][0] = xp[0];
          xv[t][1] = xp[1];
        }
      }
      const uint16_t *p0 = reinterpret_cast<const uint16_t *>(&hv0);
      const uint16_t *p1 = reinterpret_cast<const uint16_t *>(&hv1);
#pragma unroll
      for (int t = 0; t < MAXT; ++t) {
        if (t < nt) {
          const float xe[8] = {xv[t][0].x, xv[t][0].y, xv[t][0].z, xv[t][0].w,
                               xv[t][1].x, xv[t][1].y, xv[t][1].z, xv[t][1].w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const double xd = (double)xe[i];
            acc0[t] = fma((double)half_bits_to_float(p0[i]), xd, acc0[t]);
            acc1[t] = fma((double)half_bits_to_float(p1[i]), xd, acc1[t]);
            ssq[t] = fma(xd, xd, ssq[t]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < MAXT; ++t) {
      if (t < nt) {
        const double v0 = warp_sum_d(acc0[t]);
        const double v1 = warp_sum_d(acc1[t]);
        const double v2 = warp_sum_d(ssq[t]);
        if (lane == 0) {
          red[warp][t] = v0;
          red[warp][MAXT + t] = v1;
          red[warp][2 * MAXT + t] = v2;
        }
      }
    }
    __syncthreads();
    if (tid < 2 * nt) {
      const int t = tid >> 1, which = tid & 1;
      if (which == 0 || two) {
        double z = 0.0, s2 = 0.0;
        for (int w = 0; w < NW; ++w) {
          z += red[w][which * MAXT + t];
          s2 += red[w][2 * MAXT + t];
        }
        if (d.flags & MOE_FLAG_PRENORM_RESIDUAL) z *= 1.0 / sqrt(s2 / (double)d.H + (double)d.eps);
        const int e = e0 + which;
        const double sc = sqrtsoftplus(z);
        a.s.sc[(size_t)(t0 + t) * d.E + e] = sc;
        a.s.z[(size_t)(t0 + t) * d.E + e] = sc + (double)a.wt.bias[e];
      }
    }
    __syncthreads();  // red is reused by the next group
  }
}

// ------------------------------------------------------------------ routing

// One warp: top-k of token t by key (ties to the lower id), ids in ascending
// order, weights scaling * s / sum(s) with the sum taken in ascending id
// order.  Keys come from k1 (router mode) or the token-id table (hash mode).
// Every lane loads its 8 keys and scores at once; each of the k rounds is a
// warp arg-max over (key, id) followed by a broadcast of the winner's score;
// the ids are then ranked in registers, so nothing waits on memory twice.
__device__ void warp_route_token(const DecodeArgs &a, int t, int32_t *idx_out, float *w_out) {
  const LayerDims &d = a.d;
  const int lane = threadIdx.x & 31;
  const int k = d.k;
  int sel[kMaxK];
  double ssel[kMaxK];
  if (d.mode == MOE_ROUTE_HASH) {
    int tid = a.token_ids[t];
    if (tid < 0 || tid >= d.vocab) {
      if (lane == 0) set_error(a.err, kErrTokenId);
      tid = 0;
    }
#pragma unroll
    for (int i = 0; i < kMaxK; ++i) {
      sel[i] = i < k ? a.wt.tid2eid[(size_t)tid * k + i] : INT_MAX;
      ssel[i] = 0.0;
    }
  } else {
    const double *kt = a.s.z + (size_t)t * d.E;
    const double *stt = a.s.sc + (size_t)t * d.E;
    double key[8], scv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      key[i] = e < d.E ? kt[e] : -DBL_MAX;
      scv[i] = e < d.E ? stt[e] : 0.0;
    }
    unsigned taken = 0;
#pragma unroll
    for (int r = 0; r < kMaxK; ++r) {
      sel[r] = INT_MAX;
      ssel[r] = 0.0;
      if (r < k) {
        // this lane's best untaken key (slots in id order, so the first wins ties)
        double bk = -INFINITY, bs = 0.0;
        int be = INT_MAX;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = lane + 32 * i;
          if (e < d.E && !((taken >> i) & 1u) && key[i] > bk) {
            bk = key[i];
            be = e;
            bs = scv[i];
          }
        }
        const double my_s = bs;
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
        ssel[r] = __shfl_sync(0xffffffffu, my_s, be & 31);
      }
    }
  }
  // rank the ids (stable for repeated ids of the hash table)
  int rank[kMaxK];
#pragma unroll
  for (int i = 0; i < kMaxK; ++i) {
    rank[i] = 0;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k && i < k) rank[i] += (sel[j] < sel[i]) || (sel[j] == sel[i] && j < i);
  }
  int ids[kMaxK];
  double srt[kMaxK];
#pragma unroll
  for (int pos = 0; pos < kMaxK; ++pos) {
    ids[pos] = INT_MAX;
    srt[pos] = 0.0;
#pragma unroll
    for (int i = 0; i < kMaxK; ++i)
      if (i < k && rank[i] == pos) {
        ids[pos] = sel[i];
        srt[pos] = ssel[i];
      }
  }
  double tot = 0.0;
#pragma unroll
  for (int pos = 0; pos < kMaxK; ++pos)
    if (pos < k) tot += srt[pos];
#pragma unroll
  for (int pos = 0; pos < kMaxK; ++pos) {
    if (pos < k && lane == pos) {
      idx_out[pos] = ids[pos];
      w_out[pos] = d.mode == MOE_ROUTE_HASH ? d.scaling / (float)k : (float)((double)d.scaling * srt[pos] / tot);
    }
  }
}

// Job table: the distinct selected experts in ascending order, each with its
// (token, slot) pairs in ascending token order; an expert with more than
// uw pairs (the kernel's unit width) is split into consecutive jobs of at most uw.
struct Jobs {
  int n;
  int e[kDecodeMaxT * kMaxK];
  int first[kDecodeMaxT * kMaxK];
  int cnt[kDecodeMaxT * kMaxK];
  int pair[kDecodeMaxT * kMaxK];  // sorted t*k + slot
  int rank_e[kDecodeMaxT * kMaxK];
};
static_assert(sizeof(Jobs) == sizeof(int) * kJobsInts, "job table layout");

// Built by one warp (no block barrier): ranks of the (token, slot) pairs by
// (expert, token), then the group starts by ballot.
__device__ void warp_build_jobs(const int32_t *idx_s, int T, int k, int uw, Jobs &J) {
  const int lane = threadIdx.x & 31;
  const int np = T * k;
  for (int i = lane; i < np; i += 32) {
    const int ei = idx_s[i], ti = i / k;
    int rank = 0;
    for (int j = 0; j < np; ++j) {
      const int ej = idx_s[j], tj = j / k;
      rank += (ej < ei) || (ej == ei && tj < ti);
    }
    J.pair[rank] = i;
    J.rank_e[rank] = ei;
  }
  __syncwarp();
  int ng = 0;
  for (int base = 0; base < np; base += 32) {
    const int rr = base + lane;
    const bool first = rr < np && (rr == 0 || J.rank_e[rr] != J.rank_e[rr - 1]);
    const unsigned m = __ballot_sync(0xffffffffu, first);
    if (first) {
      const int g = ng + __popc(m & ((1u << lane) - 1u));
      J.e[g] = J.rank_e[rr];
      J.first[g] = rr;
    }
    ng += __popc(m);
  }
  __syncwarp();
  for (int g = lane; g < ng; g += 32) J.cnt[g] = (g + 1 < ng ? J.first[g + 1] : np) - J.first[g];
  __syncwarp();
  if (T <= uw) {  // an expert holds at most one pair per token: none exceeds a unit
    if (lane == 0) J.n = ng;
    __syncwarp();
    return;
  }
  // split: every lane takes groups lane, lane + 32, ... (at most 8 with
  // np <= 256); exclusive prefix of the job counts over the groups in order
  int ge[8], gf[8], gc[8], nj[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int g = lane + 32 * q;
    ge[q] = g < ng ? J.e[g] : 0;
    gf[q] = g < ng ? J.first[g] : 0;
    gc[q] = g < ng ? J.cnt[g] : 0;
    nj[q] = (gc[q] + uw - 1) / uw;
  }
  __syncwarp();
  int base = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    // jobs of the groups before lane + 32q: all of round q's lower lanes plus base
    int incl = nj[q];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int start = base + incl - nj[q];
    for (int c = 0; c < nj[q]; ++c) {
      J.e[start + c] = ge[q];
      J.first[start + c] = gf[q] + uw * c;
      J.cnt[start + c] = min(uw, gc[q] - uw * c);
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) J.n = base;
  __syncwarp();
}

// ------------------------------------------------------------------ staging

__device__ __forceinline__ void cp_async8(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ int stage_rs(int bpr) { return (int)align_up((size_t)bpr, 16); }

struct Chunk {
  const uint8_t *g;  // row 0 of the tile at the chunk's first block
  size_t gstride;    // global row stride (bytes)
  int bpr;           // bytes per row in the chunk
  int nb;            // blocks in the chunk
  int k0;            // first element (K index) of the chunk
  int piece;         // copy granularity: 16, 8, 4 (cp.async) or 2 (plain loads)
  int align;         // alignment the decoder needs at the start of a staged row (4 or 8)
  int tm;            // TMA: tensor map index
  int tx, ty;        // TMA: box origin (16-bit elements along the row, first row)
  int tshift;        // TMA: bytes from the box origin to the chunk's first byte
};

// TMA chunk load: one lane arms the stage's mbarrier with the box bytes and
// issues one 2-D tensor copy of 16 rows x the staged row width; returns where
// the chunk's data starts in each staged row.
__device__ __forceinline__ int stage_chunk_tma(uint8_t *st, uint64_t *mbar, const TensorMap *tm, const Chunk &c) {
  if ((threadIdx.x & 31) == 0) {
    const uint32_t bytes = 16u * (uint32_t)stage_rs(c.bpr);
    const uint32_t mb = smem_u32(mbar);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(mb), "r"(bytes) : "memory");
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::
            "r"(smem_u32(st)),
        "l"(reinterpret_cast<uint64_t>(tm + c.tm)), "r"(c.tx), "r"(c.ty), "r"(mb)
        : "memory");
  }
  return c.tshift;
}

// Bounded wait for phase `parity` of an mbarrier; false (and the timeout
// error recorded) if it does not complete.  Each try_wait may suspend the
// warp for up to kSuspendNs (it resumes as soon as the phase completes), so
// a waiting warp takes few issue slots from the warps that compute.
#ifndef MOE_MBAR_SUSPEND_NS
#define MOE_MBAR_SUSPEND_NS 0
#endif
constexpr unsigned kSuspendNs = MOE_MBAR_SUSPEND_NS;
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *mbar, uint32_t parity, int *err) {
  const uint32_t mb = smem_u32(mbar);
  const long long t0 = clock64();
  while (true) {
    uint32_t ok;
    if (kSuspendNs > 0)
      asm volatile(
          "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}\n"
          : "=r"(ok)
          : "r"(mb), "r"(parity), "n"(kSuspendNs)
          : "memory");
    else
      asm volatile(
          "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
          : "=r"(ok)
          : "r"(mb), "r"(parity)
          : "memory");
    if (ok) return true;
    if (clock64() - t0 > kDefaultWaitCycles) {
      set_error(err, kErrTimeout);
      return false;
    }
  }
}

__host__ __device__ __forceinline__ int piece_for(size_t gstride, size_t off, int bpr) {
  const size_t m = gstride | off | (size_t)bpr;
  return (m & 15) == 0 ? 16 : (m & 7) == 0 ? 8 : (m & 3) == 0 ? 4 : 2;
}


// Copies one chunk (16 rows x bpr bytes) into the stage (row stride RS) and
// returns where the chunk's data starts in each staged row.
//
// Fast path, when all rows start at the same 4-byte phase of a 16-byte line
// (row stride a multiple of 16): each row is copied from the 16-byte boundary
// at or below its start, in 16-byte pieces plus an 8- and a 4-byte tail, two
// rows per pass of the warp; the data then starts `shift` (0, 4, 8 or 12)
// bytes into the staged row.  The bytes before the chunk belong to the same
// row.
// Otherwise rows are walked in order and each lane issues the pieces lane,
// lane + 32, ... of a row in the chunk's own granularity (data at offset 0).
__device__ __forceinline__ int stage_chunk(uint8_t *st, const Chunk &c) {
  const int lane = threadIdx.x & 31;
  const int RS = stage_rs(c.bpr);
  const int shift = (int)(reinterpret_cast<uintptr_t>(c.g) & 15);
  if ((c.gstride & 15) == 0 && (shift & (c.align - 1)) == 0 && shift + c.bpr <= RS && ((shift + c.bpr) & 3) == 0) {
    const int end = shift + c.bpr;
    const int n16 = end >> 4;
    const int t8 = end & 8, t4 = end & 4;  // tail: an 8-byte piece, then a 4-byte piece
    const uint8_t *g0 = c.g - shift;
    const int half = lane >> 4, l16 = lane & 15;
#pragma unroll 1
    for (int i = 0; i < 8; ++i) {
      const int row = 2 * i + half;
      const uint8_t *gr = g0 + (size_t)row * c.gstride;
      uint8_t *sr = st + row * RS;
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int pc = l16 + 16 * m;
        if (pc < n16) {
          cp_async16(sr + 16 * pc, gr + 16 * pc);
        } else if (pc == n16) {
          if (t8) cp_async8(sr + 16 * pc, gr + 16 * pc);
          if (t4) cp_async4(sr + 16 * pc + t8, gr + 16 * pc + t8);
        }
      }
    }
    cp_async_commit();
    return shift;
  }
  const int n = c.bpr / c.piece;
  const uint8_t *g = c.g;
  uint8_t *s = st;
  if (c.piece == 8) {
    for (int row = 0; row < 16; ++row, g += c.gstride, s += RS) {
      for (int o = lane; o < n; o += 32) cp_async8(s + 8 * o, g + 8 * o);
    }
  } else if (c.piece == 16) {
    for (int row = 0; row < 16; ++row, g += c.gstride, s += RS) {
      for (int o = lane; o < n; o += 32) cp_async16(s + 16 * o, g + 16 * o);
    }
  } else if (c.piece == 4) {
    for (int row = 0; row < 16; ++row, g += c.gstride, s += RS) {
      for (int o = lane; o < n; o += 32) cp_async4(s + 4 * o, g + 4 * o);
    }
  } else {
    for (int row = 0; row < 16; ++row, g += c.gstride, s += RS) {
      for (int o = lane; o < n; o += 32)
        *reinterpret_cast<uint16_t *>(s + 2 * o) = *reinterpret_cast<const uint16_t *>(g + 2 * o);
    }
  }
  cp_async_commit();
  return 0;
}

// Runs a list of chunks through the warp's two-stage ring; `compute(i, data)`
// consumes chunk i, whose staged rows start at `data` (row stride RS).
template <typename ChunkAt, typename Compute>
__device__ __forceinline__ void run_chunks(uint8_t *stage0, uint8_t *stage1, int n, ChunkAt chunk_at,
                                           Compute compute) {
  int sh_cur = stage_chunk(stage0, chunk_at(0));
  for (int i = 0; i < n; ++i) {
    uint8_t *cur = (i & 1) ? stage1 : stage0;
    uint8_t *nxt = (i & 1) ? stage0 : stage1;
    int sh_next = 0;
    if (i + 1 < n)
      sh_next = stage_chunk(nxt, chunk_at(i + 1));
    else
      cp_async_commit();
    cp_async_wait<1>();
    __syncwarp();
    compute(i, cur + sh_cur);
    __syncwarp();
    sh_cur = sh_next;
  }
}

// Dynamic unit scheduling on the warp's two-stage ring.  A warp claims G
// consecutive units at a time (claim() returns the first, warp-uniform); the
// ring runs on across unit boundaries.
//   valid(u)          -> false once u is past the last unit (may wait until
//                        the unit count is known)
//   unit_at(u)        -> UnitT with field nch (chunks of the unit)
//   chunk_of(unit, c) -> Chunk c of the unit
//   compute(unit, u, c, data, next_u): consume chunk c of unit u, staged at
//                        `data`; next_u is the unit of the next chunk the warp
//                        computes (-1 when none), for segment bookkeeping
template <int G, bool AHEAD, bool TMA, typename UnitT, typename Claim, typename Valid, typename UnitAt,
          typename ChunkOf, typename Compute>
__device__ __forceinline__ void run_units(uint8_t *st0, uint8_t *st1, uint64_t *mbar, const TensorMap *tm,
                                          int *err, Claim claim, Valid valid, UnitAt unit_at, ChunkOf chunk_of,
                                          Compute compute) {
  int s_u = 0, s_left = 0, s_c = 0;
  UnitT su;
  // stages the next chunk into slot `slot` (TMA) or commits its cp.async group
  auto stage_next = [&](uint8_t *dst, int slot, int &uid, int &cidx, int &shift) -> bool {
    if (s_c == 0) {
      if (s_left == 0) {
        s_u = claim();
        s_left = G;
      } else {
        ++s_u;
      }
      --s_left;
      if (!valid(s_u)) {
        s_left = 0;
        if (!TMA) cp_async_commit();
        return false;
      }
      su = unit_at(s_u);
    }
    uid = s_u;
    cidx = s_c;
    shift = TMA ? stage_chunk_tma(dst, mbar + slot, tm, chunk_of(su, s_c)) : stage_chunk(dst, chunk_of(su, s_c));
    if (++s_c == su.nch) s_c = 0;
    return true;
  };
  int uA = 0, cA = 0, shA = 0;
  bool haveA = stage_next(st0, 0, uA, cA, shA);
  UnitT cu;
  for (int i = 0; haveA; ++i) {
    uint8_t *cur = (i & 1) ? st1 : st0;
    uint8_t *nxt = (i & 1) ? st0 : st1;
    if (cA == 0) cu = unit_at(uA);
    int uB = 0, cB = 0, shB = 0;
    bool haveB = false;
    // with AHEAD the next unit is claimed while this chunk is computed,
    // otherwise only after it
    const bool defer = !AHEAD && s_c == 0 && s_left == 0;
    if (!defer) haveB = stage_next(nxt, (i + 1) & 1, uB, cB, shB);
    else if (!TMA) cp_async_commit();
    if (TMA) {
      // chunk i is the (i / 2)-th use of its slot
      if (!mbar_wait_bounded(mbar + (i & 1), (uint32_t)(i >> 1) & 1u, err)) {
        // leave after the other slot's copy (if any) has landed
        if (haveB) mbar_wait_bounded(mbar + ((i + 1) & 1), (uint32_t)((i + 1) >> 1) & 1u, err);
        __syncwarp();
        return;
      }
    } else {
      cp_async_wait<1>();
    }
    __syncwarp();
    compute(cu, uA, cA, cur + shA, defer ? -1 : (haveB ? uB : -1));
    __syncwarp();
    if (defer) haveB = stage_next(nxt, (i + 1) & 1, uB, cB, shB);
    uA = uB;
    cA = cB;
    shA = shB;
    haveA = haveB;
  }
}

// This CTA's share of the next layer's prefetch regions, in pieces of at
// most 64 KB (one thread issues them; they complete on their own).
__device__ void prefetch_next_layer(const NextLayerPrefetch &pf) {
  for (int r = 0; r < kPrefetchRegions; ++r) {
    const size_t n = pf.bytes[r];
    if (!pf.ptr[r] || n == 0) continue;
    const size_t per = (n / gridDim.x + 15) & ~(size_t)15;
    const size_t b0 = per * blockIdx.x;
    const size_t b1 = min(n, b0 + per);
    const uint8_t *base = static_cast<const uint8_t *>(pf.ptr[r]);
    for (size_t o = b0; o < b1; o += 65536) {
      const uint32_t sz = (uint32_t)min((size_t)65536, b1 - o);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(base + o), "r"(sz) : "memory");
    }
  }
}

// ------------------------------------------------------------------ decoders

// B operand column (the int8 limbs of one vector) in shared or global memory;
// `ok` is false for the padding columns, which read as zero.
struct BColS {
  const int8_t *p;  // shared memory
  bool ok;
};
struct BColG {
  const int8_t *p;  // global memory
  bool ok;
};
__device__ __forceinline__ uint2 ldb(const BColS &b, int kel) {
  uint2 v = make_uint2(0u, 0u);
  if (b.ok) v = *reinterpret_cast<const uint2 *>(b.p + kel);
  return v;
}
__device__ __forceinline__ uint2 ldb(const BColG &b, int kel) {
  uint2 v = make_uint2(0u, 0u);
  if (b.ok) v = __ldcg(reinterpret_cast<const uint2 *>(b.p + kel));  // via L2: may be written by this kernel
  return v;
}
__device__ __forceinline__ uint32_t ldx(const BColG &b, int off) {
  return b.ok ? __ldcg(reinterpret_cast<const unsigned *>(b.p + off)) : 0u;
}

// IQ2_XXS group of one staged row -> the A fragment halves of sub-vector c,
// and the group's scale factor 2s+1.  `o` is the group's byte offset in the row
// (a compile-time constant once the loops are unrolled, so is its alignment).
__device__ __forceinline__ void iq2_group(const uint8_t *rowc, const uint8_t *row, int o, int sh7,
                                          const uint8_t *gpm_l, const uint8_t *sel_l, uint32_t &lo, uint32_t &hi,
                                          int &f) {
  const uint32_t ix = rowc[o];  // rowc = row + c
  uint32_t S;
  if (((o + 4) & 3) == 0)
    S = lds_u32(row + o + 4);
  else
    S = lds_u16(row + o + 4) | (lds_u16(row + o + 6) << 16);
  const uint32_t m7 = (S >> sh7) & 127u;
  const uint4 gv = *reinterpret_cast<const uint4 *>(gpm_l + (ix << 7));
  const uint2 sv = *reinterpret_cast<const uint2 *>(sel_l + (m7 << 7));
  lo = __byte_perm(gv.x, gv.y, sv.x);
  hi = __byte_perm(gv.z, gv.w, sv.y);
  f = (int)((S >> 27) | 1u);  // 2s + 1
}

template <int NB, int MAXP, typename BCol>
__device__ __forceinline__ void iq2_chunk(const uint8_t *st, int k0, const uint8_t *gpm_l, const uint8_t *sel_l,
                                          const BCol (&bcol)[MAXP], int npairs, float (&F)[MAXP][4]) {
  constexpr int RS = (NB * 66 + 15) / 16 * 16;
  const int lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
  const int sh7 = 7 * c;
  const uint8_t *row0 = st + r * RS;
  const uint8_t *row1 = row0 + 8 * RS;
#pragma unroll kBUnroll
  for (int b = 0; b < NB; ++b) {
    const float d0 = half_bits_to_float(lds_u16(row0 + 66 * b)) * 0.125f;
    const float d1 = half_bits_to_float(lds_u16(row1 + 66 * b)) * 0.125f;
    int acc[MAXP][4];
#pragma unroll
    for (int p = 0; p < MAXP; ++p) acc[p][0] = acc[p][1] = acc[p][2] = acc[p][3] = 0;
#pragma unroll kGUnroll
    for (int g = 0; g < 8; ++g) {
      const int o = 66 * b + 2 + 8 * g;
      uint32_t A[4];
      int f0, f1;
      iq2_group(row0 + c, row0, o, sh7, gpm_l, sel_l, A[0], A[2], f0);
      iq2_group(row1 + c, row1, o, sh7, gpm_l, sel_l, A[1], A[3], f1);
      const int kel = k0 + 256 * b + 32 * g;  // the column base includes 8c
#pragma unroll
      for (int p = 0; p < MAXP; ++p) {
        if (MAXP == 1 || p < npairs) {
          const uint2 bb = ldb(bcol[p], kel);
          const int zero[4] = {0, 0, 0, 0};
          int cg[4];
          mma_s8(cg, A, bb.x, bb.y, zero);
          acc[p][0] += cg[0] * f0;
          acc[p][1] += cg[1] * f0;
          acc[p][2] += cg[2] * f1;
          acc[p][3] += cg[3] * f1;
        }
      }
    }
#pragma unroll
    for (int p = 0; p < MAXP; ++p) {
      F[p][0] = fmaf(d0, (float)acc[p][0], F[p][0]);
      F[p][1] = fmaf(d0, (float)acc[p][1], F[p][1]);
      F[p][2] = fmaf(d1, (float)acc[p][2], F[p][2]);
      F[p][3] = fmaf(d1, (float)acc[p][3], F[p][3]);
    }
  }
}

// Q8_0: 34-byte block at row offset `o`; the 8 int8 values of sub-range c.
__device__ __forceinline__ void q80_vals(const uint8_t *row, int o, int c, uint32_t &lo, uint32_t &hi) {
  const uint8_t *p = row + o + 2 + 8 * c;
  if (((o + 2) & 3) == 0) {
    lo = lds_u32(p);
    hi = lds_u32(p + 4);
  } else {  // two bytes past a multiple of 4
    const uint32_t u0 = lds_u32(p - 2), u1 = lds_u32(p + 2), u2 = lds_u32(p + 6);
    lo = __byte_perm(u0, u1, 0x5432);
    hi = __byte_perm(u1, u2, 0x5432);
  }
}

template <int NB, int MAXP, typename BCol>
__device__ __forceinline__ void q80_chunk(const uint8_t *st, int k0, const BCol (&bcol)[MAXP], int npairs,
                                          float (&F)[MAXP][4]) {
  constexpr int RS = (NB * 34 + 15) / 16 * 16;
  const int lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
  const uint8_t *row0 = st + r * RS;
  const uint8_t *row1 = row0 + 8 * RS;
  // one token pair: the B fragments of the whole chunk are loaded first (from
  // global memory they are the long-latency loads of this loop); more pairs
  // load them next to their MMAs (registers)
  constexpr bool kPre = MAXP == 1;
  uint2 B[kPre ? NB : 1][MAXP];
  if (kPre) {
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int p = 0; p < MAXP; ++p) B[kPre ? b : 0][p] = (MAXP == 1 || p < npairs) ? ldb(bcol[p], k0 + 32 * b) : make_uint2(0u, 0u);
  }
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const int o = 34 * b;
    const float d0 = half_bits_to_float(lds_u16(row0 + o));
    const float d1 = half_bits_to_float(lds_u16(row1 + o));
    uint32_t A[4];
    q80_vals(row0, o, c, A[0], A[2]);
    q80_vals(row1, o, c, A[1], A[3]);
#pragma unroll
    for (int p = 0; p < MAXP; ++p) {
      if (MAXP == 1 || p < npairs) {
        const uint2 bb = kPre ? B[kPre ? b : 0][p] : ldb(bcol[p], k0 + 32 * b);
        const int zero[4] = {0, 0, 0, 0};
        int cg[4];
        mma_s8(cg, A, bb.x, bb.y, zero);
        F[p][0] = fmaf(d0, (float)cg[0], F[p][0]);
        F[p][1] = fmaf(d0, (float)cg[1], F[p][1]);
        F[p][2] = fmaf(d1, (float)cg[2], F[p][2]);
        F[p][3] = fmaf(d1, (float)cg[3], F[p][3]);
      }
    }
  }
}

// 8 bytes at a 4-byte aligned shared address: one 8-byte load when `al8`
// (a compile-time constant at every call site), else two 4-byte loads.
__device__ __forceinline__ uint2 lds_u64_al4(const uint8_t *p, bool al8) {
  if (al8) return *reinterpret_cast<const uint2 *>(p);
  return make_uint2(lds_u32(p), lds_u32(p + 4));
}

// Q2_K: value = d*sc*q - dmin*m.  Main term: A = q*sc (exact int8) against
// the limbs of h.  Min term: A = m (per 16-element sub-block) against the
// limbs of the 16-element sums of h.
template <int NB, int MAXP, typename BCol>
__device__ __forceinline__ void q2k_chunk(const uint8_t *st, int k0, const BCol (&bcol)[MAXP],
                                          const BCol (&xcol)[MAXP], int npairs, float (&F)[MAXP][4],
                                          float (&G)[MAXP][4]) {
  constexpr int RS = (NB * 84 + 15) / 16 * 16;
  const int lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
  const int cs = 8 * (c >> 1);  // byte of the scale word holding this lane's sub-block, within a pair
  const uint8_t *row0 = st + r * RS;
  const uint8_t *row1 = row0 + 8 * RS;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const uint8_t *p0 = row0 + 84 * b;
    const uint8_t *p1 = row1 + 84 * b;
    const uint32_t dd0 = lds_u32(p0 + 80), dd1 = lds_u32(p1 + 80);
    const float d0 = half_bits_to_float((uint16_t)(dd0 & 0xFFFFu)), m0 = half_bits_to_float((uint16_t)(dd0 >> 16));
    const float d1 = half_bits_to_float((uint16_t)(dd1 & 0xFFFFu)), m1 = half_bits_to_float((uint16_t)(dd1 >> 16));
    int Cm[MAXP][4];
#pragma unroll
    for (int p = 0; p < MAXP; ++p) Cm[p][0] = Cm[p][1] = Cm[p][2] = Cm[p][3] = 0;
    const int kb = (k0 >> 8) + b;  // global block index along K
    // one token pair: the B fragments of the block's 8 MMAs and its min-term
    // column are loaded first (from global memory they are the long-latency
    // loads of this loop); more pairs load them next to their MMAs
    constexpr bool kPre = MAXP == 1;
    uint2 B[kPre ? 2 : 1][kPre ? 4 : 1][MAXP];
    uint32_t BX[MAXP];
    if (kPre) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int sh = 0; sh < 4; ++sh)
#pragma unroll
          for (int p = 0; p < MAXP; ++p)
            B[kPre ? hf : 0][kPre ? sh : 0][p] =
                (MAXP == 1 || p < npairs) ? ldb(bcol[p], k0 + 256 * b + 128 * hf + 32 * sh) : make_uint2(0u, 0u);
#pragma unroll
      for (int p = 0; p < MAXP; ++p) BX[p] = (MAXP == 1 || p < npairs) ? ldx(xcol[p], kb * 16) : 0u;  // base includes 4c
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      // a block at an odd position of the staged row starts 4 (not 8) bytes aligned
      const bool al8 = ((84 * b) & 7) == 0;
      const uint2 q0 = lds_u64_al4(p0 + 16 + 32 * hf + 8 * c, al8);
      const uint2 q1 = lds_u64_al4(p1 + 16 + 32 * hf + 8 * c, al8);
      const uint2 s0 = lds_u64_al4(p0 + 8 * hf, al8);
      const uint2 s1 = lds_u64_al4(p1 + 8 * hf, al8);
#pragma unroll
      for (int sh = 0; sh < 4; ++sh) {
        const int bsh = 16 * (sh & 1) + cs;
        const uint32_t sc0 = ((sh < 2 ? s0.x : s0.y) >> bsh) & 15u;
        const uint32_t sc1 = ((sh < 2 ? s1.x : s1.y) >> bsh) & 15u;
        uint32_t A[4];
        A[0] = ((q0.x >> (2 * sh)) & 0x03030303u) * sc0;
        A[2] = ((q0.y >> (2 * sh)) & 0x03030303u) * sc0;
        A[1] = ((q1.x >> (2 * sh)) & 0x03030303u) * sc1;
        A[3] = ((q1.y >> (2 * sh)) & 0x03030303u) * sc1;
#pragma unroll
        for (int p = 0; p < MAXP; ++p) {
          if (MAXP == 1 || p < npairs) {
            const uint2 bb = kPre ? B[kPre ? hf : 0][kPre ? sh : 0][p] : ldb(bcol[p], k0 + 256 * b + 128 * hf + 32 * sh);
            mma_s8(Cm[p], A, bb.x, bb.y, Cm[p]);
          }
        }
      }
    }
    // min term over the 16 sub-blocks: thread c covers sub-blocks 4c..4c+3
    uint32_t Am[4];
    Am[0] = (lds_u32(p0 + 4 * c) >> 4) & 0x0F0F0F0Fu;
    Am[1] = (lds_u32(p1 + 4 * c) >> 4) & 0x0F0F0F0Fu;
    Am[2] = 0u;
    Am[3] = 0u;
#pragma unroll
    for (int p = 0; p < MAXP; ++p) {
      if (MAXP == 1 || p < npairs) {
        const uint32_t bx = kPre ? BX[p] : ldx(xcol[p], kb * 16);  // base includes 4c
        const int zero[4] = {0, 0, 0, 0};
        int cn[4];
        mma_s8(cn, Am, bx, 0u, zero);
        F[p][0] = fmaf(d0, (float)Cm[p][0], F[p][0]);
        F[p][1] = fmaf(d0, (float)Cm[p][1], F[p][1]);
        F[p][2] = fmaf(d1, (float)Cm[p][2], F[p][2]);
        F[p][3] = fmaf(d1, (float)Cm[p][3], F[p][3]);
        G[p][0] = fmaf(m0, (float)cn[0], G[p][0]);
        G[p][1] = fmaf(m0, (float)cn[1], G[p][1]);
        G[p][2] = fmaf(m1, (float)cn[2], G[p][2]);
        G[p][3] = fmaf(m1, (float)cn[3], G[p][3]);
      }
    }
  }
}

// Sum of the limb columns: thread (r, c) holds columns 2c, 2c+1 = limbs
// 2(c&1), 2(c&1)+1 of token slot c>>1 of the pair.  Returns the row-r and
// row-(r+8) values of that token (identical in lanes c and c^1).
__device__ __forceinline__ void combine_limbs(const float (&F)[4], const float *scale, float &v0, float &v1) {
  const int c = threadIdx.x & 3;
  const int l0 = 2 * (c & 1);
  const float s0 = scale ? scale[l0] : 0.f;
  const float s1 = (scale && l0 + 1 < 3) ? scale[l0 + 1] : 0.f;
  v0 = s0 * F[0] + s1 * F[1];
  v1 = s0 * F[2] + s1 * F[3];
  v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
  v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
}

// Three-limb int8 quantisation of n floats with scale max/127 (n a multiple
// of 4; src 16-byte and dst 4-byte aligned).  Every lane takes 4 consecutive
// elements per step and a batch of steps is loaded before any is used, so
// the warp waits for memory once per batch rather than once per element.
__device__ void quantise_vector(const float *src, int n, float vmax, int8_t *dst, int dstride, float *scales) {
  const int lane = threadIdx.x & 31;
  const float s1 = vmax > 0.f ? vmax / 127.f : 1.f;
  const float s2 = s1 / 254.f, s3 = s2 / 254.f;
  const float r1 = 1.f / s1, r2 = 1.f / s2, r3 = 1.f / s3;
  constexpr int kBatch = 8;
  for (int base = 0; base < n; base += 4 * 32 * kBatch) {
    float4 v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int j = base + 4 * (lane + 32 * i);
      v[i] = j < n ? __ldcg(reinterpret_cast<const float4 *>(src + j)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int j = base + 4 * (lane + 32 * i);
      if (j < n) {
        const float e[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        uint32_t w1 = 0u, w2 = 0u, w3 = 0u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float q1 = fminf(fmaxf(rintf(e[q] * r1), -127.f), 127.f);
          const float e1 = fmaf(-q1, s1, e[q]);
          const float q2 = fminf(fmaxf(rintf(e1 * r2), -127.f), 127.f);
          const float e2 = fmaf(-q2, s2, e1);
          const float q3 = fminf(fmaxf(rintf(e2 * r3), -127.f), 127.f);
          w1 |= ((uint32_t)(int)q1 & 255u) << (8 * q);
          w2 |= ((uint32_t)(int)q2 & 255u) << (8 * q);
          w3 |= ((uint32_t)(int)q3 & 255u) << (8 * q);
        }
        *reinterpret_cast<uint32_t *>(dst + j) = w1;
        *reinterpret_cast<uint32_t *>(dst + dstride + j) = w2;
        *reinterpret_cast<uint32_t *>(dst + 2 * dstride + j) = w3;
      }
    }
  }
  if (lane == 0) {
    scales[0] = s1;
    scales[1] = s2;
    scales[2] = s3;
    scales[3] = 0.f;
  }
}

// Shared-memory tables of k2: +/- codebook and byte-permute selectors.
__device__ void build_tables(const uint8_t *grid, uint8_t *gpm, uint8_t *selt, int *err, int tid, int nthreads) {
  for (int ix = tid; ix < 256; ix += nthreads) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(grid + 8 * ix);
    if ((raw.x | raw.y) & 0x80808080u) set_error(err, kErrGrid);
    // negate each byte: (0x80 - b) ^ 0x80 computed per byte without carries
    const uint32_t n0 = __vsub4(0u, raw.x), n1 = __vsub4(0u, raw.y);
    const uint4 e = make_uint4(raw.x, n0, raw.y, n1);
#pragma unroll
    for (int rep = 0; rep < 8; ++rep) *reinterpret_cast<uint4 *>(gpm + ix * 128 + rep * 16) = e;
  }
  for (int m7 = tid; m7 < 128; m7 += nthreads) {
    const uint32_t m8 = (uint32_t)m7 | ((uint32_t)(__popc(m7) & 1) << 7);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      lo |= (uint32_t)(l + 4 * ((m8 >> l) & 1u)) << (4 * l);
      hi |= (uint32_t)(l + 4 * ((m8 >> (l + 4)) & 1u)) << (4 * l);
    }
    const uint2 e = make_uint2(lo, hi);
#pragma unroll
    for (int rep = 0; rep < 16; ++rep) *reinterpret_cast<uint2 *>(selt + m7 * 128 + rep * 8) = e;
  }
}


// ------------------------------------------------------------------ k2

// Counter increment that publishes this warp's earlier writes (release) and,
// for the warp that sees the final count, makes the other warps' writes
// visible (acquire).  Call from one lane after __syncwarp().
__device__ __forceinline__ int atomic_add_acq_rel(int *p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;\n" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void store_release(int *p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}

struct K2Shared {
  int32_t idx[kDecodeMaxT * kMaxK];
  float w[kDecodeMaxT * kMaxK];
  Jobs J;
  int jobs_ready;  // set once the routing warps have published idx, w and J
  int limbs_ready;  // set once the x limbs made in this block are in xsm
  float hsm[kWarps2][kUnitMaxTok][16];
  uint64_t mbar[kWarps2][2];  // TMA completion of each warp's two stages
  float xs[kDecodeMaxT * 4];  // limb scales of x (when its limbs are made here)
  double red[kWarps2];
  float redf[kWarps2];
};

// Writes the 16 x ntok SwiGLU outputs held in hs (token slot, row) for the
// vectors vec[slot] (rows r0.. of h), updates the slice maxima, the 16-row
// sums and the slice's tile counter; the warp that completes a slice
// (slice_len / 16 tiles) quantises it into limbs and then sets its ready flag.
__device__ void finish_h_tile(const DecodeArgs &a, const float (*hs)[16], int ntok, const int *vec, int r0,
                              int slice_len) {
  const int lane = threadIdx.x & 31;
  const DecodeScratch &s = a.s;
  const int sl = r0 / slice_len;
  const int Im16 = s.Imax / 16;
  for (int base = 0; base < ntok; base += 2) {
    const int slot = base + (lane >> 4), row = lane & 15;
    const bool ok = slot < ntok;
    const float h = ok ? hs[slot][row] : 0.f;
    float m = fabsf(h), sum = h;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
    if (ok) {
      const int v = vec[slot];
      s.hbuf[(size_t)v * s.Imax + r0 + row] = h;
      if (row == 0) {
        s.Xbuf[(size_t)v * Im16 + r0 / 16] = sum;
        atomicMax(s.hmax + v * s.NSL + sl, __float_as_uint(m));
        atomicMax(s.Xmax + v * s.NSL + sl, __float_as_uint(fabsf(sum)));
      }
    }
  }
  __syncwarp();
  for (int slot = 0; slot < ntok; ++slot) {
    const int v = vec[slot];
    const int vs = v * s.NSL + sl;
    int last = 0;
    if (lane == 0) last = atomic_add_acq_rel(s.scount + vs, 1) == slice_len / 16 - 1;
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      __syncwarp();
      const float hm = __uint_as_float(__ldcg(s.hmax + vs));
      const float xm = __uint_as_float(__ldcg(s.Xmax + vs));
      const int k0 = sl * slice_len;
      quantise_vector(s.hbuf + (size_t)v * s.Imax + k0, slice_len, hm, s.hq + (size_t)v * 3 * s.Imax + k0, s.Imax,
                      s.hsc + 4 * vs);
      quantise_vector(s.Xbuf + (size_t)v * Im16 + k0 / 16, slice_len / 16, xm,
                      s.Xq + (size_t)v * 3 * Im16 + k0 / 16, Im16, s.Xsc + 4 * vs);
      __syncwarp();
      if (lane == 0) store_release(s.ready + vs, 1);
    }
  }
}

// Each lane with a flag waits (bounded) until it is set; the warp then reads
// what the flag's writer published.  A flag that is never set records the
// timeout error and lets the warp go on.
__device__ void wait_slice(const int *flag, int *err, long long limit) {
  if (flag) {
    const long long t0 = clock64();
    while (true) {
      int v;
      asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(flag) : "memory");
      if (v) break;
      if (clock64() - t0 > limit) {
        set_error(err, kErrTimeout);
        break;
      }
      __nanosleep(256);
    }
  }
  __syncwarp();
}

// The expert kernel: every unit of the layer's expert work, gate/up and
// down, on one unit counter.
//   units [0, n_sh)            shared gate/up (16-row tile of Is, K part of H)
//   units [n_sh, n2)           routed gate/up (job, tile of I, K part of H)
//   units [n2, n2 + n3s)       shared down (K part q of Is, 16-row tile of H)
//   units [n2 + n3s, n_units)  routed down (job, K part of I, 16-row tile of H)
// A down unit waits for the h slices it reads; every gate/up unit has been
// claimed by a running warp before the first down unit is claimed, so the
// waits end.  XSMEM: the x limbs of all tokens are staged in shared memory
// (rows of H + 32 bytes, which spreads the B-fragment loads over all banks).
template <int MAXP, bool XSMEM, bool TMA>
__global__ void __launch_bounds__(k2_threads(MAXP), 1) k2_experts(const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const LayerDims &d = a.d;
  const DecodeScratch &s = a.s;
  const int T = a.T;
  uint8_t *gpm = smem;
  uint8_t *selt = gpm + kGpmBytes;
  uint8_t *stages = selt + kSelBytes;
  K2Shared &S = *reinterpret_cast<K2Shared *>(stages + 2 * kWarps2 * kStage2);
  int8_t *xsm = reinterpret_cast<int8_t *>(reinterpret_cast<uint8_t *>(&S) + align_up(sizeof(K2Shared), 128));
  const int XS = d.H + 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (tid == 0) {
    S.jobs_ready = 0;
    S.limbs_ready = 0;
  }
  __syncthreads();
  if (TMA && lane == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(&S.mbar[warp][0])) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(&S.mbar[warp][1])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  const int nw = (int)(blockDim.x >> 5);
  if (XSMEM) {
    // the warps that make the x limbs also build the tables (below), on their
    // own named barrier, and publish both with limbs_ready
    __syncthreads();  // the mbarriers are initialised
  } else {
    build_tables(a.wt.grid, gpm, selt, a.err, tid, (int)blockDim.x);
    __syncthreads();  // tables in place for every warp
  }
  constexpr int kUW = 2 * MAXP;  // tokens per unit: 2 per MMA column pair
  if (XSMEM && warp >= T) {
    // The decoding tables and the x limbs of the T tokens are made here (the
    // limbs from x itself, as k1 makes them) by the warps that do not copy
    // the routing, on a named barrier of their own, so the shared expert's
    // gate/up units can run before the routing is known: nothing before the
    // first counter update below reads the earlier kernels' results.
    const int ltid = tid - 32 * T, lthreads = (nw - T) * 32;
    build_tables(a.wt.grid, gpm, selt, a.err, ltid, lthreads);
    const int n4 = d.H / 4;
    for (int t = 0; t < T; ++t) {
      const float4 *xt = reinterpret_cast<const float4 *>(a.x + (size_t)t * d.H);
      double ss = 0.0;
      float amax = 0.f;
      for (int j = ltid; j < n4; j += lthreads) {
        const float4 v = xt[j];
        ss += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
        amax = fmaxf(fmaxf(fmaxf(amax, fabsf(v.x)), fmaxf(fabsf(v.y), fabsf(v.z))), fabsf(v.w));
      }
      ss = warp_sum_d(ss);
      amax = warp_max(amax);
      if (lane == 0) {
        S.red[warp] = ss;
        S.redf[warp] = amax;
      }
      asm volatile("bar.sync 2, %0;\n" ::"r"(lthreads) : "memory");
      ss = 0.0;
      amax = 0.f;
      for (int w = T; w < nw; ++w) {
        ss += S.red[w];
        amax = fmaxf(amax, S.redf[w]);
      }
      float inv = 1.f;
      if (d.flags & MOE_FLAG_PRENORM_RESIDUAL) {
        inv = (float)(1.0 / sqrt(ss / (double)d.H + (double)d.eps));
        amax = amax * inv;
      }
      const float s1 = amax > 0.f ? amax / 127.f : 1.f;
      const float s2 = s1 / 254.f, s3 = s2 / 254.f;
      const float r1 = 1.f / s1, r2 = 1.f / s2, r3 = 1.f / s3;
      for (int j = ltid; j < n4; j += lthreads) {
        const float4 v = xt[j];
        const float e[4] = {v.x, v.y, v.z, v.w};
        uint32_t w1 = 0u, w2 = 0u, w3 = 0u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float xv = e[q] * inv;
          const float q1 = fminf(fmaxf(rintf(xv * r1), -127.f), 127.f);
          const float e1 = fmaf(-q1, s1, xv);
          const float q2 = fminf(fmaxf(rintf(e1 * r2), -127.f), 127.f);
          const float e2 = fmaf(-q2, s2, e1);
          const float q3 = fminf(fmaxf(rintf(e2 * r3), -127.f), 127.f);
          w1 |= ((uint32_t)(int)q1 & 255u) << (8 * q);
          w2 |= ((uint32_t)(int)q2 & 255u) << (8 * q);
          w3 |= ((uint32_t)(int)q3 & 255u) << (8 * q);
        }
        *reinterpret_cast<uint32_t *>(xsm + (size_t)(t * 3 + 0) * XS + 4 * j) = w1;
        *reinterpret_cast<uint32_t *>(xsm + (size_t)(t * 3 + 1) * XS + 4 * j) = w2;
        *reinterpret_cast<uint32_t *>(xsm + (size_t)(t * 3 + 2) * XS + 4 * j) = w3;
      }
      if (ltid == 0) {
        S.xs[4 * t] = s1;
        S.xs[4 * t + 1] = s2;
        S.xs[4 * t + 2] = s3;
        S.xs[4 * t + 3] = 0.f;
      }
      asm volatile("bar.sync 2, %0;\n" ::"r"(lthreads) : "memory");
    }
    if (ltid == 0) {
      __threadfence_block();
      *reinterpret_cast<volatile int *>(&S.limbs_ready) = 1;
    }
  } else if (!XSMEM) {
    pdl_wait();  // k1's limbs and keys are visible from here on
    __syncthreads();
  }
  // Warps 0..T-1 route one token each and warp 0 builds the job table; the
  // other warps start on the shared expert's gate/up units, which need no
  // routing, and wait for the table only when they claim a routed unit.
  // (Routing in every CTA beats one routing block followed by copies: the
  // copies would wait for that block's whole kernel to finish.)
  const int nr = T < nw ? T : nw;  // routing warps
  if (warp < nr) {
    pdl_wait();  // the router's keys
    for (int t = warp; t < T; t += nr) warp_route_token(a, t, S.idx + t * d.k, S.w + t * d.k);
    asm volatile("bar.sync 1, %0;\n" ::"r"(32 * nr) : "memory");
    if (warp == 0) {
      warp_build_jobs(S.idx, T, d.k, kUW, S.J);
      if (blockIdx.x == 0)
        for (int i = lane; i < T * d.k; i += 32) {
          s.idx[i] = S.idx[i];
          s.w[i] = S.w[i];
        }
      __threadfence_block();
      if (lane == 0) *reinterpret_cast<volatile int *>(&S.jobs_ready) = 1;
    }
  }

  const uint8_t *gpm_l = gpm + (lane & 7) * 16;
  const uint8_t *sel_l = selt + (lane & 15) * 8;
  uint8_t *st0 = stages + warp * 2 * kStage2;
  uint8_t *st1 = st0 + kStage2;
  const int r = lane >> 2, c = lane & 3;
  using BCol = typename std::conditional<XSMEM, BColS, BColG>::type;
  // column of limb `limb` of token t, offset by this lane's 8-element sub-range
  auto xcol = [&](int t, int limb) -> const int8_t * {
    return (XSMEM ? xsm + (size_t)(t * 3 + limb) * XS : s.xq + ((size_t)t * 3 + limb) * d.H) + 8 * c;
  };
  // limb `limb` of vector v of h (and of its 16-element sums), offset likewise
  auto hcol = [&](int v, int limb) -> const int8_t * { return s.hq + ((size_t)v * 3 + limb) * s.Imax + 8 * c; };
  auto Xcol = [&](int v, int limb) -> const int8_t * {
    return s.Xq + ((size_t)v * 3 + limb) * (s.Imax / 16) + 4 * c;
  };

  // ---- gate/up geometry
  const int tilesI = d.I / 16, tilesS = d.Is / 16;
  const int PH = s.PH;
  const int kpart = d.H / PH;  // K elements of a gate/up unit
  const int cbI = kpart / 256;  // IQ2_XXS blocks per unit (4, 2 or 1): one chunk per matrix
  const int nq8 = kpart / 256;  // Q8_0 chunks of 8 blocks per unit and matrix
  const size_t rbI = (size_t)(d.H / 256) * 66;
  const size_t rbQ = (size_t)(d.H / 32) * 34;
  const int V = T * d.k + T;
  // ---- down geometry
  const int tilesH = d.H / 16;
  const int PD = s.PD, PS = s.PS;
  const int kpd = d.I / PD;           // K elements of a routed down unit (one slice)
  const int cbD = kpd / 256;          // Q2_K blocks per routed down unit
  const int nbD = cbD < 2 ? cbD : 2;  // Q2_K blocks per chunk (rows of <= 168 bytes)
  const int kps = d.Is / PS;          // K elements of a shared down unit (one slice)
  const int nqd = kps / 256;          // Q8_0 chunks of 8 blocks per shared down unit
  const size_t rbD = (size_t)(d.I / 256) * 84;
  const size_t rbQd = (size_t)(d.Is / 32) * 34;
  const int NS = s.NS;
  // ---- unit ranges; the ones past the shared gate/up units depend on the
  // number of jobs and are set once the job table is ready
  const int n_sh = s.G * tilesS * PH;
  const int n3s = s.G * PS * tilesH;
  int nparts = 0, n2 = 0, n_units = -1;  // parts of an output tile, unit ranges
  auto valid = [&](int u) {
    if (u < n_sh) return true;
    if (n_units < 0) {
      const long long t0 = clock64();
      bool ok = true;
      while (*reinterpret_cast<volatile int *>(&S.jobs_ready) == 0) {
        if (clock64() - t0 > d.wait_cycles) {
          set_error(a.err, kErrTimeout);
          ok = false;
          break;
        }
        __nanosleep(256);
      }
      __syncwarp();
      __threadfence_block();
      if (!ok) return false;
      nparts = S.J.n * PD + s.G * PS;
      n2 = n_sh + S.J.n * tilesI * PH;
      n_units = n2 + n3s + S.J.n * PD * tilesH;
    }
    return u < n_units;
  };

  struct Unit {
    int kind;  // 0 shared gate/up, 1 routed gate/up, 2 shared down, 3 routed down
    int j, e, tile, part, ntok, per, nch;  // gate/up: 16-row tile, K part of H, chunks per matrix
    int ot, kp;                            // down: output tile, K part (slice) of I or Is
    int t0;                                // shared: first token of the unit's token group
    const int *pairs;
  };
  // the shared expert's tokens in groups of kUW: group g holds tokens
  // kUW * g ..; its units are numbered like one group's, group-major
  const int shG = s.G;
  const int nshg = tilesS * PH, n3sg = PS * tilesH;  // units of one group
  auto shared_group = [&](int w, int per_group, int &rem) {
    const int g = shG == 1 ? 0 : w / per_group;
    rem = w - g * per_group;
    return g;
  };
  auto unit_at = [&](int u) {
    Unit x;
    x.j = x.e = x.tile = x.part = x.ot = x.kp = x.t0 = 0;
    x.per = 1;
    x.pairs = nullptr;
    x.ntok = T;
    if (u < n_sh) {
      x.kind = 0;
      int rem;
      const int g = shared_group(u, nshg, rem);
      x.t0 = kUW * g;
      x.ntok = min(kUW, T - x.t0);
      x.tile = s.fPH.div(rem);
      x.part = rem - x.tile * PH;
      x.per = nq8;
      x.nch = 2 * nq8;
    } else if (u < n2) {
      x.kind = 1;
      const int uu = u - n_sh;
      x.j = s.fTIPH.div(uu);
      const int rem = uu - x.j * tilesI * PH;
      x.tile = s.fPH.div(rem);
      x.part = rem - x.tile * PH;
      x.nch = 2;
    } else if (u < n2 + n3s) {
      x.kind = 2;
      int w;
      const int g = shared_group(u - n2, n3sg, w);
      x.t0 = kUW * g;
      x.ntok = min(kUW, T - x.t0);
      x.kp = s.fTH.div(w);
      x.ot = w - x.kp * tilesH;
      x.nch = nqd;
    } else {
      x.kind = 3;
      const int w = u - n2 - n3s;
      const int jp = s.fTH.div(w);
      x.ot = w - jp * tilesH;
      x.j = s.fPD.div(jp);
      x.kp = jp - x.j * PD;
      x.nch = cbD / nbD;
    }
    if (x.kind & 1) {
      x.e = S.J.e[x.j];
      x.ntok = S.J.cnt[x.j];
      x.pairs = S.J.pair + S.J.first[x.j];
    }
    return x;
  };
  // token slot ts of a unit -> row of x / vector of h
  auto xrow = [&](const Unit &x, int ts) { return (x.kind & 1) ? x.pairs[ts] / d.k : x.t0 + ts; };
  auto hvec = [&](const Unit &x, int ts) { return (x.kind & 1) ? x.pairs[ts] : T * d.k + x.t0 + ts; };
  auto chunk_of = [&](const Unit &su, int cs) {
    Chunk ch;
    size_t off;  // byte offset of the chunk within its row
    int row;     // first row of the chunk in its tensor
    if (su.kind == 0) {
      const bool up = cs >= su.per;
      const int ck = up ? cs - su.per : cs;
      off = (size_t)(su.part * kpart / 32 + ck * 8) * 34;
      row = su.tile * 16;
      ch.g = (up ? a.wt.sh_up : a.wt.sh_gate) + (size_t)row * rbQ + off;
      ch.gstride = rbQ;
      ch.bpr = 8 * 34;
      ch.nb = 8;
      ch.k0 = su.part * kpart + ck * 256;
      ch.align = 4;
      ch.tm = up ? kTmShUp : kTmShGate;
    } else if (su.kind == 1) {
      off = (size_t)su.part * cbI * 66;
      row = su.e * d.I + su.tile * 16;
      ch.g = (cs ? a.wt.up : a.wt.gate) + (size_t)row * rbI + off;
      ch.gstride = rbI;
      ch.bpr = cbI * 66;
      ch.nb = cbI;
      ch.k0 = su.part * kpart;
      ch.align = 4;
      ch.tm = cs ? kTmUp : kTmGate;
    } else if (su.kind == 2) {
      off = (size_t)(su.kp * kps / 32 + cs * 8) * 34;
      row = su.ot * 16;
      ch.g = a.wt.sh_down + (size_t)row * rbQd + off;
      ch.gstride = rbQd;
      ch.bpr = 8 * 34;
      ch.nb = 8;
      ch.k0 = su.kp * kps + cs * 256;
      ch.align = 4;
      ch.tm = kTmShDown;
    } else {
      off = (size_t)(su.kp * cbD + cs * nbD) * 84;
      row = su.e * d.H + su.ot * 16;
      ch.g = a.wt.down + (size_t)row * rbD + off;
      ch.gstride = rbD;
      ch.bpr = nbD * 84;
      ch.nb = nbD;
      ch.k0 = su.kp * kpd + cs * nbD * 256;
      ch.align = 8;
      ch.tm = kTmDown;
    }
    ch.piece = piece_for(ch.gstride, reinterpret_cast<uintptr_t>(ch.g) & 15, ch.bpr);
    ch.tx = (int)((off & ~(size_t)15) / 2);
    ch.ty = row;
    ch.tshift = (int)(off & 15);
    return ch;
  };

  int seg_parts = 0, npairs = 0;
  BCol bcol[MAXP];
  BColG hb[MAXP], xb[MAXP];
  float F[MAXP][4] = {}, G[MAXP][4] = {};
  // gate/up: each matrix's sums of a unit are combined over limbs and stored as
  // the partials of the unit's K part (m = 0 gate, 1 up)
  auto store_part = [&](const Unit &cu, int m) {
#pragma unroll
    for (int p = 0; p < MAXP; ++p) {
      if (MAXP == 1 || p < npairs) {
        const int ts = 2 * p + (c >> 1);
        float v0, v1;
        combine_limbs(F[p], ts < cu.ntok ? (XSMEM ? S.xs : s.xs) + 4 * xrow(cu, ts) : nullptr, v0, v1);
        if ((c & 1) == 0 && ts < cu.ntok) {
          float *pp = s.gpart + ((size_t)(m * PH + cu.part) * V + hvec(cu, ts)) * s.Imax + cu.tile * 16;
          pp[r] = v0;
          pp[r + 8] = v1;
        }
      }
      F[p][0] = F[p][1] = F[p][2] = F[p][3] = 0.f;
    }
  };
  // gate/up: count the segment's parts in; the warp that completes the tile
  // sums the parts in order, applies the SwiGLU and hands the tile on
  auto end_gateup = [&](const Unit &cu) {
    pdl_wait();  // the counters are reset by k1
    __syncwarp();
    const int set = cu.kind == 0 ? cu.t0 / kUW : s.G + cu.j;
    int last = 0;
    if (lane == 0) last = atomic_add_acq_rel(s.hcount + set * s.TM + cu.tile, seg_parts) + seg_parts == PH;
    last = __shfl_sync(0xffffffffu, last, 0);
    seg_parts = 0;
    if (!last) return;
    __syncwarp();
    const int r0 = cu.tile * 16;
    for (int i = lane; i < 16 * cu.ntok; i += 32) {
      const int ts = i >> 4, row = i & 15;
      const int v = hvec(cu, ts);
      float ga = 0.f, ub = 0.f;
      for (int p0 = 0; p0 < PH; p0 += 4) {  // loads of a batch are independent; sums keep part order
        float gb[4], ubb[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const bool in = p0 + q < PH;
          gb[q] = in ? __ldcg(s.gpart + ((size_t)(0 * PH + p0 + q) * V + v) * s.Imax + r0 + row) : 0.f;
          ubb[q] = in ? __ldcg(s.gpart + ((size_t)(1 * PH + p0 + q) * V + v) * s.Imax + r0 + row) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          ga += gb[q];
          ub += ubb[q];
        }
      }
      S.hsm[warp][ts][row] = silu(ga) * ub;
    }
    __syncwarp();
    int vec[kUnitMaxTok];
#pragma unroll
    for (int t = 0; t < kUnitMaxTok; ++t) vec[t] = t < cu.ntok ? hvec(cu, t) : 0;
    finish_h_tile(a, S.hsm[warp], cu.ntok, vec, r0, cu.kind == 0 ? kps : kpd);
  };
  // down: the part is in its slot; the warp that completes the output tile
  // sums its slots in a fixed order into y
  auto end_down = [&](const Unit &cu) {
    __syncwarp();
    int last = 0;
    if (lane == 0) last = atomic_add_acq_rel(s.ycount + cu.ot, 1) == nparts - 1;
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    __syncwarp();
    const int r0 = cu.ot * 16;
    const float *ytile = s.ypart + (size_t)cu.ot * NS * 16;
    for (int i = lane; i < 16 * T; i += 32) {
      const int t = i >> 4, row = i & 15;
      float acc = (d.flags & MOE_FLAG_PRENORM_RESIDUAL) ? a.x[(size_t)t * d.H + r0 + row] : 0.f;
      // slots in a fixed order: the token's routed parts, then its shared parts;
      // the loads of a batch are independent
      const int nr = d.k * PD, ns = nr + PS;
      for (int s0 = 0; s0 < ns; s0 += 8) {
        float vb[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int sl = s0 + q;
          const size_t slot = sl < nr ? (size_t)t * nr + sl : (size_t)T * nr + (size_t)t * PS + (sl - nr);
          vb[q] = sl < ns ? __ldcg(ytile + slot * 16 + row) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) acc += vb[q];
      }
      a.y[(size_t)t * d.H + r0 + row] = acc;
    }
  };

  if (XSMEM && warp < T) {
    // the routing warps compute units only once the limbs are in place
    const long long t0 = clock64();
    while (*reinterpret_cast<volatile int *>(&S.limbs_ready) == 0) {
      if (clock64() - t0 > d.wait_cycles) {
        set_error(a.err, kErrTimeout);
        break;
      }
      __nanosleep(64);
    }
    __syncwarp();
    __threadfence_block();
  }
  // Claims: with the x limbs made here, every non-routing warp first takes
  // one shared gate/up unit by its number (no counter: k1 resets the
  // counters); the remaining units come from the counter after k1 is done.
  const int gwn = (warp - T) * (int)gridDim.x + (int)blockIdx.x;
  bool first_static = XSMEM && warp >= T && gwn < n_sh;
  const int n_static = XSMEM ? min(n_sh, (nw - T) * (int)gridDim.x) : 0;
  auto claim = [&]() -> int {
    if (first_static) {
      first_static = false;
      return gwn;
    }
    pdl_wait();
    int u = 0;
    if (lane == 0) u = atomicAdd(s.work + 0, kClaim);
    return n_static + __shfl_sync(0xffffffffu, u, 0);
  };
  run_units<kClaim, kAheadClaim, TMA, Unit>(
      st0, st1, &S.mbar[warp][0], a.wt.tm, a.err, claim, valid, unit_at, chunk_of,
      [&](const Unit &cu, int u, int cc, const uint8_t *st, int next_u) {
        if (cu.kind <= 1) {
          // ------------------------------------------------ gate/up
          if (cc == 0) {
            npairs = (cu.ntok + 1) >> 1;
#pragma unroll
            for (int p = 0; p < MAXP; ++p) {
              const int ts = 2 * p + (r >> 2), limb = r & 3;
              bcol[p].ok = ts < cu.ntok && limb < 3;
              bcol[p].p = bcol[p].ok ? xcol(xrow(cu, ts), limb) : nullptr;
            }
          }
          if (cu.kind == 0) {
            q80_chunk<8, MAXP>(st, cu.part * kpart + (cc < nq8 ? cc : cc - nq8) * 256, bcol, npairs, F);
          } else if (cbI == 4) {
            iq2_chunk<4, MAXP>(st, cu.part * kpart, gpm_l, sel_l, bcol, npairs, F);
          } else if (cbI == 2) {
            iq2_chunk<2, MAXP>(st, cu.part * kpart, gpm_l, sel_l, bcol, npairs, F);
          } else {
            iq2_chunk<1, MAXP>(st, cu.part * kpart, gpm_l, sel_l, bcol, npairs, F);
          }
          if (cc == cu.per - 1) store_part(cu, 0);
          if (cc == cu.nch - 1) {
            store_part(cu, 1);
            ++seg_parts;
            if (next_u != u + 1 || s.fPH.div(u + 1) != s.fPH.div(u)) end_gateup(cu);
          }
          return;
        }
        // -------------------------------------------------- down
        if (cc == 0) {
          // the h slices this unit reads: one per token slot
          wait_slice(lane < cu.ntok ? s.ready + hvec(cu, lane) * s.NSL + cu.kp : nullptr, a.err, d.wait_cycles);
          npairs = (cu.ntok + 1) >> 1;
#pragma unroll
          for (int p = 0; p < MAXP; ++p) {
            const int ts = 2 * p + (r >> 2), limb = r & 3;
            const bool ok = ts < cu.ntok && limb < 3;
            const int v = ok ? hvec(cu, ts) : 0;
            hb[p].ok = xb[p].ok = ok;
            hb[p].p = ok ? hcol(v, limb) : nullptr;
            xb[p].p = ok ? Xcol(v, limb) : nullptr;
          }
        }
        float *ytile = s.ypart + (size_t)cu.ot * NS * 16;
        if (cu.kind == 3) {
          if (nbD == 2)
            q2k_chunk<2, MAXP>(st, cu.kp * kpd + cc * 512, hb, xb, npairs, F, G);
          else
            q2k_chunk<1, MAXP>(st, cu.kp * kpd + cc * 256, hb, xb, npairs, F, G);
          if (cc == cu.nch - 1) {
#pragma unroll
            for (int p = 0; p < MAXP; ++p) {
              if (MAXP == 1 || p < npairs) {
                const int ts = 2 * p + (c >> 1);
                const bool ok = ts < cu.ntok;
                const int v = ok ? cu.pairs[ts] : 0;
                const int l0 = 2 * (c & 1);
                float v0 = 0.f, v1 = 0.f;
                if (ok) {
                  const float *hs = s.hsc + 4 * (v * s.NSL + cu.kp);
                  const float *xs = s.Xsc + 4 * (v * s.NSL + cu.kp);
                  v0 = hs[l0] * F[p][0] - xs[l0] * G[p][0];
                  v1 = hs[l0] * F[p][2] - xs[l0] * G[p][2];
                  if (l0 + 1 < 3) {
                    v0 += hs[l0 + 1] * F[p][1] - xs[l0 + 1] * G[p][1];
                    v1 += hs[l0 + 1] * F[p][3] - xs[l0 + 1] * G[p][3];
                  }
                }
                v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
                v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
                if ((c & 1) == 0 && ok) {
                  const float wt = S.w[v];
                  float *dst = ytile + (size_t)(v * PD + cu.kp) * 16;
                  dst[r] = wt * v0;
                  dst[r + 8] = wt * v1;
                }
              }
#pragma unroll
              for (int i = 0; i < 4; ++i) F[p][i] = G[p][i] = 0.f;
            }
            end_down(cu);
          }
        } else {
          q80_chunk<8, MAXP>(st, cu.kp * kps + cc * 256, hb, npairs, F);
          if (cc == cu.nch - 1) {
#pragma unroll
            for (int p = 0; p < MAXP; ++p) {
              if (MAXP == 1 || p < npairs) {
                const int ts = 2 * p + (c >> 1);
                const float *sc = ts < cu.ntok ? s.hsc + 4 * ((T * d.k + cu.t0 + ts) * s.NSL + cu.kp) : nullptr;
                float v0, v1;
                combine_limbs(F[p], sc, v0, v1);
                if ((c & 1) == 0 && ts < cu.ntok) {
                  float *dst = ytile + (size_t)(T * d.k * PD + (cu.t0 + ts) * PS + cu.kp) * 16;
                  dst[r] = v0;
                  dst[r + 8] = v1;
                }
              }
#pragma unroll
              for (int i = 0; i < 4; ++i) F[p][i] = 0.f;
            }
            end_down(cu);
          }
        }
      });
  // the CTA's last warp, once out of units, starts this CTA's share of the
  // next layer's prefetch (set only when the layer runs in a stack)
  if (warp == nw - 1 && lane == 0) prefetch_next_layer(a.pf);
}

// ------------------------------------------------------------------ route only

__global__ void k_route_only(DecodeArgs a, int32_t *idx, float *w) {
  const int warp = threadIdx.x >> 5;
  for (int t = blockIdx.x * (blockDim.x / 32) + warp; t < a.T; t += gridDim.x * (blockDim.x / 32))
    warp_route_token(a, t, idx + (size_t)t * a.d.k, w + (size_t)t * a.d.k);
}

size_t k2_smem_bytes(const LayerDims &d, int T, bool xsmem) {
  size_t b = kGpmBytes + kSelBytes + 2 * kWarps2 * kStage2 + align_up(sizeof(K2Shared), 128);
  if (xsmem) b += (size_t)T * 3 * (d.H + 32);
  return b;
}
constexpr size_t kSmemLimit = kSmemOptInMax;

template <typename K>
cudaError_t launch_pdl(K kernel, int grid, int block, size_t smem, cudaStream_t stream, const DecodeArgs &a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

template <int MAXP, bool XSMEM, bool TMA>
cudaError_t launch_k2(const DecodeArgs &a, cudaStream_t stream, int num_sms) {
  static SmemOptIn opt;
  cudaError_t e = opt_in_smem(k2_experts<MAXP, XSMEM, TMA>, kSmemLimit, opt);
  if (e != cudaSuccess) return e;
  if (a.ev_begin) cudaEventRecord(a.ev_begin, stream);
  e = launch_pdl(k2_experts<MAXP, XSMEM, TMA>, num_sms, k2_threads(MAXP), k2_smem_bytes(a.d, a.T, XSMEM), stream,
                 a);
  if (e != cudaSuccess) return e;
  if (a.ev_end) cudaEventRecord(a.ev_end, stream);
  return cudaSuccess;
}

template <int MAXP, bool XSMEM>
cudaError_t launch_k2_tma(const DecodeArgs &a, cudaStream_t stream, int num_sms) {
  return a.wt.tma ? launch_k2<MAXP, XSMEM, true>(a, stream, num_sms) : launch_k2<MAXP, XSMEM, false>(a, stream, num_sms);
}

cudaError_t launch_k1(const DecodeArgs &a, cudaStream_t stream) {
  const int nr = a.d.mode == MOE_ROUTE_ROUTER ? (a.d.E + 1) / 2 : 0;
  const int grid = a.T + nr;
  if (a.T <= 1)
    k1_prep_router<1><<<grid, kRouterThreads, 0, stream>>>(a);
  else if (a.T <= 2)
    k1_prep_router<2><<<grid, kRouterThreads, 0, stream>>>(a);
  else if (a.T <= 4)
    k1_prep_router<4><<<grid, kRouterThreads, 0, stream>>>(a);
  else
    k1_prep_router<8><<<grid, kRouterThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

void build_chunk_tensor_maps(LayerWeights &wt, const LayerDims &d) {
  wt.tma = 0;
  const int PH = decode_kparts(d.H), PD = decode_kparts(d.I);
  const int cbI = d.H / PH / 256;       // IQ2_XXS blocks per gate/up chunk
  const int cbD = d.I / PD / 256;       // Q2_K blocks per down unit
  const int nbD = cbD < 2 ? cbD : 2;    // Q2_K blocks per down chunk
  const size_t rbI = (size_t)(d.H / 256) * 66, rbD = (size_t)(d.I / 256) * 84;
  const size_t rbQ = (size_t)(d.H / 32) * 34, rbQd = (size_t)(d.Is / 32) * 34;
  // 16-byte row strides, and chunk starts at 0 or 4/8 (IQ2_XXS) or 0/8 (Q2_K)
  // bytes past a 16-byte boundary, which the decoders' alignment allows
  if (rbI % 16 || rbD % 16 || rbQ % 16 || rbQd % 16 || cbI % 2 || nbD != 2) return;
  PFN_cuTensorMapEncodeTiled encode = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", reinterpret_cast<void **>(&encode), cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !encode)
    return;
  auto make = [&](TensorMap &m, const void *base, size_t row_bytes, size_t rows, int box_bytes) {
    const cuuint64_t dims[2] = {row_bytes / 2, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)(box_bytes / 2), 16};
    const cuuint32_t es[2] = {1, 1};
    return encode(reinterpret_cast<CUtensorMap *>(&m), CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(base),
                  dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  const int boxI = (int)align_up((size_t)cbI * 66, 16), boxD = (int)align_up((size_t)nbD * 84, 16), boxQ = 8 * 34;
  const bool ok = make(wt.tm[kTmGate], wt.gate, rbI, (size_t)d.E * d.I, boxI) &&
                  make(wt.tm[kTmUp], wt.up, rbI, (size_t)d.E * d.I, boxI) &&
                  make(wt.tm[kTmDown], wt.down, rbD, (size_t)d.E * d.H, boxD) &&
                  make(wt.tm[kTmShGate], wt.sh_gate, rbQ, (size_t)d.Is, boxQ) &&
                  make(wt.tm[kTmShUp], wt.sh_up, rbQ, (size_t)d.Is, boxQ) &&
                  make(wt.tm[kTmShDown], wt.sh_down, rbQd, (size_t)d.H, boxQ);
  wt.tma = ok ? 1 : 0;
}

// Tokens per unit of the expert kernel (2, 4 or 8: MAXP = width / 2 MMA
// column pairs).  Wider units decode a weight tile once for more tokens, but
// need more registers (12 warps per block instead of 16) and load their
// activation fragments inside the MMA loop; since nearly every expert holds
// one or two of a call's tokens, 2-token units measured fastest at every T up
// to 32 (the layer at T = 8 / 16 / 32: 0.32 / 0.60 / 1.07 ms against 0.38 /
// 0.67 / 1.16 ms with 4-token and 0.53 / 0.92 / 1.54 ms with 8-token units).
#ifndef MOE_DECODE_UNIT_TOKENS
#define MOE_DECODE_UNIT_TOKENS 2
#endif
static_assert(MOE_DECODE_UNIT_TOKENS == 2 || MOE_DECODE_UNIT_TOKENS == 4 || MOE_DECODE_UNIT_TOKENS == 8,
              "unit width");
static int decode_unit_tokens(int T) { return T <= 2 ? 2 : MOE_DECODE_UNIT_TOKENS; }

size_t decode_scratch_bytes(const LayerDims &d, int T) {
  // the largest carve of any call with up to T tokens (the unit width, and so
  // the number of shared token groups, depends on the call's T)
  size_t most = 0;
  for (int t = 1; t <= T; ++t) {
    DecodeScratch s;
    decode_carve(s, d, t, nullptr);
    const size_t b = reinterpret_cast<size_t>(s.jobs) + kJobsInts * sizeof(int) + 256;
    most = b > most ? b : most;
  }
  return most;
}

void decode_carve(DecodeScratch &s, const LayerDims &d, int T, void *base) {
  const int V = T * d.k + T;
  const int Imax = d.I > d.Is ? d.I : d.Is;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    off = align_up(off, 256);
    uint8_t *p = static_cast<uint8_t *>(base) + off;
    off += bytes;
    return p;
  };
  s.Imax = Imax;
  s.PH = decode_kparts(d.H);
  s.PD = decode_kparts(d.I);
  s.PS = decode_kparts(d.Is);
  s.Jmax = T * d.k;
  s.UW = decode_unit_tokens(T);
  s.G = (T + s.UW - 1) / s.UW;
  s.TM = Imax / 16;
  s.NS = T * d.k * s.PD + T * s.PS;
  s.NSL = s.PD > s.PS ? s.PD : s.PS;
  s.fPH.init(s.PH);
  s.fTIPH.init((d.I / 16) * s.PH);
  s.fTH.init(d.H / 16);
  s.fPD.init(s.PD);
  s.z = reinterpret_cast<double *>(take(sizeof(double) * T * d.E));
  s.sc = reinterpret_cast<double *>(take(sizeof(double) * T * d.E));
  s.idx = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * T * d.k));
  s.w = reinterpret_cast<float *>(take(sizeof(float) * T * d.k));
  s.xq = reinterpret_cast<int8_t *>(take((size_t)T * 3 * d.H));
  s.xs = reinterpret_cast<float *>(take(sizeof(float) * 4 * T));
  s.hbuf = reinterpret_cast<float *>(take(sizeof(float) * (size_t)V * Imax));
  s.hq = reinterpret_cast<int8_t *>(take((size_t)V * 3 * Imax));
  s.hsc = reinterpret_cast<float *>(take(sizeof(float) * 4 * V * s.NSL));
  s.Xbuf = reinterpret_cast<float *>(take(sizeof(float) * (size_t)V * (Imax / 16)));
  s.Xq = reinterpret_cast<int8_t *>(take((size_t)V * 3 * (Imax / 16)));
  s.Xsc = reinterpret_cast<float *>(take(sizeof(float) * 4 * V * s.NSL));
  s.hmax = reinterpret_cast<unsigned *>(take(sizeof(unsigned) * V * s.NSL));
  s.Xmax = reinterpret_cast<unsigned *>(take(sizeof(unsigned) * V * s.NSL));
  s.scount = reinterpret_cast<int *>(take(sizeof(int) * V * s.NSL));
  s.ready = reinterpret_cast<int *>(take(sizeof(int) * V * s.NSL));
  s.gpart = reinterpret_cast<float *>(take(sizeof(float) * 2 * (size_t)s.PH * V * Imax));
  s.hcount = reinterpret_cast<int *>(take(sizeof(int) * (size_t)(s.G + s.Jmax) * s.TM));
  s.ypart = reinterpret_cast<float *>(take(sizeof(float) * (size_t)(d.H / 16) * s.NS * 16));
  s.ycount = reinterpret_cast<int *>(take(sizeof(int) * (d.H / 16)));
  s.work = reinterpret_cast<int *>(take(sizeof(int) * 4));
  s.jobs = reinterpret_cast<int *>(take(sizeof(int) * kJobsInts));
}

cudaError_t decode_forward(const DecodeArgs &a, cudaStream_t stream, int num_sms) {
  cudaError_t e = launch_k1(a, stream);
  if (e != cudaSuccess) return e;
  // the variant whose unit width the scratch was carved for
  switch (a.s.UW) {
    case 2:
      if (a.T <= 2 && k2_smem_bytes(a.d, a.T, true) <= kSmemLimit) return launch_k2_tma<1, true>(a, stream, num_sms);
      return launch_k2_tma<1, false>(a, stream, num_sms);
    case 4:
      return launch_k2_tma<2, false>(a, stream, num_sms);
    case 8:
      return launch_k2_tma<4, false>(a, stream, num_sms);
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t decode_route(const DecodeArgs &a, int32_t *idx, float *w, cudaStream_t stream) {
  cudaError_t e = launch_k1(a, stream);
  if (e != cudaSuccess) return e;
  k_route_only<<<(a.T + 7) / 8, 256, 0, stream>>>(a, idx, w);
  return cudaGetLastError();
}

}  // namespace moe
