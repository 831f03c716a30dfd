// layer.cuh -- argument block and scratch layout shared by the layer's host
// code and kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

constexpr int kDecodeMaxT = 32;  // token counts handled by the GEMV (mma.sync) path
constexpr int kUnitMaxTok = 8;   // most tokens of one warp unit (4 MMA column pairs)
constexpr int kMaxK = 8;
constexpr int kMaxE = 256;

struct LayerDims {
  int H, I, Is, E, k, mode, flags, vocab;
  float scaling, eps;
  // bound, in clock cycles, of a device wait on other warps' results (an h
  // slice, the job table, a tensor-core pipeline hand-off); waits on a
  // warp's own copies keep the default
  long long wait_cycles;
  // batched path: 1 = the shared expert's weights are expanded to 16-bit
  // rows once per call and multiplied by a TMA-fed GEMM when the call has at
  // least kSharedDenseMinT tokens; 0 = its producers decode Q8_0 per tile
  int shared_dense;
};
constexpr long long kDefaultWaitCycles = 4000000000ll;  // about 2 s
#ifndef MOE_SHARED_DENSE_MIN_T
#define MOE_SHARED_DENSE_MIN_T 257
#endif
constexpr int kSharedDenseMinT = MOE_SHARED_DENSE_MIN_T;

// Opaque TMA tensor descriptor (the driver's 128-byte, 64-byte aligned
// CUtensorMap), built on the host and read by the TMA unit from the kernel's
// parameter space.
struct alignas(64) TensorMap {
  uint64_t v[16];
};

// Tensor maps of the packed weights for the small-T kernel's chunk loads:
// each matrix viewed as [rows][row_bytes / 2] 16-bit elements, box = 16 rows x
// the staged row width.  Order: gate, up, down, shared gate, shared up, shared
// down.
enum { kTmGate = 0, kTmUp, kTmDown, kTmShGate, kTmShUp, kTmShDown, kNumTm };

struct LayerWeights {
  const uint16_t *Wr;
  const float *bias;
  const int32_t *tid2eid;
  const uint8_t *gate, *up, *down, *sh_gate, *sh_up, *sh_down, *grid;
  int tma;  // 1 when tm[] is valid and every chunk start keeps the decoders' alignment
  TensorMap tm[kNumTm];
  // device copies of the batched path's tensor maps of gate, up and down
  // (128 bytes each, 64-byte aligned) for the TMA staging of its packed
  // weight tiles; nullptr: that path loads the packed bytes without TMA
  const void *gemm_tm;
};

// Builds wt.tm[] and sets wt.tma (0 when a shape does not allow TMA chunk
// loads or the driver entry point is missing); the small-T kernel then
// stages its chunks with TMA instead of cp.async.
void build_chunk_tensor_maps(LayerWeights &wt, const struct LayerDims &d);

// K parts of the decode path's warp units: every unit covers 16 weight rows
// and a K range of kDecodeKPart elements (256 where the dimension is not a
// multiple of it), so routed and shared units carry the same work.
#ifndef MOE_DECODE_KPART
#define MOE_DECODE_KPART 1024
#endif
constexpr int kDecodeKPart = MOE_DECODE_KPART;  // 1024, 512 or 256
__host__ __device__ inline int decode_kparts(int K) { return (K % kDecodeKPart == 0) ? K / kDecodeKPart : K / 256; }

// Job table of the decode path (distinct experts of a call and their
// (token, slot) pairs) as ints: n, then e, first, cnt, pair, rank_e.
constexpr int kJobsInts = 1 + 5 * kDecodeMaxT * kMaxK;

// Division by a constant d >= 1 as a multiply-high and a shift (round-up
// method): l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1; for
// 0 <= n < 2^31, n / d = (umulhi(n, m) + n) >> l.
struct FastDiv {
  uint32_t d, m, l;
  void init(uint32_t div) {
    d = div;
    l = 0;
    while ((1ull << l) < div) ++l;
    m = (uint32_t)(((1ull << 32) * ((1ull << l) - div)) / div + 1);
  }
#ifdef __CUDACC__
  __device__ __forceinline__ int div(int n) const { return (int)((__umulhi((uint32_t)n, m) + (uint32_t)n) >> l); }
#endif
};

// Scratch of the decode (GEMV) path.  V = T*k + T vectors: routed vector
// t*k + slot, shared vector T*k + t.  The SwiGLU output h of a vector is
// quantised slice by slice: a slice is the K range of one down-projection
// unit (I/PD elements for a routed vector, Is/PS for a shared one), NSL =
// max(PD, PS) slices per vector.
struct DecodeScratch {
  double *z;        // [T][E] selection keys sqrtsoftplus(z) + bias (fp64)
  double *sc;       // [T][E] scores sqrtsoftplus(z) (fp64)
  int32_t *idx;     // [T][k]
  float *w;         // [T][k]
  int8_t *xq;       // [T][3][H] int8 limbs of the expert input
  float *xs;        // [T][4] limb scales
  float *hbuf;      // [V][Imax] SwiGLU outputs
  int8_t *hq;       // [V][3][Imax] int8 limbs of h
  float *hsc;       // [V][NSL][4] limb scales per slice
  float *Xbuf;      // [V][Imax/16] sums of 16 consecutive h
  int8_t *Xq;       // [V][3][Imax/16]
  float *Xsc;       // [V][NSL][4]
  unsigned *hmax;   // [V][NSL] max |h| per slice (float bits)
  unsigned *Xmax;   // [V][NSL]
  int *scount;      // [V][NSL] finished 16-row tiles per slice
  int *ready;       // [V][NSL] 1 once the slice's limbs are written
  float *gpart;     // [2][PH][V][Imax] gate/up partial sums per K part of H
  int *hcount;      // [G + Jmax][TM] finished K parts per (vector set, 16-row tile)
  float *ypart;     // [H/16][NS][16] partial output tiles, NS = T*k*PD + T*PS slots
  int *ycount;      // [H/16]
  int *work;        // [4] unit counters
  int *jobs;        // [kJobsInts] job table (first block of the expert kernel)
  int Imax;
  int PH, PD, PS;   // K parts of H (gate/up), I (routed down), Is (shared down)
  int NSL;          // slices per vector = max(PD, PS)
  int UW;           // tokens per unit of this call's kernel variant (2 per MMA column pair)
  int Jmax;         // max routed jobs (an expert's tokens, at most UW per job) = T*k
  int G;            // token groups of the shared expert (UW tokens each)
  int TM;           // max(I, Is) / 16
  int NS;           // output slots per 16-row tile of y
  FastDiv fPH, fTIPH, fTH, fPD;  // divisors PH, (I/16)*PH, H/16, PD of the unit numbering
};

// Weights of the next layer of a stack that the expert kernel brings into
// L2 near its end (the router rows and the shared expert's gate/up rows that
// the next layer reads first); bytes are multiples of 16, pointers 16-byte
// aligned, unused entries 0.
constexpr int kPrefetchRegions = 3;
struct NextLayerPrefetch {
  const void *ptr[kPrefetchRegions];
  size_t bytes[kPrefetchRegions];
};

struct DecodeArgs {
  LayerDims d;
  LayerWeights wt;
  NextLayerPrefetch pf;
  int T;
  const float *x;
  const int32_t *token_ids;
  float *y;
  DecodeScratch s;
  int *err;
  cudaEvent_t ev_begin, ev_end;  // recorded around the expert kernel when set
};

size_t decode_scratch_bytes(const LayerDims &d, int T);
void decode_carve(DecodeScratch &s, const LayerDims &d, int T, void *base);
cudaError_t decode_forward(const DecodeArgs &a, cudaStream_t stream, int num_sms);
cudaError_t decode_route(const DecodeArgs &a, int32_t *idx, float *w, cudaStream_t stream);

}  // namespace moe
