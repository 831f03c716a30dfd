// gemm.cu -- persistent, warp-specialised grouped GEMM on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// One CTA per SM, 25 warps (26 with TMA staging):
//   warps 0-7   epilogue: tcgen05.ld of the 128-lane accumulator, SwiGLU /
//               scatter-add / store
//   warps 8-23  producers: dequantise the 128 x 64 weight tile(s) of a K step
//               into 16-bit values written straight into the 128-byte-swizzled
//               K-major operand layout, and gather the N x 64 activation tile
//               with cp.async
//   warp 24     allocates tensor memory and issues tcgen05.mma (one thread)
//   warp 25     TMA staging only: issues the tensor copies of the packed
//               weight tiles (one thread)
// Shared memory holds a ring of A stages (dequantised weight tiles, written
// in the step that hands them over), a ring of B stages (token rows,
// loaded two K steps ahead) and, with TMA staging, a ring of packed stages
// (one 256-value block of each of the tile's 128 weight rows, i.e. four K
// steps, brought by one 2-D tensor copy per matrix as soon as the stage is
// free); without it each producer keeps the packed bytes of its next K steps
// in a ring of registers.  mbarriers carry the full/empty hand-offs of every
// ring and of the accumulator between the MMA thread and the epilogue.
// Every wait is bounded: on expiry the CTA records MOE_ERR_TIMEOUT in the
// device error word, every role leaves its loop, the MMA thread drains its
// outstanding tensor-core work, the copy thread waits for its copies in
// flight, and tensor memory is freed before the kernel returns.
//
// Tiles: M = 128 weight rows, N = up to 256 columns (tokens) of one group, K
// stepped 64 at a time (four K=16 MMAs per step).  A gate/up pair shares the
// B tile and uses two accumulators.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "gemm.cuh"
#include "layer.cuh"
#include "launch.cuh"

namespace moe {

namespace {

constexpr int kEpiWarps = 8;  // two per TMEM lane quadrant, splitting the column groups
constexpr int kProdWarps = 16;
constexpr int kMmaWarp = kEpiWarps + kProdWarps;  // 24
constexpr int kTmaWarp = kMmaWarp + 1;             // 25: packed-tile copies (TMA staging only)
__host__ __device__ constexpr int gemm_threads(bool tma) { return (kMmaWarp + (tma ? 2 : 1)) * 32; }  // 832 / 800
constexpr int kProd = kProdWarps * 32;             // 512 producer threads
// Codebook and sign tables: an entry is read as 16 bytes by 8 lanes per
// shared-memory wavefront; with 8 replicas, lane l reads replica l % 8, so
// the 8 lanes of a wavefront hit 8 different 16-byte bank groups whatever
// the entries.  (Measured on B200 at 4096 tokens: with 4 and 2 replicas the
// gate/up GEMM took 3.12 ms against 2.44, and spending the freed shared
// memory on a third A stage did not win it back.)
#ifndef MOE_GEMM_GRID_REP
#define MOE_GEMM_GRID_REP 8
#endif
#ifndef MOE_GEMM_SIGN_REP
#define MOE_GEMM_SIGN_REP 8
#endif
constexpr int kGridRep = MOE_GEMM_GRID_REP;  // replicas of the f16 codebook table
constexpr int kSignRep = MOE_GEMM_SIGN_REP;  // replicas of the sign-mask table
// K steps of packed weights a producer fetches ahead, by format: the ring
// holds (ahead + 1) items of 3 (IQ2_XXS), 6 (Q2_K) or 9 (Q8_0, Q4_K) words
__host__ __device__ constexpr int ahead_of(int fmt) { return fmt == 0 ? 6 : fmt == 1 ? 4 : 3; }
constexpr int BM = 128, BK = 64;
constexpr int kATile = BM * BK * 2;  // 16 KB
// token columns per tile: 128 for a routed gate/up pair (two accumulators
// per tile, two tiles in flight fill the 512 TMEM columns; experts hold few
// tokens, so narrow tiles waste less) and for the routed Q2_K down matrix
// (measured on B200 at 4096 tokens: the layer 5.08 ms against 5.28 ms with
// 256-column tiles, whose producers each copy twice the token rows per K
// step), 256 for the shared expert (all T tokens: wide tiles decode each
// weight tile fewer times; its pair's one tile fills TMEM alone)
#ifndef MOE_GEMM_BN_Q2K
#define MOE_GEMM_BN_Q2K 128
#endif
__host__ __device__ constexpr int bn_of(int fmt, bool paired) {
  return paired && fmt != 2 ? 128 : (!paired && fmt == 1 ? MOE_GEMM_BN_Q2K : 256);
}
__host__ __device__ constexpr int btile_of(int fmt, bool paired) { return bn_of(fmt, paired) * BK * 2; }
__host__ __device__ constexpr int nacc_of(int fmt, bool paired) { return (paired ? 2 : 1) * bn_of(fmt, paired) <= 256 ? 2 : 1; }
// stages of the dequantised A ring: how many K steps the producers may run
// ahead of the MMA (a pair's stage holds both matrices' tiles)
#ifndef MOE_GEMM_SA_PAIRED
#define MOE_GEMM_SA_PAIRED 2
#endif
#ifndef MOE_GEMM_SA_Q2K
#define MOE_GEMM_SA_Q2K 4
#endif
#ifndef MOE_GEMM_SA_IQ2
#define MOE_GEMM_SA_IQ2 MOE_GEMM_SA_PAIRED
#endif
__host__ __device__ constexpr int sa_of(int fmt, bool paired) {
  return paired ? (fmt == kFmtIQ2 ? MOE_GEMM_SA_IQ2 : MOE_GEMM_SA_PAIRED) : fmt == kFmtQ2K ? MOE_GEMM_SA_Q2K : 4;
}

// stages of the B (token rows) ring; a B tile is loaded kSB - 2 K steps
// ahead of its use (the stage it reuses was read by the MMA two steps back)
#ifndef MOE_GEMM_BSTAGES_NARROW
#define MOE_GEMM_BSTAGES_NARROW 4
#endif
constexpr int kSBMax = 8;
__host__ __device__ constexpr int sb_of(int fmt, bool paired) {
  return bn_of(fmt, paired) == 128 ? MOE_GEMM_BSTAGES_NARROW : 4;
}

// TMA staging of packed A tiles: a unit is one 256-value block (four K
// steps) of each of the tile's 128 rows.  A block starts 2 (IQ2_XXS, 66-byte
// blocks) or 4 (Q2_K, 84-byte blocks) bytes times its index past a 16-byte
// boundary; a copy's first byte must sit on one, so the box starts at the
// boundary below the block and is wide enough for the largest offset
// (14 + 66 <= 80, 12 + 84 <= 96).
__host__ __device__ constexpr int blk_bytes_of(int fmt) { return fmt == kFmtIQ2 ? 66 : 84; }
__host__ __device__ constexpr int pbox_of(int fmt) { return fmt == kFmtIQ2 ? 80 : 96; }
__host__ __device__ constexpr int pmat_of(int fmt) { return pbox_of(fmt) * BM; }
__host__ __device__ constexpr int pstage_of(int fmt, bool paired) { return (paired ? 2 : 1) * pmat_of(fmt); }
// packed stages: with s stages the copy of block b + s - 1 is issued when
// block b starts (the pair's two 10 KB boxes leave room for two stages only)
#ifndef MOE_GEMM_SP_Q2K
#define MOE_GEMM_SP_Q2K 2
#endif
constexpr int kSPMax = 4;
__host__ __device__ constexpr int sp_of(bool paired) { return paired ? 2 : MOE_GEMM_SP_Q2K; }
// Q2_K (down) tiles by TMA as well (1) or by the producers' own loads (0).
// Measured on B200 (prefill, 4096 tokens): the IQ2_XXS gate/up GEMM takes
// 2.47 ms with TMA staging against 2.86 ms without; the Q2_K down GEMM 2.30
// ms against 2.08 ms (its 16-value items leave little decode to hide the
// staged reads behind, and the 96-byte staged rows put two of every eight
// rows of a warp on the same banks), whatever the depth of the rings; with
// 128-column down tiles the layer took 5.18 ms with staging against 5.09.
#ifndef MOE_GEMM_TMA_Q2K
#define MOE_GEMM_TMA_Q2K 0
#endif

struct alignas(8) GemmCtl {
  uint64_t full[kSBMax], emptyA[4], emptyB[kSBMax], acc_full[2], acc_empty[2], drain;
  uint64_t pfull[kSPMax], pempty[kSPMax];
  uint32_t tmem_base;
  int abort;
  long long wait;  // bound of the role hand-off waits (cycles)
  int n_groups;
  int total_tiles;
  int tile_prefix[257];  // tiles before group g
  int col_off[257];      // first column of group g
};

__device__ __forceinline__ void mbar_init(uint64_t *b, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(b)) : "memory");
}
// try_wait may suspend the thread until the phase completes; with a
// suspend-time hint (ns) the hardware may keep it suspended that long, so a
// waiting warp spins less and leaves issue slots to the others.
#ifndef MOE_GEMM_SUSPEND_NS
#define MOE_GEMM_SUSPEND_NS 0
#endif
__device__ __forceinline__ bool mbar_try(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  if (MOE_GEMM_SUSPEND_NS > 0)
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(b)), "r"(parity), "n"(MOE_GEMM_SUSPEND_NS)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(b)), "r"(parity)
        : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_test(uint64_t *b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; false when this CTA is aborting (timeout here or elsewhere).
// try_wait may suspend the thread until the phase completes, which can
// outlast a bound shorter than the default; such bounds poll with the
// non-blocking test_wait instead.
template <typename Ctl>
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity, Ctl &ctl, int *err) {
  if (ctl.wait < kDefaultWaitCycles) {
    const long long t0 = clock64();
    while (!mbar_test(b, parity)) {
      if (*((volatile int *)&ctl.abort)) return false;
      if (clock64() - t0 > ctl.wait) {
        *((volatile int *)&ctl.abort) = 1;
        set_error(err, kErrTimeout);
        return false;
      }
    }
    return true;
  }
  if (mbar_try(b, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try(b, parity)) {
    if (*((volatile int *)&ctl.abort)) return false;
    if (clock64() - t0 > ctl.wait) {
      *((volatile int *)&ctl.abort) = 1;
      set_error(err, kErrTimeout);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_tx(uint64_t *b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}
// 2-D tensor copy global -> this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// K-major operand tile, 128-byte rows, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;               // leading byte offset (unused for this layout)
  d |= (uint64_t)(1024u >> 4) << 32;     // stride byte offset
  d |= (uint64_t)1u << 46;               // descriptor version
  d |= (uint64_t)2u << 61;               // 128-byte swizzle
  return d;
}

// kind::f16 instruction descriptor: fp32 accumulate, K-major A and B, M = 128.
__device__ __forceinline__ uint32_t instr_desc(int n, int bf16) {
  return (1u << 4) | ((uint32_t)bf16 << 7) | ((uint32_t)bf16 << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
__device__ __forceinline__ void mma_commit(uint64_t *b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(b))
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

// Packed weights are read once per tile; with MOE_GEMM_EVICT_FIRST their
// loads carry an L2 evict-first policy so the activation rows that every
// tile of a group re-reads stay in L2.
#ifndef MOE_GEMM_EVICT_FIRST
#define MOE_GEMM_EVICT_FIRST 0
#endif
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint32_t ldg16(const uint8_t *p) {
  if (MOE_GEMM_EVICT_FIRST) {
    uint16_t v;
    asm volatile("ld.global.L2::cache_hint.u16 %0, [%1], %2;\n" : "=h"(v) : "l"(p), "l"(l2_evict_first()));
    return v;
  }
  return *reinterpret_cast<const uint16_t *>(p);
}
__device__ __forceinline__ uint32_t ldg32(const uint8_t *p) {
  if (MOE_GEMM_EVICT_FIRST) {
    uint32_t v;
    asm volatile("ld.global.L2::cache_hint.u32 %0, [%1], %2;\n" : "=r"(v) : "l"(p), "l"(l2_evict_first()));
    return v;
  }
  return *reinterpret_cast<const uint32_t *>(p);
}

__device__ __forceinline__ void sts128(uint8_t *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  *reinterpret_cast<uint4 *>(p) = make_uint4(a, b, c, d);
}

// 16-byte chunk `chunk` (0..7) of row `row` in a 128-byte-swizzled tile.
__device__ __forceinline__ uint8_t *swz(uint8_t *tile, int row, int chunk) {
  return tile + row * 128 + ((chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ uint32_t h2bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 bits2h(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

// One accumulator element (row m of the tile's weights, global column c):
// dv = D of the first matrix, u = D of the pair's second (SwiGLU only).
__device__ __forceinline__ void epilogue_one(const GemmArgs &a, float dv, float u, int c, int m) {
  if (a.epi == kEpiSwiGLU) {
    // SiLU with the fast exponential and reciprocal (rcp(inf) = 0 for large -dv)
    const float h = dv * __frcp_rn(1.f + __expf(-dv)) * u;
    uint16_t hb;
    if (a.h_bf16) {
      __nv_bfloat16 v = __float2bfloat16_rn(h);
      hb = *reinterpret_cast<uint16_t *>(&v);
    } else {
      __half v = __float2half_rn(h);
      hb = *reinterpret_cast<uint16_t *>(&v);
    }
    a.h_out[(size_t)c * a.h_ld + m] = hb;
  } else if (a.epi == kEpiScatterAdd) {
    const int pr = a.perm[c];
    atomicAdd(a.y + (size_t)(pr / a.k) * a.y_ld + m, a.w[pr] * dv);
  } else if (a.epi == kEpiSlotStore) {
    const int pr = a.perm[c];
    a.y[(size_t)pr * a.y_ld + m] = a.w[pr] * dv;
  } else {
    float v = dv;
    if (a.res) v += a.res[(size_t)c * a.y_ld + m];
    a.y[(size_t)c * a.y_ld + m] = v;
  }
}

// ---------------------------------------------------------------- tile map

struct Tile {
  int g, m0, n0, nt, col0;
};

template <int BN>
__device__ __forceinline__ Tile tile_at(const GemmCtl &ctl, int t, int m_tiles) {
  int lo = 0, hi = ctl.n_groups - 1;
  while (lo < hi) {  // last group with prefix <= t
    const int mid = (lo + hi + 1) >> 1;
    if (ctl.tile_prefix[mid] <= t)
      lo = mid;
    else
      hi = mid - 1;
  }
  Tile r;
  r.g = lo;
  const int local = t - ctl.tile_prefix[lo];
  const int n = ctl.col_off[lo + 1] - ctl.col_off[lo];
  const int ntl = (n + BN - 1) / BN;
  const int mt = local / ntl, nti = local - mt * ntl;
  r.m0 = mt * BM;
  r.n0 = nti * BN;
  r.nt = min(BN, n - r.n0);
  r.col0 = ctl.col_off[lo] + r.n0;
  return r;
}

// ---------------------------------------------------------------- producers
//
// A producer thread owns one (row, 32-element half) item of the 128 x 64 K
// step (for a gate/up pair, the same item of both matrices).  fetch() reads
// the packed bytes of an item into registers (issued two K steps ahead of
// their use); decode() turns them into 16-bit values in the swizzled tile.

template <int FMT>
struct Raw;
template <>
struct Raw<kFmtIQ2> {
  uint32_t d16, idx4, S;
};
template <>
struct Raw<kFmtQ2K> {
  uint32_t dd, sb, q[4];
};
template <>
struct Raw<kFmtQ80> {
  uint32_t d16, q[8];
};
template <>
struct Raw<kFmtQ4K> {
  uint32_t sm, q[8];  // half2 (d * scale, -dmin * min) of the sub-block; its 32 code bytes
};

// IQ2_XXS: group (kel/32) of the row.
__device__ __forceinline__ void fetch(Raw<kFmtIQ2> &r, const uint8_t *rowp, int ks, int item) {
  const int kel = ks * BK + 32 * item;
  const int blk = kel >> 8, gib = (kel >> 5) & 7;
  const uint8_t *bp = rowp + (size_t)blk * 66;
  const uint8_t *gp = bp + 2 + 8 * gib;
  r.d16 = ldg16(bp);
  if ((reinterpret_cast<uintptr_t>(gp) & 3u) == 0) {
    r.idx4 = ldg32(gp);
    r.S = ldg32(gp + 4);
  } else {
    r.idx4 = ldg16(gp) | (ldg16(gp + 2) << 16);
    r.S = ldg16(gp + 4) | (ldg16(gp + 6) << 16);
  }
}

__device__ __forceinline__ void decode(const Raw<kFmtIQ2> &r, uint8_t *tile, int row, int item, int,
                                       const uint8_t *gridh, const uint8_t *signm) {
  const __half2 f2 = __half2half2(__int2half_rn(2 * (int)(r.S >> 28) + 1));
  const __half2 d2 = __half2half2(__hmul(__ushort_as_half((unsigned short)r.d16), __float2half(0.125f)));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t ix = (r.idx4 >> (8 * j)) & 255u;
    const uint32_t m7 = (r.S >> (7 * j)) & 127u;
    const uint4 g = *reinterpret_cast<const uint4 *>(gridh + ix * (16u * kGridRep));
    const uint4 sm = *reinterpret_cast<const uint4 *>(signm + m7 * (16u * kSignRep));
    // grid value times 2s+1 is exact in f16 (at most 43 * 31); one rounding by d/8
    const uint32_t o0 = h2bits(__hmul2(__hmul2(bits2h(g.x ^ sm.x), f2), d2));
    const uint32_t o1 = h2bits(__hmul2(__hmul2(bits2h(g.y ^ sm.y), f2), d2));
    const uint32_t o2 = h2bits(__hmul2(__hmul2(bits2h(g.z ^ sm.z), f2), d2));
    const uint32_t o3 = h2bits(__hmul2(__hmul2(bits2h(g.w ^ sm.w), f2), d2));
    sts128(swz(tile, row, 4 * item + j), o0, o1, o2, o3);
  }
}

__device__ __forceinline__ uint32_t bf16pair(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Q2_K: the K step covers 64 elements of block ks/4 (two shifts of one half);
// item (0..3) = shift (item >> 1) and 16-element sub-block (item & 1) of it.
__device__ __forceinline__ void fetch(Raw<kFmtQ2K> &r, const uint8_t *rowp, int ks, int item) {
  const int blk = ks >> 2, qq = ks & 3;
  const uint8_t *bp = rowp + (size_t)blk * 84;
  const int hf = qq >> 1, sh = 2 * (qq & 1) + (item >> 1), sub = item & 1;
  r.dd = ldg32(bp + 80);
  r.sb = bp[8 * hf + 2 * sh + sub];  // scale/min byte of the sub-block
#pragma unroll
  for (int i = 0; i < 4; ++i) r.q[i] = ldg32(bp + 16 + 32 * hf + 16 * sub + 4 * i);
}

__device__ __forceinline__ void decode(const Raw<kFmtQ2K> &r, uint8_t *tile, int row, int item, int ks,
                                       const uint8_t *, const uint8_t *) {
  const int sh = 2 * (ks & 1) + (item >> 1), sub = item & 1;
  const float d = __half2float(__ushort_as_half((unsigned short)(r.dd & 0xFFFFu)));
  const float dmin = __half2float(__ushort_as_half((unsigned short)(r.dd >> 16)));
  const float dsc = d * (float)(r.sb & 15u);
  const float mn = -dmin * (float)(r.sb >> 4);
  const uint32_t V0 = bf16pair(mn, fmaf(dsc, 1.f, mn));
  const uint32_t V1 = bf16pair(fmaf(dsc, 2.f, mn), fmaf(dsc, 3.f, mn));
  uint32_t o[8];
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    const uint32_t q = (r.q[wi] >> (2 * sh)) & 0x03030303u;
    const uint32_t t = q * 0x22u + 0x10101010u;
    o[2 * wi] = __byte_perm(V0, V1, t & 0xFFFFu);
    o[2 * wi + 1] = __byte_perm(V0, V1, t >> 16);
  }
  // elements 32*(shift in the step) + 16*sub .. +15 of the 64-element step
  const int chunk = 4 * (item >> 1) + 2 * sub;
  sts128(swz(tile, row, chunk), o[0], o[1], o[2], o[3]);
  sts128(swz(tile, row, chunk + 1), o[4], o[5], o[6], o[7]);
}

// The same items read from a staged block (TMA path): `bp` is this row's
// block in the packed stage.  The block's offset in the staged row is that of
// the global block from a 16-byte boundary, so the alignment tests are the
// same for every row of a unit.
__device__ __forceinline__ uint32_t lds16(const uint8_t *p) { return *reinterpret_cast<const uint16_t *>(p); }
__device__ __forceinline__ uint32_t lds32(const uint8_t *p) { return *reinterpret_cast<const uint32_t *>(p); }
__device__ __forceinline__ void fetch_staged(Raw<kFmtIQ2> &r, const uint8_t *bp, int ks, int item) {
  const uint8_t *gp = bp + 2 + 8 * (2 * (ks & 3) + item);
  r.d16 = lds16(bp);
  if ((smem_u32(gp) & 3u) == 0) {
    r.idx4 = lds32(gp);
    r.S = lds32(gp + 4);
  } else {
    r.idx4 = lds16(gp) | (lds16(gp + 2) << 16);
    r.S = lds16(gp + 4) | (lds16(gp + 6) << 16);
  }
}
__device__ __forceinline__ void fetch_staged(Raw<kFmtQ2K> &r, const uint8_t *bp, int ks, int item) {
  const int qq = ks & 3, hf = qq >> 1, sh = 2 * (qq & 1) + (item >> 1), sub = item & 1;
  r.dd = lds32(bp + 80);
  r.sb = bp[8 * hf + 2 * sh + sub];
  const uint8_t *qp = bp + 16 + 32 * hf + 16 * sub;  // 4-byte aligned (blocks start 0, 4, 8 or 12 bytes in)
#pragma unroll
  for (int i = 0; i < 4; ++i) r.q[i] = lds32(qp + 4 * i);
}
// Q8_0: 32-element block (kel/32) of the row.
__device__ __forceinline__ void fetch(Raw<kFmtQ80> &r, const uint8_t *rowp, int ks, int item) {
  const int kel = ks * BK + 32 * item;
  const uint8_t *bp = rowp + (size_t)(kel >> 5) * 34;
  r.d16 = ldg16(bp);
  const uint8_t *qp = bp + 2;
  if ((reinterpret_cast<uintptr_t>(qp) & 3u) == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) r.q[i] = ldg32(qp + 4 * i);
  } else {
    const uint8_t *base = qp - 2;  // 4-byte aligned; the last word is read as 16 bits to stay in the block
    uint32_t u[9];
#pragma unroll
    for (int i = 0; i < 8; ++i) u[i] = ldg32(base + 4 * i);
    u[8] = ldg16(base + 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) r.q[i] = __byte_perm(u[i], u[i + 1], 0x5432);
  }
}

// Q4_K (144-byte blocks: f16 d, f16 dmin, 12 bytes of 6-bit scales and mins,
// 128 code bytes; value e of a block has code byte 32*(e/64) + e%32, nibble
// (e%64)/32): the K step covers the 64-value chunk ks%4 of block ks/4, and
// item (0, 1) is its sub-block 2*(ks%4) + item, whose 32 codes are the low or
// the high nibbles of the chunk's 32 code bytes.  The sub-block's step
// d * scale and offset -dmin * min travel as one f16 pair: their rounding (a
// relative 2^-11 at most while they are normal binary16 values, >= 2^-14) is
// that of one more f16 rounding, next to the f16 / bf16 rounding of every
// tile value.
__device__ __forceinline__ void fetch(Raw<kFmtQ4K> &r, const uint8_t *rowp, int ks, int item) {
  const uint8_t *bp = rowp + (size_t)(ks >> 2) * 144;
  const int c = ks & 3, j = 2 * c + item;
  const uint32_t dd = ldg32(bp);
  const uint8_t *sm = bp + 4;
  int sc, mn;
  if (j < 4) {
    sc = sm[j] & 63;
    mn = sm[j + 4] & 63;
  } else {
    sc = (sm[j + 4] & 15) | ((sm[j - 4] >> 6) << 4);
    mn = (sm[j + 4] >> 4) | ((sm[j] >> 6) << 4);
  }
  const float d = __half2float(__ushort_as_half((unsigned short)(dd & 0xFFFFu)));
  const float dmin = __half2float(__ushort_as_half((unsigned short)(dd >> 16)));
  r.sm = h2bits(__floats2half2_rn(d * (float)sc, -dmin * (float)mn));
#pragma unroll
  for (int i = 0; i < 8; ++i) r.q[i] = ldg32(bp + 16 + 32 * c + 4 * i);
}

__device__ __forceinline__ void decode(const Raw<kFmtQ4K> &r, uint8_t *tile, int row, int item, int bf16,
                                       const uint8_t *, const uint8_t *) {
  const float2 f = __half22float2(bits2h(r.sm));
  const float dsc = f.x, mn = f.y;
  // 16-byte chunk c of the item: values 8c .. 8c+7 (code words 2c, 2c+1),
  // stored as soon as they are made
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t x = (r.q[2 * c + h] >> (4 * item)) & 0x0F0F0F0Fu;
      const float v0 = fmaf(dsc, (float)(x & 255u), mn), v1 = fmaf(dsc, (float)((x >> 8) & 255u), mn);
      const float v2 = fmaf(dsc, (float)((x >> 16) & 255u), mn), v3 = fmaf(dsc, (float)(x >> 24), mn);
      o[2 * h] = bf16 ? bf16pair(v0, v1) : h2bits(__floats2half2_rn(v0, v1));
      o[2 * h + 1] = bf16 ? bf16pair(v2, v3) : h2bits(__floats2half2_rn(v2, v3));
    }
    sts128(swz(tile, row, 4 * item + c), o[0], o[1], o[2], o[3]);
  }
}

template <bool BF16>
__device__ __forceinline__ void decode_q80(const Raw<kFmtQ80> &r, uint8_t *tile, int row, int item) {
  uint32_t o[16];
  const __half dh = __ushort_as_half((unsigned short)r.d16);
  const __half2 bias = __half2half2(__float2half(1152.f));
  if (!BF16) {
    const __half2 d2 = __half2half2(dh);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t x = r.q[i] ^ 0x80808080u;
      const __half2 lo = __hsub2(bits2h(__byte_perm(x, 0x64646464u, 0x5140)), bias);
      const __half2 hi = __hsub2(bits2h(__byte_perm(x, 0x64646464u, 0x7362)), bias);
      o[2 * i] = h2bits(__hmul2(lo, d2));
      o[2 * i + 1] = h2bits(__hmul2(hi, d2));
    }
  } else {
    const float d = __half2float(dh);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t x = r.q[i] ^ 0x80808080u;
      const float2 lo = __half22float2(__hsub2(bits2h(__byte_perm(x, 0x64646464u, 0x5140)), bias));
      const float2 hi = __half22float2(__hsub2(bits2h(__byte_perm(x, 0x64646464u, 0x7362)), bias));
      o[2 * i] = bf16pair(lo.x * d, lo.y * d);
      o[2 * i + 1] = bf16pair(hi.x * d, hi.y * d);
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) sts128(swz(tile, row, 4 * item + c), o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
}

__device__ __forceinline__ void decode(const Raw<kFmtQ80> &r, uint8_t *tile, int row, int item, int bf16,
                                       const uint8_t *, const uint8_t *) {
  if (bf16)
    decode_q80<true>(r, tile, row, item);
  else
    decode_q80<false>(r, tile, row, item);
}

// ---------------------------------------------------------------- kernel

template <int FMT, bool PAIRED, bool TMA>
__global__ void __launch_bounds__(gemm_threads(TMA), 1) k_grouped_gemm(GemmArgs a) {
  static_assert(!TMA || FMT == kFmtIQ2 || FMT == kFmtQ2K, "TMA staging of IQ2_XXS and Q2_K tiles only");
  // A (dequantised weights) and B (gathered token rows) have rings of their
  // own: a B tile is loaded kBAhead steps before its use, an A tile is
  // written in the step that hands it to the MMA; step `it` uses A stage
  // it % SA and B stage it % kSB, and its full barrier is full[it % kSB]
  constexpr int NA = PAIRED ? 2 : 1;
  constexpr int SA = sa_of(FMT, PAIRED);
  constexpr int BN = bn_of(FMT, PAIRED);
  constexpr int kBTile = btile_of(FMT, PAIRED);
  constexpr int kSB = sb_of(FMT, PAIRED);
  constexpr int kBAhead = kSB - 2;
  static_assert(kSB <= kSBMax, "B ring");
  // accumulator buffers in tensor memory: two tiles alternate (a pair's two
  // 128-column accumulators, or one 256-column accumulator, per tile), so the
  // epilogue of one tile overlaps the main loop of the next
  constexpr int NACC = nacc_of(FMT, PAIRED);
  constexpr int ACC_COLS = NA * BN;  // columns of one tile's accumulators
  constexpr int ASTAGE = NA * kATile;
  constexpr bool kTables = FMT == kFmtIQ2;
  constexpr int kAhead = ahead_of(FMT);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kPMat = pmat_of(FMT), kPStage = TMA ? pstage_of(FMT, PAIRED) : 0;
  constexpr int kSP = sp_of(PAIRED);
  static_assert(kSP <= kSPMax, "packed ring");
  uint8_t *stagesA = smem;
  uint8_t *stagesB = stagesA + SA * ASTAGE;
  uint8_t *stagesP = stagesB + kSB * kBTile;              // packed stages (TMA staging)
  uint8_t *gridh = stagesP + kSP * kPStage;               // 256 x kGridRep x 16 B: codebook as f16
  uint8_t *signm = gridh + (kTables ? 4096 * kGridRep : 0);  // 128 x kSignRep x 16 B: f16 sign masks
  GemmCtl &ctl = *reinterpret_cast<GemmCtl *>(signm + (kTables ? 2048 * kSignRep : 0));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m_tiles = a.M / BM;
  const int ksteps = a.K / BK;

  // ---- set-up
  if (tid == 0) {
    for (int s = 0; s < kSB; ++s) {
      mbar_init(&ctl.full[s], kProd);
      mbar_init(&ctl.emptyB[s], 1);
    }
    for (int s = 0; s < SA; ++s) mbar_init(&ctl.emptyA[s], 1);
    for (int s = 0; s < kSP; ++s) {
      mbar_init(&ctl.pfull[s], 1);       // the issuing thread's expect_tx arrival (+ the copies' bytes)
      mbar_init(&ctl.pempty[s], kProd);  // every producer, after its last read of the unit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl.acc_full[b], 1);
      mbar_init(&ctl.acc_empty[b], kEpiWarps * 32);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    ctl.wait = a.wait_cycles > 0 ? a.wait_cycles : kDefaultWaitCycles;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (tid == 32) {  // group table
    const int G = a.offsets ? a.n_groups : 1;
    int pre = 0;
    for (int g = 0; g < G; ++g) {
      const int c0 = a.offsets ? a.offsets[g] : 0;
      const int c1 = a.offsets ? a.offsets[g + 1] : a.cols;
      ctl.col_off[g] = c0;
      ctl.tile_prefix[g] = pre;
      pre += m_tiles * ((c1 - c0 + BN - 1) / BN);
    }
    ctl.col_off[G] = a.offsets ? a.offsets[G] : a.cols;
    ctl.tile_prefix[G] = pre;
    ctl.n_groups = G;
    ctl.total_tiles = pre;
  }
  if (FMT == kFmtIQ2) {
    for (int i = tid; i < 256 * 8 * kGridRep; i += blockDim.x) {  // codebook -> f16
      const int l = i & 7, rep = (i >> 3) % kGridRep, ix = (i >> 3) / kGridRep;
      reinterpret_cast<__half *>(gridh)[(ix * kGridRep + rep) * 8 + l] = __int2half_rn(a.grid[ix * 8 + l]);
    }
    for (int i = tid; i < 128 * kSignRep; i += blockDim.x) {
      const int m7 = i / kSignRep, rep = i % kSignRep;
      const uint32_t m8 = (uint32_t)m7 | ((uint32_t)(__popc(m7) & 1) << 7);
      uint32_t *e = reinterpret_cast<uint32_t *>(signm + (m7 * kSignRep + rep) * 16);
#pragma unroll
      for (int p = 0; p < 4; ++p)
        e[p] = (((m8 >> (2 * p)) & 1u) << 15) | (((m8 >> (2 * p + 1)) & 1u) << 31);
    }
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&ctl.tmem_base)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  const int total = ctl.total_tiles;

  if (warp >= kEpiWarps && warp < kMmaWarp) {
    // =================================================== producers
    const int p = tid - kEpiWarps * 32;
    const uint8_t *gridh_l = gridh + 16 * (lane % kGridRep);
    const uint8_t *signm_l = signm + 16 * (lane % kSignRep);
    constexpr int kBRows = BN / 64;  // B rows per producer thread and step
    uint32_t it = 0, pu = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile tl = tile_at<BN>(ctl, t, m_tiles);
      // B rows this thread copies: rows (p >> 3) + 64 i, chunk p & 7
      const int ch = p & 7;
      const uint16_t *brow[kBRows];
#pragma unroll
      for (int i = 0; i < kBRows; ++i) {
        const int r = (p >> 3) + 64 * i;
        brow[i] = nullptr;
        if (r < tl.nt) {
          const int c = tl.col0 + r;
          const int br = a.b_perm ? a.b_perm[c] / a.b_div : c;
          brow[i] = a.b_base + (size_t)br * a.b_ld + ch * 8;
        }
      }
      // A item of this thread: paired formats: matrix p/256, row (p/2)%128, 32-element half p%2;
      // Q2_K: row p/4, item p%4 (16 elements); unpaired Q8_0 / Q4_K: row p/2, half p%2 (threads < 256)
      const int mat = PAIRED ? (p >> 8) : 0;
      const int row = FMT == kFmtQ2K ? (p >> 2) : ((p >> 1) & 127);
      const int item = FMT == kFmtQ2K ? (p & 3) : (p & 1);
      const bool has_a = PAIRED || FMT == kFmtQ2K || p < 256;
      const int dsel = (FMT == kFmtQ80 || FMT == kFmtQ4K) ? a.bf16 : 0;
      // B tile of tile-local step ks into B stage `sb` (one cp.async group)
      auto issue_b = [&](int ks, int sb) {
        uint8_t *Bs = stagesB + sb * kBTile;
#pragma unroll
        for (int i = 0; i < kBRows; ++i) {
          if (brow[i]) cp_async16(swz(Bs, (p >> 3) + 64 * i, ch), brow[i] + ks * BK);
        }
        cp_async_commit();
      };
      // waits until the B stage of global step g is free, then loads it (or
      // commits an empty group past the tile's last step)
      auto load_b = [&](int ks, uint32_t g) -> bool {
        if (ks >= ksteps) {
          cp_async_commit();
          return true;
        }
        if (!mbar_wait(&ctl.emptyB[g % kSB], ((g / kSB) & 1u) ^ 1u, ctl, a.err)) return false;
        issue_b(ks, g % kSB);
        return true;
      };
      bool ok = true;
#pragma unroll
      for (int q = 0; q < kBAhead; ++q)
        if (ok) ok = load_b(q, it + q);
      if constexpr (TMA) {
        // packed unit (block) ks / 4 of this tile is global unit pu; its
        // stage holds each row's block at the block's offset from a 16-byte
        // boundary.  The words of step ks + 1 are read from the stage while
        // step ks is handed over.
        auto staged = [&](int ks) {
          const int off = ((ks >> 2) * blk_bytes_of(FMT)) & 15;
          return stagesP + (pu % kSP) * kPStage + mat * kPMat + row * pbox_of(FMT) + off;
        };
        Raw<FMT> rn;
        if (ok && !mbar_wait(&ctl.pfull[pu % kSP], (pu / kSP) & 1u, ctl, a.err)) ok = false;
        if (ok) fetch_staged(rn, staged(0), 0, item);
        for (int ks = 0; ok && ks < ksteps; ++ks) {
          const Raw<FMT> r = rn;
          if (!load_b(ks + kBAhead, it + kBAhead) ||
              !mbar_wait(&ctl.emptyA[it % SA], ((it / SA) & 1u) ^ 1u, ctl, a.err)) {
            ok = false;
            break;
          }
          decode(r, stagesA + (it % SA) * ASTAGE + mat * kATile, row, item, FMT == kFmtQ2K ? ks : dsel, gridh_l,
                 signm_l);
          if ((ks & 3) == 3) {  // every read of this unit is done
            mbar_arrive(&ctl.pempty[pu % kSP]);
            ++pu;
          }
          if (ks + 1 < ksteps) {
            if (((ks + 1) & 3) == 0 && !mbar_wait(&ctl.pfull[pu % kSP], (pu / kSP) & 1u, ctl, a.err)) {
              ok = false;
              break;
            }
            fetch_staged(rn, staged(ks + 1), ks + 1, item);
          }
          cp_async_wait<kBAhead>();  // this step's B tile has landed
          fence_proxy_async();
          mbar_arrive(&ctl.full[it % kSB]);
          ++it;
        }
        if (!ok) break;
        continue;
      }
      const uint8_t *arow = (mat ? a.A1 : a.A0) + a.a_group_stride * tl.g + a.a_row_bytes * (size_t)(tl.m0 + row);
      // packed bytes of K steps ks .. ks + kAhead - 1 are in flight in a ring of
      // registers; slots are compile-time indices of the unrolled loop below, so
      // no register copy ever waits on a load
      Raw<FMT> R[kAhead + 1];
      if (has_a) {
#pragma unroll
        for (int j = 0; j < kAhead; ++j)
          if (j < ksteps) fetch(R[j], arow, j, item);
      }
      for (int ks0 = 0; ok && ks0 < ksteps; ks0 += kAhead + 1) {
#pragma unroll
        for (int j = 0; j <= kAhead; ++j) {
          const int ks = ks0 + j;
          if (!ok || ks >= ksteps) break;
          if (!load_b(ks + kBAhead, it + kBAhead) ||
              !mbar_wait(&ctl.emptyA[it % SA], ((it / SA) & 1u) ^ 1u, ctl, a.err)) {
            ok = false;
            break;
          }
          uint8_t *A0s = stagesA + (it % SA) * ASTAGE;
          if (has_a) decode(R[j], A0s + mat * kATile, row, item, FMT == kFmtQ2K ? ks : dsel, gridh_l, signm_l);
          cp_async_wait<kBAhead>();  // this step's B tile has landed
          fence_proxy_async();
          mbar_arrive(&ctl.full[it % kSB]);
          // the next look-ahead fetch goes out after this step is handed over
          if (has_a && ks + kAhead < ksteps) fetch(R[(j + kAhead) % (kAhead + 1)], arow, ks + kAhead, item);
          ++it;
        }
      }
      if (!ok) break;
    }
    cp_async_wait<0>();
  } else if (warp == kMmaWarp) {
    // =================================================== MMA issue
    uint32_t it = 0, tc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++tc) {
      const Tile tl = tile_at<BN>(ctl, t, m_tiles);
      const int nmma = (tl.nt + 15) & ~15;
      const uint32_t idesc = instr_desc(nmma, a.bf16);
      const uint32_t buf = tc % NACC;
      const uint32_t dacc = tmem + buf * ACC_COLS;  // accumulator columns of this tile
      if (!mbar_wait(&ctl.acc_empty[buf], ((tc / NACC) & 1u) ^ 1u, ctl, a.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int ks = 0; ks < ksteps; ++ks, ++it) {
        const uint32_t ph = (it / kSB) & 1u;
        if (!mbar_wait(&ctl.full[it % kSB], ph, ctl, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(stagesA + (it % SA) * ASTAGE);
          const uint32_t b0 = smem_u32(stagesB + (it % kSB) * kBTile);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            mma_f16(dacc, smem_desc(a0 + 32 * kk), smem_desc(b0 + 32 * kk), idesc, acc);
            if (PAIRED) mma_f16(dacc + BN, smem_desc(a0 + kATile + 32 * kk), smem_desc(b0 + 32 * kk), idesc, acc);
          }
          mma_commit(&ctl.emptyA[it % SA]);
          mma_commit(&ctl.emptyB[it % kSB]);
        }
        __syncwarp();
      }
      if (ok && lane == 0) mma_commit(&ctl.acc_full[buf]);
      __syncwarp();
    }
    // drain: every MMA this thread issued has finished before tensor memory is freed
    if (lane == 0) {
      mma_commit(&ctl.drain);
      const long long t0 = clock64();
      while (!mbar_try(&ctl.drain, 0u)) {
        if (clock64() - t0 > kDefaultWaitCycles) {
          set_error(a.err, kErrTimeout);
          break;
        }
      }
    }
    __syncwarp();
  } else if (TMA && warp == kTmaWarp) {
    // =================================================== packed-tile copies
    // Units in the producers' order (this CTA's tiles, K blocks within a
    // tile): unit u goes to packed stage u % kSP as soon as every producer
    // has read unit u - kSP from it.
    if (lane == 0) {
      // the maps were written to global memory by a copy from the host
      // (possibly over older maps at the same address): order that write
      // before the tensor copies read them
      asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;\n" ::"l"(a.tmA) : "memory");
      if (PAIRED)
        asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;\n" ::"l"(
                         static_cast<const uint8_t *>(a.tmA) + 128)
                     : "memory");
      const int kunits = ksteps / 4;
      uint32_t pu = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        const Tile tn = tile_at<BN>(ctl, t, m_tiles);
        const int y0 = tn.g * a.M + tn.m0;
        for (int pk = 0; pk < kunits; ++pk, ++pu) {
          const uint32_t ps = pu % kSP;
          if (!mbar_wait(&ctl.pempty[ps], ((pu / kSP) & 1u) ^ 1u, ctl, a.err)) {
            ok = false;
            break;
          }
          const int x0 = (pk * blk_bytes_of(FMT)) & ~15;  // 16-byte aligned start of the box
          uint8_t *dst = stagesP + ps * kPStage;
          mbar_arrive_tx(&ctl.pfull[ps], (uint32_t)kPStage);
          tma_load_2d(dst, a.tmA, x0, y0, &ctl.pfull[ps]);
          if (PAIRED) tma_load_2d(dst + kPMat, static_cast<const uint8_t *>(a.tmA) + 128, x0, y0, &ctl.pfull[ps]);
        }
      }
      // every copy issued has landed before the CTA exits
      for (uint32_t q = pu > kSP ? pu - kSP : 0; q < pu; ++q) {  // the last unit of each stage
        const long long t1 = clock64();
        while (!mbar_try(&ctl.pfull[q % kSP], (q / kSP) & 1u)) {
          if (clock64() - t1 > kDefaultWaitCycles) {
            set_error(a.err, kErrTimeout);
            break;
          }
        }
      }
    }
    __syncwarp();
  } else {
    // =================================================== epilogue
    // warp w reads TMEM lanes 32 (w % 4) .. + 31 (the quadrant it may access)
    // and the 16-column groups g with g % 2 == w / 4
    const int row = (warp & 3) * 32 + lane;  // TMEM lane = weight row in the tile
    const int half = warp >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    uint32_t tc = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tc) {
      const Tile tl = tile_at<BN>(ctl, t, m_tiles);
      const uint32_t buf = tc % NACC;
      if (!mbar_wait(&ctl.acc_full[buf], (tc / NACC) & 1u, ctl, a.err)) break;
      tc_fence_after();
      const int m = tl.m0 + row;
      for (int c0 = 16 * half; c0 < tl.nt; c0 += 32) {
        uint32_t r0[16], r1[16];
        tmem_ld16(lane_base + buf * ACC_COLS + c0, r0);
        if (PAIRED) tmem_ld16(lane_base + buf * ACC_COLS + BN + c0, r1);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = c0 + j;
          if (n >= tl.nt) break;
          epilogue_one(a, __uint_as_float(r0[j]), __uint_as_float(PAIRED ? r1[j] : 0u), tl.col0 + n, m);
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl.acc_empty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(512));
  }
}

// ---------------------------------------------------------------- dense GEMM
//
// D = A B^T with A [M][K] and B [N][K] both plain 16-bit rows in global
// memory (the shared expert at large T: its Q8_0 rows expanded once per call
// by k_expand_q80, the tokens' activation rows as they are).  Both operands
// arrive by TMA as 128-byte-swizzled K-major tiles, so there are no producer
// warps: warps 0-7 epilogue (as above), warp 8 tensor memory and
// tcgen05.mma, warp 9 the tensor copies.  Tiles, MMA order and epilogue are
// those of the grouped kernel for the same matrix, so the results are the
// same bits.

constexpr int kDenseMmaWarp = kEpiWarps;       // 8
constexpr int kDenseCopyWarp = kEpiWarps + 1;  // 9
constexpr int kDenseThreads = (kEpiWarps + 2) * 32;
constexpr int kDenseBN = 256;
__host__ __device__ constexpr int dense_stages(bool paired) { return paired ? 3 : 4; }
__host__ __device__ constexpr int dense_stage_bytes(bool paired) { return (paired ? 2 : 1) * kATile + kDenseBN * BK * 2; }

struct alignas(8) DenseCtl {
  uint64_t full[4], empty[4], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int abort;
  long long wait;
};

template <bool PAIRED>
__global__ void __launch_bounds__(kDenseThreads, 1)
    k_dense_gemm(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                 const __grid_constant__ CUtensorMap tmB, GemmArgs a) {
  constexpr int NA = PAIRED ? 2 : 1;
  constexpr int BN = kDenseBN;
  constexpr int NACC = nacc_of(kFmtQ80, PAIRED);  // a pair's 2 x 256 columns fill TMEM: one buffer
  constexpr int ACC_COLS = NA * BN;
  constexpr int KS = dense_stages(PAIRED);
  constexpr int STAGE = dense_stage_bytes(PAIRED);
  static_assert(bn_of(kFmtQ80, PAIRED) == BN, "same tiles as the grouped kernel");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  DenseCtl &ctl = *reinterpret_cast<DenseCtl *>(smem + KS * STAGE);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m_tiles = a.M / BM, n_tiles = (a.cols + BN - 1) / BN, total = m_tiles * n_tiles;
  const int ksteps = a.K / BK;

  if (tid == 0) {
    for (int s = 0; s < KS; ++s) {
      mbar_init(&ctl.full[s], 1);   // the copy thread's expect_tx arrival (+ the copies' bytes)
      mbar_init(&ctl.empty[s], 1);  // the MMA thread's commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl.acc_full[b], 1);
      mbar_init(&ctl.acc_empty[b], kEpiWarps * 32);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    ctl.wait = a.wait_cycles > 0 ? a.wait_cycles : kDefaultWaitCycles;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kDenseMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&ctl.tmem_base)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == kDenseCopyWarp) {
    // =================================================== tensor copies
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        const int m0 = (t / n_tiles) * BM, n0 = (t % n_tiles) * BN;
        for (int ks = 0; ks < ksteps; ++ks, ++it) {
          const uint32_t s = it % KS;
          if (!mbar_wait(&ctl.empty[s], ((it / KS) & 1u) ^ 1u, ctl, a.err)) {
            ok = false;
            break;
          }
          uint8_t *st = smem + s * STAGE;
          mbar_arrive_tx(&ctl.full[s], (uint32_t)STAGE);
          tma_load_2d(st, &tmA0, ks * BK, m0, &ctl.full[s]);
          if (PAIRED) tma_load_2d(st + kATile, &tmA1, ks * BK, m0, &ctl.full[s]);
          tma_load_2d(st + NA * kATile, &tmB, ks * BK, n0, &ctl.full[s]);  // rows past N read as zeros
        }
      }
      // every copy issued has landed before the CTA exits
      for (uint32_t q = it > KS ? it - KS : 0; q < it; ++q) {
        const long long t1 = clock64();
        while (!mbar_try(&ctl.full[q % KS], (q / KS) & 1u)) {
          if (clock64() - t1 > kDefaultWaitCycles) {
            set_error(a.err, kErrTimeout);
            break;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == kDenseMmaWarp) {
    // =================================================== MMA issue
    uint32_t it = 0, tc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++tc) {
      const int n0 = (t % n_tiles) * BN;
      const int nt = min(BN, a.cols - n0);
      const uint32_t idesc = instr_desc((nt + 15) & ~15, a.bf16);
      const uint32_t buf = tc % NACC;
      const uint32_t dacc = tmem + buf * ACC_COLS;
      if (!mbar_wait(&ctl.acc_empty[buf], ((tc / NACC) & 1u) ^ 1u, ctl, a.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int ks = 0; ks < ksteps; ++ks, ++it) {
        const uint32_t s = it % KS;
        if (!mbar_wait(&ctl.full[s], (it / KS) & 1u, ctl, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(smem + s * STAGE), b0 = a0 + NA * kATile;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            mma_f16(dacc, smem_desc(a0 + 32 * kk), smem_desc(b0 + 32 * kk), idesc, acc);
            if (PAIRED) mma_f16(dacc + BN, smem_desc(a0 + kATile + 32 * kk), smem_desc(b0 + 32 * kk), idesc, acc);
          }
          mma_commit(&ctl.empty[s]);
        }
        __syncwarp();
      }
      if (ok && lane == 0) mma_commit(&ctl.acc_full[buf]);
      __syncwarp();
    }
    if (lane == 0) {
      mma_commit(&ctl.drain);
      const long long t0 = clock64();
      while (!mbar_try(&ctl.drain, 0u)) {
        if (clock64() - t0 > kDefaultWaitCycles) {
          set_error(a.err, kErrTimeout);
          break;
        }
      }
    }
    __syncwarp();
  } else {
    // =================================================== epilogue (warps 0-7)
    const int row = (warp & 3) * 32 + lane;
    const int half = warp >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    uint32_t tc = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tc) {
      const int m0 = (t / n_tiles) * BM, n0 = (t % n_tiles) * BN;
      const int nt = min(BN, a.cols - n0);
      const uint32_t buf = tc % NACC;
      if (!mbar_wait(&ctl.acc_full[buf], (tc / NACC) & 1u, ctl, a.err)) break;
      tc_fence_after();
      for (int c0 = 16 * half; c0 < nt; c0 += 32) {
        uint32_t r0[16], r1[16];
        tmem_ld16(lane_base + buf * ACC_COLS + c0, r0);
        if (PAIRED) tmem_ld16(lane_base + buf * ACC_COLS + BN + c0, r1);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = c0 + j;
          if (n >= nt) break;
          epilogue_one(a, __uint_as_float(r0[j]), __uint_as_float(PAIRED ? r1[j] : 0u), n0 + n, m0 + row);
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl.acc_empty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kDenseMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(512));
  }
}

// out[r][k] = the Q8_0 value d * q of W's row r, rounded once to f16 (bf16 =
// 0) or bf16 (bf16 = 1): the operand the grouped kernel's Q8_0 producers make.
// One thread per 8 values.
__global__ void k_expand_q80(const uint8_t *__restrict__ W, int rows, int K, int bf16, uint16_t *__restrict__ out) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int per_row = K / 8;
  if (i >= (size_t)rows * per_row) return;
  const size_t r = i / per_row;
  const int c8 = (int)(i - r * per_row);
  const uint8_t *bp = W + r * (size_t)(K / 32) * 34 + (size_t)(c8 >> 2) * 34;
  const float d = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t *>(bp)));
  const uint8_t *qp = bp + 2 + 8 * (c8 & 3);  // 2-byte aligned
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t qq = *reinterpret_cast<const uint16_t *>(qp + 2 * j);
    const float v0 = (float)(int8_t)(qq & 255u) * d, v1 = (float)(int8_t)(qq >> 8) * d;  // exact products
    o[j] = bf16 ? bf16pair(v0, v1) : h2bits(__floats2half2_rn(v0, v1));
  }
  *reinterpret_cast<uint4 *>(out + r * (size_t)K + 8 * (size_t)c8) = make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace

size_t grouped_gemm_smem(int fmt, int paired, int tma) {
  const int na = paired ? 2 : 1;
  const int sa = sa_of(fmt, paired != 0);
  const size_t tables = fmt == kFmtIQ2 ? 4096 * kGridRep + 2048 * kSignRep : 0;
  const size_t packed = tma ? (size_t)sp_of(paired != 0) * pstage_of(fmt, paired != 0) : 0;
  return 1024 + (size_t)sa * na * kATile + (size_t)sb_of(fmt, paired != 0) * btile_of(fmt, paired != 0) + packed +
         tables + sizeof(GemmCtl);
}

template <int FMT, bool PAIRED, bool TMA>
static cudaError_t launch_gemm(const GemmArgs &a, cudaStream_t s, int num_sms) {
  static SmemOptIn opt;
  const size_t smem = grouped_gemm_smem(FMT, PAIRED, TMA);
  cudaError_t e = opt_in_smem(k_grouped_gemm<FMT, PAIRED, TMA>, smem, opt);
  if (e != cudaSuccess) return e;
  k_grouped_gemm<FMT, PAIRED, TMA><<<num_sms, gemm_threads(TMA), smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t grouped_gemm(const GemmArgs &a, cudaStream_t s, int num_sms) {
  const bool paired = a.A1 != nullptr;
  // TMA staging needs the groups' matrices back to back (row g * M + m of
  // the tensor map is row m of group g) and K a whole number of blocks
  const bool tma = a.tmA != nullptr && a.a_group_stride == (size_t)a.M * a.a_row_bytes && a.K % 256 == 0;
  if (a.fmt == kFmtIQ2 && paired)
    return tma ? launch_gemm<kFmtIQ2, true, true>(a, s, num_sms) : launch_gemm<kFmtIQ2, true, false>(a, s, num_sms);
  if (a.fmt == kFmtQ2K && !paired)
    return tma && MOE_GEMM_TMA_Q2K ? launch_gemm<kFmtQ2K, false, true>(a, s, num_sms)
                                   : launch_gemm<kFmtQ2K, false, false>(a, s, num_sms);
  if (a.fmt == kFmtQ80 && paired) return launch_gemm<kFmtQ80, true, false>(a, s, num_sms);
  if (a.fmt == kFmtQ80 && !paired) return launch_gemm<kFmtQ80, false, false>(a, s, num_sms);
  if (a.fmt == kFmtQ4K && paired) return launch_gemm<kFmtQ4K, true, false>(a, s, num_sms);
  if (a.fmt == kFmtQ4K && !paired) return launch_gemm<kFmtQ4K, false, false>(a, s, num_sms);
  return cudaErrorInvalidValue;
}

static PFN_cuTensorMapEncodeTiled tensor_map_encoder() {
  PFN_cuTensorMapEncodeTiled encode = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", reinterpret_cast<void **>(&encode), cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return encode;
}

// [rows][K] 16-bit rows, box 64 values x box_rows rows, 128-byte swizzle.
static bool rows16_map(CUtensorMap *m, const void *base, int bf16, size_t rows, size_t K, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled encode = tensor_map_encoder();
  if (!encode || !base || (reinterpret_cast<uintptr_t>(base) & 15u) || (K * 2) % 16 || K % BK) return false;
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return encode(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t dense_gemm_smem(int paired) {
  return 1024 + (size_t)dense_stages(paired != 0) * dense_stage_bytes(paired != 0) + sizeof(DenseCtl);
}

template <bool PAIRED>
static cudaError_t launch_dense(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b, const GemmArgs &a,
                                cudaStream_t s, int num_sms) {
  static SmemOptIn opt;
  const size_t smem = dense_gemm_smem(PAIRED);
  cudaError_t e = opt_in_smem(k_dense_gemm<PAIRED>, smem, opt);
  if (e != cudaSuccess) return e;
  k_dense_gemm<PAIRED><<<num_sms, kDenseThreads, smem, s>>>(a0, a1, b, a);
  return cudaGetLastError();
}

cudaError_t dense_gemm(const GemmArgs &a, const uint16_t *A0, const uint16_t *A1, const uint16_t *B, cudaStream_t s,
                       int num_sms) {
  if (a.M % BM || a.K % BK || a.cols <= 0 || a.epi == kEpiScatterAdd || a.epi == kEpiSlotStore ||
      (a.epi == kEpiSwiGLU) != (A1 != nullptr))
    return cudaErrorInvalidValue;
  CUtensorMap m0, m1, mb;
  if (!rows16_map(&m0, A0, a.bf16, (size_t)a.M, (size_t)a.K, BM) ||
      (A1 && !rows16_map(&m1, A1, a.bf16, (size_t)a.M, (size_t)a.K, BM)) ||
      !rows16_map(&mb, B, a.bf16, (size_t)a.cols, (size_t)a.K, kDenseBN))
    return cudaErrorInvalidValue;
  if (!A1) m1 = m0;
  return A1 ? launch_dense<true>(m0, m1, mb, a, s, num_sms) : launch_dense<false>(m0, m1, mb, a, s, num_sms);
}

cudaError_t expand_q80(const uint8_t *W, int rows, int K, int bf16, uint16_t *out, cudaStream_t s) {
  const size_t n = (size_t)rows * (K / 8);
  if (n == 0) return cudaSuccess;
  k_expand_q80<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(W, rows, K, bf16, out);
  return cudaGetLastError();
}

bool gemm_tensor_map(void *map, const void *base, size_t row_bytes, size_t rows, int fmt) {
  if (fmt != kFmtIQ2 && fmt != kFmtQ2K) return false;
  const int box = pbox_of(fmt);
  if (!base || (reinterpret_cast<uintptr_t>(base) & 15u) || row_bytes % 16 || row_bytes < (size_t)box || rows == 0 ||
      rows > 0xFFFFFFFFull)
    return false;
  PFN_cuTensorMapEncodeTiled encode = tensor_map_encoder();
  if (!encode) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t boxd[2] = {(cuuint32_t)box, (cuuint32_t)BM};
  const cuuint32_t es[2] = {1, 1};
  return encode(reinterpret_cast<CUtensorMap *>(map), CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims,
                strides, boxd, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace moe
