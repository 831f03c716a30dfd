// gemm.cuh -- grouped tensor-core GEMM of the large-T path.
//
// D[m][n] = sum_k A[m][k] * B[n][k] for column groups (one per expert, or one
// for the shared expert), A = packed weight rows dequantised on the fly, B =
// 16-bit activation rows gathered per column.  Epilogues: SwiGLU of a paired
// gate/up product into 16-bit h rows; routing-weighted scatter-add into y;
// plain store into y.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

enum GemmFmt { kFmtIQ2 = 0, kFmtQ2K = 1, kFmtQ80 = 2, kFmtQ4K = 3 };
enum GemmEpi { kEpiSwiGLU = 0, kEpiScatterAdd = 1, kEpiStore = 2, kEpiSlotStore = 3 };

struct GemmArgs {
  int fmt;    // GemmFmt of the A operand
  int bf16;   // operand type: 0 = f16, 1 = bf16
  int epi;    // GemmEpi
  int M, K;   // weight rows / reduction length (multiples of 128 / 256)
  int n_groups;
  const int32_t *offsets;  // [n_groups+1] column ranges; nullptr: one group of `cols` columns
  int cols;
  const uint8_t *A0, *A1;  // packed weights of group 0 (A1: the up matrix of a gate/up pair)
  size_t a_group_stride;   // bytes between consecutive groups' matrices
  size_t a_row_bytes;
  const uint8_t *grid;     // IQ2_XXS codebook [256][8]
  // B: row of column c (global column index, offsets[g] + n) is
  //    b_base + b_ld * (b_perm ? b_perm[c] / b_div : c)
  const uint16_t *b_base;
  int b_ld;
  const int32_t *b_perm;
  int b_div;
  // epilogues
  uint16_t *h_out;   // SwiGLU: h_out[c * h_ld + m] (16-bit, same type as `h_bf16`)
  int h_ld;
  int h_bf16;
  float *y;          // ScatterAdd: y[(perm[c]/k) * y_ld + m] += w[perm[c]] * D
  int y_ld;          // Store: y[c * y_ld + m] = D (+ res[c * y_ld + m])
                     // SlotStore: y[perm[c] * y_ld + m] = w[perm[c]] * D (one row per pair)
  const float *res;
  const float *w;
  const int32_t *perm;
  int k;
  int *err;
  long long wait_cycles;  // bound of the waits between the kernel's roles (0: the default)
  // TMA staging of the packed A tiles (IQ2_XXS pairs and Q2_K only): device
  // address of the tensor maps built by gemm_tensor_map, A0's then (paired)
  // A1's, 128 bytes each; nullptr: producers load the packed bytes themselves
  const void *tmA;
};

cudaError_t grouped_gemm(const GemmArgs &a, cudaStream_t s, int num_sms);
size_t grouped_gemm_smem(int fmt, int paired, int tma);

// D = A B^T for plain 16-bit operand rows (A0 [M][K], B [cols][K], both with
// row stride K, f16 or bf16 as a.bf16 says): the same tiles, MMA order and
// epilogues (SwiGLU with A1 = the pair's up rows, or store) as grouped_gemm on
// one group, fed by TMA instead of producer warps.  Reads a.bf16, epi, M, K,
// cols, the epilogue fields, err and wait_cycles.
cudaError_t dense_gemm(const GemmArgs &a, const uint16_t *A0, const uint16_t *A1, const uint16_t *B, cudaStream_t s,
                       int num_sms);
size_t dense_gemm_smem(int paired);

// out [rows][K] = the values of Q8_0 rows W (K a multiple of 32), each d * q
// rounded once to f16 (bf16 = 0) or bf16: the operands grouped_gemm's Q8_0
// producers make, for dense_gemm.
cudaError_t expand_q80(const uint8_t *W, int rows, int K, int bf16, uint16_t *out, cudaStream_t s);

// Tensor map (128 bytes, written to `map`) of a packed weight array of `rows`
// rows of `row_bytes` bytes in `fmt` (kFmtIQ2 or kFmtQ2K) for the TMA staging
// of the grouped GEMM's A tiles: one copy brings one 256-value block of 128
// consecutive rows.  False when the shape or the driver does not allow it
// (rows not a multiple of 16 bytes, a misaligned base, no encoder entry
// point); the GEMM then runs without TMA staging.
bool gemm_tensor_map(void *map, const void *base, size_t row_bytes, size_t rows, int fmt);

}  // namespace moe
