/*
 * oracle.h -- plain, slow, fp64 CPU oracle for one DwarfStar-quantised
 * DeepSeek-V4-Flash MoE FFN layer.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this code.  It shares nothing with the CUDA layer
 * (no headers, helpers, tables or constants); both read the same seeded
 * inputs from the synth package and nothing else.
 *
 * Sources (cited below by tag):
 *  [FLOW]  DeepSeek-V4-Flash one-token computation flow for the Dwarf Star
 *          (ds4) q2 build, qiita.com/sukimaengineer/items/cd76fec76d49a098abed
 *          -- the config.json table ("DeepSeek-V4-Flash の実像"); section
 *          "MoE FFN 部の中身: router → top-6 → expert → 加重和"; section
 *          "Dwarf Star の量子化の工夫" (bit-allocation table and the format
 *          paragraph after it).
 *  [QUANT] "2bit 量子化はなぜ「冗談ではない」のか: DwarfStar の非対称量子化と
 *          imatrix を読む" (ds4.c を読み解く #2),
 *          qiita.com/yoshiyakato/items/4678be0e7860ddb444ec -- section 3
 *          "Q2_K: 256 要素を 84 バイトにする K-quant" (type-trait table, the
 *          offsets enum and the 2-bit packing expression) and section 4
 *          "IQ2_XXS: 小さいが、imatrix 前提の 2bit" (structure list).
 *  [ARCH]  "2023-2026年の大規模モデルアーキテクチャ総復習", knightli.com MoE
 *          tag feed -- sections "正規化：RMSNorm が一般的に" and
 *          "活性化関数：ReLU/GELU から SwiGLU へ" (both give no formula; the
 *          textbook definitions are used).
 *
 * Readings where the sources leave a step open are listed where they are
 * used; each is one fixed choice that the CUDA layer implements separately.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* IEEE binary16 (little-endian bits) to double, subnormals included. */
double oracle_f16(uint16_t bits);

/* Decode one element / one full row of `cols` elements.  Formats (kind):
 * 0 IQ2_XXS, 1 Q2_K, 2 Q8_0, 3 Q4_K. */
double oracle_iq2xxs_elem(const uint8_t *block66, const uint8_t *grid, int e);
double oracle_q2k_elem(const uint8_t *block84, int e);
double oracle_q80_elem(const uint8_t *block34, int e);
double oracle_q4k_elem(const uint8_t *block144, int e);
void oracle_row_iq2xxs(const uint8_t *row, int cols, const uint8_t *grid, double *out);
void oracle_row_q2k(const uint8_t *row, int cols, double *out);
void oracle_row_q80(const uint8_t *row, int cols, double *out);
void oracle_row_q4k(const uint8_t *row, int cols, double *out);

/* Every row of a [rows][cols] matrix decoded into out (row-major fp64). */
void oracle_decode_matrix(int kind, const uint8_t *W, int rows, int cols, const uint8_t *grid, double *out);

/* y[r] = sum_c W[r][c] x[c] with W decoded row by row (fused route). */
void oracle_matvec(int kind, const uint8_t *W, int rows, int cols, const uint8_t *grid, const double *x,
                   double *y);

/* Router. */
double oracle_sqrtsoftplus(double z);
void oracle_router_logits(const double *x, int T, int H, const uint16_t *Wr, int E, double *z);
void oracle_select(const double *z, const float *bias, int T, int E, int k, double scaling, int32_t *idx,
                   double *w, double *margin);
/* Hash routing; returns 0, -1 (a token id outside [0, vocab)) or -2 (a used
 * table row with an id outside [0, n_experts) or a repeated id). */
int oracle_hash_select(const int32_t *token_ids, int T, const int32_t *tid2eid, int vocab, int n_experts, int k,
                       double scaling, int32_t *idx, double *w);

/* SwiGLU pieces. */
double oracle_silu(double u);
void oracle_swiglu_expert(int gate_kind, int down_kind, const uint8_t *gate, const uint8_t *up,
                          const uint8_t *down, int hidden, int inter, const uint8_t *grid, const double *x,
                          double *out);

/* One layer for T tokens given the routing.  gate/up/down are per-expert
 * pointers (NULL for experts no token selects). */
typedef struct {
  int hidden, inter, shared_inter, n_experts, top_k;
  const uint8_t *const *gate; /* [n_experts] -> [inter][hidden/256] blocks of gate_kind */
  const uint8_t *const *up;   /* [n_experts] -> [inter][hidden/256] blocks of gate_kind */
  const uint8_t *const *down; /* [n_experts] -> [hidden][inter/256] blocks of down_kind */
  const uint8_t *sh_gate;     /* Q8_0 [shared_inter][hidden/32][34] */
  const uint8_t *sh_up;       /* Q8_0 [shared_inter][hidden/32][34] */
  const uint8_t *sh_down;     /* Q8_0 [hidden][shared_inter/32][34] */
  const uint8_t *grid;        /* [256][8] */
  int gate_kind;              /* routed gate/up format: 0 IQ2_XXS (q2 build), 3 Q4_K (q2-q4 layers) */
  int down_kind;              /* routed down format: 1 Q2_K (q2 build), 3 Q4_K */
} oracle_layer_w;

int oracle_layer(const oracle_layer_w *Wt, const double *x, int T, const int32_t *idx, const double *w,
                 double *y);

/* oracle_layer with the tokens split over `nthreads` threads (same results). */
int oracle_layer_mt(const oracle_layer_w *Wt, const double *x, int T, const int32_t *idx, const double *w,
                    double *y, int nthreads);

/* Stable counting sort of the T*k (token, slot) pairs by expert. */
void oracle_permutation(const int32_t *idx, int T, int k, int E, int32_t *offsets, int32_t *perm);

/* x / sqrt(mean(x^2) + eps), unit gain. */
void oracle_rmsnorm(const double *x, int H, double eps, double *out);

/* Encoders (binary32 decisions, see oracle.c).  n is a multiple of the block
 * size (32 / 256 / 256); out receives n/32 34-byte, n/256 84-byte or n/256
 * 144-byte blocks.  Return 0, -1 for a non-finite input, -2 for a bad n. */
uint16_t oracle_f32_to_f16(float f);
int oracle_quantize_q80(const float *x, int n, uint8_t *out);
int oracle_quantize_q2k(const float *x, int n, uint8_t *out);
int oracle_quantize_q4k(const float *x, int n, uint8_t *out);

#ifdef __cplusplus
}
#endif
#endif
