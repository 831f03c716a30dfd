/*
 * oracle.c -- plain fp64 CPU oracle (TEST INFRASTRUCTURE; see oracle.h for the
 * source tags and who may call it).  Everything is scalar, row by row, in the
 * order the sources describe; there is no blocking or reordering beyond
 * decoding a row once and reusing it for every token that needs it.
 *
 * Parity status of each function: pinned by the not-gpu tests unless marked
 * "parity unpinned" below.  Parity unpinned: the IQ2_XXS group byte layout
 * and the (0.5 + s) / 4 group-scale constant, and the Q2_K nibble order and
 * min sign, are readings of structure-only descriptions; they are pinned to
 * those readings by hand-built blocks but not to any real GGUF file.
 */
#include "oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ f16 */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16(uint16_t bits) {
  int sign = (bits >> 15) & 1;
  int exp = (bits >> 10) & 0x1F;
  int frac = bits & 0x3FF;
  double v;
  if (exp == 0)
    v = ldexp((double)frac, -24); /* subnormal: frac * 2^-24 */
  else if (exp == 31)
    v = frac ? NAN : INFINITY;
  else
    v = ldexp(1.0 + (double)frac / 1024.0, exp - 15);
  return sign ? -v : v;
}

static uint16_t le16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static uint32_t le32(const uint8_t *p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}

/* -------------------------------------------------------------- IQ2_XXS */
/*
 * [QUANT] section 4: a 256-value block is eight 32-value groups; each group
 * has four 8-value grid indices and four 7-bit sign masks; the block scale is
 * f16 and each group refines it with a 4-bit scale nibble; values come from a
 * 256-entry grid of 8-tuples.  [QUANT] section 3 type table: 66 bytes per 256.
 * 2 + 8 * (4*8 + 4*7 + 4) / 8 = 66, so the listed fields fill the block.
 *
 * Reading (byte layout, parity unpinned against real files): bytes 0-1 hold d;
 * group g occupies bytes 2+8g .. 9+8g: bytes 0-3 are the grid indices of its
 * four 8-element sub-vectors, bytes 4-7 a little-endian word S whose bits
 * 7j..7j+6 are the sign mask of sub-vector j and whose bits 28-31 are the scale
 * nibble s.  The eighth sign of a sub-vector is the parity of its seven mask
 * bits, so every sub-vector has an even number of negative entries.
 * Value = d * (0.5 + s) / 4 * grid[idx][l] * (-1 if sign bit l set).
 */
double oracle_iq2xxs_elem(const uint8_t *blk, const uint8_t *grid, int e) {
  double d = oracle_f16(le16(blk));
  int g = e / 32;          /* group */
  int j = (e % 32) / 8;    /* sub-vector within the group */
  int l = e % 8;           /* lane within the 8-tuple */
  const uint8_t *grp = blk + 2 + 8 * g;
  int index = grp[j];
  uint32_t S = le32(grp + 4);
  int mask7 = (int)((S >> (7 * j)) & 0x7F);
  int ones = 0;
  for (int b = 0; b < 7; ++b) ones += (mask7 >> b) & 1;
  int mask8 = mask7 | ((ones & 1) << 7);
  int s = (int)(S >> 28);
  double value = d * (0.5 + (double)s) / 4.0 * (double)grid[8 * index + l];
  return ((mask8 >> l) & 1) ? -value : value;
}

void oracle_row_iq2xxs(const uint8_t *row, int cols, const uint8_t *grid, double *out) {
  for (int c = 0; c < cols; ++c) out[c] = oracle_iq2xxs_elem(row + (size_t)(c / 256) * 66, grid, c % 256);
}

/* ----------------------------------------------------------------- Q2_K */
/*
 * [QUANT] section 3: 256 values in 84 bytes; scales_off = 0 (16 bytes of
 * per-16-element scale/min nibbles), qs_off = 16 (64 bytes of 2-bit codes),
 * d_off = 80 (f16), dmin_off = 82 (f16).  The writer packs four codes per
 * byte as qs[j/4 + l] = L[j+l] | L[j+l+32] << 2 | L[j+l+64] << 4 | L[j+l+96] << 6
 * for l = 0..31 and j in {0, 128}; so element e sits in byte 32*(e/128) + e%32
 * at shift 2*((e%128)/32).  [FLOW] format paragraph: K-quants are affine with
 * a scale and a min per sub-block, roughly w = d*q + m.
 *
 * Reading (parity unpinned against real files): scale byte e/16 holds the
 * scale nibble in its low 4 bits and the min nibble in its high 4 bits, and
 * value = d * scale * q - dmin * min (the min is an offset below zero).
 */
double oracle_q2k_elem(const uint8_t *blk, int e) {
  const uint8_t *scales = blk;
  const uint8_t *qs = blk + 16;
  double d = oracle_f16(le16(blk + 80));
  double dmin = oracle_f16(le16(blk + 82));
  int half = e / 128;
  int r = e % 128;
  int q = (qs[32 * half + r % 32] >> (2 * (r / 32))) & 3;
  int sc = scales[e / 16] & 0xF;
  int mn = scales[e / 16] >> 4;
  return d * (double)sc * (double)q - dmin * (double)mn;
}

void oracle_row_q2k(const uint8_t *row, int cols, double *out) {
  for (int c = 0; c < cols; ++c) out[c] = oracle_q2k_elem(row + (size_t)(c / 256) * 84, c % 256);
}

/* ----------------------------------------------------------------- Q8_0 */
/*
 * [FLOW] format paragraph: Q8_0 is symmetric with one scale per 32-element
 * block; bit-allocation table: about 8.5 bpw, i.e. 34 bytes per 32.
 * Reading: f16 d in bytes 0-1, then 32 signed bytes; value = d * q.
 */
double oracle_q80_elem(const uint8_t *blk, int e) {
  double d = oracle_f16(le16(blk));
  return d * (double)(int8_t)blk[2 + e];
}

void oracle_row_q80(const uint8_t *row, int cols, double *out) {
  for (int c = 0; c < cols; ++c) out[c] = oracle_q80_elem(row + (size_t)(c / 32) * 34, c % 32);
}

/* ----------------------------------------------------------------- Q4_K */
/*
 * [QUANT] section 3 type table: q4_K holds 256 values in 144 bytes; [FLOW]
 * format paragraph: like Q2_K it is affine with a scale and a min per
 * sub-block (w = d*q + m roughly); [FLOW] bit-width table after "パラメータは
 * どこにあるか: 層別の内訳": about 4.5 bpw.  144 = 2 + 2 + 12 + 128 fits two f16
 * bases, eight 6-bit scales and eight 6-bit mins (8 sub-blocks of 32) and 256
 * 4-bit codes.
 *
 * Reading (the pages print no layout; this is the public GGUF Q4_K block, so
 * that real files decode unchanged; parity unpinned against real files):
 * bytes 0-1 d, bytes 2-3 dmin, bytes 4-15 the scales and mins, bytes 16-143
 * the codes.  Sub-block j < 4: scale = low 6 bits of scale byte j, min = low
 * 6 bits of scale byte j+4.  Sub-block j >= 4: scale = low nibble of scale
 * byte j+4 with the top two bits of scale byte j-4 above it, min = high
 * nibble of scale byte j+4 with the top two bits of scale byte j above it.
 * Element e lies in sub-block e/32; its code is in code byte 32*(e/64) + e%32,
 * low nibble for e%64 < 32 and high nibble otherwise (the two-codes-per-byte
 * form of the printed Q2_K packing).  Value = d * scale * q - dmin * min, the
 * same sign convention as Q2_K.
 */
static void q4k_scale_min(const uint8_t *sm, int j, int *scale, int *min) {
  if (j < 4) {
    *scale = sm[j] & 63;
    *min = sm[j + 4] & 63;
  } else {
    *scale = (sm[j + 4] & 15) | ((sm[j - 4] >> 6) << 4);
    *min = (sm[j + 4] >> 4) | ((sm[j] >> 6) << 4);
  }
}

double oracle_q4k_elem(const uint8_t *blk, int e) {
  double d = oracle_f16(le16(blk));
  double dmin = oracle_f16(le16(blk + 2));
  int scale, min;
  q4k_scale_min(blk + 4, e / 32, &scale, &min);
  int q = (blk[16 + 32 * (e / 64) + e % 32] >> (4 * ((e % 64) / 32))) & 15;
  return d * (double)scale * (double)q - dmin * (double)min;
}

void oracle_row_q4k(const uint8_t *row, int cols, double *out) {
  for (int c = 0; c < cols; ++c) out[c] = oracle_q4k_elem(row + (size_t)(c / 256) * 144, c % 256);
}

/* ------------------------------------------------------------- mat-vec */

static void decode_row(int kind, const uint8_t *row, int cols, const uint8_t *grid, double *out) {
  if (kind == 0)
    oracle_row_iq2xxs(row, cols, grid, out);
  else if (kind == 1)
    oracle_row_q2k(row, cols, out);
  else if (kind == 3)
    oracle_row_q4k(row, cols, out);
  else
    oracle_row_q80(row, cols, out);
}

static size_t row_bytes(int kind, int cols) {
  return kind == 0   ? (size_t)cols / 256 * 66
         : kind == 1 ? (size_t)cols / 256 * 84
         : kind == 3 ? (size_t)cols / 256 * 144
                     : (size_t)cols / 32 * 34;
}

void oracle_decode_matrix(int kind, const uint8_t *W, int rows, int cols, const uint8_t *grid, double *out) {
  size_t rb = row_bytes(kind, cols);
  for (int r = 0; r < rows; ++r) decode_row(kind, W + rb * (size_t)r, cols, grid, out + (size_t)r * cols);
}

void oracle_matvec(int kind, const uint8_t *W, int rows, int cols, const uint8_t *grid, const double *x,
                   double *y) {
  double *wrow = (double *)malloc(sizeof(double) * (size_t)cols);
  size_t rb = row_bytes(kind, cols);
  for (int r = 0; r < rows; ++r) {
    decode_row(kind, W + rb * (size_t)r, cols, grid, wrow);
    double acc = 0.0;
    for (int c = 0; c < cols; ++c) acc += wrow[c] * x[c];
    y[r] = acc;
  }
  free(wrow);
}

/* --------------------------------------------------------------- router */
/*
 * [FLOW] config table: router scoring "sqrtsoftplus + noaux_tc (bias load
 * balancing)", top-k 6, routed_scaling_factor 1.5.  [FLOW] MoE FFN section:
 * the hidden state goes through the F16 router linear layer (4096 x 256) to
 * one score per routed expert; the bias is added for the selection only and
 * is not part of the gate values; the top 6 are picked and their scores are
 * normalised (norm_topk_prob = true); y = shared(h) + 1.5 * sum g_i E_i(h).
 *
 * Readings: sqrtsoftplus(z) = sqrt(ln(1 + e^z)); no expert groups; equal keys
 * go to the lower expert id; the output ids are listed in ascending order.
 */
double oracle_sqrtsoftplus(double z) {
  double softplus = (z > 0.0 ? z : 0.0) + log1p(exp(-fabs(z)));
  return sqrt(softplus);
}

void oracle_router_logits(const double *x, int T, int H, const uint16_t *Wr, int E, double *z) {
  double *wrow = (double *)malloc(sizeof(double) * (size_t)H);
  for (int e = 0; e < E; ++e) {
    for (int c = 0; c < H; ++c) wrow[c] = oracle_f16(Wr[(size_t)e * H + c]);
    for (int t = 0; t < T; ++t) {
      double acc = 0.0;
      const double *xt = x + (size_t)t * H;
      for (int c = 0; c < H; ++c) acc += wrow[c] * xt[c];
      z[(size_t)t * E + e] = acc;
    }
  }
  free(wrow);
}

typedef struct {
  double key;
  int id;
} keyed;

static int by_key_desc_then_id(const void *a, const void *b) {
  const keyed *x = (const keyed *)a, *y = (const keyed *)b;
  if (x->key > y->key) return -1;
  if (x->key < y->key) return 1;
  return (x->id > y->id) - (x->id < y->id);
}

static int by_int(const void *a, const void *b) {
  int x = *(const int32_t *)a, y = *(const int32_t *)b;
  return (x > y) - (x < y);
}

void oracle_select(const double *z, const float *bias, int T, int E, int k, double scaling, int32_t *idx,
                   double *w, double *margin) {
  keyed *ks = (keyed *)malloc(sizeof(keyed) * (size_t)E);
  double *s = (double *)malloc(sizeof(double) * (size_t)E);
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      s[e] = oracle_sqrtsoftplus(z[(size_t)t * E + e]);
      ks[e].key = s[e] + (double)bias[e];
      ks[e].id = e;
    }
    qsort(ks, (size_t)E, sizeof(keyed), by_key_desc_then_id);
    int32_t *it = idx + (size_t)t * k;
    for (int i = 0; i < k; ++i) it[i] = ks[i].id;
    qsort(it, (size_t)k, sizeof(int32_t), by_int);
    double total = 0.0;
    for (int i = 0; i < k; ++i) total += s[it[i]];
    for (int i = 0; i < k; ++i) w[(size_t)t * k + i] = scaling * s[it[i]] / total;
    if (margin) margin[t] = (k < E) ? ks[k - 1].key - ks[k].key : INFINITY;
  }
  free(ks);
  free(s);
}

/*
 * [FLOW] MoE FFN section: layers 0-2 have no router; a static table
 * (tid2eid) maps the token id to expert ids.  Reading: the k table entries
 * each get weight scaling / k (uniform weights summing to the scaling).
 * A token id outside [0, vocab), or a table row (of a token in the call)
 * with an id outside [0, n_experts) or an id twice, names no set of k
 * distinct experts: the call returns -1 (token id) or -2 (table row) and
 * leaves that token's idx and w unset, as the CUDA layer reports such input
 * instead of computing with it.
 */
int oracle_hash_select(const int32_t *token_ids, int T, const int32_t *tid2eid, int vocab, int n_experts, int k,
                       double scaling, int32_t *idx, double *w) {
  int rc = 0;
  for (int t = 0; t < T; ++t) {
    const int tid = token_ids[t];
    if (tid < 0 || tid >= vocab) {
      rc = -1;
      continue;
    }
    const int32_t *row = tid2eid + (size_t)tid * k;
    int ok = 1;
    for (int i = 0; i < k; ++i) {
      if (row[i] < 0 || row[i] >= n_experts) ok = 0;
      for (int j = 0; j < i; ++j)
        if (row[j] == row[i]) ok = 0;
    }
    if (!ok) {
      if (rc == 0) rc = -2;
      continue;
    }
    int32_t *it = idx + (size_t)t * k;
    for (int i = 0; i < k; ++i) it[i] = row[i];
    qsort(it, (size_t)k, sizeof(int32_t), by_int);
    for (int i = 0; i < k; ++i) w[(size_t)t * k + i] = scaling / (double)k;
  }
  return rc;
}

/* --------------------------------------------------------------- SwiGLU */
/*
 * [FLOW] MoE FFN section: E(h) = W_down (SiLU(W_gate h) ⊙ (W_up h)),
 * 4096 -> 2048 -> 4096; the shared expert has the same SwiGLU structure.
 * SiLU(u) = u / (1 + e^-u) (textbook).
 */
double oracle_silu(double u) { return u / (1.0 + exp(-u)); }

void oracle_swiglu_expert(int gate_kind, int down_kind, const uint8_t *gate, const uint8_t *up,
                          const uint8_t *down, int hidden, int inter, const uint8_t *grid, const double *x,
                          double *out) {
  double *a = (double *)malloc(sizeof(double) * (size_t)inter);
  double *b = (double *)malloc(sizeof(double) * (size_t)inter);
  oracle_matvec(gate_kind, gate, inter, hidden, grid, x, a);
  oracle_matvec(gate_kind, up, inter, hidden, grid, x, b);
  for (int i = 0; i < inter; ++i) a[i] = oracle_silu(a[i]) * b[i];
  oracle_matvec(down_kind, down, hidden, inter, grid, a, out);
  free(a);
  free(b);
}

/* ---------------------------------------------------------------- layer */
/*
 * y[t] = shared(x[t]) + sum over the k selected experts, in ascending expert
 * id, of w[t][i] * E_idx[t][i](x[t])   ([FLOW] MoE FFN section).  Experts are
 * visited in ascending id; each decoded row is applied to every token that
 * selected the expert, which changes no arithmetic.
 */
int oracle_layer(const oracle_layer_w *W, const double *x, int T, const int32_t *idx, const double *w,
                 double *y) {
  const int H = W->hidden, I = W->inter, Is = W->shared_inter, E = W->n_experts, k = W->top_k;
  for (int t = 0; t < T; ++t)
    oracle_swiglu_expert(2, 2, W->sh_gate, W->sh_up, W->sh_down, H, Is, W->grid, x + (size_t)t * H,
                         y + (size_t)t * H);

  int *tok = (int *)malloc(sizeof(int) * (size_t)(T > 0 ? T : 1));
  int *slot = (int *)malloc(sizeof(int) * (size_t)(T > 0 ? T : 1));
  double *wrow = (double *)malloc(sizeof(double) * (size_t)(H > I ? H : I));
  for (int e = 0; e < E; ++e) {
    int n = 0;
    for (int t = 0; t < T; ++t)
      for (int i = 0; i < k; ++i)
        if (idx[(size_t)t * k + i] == e) {
          tok[n] = t;
          slot[n] = i;
          ++n;
        }
    if (n == 0) continue;
    if (!W->gate[e] || !W->up[e] || !W->down[e]) {
      free(tok);
      free(slot);
      free(wrow);
      return -1;
    }
    double *a = (double *)calloc((size_t)n * I, sizeof(double));
    double *b = (double *)calloc((size_t)n * I, sizeof(double));
    size_t rg = row_bytes(W->gate_kind, H), rd = row_bytes(W->down_kind, I);
    for (int r = 0; r < I; ++r) {
      decode_row(W->gate_kind, W->gate[e] + rg * (size_t)r, H, W->grid, wrow);
      for (int m = 0; m < n; ++m) {
        const double *xt = x + (size_t)tok[m] * H;
        double acc = 0.0;
        for (int c = 0; c < H; ++c) acc += wrow[c] * xt[c];
        a[(size_t)m * I + r] = acc;
      }
      decode_row(W->gate_kind, W->up[e] + rg * (size_t)r, H, W->grid, wrow);
      for (int m = 0; m < n; ++m) {
        const double *xt = x + (size_t)tok[m] * H;
        double acc = 0.0;
        for (int c = 0; c < H; ++c) acc += wrow[c] * xt[c];
        b[(size_t)m * I + r] = acc;
      }
    }
    for (size_t q = 0; q < (size_t)n * I; ++q) a[q] = oracle_silu(a[q]) * b[q];
    for (int r = 0; r < H; ++r) {
      decode_row(W->down_kind, W->down[e] + rd * (size_t)r, I, W->grid, wrow);
      for (int m = 0; m < n; ++m) {
        const double *h = a + (size_t)m * I;
        double acc = 0.0;
        for (int c = 0; c < I; ++c) acc += wrow[c] * h[c];
        y[(size_t)tok[m] * H + r] += w[(size_t)tok[m] * k + slot[m]] * acc;
      }
    }
    free(a);
    free(b);
  }
  free(tok);
  free(slot);
  free(wrow);
  return 0;
}

/* The same layer with the tokens split over threads; every token's arithmetic
 * is exactly that of oracle_layer (tokens are independent). */
typedef struct {
  const oracle_layer_w *W;
  const double *x;
  int T;
  const int32_t *idx;
  const double *w;
  double *y;
  int rc;
} layer_job;

static void *layer_job_run(void *arg) {
  layer_job *j = (layer_job *)arg;
  j->rc = oracle_layer(j->W, j->x, j->T, j->idx, j->w, j->y);
  return NULL;
}

int oracle_layer_mt(const oracle_layer_w *W, const double *x, int T, const int32_t *idx, const double *w, double *y,
                    int nthreads) {
  if (nthreads <= 1 || T <= 1) return oracle_layer(W, x, T, idx, w, y);
  if (nthreads > T) nthreads = T;
  if (nthreads > 64) nthreads = 64;
  pthread_t th[64];
  layer_job jobs[64];
  const int H = W->hidden, k = W->top_k;
  int t0 = 0;
  for (int i = 0; i < nthreads; ++i) {
    const int n = T / nthreads + (i < T % nthreads);
    jobs[i].W = W;
    jobs[i].x = x + (size_t)t0 * H;
    jobs[i].T = n;
    jobs[i].idx = idx + (size_t)t0 * k;
    jobs[i].w = w + (size_t)t0 * k;
    jobs[i].y = y + (size_t)t0 * H;
    jobs[i].rc = 0;
    pthread_create(&th[i], NULL, layer_job_run, &jobs[i]);
    t0 += n;
  }
  int rc = 0;
  for (int i = 0; i < nthreads; ++i) {
    pthread_join(th[i], NULL);
    if (jobs[i].rc) rc = jobs[i].rc;
  }
  return rc;
}

/* ---------------------------------------------------------- permutation */
/*
 * Grouping tokens by expert for the batched path: offsets[e] is the number
 * of (token, slot) pairs routed to experts below e (offsets[E] = T*k), and
 * perm lists, for each expert in turn, the pairs t*k + slot in ascending
 * order of t (a stable counting sort).
 */
void oracle_permutation(const int32_t *idx, int T, int k, int E, int32_t *offsets, int32_t *perm) {
  int pos = 0;
  for (int e = 0; e < E; ++e) {
    offsets[e] = pos;
    for (int t = 0; t < T; ++t)
      for (int i = 0; i < k; ++i)
        if (idx[(size_t)t * k + i] == e) perm[pos++] = t * k + i;
  }
  offsets[E] = pos;
}

/* -------------------------------------------------------------- RMSNorm */
/* [ARCH] RMSNorm section names the root-mean-square scale; textbook form
 * x / sqrt(mean(x^2) + eps) with unit gain. */
void oracle_rmsnorm(const double *x, int H, double eps, double *out) {
  double ss = 0.0;
  for (int c = 0; c < H; ++c) ss += x[c] * x[c];
  double inv = 1.0 / sqrt(ss / (double)H + eps);
  for (int c = 0; c < H; ++c) out[c] = x[c] * inv;
}

/* ------------------------------------------------------------- encoders */
/*
 * The encoder side of the two scalar block formats.  [QUANT] section 3: the
 * Q2_K writer estimates a scale and a min for every 16-element sub-block,
 * rounds each value to a 2-bit code 0..3 and packs four codes per byte with
 * the printed expression (code of element e at byte 32*(e/128) + e%32, shift
 * 2*((e%128)/32)); d at byte 80 and dmin at 82 are the f16 bases of the
 * sub-block scale and min nibbles.  [FLOW] "Dwarf Star の量子化の工夫": Q8_0
 * keeps one symmetric scale per 32 elements.
 *
 * Readings (the pages give neither the estimator nor a precision): plain
 * min/max estimation; every decision in IEEE binary32 with round-to-nearest-
 * even, in the order written below (the arithmetic a device encoder uses, so
 * both take each integer decision in the same precision); the f16 bases are
 * the nearest binary16 values; a block holding a non-finite value is an
 * error.  The decoded value is the one the decoders above compute:
 * Q8_0 d*q, Q2_K d*sc*q - dmin*m.
 */

/* Nearest IEEE binary16 (ties to even) of a binary32 value, from the format's
 * definition: 10 fraction bits, exponent bias 15, subnormal quantum 2^-24,
 * values at or above 65520 (the midpoint past 65504) go to infinity. */
uint16_t oracle_f32_to_f16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  const uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  const float a = fabsf(f);
  if (isnan(f)) return (uint16_t)(sign | 0x7e00u);
  if (a >= 65520.0f) return (uint16_t)(sign | 0x7c00u);
  if (a == 0.0f) return sign;
  int e;
  frexp((double)a, &e); /* a = m 2^e, m in [0.5, 1): the binade's exponent is e - 1 */
  int ex = e - 1;
  if (ex < -14) ex = -14;                     /* subnormal binade: quantum 2^-24 */
  const double quantum = ldexp(1.0, ex - 10); /* spacing of binary16 values there */
  const double r = nearbyint((double)a / quantum); /* exact quotient; ties to even */
  uint32_t bits;
  if (ex == -14 && r < 1024.0) {
    bits = (uint32_t)r; /* subnormal */
  } else {
    double m = r;
    if (m >= 2048.0) { /* rounded up into the next binade */
      m = 1024.0;
      ex += 1;
    }
    bits = ((uint32_t)(ex + 15) << 10) | ((uint32_t)m - 1024u);
  }
  return (uint16_t)(sign | bits);
}

static void put16(uint8_t *p, uint16_t v) {
  p[0] = (uint8_t)(v & 0xff);
  p[1] = (uint8_t)(v >> 8);
}

static float clampf(float v, float lo, float hi) { return v < lo ? lo : v > hi ? hi : v; }

int oracle_quantize_q80(const float *x, int n, uint8_t *out) {
  if (n < 0 || n % 32) return -2;
  for (int b = 0; b < n / 32; ++b) {
    const float *v = x + (size_t)b * 32;
    uint8_t *blk = out + (size_t)b * 34;
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) {
      if (!isfinite(v[i])) return -1;
      if (fabsf(v[i]) > amax) amax = fabsf(v[i]);
    }
    const float d = amax / 127.0f;
    const uint16_t dh = oracle_f32_to_f16(d);
    const float dq = (float)oracle_f16(dh);
    put16(blk, dh);
    for (int i = 0; i < 32; ++i) {
      float q = 0.0f;
      if (dq > 0.0f) q = clampf(rintf(v[i] / dq), -127.0f, 127.0f);
      blk[2 + i] = (uint8_t)(int8_t)q;
    }
  }
  return 0;
}

int oracle_quantize_q2k(const float *x, int n, uint8_t *out) {
  if (n < 0 || n % 256) return -2;
  for (int b = 0; b < n / 256; ++b) {
    const float *v = x + (size_t)b * 256;
    uint8_t *blk = out + (size_t)b * 84;
    memset(blk, 0, 84);
    float scale[16], mn[16], maxs = 0.0f, maxm = 0.0f;
    for (int j = 0; j < 16; ++j) {
      /* the sub-block's range, widened to include 0 below: the min term
       * -dmin*m is never positive */
      float lo = 0.0f, hi = -INFINITY;
      for (int i = 0; i < 16; ++i) {
        const float t = v[16 * j + i];
        if (!isfinite(t)) return -1;
        if (t < lo) lo = t;
        if (t > hi) hi = t;
      }
      scale[j] = (hi - lo) / 3.0f; /* four codes span the range */
      mn[j] = 0.0f - lo;
      if (scale[j] > maxs) maxs = scale[j];
      if (mn[j] > maxm) maxm = mn[j];
    }
    const uint16_t dh = oracle_f32_to_f16(maxs / 15.0f), mh = oracle_f32_to_f16(maxm / 15.0f);
    const float dq = (float)oracle_f16(dh), mq = (float)oracle_f16(mh);
    put16(blk + 80, dh);
    put16(blk + 82, mh);
    for (int j = 0; j < 16; ++j) {
      const float sc = dq > 0.0f ? clampf(rintf(scale[j] / dq), 0.0f, 15.0f) : 0.0f;
      const float m = mq > 0.0f ? clampf(rintf(mn[j] / mq), 0.0f, 15.0f) : 0.0f;
      blk[j] = (uint8_t)((int)sc | ((int)m << 4));
      const float step = dq * sc, off = mq * m;
      for (int i = 0; i < 16; ++i) {
        const int e = 16 * j + i;
        float q = 0.0f;
        if (step > 0.0f) q = clampf(rintf((v[e] + off) / step), 0.0f, 3.0f);
        blk[16 + 32 * (e / 128) + e % 32] |= (uint8_t)((int)q << (2 * ((e % 128) / 32)));
      }
    }
  }
  return 0;
}

/*
 * Q4_K encoder: the same estimator one level up (reading, as for Q2_K): for
 * every 32-value sub-block j, lo = min(0, min x), hi = max x, scale = (hi -
 * lo) / 15 (sixteen codes span the range), min = 0 - lo; d = f16(max scale /
 * 63) and dmin = f16(max min / 63); sc = clamp(rint(scale / d), 0, 63), m =
 * clamp(rint(min / dmin), 0, 63); q = clamp(rint((x + dmin*m) / (d*sc)), 0, 15);
 * packed in the Q4_K layout read above.  Decisions in binary32, ties to even.
 */
int oracle_quantize_q4k(const float *x, int n, uint8_t *out) {
  if (n < 0 || n % 256) return -2;
  for (int b = 0; b < n / 256; ++b) {
    const float *v = x + (size_t)b * 256;
    uint8_t *blk = out + (size_t)b * 144;
    memset(blk, 0, 144);
    float scale[8], mn[8], maxs = 0.0f, maxm = 0.0f;
    for (int j = 0; j < 8; ++j) {
      float lo = 0.0f, hi = -INFINITY;
      for (int i = 0; i < 32; ++i) {
        const float t = v[32 * j + i];
        if (!isfinite(t)) return -1;
        if (t < lo) lo = t;
        if (t > hi) hi = t;
      }
      scale[j] = (hi - lo) / 15.0f;
      mn[j] = 0.0f - lo;
      if (scale[j] > maxs) maxs = scale[j];
      if (mn[j] > maxm) maxm = mn[j];
    }
    const uint16_t dh = oracle_f32_to_f16(maxs / 63.0f), mh = oracle_f32_to_f16(maxm / 63.0f);
    const float dq = (float)oracle_f16(dh), mq = (float)oracle_f16(mh);
    put16(blk, dh);
    put16(blk + 2, mh);
    uint8_t *sm = blk + 4;
    for (int j = 0; j < 8; ++j) {
      const float sc = dq > 0.0f ? clampf(rintf(scale[j] / dq), 0.0f, 63.0f) : 0.0f;
      const float m = mq > 0.0f ? clampf(rintf(mn[j] / mq), 0.0f, 63.0f) : 0.0f;
      const int isc = (int)sc, im = (int)m;
      if (j < 4) {
        sm[j] |= (uint8_t)isc;
        sm[j + 4] |= (uint8_t)im;
      } else {
        sm[j + 4] |= (uint8_t)((isc & 15) | ((im & 15) << 4));
        sm[j - 4] |= (uint8_t)((isc >> 4) << 6);
        sm[j] |= (uint8_t)((im >> 4) << 6);
      }
      const float step = dq * sc, off = mq * m;
      for (int i = 0; i < 32; ++i) {
        const int e = 32 * j + i;
        float q = 0.0f;
        if (step > 0.0f) q = clampf(rintf((v[e] + off) / step), 0.0f, 15.0f);
        blk[16 + 32 * (e / 64) + e % 32] |= (uint8_t)((int)q << (4 * ((e % 64) / 32)));
      }
    }
  }
  return 0;
}
