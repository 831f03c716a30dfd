/*
 * synth_host.c -- host fills built on synth.h (shared library for ctypes).
 *
 * Each fill writes the canonical layout the layer's boundary takes:
 *   routed IQ2_XXS / Q2_K / Q4_K tensors: [expert][row][block], experts
 *   [expert_begin, expert_begin + n_experts) of the tensor;
 *   shared Q8_0 tensors: [row][block].
 * Threads split the work by expert or row only; every byte is a pure
 * function of (seed, layer, tensor, block index), so the thread count never
 * changes the output.
 */
#include <pthread.h>
#include <stdlib.h>
#include "synth.h"

typedef struct {
  uint64_t key;
  uint64_t first_block;
  uint64_t n_blocks;
  int kind; /* 0 iq2xxs, 1 q2k, 2 q80, 3 q4k */
  uint8_t *out;
} fill_job;

static void *fill_run(void *arg) {
  fill_job *j = (fill_job *)arg;
  for (uint64_t b = 0; b < j->n_blocks; ++b) {
    uint64_t gb = j->first_block + b;
    if (j->kind == 0)
      synth_iq2xxs_block(j->key, gb, j->out + b * SYNTH_IQ2XXS_BYTES);
    else if (j->kind == 1)
      synth_q2k_block(j->key, gb, j->out + b * SYNTH_Q2K_BYTES);
    else if (j->kind == 3)
      synth_q4k_block(j->key, gb, j->out + b * SYNTH_Q4K_BYTES);
    else
      synth_q80_block(j->key, gb, j->out + b * SYNTH_Q80_BYTES);
  }
  return NULL;
}

static void fill_blocks(uint64_t key, uint64_t first, uint64_t n, int kind, uint8_t *out, int threads) {
  const uint64_t bytes[4] = {SYNTH_IQ2XXS_BYTES, SYNTH_Q2K_BYTES, SYNTH_Q80_BYTES, SYNTH_Q4K_BYTES};
  if (threads < 1) threads = 1;
  if (threads > 64) threads = 64;
  if (n < 4096) threads = 1;
  pthread_t tid[64];
  fill_job jobs[64];
  uint64_t per = (n + (uint64_t)threads - 1) / (uint64_t)threads;
  int started = 0;
  for (int t = 0; t < threads; ++t) {
    uint64_t b0 = per * (uint64_t)t;
    if (b0 >= n) break;
    uint64_t nb = (b0 + per > n) ? n - b0 : per;
    jobs[t].key = key;
    jobs[t].first_block = first + b0;
    jobs[t].n_blocks = nb;
    jobs[t].kind = kind;
    jobs[t].out = out + b0 * bytes[kind];
    if (threads == 1) {
      fill_run(&jobs[t]);
    } else {
      pthread_create(&tid[t], NULL, fill_run, &jobs[t]);
      started++;
    }
  }
  for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
}

/* Routed expert tensor, experts [e0, e0 + ne), rows x cols each. */
void synth_fill_routed(uint64_t seed, uint32_t layer, uint32_t tensor, int kind, int e0, int ne, int rows,
                       int cols, uint8_t *out, int threads) {
  uint64_t bpr = (uint64_t)cols / (kind == 2 ? 32u : 256u);
  uint64_t per_expert = (uint64_t)rows * bpr;
  fill_blocks(synth_key(seed, layer, tensor), (uint64_t)e0 * per_expert, (uint64_t)ne * per_expert, kind, out,
              threads);
}

void synth_fill_grid(uint64_t seed, uint32_t layer, uint8_t *out) {
  uint64_t key = synth_key(seed, layer, SYNTH_T_GRID);
  for (uint32_t r = 0; r < 256; ++r)
    for (uint32_t l = 0; l < 8; ++l) out[8 * r + l] = synth_grid_entry(key, r, l);
}

void synth_fill_bias(uint64_t seed, uint32_t layer, int n_experts, int skew, float *out) {
  uint64_t key = synth_key(seed, layer, SYNTH_T_BIAS);
  for (int e = 0; e < n_experts; ++e) out[e] = synth_bias(key, (uint32_t)e, skew);
}

void synth_fill_tid2eid(uint64_t seed, uint32_t layer, int vocab, int n_experts, int k, int32_t *out) {
  uint64_t key = synth_key(seed, layer, SYNTH_T_TID2EID);
  for (int v = 0; v < vocab; ++v) synth_tid2eid_row(key, (uint32_t)v, n_experts, k, out + (size_t)v * k);
}

uint16_t synth_f16_of(float f) { return synth_f16_bits(f); }
