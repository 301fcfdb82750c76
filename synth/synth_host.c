/* Host side of the seeded input generator (see synth_gen.h). */
#include <stdlib.h>
#include <string.h>
#include "synth_gen.h"

void synth_philox(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  synth_philox4x32_10(ctr, key, out);
}

double synth_normal_at(uint64_t seed, uint32_t purpose, uint32_t tag, uint64_t e, uint32_t j) {
  return synth_normal(seed, synth_stream(purpose, tag), e, j);
}

/* Fill rows [row0, row0 + nrows) of a (.. x cols) tensor into out (nrows x cols,
 * row-major), as binary32 or bfloat16 bits. */
int synth_fill_rows(void* out, int out_dtype, int64_t cols, int64_t row0, int64_t nrows,
                    uint64_t seed, uint32_t tag, const synth_dist* d) {
  if (!out || cols <= 0 || nrows < 0 || !d) return 1;
  #pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < nrows; r++) {
    int64_t row = row0 + r;
    double rowf = synth_row_factor(seed, tag, (uint64_t)row, d->row_sigma);
    for (int64_t c = 0; c < cols; c++) {
      float f = synth_round_f32(synth_value(seed, tag, cols, row, c, d, rowf));
      if (out_dtype == SYNTH_OUT_BF16) ((uint16_t*)out)[r * cols + c] = synth_f32_to_bf16(f);
      else ((float*)out)[r * cols + c] = f;
    }
  }
  return 0;
}

/* Fill an arbitrary list of rows (row indices in rows[]) into out (n x cols). */
int synth_fill_row_list(void* out, int out_dtype, int64_t cols, const int64_t* rows, int64_t n,
                        uint64_t seed, uint32_t tag, const synth_dist* d) {
  if (!out || cols <= 0 || n < 0 || !d || (n > 0 && !rows)) return 1;
  #pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n; r++) {
    int64_t row = rows[r];
    double rowf = synth_row_factor(seed, tag, (uint64_t)row, d->row_sigma);
    for (int64_t c = 0; c < cols; c++) {
      float f = synth_round_f32(synth_value(seed, tag, cols, row, c, d, rowf));
      if (out_dtype == SYNTH_OUT_BF16) ((uint16_t*)out)[r * cols + c] = synth_f32_to_bf16(f);
      else ((float*)out)[r * cols + c] = f;
    }
  }
  return 0;
}

typedef struct { uint64_t key; int64_t idx; } synth_kv;

static int kv_cmp(const void* a, const void* b) {
  const synth_kv* x = (const synth_kv*)a; const synth_kv* y = (const synth_kv*)b;
  if (x->key != y->key) return x->key < y->key ? -1 : 1;
  return x->idx < y->idx ? -1 : (x->idx > y->idx);
}

/* Uniform sample of k distinct items from [0, n) without replacement: the
 * items with the k smallest sampling keys, returned in key order (ties of
 * the 64-bit key broken by item index). */
int synth_sample(uint64_t seed, uint32_t tag, int64_t n, int64_t k, int64_t* out) {
  if (k < 0 || k > n || (k > 0 && !out)) return 1;
  if (k == 0) return 0;
  /* keep the k smallest in a max-heap */
  synth_kv* heap = (synth_kv*)malloc(sizeof(synth_kv) * (size_t)k);
  if (!heap) return 2;
  int64_t sz = 0;
  for (int64_t i = 0; i < n; i++) {
    synth_kv it = {synth_sample_key(seed, tag, (uint64_t)i), i};
    if (sz < k) {
      int64_t c = sz++;
      heap[c] = it;
      while (c > 0) {
        int64_t p = (c - 1) / 2;
        if (kv_cmp(&heap[p], &heap[c]) >= 0) break;
        synth_kv t = heap[p]; heap[p] = heap[c]; heap[c] = t; c = p;
      }
    } else if (kv_cmp(&it, &heap[0]) < 0) {
      heap[0] = it;
      int64_t c = 0;
      for (;;) {
        int64_t l = 2 * c + 1, r = l + 1, m = c;
        if (l < sz && kv_cmp(&heap[l], &heap[m]) > 0) m = l;
        if (r < sz && kv_cmp(&heap[r], &heap[m]) > 0) m = r;
        if (m == c) break;
        synth_kv t = heap[m]; heap[m] = heap[c]; heap[c] = t; c = m;
      }
    }
  }
  qsort(heap, (size_t)sz, sizeof(synth_kv), kv_cmp);
  for (int64_t i = 0; i < k; i++) out[i] = heap[i].idx;
  free(heap);
  return 0;
}
