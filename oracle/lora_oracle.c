/* lora_oracle.c -- plain CPU oracle of the chunked-SGMV LoRA shrink/expand pair.
 *
 * TEST INFRASTRUCTURE ONLY (see lora_oracle.h).  Deliberately slow and
 * literal: a loop over segments, then over the rows of the segment, then over
 * the outputs, with the sum written out term by term.  No blocking, no
 * vectorisation, no reordering.  The only parallelism is OpenMP over the rows
 * of a segment, which does not change any arithmetic.
 *
 * Sources for what is computed:
 *  - sgl-kernel-xpu "Decode LoRA kernels are optimized", section "Summary"
 *    (shrink = gather x rows through the permutation, multiply each segment by
 *    its adapter's A; expand = multiply by the adapter's B, scale, scatter-add
 *    into the base output's column slices) and section "Behaviour changes"
 *    (the tables: seg_indptr, adapter index range, permutation, offset table).
 *  - ms-swift "Add optional fast lora path for qwen2/qwen3 on npu", section
 *    "Compatibility checks" (dropout 0, one active adapter: the update is
 *    scaling * (x A^T) B^T with no other term).
 * Readings where the pages are silent are listed in the design notes; the
 * ones that shape this file: rank activations are stored in sorted order
 * (row i belongs to token permutation[i]); slice q of the rank activations
 * is columns [q*rs, q*rs + r); a zero scaling skips the segment.
 */
#include "lora_oracle.h"

#include <omp.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- codec */

float oracle_decode(uint16_t h, int dtype) {
  if (dtype == ORACLE_BF16) {
    /* bf16 is the top half of an IEEE binary32 */
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
  }
  _Float16 v;
  memcpy(&v, &h, sizeof v);
  return (float)v;
}

/* round to nearest, ties to even, via the compiler's IEEE conversions */
uint16_t oracle_encode(float f, int dtype) {
  uint16_t h;
  if (dtype == ORACLE_BF16) {
    __bf16 b = (__bf16)f;
    memcpy(&h, &b, sizeof h);
  } else {
    _Float16 v = (_Float16)f;
    memcpy(&h, &v, sizeof h);
  }
  return h;
}

uint16_t oracle_encode_f64(double d, int dtype) {
  uint16_t h;
  if (dtype == ORACLE_BF16) {
    __bf16 b = (__bf16)d;
    memcpy(&h, &b, sizeof h);
  } else {
    _Float16 v = (_Float16)d;
    memcpy(&h, &v, sizeof h);
  }
  return h;
}

/* ---------------------------------------------------------------- tables */

int oracle_check_tables(const int32_t* seg_indptr, const int32_t* weight_indices,
                        const int32_t* permutation, const int32_t* slice_offsets,
                        int tok, int nseg, int L, int S, int64_t ld_base) {
  int bad = 0;
  if (tok < 0 || nseg < 0 || L < 1 || S < 1) return ORACLE_BAD_DIMS;

  for (int s = 0; s <= nseg; ++s) {
    if (seg_indptr[s] < 0 || seg_indptr[s] > tok) bad |= ORACLE_BAD_INDPTR;
    if (s > 0 && seg_indptr[s] < seg_indptr[s - 1]) bad |= ORACLE_BAD_INDPTR;
  }
  for (int s = 0; s < nseg; ++s)
    if (weight_indices[s] < 0 || weight_indices[s] >= L) bad |= ORACLE_BAD_ADAPTER;

  if (tok > 0) {
    unsigned char* seen = (unsigned char*)calloc((size_t)tok, 1);
    for (int i = 0; i < tok; ++i) {
      int32_t t = permutation[i];
      if (t < 0 || t >= tok || seen[t]) {
        bad |= ORACLE_BAD_PERMUTATION;
      } else {
        seen[t] = 1;
      }
    }
    free(seen);
  }

  if (slice_offsets) {
    for (int q = 0; q <= S; ++q) {
      if (slice_offsets[q] < 0 || slice_offsets[q] > ld_base) bad |= ORACLE_BAD_SLICES;
      if (q > 0 && slice_offsets[q] < slice_offsets[q - 1]) bad |= ORACLE_BAD_SLICES;
    }
  }
  return bad;
}

/* ---------------------------------------------------------------- shrink */

int oracle_shrink(const uint16_t* x, int64_t ld_x, const uint16_t* A_stack,
                  const int32_t* seg_indptr, const int32_t* weight_indices,
                  const int32_t* permutation, void* out_r, int64_t ld_out,
                  int tok, int K, int S, int r, int rs, int nseg, int L,
                  int dtype, int mode) {
  if (K < 1 || r < 1 || rs < r || ld_x < K || ld_out < (int64_t)S * rs ||
      (mode != ORACLE_F32 && mode != ORACLE_F64))
    return ORACLE_BAD_DIMS;
  int bad = oracle_check_tables(seg_indptr, weight_indices, permutation, NULL,
                                tok, nseg, L, S, 0);
  if (bad) return bad;

  const int64_t a_rows = (int64_t)S * rs; /* rows of one adapter's stacked A */

#pragma omp parallel
  for (int s = 0; s < nseg; ++s) {
    const int a = weight_indices[s];
    const int lo = seg_indptr[s], hi = seg_indptr[s + 1];
    const uint16_t* A = A_stack + (int64_t)a * a_rows * K;

#pragma omp for schedule(static) nowait
    for (int i = lo; i < hi; ++i) {
      const uint16_t* xrow = x + (int64_t)permutation[i] * ld_x;
      for (int q = 0; q < S; ++q) {
        for (int j = 0; j < r; ++j) {
          const int64_t n = (int64_t)q * rs + j;
          const uint16_t* arow = A + n * K;
          if (mode == ORACLE_F32) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k)
              acc += oracle_decode(xrow[k], dtype) * oracle_decode(arow[k], dtype);
            ((uint16_t*)out_r)[(int64_t)i * ld_out + n] = oracle_encode(acc, dtype);
          } else {
            double acc = 0.0;
            for (int k = 0; k < K; ++k)
              acc += (double)oracle_decode(xrow[k], dtype) * (double)oracle_decode(arow[k], dtype);
            ((double*)out_r)[(int64_t)i * ld_out + n] = acc;
          }
        }
      }
    }
  }
  return 0;
}

/* ---------------------------------------------------------------- expand */

int oracle_expand(const void* in_r, int64_t ld_in, const uint16_t* B_stack,
                  const int32_t* seg_indptr, const int32_t* weight_indices,
                  const int32_t* permutation, const int32_t* slice_offsets,
                  const float* scalings, void* base_out, int64_t ld_base,
                  int tok, int S, int r, int rs, int nseg, int L,
                  int dtype, int mode) {
  if (r < 1 || rs < r || ld_in < (int64_t)S * rs ||
      (mode != ORACLE_F32 && mode != ORACLE_F64 && mode != ORACLE_F64_IN))
    return ORACLE_BAD_DIMS;
  int bad = oracle_check_tables(seg_indptr, weight_indices, permutation, slice_offsets,
                                tok, nseg, L, S, ld_base);
  if (bad) return bad;

  const int64_t n_tot = (int64_t)slice_offsets[S] - slice_offsets[0];

#pragma omp parallel
  for (int s = 0; s < nseg; ++s) {
    const int a = weight_indices[s];
    const float scaling = scalings[a];
    const int lo = seg_indptr[s], hi = seg_indptr[s + 1];
    const uint16_t* B = B_stack + (int64_t)a * n_tot * rs;
    if (scaling == 0.0f) continue; /* a zero scaling leaves the segment untouched */

#pragma omp for schedule(static) nowait
    for (int i = lo; i < hi; ++i) {
      const int64_t t = permutation[i];
      for (int q = 0; q < S; ++q) {
        for (int64_t c = slice_offsets[q]; c < slice_offsets[q + 1]; ++c) {
          const uint16_t* brow = B + (c - slice_offsets[0]) * rs;
          if (mode == ORACLE_F32) {
            const uint16_t* v = (const uint16_t*)in_r + (int64_t)i * ld_in + (int64_t)q * rs;
            float acc = 0.0f;
            for (int j = 0; j < r; ++j)
              acc += oracle_decode(v[j], dtype) * oracle_decode(brow[j], dtype);
            uint16_t* o = (uint16_t*)base_out + t * ld_base + c;
            float prod = scaling * acc;
            float sum = oracle_decode(*o, dtype) + prod;
            *o = oracle_encode(sum, dtype);
          } else {
            double acc = 0.0;
            for (int j = 0; j < r; ++j) {
              double v;
              if (mode == ORACLE_F64_IN)
                v = ((const double*)in_r)[(int64_t)i * ld_in + (int64_t)q * rs + j];
              else
                v = (double)oracle_decode(((const uint16_t*)in_r)[(int64_t)i * ld_in + (int64_t)q * rs + j], dtype);
              acc += v * (double)oracle_decode(brow[j], dtype);
            }
            double* o = (double*)base_out + t * ld_base + c;
            *o = *o + (double)scaling * acc;
          }
        }
      }
    }
  }
  return 0;
}

/* ---------------------------------------------------------------- embedding A */

/* ---------------------------------------------------------------- base projection + expand
 *
 * The expand folded into the base projection that produces its output: on the
 * sglang page "fused split_qkv / norm / RoPE for Qwen3.5/Next on NPU" (section
 * of key source snippets, forward_prepare_npu) the qkv_proj output goes
 * straight to the split step, and with LoRA the expand rewrites that output
 * first.  The base sum over K and the rank sum over r are kept apart and
 * combined once, as base + scaling * lora, then rounded. */
int oracle_base_expand(const uint16_t* x, int64_t ld_x, const uint16_t* W, int64_t ld_w,
                       const uint16_t* in_r, int64_t ld_in, const uint16_t* B_stack,
                       const int32_t* seg_indptr, const int32_t* weight_indices,
                       const int32_t* permutation, const int32_t* slice_offsets,
                       const float* scalings, void* out, int64_t ld_out, int tok, int K,
                       int S, int r, int rs, int nseg, int L, int dtype, int mode) {
  if (K < 1 || r < 1 || rs < r || ld_x < K || ld_w < K || ld_in < (int64_t)S * rs ||
      (mode != ORACLE_F32 && mode != ORACLE_F64))
    return ORACLE_BAD_DIMS;
  int bad = oracle_check_tables(seg_indptr, weight_indices, permutation, slice_offsets,
                                tok, nseg, L, S, ld_out);
  if (bad) return bad;

  const int64_t n_tot = (int64_t)slice_offsets[S] - slice_offsets[0];

#pragma omp parallel
  for (int s = 0; s < nseg; ++s) {
    const int a = weight_indices[s];
    const float scaling = scalings[a];
    const int lo = seg_indptr[s], hi = seg_indptr[s + 1];
    const uint16_t* B = B_stack + (int64_t)a * n_tot * rs;

#pragma omp for schedule(static) nowait
    for (int i = lo; i < hi; ++i) {
      const int64_t t = permutation[i];
      const uint16_t* xrow = x + t * ld_x;
      for (int q = 0; q < S; ++q) {
        const uint16_t* v = in_r + (int64_t)i * ld_in + (int64_t)q * rs;
        for (int64_t c = slice_offsets[q]; c < slice_offsets[q + 1]; ++c) {
          const uint16_t* wrow = W + (c - slice_offsets[0]) * ld_w;
          const uint16_t* bcol = B + (c - slice_offsets[0]) * rs;  /* B row of column c */
          if (mode == ORACLE_F32) {
            float base = 0.0f;
            for (int k = 0; k < K; ++k)
              base += oracle_decode(xrow[k], dtype) * oracle_decode(wrow[k], dtype);
            float lora = 0.0f;
            for (int j = 0; j < r; ++j)
              lora += oracle_decode(v[j], dtype) * oracle_decode(bcol[j], dtype);
            const float sum = scaling == 0.0f ? base : base + scaling * lora;
            ((uint16_t*)out)[t * ld_out + c] = oracle_encode(sum, dtype);
          } else {
            double base = 0.0;
            for (int k = 0; k < K; ++k)
              base += (double)oracle_decode(xrow[k], dtype) * (double)oracle_decode(wrow[k], dtype);
            double lora = 0.0;
            for (int j = 0; j < r; ++j)
              lora += (double)oracle_decode(v[j], dtype) * (double)oracle_decode(bcol[j], dtype);
            ((double*)out)[t * ld_out + c] =
                scaling == 0.0f ? base : base + (double)scaling * lora;
          }
        }
      }
    }
  }
  return 0;
}

/* The embedding variant of the shrink (sgl-kernel-xpu page, file table:
 * EmbeddingLoraAFwd): the "x" row of a token is the one-hot vector of its id,
 * so the product with A selects one column of the adapter's A. */
int oracle_embedding_a(const int32_t* ids, const uint16_t* A_emb, const int32_t* seg_indptr,
                       const int32_t* weight_indices, uint16_t* out, int64_t ld_out,
                       int tok, int V, int r, int rs, int nseg, int L) {
  if (V < 1 || r < 1 || rs < r || ld_out < rs || tok < 0 || nseg < 0 || L < 1)
    return ORACLE_BAD_DIMS;
  for (int s = 0; s <= nseg; ++s)
    if (seg_indptr[s] < 0 || seg_indptr[s] > tok || (s > 0 && seg_indptr[s] < seg_indptr[s - 1]))
      return ORACLE_BAD_INDPTR;
  for (int s = 0; s < nseg; ++s) {
    const int a = weight_indices[s];
    if (a < 0 || a >= L) return ORACLE_BAD_ADAPTER;
    for (int i = seg_indptr[s]; i < seg_indptr[s + 1]; ++i) {
      const int id = ids[i];
      if (id < 0 || id >= V) return ORACLE_BAD_DIMS;
      for (int j = 0; j < r; ++j)
        out[(int64_t)i * ld_out + j] = A_emb[((int64_t)a * rs + j) * V + id];
    }
  }
  return 0;
}

/* ---------------------------------------------------------------- threads */

void oracle_set_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }

int oracle_max_threads(void) { return omp_get_max_threads(); }
