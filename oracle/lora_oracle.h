/* lora_oracle.h -- plain CPU oracle of the chunked-SGMV LoRA shrink/expand pair.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link
 * or call this; only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code with the CUDA library.
 *
 * What it computes follows the sgl-kernel-xpu page "Decode LoRA kernels are
 * optimized" (section "Summary": the shrink gathers token rows through a
 * permutation and multiplies each segment by its adapter's A; the expand
 * multiplies by the adapter's B, scales, and scatter-adds into the column
 * slices of the base output) and the ms-swift page "Add optional fast lora
 * path for qwen2/qwen3 on npu" (section "Compatibility checks": the LoRA
 * update with no dropout, one adapter per token).
 *
 * Element types: 0 = bf16, 1 = fp16, stored as uint16 bit patterns.
 *
 * Modes:
 *   ORACLE_F32  fp32 accumulation in order k = 0..K-1 (shrink) or
 *               j = 0..r-1 (expand), one round-to-nearest-even into the
 *               element type; every buffer in the element type.
 *   ORACLE_F64  fp64 accumulation; shrink writes double out_r; expand reads
 *               in_r in the element type and a double base_out (read and
 *               written in place, no rounding).
 *   ORACLE_F64_IN (expand only) like ORACLE_F64 but in_r is double too.
 *
 * Return value: 0 on success, otherwise the ORACLE_BAD_* bitmask of
 * oracle_check_tables (the oracle refuses invalid tables and writes nothing).
 */
#ifndef LORA_ORACLE_H
#define LORA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORACLE_BF16 = 0, ORACLE_FP16 = 1 };
enum { ORACLE_F32 = 0, ORACLE_F64 = 1, ORACLE_F64_IN = 2 };

/* bits of the table-check result */
enum {
  ORACLE_BAD_DIMS = 1,        /* a size or leading dimension is out of range   */
  ORACLE_BAD_INDPTR = 2,      /* seg_indptr decreasing or outside [0, tok]     */
  ORACLE_BAD_ADAPTER = 4,     /* weight_indices[s] outside [0, L)              */
  ORACLE_BAD_PERMUTATION = 8, /* permutation not a bijection of [0, tok)       */
  ORACLE_BAD_SLICES = 16      /* slice_offsets negative, decreasing or > ld    */
};

/* Table checks (slice_offsets may be NULL for the shrink tables only). */
int oracle_check_tables(const int32_t* seg_indptr, const int32_t* weight_indices,
                        const int32_t* permutation, const int32_t* slice_offsets,
                        int tok, int nseg, int L, int S, int64_t ld_base);

/* out_r[i, q*rs + j] = sum_k x[perm[i], k] * A[a, q*rs + j, k]  (j < r)
 * for every segment s, a = weight_indices[s], i in [seg_indptr[s], seg_indptr[s+1]). */
int oracle_shrink(const uint16_t* x, int64_t ld_x, const uint16_t* A_stack,
                  const int32_t* seg_indptr, const int32_t* weight_indices,
                  const int32_t* permutation, void* out_r, int64_t ld_out,
                  int tok, int K, int S, int r, int rs, int nseg, int L,
                  int dtype, int mode);

/* base_out[perm[i], c] = base_out[perm[i], c]
 *                        + scalings[a] * sum_j in_r[i, q*rs + j] * B[a, c - off[0], j]
 * for c in slice q = [off[q], off[q+1]), j < r; segments whose scaling is 0
 * are skipped entirely. */
int oracle_expand(const void* in_r, int64_t ld_in, const uint16_t* B_stack,
                  const int32_t* seg_indptr, const int32_t* weight_indices,
                  const int32_t* permutation, const int32_t* slice_offsets,
                  const float* scalings, void* base_out, int64_t ld_base,
                  int tok, int S, int r, int rs, int nseg, int L,
                  int dtype, int mode);

/* The base projection with the expand folded into it: for every row i of
 * segment s (adapter a, token t = permutation[i]) and column c of slice q,
 *   base = sum_k x[t, k] * W[c - off[0], k]                  (W is [N_tot, ld_w])
 *   lora = sum_{j<r} in_r[i, q*rs + j] * B[a, c - off[0], j]
 *   out[t, c] = rn(base + scalings[a] * lora)   (rn(base) when scalings[a] == 0)
 * with sequential sums (fp32 in ORACLE_F32; fp64 and no rounding in ORACLE_F64,
 * where out is double).  Only rows of tokens in segments and columns
 * [off[0], off[S]) are written. */
int oracle_base_expand(const uint16_t* x, int64_t ld_x, const uint16_t* W, int64_t ld_w,
                       const uint16_t* in_r, int64_t ld_in, const uint16_t* B_stack,
                       const int32_t* seg_indptr, const int32_t* weight_indices,
                       const int32_t* permutation, const int32_t* slice_offsets,
                       const float* scalings, void* out, int64_t ld_out, int tok, int K,
                       int S, int r, int rs, int nseg, int L, int dtype, int mode);

/* out[i, j] = A_emb[a, j, ids[i]]  (j < r) for every segment s, a = weight_indices[s],
 * i in [seg_indptr[s], seg_indptr[s+1]); rows are in token order (no permutation).
 * A_emb is [L, rs, V] with the vocabulary dimension contiguous.  Returns
 * ORACLE_BAD_DIMS for a token id outside [0, V). */
int oracle_embedding_a(const int32_t* ids, const uint16_t* A_emb, const int32_t* seg_indptr,
                       const int32_t* weight_indices, uint16_t* out, int64_t ld_out,
                       int tok, int V, int r, int rs, int nseg, int L);

/* element codec, exposed so the tests can pin it against other libraries */
float oracle_decode(uint16_t h, int dtype);
uint16_t oracle_encode(float f, int dtype);
uint16_t oracle_encode_f64(double d, int dtype);

/* OpenMP thread count used by the row loops */
void oracle_set_threads(int n);
int oracle_max_threads(void);

#ifdef __cplusplus
}
#endif
#endif
