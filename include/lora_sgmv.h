/* lora_sgmv.h -- C ABI of liblora_sgmv, the multi-adapter LoRA chunked-SGMV
 * shrink/expand pair for NVIDIA B200 (sm_100a).
 *
 * The operations follow the sgl-kernel-xpu page "Decode LoRA kernels are
 * optimized" (section "Summary": the shrink gathers token rows of x through a
 * permutation and multiplies each segment by its adapter's A; the expand
 * multiplies those rank activations by the segment's adapter B, scales the
 * result and scatter-adds it into column slices of the base projection
 * output; section "Behaviour changes": the tables seg_indptr, adapter index,
 * permutation and offset table, and the contract that callers pass one
 * coalesced segment per adapter).  The update itself is the LoRA update of
 * the ms-swift page "Add optional fast lora path for qwen2/qwen3 on npu"
 * (section "Compatibility checks": no dropout, one adapter per token).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Element type: bf16 or fp16 (lora_dtype), the same for every floating
 *    tensor of a call except `scalings`, which is fp32.  Accumulation is fp32;
 *    each output element is rounded once, to nearest even.
 *  - All tensors are row-major with an explicit leading dimension (in
 *    elements).  Any element-aligned pointer is accepted.  The tensor-core
 *    kernels take rows at any 2-byte offset: 16-byte-aligned rows go straight
 *    into their stages, others are staged as the 16-byte blocks that cover
 *    them and shifted into place.  CUDA-core kernels remain for ranks above
 *    64 and, in the shrink, S*rs above 256.
 *  - Tables (int32, in device memory):
 *      seg_indptr[nseg+1]   segment s covers sorted rows [seg_indptr[s], seg_indptr[s+1]);
 *                           non-decreasing, inside [0, tok]; empty segments allowed;
 *                           rows outside [seg_indptr[0], seg_indptr[nseg]) are not touched.
 *      weight_indices[nseg] adapter of segment s, in [0, L).
 *      permutation[tok]     sorted row i belongs to token permutation[i]; a bijection of
 *                           [0, tok).  NULL means the identity.
 *  - Rank layout: an adapter has S slices (q/k/v: S = 3, gate/up: S = 2) of
 *    valid rank r stored with stride rs >= r.  Storage padding (j >= r) is
 *    never read and never written.
 *  - Rank activations (out_r of the shrink, in_r of the expand) are stored in
 *    SORTED order: row i holds token permutation[i]; slice q occupies columns
 *    [q*rs, q*rs + r).
 *  - Nothing is synchronised with the host: the calls read no table on the
 *    host, enqueue their kernels on `stream` (a cudaStream_t, NULL = legacy
 *    default stream) and return.  The library allocates no device memory and
 *    keeps no state between calls; calls may be made from several host
 *    threads and on several streams at once.  Kernels of calls that overlap on
 *    the GPU never wait for each other: every kernel that holds tensor memory
 *    (TMEM) takes at most 256 of an SM's 512 columns and enough shared memory
 *    that at most two of its thread blocks share an SM.  The exception is other
 *    software's kernels: a kernel outside this library that holds more TMEM
 *    on an SM while it waits for thread blocks elsewhere can make a thread
 *    block of this library wait for its TMEM; do not overlap such kernels with
 *    these calls.
 *  - Every wait of a kernel on an mbarrier gives up after 1 s, records an
 *    error code (lora_device_error) and lets the kernel finish without
 *    writing further results.  Thread-block-cluster barriers and the TMEM
 *    allocation are not bounded this way; the rule above keeps them from
 *    waiting on anything but the cluster's own thread blocks.  A kernel that
 *    follows the adapter-grouping pass may start before the pass ends and
 *    then waits for it (programmatic dependent launch); the pass is one
 *    thread block with no waits of its own.
 *  - Invalid table VALUES (a decreasing seg_indptr, an adapter index out of
 *    range, a permutation that is not a bijection) are undefined behaviour in
 *    lora_shrink / lora_expand, as on the pages (section "Behaviour changes");
 *    lora_validate checks them.  Every index a kernel reads is clamped to its
 *    tensor, so bad tables give wrong values, never an out-of-bounds access.
 *  - Errors in the ARGUMENTS (null pointers, sizes, strides, dtype) are
 *    reported before anything is enqueued.
 */
#ifndef LORA_SGMV_H
#define LORA_SGMV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LORA_API __attribute__((visibility("default")))
#else
#define LORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LORA_OK = 0,
  LORA_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative or inconsistent size or stride   */
  LORA_ERR_UNSUPPORTED = 2,      /* valid but not implemented (dtype, sizes beyond limits)   */
  LORA_ERR_CUDA = 3,             /* a CUDA runtime call or a kernel launch failed            */
  LORA_ERR_BAD_VALUES = 4        /* lora_validate only: the tables hold invalid values       */
} lora_status;

typedef enum { LORA_BF16 = 0, LORA_FP16 = 1 } lora_dtype;

/* Bits that lora_validate writes into *d_result. */
enum {
  LORA_BAD_INDPTR = 2,      /* seg_indptr decreasing or outside [0, tok]       */
  LORA_BAD_ADAPTER = 4,     /* a weight index outside [0, L)                   */
  LORA_BAD_PERMUTATION = 8, /* permutation not a bijection of [0, tok)         */
  LORA_BAD_SLICES = 16      /* slice_offsets negative, decreasing or > ld_base */
};

/* Kernel path bits reported by lora_last_path. */
enum {
  LORA_PATH_GENERAL = 1, /* CUDA-core kernel (r > 64; shrink S*rs > 256)           */
  LORA_PATH_TENSOR = 2,  /* tcgen05 tensor-core kernel (any element alignment)      */
  LORA_PATH_GROUPED = 4, /* rows grouped by adapter first (workspace, many segments) */
  LORA_PATH_SPLITK = 8,  /* shrink K range split over a thread-block cluster        */
  LORA_PATH_FUSED = 16   /* lora_shrink_expand ran both ops in one launch            */
};

/* Compile-time limits of the library. */
#define LORA_MAX_SLICES 8

/* lora_shrink -- the shrink of the chunked-SGMV pair (sgl-kernel-xpu page, section "Summary").
 *
 *   out_r[i, q*rs + j] = round( sum_{k<K} x[permutation[i], k] * A_stack[a, q*rs + j, k] )
 *   for every segment s, a = weight_indices[s], i in its rows, q < S, j < r.
 *
 *   x        [tok, ld_x]      device, ld_x >= K; read
 *   A_stack  [L, S*rs, K]     device, contiguous (K contiguous, "output-dim major"); read
 *   out_r    [tok, ld_out]    device, ld_out >= S*rs; only the valid columns of rows in
 *                             segments are written
 *   workspace, workspace_bytes  optional device scratch (may be NULL / 0).  With at least
 *                             lora_workspace_size(tok, nseg, L) bytes the call may group
 *                             the rows of many small segments by adapter first; the results
 *                             agree within rounding either way.  It must not be used by
 *                             another call that runs at the same time.
 * Returns LORA_OK, LORA_ERR_INVALID_ARGUMENT, LORA_ERR_UNSUPPORTED or LORA_ERR_CUDA.
 * tok == 0 or nseg == 0 returns LORA_OK and enqueues nothing.
 */
LORA_API lora_status lora_shrink(const void* x, int64_t ld_x, const void* A_stack,
                        const int32_t* seg_indptr, const int32_t* weight_indices,
                        const int32_t* permutation, void* out_r, int64_t ld_out,
                        int tok, int K, int S, int r, int rs, int nseg, int L,
                        lora_dtype dtype, void* workspace, size_t workspace_bytes,
                        void* stream);

/* lora_expand -- the expand of the chunked-SGMV pair (sgl-kernel-xpu page, section "Summary").
 *
 *   for every segment s with a = weight_indices[s] and scalings[a] != 0, every row i of s,
 *   every slice q < S and column c in [slice_offsets[q], slice_offsets[q+1]):
 *     t = permutation[i]
 *     base_out[t, c] = round( base_out[t, c]
 *                            + scalings[a] * sum_{j<r} in_r[i, q*rs + j] * B_stack[a, c - off0, j] )
 *   with off0 = slice_offsets[0].  A segment whose scaling is exactly 0 is skipped: its
 *   base rows stay bit-identical.
 *
 *   in_r           [tok, ld_in]       device, ld_in >= S*rs; read (valid columns only)
 *   B_stack        [L, N_tot, rs]     device, contiguous, N_tot = off[S] - off[0]; read
 *   slice_offsets  [S+1]              HOST int32 array, non-decreasing, off[S] <= ld_base;
 *                                     read during the call only (no device copy, no sync)
 *   scalings       [L]                device fp32
 *   base_out       [tok, ld_base]     device; read and written in place
 *   workspace      as for lora_shrink.
 * Returns as lora_shrink.
 */
LORA_API lora_status lora_expand(const void* in_r, int64_t ld_in, const void* B_stack,
                        const int32_t* seg_indptr, const int32_t* weight_indices,
                        const int32_t* permutation, const int32_t* slice_offsets,
                        const float* scalings, void* base_out, int64_t ld_base,
                        int tok, int S, int r, int rs, int nseg, int L,
                        lora_dtype dtype, void* workspace, size_t workspace_bytes,
                        void* stream);

/* Bytes of optional workspace that lets lora_shrink / lora_expand use the
 * adapter-grouped schedule for tables with many small segments.  The grouping
 * pass is skipped when it would save under 64 KB of adapter-weight reads
 * ((nseg - L) times the weights one 128-row piece reads). */
LORA_API size_t lora_workspace_size(int tok, int nseg, int L);

/* lora_validate -- the value checks of the tables (sgl-kernel-xpu page, section "Behaviour
 * changes": seg_indptr, index range, permutation, offset table), run on the
 * device.  Writes the OR of the LORA_BAD_* bits that apply into *d_result
 * (device int32, overwritten; 0 = valid).  slice_offsets is a HOST array and
 * may be NULL (then the offset table is not checked); it is checked on the
 * host and its bit is folded into *d_result.  Needs device scratch of
 * lora_validate_workspace_size(tok) bytes.  Asynchronous: read *d_result after
 * synchronising `stream`.
 */
LORA_API lora_status lora_validate(const int32_t* seg_indptr, const int32_t* weight_indices,
                          const int32_t* permutation, const int32_t* slice_offsets,
                          int tok, int nseg, int L, int S, int64_t ld_base,
                          int32_t* d_result, void* workspace, size_t workspace_bytes,
                          void* stream);

LORA_API size_t lora_validate_workspace_size(int tok);

/* ---- identity-permutation variants --------------------------------------
 * The other LoRA ops of the sgl-kernel-xpu page's file table (SGEMMLoraAFwd,
 * SGEMMLoraBFwd, QKVLoraBFwd, GateUpLoraBFwd, EmbeddingLoraAFwd) take segments
 * in token order: row i of every tensor belongs to token i.  The first four are
 * lora_shrink / lora_expand with permutation = NULL and a fixed slice layout;
 * arguments, errors and results are those of the call they forward to.
 */

/* lora_sgemm_a: out[i, q*rs + j] = sum_k x[i, k] * A_stack[a, q*rs + j, k]. */
LORA_API lora_status lora_sgemm_a(const void* x, int64_t ld_x, const void* A_stack,
                                  const int32_t* seg_indptr, const int32_t* weight_indices,
                                  void* out, int64_t ld_out, int tok, int K, int S, int r,
                                  int rs, int nseg, int L, lora_dtype dtype, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* lora_sgemm_b: one slice of width N at column 0:
 * base_out[i, c] += scalings[a] * sum_j in_r[i, j] * B_stack[a, c, j]   (B_stack [L, N, rs]). */
LORA_API lora_status lora_sgemm_b(const void* in_r, int64_t ld_in, const void* B_stack,
                                  const int32_t* seg_indptr, const int32_t* weight_indices,
                                  const float* scalings, void* base_out, int64_t ld_base,
                                  int tok, int N, int r, int rs, int nseg, int L,
                                  lora_dtype dtype, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* lora_qkv_b: three slices (q, k, v) at the HOST column offsets qkv_offsets[0..3]. */
LORA_API lora_status lora_qkv_b(const void* in_r, int64_t ld_in, const void* B_stack,
                                const int32_t* seg_indptr, const int32_t* weight_indices,
                                const int32_t* qkv_offsets, const float* scalings,
                                void* base_out, int64_t ld_base, int tok, int r, int rs,
                                int nseg, int L, lora_dtype dtype, void* workspace,
                                size_t workspace_bytes, void* stream);

/* lora_gate_up_b: two slices (gate, up) of width N each, at columns 0 and N. */
LORA_API lora_status lora_gate_up_b(const void* in_r, int64_t ld_in, const void* B_stack,
                                    const int32_t* seg_indptr, const int32_t* weight_indices,
                                    const float* scalings, void* base_out, int64_t ld_base,
                                    int tok, int N, int r, int rs, int nseg, int L,
                                    lora_dtype dtype, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* lora_embedding_a: LoRA A of an embedding layer.  The input row of a token is
 * the one-hot vector of its id, so
 *   out[i, j] = A_emb[a, j, ids[i]]   (j < r)
 * for every segment s, a = weight_indices[s], i in its rows.
 *   ids     [tok]        device int32 token ids in [0, V) (out-of-range ids are clamped)
 *   A_emb   [L, rs, V]   device, vocabulary contiguous
 *   out     [tok, ld_out] device, ld_out >= rs; only the valid columns j < r of rows in
 *                        segments are written
 * The grid bound ceil(tok/128) + nseg is known on the host, so no maximum
 * segment length is needed and nothing is read back from the device. */
LORA_API lora_status lora_embedding_a(const int32_t* ids, const void* A_emb,
                                      const int32_t* seg_indptr, const int32_t* weight_indices,
                                      void* out, int64_t ld_out, int tok, int V, int r, int rs,
                                      int nseg, int L, lora_dtype dtype, void* stream);

/* lora_shrink_static_scratch -- lora_shrink for callers that cannot allocate.
 *
 * The pages have no counterpart of this call.  Some callers of this library
 * are handed only input and output buffers by a host framework (a custom-op or
 * plugin interface of an inference engine) and have no allocator of their own:
 * they cannot call cudaMalloc, which would bypass the framework's memory
 * accounting and can synchronise the device, and they have no workspace to
 * pass.  This entry point computes exactly what lora_shrink computes, with the
 * same arguments minus the workspace, and allocates nothing: the scratch of the
 * adapter-grouped schedule lives in a fixed array of LORA_STATIC_SCRATCH_BYTES
 * (1 MiB) compiled into the library, which every GPU that loads the library
 * holds until the process exits.
 *
 *  - Limit: only calls that group use the scratch: more segments than
 *    adapters (nseg > L), and at least 64 KB of weight reads saved
 *    ((nseg - L) * S * rs * K * 2 bytes).  For them lora_workspace_size(tok,
 *    nseg, L) must not exceed LORA_STATIC_SCRATCH_BYTES (about
 *    tok + nseg + L <= 262,000); larger problems return LORA_ERR_UNSUPPORTED
 *    before anything is enqueued.  Other calls need no scratch and have no
 *    such limit.
 *  - The first call on each device looks up the array's device address with
 *    that device current (a CUDA runtime query, no allocation) and caches it;
 *    make that first call before any stream capture.  The cached address
 *    belongs to the device's context at that time: resetting the device
 *    (cudaDeviceReset) after the first call is not supported.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; nothing in it has to start at zero.  Calls whose kernels overlap
 *    on the GPU (e.g. on two streams) race on the array: serialise them.
 * Returns as lora_shrink.
 */
#define LORA_STATIC_SCRATCH_BYTES (1u << 20)
LORA_API lora_status lora_shrink_static_scratch(const void* x, int64_t ld_x, const void* A_stack,
                                                const int32_t* seg_indptr,
                                                const int32_t* weight_indices,
                                                const int32_t* permutation, void* out_r,
                                                int64_t ld_out, int tok, int K, int S, int r,
                                                int rs, int nseg, int L, lora_dtype dtype,
                                                void* stream);

/* lora_shrink_expand -- the pair in one call: lora_shrink into out_r, then
 * lora_expand with in_r = out_r (the rank activations rounded once to the
 * element type in between, as in the sgl-kernel-xpu page, section "Summary").
 *   x, A_stack, seg_indptr, weight_indices, permutation, out_r, ld_out: as lora_shrink
 *   B_stack, slice_offsets (HOST), scalings, base_out, ld_base:          as lora_expand
 * out_r [tok, ld_out >= S*rs] is written (valid columns j < r of the rows in
 * segments) and base_out updated, with the results of the two calls made
 * one after the other, up to the fp32 summation order of the shrink.  For
 * decode-sized batches (tok <= 512, few segments, 16-byte-aligned tensors)
 * one kernel does both: a thread-block cluster per piece runs a split-K
 * shrink, shares the rounded rank activations through distributed shared
 * memory and runs the expand of that piece (LORA_PATH_FUSED).  Otherwise the
 * two calls run in sequence on the stream (using `workspace` as they do).
 * Errors: those of lora_shrink and lora_expand. */
LORA_API lora_status lora_shrink_expand(const void* x, int64_t ld_x, const void* A_stack,
                                        const void* B_stack, const int32_t* seg_indptr,
                                        const int32_t* weight_indices,
                                        const int32_t* permutation,
                                        const int32_t* slice_offsets, const float* scalings,
                                        void* out_r, int64_t ld_out, void* base_out,
                                        int64_t ld_base, int tok, int K, int S, int r, int rs,
                                        int nseg, int L, lora_dtype dtype, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* lora_base_expand -- the base projection with the expand folded into it.
 *   out[perm[i], c] = rn( sum_k x[perm[i], k] * W[c - off[0], k]
 *                         + scalings[a] * sum_{j<r} in_r[i, q*rs + j] * B_stack[a, c - off[0], j] )
 * for the rows i of every segment (adapter a) and the columns c of slice q;
 * rn(projection) alone where scalings[a] == 0.  On the sglang page for
 * Qwen3.5/Next on NPU (key source snippets, forward_prepare_npu) the qkv_proj
 * output goes straight to the split step: computing it with the LoRA term
 * included writes it once, instead of writing it and then reading and
 * rewriting it in lora_expand.
 *   x [tok, ld_x], W [N_tot, ld_w] (the projection weight, output-dimension-
 *   major, K contiguous), in_r [tok, ld_in] (sorted order, as lora_expand),
 *   B_stack [L, N_tot, rs], slice_offsets (HOST, S+1), scalings [L] fp32,
 *   out [tok, ld_out >= off[S]]: written at the rows of tokens in segments and
 *   columns [off[0], off[S]); nothing else.
 * The two sums are formed in fp32 (the projection over K on the tensor cores)
 * and rounded once.  Tensor-core layout only: x, W, in_r, B_stack, out 16-byte
 * aligned, K, rs, ld_* and slice starts multiples of 8, r <= 64; otherwise
 * LORA_ERR_UNSUPPORTED.  Other errors as lora_expand. */
LORA_API lora_status lora_base_expand(const void* x, int64_t ld_x, const void* W, int64_t ld_w,
                                      const void* in_r, int64_t ld_in, const void* B_stack,
                                      const int32_t* seg_indptr, const int32_t* weight_indices,
                                      const int32_t* permutation, const int32_t* slice_offsets,
                                      const float* scalings, void* out, int64_t ld_out,
                                      int tok, int K, int S, int r, int rs, int nseg, int L,
                                      lora_dtype dtype, void* stream);

/* ---- 64-bit index tables ------------------------------------------------
 * lora_shrink_i64 / lora_expand_i64 take seg_indptr, weight_indices and
 * permutation as int64_t (the default index type of PyTorch), as the
 * ring-attention page ("Tests") does for its cu_seqlens; everything else is
 * exactly lora_shrink / lora_expand.  One small kernel narrows the three
 * tables into the front of `workspace` (device memory, 16-byte aligned, owned
 * by the caller, stream-ordered like the call), and the call then continues
 * on the int32 path with the rest of the workspace.  Values outside int32
 * saturate; like any other invalid table value they are clamped by the
 * kernels and reported by lora_validate on the narrowed tables.
 * workspace_bytes must be at least lora_index64_workspace_size(tok, nseg),
 * else LORA_ERR_INVALID_ARGUMENT; adding lora_workspace_size(tok, nseg, L)
 * keeps the adapter-grouped schedule.  The narrowing counts in
 * lora_launch_count. */
LORA_API size_t lora_index64_workspace_size(int tok, int nseg);

LORA_API lora_status lora_shrink_i64(const void* x, int64_t ld_x, const void* A_stack,
                                     const int64_t* seg_indptr, const int64_t* weight_indices,
                                     const int64_t* permutation, void* out_r, int64_t ld_out,
                                     int tok, int K, int S, int r, int rs, int nseg, int L,
                                     lora_dtype dtype, void* workspace, size_t workspace_bytes,
                                     void* stream);

LORA_API lora_status lora_expand_i64(const void* in_r, int64_t ld_in, const void* B_stack,
                                     const int64_t* seg_indptr, const int64_t* weight_indices,
                                     const int64_t* permutation, const int32_t* slice_offsets,
                                     const float* scalings, void* base_out, int64_t ld_base,
                                     int tok, int S, int r, int rs, int nseg, int L,
                                     lora_dtype dtype, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* Kernel path (LORA_PATH_* bits) chosen by the last lora_shrink / lora_expand
 * call made on this host thread; 0 if none launched a kernel. */
LORA_API int lora_last_path(void);

/* Failure detection of the tensor-core kernels.  Every mbarrier wait inside
 * them is bounded (1 s); a wait that runs out records a nonzero code in a
 * device word, and the kernel releases its resources and returns without
 * further writes.
 * This call reads that word (synchronously, on the current device) into *code
 * and clears it if `clear` is nonzero. */
LORA_API lora_status lora_device_error(int32_t* code, int clear);

/* Static description of a status code; never NULL. */
LORA_API const char* lora_status_string(lora_status status);

/* Kernel launches this thread has enqueued through the library since the last
 * reset (a host-side counter, for accounting in benchmarks). */
LORA_API uint64_t lora_launch_count(void);
LORA_API void lora_reset_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* LORA_SGMV_H */
