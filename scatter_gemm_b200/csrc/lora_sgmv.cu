// lora_sgmv.cu -- C ABI of liblora_sgmv: argument checks, kernel selection and
// launches of the chunked-SGMV LoRA shrink/expand pair (sgl-kernel-xpu page
// "Decode LoRA kernels are optimized", sections "Summary" and "Behaviour
// changes").  Nothing here reads a device table on the host and nothing is
// synchronised: every call enqueues its kernels on the caller's stream.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "../../include/lora_sgmv.h"
#include "common.cuh"
#include "general.cuh"
#include "sched.cuh"

namespace {

thread_local uint64_t g_launches = 0;

inline bool aligned_to(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

inline lora_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

template <class E>
lora_status shrink_general(const lora::ShrinkArgs& a, cudaStream_t st) {
  const int slots = lora::num_piece_slots(a.tok, a.nseg, lora::kGBM);
  const int groups = (a.S * a.r + lora::kGNPC - 1) / lora::kGNPC;
  if (groups > 65535) return LORA_ERR_UNSUPPORTED;
  dim3 grid(slots, groups);
  lora::shrink_general_kernel<E><<<grid, lora::kGWarps * 32, 0, st>>>(a);
  ++g_launches;
  return launch_status();
}

template <class E>
lora_status expand_general(const lora::ExpandArgs& a, cudaStream_t st) {
  const int n_tot = a.slices.off[a.S] - a.slices.off[0];
  const int slots = lora::num_piece_slots(a.tok, a.nseg, lora::kGBM);
  const int chunks = (n_tot + lora::kGECols - 1) / lora::kGECols;
  if (chunks > 65535) return LORA_ERR_UNSUPPORTED;
  const size_t smem = sizeof(float) * lora::kGBM * a.S * a.r;
  if (smem > 200 * 1024) return LORA_ERR_UNSUPPORTED;
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(lora::expand_general_kernel<E>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return LORA_ERR_CUDA;
  }
  dim3 grid(slots, chunks);
  lora::expand_general_kernel<E><<<grid, lora::kGECols, smem, st>>>(a);
  ++g_launches;
  return launch_status();
}

}  // namespace

extern "C" {

const char* lora_status_string(lora_status s) {
  switch (s) {
    case LORA_OK: return "ok";
    case LORA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case LORA_ERR_UNSUPPORTED: return "unsupported argument combination";
    case LORA_ERR_CUDA: return "CUDA error";
    case LORA_ERR_BAD_VALUES: return "tables hold invalid values";
  }
  return "unknown status";
}

uint64_t lora_launch_count(void) { return g_launches; }
void lora_reset_launch_count(void) { g_launches = 0; }

size_t lora_workspace_size(int tok, int nseg, int L) {
  if (tok < 0 || nseg < 0 || L < 1) return 0;
  // adapter-grouped schedule: grouped row list + per-adapter row offsets
  return sizeof(int32_t) * (static_cast<size_t>(tok) + static_cast<size_t>(L) + 1 + 64);
}

size_t lora_validate_workspace_size(int tok) {
  if (tok < 0) return 0;
  return sizeof(uint32_t) * ((static_cast<size_t>(tok) + 31) / 32 + 1);
}

lora_status lora_shrink(const void* x, int64_t ld_x, const void* A_stack,
                        const int32_t* seg_indptr, const int32_t* weight_indices,
                        const int32_t* permutation, void* out_r, int64_t ld_out, int tok,
                        int K, int S, int r, int rs, int nseg, int L, lora_dtype dtype,
                        void* workspace, size_t workspace_bytes, void* stream) {
  if (dtype != LORA_BF16 && dtype != LORA_FP16) return LORA_ERR_UNSUPPORTED;
  if (tok < 0 || nseg < 0 || K < 1 || S < 1 || r < 1 || rs < r || L < 1)
    return LORA_ERR_INVALID_ARGUMENT;
  if (S > LORA_MAX_SLICES) return LORA_ERR_UNSUPPORTED;
  if (!x || !A_stack || !seg_indptr || !weight_indices || !out_r)
    return LORA_ERR_INVALID_ARGUMENT;
  if (ld_x < K || ld_out < static_cast<int64_t>(S) * rs) return LORA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes > 0 && !workspace) return LORA_ERR_INVALID_ARGUMENT;
  if (!aligned_to(x, 2) || !aligned_to(A_stack, 2) || !aligned_to(out_r, 2) ||
      !aligned_to(seg_indptr, 4) || !aligned_to(weight_indices, 4) ||
      (permutation && !aligned_to(permutation, 4)))
    return LORA_ERR_INVALID_ARGUMENT;
  if (tok == 0 || nseg == 0) return LORA_OK;

  lora::ShrinkArgs a{static_cast<const uint16_t*>(x), ld_x,
                     static_cast<const uint16_t*>(A_stack), seg_indptr, weight_indices,
                     permutation, static_cast<uint16_t*>(out_r), ld_out, tok, K, S, r, rs,
                     nseg, L};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dtype == LORA_BF16 ? shrink_general<lora::Bf16>(a, st)
                            : shrink_general<lora::Fp16>(a, st);
}

lora_status lora_expand(const void* in_r, int64_t ld_in, const void* B_stack,
                        const int32_t* seg_indptr, const int32_t* weight_indices,
                        const int32_t* permutation, const int32_t* slice_offsets,
                        const float* scalings, void* base_out, int64_t ld_base, int tok, int S,
                        int r, int rs, int nseg, int L, lora_dtype dtype, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (dtype != LORA_BF16 && dtype != LORA_FP16) return LORA_ERR_UNSUPPORTED;
  if (tok < 0 || nseg < 0 || S < 1 || r < 1 || rs < r || L < 1)
    return LORA_ERR_INVALID_ARGUMENT;
  if (S > LORA_MAX_SLICES) return LORA_ERR_UNSUPPORTED;
  if (!in_r || !B_stack || !seg_indptr || !weight_indices || !slice_offsets || !scalings ||
      !base_out)
    return LORA_ERR_INVALID_ARGUMENT;
  if (ld_in < static_cast<int64_t>(S) * rs) return LORA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes > 0 && !workspace) return LORA_ERR_INVALID_ARGUMENT;
  lora::SliceTable tab{};
  tab.S = S;
  for (int q = 0; q <= S; ++q) {
    tab.off[q] = slice_offsets[q];
    if (slice_offsets[q] < 0 || slice_offsets[q] > ld_base) return LORA_ERR_INVALID_ARGUMENT;
    if (q > 0 && slice_offsets[q] < slice_offsets[q - 1]) return LORA_ERR_INVALID_ARGUMENT;
  }
  if (!aligned_to(in_r, 2) || !aligned_to(B_stack, 2) || !aligned_to(base_out, 2) ||
      !aligned_to(seg_indptr, 4) || !aligned_to(weight_indices, 4) ||
      !aligned_to(scalings, 4) || (permutation && !aligned_to(permutation, 4)))
    return LORA_ERR_INVALID_ARGUMENT;
  if (tok == 0 || nseg == 0 || tab.off[S] == tab.off[0]) return LORA_OK;

  lora::ExpandArgs a{static_cast<const uint16_t*>(in_r), ld_in,
                     static_cast<const uint16_t*>(B_stack), seg_indptr, weight_indices,
                     permutation, scalings, static_cast<uint16_t*>(base_out), ld_base, tok, S,
                     r, rs, nseg, L, tab};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dtype == LORA_BF16 ? expand_general<lora::Bf16>(a, st)
                            : expand_general<lora::Fp16>(a, st);
}

lora_status lora_validate(const int32_t* seg_indptr, const int32_t* weight_indices,
                          const int32_t* permutation, const int32_t* slice_offsets, int tok,
                          int nseg, int L, int S, int64_t ld_base, int32_t* d_result,
                          void* workspace, size_t workspace_bytes, void* stream) {
  if (tok < 0 || nseg < 0 || L < 1 || S < 1 || !seg_indptr || !d_result ||
      (nseg > 0 && !weight_indices))
    return LORA_ERR_INVALID_ARGUMENT;
  if (permutation && (!workspace || workspace_bytes < lora_validate_workspace_size(tok)))
    return LORA_ERR_INVALID_ARGUMENT;
  int host_bad = 0;
  if (slice_offsets) {
    if (S > LORA_MAX_SLICES) return LORA_ERR_UNSUPPORTED;
    for (int q = 0; q <= S; ++q) {
      if (slice_offsets[q] < 0 || slice_offsets[q] > ld_base) host_bad |= LORA_BAD_SLICES;
      if (q > 0 && slice_offsets[q] < slice_offsets[q - 1]) host_bad |= LORA_BAD_SLICES;
    }
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The result word starts as the host-side findings; the kernel ORs in the rest.
  lora::set_word_kernel<<<1, 1, 0, st>>>(d_result, host_bad);
  ++g_launches;
  if (permutation &&
      cudaMemsetAsync(workspace, 0, lora_validate_workspace_size(tok), st) != cudaSuccess)
    return LORA_ERR_CUDA;
  const int work = tok > nseg + 1 ? tok : nseg + 1;
  int blocks = (work + 255) / 256;
  if (blocks > 1184) blocks = 1184;
  if (blocks < 1) blocks = 1;
  lora::validate_kernel<<<blocks, 256, 0, st>>>(seg_indptr, weight_indices, permutation, tok,
                                                nseg, L, static_cast<unsigned*>(workspace),
                                                d_result);
  ++g_launches;
  return launch_status();
}

}  // extern "C"
