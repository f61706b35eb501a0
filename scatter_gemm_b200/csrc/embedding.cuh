// embedding.cuh -- LoRA A of an embedding layer (the EmbeddingLoraAFwd op of the
// sgl-kernel-xpu page's file table): the "x" row of a token is the one-hot
// vector of its id, so the shrink reduces to selecting one column of the
// segment adapter's A:   out[i, j] = A_emb[a, j, ids[i]]   (j < r).
// A_emb is [L, rs, V] (vocabulary contiguous, as every A here is laid out with
// the contraction dimension contiguous).  Rows are in token order.  Pieces come
// from the warp lookup of sched.cuh, so the launch bound ceil(tok/128) + nseg
// is known on the host without reading any table (the pages needed a max_len
// argument, or a device-to-host read of it, to size their grid).
#pragma once

#include "common.cuh"
#include "sched.cuh"

namespace lora {

constexpr int kEmbBM = 128;

__global__ void __launch_bounds__(128)
embedding_a_kernel(const int32_t* __restrict__ ids, const uint16_t* __restrict__ A,
                   const int32_t* __restrict__ seg_indptr,
                   const int32_t* __restrict__ weight_indices, uint16_t* __restrict__ out,
                   int64_t ld_out, int tok, int V, int r, int rs, int nseg, int L) {
  PieceInfo pc;
  if (!find_piece_warp(seg_indptr, weight_indices, nullptr, nseg, L, tok, kEmbBM, blockIdx.x, pc))
    return;
  const int rows = pc.hi - pc.lo;
  const uint16_t* Aa = A + static_cast<int64_t>(pc.adapter) * rs * V;
  for (int e = threadIdx.x; e < rows * r; e += blockDim.x) {
    const int m = e / r, j = e % r;
    const int i = pc.lo + m;
    const int id = clampi(__ldg(ids + i), 0, V - 1);
    out[static_cast<int64_t>(i) * ld_out + j] = __ldg(Aa + static_cast<int64_t>(j) * V + id);
  }
}

}  // namespace lora
