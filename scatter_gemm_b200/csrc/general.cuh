// general.cuh -- CUDA-core kernels of the shrink and expand.
//
// These accept any pointer alignment, leading dimension, rank, K and slice
// layout (2-byte accesses only), so they are the path for shapes the
// tensor-core kernels do not take: ranks above 64, a padded shrink width
// S*rs above 256.  Both use the on-device piece scheduler of sched.cuh.
#pragma once

#include "common.cuh"
#include "sched.cuh"

namespace lora {

struct ShrinkArgs {
  const uint16_t* x;
  int64_t ld_x;
  const uint16_t* A;  // [L, S*rs, K]
  const int32_t* seg_indptr;
  const int32_t* weight_indices;
  const int32_t* permutation;  // may be null (identity)
  uint16_t* out;
  int64_t ld_out;
  int tok, K, S, r, rs, nseg, L;
};

struct ExpandArgs {
  const uint16_t* in_r;
  int64_t ld_in;
  const uint16_t* B;  // [L, N_tot, rs]
  const int32_t* seg_indptr;
  const int32_t* weight_indices;
  const int32_t* permutation;  // may be null (identity)
  const float* scalings;
  uint16_t* base;
  int64_t ld_base;
  int tok, S, r, rs, nseg, L;
  SliceTable slices;
};

__device__ __forceinline__ int token_of(const int32_t* __restrict__ perm, int i, int tok) {
  return perm ? clampi(__ldg(perm + i), 0, tok - 1) : i;
}

// ---------------------------------------------------------------------------
// shrink, general: CTA = one piece (<= kGBM rows) x one group of outputs.
// Warp w owns kNPW valid outputs n = (q, j); lanes split K; the x rows of the
// piece are staged in shared memory in K chunks as fp32; the per-lane partial
// sums are reduced with warp shuffles at the end.
// ---------------------------------------------------------------------------
constexpr int kGBM = 16;      // rows per piece
constexpr int kGKC = 256;     // K chunk staged in shared memory
constexpr int kGWarps = 8;
constexpr int kGNPW = 2;      // outputs per warp
constexpr int kGNPC = kGWarps * kGNPW;  // outputs per CTA

template <class E>
__global__ void __launch_bounds__(kGWarps * 32)
shrink_general_kernel(const ShrinkArgs p) {
  __shared__ float xs[kGBM][kGKC + 1];
  __shared__ int tok_of_row[kGBM];
  Piece pc;
  if (!find_piece(p.seg_indptr, p.nseg, p.tok, kGBM, blockIdx.x, pc)) return;
  const int rows = pc.hi - pc.lo;
  const int a = clampi(__ldg(p.weight_indices + pc.seg), 0, p.L - 1);
  const int nvalid = p.S * p.r;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < kGBM)
    tok_of_row[threadIdx.x] =
        threadIdx.x < rows ? token_of(p.permutation, pc.lo + threadIdx.x, p.tok) : 0;

  int nidx[kGNPW];
  const uint16_t* arow[kGNPW];
#pragma unroll
  for (int w = 0; w < kGNPW; ++w) {
    const int v = blockIdx.y * kGNPC + warp * kGNPW + w;
    const int q = v / p.r, j = v % p.r;
    nidx[w] = v < nvalid ? q * p.rs + j : -1;
    arow[w] = p.A + ((int64_t)a * p.S * p.rs + (v < nvalid ? q * p.rs + j : 0)) * p.K;
  }

  float acc[kGBM][kGNPW];
#pragma unroll
  for (int m = 0; m < kGBM; ++m)
#pragma unroll
    for (int w = 0; w < kGNPW; ++w) acc[m][w] = 0.f;

  for (int k0 = 0; k0 < p.K; k0 += kGKC) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kGBM * kGKC; idx += blockDim.x) {
      const int m = idx / kGKC, kk = idx % kGKC;
      float v = 0.f;
      if (m < rows && k0 + kk < p.K)
        v = E::bits_to_f32(__ldg(p.x + (int64_t)tok_of_row[m] * p.ld_x + k0 + kk));
      xs[m][kk] = v;
    }
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kGNPW; ++w) {
      if (nidx[w] < 0) continue;
      for (int kk = lane; kk < kGKC && k0 + kk < p.K; kk += 32) {
        const float av = E::bits_to_f32(__ldg(arow[w] + k0 + kk));
#pragma unroll
        for (int m = 0; m < kGBM; ++m) acc[m][w] = fmaf(xs[m][kk], av, acc[m][w]);
      }
    }
  }

#pragma unroll
  for (int w = 0; w < kGNPW; ++w) {
#pragma unroll
    for (int m = 0; m < kGBM; ++m) {
      const float s = warp_sum(acc[m][w]);
      if (lane == 0 && nidx[w] >= 0 && m < rows)
        p.out[(int64_t)(pc.lo + m) * p.ld_out + nidx[w]] = E::f32_to_bits(s);
    }
  }
}

// ---------------------------------------------------------------------------
// expand, general: CTA = one piece (<= kGBM rows) x 256 global columns; a
// thread per column keeps the column's B row in registers (rank chunks of
// kGRC) and the piece's rank activations sit in shared memory as fp32.
// ---------------------------------------------------------------------------
constexpr int kGECols = 256;
constexpr int kGRC = 16;  // rank chunk held in registers

template <class E>
__global__ void __launch_bounds__(kGECols)
expand_general_kernel(const ExpandArgs p) {
  extern __shared__ float rs_smem[];  // [kGBM][S*r]
  __shared__ int tok_of_row[kGBM];
  Piece pc;
  if (!find_piece(p.seg_indptr, p.nseg, p.tok, kGBM, blockIdx.x, pc)) return;
  const int a = clampi(__ldg(p.weight_indices + pc.seg), 0, p.L - 1);
  const float scale = __ldg(p.scalings + a);
  if (scale == 0.f) return;  // a zero scaling leaves the rows untouched
  const int rows = pc.hi - pc.lo;
  const int sr = p.S * p.r;
  if (threadIdx.x < kGBM)
    tok_of_row[threadIdx.x] =
        threadIdx.x < rows ? token_of(p.permutation, pc.lo + threadIdx.x, p.tok) : 0;
  for (int idx = threadIdx.x; idx < kGBM * sr; idx += blockDim.x) {
    const int m = idx / sr, v = idx % sr;
    const int q = v / p.r, j = v % p.r;
    rs_smem[idx] = m < rows
        ? E::bits_to_f32(__ldg(p.in_r + (int64_t)(pc.lo + m) * p.ld_in + q * p.rs + j)) : 0.f;
  }
  __syncthreads();

  const int off0 = p.slices.off[0];
  const int c = off0 + blockIdx.y * kGECols + threadIdx.x;
  if (c >= p.slices.off[p.S]) return;
  const int q = slice_of(p.slices, c);
  const int64_t n_tot = p.slices.off[p.S] - off0;
  const uint16_t* brow = p.B + ((int64_t)a * n_tot + (c - off0)) * p.rs;
  // the base elements of this column first: their loads stay in flight while
  // the rank sums are formed
  uint16_t old[kGBM];
#pragma unroll
  for (int m = 0; m < kGBM; ++m)
    old[m] = m < rows ? p.base[(int64_t)tok_of_row[m] * p.ld_base + c] : uint16_t(0);

  float acc[kGBM];
#pragma unroll
  for (int m = 0; m < kGBM; ++m) acc[m] = 0.f;
  for (int j0 = 0; j0 < p.r; j0 += kGRC) {
    float b[kGRC];
#pragma unroll
    for (int jj = 0; jj < kGRC; ++jj)
      b[jj] = (j0 + jj < p.r) ? E::bits_to_f32(__ldg(brow + j0 + jj)) : 0.f;
#pragma unroll
    for (int m = 0; m < kGBM; ++m) {
      const float* v = rs_smem + m * sr + q * p.r + j0;
#pragma unroll
      for (int jj = 0; jj < kGRC; ++jj)
        if (j0 + jj < p.r) acc[m] = fmaf(v[jj], b[jj], acc[m]);
    }
  }
#pragma unroll
  for (int m = 0; m < kGBM; ++m)
    if (m < rows)
      p.base[(int64_t)tok_of_row[m] * p.ld_base + c] =
          E::f32_to_bits(E::bits_to_f32(old[m]) + scale * acc[m]);
}

// ---------------------------------------------------------------------------
// table validation (device side of lora_validate)
// ---------------------------------------------------------------------------
__global__ void set_word_kernel(int32_t* __restrict__ w, int32_t v) { *w = v; }

// Narrows three int64 index tables to int32, saturating, one thread per
// destination word.  Table a (na entries) goes to out[0..pa), table b (nb
// entries) to out[pa..pa+pb), table c (nc entries) to out[pa+pb..pa+pb+nc);
// pa >= na and pb >= nb are padded sizes whose extra words are set to 0.
__global__ void narrow_index_kernel(const int64_t* __restrict__ a, int na, int pa,
                                    const int64_t* __restrict__ b, int nb, int pb,
                                    const int64_t* __restrict__ c, int nc,
                                    int32_t* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t n = static_cast<int64_t>(pa) + pb + nc;
  if (i >= n) return;
  int64_t v = 0;
  if (i < pa) {
    if (i < na) v = __ldg(a + i);
  } else if (i < static_cast<int64_t>(pa) + pb) {
    const int64_t j = i - pa;
    if (j < nb) v = __ldg(b + j);
  } else {
    v = __ldg(c + (i - pa - pb));
  }
  out[i] = v > INT32_MAX ? INT32_MAX : (v < INT32_MIN ? INT32_MIN : static_cast<int32_t>(v));
}

__global__ void validate_kernel(const int32_t* __restrict__ seg_indptr,
                                const int32_t* __restrict__ weight_indices,
                                const int32_t* __restrict__ perm, int tok, int nseg, int L,
                                unsigned* __restrict__ seen, int32_t* __restrict__ result) {
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int stride = gridDim.x * blockDim.x;
  int bad = 0;
  for (int s = tid; s <= nseg; s += stride) {
    const int v = seg_indptr[s];
    if (v < 0 || v > tok) bad |= 2;
    if (s > 0 && v < seg_indptr[s - 1]) bad |= 2;
    if (s < nseg) {
      const int w = weight_indices[s];
      if (w < 0 || w >= L) bad |= 4;
    }
  }
  if (perm) {
    for (int i = tid; i < tok; i += stride) {
      const int t = perm[i];
      if (t < 0 || t >= tok) {
        bad |= 8;
      } else {
        const unsigned bit = 1u << (t & 31);
        if (atomicOr(seen + (t >> 5), bit) & bit) bad |= 8;
      }
    }
  }
  if (bad) atomicOr(reinterpret_cast<unsigned*>(result), static_cast<unsigned>(bad));
}

}  // namespace lora
