// group.cuh -- adapter-grouped schedule for tables with many small segments.
//
// The sgl-kernel-xpu page ("Decode LoRA kernels are optimized", section
// "Behaviour changes") asks callers to pass one coalesced segment per adapter
// because the kernels tile M themselves.  When a caller does not (here: more
// segments than adapters and a workspace to work in), this single-CTA pass
// coalesces on the device instead: it lists the rows of every adapter's
// segments contiguously, so the tensor-core kernels tile each adapter's rows
// in 128-row pieces and read each adapter's weights once per piece instead of
// once per segment.  Nothing is synchronised with the host.
//
// Workspace layout (int32): vseg_indptr[L+1] | seg_base[nseg] | row_list[tok]
//   vseg_indptr  rows of adapter a are grouped rows [vseg_indptr[a], vseg_indptr[a+1])
//   row_list     grouped row g -> sorted row i (and so token permutation[i])
// The order of segments inside one adapter's group follows an atomic
// counter; each output row's value does not depend on it.
#pragma once

#include "common.cuh"
#include "sched.cuh"

namespace lora {

constexpr int kGroupThreads = 1024;
constexpr int kGroupMaxAdapters = 8192;
// Shared-memory bound (bytes, the kernel's dynamic limit) for staging
// seg_indptr and the segment bases next to the adapter counts (up to about
// 25,000 segments); larger tables are read from global memory.
constexpr int kGroupStageBytes = 200 * 1024;

__host__ __device__ __forceinline__ bool group_stages_tables(int nseg, int L) {
  return 4ll * (static_cast<long long>(L) + 2ll * nseg + 1) <= kGroupStageBytes;
}

// Entries of a[0..n) that are <= v (a sorted), in shared memory.
__device__ __forceinline__ int count_le_smem(const int* a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] <= v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kGroupThreads)
group_rows_kernel(const int32_t* __restrict__ seg_indptr, const int32_t* __restrict__ weight_indices,
                  int nseg, int L, int tok, int32_t* __restrict__ vseg_indptr,
                  int32_t* __restrict__ seg_base, int32_t* __restrict__ row_list) {
  // [L] counts, then cursors; when the tables fit (group_stages_tables):
  // [nseg + 1] clamped seg_indptr and [nseg] segment bases, so that the row
  // pass below searches shared memory instead of chasing global loads
  extern __shared__ int cnt[];
  __shared__ int warp_tot[32];
  const int tid = threadIdx.x;
  const bool staged = group_stages_tables(nseg, L);
  int* sidx = cnt + L;
  int* sbase = sidx + nseg + 1;
  for (int a = tid; a < L; a += blockDim.x) cnt[a] = 0;
  if (staged)
    for (int i = tid; i <= nseg; i += blockDim.x) sidx[i] = clampi(seg_indptr[i], 0, tok);
  __syncthreads();
  auto bound = [&](int i) { return staged ? sidx[i] : clampi(seg_indptr[i], 0, tok); };
  for (int s = tid; s < nseg; s += blockDim.x) {
    const int lo = bound(s), hi = bound(s + 1);
    if (hi > lo) atomicAdd(&cnt[clampi(weight_indices[s], 0, L - 1)], hi - lo);
  }
  __syncthreads();

  // exclusive scan of cnt[0..L) -> vseg_indptr and cursors (block-wide, chunked)
  const int per = (L + blockDim.x - 1) / blockDim.x;
  const int a0 = tid * per, a1 = min(L, a0 + per);
  int local = 0;
  for (int a = a0; a < a1; ++a) local += cnt[a];
  // inclusive scan of `local` over the block
  const int lane = tid & 31, wid = tid >> 5;
  int v = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[wid] = v;
  __syncthreads();
  if (wid == 0) {
    int w = lane < (blockDim.x >> 5) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    warp_tot[lane] = w;  // inclusive prefix of warp totals
  }
  __syncthreads();
  int run = v - local + (wid > 0 ? warp_tot[wid - 1] : 0);  // exclusive prefix of this thread
  for (int a = a0; a < a1; ++a) {
    const int c = cnt[a];
    vseg_indptr[a] = run;
    cnt[a] = run;  // becomes the cursor of adapter a
    run += c;
  }
  if (tid == blockDim.x - 1) vseg_indptr[L] = run;
  __syncthreads();

  for (int s = tid; s < nseg; s += blockDim.x) {
    const int lo = bound(s), hi = bound(s + 1);
    const int b = hi > lo ? atomicAdd(&cnt[clampi(weight_indices[s], 0, L - 1)], hi - lo) : 0;
    if (staged) sbase[s] = b; else seg_base[s] = b;
  }
  __syncthreads();

  const int rlo = bound(0), rhi = bound(nseg);
  for (int i = rlo + tid; i < rhi; i += blockDim.x) {
    const int s = (staged ? count_le_smem(sidx, nseg + 1, i) : count_le(seg_indptr, nseg + 1, i)) - 1;
    if (s < 0 || s >= nseg) continue;
    const int g = (staged ? sbase[s] : seg_base[s]) + (i - bound(s));
    if (g >= 0 && g < tok) row_list[g] = i;
  }
}

}  // namespace lora
