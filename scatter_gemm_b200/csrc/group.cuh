// group.cuh -- adapter-grouped schedule for tables with many small segments.
//
// The sgl-kernel-xpu page ("Decode LoRA kernels are optimized", section
// "Behaviour changes") asks callers to pass one coalesced segment per adapter
// because the kernels tile M themselves.  When a caller does not (here: more
// segments than adapters, at least 64 KB of weight reads to save, and a
// workspace to work in), this single-CTA pass coalesces on the device
// instead: it lists the rows of every adapter's segments contiguously, so the
// tensor-core kernels tile each adapter's rows in 128-row pieces and read each
// adapter's weights once per piece instead of once per segment.  Nothing is
// synchronised with the host; the kernel after the pass may start its CTAs
// while the pass runs (programmatic dependent launch) and waits for it before
// reading the lists.
//
// Workspace layout (int32): vseg_indptr[L+1] | seg_base[nseg] | row_list[tok]
//   vseg_indptr  rows of adapter a are grouped rows [vseg_indptr[a], vseg_indptr[a+1])
//   row_list     grouped row g -> sorted row i (and so token permutation[i])
// The order of segments inside one adapter's group follows an atomic
// counter; each output row's value does not depend on it.
#pragma once

#include "common.cuh"
#include "sched.cuh"
#include "sm100.cuh"

namespace lora {

constexpr int kGroupThreads = 1024;
constexpr int kGroupMaxAdapters = 8192;
// Shared-memory bound (bytes, the kernel's dynamic limit) for staging the
// tables next to the adapter counts (up to about 16,000 segments); larger
// tables are read from global memory.
constexpr int kGroupStageBytes = 200 * 1024;

__host__ __device__ __forceinline__ bool group_stages_tables(int nseg, int L) {
  return 4ll * (static_cast<long long>(L) + 3ll * nseg + 1) <= kGroupStageBytes;
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
  // [nseg + 1] clamped seg_indptr, [nseg] clamped adapter ids and [nseg]
  // segment bases.  The tables are read from global memory once, with every
  // thread's loads in flight together; the passes below then touch shared
  // memory only (a global load behind a shared-memory atomic would wait for
  // it, one round trip per segment a thread handles).
  extern __shared__ int cnt[];
  __shared__ int warp_tot[32];
  const int tid = threadIdx.x;
  griddep_launch_dependents();  // the kernel that reads the lists may start its CTAs
  const bool staged = group_stages_tables(nseg, L);
  int* sidx = cnt + L;
  int* swi = sidx + nseg + 1;
  int* sbase = swi + nseg;
  for (int a = tid; a < L; a += blockDim.x) cnt[a] = 0;
  if (staged) {
    for (int i = tid; i <= nseg; i += blockDim.x) sidx[i] = clampi(seg_indptr[i], 0, tok);
    for (int i = tid; i < nseg; i += blockDim.x) swi[i] = clampi(weight_indices[i], 0, L - 1);
  }
  __syncthreads();
  auto bound = [&](int i) { return staged ? sidx[i] : clampi(seg_indptr[i], 0, tok); };
  auto adapter_of = [&](int s) { return staged ? swi[s] : clampi(weight_indices[s], 0, L - 1); };
  for (int s = tid; s < nseg; s += blockDim.x) {
    const int lo = bound(s), hi = bound(s + 1);
    if (hi > lo) atomicAdd(&cnt[adapter_of(s)], hi - lo);
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
    const int b = hi > lo ? atomicAdd(&cnt[adapter_of(s)], hi - lo) : 0;
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

// ---------------------------------------------------------------------------
// The same grouping for up to 256 adapters, without contended atomics: every
// warp counts the rows of its own contiguous run of segments per adapter in a
// private counter row, a scan over (adapter, warp) turns the counts into
// cursors, and each warp then walks its run again, takes a base for each
// segment from its own cursors and lists the segment's rows.  A lane lists the
// rows of a segment of at most kGroupShortRows rows itself; longer segments
// are queued and listed by whole warps afterwards.  The tables are staged in
// shared memory (group_small_smem bytes, within kGroupStageBytes).
constexpr int kGroupSmallAdapters = 256;
constexpr int kGroupShortRows = 64;

__host__ __device__ __forceinline__ long long group_small_long_slots(int nseg, int tok) {
  const long long by_rows = static_cast<long long>(tok) / (kGroupShortRows + 1) + 1;
  return nseg < by_rows ? nseg : by_rows;
}

__host__ __device__ __forceinline__ long long group_small_smem(int nseg, int L, int tok) {
  // hist[32][L] | sidx[nseg + 1] | swi[nseg] | long segments [slots][2] | queue count
  return 4ll * (32ll * L + 2ll * nseg + 1 + 2 * group_small_long_slots(nseg, tok) + 1);
}

// Used from this many segments on: below it the block-wide counters see
// little contention and the extra passes of this kernel cost more (3
// segments: 15.5 -> 17.4 us per call; 1,024 segments: no difference).
constexpr int kGroupSmallMinSegments = 2048;

__host__ __device__ __forceinline__ bool group_small_fits(int nseg, int L, int tok) {
  return nseg >= kGroupSmallMinSegments && L <= kGroupSmallAdapters &&
         group_small_smem(nseg, L, tok) <= kGroupStageBytes;
}

__global__ void __launch_bounds__(kGroupThreads)
group_rows_small_kernel(const int32_t* __restrict__ seg_indptr,
                        const int32_t* __restrict__ weight_indices, int nseg, int L, int tok,
                        int32_t* __restrict__ vseg_indptr, int32_t* __restrict__ row_list) {
  extern __shared__ int sm[];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  griddep_launch_dependents();  // the kernel that reads the lists may start its CTAs
  constexpr int kWarps = kGroupThreads / 32;
  int* hist = sm;                       // [32][L]: counts, then cursors
  int* sidx = hist + kWarps * L;        // clamped seg_indptr
  int* swi = sidx + nseg + 1;           // clamped adapter ids
  int* lq = swi + nseg;                 // long segments: (first row, base)
  const int nlong = static_cast<int>(group_small_long_slots(nseg, tok));
  int* lq_n = lq + 2 * nlong;
  for (int i = tid; i < kWarps * L; i += kGroupThreads) hist[i] = 0;
  for (int i = tid; i <= nseg; i += kGroupThreads) sidx[i] = clampi(seg_indptr[i], 0, tok);
  for (int i = tid; i < nseg; i += kGroupThreads) swi[i] = clampi(weight_indices[i], 0, L - 1);
  if (tid == 0) *lq_n = 0;
  __syncthreads();

  // each warp's contiguous run of segments
  const int per = (nseg + kWarps - 1) / kWarps;
  const int s_lo = min(nseg, w * per), s_hi = min(nseg, s_lo + per);
  for (int s = s_lo + lane; s < s_hi; s += 32) {
    const int n = sidx[s + 1] - sidx[s];
    if (n > 0) atomicAdd(&hist[w * L + swi[s]], n);
  }
  __syncthreads();

  // adapter totals, their exclusive scan (vseg_indptr), then per-warp cursors
  if (w == 0) {
    // lane l owns adapters [l * k, l * k + k), k = ceil(L / 32)
    const int k = (L + 31) / 32;
    int mine = 0;
#pragma unroll
    for (int j = 0; j < kGroupSmallAdapters / 32; ++j) {
      const int a = lane * k + j;
      if (j < k && a < L)
        for (int ww = 0; ww < kWarps; ++ww) mine += hist[ww * L + a];
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - mine;
#pragma unroll
    for (int j = 0; j < kGroupSmallAdapters / 32; ++j) {
      const int a = lane * k + j;
      if (j < k && a < L) {
        vseg_indptr[a] = run;
        for (int ww = 0; ww < kWarps; ++ww) {
          const int c = hist[ww * L + a];
          hist[ww * L + a] = run;
          run += c;
        }
      }
    }
    if (lane == 31) vseg_indptr[L] = incl;
  }
  __syncthreads();

  // bases and rows: a lane lists a short segment itself and queues a long one
  for (int s = s_lo + lane; s < s_hi; s += 32) {
    const int lo = sidx[s], n = sidx[s + 1] - lo;
    if (n <= 0) continue;
    const int b = atomicAdd(&hist[w * L + swi[s]], n);
    if (n <= kGroupShortRows) {
      for (int r = 0; r < n; ++r)
        if (b + r < tok) row_list[b + r] = lo + r;
    } else {
      const int q = atomicAdd(lq_n, 1);
      if (q < nlong) {
        lq[2 * q] = s;
        lq[2 * q + 1] = b;
      }
    }
  }
  __syncthreads();
  const int nq = min(*lq_n, nlong);
  for (int q = w; q < nq; q += kWarps) {
    const int s = lq[2 * q], b = lq[2 * q + 1];
    const int lo = sidx[s], n = sidx[s + 1] - lo;
    for (int r = lane; r < n; r += 32)
      if (b + r < tok) row_list[b + r] = lo + r;
  }
}

}  // namespace lora
