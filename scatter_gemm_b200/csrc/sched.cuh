// sched.cuh -- on-device segment scheduler.
//
// The sgl-kernel-xpu page ("Decode LoRA kernels are optimized", sections
// "Summary" and "Behaviour changes") maps work tiles to segments on the
// device so that no call synchronises with the host, and tiles M per segment
// itself.  Here the sorted row range is cut at every multiple of BM and at
// every segment start; each cut-out "piece" has at most BM rows and lies in
// one segment.  There are at most ceil(tok/BM) + nseg pieces -- a bound the
// host knows without reading any table -- and CTA slot p finds its piece with
// one binary search over seg_indptr (O(log nseg)), or in O(1):
//   p <  nblk : the piece that starts at row p*BM (if that row is in a segment)
//   p >= nblk : the piece that starts at segment (p - nblk)'s first row, if that
//               row is not a multiple of BM (otherwise the block slot has it).
// Every row of every segment lands in exactly one piece.  Table values are
// clamped, so invalid tables never send a kernel outside its tensors.
#pragma once

#include "common.cuh"

namespace lora {

struct Piece {
  int lo;   // first sorted row
  int hi;   // one past the last sorted row (hi - lo <= BM)
  int seg;  // segment index
};

// Number of entries of seg_indptr[0..n) that are <= v (seg_indptr sorted).
__device__ __forceinline__ int count_le(const int32_t* __restrict__ a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (__ldg(a + mid) <= v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__host__ __device__ __forceinline__ int num_piece_slots(int tok, int nseg, int bm) {
  return (tok + bm - 1) / bm + nseg;
}

// Rows [lo, hi) of segment `seg` handled by slot p, or false if slot p has none.
__device__ __forceinline__ bool find_piece(const int32_t* __restrict__ seg_indptr, int nseg,
                                           int tok, int bm, int p, Piece& out) {
  const int nblk = (tok + bm - 1) / bm;
  if (p < nblk) {
    const int start = p * bm;
    const int s = count_le(seg_indptr, nseg + 1, start) - 1;
    if (s < 0 || s >= nseg) return false;
    const int end = min(clampi(__ldg(seg_indptr + s + 1), 0, tok), start + bm);
    if (end <= start) return false;
    out.lo = start;
    out.hi = end;
    out.seg = s;
    return true;
  }
  const int s = p - nblk;
  if (s >= nseg) return false;
  const int a = clampi(__ldg(seg_indptr + s), 0, tok);
  const int b = clampi(__ldg(seg_indptr + s + 1), 0, tok);
  if (a >= b || a % bm == 0) return false;
  out.lo = a;
  out.hi = min(b, (a / bm + 1) * bm);
  out.seg = s;
  return true;
}

}  // namespace lora

namespace lora {

// ---------------------------------------------------------------------------
// Warp-cooperative piece lookup for the tensor-core kernels.
//
// Same mapping as find_piece, but one warp reads the tables together: for up
// to 255 segments every lane loads 8 entries of seg_indptr and weight_indices
// (and of `per_adapter`, e.g. the scalings, for up to 256 adapters) in one
// round trip to memory, the segment is found with a ballot count, and its
// neighbours come out of registers by shuffle.  Larger tables use a 32-way
// sampled search (three round trips for 16,384 segments) and direct loads.
// All 32 lanes must call it; all get the same result.
// ---------------------------------------------------------------------------
struct PieceInfo {
  int lo, hi, seg, adapter;
  float per_adapter;  // per_adapter[adapter] (0 when no table is given)
};

constexpr int kTabPerLane = 8;
constexpr int kTabMax = 32 * kTabPerLane;

// Value of table entry i, held as v[i / 32] by lane i % 32 (i uniform over the
// warp).  Every register is shuffled with a constant index and the result is
// picked by a select chain: indexing v with i / 32 would put the table in
// local memory, which misses L1 when shared memory fills the SM.
__device__ __forceinline__ int pick(const int (&v)[kTabPerLane], int i) {
  const int src = i & 31, k = i >> 5;
  int r = 0;
#pragma unroll
  for (int j = 0; j < kTabPerLane; ++j) {
    const int t = __shfl_sync(0xffffffffu, v[j], src);
    r = (k == j) ? t : r;
  }
  return r;
}

__device__ __forceinline__ float pickf(const float (&v)[kTabPerLane], int i) {
  const int src = i & 31, k = i >> 5;
  float r = 0.f;
#pragma unroll
  for (int j = 0; j < kTabPerLane; ++j) {
    const float t = __shfl_sync(0xffffffffu, v[j], src);
    r = (k == j) ? t : r;
  }
  return r;
}

__device__ __forceinline__ bool find_piece_warp(const int32_t* __restrict__ seg_indptr,
                                                const int32_t* __restrict__ weight_indices,
                                                const float* __restrict__ per_adapter,
                                                int nseg, int L, int tok, int bm, int p,
                                                PieceInfo& out) {
  const int lane = threadIdx.x & 31;
  const int n = nseg + 1;
  const bool small = n <= kTabMax;
  int iv[kTabPerLane], wv[kTabPerLane];
  float av[kTabPerLane];
#pragma unroll
  for (int k = 0; k < kTabPerLane; ++k) {
    const int i = lane + 32 * k;
    iv[k] = (small && i < n) ? __ldg(seg_indptr + i) : 0x7fffffff;
    wv[k] = (small && weight_indices && i < nseg) ? __ldg(weight_indices + i) : 0;
    av[k] = (per_adapter && L <= kTabMax && i < L) ? __ldg(per_adapter + i) : 0.f;
  }
  auto entry = [&](int i) { return small ? pick(iv, i) : __ldg(seg_indptr + i); };

  const int nblk = (tok + bm - 1) / bm;
  int s, lo, hi;
  if (p < nblk) {
    const int start = p * bm;
    int cnt;
    if (small) {
      int c = 0;
#pragma unroll
      for (int k = 0; k < kTabPerLane; ++k) c += (iv[k] <= start) ? 1 : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
      cnt = c;
    } else {
      int a = 0, b = n;  // entries below a are <= start, entries from b on are > start
      while (b - a > 32) {
        const int step = (b - a + 31) / 32;
        const int idx = a + lane * step;
        const bool le = idx < b && __ldg(seg_indptr + idx) <= start;
        const int c = __popc(__ballot_sync(0xffffffffu, le));
        if (c == 0) { b = a; break; }
        const int na = a + (c - 1) * step + 1;
        const int nb = min(b, a + c * step);
        a = na;
        b = nb;
      }
      const int idx = a + lane;
      const bool le = idx < b && __ldg(seg_indptr + idx) <= start;
      cnt = a + __popc(__ballot_sync(0xffffffffu, le));
    }
    s = cnt - 1;
    if (s < 0 || s >= nseg) return false;
    lo = start;
    hi = min(clampi(entry(s + 1), 0, tok), start + bm);
    if (hi <= lo) return false;
  } else {
    s = p - nblk;
    if (s >= nseg) return false;
    const int a = clampi(entry(s), 0, tok), b = clampi(entry(s + 1), 0, tok);
    if (a >= b || a % bm == 0) return false;
    lo = a;
    hi = min(b, (a / bm + 1) * bm);
  }
  int adapter;
  if (!weight_indices) adapter = s;
  else adapter = small ? pick(wv, s) : __ldg(weight_indices + s);
  adapter = clampi(adapter, 0, L - 1);
  out.lo = lo;
  out.hi = hi;
  out.seg = s;
  out.adapter = adapter;
  out.per_adapter = !per_adapter ? 0.f
                    : (L <= kTabMax ? pickf(av, adapter) : __ldg(per_adapter + adapter));
  return true;
}

}  // namespace lora
