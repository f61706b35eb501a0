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
