// expand_unaligned_tc.cuh -- tensor-core expand for element-aligned inputs
// (sm_100a): rank activations, B and base rows at any 2-byte offset, any
// leading dimensions, any slice starts and widths (the tail workload of the
// sgl-kernel-xpu page, "Decode LoRA kernels are optimized", section
// "Testing": K tails, odd N, odd ranks, unaligned slice starts, misaligned
// pointers).
//
// The contraction and the scatter epilogue are those of expand_tc.cuh
//     D[128 x 128] = R_q[128 x r] * B_a[c0-off0 : c0-off0+128, 0:r]^T
//     base[perm[row], c] = round(base[perm[row], c] + scaling[a] * D[row, c])
// (tcgen05.mma, double-buffered TMEM accumulator).  What changes is the data
// movement: 16-byte copies and TMA need 16-byte aligned rows, so every row
// segment is moved as the aligned 16-byte blocks that cover it.
//   - rank activations and B rows: the covering blocks are staged with
//     cp.async and shifted (__funnelshift_r) into the swizzled K-major layout
//     the MMA reads, zero past r;
//   - base rows: the covering blocks of a tile row (at most 17 for 128
//     columns) are staged as they are; the consumers read each 8-column chunk
//     out of two blocks, add the scaled accumulator and write the result to a
//     logical tile; the write-back shifts the logical chunks back onto the
//     16-byte grid of the row and stores whole blocks with 16-byte stores,
//     the partial blocks at the two ends element by element, so no byte
//     outside the tile's columns is written.
// Warp roles (416 threads): warp 0 TMEM and MMA issue, warps 1-8 consumers as
// in expand_tc.cuh; warps 9-11 stage base blocks, warp 12 stages and realigns
// the B tiles one tile ahead (the four stage the rank activations first, all
// slices in one round trip, while the first base tiles are on their way).
// One CTA per SM.
#pragma once

#include "common.cuh"
#include "expand_tc.cuh"
#include "general.cuh"
#include "sched.cuh"
#include "sm100.cuh"

namespace lora {

constexpr int kEuRawBlocks = 17;                  // 16-byte blocks covering 128 columns
constexpr int kEuRawRow = kEuRawBlocks * 16;      // 272 bytes per staged base row
constexpr int kEuRawBase = kExBM * kEuRawRow;     // one staged base tile
constexpr int kEuStageRow = 144;                  // staged rank / B row (<= 9 blocks)

struct ExpandUnalignedParams {
  ExpandArgs a;
  const int32_t* row_list;     // grouped schedule (or null)
  const int32_t* vseg_indptr;  // grouped schedule (or null)
  int nvseg;
  int rpad;                    // 16, 32 or 64
  int tiles_total;
  int tiles_per_cta;
  int tile_prefix[LORA_MAX_SLICES + 1];
  int stages;                  // ring depth (base blocks + B tile + B staging per stage)
  uint32_t idesc;
  uint32_t sw_layout;
  uint32_t rin_bytes;          // one slice of rank activations (128 * rpad * 2)
  uint32_t btile_bytes;        // one B tile (128 * rpad * 2)
  uint32_t stage_bytes;        // kEuRawBase + btile_bytes + 128 * kEuStageRow, 1024-aligned
};

// Copies the aligned 16-byte blocks that cover bytes [a, a + nbytes) (a even)
// to shared memory at dst (16-byte blocks, in order); blocks with no byte of
// the range are not read.
__device__ __forceinline__ void stage_blocks(uint32_t dst, const void* a, int nbytes) {
  if (nbytes <= 0) return;
  const uintptr_t p = reinterpret_cast<uintptr_t>(a);
  const uintptr_t p0 = p & ~static_cast<uintptr_t>(15);
  const uintptr_t p1 = (p + nbytes + 15) & ~static_cast<uintptr_t>(15);
  for (uintptr_t b = p0; b < p1; b += 16)
    cp_async_16_ca(dst + static_cast<uint32_t>(b - p0), reinterpret_cast<const void*>(b));
}

// Row m of a swizzled K-major operand tile (rows of rpad*2 bytes) from `n`
// elements staged by stage_blocks (source offset `off` = source address & 15);
// elements n..rpad-1 are zero.
__device__ __forceinline__ void realign_row(uint8_t* tile, int m, int rpad, const uint8_t* raw,
                                            int off, int n) {
  const uint4* blk = reinterpret_cast<const uint4*>(raw);
  const int nch = rpad / 8;
  for (int c = 0; c < nch; ++c) {
    const int keep = min(8, max(0, n - 8 * c));
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (keep > 0) {
      const int pos = off + 16 * c, b = pos >> 4, sh = pos & 15;
      const uint4 w0 = blk[b];
      const uint4 w1 = (sh != 0 && b + 1 < 9) ? blk[b + 1] : make_uint4(0u, 0u, 0u, 0u);
      v = keep_elems(bytes_at(w0, w1, sh), keep);
    }
    *reinterpret_cast<uint4*>(tile + m * (rpad * 2) + (swz_chunk(c, m, rpad) << 4)) = v;
  }
}

template <class E>
__global__ void __launch_bounds__(kExThreads, 1)
expand_unaligned_kernel(const __grid_constant__ ExpandUnalignedParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const ExpandArgs& p = P.a;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int ncg = (P.tiles_total + P.tiles_per_cta - 1) / P.tiles_per_cta;
  const int slot = blockIdx.x / ncg;
  const int cg = blockIdx.x % ncg;
  const int ntl = cg < P.tiles_total ? (P.tiles_total - cg + ncg - 1) / ncg : 0;
  if (ntl <= 0) return;

  // ---- shared memory: [stages: base blocks | B tile | B staging][logical tile]
  //      [rank activations S x][tokens][barriers]
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int NB = P.stages;
  uint8_t* logical = smem + NB * P.stage_bytes;                  // [128][256 B], swizzled
  uint8_t* rin_p = logical + kExStageBytes;                      // S x [128][rpad*2]
  int* trow = reinterpret_cast<int*>(rin_p + p.S * P.rin_bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(trow + kExBM);
  const uint32_t xfull0 = smem_u32(bars);           // base blocks landed (warps 9-11)
  const uint32_t bfull0 = xfull0 + 8 * NB;          // B tile realigned (warp 12)
  const uint32_t xempty0 = bfull0 + 8 * NB;         // stage consumed (256)
  const uint32_t tfull0 = xempty0 + 8 * NB;         // accumulator buffer complete
  const uint32_t tempty0 = tfull0 + 16;             // accumulator buffer read (256)
  const uint32_t rin_bar = tempty0 + 16;            // rank activations realigned (128)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * NB + 5);
  const uint32_t rin = smem_u32(rin_p);

  if (tid == 32) {
    for (int s = 0; s < NB; ++s) {
      mbar_init(xfull0 + 8 * s, 96);  // copy completions of the three base warps
      mbar_init(bfull0 + 8 * s, 32);  // the B warp's realigned rows
      mbar_init(xempty0 + 8 * s, kExConsumers);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, kExConsumers);
    }
    mbar_init(rin_bar, kExProducers);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kExTmemCols);
    tmem_relinquish();
  }

  PieceInfo pc;
  const int32_t* indptr = P.vseg_indptr ? P.vseg_indptr : p.seg_indptr;
  const bool have = find_piece_warp(indptr, P.vseg_indptr ? nullptr : p.weight_indices,
                                    p.scalings, P.nvseg, p.L, p.tok, kExBM, slot, pc);
  if (!have || pc.per_adapter == 0.f) {
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(*tmem_slot, kExTmemCols);
    }
    return;
  }
  const int rows = pc.hi - pc.lo;
  const int adapter = pc.adapter;
  const float scale = pc.per_adapter;
  const int off0 = p.slices.off[0];
  const int64_t n_tot = p.slices.off[p.S] - off0;

  auto tile_info = [&](int t, int& q, int& c0) {
    const int g = cg + t * ncg;
    q = 0;
#pragma unroll
    for (int k = 1; k < LORA_MAX_SLICES; ++k)
      if (k < p.S && g >= P.tile_prefix[k]) q = k;
    c0 = p.slices.off[q] + (g - P.tile_prefix[q]) * kExBN;
  };
  // first byte of row `row`'s tile segment starting at column c0
  auto seg_addr = [&](int row, int c0) {
    return p.base + static_cast<int64_t>(trow[row]) * p.ld_base + c0;
  };

  // tokens of the piece's rows
  if (warp >= 9) {
    const int m = tid - 9 * 32;
    int sr = pc.lo + (m < rows ? m : 0);
    if (P.row_list) sr = clampi(__ldg(P.row_list + sr), 0, p.tok - 1);
    trow[m] = p.permutation ? clampi(__ldg(p.permutation + sr), 0, p.tok - 1) : sr;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp >= 9) {
    // =========================== producers (128 threads)
    const int m = tid - 9 * 32;
    // base tile t into stage t % NB: block u = j*96 + i -> row u / 17, block u % 17
    auto issue_base = [&](int t, int i) {
      constexpr int kBaseThreads = 96;
      int q, c0;
      tile_info(t, q, c0);
      const int ncols = min(kExBN, p.slices.off[q + 1] - c0);
      const uint32_t st = sbase + (t % NB) * P.stage_bytes;
      for (int u = i; u < kExBM * kEuRawBlocks; u += kBaseThreads) {
        const int row = u / kEuRawBlocks, b = u % kEuRawBlocks;
        if (row >= rows) break;  // u grows with the row
        const uintptr_t a = reinterpret_cast<uintptr_t>(seg_addr(row, c0));
        const uintptr_t a0 = a & ~static_cast<uintptr_t>(15);
        const uintptr_t a1 = (a + 2 * ncols + 15) & ~static_cast<uintptr_t>(15);
        const uintptr_t blk = a0 + 16 * static_cast<uintptr_t>(b);
        if (blk < a1)
          cp_async_16_ca(st + row * kEuRawRow + b * 16, reinterpret_cast<const void*>(blk));
      }
      cp_async_arrive_noinc(xfull0 + 8 * (t % NB));
      cp_async_commit();
    };
    // (1) the rank activations of row m, every slice at once: slice 0 staged
    //     in the logical tile, slice q >= 1 in stage q-1's B staging area
    //     (all still unused; the host keeps S <= stages + 1)
    int sr = pc.lo + (m < rows ? m : 0);
    if (P.row_list) sr = clampi(__ldg(P.row_list + sr), 0, p.tok - 1);
    const uint16_t* rsrc = p.in_r + static_cast<int64_t>(sr) * p.ld_in;
    auto rin_staging = [&](int q) {
      return q == 0 ? logical + m * kEuStageRow
                    : smem + (q - 1) * P.stage_bytes + kEuRawBase + P.btile_bytes +
                          m * kEuStageRow;
    };
    if (m < rows)
      for (int q = 0; q < p.S; ++q) stage_blocks(smem_u32(rin_staging(q)), rsrc + q * p.rs, 2 * p.r);
    cp_async_commit();
    // (2) the base warps send their first tiles out while those land
    const int pre = warp != 12 ? min(NB, ntl) : 0;
    for (int t = 0; t < pre; ++t) issue_base(t, tid - 9 * 32);
    // (3) every group but the base tiles' has landed: realign the rank rows
    cp_async_wait_dyn(pre);
    for (int q = 0; q < p.S; ++q)
      realign_row(rin_p + q * P.rin_bytes, m, P.rpad, rin_staging(q),
                  static_cast<int>(reinterpret_cast<uintptr_t>(rsrc + q * p.rs) & 15),
                  m < rows ? p.r : 0);
    fence_proxy_async_smem();
    mbar_arrive(rin_bar);
    if (warp == 12) {
      // ---- B tiles (warp 12): rows l, l+32, l+64, l+96 of each tile, staged
      //      one tile ahead and realigned; this warp issues no other copies,
      //      so waiting for its own copies waits for nothing else
      const int l = tid - 12 * 32;
      ok = mbar_wait(rin_bar, 0);  // no B staging area holds rank rows any more
      auto brow = [&](int c0, int k, bool& okk) {
        const int n = l + 32 * k;  // output column c0 + n; past the last slice: zero
        okk = c0 + n < p.slices.off[p.S];
        return p.B + (static_cast<int64_t>(adapter) * n_tot + (okk ? c0 - off0 + n : 0)) * p.rs;
      };
      auto stage_b = [&](int t) {
        int q, c0;
        tile_info(t, q, c0);
        const uint32_t st = sbase + (t % NB) * P.stage_bytes;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          bool okk;
          const uint16_t* src = brow(c0, k, okk);
          if (okk)
            stage_blocks(st + kEuRawBase + P.btile_bytes + (l + 32 * k) * kEuStageRow, src,
                         2 * p.r);
        }
        cp_async_commit();
      };
      if (ok && ntl > 0) stage_b(0);
      for (int t = 0; t < ntl && ok; ++t) {
        const int s = t % NB;
        cp_async_wait<0>();  // tile t's rows have landed (the only copies in flight)
        int q, c0;
        tile_info(t, q, c0);
        uint8_t* stp = smem + s * P.stage_bytes;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          bool okk;
          const uint16_t* src = brow(c0, k, okk);
          const int n = l + 32 * k;
          realign_row(stp + kEuRawBase, n, P.rpad,
                      stp + kEuRawBase + P.btile_bytes + n * kEuStageRow,
                      static_cast<int>(reinterpret_cast<uintptr_t>(src) & 15), okk ? p.r : 0);
        }
        fence_proxy_async_smem();
        mbar_arrive(bfull0 + 8 * s);
        // the next tile's rows go out while this tile is multiplied
        if (t + 1 < ntl) {
          const int s1 = (t + 1) % NB;
          if (t + 1 >= NB) ok = mbar_wait(xempty0 + 8 * s1, (((t + 1) / NB) - 1) & 1);
          if (ok) stage_b(t + 1);
        }
      }
    } else {
      // ---- base blocks (warps 9-11), from tile `pre` on
      for (int t = pre; t < ntl && ok; ++t) {
        const int s = t % NB;
        if (t >= NB) ok = mbar_wait(xempty0 + 8 * s, ((t / NB) - 1) & 1);
        if (!ok) break;
        issue_base(t, tid - 9 * 32);
      }
    }
    cp_async_wait<0>();
  } else if (warp == 0) {
    // =========================== MMA issuer
    if (lane == 0) {
      ok = mbar_wait(rin_bar, 0);
      for (int t = 0; t < ntl && ok; ++t) {
        const int s = t % NB, buf = t & 1;
        if (t >= 2) ok = mbar_wait(tempty0 + 8 * buf, ((t - 2) >> 1) & 1);
        if (ok) ok = mbar_wait(bfull0 + 8 * s, (t / NB) & 1);
        if (!ok) break;
        tc_fence_after();
        int q, c0;
        tile_info(t, q, c0);
        const uint32_t a_s = rin + q * P.rin_bytes;
        const uint32_t b_s = sbase + s * P.stage_bytes + kEuRawBase;
        for (int kk = 0; kk < P.rpad / 16; ++kk) {
          const uint64_t ad = make_sdesc(a_s + kk * 32, P.rpad * 2, P.sw_layout);
          const uint64_t bd = make_sdesc(b_s + kk * 32, P.rpad * 2, P.sw_layout);
          tc_mma_f16(tmem + buf * kExBN, ad, bd, P.idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(tfull0 + 8 * buf);
      }
    }
    __syncwarp();
  } else {
    // =========================== consumers (warps 1-8)
    const int quarter = warp & 3;
    const int half = (warp - 1) >> 2;
    const int m = quarter * 32 + lane;  // accumulator row of this thread
    const int ct = tid - 32;            // 0..255 for the write-back
    for (int t = 0; t < ntl; ++t) {
      const int s = t % NB, buf = t & 1;
      if (ok) ok = mbar_wait(xfull0 + 8 * s, (t / NB) & 1);
      if (ok) ok = mbar_wait(tfull0 + 8 * buf, (t >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
      tc_fence_after();
      int q, c0;
      tile_info(t, q, c0);
      const int ncols = min(kExBN, p.slices.off[q + 1] - c0);
      const uint8_t* stp = smem + s * P.stage_bytes;
      const uint32_t tacc = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * kExBN;
      // (a) row m, this warp's half of the columns: the base chunk out of its
      //     two staged blocks, plus scaling * acc, into the logical tile
      const int off = m < rows ? static_cast<int>(
                                     reinterpret_cast<uintptr_t>(seg_addr(m, c0)) & 15)
                               : 0;
      const uint4* raw = reinterpret_cast<const uint4*>(stp + m * kEuRawRow);
      constexpr int kHalfChunks = kExBN / 32;
#pragma unroll
      for (int k0 = 0; k0 < kHalfChunks; ++k0) {
        float v[16];
        if (ok) {
          tmem_ld16(tacc + (half * kHalfChunks + k0) * 16, v);
          tmem_ld_wait();
        }
        if (ok && m < rows) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int c = 2 * (half * kHalfChunks + k0) + hh;  // logical 8-column chunk
            const int pos = off + 16 * c, b = pos >> 4, sh = pos & 15;
            const uint4 w0 = raw[b];
            const uint4 w1 = (sh != 0 && b + 1 < kEuRawBlocks) ? raw[b + 1]
                                                              : make_uint4(0u, 0u, 0u, 0u);
            uint4 w = bytes_at(w0, w1, sh);
            uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 bv = E::u32_to_f2(wv[e]);
              wv[e] = E::f2_to_u32(fmaf(scale, v[8 * hh + 2 * e], bv.x),
                                   fmaf(scale, v[8 * hh + 2 * e + 1], bv.y));
            }
            *reinterpret_cast<uint4*>(logical + m * (kExBN * 2) +
                                      ((c ^ (m & (kExCh - 1))) << 4)) = w;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * buf);
      named_bar_sync(1, kExConsumers);  // every row of the logical tile is written
      mbar_arrive(xempty0 + 8 * s);     // the staged blocks may be refilled
      // (b) write-back on the row's own 16-byte grid: block u = j*256 + ct ->
      //     row u / 17, block u % 17; whole blocks with 16-byte stores, the
      //     partial blocks at the two ends element by element
      if (ok) {
        for (int j = 0; j < (kExBM * kEuRawBlocks + kExConsumers - 1) / kExConsumers; ++j) {
          const int u = j * kExConsumers + ct;
          const int row = u / kEuRawBlocks, b = u % kEuRawBlocks;
          if (row >= rows) continue;
          uint16_t* sa = seg_addr(row, c0);
          const int roff = static_cast<int>(reinterpret_cast<uintptr_t>(sa) & 15);
          const uintptr_t a0 = reinterpret_cast<uintptr_t>(sa) & ~static_cast<uintptr_t>(15);
          const uintptr_t a1 =
              (reinterpret_cast<uintptr_t>(sa) + 2 * ncols + 15) & ~static_cast<uintptr_t>(15);
          const uintptr_t ga = a0 + 16 * static_cast<uintptr_t>(b);
          if (ga >= a1) continue;
          // logical bytes [16b - roff, 16b - roff + 16): chunks k and k + 1
          const int lpos = 16 * b - roff;
          const int k = lpos >= 0 ? lpos >> 4 : -1;
          const int sh = lpos - 16 * k;
          const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
          const uint4 l0 = k >= 0 ? *reinterpret_cast<const uint4*>(
                                        logical + row * (kExBN * 2) +
                                        ((k ^ (row & (kExCh - 1))) << 4))
                                  : zero;
          const uint4 l1 = (sh != 0 && k + 1 < kExCh)
                               ? *reinterpret_cast<const uint4*>(
                                     logical + row * (kExBN * 2) +
                                     (((k + 1) ^ (row & (kExCh - 1))) << 4))
                               : zero;
          const uint4 w = bytes_at(l0, l1, sh);
          const int e0 = lpos / 2;  // logical element of the block's first element
          if (e0 >= 0 && e0 + 8 <= ncols) {
            *reinterpret_cast<uint4*>(ga) = w;
          } else {
            const uint16_t* we = reinterpret_cast<const uint16_t*>(&w);
            uint16_t* gp = reinterpret_cast<uint16_t*>(ga);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (e0 + i >= 0 && e0 + i < ncols) gp[i] = we[i];
          }
        }
      }
      named_bar_sync(1, kExConsumers);  // the logical tile may be rewritten
    }
  }

  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kExTmemCols);
  }
}

}  // namespace lora
