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
//     cp.async and shifted into the swizzled K-major layout the MMA reads,
//     zero past r;
//   - base rows: the covering blocks of a tile row (at most 17 for 128
//     columns) are staged as they are, on the row's own 16-byte grid.  A
//     consumer thread walks its row once, word by word: the base word of
//     columns 2k, 2k+1 is read at byte offset off + 4k of the staged row
//     (off = the row's address & 15), the scaled accumulator is added, and
//     the result is written back in place at the same byte offset.  Both
//     shifts are a word index plus a 0- or 16-bit funnel shift, so the walk
//     costs a load, a shift, the arithmetic and a store per word.  The
//     write-back then stores whole blocks with 16-byte stores, the partial
//     blocks at the two ends element by element, so no byte outside the
//     tile's columns is written.
// Warp roles (416 threads): warp 0 TMEM and MMA issue; warps 1-4 and 5-8 are
// two consumer groups that take alternate tiles (each group reads one of the
// two accumulator buffers, so two tile epilogues overlap); warps 9-11 stage
// base blocks; warp 12 stages and realigns the B tiles one tile ahead.  The
// four producer warps copy the rank activations (all slices, one round trip)
// and the first B tile as soon as the piece is known, before the row tokens
// arrive, then go on with the first base tiles; consumer group 0 shifts the
// rank rows and group 1 the first B tile into place when they land.  Two
// CTAs per SM when the stages fit.
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
constexpr int kEuGroup = kExConsumers / 2;        // threads of one consumer group
static_assert(kExBN == 128, "the element-aligned expand stages 128-column tiles");

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
  uint32_t srow;               // one staged rank / B row: 16 * (rpad / 8 + 1) bytes
  uint32_t stage_bytes;        // kEuRawBase + btile_bytes + 128 * srow, 1024-aligned
  int rin_in_stage0;           // stage 0's B staging holds rank rows too
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
// elements staged by stage_blocks (source offset `off` = source address & 15):
// word k of the row is the 4 bytes at staged byte off + 4k (a word index and a
// 0- or 16-bit funnel shift); elements n..rpad-1 are zero.
__device__ __forceinline__ void realign_row(uint8_t* tile, int m, int rpad, const uint8_t* raw,
                                            int off, int n) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(raw) + (off >> 2);
  const uint32_t fs = static_cast<uint32_t>(off & 2) * 8;
  const int nch = rpad / 8;
  uint32_t prev = w[0];
  for (int c = 0; c < nch; ++c) {
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t next = w[4 * c + i + 1];
      o[i] = __funnelshift_r(prev, next, fs);
      prev = next;
    }
    const uint4 v = keep_elems(make_uint4(o[0], o[1], o[2], o[3]), n - 8 * c);
    *reinterpret_cast<uint4*>(tile + m * (rpad * 2) + (swz_chunk(c, m, rpad) << 4)) = v;
  }
}

// Barrier of one consumer group (named barriers 1 and 2; constant ids keep
// the CTA's barrier count at three).
__device__ __forceinline__ void group_sync(int grp) {
  if (grp == 0)
    named_bar_sync(1, kEuGroup);
  else
    named_bar_sync(2, kEuGroup);
}

template <class E>
__global__ void __launch_bounds__(kExThreads, 2)
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

  // ---- shared memory: [stages: base blocks | B tile | B staging]
  //      [rank activations S x][tokens][barriers]
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int NB = P.stages;
  uint8_t* rin_p = smem + NB * P.stage_bytes;                    // S x [128][rpad*2]
  int* trow = reinterpret_cast<int*>(rin_p + p.S * P.rin_bytes);
  uintptr_t* rsa = reinterpret_cast<uintptr_t*>(trow + kExBM);  // [2][128] row addresses
  uint64_t* bars = reinterpret_cast<uint64_t*>(rsa + 2 * kExBM);
  const uint32_t xfull0 = smem_u32(bars);           // base blocks landed (warps 9-11)
  const uint32_t bfull0 = xfull0 + 8 * NB;          // B tile realigned (warp 12)
  const uint32_t xempty0 = bfull0 + 8 * NB;         // stage consumed (one group)
  const uint32_t tfull0 = xempty0 + 8 * NB;         // accumulator buffer complete
  const uint32_t tempty0 = tfull0 + 16;             // accumulator buffer read (one group)
  const uint32_t rin_bar = tempty0 + 16;            // rank activations realigned (group 0)
  const uint32_t rin_land = rin_bar + 8;            // rank rows and first B tile landed (128)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * NB + 6);
  const uint32_t rin = smem_u32(rin_p);

  if (tid == 32) {
    for (int s = 0; s < NB; ++s) {
      mbar_init(xfull0 + 8 * s, 96);  // copy completions of the three base warps
      mbar_init(bfull0 + 8 * s, 32);  // the B warp's realigned rows
      mbar_init(xempty0 + 8 * s, kEuGroup);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, kEuGroup);
    }
    mbar_init(rin_bar, kEuGroup);
    mbar_init(rin_land, kExProducers);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kExTmemCols);
    tmem_relinquish();
  }
  // the grouping pass ahead of this kernel (when there is one) has finished
  griddep_wait();

  // a block slot's piece starts at row slot * 128: the producers fetch the
  // tokens of its rows while the tables are read
  const bool block_slot = slot < (p.tok + kExBM - 1) / kExBM;
  int spec_tok = 0;
  if (warp >= 9 && block_slot) {
    int sr = min(slot * kExBM + (tid - 9 * 32), p.tok - 1);
    if (P.row_list) sr = clampi(__ldg(P.row_list + sr), 0, p.tok - 1);
    spec_tok = p.permutation ? clampi(__ldg(p.permutation + sr), 0, p.tok - 1) : sr;
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
  // the rank activations of piece row m (any slice) and where their covering
  // blocks are staged: the first slices in the last stage's base area, the
  // others in the B staging areas of stages NB-1, NB-2, ... (the host keeps S
  // within that room); stage 0's B staging, which the first B tile needs, is
  // the last one used
  auto rin_src = [&](int m) {
    int sr = pc.lo + (m < rows ? m : 0);
    if (P.row_list) sr = clampi(__ldg(P.row_list + sr), 0, p.tok - 1);
    return p.in_r + static_cast<int64_t>(sr) * p.ld_in;
  };
  auto rin_staging = [&](int q, int m) {
    const int nfit = kEuRawBase / (kExBM * static_cast<int>(P.srow));
    if (q < nfit) return smem + (NB - 1) * P.stage_bytes + (q * kExBM + m) * P.srow;
    return smem + (NB - 1 - (q - nfit)) * P.stage_bytes + kEuRawBase + P.btile_bytes + m * P.srow;
  };

  // B rows of a tile: output column c0 + n (n = 0..127) is B row
  // adapter * n_tot + c0 - off0 + n; past the last slice, zero
  auto brow = [&](int c0, int n, bool& okk) {
    okk = c0 + n < p.slices.off[p.S];
    return p.B + (static_cast<int64_t>(adapter) * n_tot + (okk ? c0 - off0 + n : 0)) * p.rs;
  };
  auto stage_b_row = [&](int t, int n) {  // covering blocks of tile t's B row n
    int q, c0;
    tile_info(t, q, c0);
    bool okk;
    const uint16_t* src = brow(c0, n, okk);
    if (okk)
      stage_blocks(sbase + (t % NB) * P.stage_bytes + kEuRawBase + P.btile_bytes + n * P.srow,
                   src, 2 * p.r);
  };
  auto realign_b_row = [&](int t, int n) {  // tile t's B row n into the stage's B tile
    int q, c0;
    tile_info(t, q, c0);
    bool okk;
    const uint16_t* src = brow(c0, n, okk);
    uint8_t* stp = smem + (t % NB) * P.stage_bytes;
    realign_row(stp + kEuRawBase, n, P.rpad, stp + kEuRawBase + P.btile_bytes + n * P.srow,
                static_cast<int>(reinterpret_cast<uintptr_t>(src) & 15), okk ? p.r : 0);
  };
  // the first B tile goes out with the rank activations unless stage 0's B
  // staging holds rank rows; consumer group 1 then shifts it into place
  const bool b0_early = !P.rin_in_stage0;

  // base tile t into stage t % NB: block u = i + 96 j -> row u / 17, block
  // u % 17 (96 = 5 * 17 + 11), so a warp copies two rows' blocks at a time.
  // Eight blocks at a time: their row tokens are read first, then the eight
  // copies issue back to back (a copy may not pass a shared-memory load).
  auto issue_base = [&](int t, int i) {
    constexpr int kBaseThreads = 96;
    constexpr int kBatch = 8;
    int q, c0;
    tile_info(t, q, c0);
    const int ncols = min(kExBN, p.slices.off[q + 1] - c0);
    const uint32_t st = sbase + (t % NB) * P.stage_bytes;
    int row = i / kEuRawBlocks, b = i - row * kEuRawBlocks;
    while (row < rows) {
      const uint8_t* src[kBatch];
      uint32_t dst[kBatch];
      bool go[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        go[k] = row < rows;
        const uintptr_t a = reinterpret_cast<uintptr_t>(seg_addr(go[k] ? row : 0, c0));
        const uintptr_t a0 = a & ~static_cast<uintptr_t>(15);
        const uintptr_t a1 = (a + 2 * ncols + 15) & ~static_cast<uintptr_t>(15);
        const uintptr_t blk = a0 + 16 * static_cast<uintptr_t>(b);
        go[k] = go[k] && blk < a1;
        src[k] = reinterpret_cast<const uint8_t*>(blk);
        dst[k] = st + row * kEuRawRow + b * 16;
        row += kBaseThreads / kEuRawBlocks;
        b += kBaseThreads % kEuRawBlocks;
        if (b >= kEuRawBlocks) {
          b -= kEuRawBlocks;
          ++row;
        }
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k)
        if (go[k]) cp_async_16(dst[k], src[k], 16u);
    }
    cp_async_arrive_noinc(xfull0 + 8 * (t % NB));
    cp_async_commit();
  };
  const int pre = min(NB - 1, ntl);  // base tiles sent at once
  if (warp >= 9) {
    const int m = tid - 9 * 32;
    // tokens of the piece's rows (a block slot's are already on their way);
    // the loads go out before the copies below
    int sr = pc.lo + (m < rows ? m : 0);
    if (P.row_list) sr = clampi(__ldg(P.row_list + sr), 0, p.tok - 1);
    const int tk = block_slot ? spec_tok
                              : (p.permutation ? __ldg(p.permutation + sr) : sr);
    // the rank activations of row m (every slice, one round trip) and, from
    // warp 12, the first B tile
    const uint16_t* rsrc = p.in_r + static_cast<int64_t>(sr) * p.ld_in;
    if (m < rows)
      for (int q = 0; q < p.S; ++q)
        stage_blocks(smem_u32(rin_staging(q, m)), rsrc + q * p.rs, 2 * p.r);
    if (warp == 12 && b0_early)
#pragma unroll
      for (int k = 0; k < 4; ++k) stage_b_row(0, (tid - 12 * 32) + 32 * k);
    cp_async_commit();
    trow[m] = clampi(tk, 0, p.tok - 1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp >= 9) {
    // =========================== producers (128 threads)
    // rin_land completes once the copies issued before the CTA barrier have
    // landed; consumer groups 0 and 1 then shift the rank rows and the first
    // B tile into place.  Then the first base tiles (not into the last stage,
    // whose base area holds staged rank rows until rin_bar).
    cp_async_arrive_noinc(rin_land);
    if (warp != 12)
      for (int t = 0; t < pre; ++t) issue_base(t, tid - 9 * 32);
    if (warp == 12) {
      // ---- B tiles (warp 12): rows l, l+32, l+64, l+96 of each tile, staged
      //      one tile ahead and realigned; this warp's copies are only its
      //      own, so waiting for them waits for nothing else
      const int l = tid - 12 * 32;
      auto stage_b = [&](int t) {
#pragma unroll
        for (int k = 0; k < 4; ++k) stage_b_row(t, l + 32 * k);
        cp_async_commit();
      };
      bool rin_done = false;
      if (!b0_early) {  // stage 0's B staging held rank rows
        ok = mbar_wait(rin_bar, 0);
        rin_done = true;
        if (ok) stage_b(0);
      }
      for (int t = 0; t < ntl && ok; ++t) {
        const int s = t % NB;
        if (t > 0 || !b0_early) {
          cp_async_wait<0>();  // tile t's rows have landed
#pragma unroll
          for (int k = 0; k < 4; ++k) realign_b_row(t, l + 32 * k);
          fence_proxy_async_smem();
          mbar_arrive(bfull0 + 8 * s);
        }
        // the next tile's rows go out while this tile is multiplied
        if (t + 1 < ntl) {
          const int s1 = (t + 1) % NB;
          if (!rin_done) {  // no B staging area holds rank rows any more
            ok = mbar_wait(rin_bar, 0);
            rin_done = true;
          }
          if (ok && t + 1 >= NB) ok = mbar_wait(xempty0 + 8 * s1, (((t + 1) / NB) - 1) & 1);
          if (ok) stage_b(t + 1);
        }
      }
    } else {
      // ---- base blocks (warps 9-11), from tile `pre` on
      for (int t = pre; t < ntl && ok; ++t) {
        const int s = t % NB;
        // the last stage holds staged rank rows until they are realigned
        if (t == NB - 1) ok = mbar_wait(rin_bar, 0);
        if (ok && t >= NB) ok = mbar_wait(xempty0 + 8 * s, ((t / NB) - 1) & 1);
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
    // =========================== consumers: group g (warps 1-4 or 5-8) takes
    // tiles g, g+2, ... and accumulator buffer g
    const int quarter = warp & 3;
    const int grp = (warp - 1) >> 2;
    const int m = quarter * 32 + lane;      // accumulator row of this thread
    const int gt = tid - 32 - grp * kEuGroup;  // 0..127 for the write-back
    uintptr_t* my_rsa = rsa + grp * kExBM;
    if (grp == 0) {
      // the rank rows of piece row gt, shifted into the MMA layout
      ok = mbar_wait(rin_land, 0);
      const uint16_t* rsrc = rin_src(gt);
      if (ok)
        for (int q = 0; q < p.S; ++q)
          realign_row(rin_p + q * P.rin_bytes, gt, P.rpad, rin_staging(q, gt),
                      static_cast<int>(reinterpret_cast<uintptr_t>(rsrc + q * p.rs) & 15),
                      gt < rows ? p.r : 0);
      fence_proxy_async_smem();
      mbar_arrive(rin_bar);
    } else if (b0_early) {
      // row gt of the first B tile; one warp of the group publishes it
      ok = mbar_wait(rin_land, 0);
      if (ok) realign_b_row(0, gt);
      fence_proxy_async_smem();
      group_sync(1);
      if (warp == 5) mbar_arrive(bfull0);
    }
    for (int t = grp; t < ntl; t += 2) {
      const int s = t % NB, buf = t & 1;
      if (ok) ok = mbar_wait(xfull0 + 8 * s, (t / NB) & 1);
      if (ok) ok = mbar_wait(tfull0 + 8 * buf, (t >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
      tc_fence_after();
      int q, c0;
      tile_info(t, q, c0);
      const int ncols = min(kExBN, p.slices.off[q + 1] - c0);
      uint8_t* stp = smem + s * P.stage_bytes;
      const uint32_t tacc = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * kExBN;
      // (a) row m, all 128 columns, in place: word k (columns 2k, 2k+1) of the
      //     row sits at staged byte roff + 4k, i.e. staged words qw + k and
      //     qw + k + 1 funnel-shifted by fs; the result goes back to the same
      //     bytes (the staged word qw + k - 1 + hs is written once both words
      //     that feed it have been read)
      if (ok) {
        const uintptr_t sa = m < rows ? reinterpret_cast<uintptr_t>(seg_addr(m, c0)) : 0;
        const int roff = static_cast<int>(sa & 15);
        uint8_t* rowp = stp + m * kEuRawRow;
        uint32_t* w = reinterpret_cast<uint32_t*>(rowp) + (roff >> 2);
        const uint32_t fs = static_cast<uint32_t>(roff & 2) * 8;
        const int hs = (roff >> 1) & 1;
        uint32_t* wo = w + hs - 1;
        uint32_t bprev = w[0];
        uint32_t oprev = 0u;
#pragma unroll
        for (int j = 0; j < kExBN / 16; ++j) {
          float v[16];
          tmem_ld16(tacc + 16 * j, v);
          tmem_ld_wait();
          if (m < rows) {
            // the group's eight staged words are read before any of its
            // results is written back over them
            uint32_t bw[9];
            bw[0] = bprev;
#pragma unroll
            for (int i = 1; i <= 8; ++i) bw[i] = w[8 * j + i];
            bprev = bw[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int k = 8 * j + i;
              const float2 bv = E::u32_to_f2(__funnelshift_r(bw[i], bw[i + 1], fs));
              const uint32_t ow =
                  E::f2_to_u32(fmaf(scale, v[2 * i], bv.x), fmaf(scale, v[2 * i + 1], bv.y));
              if (k > 0 || hs) wo[k] = __funnelshift_r(oprev, ow, fs);
              oprev = ow;
            }
          }
        }
        if (m < rows) {
          wo[kExBN / 2] = __funnelshift_r(oprev, 0u, fs);
          // the partial blocks at the two ends of the row (the write-back
          // takes the whole ones), in aligned pieces of 8, 4 and 2 bytes
          my_rsa[m] = sa;
          const uintptr_t se = sa + 2 * static_cast<uintptr_t>(ncols);
          const uintptr_t a0 = sa & ~static_cast<uintptr_t>(15);
          const int nb = static_cast<int>(((se + 15) & ~static_cast<uintptr_t>(15)) - a0) >> 4;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int b = e == 0 ? 0 : nb - 1;
            if (e == 1 && b == 0) break;
            const uintptr_t ga = a0 + 16 * static_cast<uintptr_t>(b);
            if (ga >= sa && ga + 16 <= se) continue;  // whole block
            const int i1 = static_cast<int>(min(se - ga, static_cast<uintptr_t>(16))) >> 1;
            for (int i = ga >= sa ? 0 : static_cast<int>(sa - ga) >> 1; i < i1;) {
              const uint8_t* src = rowp + 16 * b + 2 * i;
              uint8_t* dst = reinterpret_cast<uint8_t*>(ga) + 2 * i;
              if ((i & 3) == 0 && i + 4 <= i1) {
                stg64(dst, *reinterpret_cast<const uint2*>(src));
                i += 4;
              } else if ((i & 1) == 0 && i + 2 <= i1) {
                stg32(dst, *reinterpret_cast<const uint32_t*>(src));
                i += 2;
              } else {
                stg16(dst, *reinterpret_cast<const uint16_t*>(src));
                i += 1;
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * buf);
      group_sync(grp);  // every row of the tile is updated
      // (b) write-back of the whole blocks on the rows' own 16-byte grid:
      //     block u = gt + 128 j -> row u / 17, block u % 17 (128 = 7 * 17 + 9)
      //     Four blocks at a time: every shared-memory load first, then the
      //     four stores (global-space stores: the next loads need not wait on them).
      if (ok) {
        constexpr int kBatch = 4;
        int row = gt / kEuRawBlocks, b = gt - row * kEuRawBlocks;
        while (row < rows) {
          uint4 val[kBatch];
          uintptr_t ga[kBatch];
          bool go[kBatch];
#pragma unroll
          for (int k = 0; k < kBatch; ++k) {
            go[k] = row < rows;
            const uintptr_t sa = my_rsa[go[k] ? row : 0];
            ga[k] = (sa & ~static_cast<uintptr_t>(15)) + 16 * static_cast<uintptr_t>(b);
            go[k] = go[k] && ga[k] >= sa && ga[k] + 16 <= sa + 2 * static_cast<uintptr_t>(ncols);
            val[k] = *reinterpret_cast<const uint4*>(stp + (go[k] ? row : 0) * kEuRawRow + 16 * b);
            row += kEuGroup / kEuRawBlocks;
            b += kEuGroup % kEuRawBlocks;
            if (b >= kEuRawBlocks) {
              b -= kEuRawBlocks;
              ++row;
            }
          }
#pragma unroll
          for (int k = 0; k < kBatch; ++k)
            if (go[k]) stg128(reinterpret_cast<void*>(ga[k]), val[k]);
        }
      }
      group_sync(grp);  // the stage may be refilled
      mbar_arrive(xempty0 + 8 * s);
    }
  }

  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kExTmemCols);
  }
}

}  // namespace lora
