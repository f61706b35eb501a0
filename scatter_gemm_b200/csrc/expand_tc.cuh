// expand_tc.cuh -- tensor-core expand with a fused scale-and-add scatter
// epilogue, for 16-byte-aligned inputs (sm_100a).
//
// One CTA handles one piece (<= 128 sorted rows of one segment) times a run of
// 128-column tiles of the base output.  For every tile (slice q, columns
// [c0, c0+128) inside the slice):
//     D[128 x 128] = R_q[128 x r] * B_a[c0-off0 : c0-off0+128, 0:r]^T
// on tcgen05.mma (M = 128 tokens, N = 128 columns, K = r padded to 16/32/64)
// with a double-buffered fp32 accumulator in TMEM, and then
//     base[perm[row], c] = round(base[perm[row], c] + scaling[a] * D[row, c]).
// This is the expand and the "scatter epilogue" of the sgl-kernel-xpu page
// ("Decode LoRA kernels are optimized", section "Summary"), rebuilt for B200.
//
// Warp roles (416 threads):
//   warp 0      TMEM allocation; lane 0 loads B tiles by TMA (the tensor map's
//               inner extent is r, so the storage padding j >= r reads as zero)
//               and issues the MMAs;
//   warps 1-8   consumers, two per TMEM lane quarter (one per half of the
//               tile's columns): (a) one accumulator row per thread updates its
//               staged base row in shared memory, (b) the eight warps write the
//               tile back with coalesced 16-byte stores;
//   warps 9-12  producers: the piece's rank activations (cp.async, whose
//               partial-size form zero-fills the padding j >= r) overlapped
//               with the first base tiles, then the base tiles with coalesced
//               16-byte cp.async (two 256-byte rows per warp instruction) into a
//               ring of stages; completion reaches the consumers through
//               cp.async.mbarrier.arrive, so producers never block on a tile.
// The 16-byte chunks of a staged row are XOR-swizzled by the row index, so the
// row-per-thread phase and the coalesced phases are free of bank conflicts.
#pragma once

#include "common.cuh"
#include "general.cuh"
#include "sched.cuh"
#include "sm100.cuh"

#ifndef LORA_EXPAND_INTERLEAVE
#define LORA_EXPAND_INTERLEAVE 1
#endif

namespace lora {

#ifndef LORA_EXPAND_BN
#define LORA_EXPAND_BN 128  // columns per tile (64, 128 or 256)
#endif
#ifndef LORA_EXPAND_LD_BATCH
#define LORA_EXPAND_LD_BATCH 2  // 16-column TMEM loads in flight per consumer thread
#endif
#ifndef LORA_EXPAND_MIN_BLOCKS
#define LORA_EXPAND_MIN_BLOCKS 2  // co-resident CTAs per SM the register budget must allow
#endif
constexpr int kExBM = 128;               // rows per piece
constexpr int kExBN = LORA_EXPAND_BN;    // columns per tile
constexpr int kExCh = kExBN / 8;         // 16-byte chunks per staged row
constexpr int kExTmemCols = 2 * kExBN;   // double-buffered accumulator
constexpr int kExConsumers = 256;        // warps 1-8: two warps per TMEM lane quarter
constexpr int kExProducers = 128;        // warps 9-12
constexpr int kExThreads = 32 + kExConsumers + kExProducers;
constexpr int kExStageBytes = kExBM * kExBN * 2;  // one staged base tile
constexpr int kExLdBatch = LORA_EXPAND_LD_BATCH;   // TMEM chunks loaded per wait
static_assert((kExBN / 32) % kExLdBatch == 0, "batch must divide a half tile");
static_assert(kExBN == 64 || kExBN == 128 || kExBN == 256, "expand tile width");

struct ExpandTcParams {
  CUtensorMap tmap_B;  // 2-D [L*N_tot rows, r cols] (row stride rs), box {rpad, 128}
  CUtensorMap tmap_R;  // 3-D [tok rows, S slices, r cols] of in_r, box {rpad, 1, 128}
  int rin_tma;         // the rank activations by TMA (sorted rows contiguous: no grouping)
  ExpandArgs a;
  const int32_t* row_list;     // grouped schedule (or null)
  const int32_t* vseg_indptr;  // grouped schedule (or null)
  int nvseg;
  int rpad;                    // 16, 32 or 64
  int tiles_total;             // 128-column tiles over all slices
  int tiles_per_cta;
  int tile_prefix[LORA_MAX_SLICES + 1];  // first tile of each slice
  int base_stages;             // ring depth of base tiles
  int b_stages;                // ring depth of B tiles
  uint32_t idesc;
  uint32_t sw_layout;          // UMMA layout code of rows of rpad*2 bytes
  uint32_t rin_bytes;          // one slice of staged rank activations (128 * rpad * 2)
  uint32_t btile_bytes;        // one B tile (128 * rpad * 2)
};

// physical 16-byte chunk of logical chunk c in a row of the rank-activation /
// B tiles (rows of rpad*2 bytes, canonical UMMA swizzle)
__device__ __forceinline__ int swz_chunk(int c, int m, int rpad) {
  return rpad == 64 ? (c ^ (m & 7)) : rpad == 32 ? (c ^ ((m >> 1) & 3)) : (c ^ ((m >> 2) & 1));
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

template <class E>
__global__ void __launch_bounds__(kExThreads, LORA_EXPAND_MIN_BLOCKS)
expand_tc_kernel(const __grid_constant__ ExpandTcParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const ExpandArgs& p = P.a;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int ncg = (P.tiles_total + P.tiles_per_cta - 1) / P.tiles_per_cta;
  const int slot = blockIdx.x / ncg;
  const int cg = blockIdx.x % ncg;
#if LORA_EXPAND_INTERLEAVE
  // column group cg takes tiles cg, cg+ncg, cg+2*ncg, ...: the CTAs of one piece
  // (consecutive blocks, launched together) stream adjacent column tiles of the
  // same rows at about the same time, so DRAM sees long runs of each row
  const int ntl = cg < P.tiles_total ? (P.tiles_total - cg + ncg - 1) / ncg : 0;
#define LORA_TILE(t) (cg + (t) * ncg)
#else
  const int t_begin = cg * P.tiles_per_cta;
  const int ntl = min(P.tiles_total, t_begin + P.tiles_per_cta) - t_begin;
#define LORA_TILE(t) (t_begin + (t))
#endif
  if (ntl <= 0) return;

  // ---- shared memory: [base ring][rank activations S x][B ring][token of each row][barriers]
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t base_ring = sbase;
  const uint32_t rin = base_ring + P.base_stages * kExStageBytes;
  const uint32_t bring = rin + p.S * P.rin_bytes;
  int* trow = reinterpret_cast<int*>(smem + (bring - sbase) + P.b_stages * P.btile_bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(trow + kExBM);
  const uint32_t bfull0 = smem_u32(bars);
  const uint32_t bempty0 = bfull0 + 8 * P.b_stages;
  const uint32_t tfull0 = bempty0 + 8 * P.b_stages;  // 2 accumulator buffers
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t rin_bar = tempty0 + 16;
  const uint32_t xfull0 = rin_bar + 8;                  // base tile landed
  const uint32_t xempty0 = xfull0 + 8 * P.base_stages;  // base tile written back
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * P.b_stages + 5 +
                                                    2 * P.base_stages);

  // Barriers (one consumer thread; the B ring's by warp 0, which uses them
  // before the CTA barrier) and TMEM (warp 0) first, so that both overlap the
  // table reads.
  if (tid == 0) {
    for (int s = 0; s < P.b_stages; ++s) {
      mbar_init(bfull0 + 8 * s, 1);
      mbar_init(bempty0 + 8 * s, 1);
    }
    mbar_init(rin_bar, P.rin_tma ? 1 : kExProducers);
    fence_mbar_init();
  }
  if (tid == 32) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, kExConsumers);
    }
    for (int s = 0; s < P.base_stages; ++s) {
      mbar_init(xfull0 + 8 * s, kExProducers);
      mbar_init(xempty0 + 8 * s, kExConsumers);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&P.tmap_B);
      if (P.rin_tma) tma_prefetch_desc(&P.tmap_R);
    }
    tmem_alloc(smem_u32(tmem_slot), kExTmemCols);
    tmem_relinquish();
  }
  // the grouping pass ahead of this kernel (when there is one) has finished
  griddep_wait();

  // Producer thread pt owns row pt of the piece.  Rows of a block slot start
  // at slot*128: their sorted rows and tokens are fetched while the tables are read.
  const bool producer = warp >= 9;
  const int pt = tid - 9 * 32;
  const bool block_slot = slot < (p.tok + kExBM - 1) / kExBM;
  int spec_srow = 0, spec_tok = 0;
  if (producer && block_slot) {
    spec_srow = min(slot * kExBM + pt, p.tok - 1);
    if (P.row_list) spec_srow = clampi(__ldg(P.row_list + spec_srow), 0, p.tok - 1);
    spec_tok = p.permutation ? clampi(__ldg(p.permutation + spec_srow), 0, p.tok - 1)
                             : spec_srow;
  }
  PieceInfo pc;
  const int32_t* indptr = P.vseg_indptr ? P.vseg_indptr : p.seg_indptr;
  const bool have = find_piece_warp(indptr, P.vseg_indptr ? nullptr : p.weight_indices,
                                    p.scalings, P.nvseg, p.L, p.tok, kExBM, slot, pc);
  // no rows here, or a zero scaling (the rows then stay bit-identical): leave
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

  // tile t of this CTA -> (slice, first column)
  auto tile_info = [&](int t, int& q, int& c0) {
    const int g = LORA_TILE(t);
    q = 0;
#pragma unroll
    for (int k = 1; k < LORA_MAX_SLICES; ++k)
      if (k < p.S && g >= P.tile_prefix[k]) q = k;
    c0 = p.slices.off[q] + (g - P.tile_prefix[q]) * kExBN;
  };
  // base tile t into ring stage s: chunk u = j*128 + pt -> row u / kExCh,
  // logical chunk u % kExCh (two 256-byte rows per warp instruction)
  // A producer's rows are the same for every tile (pt / kExCh + j * 128 /
  // kExCh), so their tokens are read from shared memory once (ptok) and the
  // copies of a tile issue back to back, none waiting on a shared-memory load.
  int ptok[kExCh];
  auto issue_tile = [&](int t, int s) {
    int q, c0;
    tile_info(t, q, c0);
    const int cend = p.slices.off[q + 1];
    const uint32_t stage = base_ring + s * kExStageBytes;
#pragma unroll
    for (int j = 0; j < kExCh; ++j) {
      const int u = j * kExBM + pt;
      const int row = u / kExCh, c = u % kExCh;
      const int col = c0 + 8 * c;
      // rows past the piece and columns past the slice are not loaded: the
      // epilogue never stores them
      if (row < rows && col < cend)
        cp_async_16(stage + row * (kExBN * 2) + ((c ^ (row & (kExCh - 1))) << 4),
                    p.base + static_cast<int64_t>(ptok[j]) * p.ld_base + col, 16u);
    }
  };
  // The first base tile goes out before the CTA barrier, the others after it:
  // a second early tile held the barrier back while its copies issued
  // (measured up to 1.8 us slower, at no size faster).
  const int pre = min(1, ntl);
  // The first B tiles depend only on the adapter: warp 0 requests them now,
  // before the row tokens are known and the CTA barrier is passed.
  const int pre_b = min(P.b_stages, ntl);
  if (tid == 0) {
    for (int t = 0; t < pre_b; ++t) {
      int q, c0;
      tile_info(t, q, c0);
      mbar_arrive_expect_tx(bfull0 + 8 * t, P.btile_bytes);
      tma_load_2d(bring + t * P.btile_bytes, &P.tmap_B, bfull0 + 8 * t, 0,
                  static_cast<int>(adapter * n_tot + (c0 - off0)));
    }
    // Without grouping the piece's rows are contiguous sorted rows: the rank
    // activations of every slice are one TMA box each (columns j >= r and
    // rows past the tensor read as zero; rows past the piece feed
    // accumulator rows that are never stored).
    if (P.rin_tma) {
      mbar_arrive_expect_tx(rin_bar, static_cast<uint32_t>(p.S) * P.rin_bytes);
      for (int q = 0; q < p.S; ++q)
        tma_load_3d(rin + q * P.rin_bytes, &P.tmap_R, rin_bar, 0, q, pc.lo);
    }
  }

  if (producer) {
    // Row tables, then every load that needs no barrier goes out before the
    // CTA-wide barrier: the rank activations of row pt (zero-filled beyond r,
    // their own cp.async group) and the first `pre` base tiles (one group each).
    const int m = pt;
    int sr, tk;
    if (block_slot) {
      sr = spec_srow;
      tk = spec_tok;
    } else {
      sr = pc.lo + (m < rows ? m : 0);
      if (P.row_list) sr = clampi(__ldg(P.row_list + sr), 0, p.tok - 1);
      tk = p.permutation ? clampi(__ldg(p.permutation + sr), 0, p.tok - 1) : sr;
    }
    trow[m] = tk;
    const bool row_ok = m < rows && !P.rin_tma;
    const uint16_t* src0 = p.in_r + static_cast<int64_t>(sr) * p.ld_in;
    const int nchunk = P.rpad / 8;
    for (int q = 0; q < (P.rin_tma ? 0 : p.S); ++q) {
      for (int c = 0; c < nchunk; ++c) {
        const int left = p.r - 8 * c;
        const uint32_t nb = row_ok ? static_cast<uint32_t>(max(0, min(left, 8)) * 2) : 0u;
        const uint32_t dst = rin + q * P.rin_bytes + m * (P.rpad * 2) +
                             (swz_chunk(c, m, P.rpad) << 4);
        // rows past the piece are not loaded (their accumulator rows are never
        // stored); a row of the piece is zero-filled beyond r
        if (row_ok)
          cp_async_16(dst, nb ? static_cast<const void*>(src0 + q * p.rs + 8 * c)
                              : static_cast<const void*>(p.in_r), nb);
      }
    }
    cp_async_commit();
    named_bar_sync(2, kExProducers);  // trow of every row is in shared memory
#pragma unroll
    for (int j = 0; j < kExCh; ++j) ptok[j] = trow[(j * kExBM + pt) / kExCh];
    for (int t = 0; t < pre; ++t) {
      issue_tile(t, t);
      cp_async_commit();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // =========================== B tiles (TMA) and MMA issue
    if (lane == 0) {
      ok = mbar_wait(rin_bar, 0);
      for (int t = 0; t < ntl && ok; ++t) {
        const int s = t % P.b_stages, buf = t & 1;
        if (t >= 2) ok = mbar_wait(tempty0 + 8 * buf, ((t - 2) >> 1) & 1);
        if (ok) ok = mbar_wait(bfull0 + 8 * s, (t / P.b_stages) & 1);
        if (!ok) break;
        tc_fence_after();
        int q, c0;
        tile_info(t, q, c0);
        const uint32_t a_s = rin + q * P.rin_bytes;
        const uint32_t b_s = bring + s * P.btile_bytes;
        for (int kk = 0; kk < P.rpad / 16; ++kk) {
          const uint64_t ad = make_sdesc(a_s + kk * 32, P.rpad * 2, P.sw_layout);
          const uint64_t bd = make_sdesc(b_s + kk * 32, P.rpad * 2, P.sw_layout);
          tc_mma_f16(tmem + buf * kExBN, ad, bd, P.idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(tfull0 + 8 * buf);
        tc_commit(bempty0 + 8 * s);
        // refill the slot of tile t-1 with tile t-1+b_stages
        const int tn = t - 1 + P.b_stages;
        if (t >= 1 && tn < ntl) {
          const int sp = (t - 1) % P.b_stages;
          ok = mbar_wait(bempty0 + 8 * sp, ((t - 1) / P.b_stages) & 1);
          if (!ok) break;
          int q2, c2;
          tile_info(tn, q2, c2);
          mbar_arrive_expect_tx(bfull0 + 8 * sp, P.btile_bytes);
          tma_load_2d(bring + sp * P.btile_bytes, &P.tmap_B, bfull0 + 8 * sp, 0,
                      static_cast<int>(adapter * n_tot + (c2 - off0)));
        }
      }
    }
    __syncwarp();
  } else if (warp >= 9) {
    // =========================== producers (128 threads)
    // Publish what went out before the barrier, oldest group first: the rank
    // activations (read by the MMA through the async proxy), then each early tile.
    if (!P.rin_tma) {
      cp_async_wait_dyn(pre);
      fence_proxy_async_smem();
      mbar_arrive(rin_bar);
    }
    for (int t = 0; t < pre; ++t) {
      cp_async_wait_dyn(pre - 1 - t);
      mbar_arrive(xfull0 + 8 * t);
    }
    // The remaining tiles: completion reaches the consumers through
    // cp.async.mbarrier.arrive, so the producers never block on a tile.
    for (int t = pre; t < ntl && ok; ++t) {
      const int s = t % P.base_stages;
      ok = mbar_wait(xempty0 + 8 * s, ((t / P.base_stages) - 1) & 1);
      if (!ok) break;
      issue_tile(t, s);
      cp_async_arrive_noinc(xfull0 + 8 * s);
      cp_async_commit();
    }
    cp_async_wait<0>();
  } else {
    // =========================== consumers (warps 1-8)
    const int quarter = warp & 3;
    const int half = (warp - 1) >> 2;
    const int m = quarter * 32 + lane;  // accumulator row of this thread
    const int ct = tid - 32;            // 0..255 for the coalesced phase
    for (int t = 0; t < ntl; ++t) {
      const int s = t % P.base_stages, buf = t & 1;
      if (ok) ok = mbar_wait(xfull0 + 8 * s, (t / P.base_stages) & 1);
      if (ok) ok = mbar_wait(tfull0 + 8 * buf, (t >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
      tc_fence_after();
      int q, c0;
      tile_info(t, q, c0);
      uint8_t* stage_p = smem + (base_ring - sbase) + s * kExStageBytes;
      const uint32_t tacc = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * kExBN;
      // (a) row-per-thread on this warp's half of the columns: base + scaling * acc.
      //     TMEM loads go out kExLdBatch chunks at a time, one wait per batch.
      constexpr int kHalfChunks = kExBN / 32;  // 16-column TMEM chunks per half
#pragma unroll
      for (int k0 = 0; k0 < kHalfChunks; k0 += kExLdBatch) {
        float v[kExLdBatch][16];
        if (ok) {
#pragma unroll
          for (int k = 0; k < kExLdBatch; ++k)
            tmem_ld16(tacc + (half * kHalfChunks + k0 + k) * 16, v[k]);
          tmem_ld_wait();
        }
        if (ok && m < rows) {
#pragma unroll
          for (int k = 0; k < kExLdBatch; ++k) {
            const int cc = half * kHalfChunks + k0 + k;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int c = 2 * cc + h;
              uint4* ptr = reinterpret_cast<uint4*>(stage_p + m * (kExBN * 2) +
                                                    ((c ^ (m & (kExCh - 1))) << 4));
              uint4 w = *ptr;
              uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 b = E::u32_to_f2(wv[e]);
                wv[e] = E::f2_to_u32(fmaf(scale, v[k][8 * h + 2 * e], b.x),
                                     fmaf(scale, v[k][8 * h + 2 * e + 1], b.y));
              }
              *ptr = w;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * buf);
      named_bar_sync(1, kExConsumers);  // every row of the tile is updated
      // (b) coalesced write-back: chunk u = j*256 + ct -> row u / kExCh, chunk u % kExCh;
      //     all shared-memory reads first, then the stores
      const int cend = p.slices.off[q + 1];
      if (ok) {
        constexpr int kPer = (kExBM * kExCh) / kExConsumers;
        uint4 w[kPer];
        int tk[kPer];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          const int u = j * kExConsumers + ct;
          const int row = u / kExCh, c = u % kExCh;
          w[j] = *reinterpret_cast<const uint4*>(stage_p + row * (kExBN * 2) +
                                                 ((c ^ (row & (kExCh - 1))) << 4));
          tk[j] = trow[row];
        }
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          const int u = j * kExConsumers + ct;
          const int row = u / kExCh, c = u % kExCh;
          const int col = c0 + 8 * c;
          if (row < rows && col < cend)
            stg128(p.base + static_cast<int64_t>(tk[j]) * p.ld_base + col, w[j]);
        }
      }
      mbar_arrive(xempty0 + 8 * s);  // the stage's shared memory may be refilled
    }
  }

  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kExTmemCols);
  }
}

}  // namespace lora

#undef LORA_TILE
