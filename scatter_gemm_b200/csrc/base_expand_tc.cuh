// base_expand_tc.cuh -- the base projection with the expand folded into its
// epilogue (sm_100a).
//
// On the sglang page "fused split_qkv / norm / RoPE for Qwen3.5/Next on NPU"
// (key source snippets, forward_prepare_npu) the qkv_proj output goes straight
// to the split step; with LoRA, the expand of the chunked-SGMV pair (the
// sgl-kernel-xpu page, "Decode LoRA kernels are optimized", section "Summary")
// first reads and rewrites that whole output.  Here the projection and the
// expand are one kernel, and the output is written once:
//     out[perm[i], c] = rn( sum_k x[perm[i], k] W[c - off0, k]
//                           + s_a sum_{j<r} in_r[i, q*rs + j] B_a[c - off0, j] )
// for the rows i of every segment (adapter a) and the columns c of slice q.
//
// One CTA computes one piece (<= 128 sorted rows of one segment, from the
// scheduler of sched.cuh) times one 128-column tile:
//  - warps 0-3 gather the piece's x rows with cp.async into 128-byte-swizzled
//    K-major stages; thread 0 loads the stage's W tile (128 rows x 64 K) by
//    TMA; the same warps load the piece's rank activations of the tile's slice
//    (zero-filled beyond r);
//  - warp 4 holds TMEM (256 columns: the projection's accumulator at column 0,
//    the rank term's at column 128), loads the adapter's B tile by TMA and
//    issues the MMAs: K/16 for the projection (M = 128, N = 128), then rpad/16
//    for the rank term;
//  - warps 0-3 then read both accumulators (one row per thread), form
//    rn(base + s_a * lora) in fp32, stage the tile in shared memory and write
//    it to the token rows with coalesced 16-byte stores.
// A zero scaling skips the rank term: the result is the rounded projection.
// The roofline is the tensor pipe: 2 * N_tot * K flops per token.
#pragma once

#include "common.cuh"
#include "expand_tc.cuh"
#include "general.cuh"
#include "sched.cuh"
#include "shrink_tc.cuh"
#include "sm100.cuh"

namespace lora {

constexpr int kBeThreads = 160;
constexpr int kBeBN = 128;        // columns per tile
constexpr int kBeTmemCols = 256;  // projection accumulator + rank-term accumulator

struct BaseExpandArgs {
  const uint16_t* x;   // [tok, ld_x]
  int64_t ld_x;
  const uint16_t* in_r;  // [tok, ld_in], sorted order
  int64_t ld_in;
  const int32_t* seg_indptr;
  const int32_t* weight_indices;
  const int32_t* permutation;
  const float* scalings;
  uint16_t* out;  // [tok, ld_out]
  int64_t ld_out;
  int tok, K, S, r, rs, nseg, L;
  SliceTable slices;
};

struct BaseExpandTcParams {
  CUtensorMap tmap_W;  // 2-D [N_tot rows, K cols] (row stride ld_w), box {64, 128}, 128B swizzle
  CUtensorMap tmap_B;  // 2-D [L*N_tot rows, r cols] (row stride rs), box {rpad, 128}
  BaseExpandArgs a;
  int tiles_total;     // 128-column tiles over all slices
  int tile_prefix[LORA_MAX_SLICES + 1];
  int stages;          // K ring depth (stages of 64 K)
  int nkb;             // 64-wide K blocks
  int rpad;            // rank term MMA K: 16, 32 or 64
  uint32_t sw_layout;  // UMMA layout code of rows of rpad*2 bytes
  uint32_t rin_bytes;  // rank activations of the tile's slice (128 * rpad * 2)
  uint32_t btile_bytes;
  uint32_t idesc;      // M = 128, N = 128
};

template <class E>
__global__ void __launch_bounds__(kBeThreads, 1)
base_expand_tc_kernel(const __grid_constant__ BaseExpandTcParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const BaseExpandArgs& p = P.a;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int T = P.tiles_total;
  const int slot = blockIdx.x / T;
  const int g = blockIdx.x % T;

  // ---- shared memory: [K ring (x 16 KB + W 16 KB per stage), later the output
  //      tile][rank activations][B tile][tokens of 128 rows][barriers]
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  constexpr uint32_t kXBytes = kTcBM * 128;
  constexpr uint32_t kStage = kXBytes + kBeBN * 128;
  const uint32_t rin = sbase + P.stages * kStage;
  const uint32_t btile = rin + P.rin_bytes;
  int* trow = reinterpret_cast<int*>(smem + (btile - sbase) + P.btile_bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(trow + kTcBM);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * P.stages;
  const uint32_t rin_bar = empty0 + 8 * P.stages;
  const uint32_t bfull = rin_bar + 8;
  const uint32_t done_bar = bfull + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * P.stages + 3);

  if (tid == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(full0 + 8 * s, kTcBM + 1);  // 128 gathering threads + the W transfer
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(rin_bar, kTcBM);
    mbar_init(bfull, 1);
    mbar_init(done_bar, 1);
    fence_mbar_init();
  }
  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch_desc(&P.tmap_W);
      tma_prefetch_desc(&P.tmap_B);
    }
    tmem_alloc(smem_u32(tmem_slot), kBeTmemCols);
    tmem_relinquish();
  }

  // ---- the piece of this slot; rows of a block slot start at slot*128, so
  // their tokens are fetched while the tables are read
  const bool block_slot = slot < (p.tok + kTcBM - 1) / kTcBM;
  int spec_tok = 0;
  if (tid < kTcBM && block_slot) {
    const int sr = min(slot * kTcBM + tid, p.tok - 1);
    spec_tok = p.permutation ? clampi(__ldg(p.permutation + sr), 0, p.tok - 1) : sr;
  }
  PieceInfo pc;
  if (!find_piece_warp(p.seg_indptr, p.weight_indices, p.scalings, p.nseg, p.L, p.tok, kTcBM,
                       slot, pc)) {
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
      tc_fence_after();
      tmem_dealloc(*tmem_slot, kBeTmemCols);
    }
    return;
  }
  const int rows = pc.hi - pc.lo;
  const int adapter = pc.adapter;
  const float scale = pc.per_adapter;
  const bool lora = scale != 0.f;  // a zero scaling leaves the rounded projection

  // tile g -> slice q, first column c0
  int q = 0;
#pragma unroll
  for (int k = 1; k < LORA_MAX_SLICES; ++k)
    if (k < p.S && g >= P.tile_prefix[k]) q = k;
  const int c0 = p.slices.off[q] + (g - P.tile_prefix[q]) * kBeBN;
  const int cend = p.slices.off[q + 1];
  const int off0 = p.slices.off[0];
  const int64_t n_tot = p.slices.off[p.S] - off0;

  if (tid < kTcBM) {
    const int m = tid;
    int tk = spec_tok;
    if (!block_slot) {
      const int sr = pc.lo + (m < rows ? m : 0);
      tk = p.permutation ? clampi(__ldg(p.permutation + sr), 0, p.tok - 1) : sr;
    }
    trow[m] = tk;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp < 4) {
    // =========================== producers: rank activations, then the K loop
    {
      // row m of the piece: slice q of its rank activations, zero-filled beyond r
      const int m = tid;
      const bool row_ok = lora && m < rows;
      const uint16_t* src = p.in_r + static_cast<int64_t>(pc.lo + (m < rows ? m : 0)) * p.ld_in +
                            static_cast<int64_t>(q) * p.rs;
      for (int c = 0; c < P.rpad / 8; ++c) {
        const int left = p.r - 8 * c;
        const uint32_t nb = row_ok ? static_cast<uint32_t>(max(0, min(left, 8)) * 2) : 0u;
        cp_async_16(rin + m * (P.rpad * 2) + (swz_chunk(c, m, P.rpad) << 4),
                    nb ? static_cast<const void*>(src + 8 * c) : static_cast<const void*>(p.in_r),
                    nb);
      }
      cp_async_commit();  // the oldest group: published after the K loop
    }
    // x stage: 128 rows x 8 chunks of 16 bytes; this thread's chunk column is
    // cc and its rows rr + 16 j, the same for every stage
    const int cc = tid % 8, rr = tid / 8;
    const uint16_t* xr[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) xr[j] = p.x + static_cast<int64_t>(trow[rr + 16 * j]) * p.ld_x;
    const int lag = P.stages - 1;
    for (int i = 0; i < P.nkb && ok; ++i) {
      const int s = i % P.stages;
      if (i >= P.stages) ok = mbar_wait(empty0 + 8 * s, ((i / P.stages) - 1) & 1);
      if (!ok) break;
      const uint32_t xs = sbase + s * kStage;
      const int k0 = i * kTcAtomK;
      if (tid == 0) {
        mbar_arrive_expect_tx(full0 + 8 * s, kBeBN * 128);
        tma_load_2d(xs + kXBytes, &P.tmap_W, full0 + 8 * s, k0, c0 - off0);
      }
      const int k = k0 + 8 * cc;
      const bool k_in = k < p.K;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int row = rr + 16 * j;
        const bool in = k_in && row < rows;
        cp_async_16(xs + row * 128 + ((cc ^ (row & 7)) << 4),
                    in ? static_cast<const void*>(xr[j] + k) : static_cast<const void*>(p.x),
                    in ? 16u : 0u);
      }
      cp_async_commit();
      if (i >= lag) {
        cp_async_wait_dyn(lag);
        fence_proxy_async_smem();
        mbar_arrive(full0 + 8 * ((i - lag) % P.stages));
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();  // x and the rank activations are read by the MMA (async proxy)
    if (ok)
      for (int i = max(0, P.nkb - lag); i < P.nkb; ++i) mbar_arrive(full0 + 8 * (i % P.stages));
    mbar_arrive(rin_bar);
  } else {
    // =========================== MMA issuer (warp 4)
    if (lane == 0) {
      if (lora) {
        mbar_arrive_expect_tx(bfull, P.btile_bytes);
        tma_load_2d(btile, &P.tmap_B, bfull, 0, static_cast<int>(adapter * n_tot + (c0 - off0)));
      }
      for (int i = 0; i < P.nkb && ok; ++i) {
        const int s = i % P.stages;
        ok = mbar_wait(full0 + 8 * s, (i / P.stages) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t xs = sbase + s * kStage;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = make_sdesc(xs + kk * 32, 128, 2);
          const uint64_t bd = make_sdesc(xs + kXBytes + kk * 32, 128, 2);
          tc_mma_f16(tmem, ad, bd, P.idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(empty0 + 8 * s);
      }
      if (ok && lora) {
        ok = mbar_wait(rin_bar, 0);
        if (ok) ok = mbar_wait(bfull, 0);
        if (ok) {
          tc_fence_after();
          for (int kk = 0; kk < P.rpad / 16; ++kk) {
            const uint64_t ad = make_sdesc(rin + kk * 32, P.rpad * 2, P.sw_layout);
            const uint64_t bd = make_sdesc(btile + kk * 32, P.rpad * 2, P.sw_layout);
            tc_mma_f16(tmem + kBeBN, ad, bd, P.idesc, kk > 0 ? 1u : 0u);
          }
        }
      }
      if (P.nkb > 0 || lora) tc_commit(done_bar); else mbar_arrive(done_bar);
    }
    __syncwarp();
  }

  // =========================== epilogue (warps 0-3): one accumulator row per thread
  if (warp < 4) {
    if (ok) ok = mbar_wait(done_bar, 0);
    ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
    tc_fence_after();
    const int m = tid;
    const uint32_t tb = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    // the output tile over the K ring: row m is 256 bytes, 16-byte chunks
    // XOR-swizzled by the row so both phases are free of bank conflicts
    uint8_t* stile = smem;
#pragma unroll 1
    for (int c16 = 0; c16 < kBeBN / 16; ++c16) {
      float vb[16], vl[16];
      if (ok) {
        tmem_ld16(tb + c16 * 16, vb);
        if (lora) tmem_ld16(tb + kBeBN + c16 * 16, vl);
        tmem_ld_wait();
      }
      if (ok && m < rows) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4 w;
          uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i0 = 8 * h + 2 * e;
            const float a0 = lora ? fmaf(scale, vl[i0], vb[i0]) : vb[i0];
            const float a1 = lora ? fmaf(scale, vl[i0 + 1], vb[i0 + 1]) : vb[i0 + 1];
            wv[e] = E::f2_to_u32(a0, a1);
          }
          const int c = 2 * c16 + h;
          *reinterpret_cast<uint4*>(stile + m * (kBeBN * 2) + ((c ^ (m & 15)) << 4)) = w;
        }
      }
    }
    tc_fence_before();
    named_bar_sync(1, kTcBM);  // the whole tile is staged
    if (ok) {
      // coalesced write-back: chunk u = j*128 + tid -> row u / 16, chunk u % 16;
      // four chunks at a time, their shared-memory reads before the stores
      constexpr int kBatch = 4;
#pragma unroll
      for (int j0 = 0; j0 < 16; j0 += kBatch) {
        uint4 w[kBatch];
        int tk[kBatch];
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
          const int u = (j0 + k) * kTcBM + tid;
          const int row = u / 16, c = u % 16;
          w[k] = *reinterpret_cast<const uint4*>(stile + row * (kBeBN * 2) + ((c ^ (row & 15)) << 4));
          tk[k] = trow[row];
        }
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
          const int u = (j0 + k) * kTcBM + tid;
          const int row = u / 16, c = u % 16;
          const int col = c0 + 8 * c;
          if (row < rows && col < cend)
            stg128(p.out + static_cast<int64_t>(tk[k]) * p.ld_out + col, w[k]);
        }
      }
    }
  }

  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, kBeTmemCols);
  }
}

}  // namespace lora
