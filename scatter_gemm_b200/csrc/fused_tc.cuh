// fused_tc.cuh -- the shrink and the expand of a piece in one launch, for
// decode-sized token counts (sm_100a).
//
// The pair computes base[perm[i], c] += s_a * (x[perm[i], :] A_a^T B_a^T)[c],
// with the rank activations rounded once to the element type in between (the
// sgl-kernel-xpu page, "Decode LoRA kernels are optimized", section
// "Summary").  At decode sizes both ops are a few microseconds of latency
// each; here one thread-block cluster of C CTAs takes a piece (<= 128 sorted
// rows of one segment, from the scheduler of sched.cuh) through both:
//
//  1. shrink: CTA c gathers the piece's x rows for its K blocks c, c+C, ...
//     (cp.async, 128-byte-swizzled K-major), the adapter's A block by TMA, and
//     accumulates its split-K partial with tcgen05.mma in TMEM;
//  2. every CTA sums its 128/C rows over the C partials (distributed shared
//     memory, rank order), rounds them once, writes them to out_r, and stores
//     the same rounded values into the rank-activation buffer of every CTA of
//     the cluster: after a cluster barrier each CTA holds the piece's complete
//     rank activations in the layout the expand MMA reads;
//  3. expand: CTA c takes the column tiles c, c+C, ...: tcgen05.mma of the
//     rank activations and B, then the fused scale-and-add scatter epilogue.
// The base tiles and B tiles of step 3 do not depend on steps 1-2; they are
// requested while the shrink runs.
//
// Roles (416 threads):
//   warp 0      TMEM (256 columns: first the shrink accumulator, then, once it
//               has been read out and the cluster has passed its barriers, the
//               expand's double-buffered accumulator); A and B tiles by TMA;
//               every MMA;
//   warps 1-8   expand epilogue as two groups of four warps taking alternate
//               tiles (group g uses accumulator buffer g); warps 1-4 also read
//               the shrink accumulator out into the split-K partial;
//   warps 9-12  x gather of the shrink, base tiles of the expand.
// All threads take part in step 2.
#pragma once

#include "common.cuh"
#include "expand_tc.cuh"
#include "general.cuh"
#include "sched.cuh"
#include "shrink_tc.cuh"
#include "sm100.cuh"

namespace lora {

constexpr int kFuThreads = 416;
constexpr int kFuTmemCols = 256;
constexpr int kFuExpandCol = 0;    // the expand accumulators reuse the shrink's columns
constexpr int kFuGroup = 128;      // threads of one consumer group (four warps)

struct FusedTcParams {
  CUtensorMap tmap_A;  // 2-D [L*S*rs rows, K cols], box {64, NPAD}, 128B swizzle
  CUtensorMap tmap_B;  // 2-D [L*N_tot rows, r cols] (row stride rs), box {rpad, 128}
  ShrinkArgs s;        // s.out = out_r (sorted order)
  ExpandArgs e;        // e.in_r = out_r
  int npad;            // shrink MMA N: S*rs rounded up to 16 (<= 256)
  int stages;          // shrink ring depth, stages of 64 K
  int nkb;             // 64-wide K blocks
  int csplit;          // CTAs per cluster
  uint32_t idesc_s;    // shrink: M = 128, N = npad
  uint32_t stage_bytes;  // x (128 rows x 128 B) + A (npad rows x 128 B)
  int rpad;            // expand MMA K: r rounded up to 16, 32 or 64
  uint32_t sw_layout;  // UMMA layout code of rows of rpad*2 bytes
  uint32_t rin_bytes;  // one slice of rank activations (128 * rpad * 2)
  uint32_t btile_bytes;
  uint32_t idesc_e;    // expand: M = 128, N = 128
  int tiles_total;
  int tile_prefix[LORA_MAX_SLICES + 1];
  int base_stages;     // expand ring stages of their own
  int xstages;         // expand ring stages in all: the rest live in the shrink ring,
                       // free once step 2 is over
  int b_stages;
};

template <class E>
__global__ void __launch_bounds__(kFuThreads, 1)
fused_tc_kernel(const __grid_constant__ FusedTcParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const ShrinkArgs& ps = P.s;
  const ExpandArgs& pe = P.e;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int C = P.csplit;
  const int split = blockIdx.x % C;  // rank in the (1-D) cluster
  const int slot = blockIdx.x / C;

  // ---- shared memory: [shrink ring, later the split-K partial][rank activations S]
  //      [base ring][B ring][tokens of 128 rows][barriers]
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t ring = sbase;
  constexpr uint32_t x_bytes = kTcBM * 128;
  const uint32_t rin = ring + P.stages * P.stage_bytes;
  const uint32_t base_ring = rin + ps.S * P.rin_bytes;
  const uint32_t bring = base_ring + P.base_stages * kExStageBytes;
  int* trow = reinterpret_cast<int*>(smem + (bring - sbase) + P.b_stages * P.btile_bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(trow + kTcBM);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * P.stages;
  const uint32_t sdone = empty0 + 8 * P.stages;  // shrink accumulator complete
  const uint32_t bfull0 = sdone + 8;
  const uint32_t bempty0 = bfull0 + 8 * P.b_stages;
  const uint32_t tfull0 = bempty0 + 8 * P.b_stages;
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t xfull0 = tempty0 + 16;
  const uint32_t xempty0 = xfull0 + 8 * P.xstages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * P.stages + 1 + 2 * P.b_stages +
                                                    4 + 2 * P.xstages);
  // expand ring stage s: the first base_stages are the CTA's own, the others
  // reuse the shrink ring after step 2
  auto xstage = [&](int s) {
    return s < P.base_stages ? base_ring + s * kExStageBytes
                             : ring + (s - P.base_stages) * kExStageBytes;
  };

  if (tid == 32) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(full0 + 8 * s, kTcBM + 1);  // 128 gathering threads + the A transfer
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(sdone, 1);
    for (int s = 0; s < P.b_stages; ++s) {
      mbar_init(bfull0 + 8 * s, 1);
      mbar_init(bempty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, kFuGroup);  // accumulator buffer b: consumer group b
    }
    for (int s = 0; s < P.xstages; ++s) {
      mbar_init(xfull0 + 8 * s, kExProducers);
      mbar_init(xempty0 + 8 * s, kFuGroup);  // released by the group that used the stage
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&P.tmap_A);
      tma_prefetch_desc(&P.tmap_B);
    }
    tmem_alloc(smem_u32(tmem_slot), kFuTmemCols);
    tmem_relinquish();
  }

  // ---- the piece of this cluster (the same in all its CTAs).  Producer thread
  // pt owns row pt; rows of a block slot start at slot*128, so their tokens are
  // fetched while the tables are read.
  const bool producer = warp >= 9;
  const int pt = tid - 9 * 32;
  const bool block_slot = slot < (ps.tok + kTcBM - 1) / kTcBM;
  int spec_tok = 0;
  if (producer && block_slot) {
    const int sr = min(slot * kTcBM + pt, ps.tok - 1);
    spec_tok = ps.permutation ? clampi(__ldg(ps.permutation + sr), 0, ps.tok - 1) : sr;
  }
  PieceInfo pc;
  if (!find_piece_warp(ps.seg_indptr, ps.weight_indices, pe.scalings, ps.nseg, ps.L, ps.tok,
                       kTcBM, slot, pc)) {
    // no rows here (the same answer in every CTA of the cluster)
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(*tmem_slot, kFuTmemCols);
    }
    return;
  }
  const int rows = pc.hi - pc.lo;
  const int adapter = pc.adapter;
  const float scale = pc.per_adapter;

  if (producer) {
    const int m = pt;
    int tk = spec_tok;
    if (!block_slot) {
      const int sr = pc.lo + (m < rows ? m : 0);
      tk = ps.permutation ? clampi(__ldg(ps.permutation + sr), 0, ps.tok - 1) : sr;
    }
    trow[m] = tk;
  }
  // The rank activations start as zeros: storage columns rs..rpad and rows
  // past the piece are never written by step 2, and the expand MMA reads them.
  for (uint32_t o = 16 * tid; o < ps.S * P.rin_bytes; o += 16 * kFuThreads)
    *reinterpret_cast<uint4*>(smem + (rin - sbase) + o) = make_uint4(0u, 0u, 0u, 0u);

  // K blocks (shrink) and column tiles (expand) of this CTA, interleaved over the cluster
  const int nk = split < P.nkb ? (P.nkb - split + C - 1) / C : 0;
  const int T = P.tiles_total;
  // a zero scaling leaves the base rows bit-identical: no expand work
  const int ntl = (scale != 0.f && split < T) ? (T - split + C - 1) / C : 0;
  const int off0 = pe.slices.off[0];
  const int64_t n_tot = pe.slices.off[pe.S] - off0;
  auto tile_cols = [&](int t, int& q, int& c0) {
    const int g = split + t * C;
    q = 0;
#pragma unroll
    for (int k = 1; k < LORA_MAX_SLICES; ++k)
      if (k < pe.S && g >= P.tile_prefix[k]) q = k;
    c0 = pe.slices.off[q] + (g - P.tile_prefix[q]) * kExBN;
  };
  // base tile t into ring stage s: chunk u = j*128 + pt -> row u / kExCh, chunk
  // u % kExCh.  A producer's rows are the same for every tile, so their tokens
  // sit in registers (ptok, filled once trow is complete) and the copies of a
  // tile issue back to back, none waiting on a shared-memory load.
  int ptok[kExCh];
  auto issue_tile = [&](int t, int s) {
    int q, c0;
    tile_cols(t, q, c0);
    const int cend = pe.slices.off[q + 1];
    const uint32_t stage = xstage(s);
#pragma unroll
    for (int j = 0; j < kExCh; ++j) {
      const int u = j * kExBM + pt;
      const int row = u / kExCh, c = u % kExCh;
      const int col = c0 + 8 * c;
      // rows past the piece and columns past the slice are not loaded: the
      // epilogue never stores them
      if (row < rows && col < cend)
        cp_async_16(stage + row * (kExBN * 2) + ((c ^ (row & (kExCh - 1))) << 4),
                    pe.base + static_cast<int64_t>(ptok[j]) * pe.ld_base + col, 16u);
    }
  };
  auto load_b = [&](int t, int sp) {
    int q, c0;
    tile_cols(t, q, c0);
    mbar_arrive_expect_tx(bfull0 + 8 * sp, P.btile_bytes);
    tma_load_2d(bring + sp * P.btile_bytes, &P.tmap_B, bfull0 + 8 * sp, 0,
                static_cast<int>(adapter * n_tot + (c0 - off0)));
  };

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  const int pre_e = min(P.base_stages, ntl);

  // =========================== 1. shrink
  if (producer) {
    // x stage: 128 rows x 8 chunks of 16 bytes; this thread's chunk column is
    // cc and its rows rr + 16 j, the same for every stage
    const int cc = pt % 8, rr = pt / 8;
    const uint32_t a_bytes = P.npad * 128;
    const uint16_t* xr[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) xr[j] = ps.x + static_cast<int64_t>(trow[rr + 16 * j]) * ps.ld_x;
#pragma unroll
    for (int j = 0; j < kExCh; ++j) ptok[j] = trow[(j * kExBM + pt) / kExCh];
    const int lag = P.stages - 1;
    for (int i = 0; i < nk && ok; ++i) {
      const int s = i % P.stages;
      if (i >= P.stages) ok = mbar_wait(empty0 + 8 * s, ((i / P.stages) - 1) & 1);
      if (!ok) break;
      const uint32_t xs = ring + s * P.stage_bytes;
      const int k0 = (split + i * C) * kTcAtomK;
      if (pt == 0) {
        mbar_arrive_expect_tx(full0 + 8 * s, a_bytes);
        tma_load_2d(xs + x_bytes, &P.tmap_A, full0 + 8 * s, k0, adapter * ps.S * ps.rs);
      }
      const int k = k0 + 8 * cc;
      const bool k_in = k < ps.K;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        // rows past the piece are not loaded (their MMA rows are never used);
        // past K a row of the piece is zero-filled
        const int row = rr + 16 * j;
        if (row < rows)
          cp_async_16(xs + row * 128 + ((cc ^ (row & 7)) << 4),
                      k_in ? static_cast<const void*>(xr[j] + k)
                           : static_cast<const void*>(ps.x),
                      k_in ? 16u : 0u);
      }
      cp_async_commit();
      if (i >= lag) {
        cp_async_wait_dyn(lag);
        fence_proxy_async_smem();
        mbar_arrive(full0 + 8 * ((i - lag) % P.stages));
      }
    }
    // the expand's first base tiles go out now; their arrivals (.noinc) wait
    // for every earlier copy of the thread, so nothing blocks here
    for (int t = 0; t < pre_e; ++t) {
      issue_tile(t, t);
      cp_async_arrive_noinc(xfull0 + 8 * t);
      cp_async_commit();
    }
    // publish the shrink stages still in flight (all groups but the base tiles')
    cp_async_wait_dyn(pre_e);
    fence_proxy_async_smem();
    if (ok)
      for (int i = max(0, nk - lag); i < nk; ++i) mbar_arrive(full0 + 8 * (i % P.stages));
  } else if (warp == 0) {
    if (lane == 0) {
      // B tiles of the first expand tiles do not depend on the shrink
      for (int t = 0; t < min(P.b_stages, ntl); ++t) load_b(t, t);
      for (int i = 0; i < nk && ok; ++i) {
        const int s = i % P.stages;
        ok = mbar_wait(full0 + 8 * s, (i / P.stages) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t xs = ring + s * P.stage_bytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = make_sdesc(xs + kk * 32, 128, 2);
          const uint64_t bd = make_sdesc(xs + x_bytes + kk * 32, 128, 2);
          tc_mma_f16(tmem, ad, bd, P.idesc_s, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(empty0 + 8 * s);
      }
      if (nk > 0) tc_commit(sdone); else mbar_arrive(sdone);
    }
    __syncwarp();
  }
  // split-K partial: [128][npad + 4] fp32 over the shrink ring (the row stride
  // keeps the row-per-thread 16-byte stores free of bank conflicts)
  float* part = reinterpret_cast<float*>(smem);
  const int pstride = P.npad + 4;
  if (warp >= 1 && warp <= 4) {
    if (ok) ok = mbar_wait(sdone, 0);
    ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
    tc_fence_after();
    const int quarter = warp & 3;
    const int m = quarter * 32 + lane;
    const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    for (int c0 = 0; c0 < P.npad; c0 += 16) {
      float v[16];
      if (nk > 0 && ok) {
        tmem_ld16(tq + c0, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
      }
      float4* dst = reinterpret_cast<float4*>(part + m * pstride + c0);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
    tc_fence_before();
  }

  // =========================== 2. reduce, round, share
  cluster_sync();  // every partial of the cluster is in shared memory
  {
    const int R = kTcBM / C;
    const int r0 = split * R;
    const int ng = P.npad / 4;
    const int nvalid = ps.S * ps.rs;
    const uint32_t pbase = smem_u32(part);
    for (int e = tid; e < R * ng; e += kFuThreads) {
      const int row = r0 + e / ng;
      const int n = 4 * (e % ng);
      if (row >= rows || n >= nvalid) continue;
      const int q = n / ps.rs, j = n % ps.rs;  // rs is a multiple of 8: 4 columns, one slice
      if (j >= P.rpad) continue;               // storage padding the expand never reads
      const uint32_t off = pbase + 4u * static_cast<uint32_t>(row * pstride + n);
      float4 pv[16];
#pragma unroll
      for (int c = 0; c < 16; ++c)
        if (c < C) pv[c] = ld_dsmem_v4(mapa_shared(off, c));
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        if (c < C) {
          sum.x += pv[c].x;
          sum.y += pv[c].y;
          sum.z += pv[c].z;
          sum.w += pv[c].w;
        }
      }
      const float sv[4] = {sum.x, sum.y, sum.z, sum.w};
      uint16_t b[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) b[k] = (j + k < ps.r) ? E::f32_to_bits(sv[k]) : uint16_t(0);
      if (ok) {
        uint16_t* orow = ps.out + static_cast<int64_t>(pc.lo + row) * ps.ld_out;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (j + k < ps.r) stg16(orow + n + k, b[k]);
      }
      // the rounded activations into every CTA's buffer, in the expand's layout
      const uint32_t dst = rin + q * P.rin_bytes + row * (P.rpad * 2) +
                           (swz_chunk(j >> 3, row, P.rpad) << 4) + ((j & 7) << 1);
      const uint32_t lo = static_cast<uint32_t>(b[0]) | (static_cast<uint32_t>(b[1]) << 16);
      const uint32_t hi = static_cast<uint32_t>(b[2]) | (static_cast<uint32_t>(b[3]) << 16);
      for (int c = 0; c < C; ++c) st_dsmem_v2(mapa_shared(dst, c), lo, hi);
    }
    fence_proxy_async_all();  // read next by the expand MMAs (async proxy)
  }
  cluster_sync();  // rank activations complete everywhere; the partials are no longer read

  // =========================== 3. expand
  if (warp == 0) {
    if (lane == 0) {
      fence_proxy_async_smem();
      for (int t = 0; t < ntl && ok; ++t) {
        const int s = t % P.b_stages, buf = t & 1;
        if (t >= 2) ok = mbar_wait(tempty0 + 8 * buf, ((t - 2) >> 1) & 1);
        if (ok) ok = mbar_wait(bfull0 + 8 * s, (t / P.b_stages) & 1);
        if (!ok) break;
        tc_fence_after();
        int q, c0;
        tile_cols(t, q, c0);
        const uint32_t a_s = rin + q * P.rin_bytes;
        const uint32_t b_s = bring + s * P.btile_bytes;
        for (int kk = 0; kk < P.rpad / 16; ++kk) {
          const uint64_t ad = make_sdesc(a_s + kk * 32, P.rpad * 2, P.sw_layout);
          const uint64_t bd = make_sdesc(b_s + kk * 32, P.rpad * 2, P.sw_layout);
          tc_mma_f16(tmem + kFuExpandCol + buf * kExBN, ad, bd, P.idesc_e, kk > 0 ? 1u : 0u);
        }
        tc_commit(tfull0 + 8 * buf);
        tc_commit(bempty0 + 8 * s);
        const int tn = t - 1 + P.b_stages;
        if (t >= 1 && tn < ntl) {
          const int sp = (t - 1) % P.b_stages;
          ok = mbar_wait(bempty0 + 8 * sp, ((t - 1) / P.b_stages) & 1);
          if (!ok) break;
          load_b(tn, sp);
        }
      }
    }
    __syncwarp();
  } else if (producer) {
    // stages of the shrink ring are fresh now: they are filled without waiting
    for (int t = pre_e; t < ntl && ok; ++t) {
      const int s = t % P.xstages;
      if (t >= P.xstages) ok = mbar_wait(xempty0 + 8 * s, ((t / P.xstages) - 1) & 1);
      if (!ok) break;
      issue_tile(t, s);
      cp_async_arrive_noinc(xfull0 + 8 * s);
      cp_async_commit();
    }
    cp_async_wait<0>();
  } else {
    // consumers: two groups of four warps (one per TMEM lane quarter) take
    // alternate tiles, so two tiles are in their epilogue at once; group g
    // uses accumulator buffer g
    const int quarter = warp & 3;
    const int grp = (warp - 1) >> 2;
    const int m = quarter * 32 + lane;  // accumulator row of this thread
    const int gt = tid - 32 - grp * kFuGroup;  // 0..127 in the group
    for (int t = grp; t < ntl; t += 2) {
      const int s = t % P.xstages, buf = grp;
      if (ok) ok = mbar_wait(xfull0 + 8 * s, (t / P.xstages) & 1);
      if (ok) ok = mbar_wait(tfull0 + 8 * buf, (t >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
      tc_fence_after();
      int q, c0;
      tile_cols(t, q, c0);
      uint8_t* stage_p = smem + (xstage(s) - sbase);
      const uint32_t tacc = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kFuExpandCol +
                            buf * kExBN;
      // (a) row m, every column: base + scaling * acc, in place in shared memory
#pragma unroll
      for (int k0 = 0; k0 < kExBN / 16; k0 += kExLdBatch) {
        float v[kExLdBatch][16];
        if (ok) {
#pragma unroll
          for (int kb = 0; kb < kExLdBatch; ++kb) tmem_ld16(tacc + (k0 + kb) * 16, v[kb]);
          tmem_ld_wait();
        }
        if (ok && m < rows) {
#pragma unroll
          for (int kb = 0; kb < kExLdBatch; ++kb) {
            const int cc = k0 + kb;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int c = 2 * cc + h;
              uint4* ptr = reinterpret_cast<uint4*>(stage_p + m * (kExBN * 2) +
                                                    ((c ^ (m & (kExCh - 1))) << 4));
              uint4 w = *ptr;
              uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 bb = E::u32_to_f2(wv[e]);
                wv[e] = E::f2_to_u32(fmaf(scale, v[kb][8 * h + 2 * e], bb.x),
                                     fmaf(scale, v[kb][8 * h + 2 * e + 1], bb.y));
              }
              *ptr = w;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * buf);
      named_bar_sync(1 + grp, kFuGroup);  // every row of the tile is updated
      // (b) coalesced write-back of the rows of the piece: chunk u = j*128 + gt
      const int cend = pe.slices.off[q + 1];
      //     four chunks at a time: their shared-memory reads first, then the
      //     stores (global-space stores: the next loads need not wait on them)
      if (ok) {
        constexpr int kPer = (kExBM * kExCh) / kFuGroup;
        constexpr int kBatch = 4;
#pragma unroll
        for (int j0 = 0; j0 < kPer; j0 += kBatch) {
          uint4 w[kBatch];
          int tk[kBatch];
#pragma unroll
          for (int k = 0; k < kBatch; ++k) {
            const int u = (j0 + k) * kFuGroup + gt;
            const int row = u / kExCh, c = u % kExCh;
            w[k] = *reinterpret_cast<const uint4*>(stage_p + row * (kExBN * 2) +
                                                   ((c ^ (row & (kExCh - 1))) << 4));
            tk[k] = trow[row];
          }
#pragma unroll
          for (int k = 0; k < kBatch; ++k) {
            const int u = (j0 + k) * kFuGroup + gt;
            const int row = u / kExCh, c = u % kExCh;
            const int col = c0 + 8 * c;
            if (row < rows && col < cend)
              stg128(pe.base + static_cast<int64_t>(tk[k]) * pe.ld_base + col, w[k]);
          }
        }
      }
      mbar_arrive(xempty0 + 8 * s);
    }
  }

  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kFuTmemCols);
  }
}

}  // namespace lora
