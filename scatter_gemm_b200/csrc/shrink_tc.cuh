// shrink_tc.cuh -- tensor-core shrink for 16-byte-aligned inputs (sm_100a).
//
// One CTA computes one piece (<= 128 sorted rows of one segment, from the
// scheduler of sched.cuh) times one K range:
//     D[128 x NPAD] = X_piece[128 x K_range] * A_a[NPAD x K_range]^T
// with NPAD = S*rs rounded up to 16.  The contraction runs on tcgen05.mma
// (M = 128, N = NPAD, K = 16 per instruction) with the fp32 accumulator in
// TMEM.  This is the "gathered-A mainloop" of the sgl-kernel-xpu page
// ("Decode LoRA kernels are optimized", section "Summary"), rebuilt for B200:
//
//  - warps 0-3 gather the piece's x rows (row m = token perm[lo+m]) with
//    16-byte cp.async straight into the 128-byte-swizzled K-major layout the
//    MMA reads, through a ring of stages of up to LORA_SHRINK_BK K elements
//    (the host picks the widest that fits two stages; 64 measured best);
//  - thread 0 loads the adapter's A block of the stage with TMA tiled copies
//    (rows a*S*rs ... + NPAD, 64 K columns each; out-of-range rows and K
//    columns are zero-filled by the TMA unit);
//  - warp 4 issues the MMAs and returns each stage with tcgen05.commit;
//  - warps 0-3 then read the accumulator back (tcgen05.ld, one row per
//    thread) and round each valid column (j < r of every slice) once.
//
// Split-K: for small token counts the K range is split over the CTAs of a
// thread-block cluster (grid = pieces x C, cluster = C CTAs along K).  Each
// CTA leaves its fp32 partial in its own shared memory; after a cluster
// barrier CTA c sums rows [c*128/C, (c+1)*128/C) over all C partials through
// distributed shared memory, in rank order (deterministic), and writes them.
// No global scratch and no atomics.
#pragma once

#include "common.cuh"
#include "general.cuh"
#include "sched.cuh"
#include "sm100.cuh"

#ifndef LORA_SHRINK_INTERLEAVE
#define LORA_SHRINK_INTERLEAVE 1
#endif

namespace lora {

constexpr int kTcBM = 128;   // rows per piece (MMA M)
constexpr int kTcAtomK = 64; // K elements of one 128-byte swizzle atom row
#ifndef LORA_SHRINK_BK
#define LORA_SHRINK_BK 64     // widest stage: K elements of every x row (64 = 128 bytes)
#endif
constexpr int kTcMaxNSub = LORA_SHRINK_BK / kTcAtomK;
static_assert(kTcMaxNSub == 1 || kTcMaxNSub == 2 || kTcMaxNSub == 4, "stage K width");
constexpr int kTcThreads = 160;

struct ShrinkTcParams {
  CUtensorMap tmap_A;  // 2-D [L*S*rs rows, K cols], box {64, NPAD}, 128B swizzle
  ShrinkArgs a;
  const int32_t* row_list;     // grouped schedule: sorted row of each grouped row (or null)
  const int32_t* vseg_indptr;  // grouped schedule: rows of each adapter group (or null)
  int nvseg;                   // number of (virtual) segments the scheduler walks
  int npad;                    // MMA N
  int tmem_cols;               // power of two >= npad, >= 32
  int stages;
  int nkb;                     // K blocks in total
  int kb_per;                  // K blocks per split
  int csplit;                  // CTAs per cluster (K splits)
  uint32_t idesc;
  uint32_t stage_bytes;
};

// NSUB: 64-K sub-tiles per stage (stage K width = 64 * NSUB)
template <class E, int NSUB>
__global__ void __launch_bounds__(kTcThreads, 1)
shrink_tc_kernel(const __grid_constant__ ShrinkTcParams P) {
  constexpr int kTcNSub = NSUB;
  constexpr int kTcBK = NSUB * kTcAtomK;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const ShrinkArgs& p = P.a;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x % P.csplit;
  const int slot = blockIdx.x / P.csplit;

  // ---- shared memory carve-up (1024-aligned stages, then barriers)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t x_bytes = kTcNSub * kTcBM * 128;  // kTcNSub sub-tiles of 128 rows x 128 B
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P.stages * P.stage_bytes);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * P.stages;
  const uint32_t done_bar = empty0 + 8 * P.stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * P.stages + 1);
  int64_t* xrow_tok = reinterpret_cast<int64_t*>(bars + 2 * P.stages + 2);  // [128] x row index

  // barriers and TMEM first, so that their latency overlaps the table reads
  if (tid == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(full0 + 8 * s, kTcBM + 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(done_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&P.tmap_A);
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), P.tmem_cols);
    tmem_relinquish();
  }

  // ---- piece of this cluster (identical in all its CTAs).  Rows of a block
  // slot start at slot*128, so their tokens are fetched while the tables are read.
  const bool block_slot = slot < (p.tok + kTcBM - 1) / kTcBM;
  int spec_tok = 0;
  if (tid < kTcBM && block_slot) {
    int sr = min(slot * kTcBM + tid, p.tok - 1);
    if (P.row_list) sr = clampi(__ldg(P.row_list + sr), 0, p.tok - 1);
    spec_tok = p.permutation ? clampi(__ldg(p.permutation + sr), 0, p.tok - 1) : sr;
  }
  PieceInfo pc;
  const int32_t* indptr = P.vseg_indptr ? P.vseg_indptr : p.seg_indptr;
  if (!find_piece_warp(indptr, P.vseg_indptr ? nullptr : p.weight_indices, nullptr, P.nvseg,
                       p.L, p.tok, kTcBM, slot, pc)) {
    // no rows here (the same answer in every CTA of the cluster): give TMEM back
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
      tc_fence_after();
      tmem_dealloc(*tmem_slot, P.tmem_cols);
    }
    return;
  }
  const int rows = pc.hi - pc.lo;
  const int adapter = pc.adapter;

  // K blocks of this CTA.  Interleaved over the cluster (CTA c takes blocks
  // c, c+C, c+2C, ...), so the C co-scheduled CTAs of a piece read C adjacent
  // 128-byte runs of every row at about the same time: DRAM sees contiguous
  // C*128-byte pieces of each gathered row instead of scattered 128-byte ones.
#if LORA_SHRINK_INTERLEAVE
  const int nk = split < P.nkb ? (P.nkb - split + P.csplit - 1) / P.csplit : 0;
#define LORA_KB(i) (split + (i) * P.csplit)
#else
  const int kb0 = split * P.kb_per;
  const int nk = max(0, min(P.nkb, kb0 + P.kb_per) - kb0);
#define LORA_KB(i) (kb0 + (i))
#endif

  if (tid < kTcBM) {
    const int m = tid;
    if (block_slot) {
      xrow_tok[m] = spec_tok;
    } else {
      int srow = pc.lo + (m < rows ? m : 0);
      if (P.row_list) srow = clampi(__ldg(P.row_list + srow), 0, p.tok - 1);
      xrow_tok[m] = p.permutation ? clampi(__ldg(p.permutation + srow), 0, p.tok - 1) : srow;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp < 4) {
    // =========================== producer: gather x rows and the A block
    // A stage holds NSUB sub-tiles of 16-byte chunks; chunk u = j*128 + tid ->
    // row u / (8*NSUB), chunk u % (8*NSUB).  The chunk column of a thread is the
    // same for every row and stage, and its x rows are the same for every stage,
    // so their addresses are formed once.  Thread 0 also loads the stage's A
    // block with TMA (measured faster than gathering A with cp.async).
    constexpr int CPR = 8 * kTcNSub;              // 16-byte chunks per row per stage
    constexpr int RSTEP = kTcBM / CPR;            // rows between a thread's chunks
    const int cc = tid % CPR;                     // this thread's chunk column
    const int rr = tid / CPR;                     // ... and first row
    const int wrow0 = (tid & ~31) / CPR;          // first row of this warp
    const uint32_t sub_off = (cc >> 3) * (kTcBM * 128);  // x sub-tile of this chunk
    const uint32_t a_sub = P.npad * 128;  // one 64-K sub-tile of A
    const uint32_t a_bytes = kTcNSub * a_sub;
    // gathered x row of each of this thread's CPR rows (rows past the piece are
    // never read)
    const uint16_t* xr[CPR];
#pragma unroll
    for (int j = 0; j < CPR; ++j) xr[j] = p.x + xrow_tok[rr + j * RSTEP] * p.ld_x;
    const int lag = P.stages - 1;
    for (int i = 0; i < nk && ok; ++i) {
      const int s = i % P.stages;
      if (i >= P.stages) ok = mbar_wait(empty0 + 8 * s, ((i / P.stages) - 1) & 1);
      if (!ok) break;
      const uint32_t xs = sbase + s * P.stage_bytes;
      const int k0 = LORA_KB(i) * kTcBK;
      if (tid == 0) {
        mbar_arrive_expect_tx(full0 + 8 * s, a_bytes);
#pragma unroll
        for (int sub = 0; sub < kTcNSub; ++sub)
          tma_load_2d(xs + x_bytes + sub * a_sub, &P.tmap_A, full0 + 8 * s, k0 + sub * kTcAtomK,
                      adapter * p.S * p.rs);
      }
      const int k = k0 + 8 * cc;
      const bool k_in = k < p.K;
      // Row j of this thread: zero-filled past the piece and past K, so the
      // copies of a warp never diverge.
      auto copy_row = [&](int j) {
        const int row = rr + j * RSTEP;
        const bool in = k_in && row < rows;
        const uint32_t dst = xs + sub_off + row * 128 + (((cc & 7) ^ (row & 7)) << 4);
        cp_async_16(dst, in ? static_cast<const void*>(xr[j] + k) : static_cast<const void*>(p.x),
                    in ? 16u : 0u);
      };
      if (rows >= kTcBM) {
#pragma unroll
        for (int j = 0; j < CPR; ++j) copy_row(j);
      } else {
        // A short piece: a warp stops once its first row for this j is past
        // the piece (warp-uniform, and true for every later j).  Those stage
        // rows are not written; the accumulator rows they feed are never
        // stored or reduced.  (Full pieces keep the loop without the test,
        // which measured faster for them.)
#pragma unroll
        for (int j = 0; j < CPR; ++j) {
          if (wrow0 + j * RSTEP >= rows) break;
          copy_row(j);
        }
      }
      cp_async_commit();
      if (i >= lag) {
        // stage i - lag has landed for this thread: publish it to the MMA (async proxy)
        cp_async_wait_dyn(lag);
        fence_proxy_async_smem();
        mbar_arrive(full0 + 8 * ((i - lag) % P.stages));
      }
    }
    // drain: publish the stages still in flight, oldest first, each as soon
    // as this thread's copies of it have landed
    if (ok) {
      for (int i = max(0, nk - lag); i < nk; ++i) {
        cp_async_wait_dyn(nk - 1 - i);
        fence_proxy_async_smem();
        mbar_arrive(full0 + 8 * (i % P.stages));
      }
    }
    cp_async_wait<0>();
  } else if (warp == 4) {
    // =========================== MMA issuer
    if (lane == 0) {
      for (int i = 0; i < nk && ok; ++i) {
        const int s = i % P.stages;
        ok = mbar_wait(full0 + 8 * s, (i / P.stages) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t xs = sbase + s * P.stage_bytes;
        const uint32_t as = xs + x_bytes;
#pragma unroll
        for (int kk = 0; kk < kTcBK / 16; ++kk) {
          const uint32_t sub = kk >> 2, k16 = kk & 3;
          const uint64_t ad = make_sdesc(xs + sub * (kTcBM * 128) + k16 * 32, 128, 2);
          const uint64_t bd = make_sdesc(as + sub * (P.npad * 128) + k16 * 32, 128, 2);
          tc_mma_f16(tmem, ad, bd, P.idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(empty0 + 8 * s);
      }
      if (nk > 0) tc_commit(done_bar); else mbar_arrive(done_bar);
    }
    __syncwarp();
  }

  // =========================== epilogue (warps 0-3: one accumulator row per thread)
  // Split-K partials reuse the stage ring as [128][npad + 4] fp32: 16-byte rows
  // whose stride (4 or 20 words mod 32) keeps the row-per-thread 16-byte
  // stores free of bank conflicts.
  float* part = reinterpret_cast<float*>(smem);
  const int pstride = P.npad + 4;
  if (warp < 4) {
    if (ok) ok = mbar_wait(done_bar, 0);
    ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
    tc_fence_after();
    const int m = tid;
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int nvalid = p.S * p.rs;
    for (int c0 = 0; c0 < P.npad; c0 += 16) {
      float v[16];
      if (nk > 0 && ok) {
        tmem_ld16(trow + c0, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
      }
      if (P.csplit == 1) {
        if (m < rows && ok) {
          const int orow_i = P.row_list ? clampi(__ldg(P.row_list + pc.lo + m), 0, p.tok - 1)
                                        : pc.lo + m;
          uint16_t* orow = p.out + static_cast<int64_t>(orow_i) * p.ld_out;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int n = c0 + i;
            if (n < nvalid && (n % p.rs) < p.r) orow[n] = E::f32_to_bits(v[i]);
          }
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(part + m * pstride + c0);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    }
    tc_fence_before();
  }

  if (P.csplit > 1) {
    cluster_sync();  // every partial of the cluster is in shared memory
    // CTA `split` owns rows [split*R, (split+1)*R); a thread sums one 4-column
    // group over all C partials: the C remote 16-byte loads are issued back to
    // back and only then added, in rank order (deterministic).
    const int R = kTcBM / P.csplit;
    const int r0 = split * R;
    const int ng = P.npad / 4;
    const int nvalid = p.S * p.rs;
    const uint32_t pbase = smem_u32(part);
    for (int e = tid; e < R * ng; e += kTcThreads) {
      const int row = r0 + e / ng;
      const int g = e % ng;
      if (row >= rows) continue;
      const uint32_t off = pbase + 4u * static_cast<uint32_t>(row * pstride + 4 * g);
      float4 pv[16];
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (q < P.csplit) pv[q] = ld_dsmem_v4(mapa_shared(off, q));
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        if (q < P.csplit) {
          sum.x += pv[q].x;
          sum.y += pv[q].y;
          sum.z += pv[q].z;
          sum.w += pv[q].w;
        }
      }
      const int orow_i = P.row_list ? clampi(__ldg(P.row_list + pc.lo + row), 0, p.tok - 1)
                                    : pc.lo + row;
      uint16_t* orow = p.out + static_cast<int64_t>(orow_i) * p.ld_out;
      const float sv[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int n = 4 * g + k;
        if (ok && n < nvalid && (n % p.rs) < p.r) orow[n] = E::f32_to_bits(sv[k]);
      }
    }
    // peers are done reading this CTA's partial (their loads have returned:
    // the sums above used them), so the arrive needs no release ordering
    cluster_sync_relaxed();
  }

  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, P.tmem_cols);
  }
}

}  // namespace lora

#undef LORA_KB
