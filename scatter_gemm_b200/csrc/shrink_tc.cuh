// shrink_tc.cuh -- tensor-core shrink (sm_100a); rows at any 2-byte offset in
// the element-aligned variant (AL = false, below).
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
// thread-block cluster (grid = pieces x C, cluster = C CTAs along K).  CTA c
// owns rows [c*128/C, (c+1)*128/C) of the piece: every CTA pushes each of its
// fp32 partial rows into the receive buffer of the row's owner with st.async
// (distributed shared memory, completion counted in bytes on the owner's
// mbarrier), and the owner sums the C partials of its rows in rank order
// (deterministic) and writes them.  No global scratch and no atomics.
#pragma once

#include "common.cuh"
#include "general.cuh"
#include "sched.cuh"
#include "sm100.cuh"

#ifndef LORA_SHRINK_INTERLEAVE
#define LORA_SHRINK_INTERLEAVE 1
#endif
// L2 hints of the x gather (sm100.cuh, cp_async_16_hint)
#ifndef LORA_X_PREFETCH
#define LORA_X_PREFETCH 0
#endif
// L2 prefetch of a block slot's x rows for this many first stages, issued
// once the piece is known (the copies into the stages follow the CTA
// barrier); aligned rows only.  One stage measured best on the qkv workload
// (tok 8192: 28.4 -> 26.8 us; every stage: 27.7 us); for element-aligned
// rows it measured slower.
#ifndef LORA_SHRINK_EARLY_PREFETCH
#define LORA_SHRINK_EARLY_PREFETCH 1
#endif
#ifndef LORA_X_EVICT_FIRST
#define LORA_X_EVICT_FIRST 1
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
  int vec_out;                 // out_r 16-byte aligned with ld_out % 8 == 0
  int recv_in_ring;            // split-K partials received in the (then idle) stage ring
};

// Row staging of the element-aligned variant: the 16-byte blocks that cover
// one row's 64 elements of a stage (at most 9), 144 bytes per row, so that
// eight consecutive rows fall in eight different bank groups.
constexpr int kRawRow = 144;

// NSUB: 64-K sub-tiles per stage (stage K width = 64 * NSUB).
// AL: x and A rows are 16-byte aligned with K % 8 == 0 (x rows by 16-byte
// cp.async, A by TMA).  Otherwise (any 2-byte alignment, any K; NSUB = 1) each
// producer thread copies the aligned 16-byte blocks that cover its own x row
// (and A row) into a staging area of the stage, then shifts them into the
// swizzled layout the MMA reads, zero-filling past K.
template <class E, int NSUB, bool AL>
__global__ void __launch_bounds__(kTcThreads, 1)
shrink_tc_kernel(const __grid_constant__ ShrinkTcParams P) {
  static_assert(AL || NSUB == 1, "the element-aligned stage is 64 K wide");
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
  // split-K receive buffer: [C sources][128/C rows][npad] fp32, after the
  // ring, or in the ring itself once every CTA of the cluster has finished its
  // MMAs (when a separate buffer would leave too few stages)
  float* recv = reinterpret_cast<float*>(smem + (P.recv_in_ring ? 0 : P.stages * P.stage_bytes));
  const uint32_t recv_bytes = P.csplit > 1 && !P.recv_in_ring ? kTcBM * P.npad * 4 : 0;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P.stages * P.stage_bytes + recv_bytes);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * P.stages;
  const uint32_t done_bar = empty0 + 8 * P.stages;
  const uint32_t recv_bar = done_bar + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * P.stages + 2);
  int64_t* xrow_tok = reinterpret_cast<int64_t*>(bars + 2 * P.stages + 3);  // [128] x row index
  // receive buffer in the ring: ready[c] completes once CTA c of the cluster
  // has finished its MMAs (its ring may then receive partials)
  const uint32_t ready0 = smem_u32(xrow_tok + kTcBM);  // [csplit] mbarriers

  // barriers and TMEM first, so that their latency overlaps the table reads
  if (tid == 0) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(full0 + 8 * s, AL ? kTcBM + 1 : kTcBM);  // + the A transfer (TMA)
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(done_bar, 1);
    mbar_init(recv_bar, 1);
    if (P.recv_in_ring)
      for (int c = 0; c < P.csplit; ++c) mbar_init(ready0 + 8 * c, 1);
    fence_mbar_init();
    if (AL) tma_prefetch_desc(&P.tmap_A);
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), P.tmem_cols);
    tmem_relinquish();
  }
  // the receive barrier (and the ready barriers) must be initialised before
  // any peer pushes or arrives: arrive now, wait after the MMAs
  const bool early_arrive = P.csplit > 1;
  if (early_arrive) cluster_arrive_relaxed();

  // the grouping pass ahead of this kernel (when there is one) has finished:
  // everything above overlapped it
  griddep_wait();

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
    if (early_arrive) cluster_wait();  // pairs the arrive above
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
      tc_fence_after();
      tmem_dealloc(*tmem_slot, P.tmem_cols);
    }
    return;
  }
  if (AL && LORA_SHRINK_EARLY_PREFETCH > 0 && tid < kTcBM && block_slot) {
    // L2 prefetch of this row's x columns for the first stages, before the
    // CTA barrier (every address lies inside row spec_tok, a valid token)
    const uint16_t* xr = p.x + static_cast<int64_t>(spec_tok) * p.ld_x;
    const int npre = min(nk, min(P.stages, LORA_SHRINK_EARLY_PREFETCH));
    for (int i = 0; i < npre; ++i) {
      const int k0 = LORA_KB(i) * kTcBK;
      const int k1 = min(p.K, k0 + kTcBK);
      // every 128-byte line holding one of the columns [k0, k1)
      const uintptr_t l0 = reinterpret_cast<uintptr_t>(xr + k0) & ~static_cast<uintptr_t>(127);
      const uintptr_t l1 = reinterpret_cast<uintptr_t>(xr + k1 - 1);
      for (uintptr_t l = l0; l <= l1; l += 128) prefetch_l2(reinterpret_cast<const void*>(l));
    }
  }
  const int rows = pc.hi - pc.lo;
  const int adapter = pc.adapter;
  const int R = kTcBM / P.csplit;  // rows owned by each CTA of the cluster
  const int nmine = max(0, min(R, rows - split * R));

  // The adapter's A blocks of the first stages do not depend on the x rows:
  // request them now, before the row tokens are known.
  const uint32_t a_sub = P.npad * 128;  // one 64-K sub-tile of A
  const uint32_t a_bytes = kTcNSub * a_sub;
  const int pre_a = AL ? min(nk, P.stages) : 0;
  if (tid == 0) {
    for (int i = 0; i < pre_a; ++i) {
      const uint32_t as = sbase + i * P.stage_bytes + x_bytes;
      const int k0 = LORA_KB(i) * kTcBK;
      mbar_arrive_expect_tx(full0 + 8 * i, a_bytes);
#pragma unroll
      for (int sub = 0; sub < kTcNSub; ++sub)
        tma_load_2d(as + sub * a_sub, &P.tmap_A, full0 + 8 * i, k0 + sub * kTcAtomK,
                    adapter * p.S * p.rs);
    }
    if (P.csplit > 1)
      mbar_arrive_expect_tx(recv_bar, static_cast<uint32_t>(P.csplit * nmine * P.npad * 4));
  }

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

  if (!AL && warp < 4) {
    // =========================== producer, element-aligned rows
    // Thread m stages x row m and A rows m and m + 128 of the stage's 64 K
    // columns: copy the covering 16-byte blocks (16-byte cp.async, one row
    // per thread), and once they have landed (lagged like the aligned path)
    // shift them into the swizzled K-major layout, zero past K.
    const int m = tid;
    const uint32_t raw_x = x_bytes + P.npad * 128;     // offsets inside a stage
    const uint32_t raw_a = raw_x + kTcBM * kRawRow;
    const uint16_t* rowp[3];
    bool rowok[3];
    uint32_t rawo[3], dsto[3];
    int rown[3];
    rowp[0] = p.x + xrow_tok[m] * p.ld_x;
    rowok[0] = m < rows;
    rawo[0] = raw_x + m * kRawRow;
    dsto[0] = m * 128;
    rown[0] = m;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = m + 128 * h;
      rowok[1 + h] = n < P.npad && n < p.S * p.rs;
      rowp[1 + h] = p.A + (static_cast<int64_t>(adapter) * p.S * p.rs + (rowok[1 + h] ? n : 0)) *
                              p.K;
      rawo[1 + h] = raw_a + n * kRawRow;
      dsto[1 + h] = x_bytes + n * 128;
      rown[1 + h] = n;
    }
    auto issue_rows = [&](uint32_t st, int k0) {
      const int nv = min(kTcAtomK, p.K - k0);
#pragma unroll
      for (int h = 0; h < 3; ++h) {
        if (!rowok[h]) continue;
        const uintptr_t a = reinterpret_cast<uintptr_t>(rowp[h] + k0);
        const uintptr_t a0 = a & ~static_cast<uintptr_t>(15);
        // blocks holding at least one of the nv elements (<= 9)
        const int nb = static_cast<int>(((a + 2 * nv + 15) & ~static_cast<uintptr_t>(15)) - a0) >> 4;
        const uint8_t* src = reinterpret_cast<const uint8_t*>(a0);
#pragma unroll
        for (int b = 0; b < 9; ++b)
          if (b < nb) cp_async_16(st + rawo[h] + 16 * b, src + 16 * b, 16u);
      }
    };
    // The staged row is a byte stream: element k0 + e sits at byte off + 2e
    // (off = source address & 15).  Word k of the shifted row (elements
    // 2k, 2k+1) is the 4 bytes at off + 4k: staged words q + k and q + k + 1
    // (q = off / 4) funnel-shifted by 16 bits when off % 4 == 2.  The word
    // index is an address offset, so every load below has a constant offset
    // from the row's base; elements past K are zeroed in the last stage only.
    auto realign_rows = [&](int j) {
      uint8_t* stp = smem + (j % P.stages) * P.stage_bytes;
      const int k0 = LORA_KB(j) * kTcBK;
      const int nv = min(kTcAtomK, p.K - k0);
#pragma unroll
      for (int h = 0; h < 3; ++h) {
        if (!rowok[h]) continue;
        const int off = static_cast<int>(reinterpret_cast<uintptr_t>(rowp[h] + k0) & 15);
        const uint32_t* w = reinterpret_cast<const uint32_t*>(stp + rawo[h]) + (off >> 2);
        const uint32_t fs = (off & 2) * 8;  // 0 or 16 bits
        uint8_t* dst = stp + dsto[h];
        const int sw = rown[h] & 7;
        uint32_t ws[33];  // every staged word first: the stores below may alias them
#pragma unroll
        for (int i = 0; i < 33; ++i) ws[i] = w[i];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) o[i] = __funnelshift_r(ws[4 * c + i], ws[4 * c + i + 1], fs);
          uint4 v = make_uint4(o[0], o[1], o[2], o[3]);
          if (nv < kTcAtomK) v = keep_elems(v, nv - 8 * c);
          *reinterpret_cast<uint4*>(dst + ((c ^ sw) << 4)) = v;
        }
      }
    };
    const int lag = P.stages - 1;
    for (int i = 0; i < nk && ok; ++i) {
      const int s = i % P.stages;
      if (i >= P.stages) ok = mbar_wait(empty0 + 8 * s, ((i / P.stages) - 1) & 1);
      if (!ok) break;
      issue_rows(sbase + s * P.stage_bytes, LORA_KB(i) * kTcBK);
      cp_async_commit();
      if (i >= lag) {
        cp_async_wait_dyn(lag);
        realign_rows(i - lag);
        fence_proxy_async_smem();
        mbar_arrive(full0 + 8 * ((i - lag) % P.stages));
      }
    }
    if (ok) {
      for (int i = max(0, nk - lag); i < nk; ++i) {
        cp_async_wait_dyn(nk - 1 - i);
        realign_rows(i);
        fence_proxy_async_smem();
        mbar_arrive(full0 + 8 * (i % P.stages));
      }
    }
    cp_async_wait<0>();
  } else if (warp < 4) {
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
    // gathered x row of each of this thread's CPR rows (rows past the piece are
    // never read)
    const uint16_t* xr[CPR];
#pragma unroll
    for (int j = 0; j < CPR; ++j) xr[j] = p.x + xrow_tok[rr + j * RSTEP] * p.ld_x;
    const int lag = P.stages - 1;
    const uint64_t pol = LORA_X_EVICT_FIRST ? policy_evict_first() : 0;
    for (int i = 0; i < nk && ok; ++i) {
      const int s = i % P.stages;
      if (i >= P.stages) ok = mbar_wait(empty0 + 8 * s, ((i / P.stages) - 1) & 1);
      if (!ok) break;
      const uint32_t xs = sbase + s * P.stage_bytes;
      const int k0 = LORA_KB(i) * kTcBK;
      if (tid == 0 && i >= pre_a) {
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
        cp_async_16_hint<LORA_X_PREFETCH, LORA_X_EVICT_FIRST != 0>(
            dst, in ? static_cast<const void*>(xr[j] + k) : static_cast<const void*>(p.x),
            in ? 16u : 0u, pol);
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
  const int nvalid = p.S * p.rs;
  // columns [n0, n0+8) of output row `orow_i`, rounded once: one 16-byte store
  // when all eight are valid outputs (j < r) and the row is 16-byte aligned,
  // otherwise element by element
  auto store8 = [&](int orow_i, int n0, const float* v) {
    uint16_t* orow = p.out + static_cast<int64_t>(orow_i) * p.ld_out;
    const bool full = P.vec_out && n0 + 8 <= nvalid && (n0 % p.rs) + 8 <= p.r;
    if (full) {
      uint4 w;
      w.x = E::f2_to_u32(v[0], v[1]);
      w.y = E::f2_to_u32(v[2], v[3]);
      w.z = E::f2_to_u32(v[4], v[5]);
      w.w = E::f2_to_u32(v[6], v[7]);
      stg128(orow + n0, w);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int n = n0 + i;
        if (n < nvalid && (n % p.rs) < p.r) stg16(orow + n, E::f32_to_bits(v[i]));
      }
    }
  };
  if (warp < 4) {
    if (ok) ok = mbar_wait(done_bar, 0);
    ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
  }
  if (P.csplit > 1) {
    cluster_wait();  // every receive and ready barrier of the cluster is initialised
    // a receive buffer in the ring: this CTA's MMAs are done, so tell every
    // CTA of the cluster that its pushes may come (release: the MMAs' reads
    // of the ring come first)
    if (P.recv_in_ring && tid < P.csplit) mbar_arrive_cluster(mapa_shared(ready0 + 8 * split, tid));
  }
  if (warp < 4) {
    tc_fence_after();
    const int m = tid;
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    // split-K: row m goes to CTA m / R of the cluster, into the slot of this
    // CTA's rank; into a ring, only once that CTA is ready (its MMAs done)
    const int owner = m / R;
    if (P.recv_in_ring) {
      if (ok) ok = mbar_wait_cluster(ready0 + 8 * owner, 0);
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
    }
    const uint32_t rdst = P.csplit > 1
        ? mapa_shared(smem_u32(recv) + 4u * static_cast<uint32_t>((split * R + m % R) * P.npad),
                      owner)
        : 0u;
    const uint32_t rbar = P.csplit > 1 ? mapa_shared(recv_bar, owner) : 0u;
    const int orow_i = P.csplit == 1 && m < rows
        ? (P.row_list ? clampi(__ldg(P.row_list + pc.lo + m), 0, p.tok - 1) : pc.lo + m)
        : 0;
    for (int c0 = 0; c0 < P.npad; c0 += 16) {
      float v[16];
      if (nk > 0 && ok) {
        tmem_ld16(trow + c0, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
      }
      if (m < rows && ok) {
        if (P.csplit == 1) {
          store8(orow_i, c0, v);
          store8(orow_i, c0 + 8, v + 8);
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            st_async_v4(rdst + 4u * static_cast<uint32_t>(c0 + 4 * k),
                        make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]), rbar);
        }
      }
    }
    tc_fence_before();
  }

  if (P.csplit > 1) {
    // rows [split*R, split*R + nmine) of the piece: the C partials of each
    // 8-column group summed in rank order (deterministic), rounded once
    if (ok) ok = mbar_wait(recv_bar, 0);
    const int ng = P.npad / 8;
    for (int e = tid; e < nmine * ng && ok; e += kTcThreads) {
      const int lr = e / ng, n0 = 8 * (e % ng);
      float sum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int src = 0; src < P.csplit; ++src) {
        const float4* pp = reinterpret_cast<const float4*>(recv + (src * R + lr) * P.npad + n0);
        const float4 a0 = pp[0], a1 = pp[1];
        sum[0] += a0.x; sum[1] += a0.y; sum[2] += a0.z; sum[3] += a0.w;
        sum[4] += a1.x; sum[5] += a1.y; sum[6] += a1.z; sum[7] += a1.w;
      }
      const int row = split * R + lr;
      const int orow_i = P.row_list ? clampi(__ldg(P.row_list + pc.lo + row), 0, p.tok - 1)
                                    : pc.lo + row;
      store8(orow_i, n0, sum);
    }
    // a CTA leaves only after its peers: none of them is still writing into it
    // (each waited for its own receive), and none still needs this CTA
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
