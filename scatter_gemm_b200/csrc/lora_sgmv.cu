// lora_sgmv.cu -- C ABI of liblora_sgmv: argument checks, kernel selection and
// launches of the chunked-SGMV LoRA shrink/expand pair (sgl-kernel-xpu page
// "Decode LoRA kernels are optimized", sections "Summary" and "Behaviour
// changes").  Nothing here reads a device table on the host and nothing is
// synchronised: every call enqueues its kernels on the caller's stream.
//
// Kernel selection (run time, from pointers and sizes only):
//   shrink: shrink_tc when the padded width S*rs <= 256, its aligned variant
//   when x and A rows are 16-byte aligned with K % 8 == 0 (else the variant
//   that stages and shifts element-aligned rows); expand: expand_tc when every
//   tensor it streams is 16-byte aligned with 16-byte-multiple row strides,
//   slice starts % 8 == 0 and r <= 64, else expand_unaligned for r <= 64; the
//   CUDA-core kernels of general.cuh for what remains (r > 64, S*rs > 256).
//   With a workspace, more segments than adapters and at least 64 KB of
//   weight reads to save, the tensor-core kernels run on the adapter-grouped
//   schedule of group.cuh.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/lora_sgmv.h"
#include "common.cuh"
#include "embedding.cuh"
#include "expand_tc.cuh"
#include "expand_unaligned_tc.cuh"
#include "base_expand_tc.cuh"
#include "fused_tc.cuh"
#include "general.cuh"
#include "group.cuh"
#include "sched.cuh"
#include "shrink_tc.cuh"
#include "sm100.cuh"

// Tuning constants of the expand (compile-time; defaults below).
#ifndef LORA_EXPAND_CTAS_PER_SM
#define LORA_EXPAND_CTAS_PER_SM 2   // 2: <= 113 KB per CTA; 1: deep ring (<= 225 KB)
#endif
#ifndef LORA_EXPAND_WAVES
#define LORA_EXPAND_WAVES 1         // resident-CTA waves the grid is sized for
#endif
#ifndef LORA_SHRINK_CTAS_PER_SM
#define LORA_SHRINK_CTAS_PER_SM 2  // 2: <= 110 KB shared memory per CTA; 1: deepest ring
#endif
#ifndef LORA_SHRINK_MIN_SPLIT
#define LORA_SHRINK_MIN_SPLIT 1    // smallest K split (CTAs per cluster) of the shrink
#endif
#ifndef LORA_EXPAND_B_STAGES
#define LORA_EXPAND_B_STAGES 3
#endif
#ifndef LORA_SHRINK_RING_BELOW
#define LORA_SHRINK_RING_BELOW 3    // split-K partials into the ring below this many stages
#endif
#ifndef LORA_BASE_EXPAND_CTAS_PER_SM
#define LORA_BASE_EXPAND_CTAS_PER_SM 2  // base projection: 2 when three stages fit in 113 KB
#endif
#ifndef LORA_EU_CTAS_PER_SM
#define LORA_EU_CTAS_PER_SM 2       // element-aligned expand: CTAs per SM when they fit
#endif
#ifndef LORA_SHRINK_WIDE_SMEM
#define LORA_SHRINK_WIDE_SMEM 0     // 1: one-CTA-per-SM budget when the grid fits the SMs
#endif

namespace {

thread_local uint64_t g_launches = 0;
thread_local int g_last_path = 0;

constexpr int kMaxDevices = 64;

// Every kernel of this library that holds TMEM allocates at most 256 columns
// and asks for at least this much dynamic shared memory, so that no more than
// two of its CTAs fit on one SM (228 KB) and their allocations (2 x 256 of 512
// columns) never wait for each other, whatever calls run concurrently on
// other streams: a CTA blocked in tcgen05.alloc while its cluster peers hold
// TMEM and wait at a cluster barrier could otherwise deadlock.
constexpr size_t kTmemCtaMinSmem = 80 * 1024;

inline bool aligned_to(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

inline lora_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

// ------------------------------------------------------------------ device facts

struct DeviceFacts {
  std::atomic<int> ready{0};
  int sms = 148;
  int max_cluster = 8;  // largest K-split cluster the shrink may use
  // clusters of 1, 2, 4, 8, 16 CTAs of the fused kernel (one CTA per SM) that
  // can be resident at once
  int fused_clusters[5] = {0, 0, 0, 0, 0};
};
DeviceFacts g_dev[kMaxDevices];
std::mutex g_dev_mu;

template <class E, int NSUB, bool AL>
void set_shrink_attrs() {
  cudaFuncSetAttribute(lora::shrink_tc_kernel<E, NSUB, AL>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  cudaFuncSetAttribute(lora::shrink_tc_kernel<E, NSUB, AL>,
                       cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
}

template <class E>
void set_kernel_attrs() {
  set_shrink_attrs<E, 1, true>();
  set_shrink_attrs<E, 2, true>();
  set_shrink_attrs<E, 4, true>();
  set_shrink_attrs<E, 1, false>();
  cudaFuncSetAttribute(lora::expand_tc_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       227 * 1024);
  cudaFuncSetAttribute(lora::expand_general_kernel<E>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  cudaFuncSetAttribute(lora::expand_unaligned_kernel<E>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  cudaFuncSetAttribute(lora::fused_tc_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       227 * 1024);
  cudaFuncSetAttribute(lora::base_expand_tc_kernel<E>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  cudaFuncSetAttribute(lora::fused_tc_kernel<E>, cudaFuncAttributeNonPortableClusterSizeAllowed,
                       1);
}

const DeviceFacts* device_facts() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceFacts& f = g_dev[dev];
  if (f.ready.load(std::memory_order_acquire)) return &f;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!f.ready.load(std::memory_order_relaxed)) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return nullptr;
    f.sms = sms;
    set_kernel_attrs<lora::Bf16>();
    set_kernel_attrs<lora::Fp16>();
    cudaFuncSetAttribute(lora::group_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         lora::kGroupStageBytes);
    cudaFuncSetAttribute(lora::group_rows_small_kernel,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, lora::kGroupStageBytes);
    // can 16 CTAs of the shrink (at its largest two-per-SM footprint) form a cluster?
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 16;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(16 * 16);
    cfg.blockDim = dim3(lora::kTcThreads);
    cfg.dynamicSmemBytes = 112 * 1024;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, lora::shrink_tc_kernel<lora::Bf16, 1, true>,
                                       &cfg) ==
            cudaSuccess &&
        nclusters > 0)
      f.max_cluster = 16;
    cudaGetLastError();  // the probe above must not leave a sticky launch error
    for (int i = 0; i < 5; ++i) {
      attr[0].val.clusterDim.x = 1u << i;
      cfg.gridDim = dim3(16u << i);
      cfg.blockDim = dim3(lora::kFuThreads);
      cfg.dynamicSmemBytes = 200 * 1024;
      int nc = 0;
      if (cudaOccupancyMaxActiveClusters(&nc, lora::fused_tc_kernel<lora::Bf16>, &cfg) ==
          cudaSuccess)
        f.fused_clusters[i] = nc;
      cudaGetLastError();
    }
    f.ready.store(1, std::memory_order_release);
  }
  return &f;
}

// ------------------------------------------------------------------ TMA tensor maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor of 16-bit elements: `cols` valid columns, `rows` rows,
// `row_bytes` between rows; box {box_cols, box_rows}.
bool encode_2d(CUtensorMap* m, lora_dtype dt, const void* base, uint64_t cols, uint64_t rows,
               uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows,
               CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, dt == LORA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                            : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D tiled map: dims {d0 (contiguous), d1, d2}, byte strides s1 (dim 1) and
// s2 (dim 2), box {b0, b1, b2}.
bool encode_3d(CUtensorMap* m, lora_dtype dt, const void* base, uint64_t d0, uint64_t d1,
               uint64_t d2, uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2,
               CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, dt == LORA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                            : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ workspace

struct Grouping {
  const int32_t* vseg_indptr = nullptr;
  const int32_t* row_list = nullptr;
  int nvseg = 0;
};

#ifndef LORA_PDL
#define LORA_PDL 1  // kernels after the grouping pass start while it runs
#endif

// Launch attributes of a tensor-core kernel: its cluster shape, and, right
// after the grouping pass, programmatic serialisation: its CTAs are placed and
// run their set-up (barriers, TMEM) while the pass finishes, then wait for it
// (griddep_wait) before reading the lists.
struct LaunchAttrs {
  cudaLaunchAttribute a[2];
  unsigned n = 0;
  void cluster(unsigned x) {
    a[n].id = cudaLaunchAttributeClusterDimension;
    a[n].val.clusterDim.x = x;
    a[n].val.clusterDim.y = 1;
    a[n].val.clusterDim.z = 1;
    ++n;
  }
  void after_grouping(const Grouping& g) {
    if (!LORA_PDL || g.vseg_indptr == nullptr) return;
    a[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  void apply(cudaLaunchConfig_t& cfg) {
    cfg.attrs = n ? a : nullptr;
    cfg.numAttrs = n;
  }
};

inline size_t a16(size_t n) { return (n + 3) / 4 * 4; }  // ints -> multiple of 4 ints

size_t workspace_ints(int tok, int nseg, int L) {
  return a16(static_cast<size_t>(L) + 1) + a16(static_cast<size_t>(nseg)) +
         a16(static_cast<size_t>(tok));
}

// Narrowed int64 tables at the front of an *_i64 call's workspace:
// [seg_indptr (nseg+1)][weight_indices (nseg)][permutation (tok)], each padded
// to 16 bytes, so the rest of the workspace stays 16-byte aligned.
size_t index64_bytes(int tok, int nseg) {
  return 4 * (a16(static_cast<size_t>(nseg) + 1) + a16(static_cast<size_t>(nseg)) +
              a16(static_cast<size_t>(tok)));
}

// Checks of the arguments of lora_shrink other than its pointers.
lora_status shrink_scalar_check(int64_t ld_x, int64_t ld_out, int tok, int K, int S, int r,
                                int rs, int nseg, int L, lora_dtype dtype, const void* workspace,
                                size_t workspace_bytes) {
  if (dtype != LORA_BF16 && dtype != LORA_FP16) return LORA_ERR_UNSUPPORTED;
  if (tok < 0 || nseg < 0 || K < 1 || S < 1 || r < 1 || rs < r || L < 1)
    return LORA_ERR_INVALID_ARGUMENT;
  if (S > LORA_MAX_SLICES) return LORA_ERR_UNSUPPORTED;
  if (ld_x < K || ld_out < static_cast<int64_t>(S) * rs) return LORA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes > 0 && !workspace) return LORA_ERR_INVALID_ARGUMENT;
  return LORA_OK;
}

// Checks of the arguments of lora_expand other than its device pointers;
// fills the slice table.
lora_status expand_scalar_check(int64_t ld_in, int64_t ld_base, int tok, int S, int r, int rs,
                                int nseg, int L, const int32_t* slice_offsets, lora_dtype dtype,
                                const void* workspace, size_t workspace_bytes,
                                lora::SliceTable& tab) {
  if (dtype != LORA_BF16 && dtype != LORA_FP16) return LORA_ERR_UNSUPPORTED;
  if (tok < 0 || nseg < 0 || S < 1 || r < 1 || rs < r || L < 1)
    return LORA_ERR_INVALID_ARGUMENT;
  if (S > LORA_MAX_SLICES) return LORA_ERR_UNSUPPORTED;
  if (!slice_offsets) return LORA_ERR_INVALID_ARGUMENT;
  if (ld_in < static_cast<int64_t>(S) * rs) return LORA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes > 0 && !workspace) return LORA_ERR_INVALID_ARGUMENT;
  tab = lora::SliceTable{};
  tab.S = S;
  for (int q = 0; q <= S; ++q) {
    tab.off[q] = slice_offsets[q];
    if (slice_offsets[q] < 0 || slice_offsets[q] > ld_base) return LORA_ERR_INVALID_ARGUMENT;
    if (q > 0 && slice_offsets[q] < slice_offsets[q - 1]) return LORA_ERR_INVALID_ARGUMENT;
  }
  return LORA_OK;
}

// Narrows the int64 tables of an *_i64 call into the front of `ws`, at the
// offsets index64_bytes lays out.
lora_status narrow_tables(const int64_t* seg_indptr, const int64_t* weight_indices,
                          const int64_t* permutation, int tok, int nseg, int32_t* ws,
                          cudaStream_t st) {
  const int pa = static_cast<int>(a16(static_cast<size_t>(nseg) + 1));
  const int pb = static_cast<int>(a16(static_cast<size_t>(nseg)));
  const int nc = permutation ? tok : 0;
  const int64_t total = static_cast<int64_t>(pa) + pb + nc;
  const int threads = 256;
  const unsigned blocks = static_cast<unsigned>((total + threads - 1) / threads);
  lora::narrow_index_kernel<<<blocks, threads, 0, st>>>(seg_indptr, nseg + 1, pa,
                                                        weight_indices, nseg, pb,
                                                        permutation, nc, ws);
  ++g_launches;
  return launch_status();
}

// Enqueues the grouping pass when the schedule calls for it.
// piece_weight_bytes: the adapter weights one piece of rows reads (A for the
// shrink, B for the expand).  Grouping saves about one such read for every
// segment beyond one per adapter; below kGroupMinSavedBytes of them the pass
// (one more kernel on the stream) costs more than it saves.
constexpr int64_t kGroupMinSavedBytes = 64 * 1024;

bool grouping_pays(int nseg, int L, int64_t piece_weight_bytes) {
  return nseg > L && L <= lora::kGroupMaxAdapters &&
         static_cast<int64_t>(nseg - L) * piece_weight_bytes >= kGroupMinSavedBytes;
}

lora_status maybe_group(const int32_t* seg_indptr, const int32_t* weight_indices, int tok,
                        int nseg, int L, int64_t piece_weight_bytes, void* ws, size_t ws_bytes,
                        cudaStream_t st, Grouping& g) {
  g = Grouping{};
  if (!ws || !grouping_pays(nseg, L, piece_weight_bytes)) return LORA_OK;
  if (!device_facts()) return LORA_ERR_CUDA;  // sets the pass's shared-memory limit
  if (!aligned_to(ws, 16) || ws_bytes < workspace_ints(tok, nseg, L) * 4) return LORA_OK;
  int32_t* w = static_cast<int32_t*>(ws);
  int32_t* vseg = w;
  int32_t* seg_base = vseg + a16(static_cast<size_t>(L) + 1);
  int32_t* rows = seg_base + a16(static_cast<size_t>(nseg));
  if (lora::group_small_fits(nseg, L, tok)) {
    lora::group_rows_small_kernel<<<1, lora::kGroupThreads,
                                    static_cast<size_t>(lora::group_small_smem(nseg, L, tok)), st>>>(
        seg_indptr, weight_indices, nseg, L, tok, vseg, rows);
  } else {
    const size_t gsmem = sizeof(int) * (lora::group_stages_tables(nseg, L)
                                            ? static_cast<size_t>(L) + 3 * static_cast<size_t>(nseg) + 1
                                            : static_cast<size_t>(L));
    lora::group_rows_kernel<<<1, lora::kGroupThreads, gsmem, st>>>(
        seg_indptr, weight_indices, nseg, L, tok, vseg, seg_base, rows);
  }
  ++g_launches;
  if (launch_status() != LORA_OK) return LORA_ERR_CUDA;
  g.vseg_indptr = vseg;
  g.row_list = rows;
  g.nvseg = L;
  return LORA_OK;
}

// ------------------------------------------------------------------ shrink

template <class E>
lora_status shrink_general(const lora::ShrinkArgs& a, cudaStream_t st) {
  const int slots = lora::num_piece_slots(a.tok, a.nseg, lora::kGBM);
  const int groups = (a.S * a.r + lora::kGNPC - 1) / lora::kGNPC;
  if (groups > 65535) return LORA_ERR_UNSUPPORTED;
  dim3 grid(slots, groups);
  lora::shrink_general_kernel<E><<<grid, lora::kGWarps * 32, 0, st>>>(a);
  ++g_launches;
  g_last_path = LORA_PATH_GENERAL;
  return launch_status();
}

// The tensor-core shrink: aligned (16-byte rows, TMA for A) or element-aligned
// (row staging and shifts); the CUDA-core kernel only beyond 256 outputs.
bool shrink_tc_eligible(const lora::ShrinkArgs& a) {
  const int npad = round_up(a.S * a.rs, 16);
  return npad <= 256 && static_cast<int64_t>(a.L) * a.S * a.rs < (int64_t(1) << 31) &&
         a.tok < (1 << 30);
}

bool shrink_tc_aligned(const lora::ShrinkArgs& a) {
  return aligned_to(a.x, 16) && (a.ld_x % 8) == 0 && (a.K % 8) == 0 && aligned_to(a.A, 16);
}

template <class E>
lora_status shrink_tc(const lora::ShrinkArgs& a, lora_dtype dt, const Grouping& g,
                      const DeviceFacts& dev, cudaStream_t st) {
  lora::ShrinkTcParams P;
  std::memset(&P, 0, sizeof(P));
  P.a = a;
  P.row_list = g.row_list;
  P.vseg_indptr = g.vseg_indptr;
  P.nvseg = g.vseg_indptr ? g.nvseg : a.nseg;
  P.npad = round_up(a.S * a.rs, 16);
  P.tmem_cols = P.npad <= 32 ? 32 : P.npad <= 64 ? 64 : P.npad <= 128 ? 128 : 256;
  // widest stage (64-K sub-tiles of x and A) that still leaves two stages
  // inside the shared-memory budget
  int budget = (LORA_SHRINK_CTAS_PER_SM >= 2 && P.npad <= 128 ? 110 : 220) * 1024;
  const bool al = shrink_tc_aligned(a);
  int nsub = al ? lora::kTcMaxNSub : 1;
  for (;; nsub /= 2) {
    const int sb = nsub * (lora::kTcBM * 128 + P.npad * 128);
    if (nsub == 1 || 2 * sb <= budget - 2048) break;
  }
  P.stage_bytes = nsub * (lora::kTcBM * 128 + P.npad * 128);
  if (!al)  // plus the staging of x rows and A rows
    P.stage_bytes = static_cast<uint32_t>(round_up(
        static_cast<int>(P.stage_bytes) + (lora::kTcBM + P.npad) * lora::kRawRow, 1024));
  P.nkb = (a.K + nsub * lora::kTcAtomK - 1) / (nsub * lora::kTcAtomK);

  if (al && !encode_2d(&P.tmap_A, dt, a.A, a.K, static_cast<uint64_t>(a.L) * a.S * a.rs,
                       static_cast<uint64_t>(a.K) * 2, lora::kTcAtomK, P.npad,
                       CU_TENSOR_MAP_SWIZZLE_128B))
    return LORA_ERR_CUDA;
  // K split over a cluster: the smallest power of two that gives every SM a CTA
  // (expected pieces: one per 128 rows plus about half a piece per segment),
  // keeping at least four stages of K per CTA.  (Splitting further, to fill
  // every resident CTA slot, measured slower: more partials to reduce.)
  const int est = (a.tok + lora::kTcBM - 1) / lora::kTcBM + (P.vseg_indptr ? a.L : a.nseg) / 2;
  // a grid that fits one CTA per SM may use the shared memory of two, with
  // clusters of at most 8 (two per GPC at one CTA per SM)
  const long nslots = lora::num_piece_slots(a.tok, P.nvseg, lora::kTcBM);
  const bool wide = LORA_SHRINK_WIDE_SMEM && nslots * 8 <= dev.sms;
  const int max_cs = wide ? std::min(dev.max_cluster, 8) : dev.max_cluster;
  int cs = 1;
  while (cs < max_cs && P.nkb >= 4 * cs && (est * cs < dev.sms || cs < LORA_SHRINK_MIN_SPLIT))
    cs *= 2;
#ifdef LORA_SHRINK_FORCE_CS
  cs = LORA_SHRINK_FORCE_CS;
  if (P.nkb < cs) cs = 1;
#endif
  P.csplit = cs;
  P.kb_per = (P.nkb + cs - 1) / cs;
  P.idesc = lora::make_idesc_f16(dt == LORA_BF16 ? 1 : 0, lora::kTcBM, P.npad);
  P.vec_out = aligned_to(a.out, 16) && (a.ld_out % 8) == 0;
  // ring stages in what the split-K receive buffer leaves of the budget; when
  // the whole grid fits one CTA per SM, the budget of one CTA per SM
  if (wide && nslots * cs <= dev.sms) budget = 220 * 1024;
#ifdef LORA_SHRINK_FORCE_WIDE
  budget = LORA_SHRINK_FORCE_WIDE ? 220 * 1024 : 110 * 1024;
#endif
  const size_t recv_full = cs > 1 ? static_cast<size_t>(lora::kTcBM) * P.npad * 4 : 0;
  auto smem_for = [&](int stages, size_t recv) {
    return static_cast<size_t>(stages) * P.stage_bytes + recv + 1024 + 8 * (2 * stages + 3) +
           8 * lora::kTcBM + 8 * 16;  // row indices, ready barriers
  };
  auto stages_for = [&](size_t recv) {
    int st = 2;
    while (st < 8 && smem_for(st + 1, recv) <= static_cast<size_t>(budget)) ++st;
    return st;
  };
  // a separate receive buffer when it leaves at least three stages; otherwise
  // the partials are received in the ring, each CTA's once its MMAs are done
  P.stages = stages_for(recv_full);
  P.recv_in_ring = 0;
  if (cs > 1 && P.stages < LORA_SHRINK_RING_BELOW) {
    P.recv_in_ring = 1;
    P.stages = stages_for(0);
    while (static_cast<size_t>(P.stages) * P.stage_bytes < recv_full) ++P.stages;
  }
  const size_t smem_need =
      std::max<size_t>(smem_for(P.stages, P.recv_in_ring ? 0 : recv_full), kTmemCtaMinSmem);
  const size_t smem = smem_need;
  const long slots = lora::num_piece_slots(a.tok, P.nvseg, lora::kTcBM);
  cudaLaunchConfig_t cfg{};
  LaunchAttrs attrs;
  cfg.gridDim = dim3(static_cast<unsigned>(slots * cs));
  cfg.blockDim = dim3(lora::kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  if (cs > 1) attrs.cluster(cs);
  attrs.after_grouping(g);
  attrs.apply(cfg);
  if (smem > 227 * 1024) return LORA_ERR_UNSUPPORTED;
  cudaError_t e;
  if (!al) e = cudaLaunchKernelEx(&cfg, lora::shrink_tc_kernel<E, 1, false>, P);
  else if (nsub == 4) e = cudaLaunchKernelEx(&cfg, lora::shrink_tc_kernel<E, 4, true>, P);
  else if (nsub == 2) e = cudaLaunchKernelEx(&cfg, lora::shrink_tc_kernel<E, 2, true>, P);
  else e = cudaLaunchKernelEx(&cfg, lora::shrink_tc_kernel<E, 1, true>, P);
  ++g_launches;
  g_last_path = LORA_PATH_TENSOR | (cs > 1 ? LORA_PATH_SPLITK : 0) |
                (P.vseg_indptr ? LORA_PATH_GROUPED : 0);
  return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

// ------------------------------------------------------------------ expand

template <class E>
lora_status expand_general(const lora::ExpandArgs& a, cudaStream_t st) {
  const int n_tot = a.slices.off[a.S] - a.slices.off[0];
  const int slots = lora::num_piece_slots(a.tok, a.nseg, lora::kGBM);
  const int chunks = (n_tot + lora::kGECols - 1) / lora::kGECols;
  if (chunks > 65535) return LORA_ERR_UNSUPPORTED;
  const size_t smem = sizeof(float) * lora::kGBM * a.S * a.r;
  if (smem > 200 * 1024) return LORA_ERR_UNSUPPORTED;
  dim3 grid(slots, chunks);
  lora::expand_general_kernel<E><<<grid, lora::kGECols, smem, st>>>(a);
  ++g_launches;
  g_last_path = LORA_PATH_GENERAL;
  return launch_status();
}

bool expand_tc_eligible(const lora::ExpandArgs& a) {
  if (!(aligned_to(a.in_r, 16) && (a.ld_in % 8) == 0 && (a.rs % 8) == 0 &&
        aligned_to(a.B, 16) && aligned_to(a.base, 16) && (a.ld_base % 8) == 0 && a.r <= 64))
    return false;
  for (int q = 0; q <= a.S; ++q)
    if (a.slices.off[q] % 8) return false;
  const int64_t n_tot = a.slices.off[a.S] - a.slices.off[0];
  return static_cast<int64_t>(a.L) * n_tot < (int64_t(1) << 31) && a.tok < (1 << 30);
}

template <class E>
lora_status expand_tc(const lora::ExpandArgs& a, lora_dtype dt, const Grouping& g,
                      const DeviceFacts& dev, cudaStream_t st) {
  lora::ExpandTcParams P;
  std::memset(&P, 0, sizeof(P));
  P.a = a;
  P.row_list = g.row_list;
  P.vseg_indptr = g.vseg_indptr;
  P.nvseg = g.vseg_indptr ? g.nvseg : a.nseg;
  P.rpad = a.r <= 16 ? 16 : (a.r <= 32 ? 32 : 64);
  P.sw_layout = P.rpad == 16 ? 6u : (P.rpad == 32 ? 4u : 2u);
  const CUtensorMapSwizzle swz = P.rpad == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                 : P.rpad == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_128B;
  P.rin_bytes = lora::kExBM * P.rpad * 2;
  P.btile_bytes = lora::kExBN * P.rpad * 2;
  int tiles = 0;
  for (int q = 0; q < a.S; ++q) {
    P.tile_prefix[q] = tiles;
    tiles += (a.slices.off[q + 1] - a.slices.off[q] + lora::kExBN - 1) / lora::kExBN;
  }
  P.tile_prefix[a.S] = tiles;
  for (int q = a.S + 1; q <= LORA_MAX_SLICES; ++q) P.tile_prefix[q] = tiles;
  if (tiles == 0) return LORA_OK;
  P.tiles_total = tiles;
  P.idesc = lora::make_idesc_f16(dt == LORA_BF16 ? 1 : 0, lora::kExBM, lora::kExBN);

  // shared memory: base ring, rank activations, B ring, row tables, barriers
  P.b_stages = LORA_EXPAND_B_STAGES;
  auto total = [&](int bs) {
    const size_t fixed = static_cast<size_t>(a.S) * P.rin_bytes +
                         static_cast<size_t>(P.b_stages) * P.btile_bytes + 1024 + 512 + 16;
    return ((static_cast<size_t>(bs) * lora::kExStageBytes + 1023) & ~size_t(1023)) + fixed +
           8 * (2 * P.b_stages + 5 + 2 * bs);
  };
  // two CTAs per SM when both accumulators fit twice in TMEM (512 columns) and
  // two base stages fit in half the shared memory, with a B ring of two if
  // three do not fit; otherwise one CTA per SM with a deeper base ring.  (The
  // grid is sized for two CTAs per SM either way: sized for one, the rank-64
  // gate_up expand measured 188 us against 140 us.)
  const int grid_ctas_per_sm =
      (LORA_EXPAND_CTAS_PER_SM >= 2 && lora::kExTmemCols <= 256) ? 2 : 1;
  int ctas_per_sm = grid_ctas_per_sm;
  if (ctas_per_sm == 2 && total(2) > 113 * 1024) {
    P.b_stages = 2;
    if (total(2) > 113 * 1024) {
      P.b_stages = LORA_EXPAND_B_STAGES;
      ctas_per_sm = 1;
    }
  }
  const size_t cap = (ctas_per_sm >= 2 ? 113 : 225) * 1024;
  P.base_stages = 2;
  while (P.base_stages < 7 && total(P.base_stages + 1) <= cap) ++P.base_stages;
  if (total(P.base_stages) > 225 * 1024) return LORA_ERR_UNSUPPORTED;
  size_t smem = total(P.base_stages);
  // keep the CTAs per SM within TMEM: 512 columns / kExTmemCols
  const size_t min_smem = lora::kExTmemCols > 256 ? 116 * 1024 : kTmemCtaMinSmem;
  if (smem < min_smem) smem = min_smem;

  const int64_t n_tot = a.slices.off[a.S] - a.slices.off[0];
  if (!encode_2d(&P.tmap_B, dt, a.B, a.r, static_cast<uint64_t>(a.L) * n_tot,
                 static_cast<uint64_t>(a.rs) * 2, P.rpad, lora::kExBN, swz))
    return LORA_ERR_CUDA;
  // the rank activations by TMA when a piece's rows are contiguous sorted rows
  P.rin_tma = g.row_list == nullptr ? 1 : 0;
  if (P.rin_tma &&
      !encode_3d(&P.tmap_R, dt, a.in_r, a.r, a.S, a.tok, static_cast<uint64_t>(a.rs) * 2,
                 static_cast<uint64_t>(a.ld_in) * 2, P.rpad, 1, lora::kExBM, swz))
    return LORA_ERR_CUDA;

  // Tiles per CTA: the split of the tiles into column groups that minimises
  // waves x (tiles per CTA + start-up) with every slot counted as a piece (the
  // start-up costs about two tiles' epilogues).  It keeps the grid within one
  // wave where the plain quotient would spill a few CTAs into a second (qkv at
  // tok 16384: 23 tiles per CTA gave three column groups and 408 CTAs for 296
  // places).
  const long slots = lora::num_piece_slots(a.tok, P.nvseg, lora::kExBM);
  const long resident = static_cast<long>(grid_ctas_per_sm) * dev.sms * LORA_EXPAND_WAVES;
  long tpc = tiles, best = -1;
  for (long t = 1; t <= tiles; ++t) {
    const long ncg_t = (tiles + t - 1) / t;
    const long waves = (slots * ncg_t + resident - 1) / resident;
    const long cost = waves * ((tiles + ncg_t - 1) / ncg_t + 2);
    if (best < 0 || cost < best) {
      best = cost;
      tpc = t;
    }
  }
  P.tiles_per_cta = static_cast<int>(tpc);
  const long ncg = (tiles + tpc - 1) / tpc;
  if (slots * ncg >= (1L << 31)) return LORA_ERR_UNSUPPORTED;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(slots * ncg));
  cfg.blockDim = dim3(lora::kExThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  LaunchAttrs attrs;
  attrs.after_grouping(g);
  attrs.apply(cfg);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, lora::expand_tc_kernel<E>, P);
  ++g_launches;
  g_last_path = LORA_PATH_TENSOR | (P.vseg_indptr ? LORA_PATH_GROUPED : 0);
  return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

// Element-aligned tensor-core expand (expand_unaligned_tc.cuh): any 2-byte
// alignment, leading dimension and slice layout, r <= 64.  *launched says
// whether it ran (else the CUDA-core kernel takes the call).
template <class E>
lora_status expand_unaligned_tc(const lora::ExpandArgs& a, lora_dtype dt, const Grouping& g,
                                const DeviceFacts& dev, cudaStream_t st, bool& launched) {
  launched = false;
  const int64_t n_tot = a.slices.off[a.S] - a.slices.off[0];
  if (a.r > 64 || static_cast<int64_t>(a.L) * n_tot >= (int64_t(1) << 31) || a.tok >= (1 << 30))
    return LORA_OK;
  lora::ExpandUnalignedParams P;
  std::memset(&P, 0, sizeof(P));
  P.a = a;
  P.row_list = g.row_list;
  P.vseg_indptr = g.vseg_indptr;
  P.nvseg = g.vseg_indptr ? g.nvseg : a.nseg;
  P.rpad = a.r <= 16 ? 16 : (a.r <= 32 ? 32 : 64);
  P.sw_layout = P.rpad == 16 ? 6u : (P.rpad == 32 ? 4u : 2u);
  P.rin_bytes = lora::kExBM * P.rpad * 2;
  P.btile_bytes = lora::kExBN * P.rpad * 2;
  int tiles = 0;
  for (int q = 0; q < a.S; ++q) {
    P.tile_prefix[q] = tiles;
    tiles += (a.slices.off[q + 1] - a.slices.off[q] + lora::kExBN - 1) / lora::kExBN;
  }
  for (int q = a.S; q <= LORA_MAX_SLICES; ++q) P.tile_prefix[q] = tiles;
  if (tiles == 0) {
    launched = true;
    return LORA_OK;
  }
  P.tiles_total = tiles;
  P.idesc = lora::make_idesc_f16(dt == LORA_BF16 ? 1 : 0, lora::kExBM, lora::kExBN);
  P.srow = static_cast<uint32_t>(16 * (P.rpad / 8 + 1));
  P.stage_bytes = static_cast<uint32_t>(round_up(
      lora::kEuRawBase + static_cast<int>(P.btile_bytes) + lora::kExBM * static_cast<int>(P.srow),
      1024));
  // rank activations, row tokens, two groups' row addresses, alignment slack
  const size_t fixed = static_cast<size_t>(a.S) * P.rin_bytes + 4 * lora::kExBM +
                       2 * sizeof(uintptr_t) * lora::kExBM + 1024 + 16;
  auto total = [&](int nb) {
    return static_cast<size_t>(nb) * P.stage_bytes + fixed + 8 * (3 * nb + 7);
  };
  // two CTAs per SM (TMEM: 2 x 256 columns) when two stages fit in half the
  // SM's shared memory, else one CTA with up to four stages
  const int ctas_per_sm = LORA_EU_CTAS_PER_SM >= 2 && total(2) <= 113 * 1024 ? 2 : 1;
  const size_t cap = ctas_per_sm == 2 ? 113 * 1024 : 225 * 1024;
  P.stages = 2;
  while (P.stages < 4 && total(P.stages + 1) <= cap) ++P.stages;
  // the rank activations of a piece are staged in the last stage's base area
  // (as many slices as fit) and the B staging areas of stages stages-1 .. 0;
  // stage 0's only when needed, since the first B tile then waits for them
  const int nfit = lora::kEuRawBase / (lora::kExBM * static_cast<int>(P.srow));
  if (total(P.stages) > cap || a.S > nfit + P.stages) return LORA_OK;
  P.rin_in_stage0 = a.S > nfit + P.stages - 1 ? 1 : 0;
  const size_t smem = std::max<size_t>(total(P.stages), kTmemCtaMinSmem);

  const long slots = lora::num_piece_slots(a.tok, P.nvseg, lora::kExBM);
  // Tiles per CTA: the split of the tiles into column groups that minimises
  // waves x (tiles per CTA + start-up), for the pieces expected (one per 128
  // rows plus half a piece per segment; slots beyond them find no piece and
  // leave at once).  The start-up (tables, rank rows, first tiles) costs about
  // two tiles' epilogues.
  const long est = (a.tok + lora::kExBM - 1) / lora::kExBM + P.nvseg / 2;
  const long resident = static_cast<long>(ctas_per_sm) * dev.sms;
  long tpc = tiles, best = -1;
  for (long t = 1; t <= tiles; ++t) {
    const long ncg_t = (tiles + t - 1) / t;
    const long waves = (std::max(est, 1L) * ncg_t + resident - 1) / resident;
    const long cost = waves * ((tiles + ncg_t - 1) / ncg_t + 2);
    if (best < 0 || cost < best) {
      best = cost;
      tpc = t;
    }
  }
  P.tiles_per_cta = static_cast<int>(tpc);
  const long ncg = (tiles + tpc - 1) / tpc;
  if (slots * ncg >= (1L << 31)) return LORA_OK;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(slots * ncg));
  cfg.blockDim = dim3(lora::kExThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  LaunchAttrs attrs;
  attrs.after_grouping(g);
  attrs.apply(cfg);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, lora::expand_unaligned_kernel<E>, P);
  ++g_launches;
  launched = true;
  g_last_path = LORA_PATH_TENSOR | (P.vseg_indptr ? LORA_PATH_GROUPED : 0);
  return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

// ------------------------------------------------------------------ fused shrink + expand

#ifndef LORA_FUSED_MAX_TOK
#define LORA_FUSED_MAX_TOK 512  // larger batches run the two kernels one after the other
#endif

// Launches the fused kernel when it applies; *launched says whether it did.
template <class E>
lora_status fused_tc(const lora::ShrinkArgs& sa, const lora::ExpandArgs& ea, lora_dtype dt,
                     const DeviceFacts& dev, cudaStream_t st, bool& launched) {
  launched = false;
  if (sa.tok > LORA_FUSED_MAX_TOK) return LORA_OK;
  lora::FusedTcParams P;
  std::memset(&P, 0, sizeof(P));
  P.s = sa;
  P.e = ea;
  P.npad = round_up(sa.S * sa.rs, 16);
  P.nkb = (sa.K + lora::kTcAtomK - 1) / lora::kTcAtomK;
  P.idesc_s = lora::make_idesc_f16(dt == LORA_BF16 ? 1 : 0, lora::kTcBM, P.npad);
  P.stage_bytes = lora::kTcBM * 128 + P.npad * 128;
  P.rpad = ea.r <= 16 ? 16 : (ea.r <= 32 ? 32 : 64);
  P.sw_layout = P.rpad == 16 ? 6u : (P.rpad == 32 ? 4u : 2u);
  const CUtensorMapSwizzle swz = P.rpad == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                 : P.rpad == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_128B;
  P.rin_bytes = lora::kExBM * P.rpad * 2;
  P.btile_bytes = lora::kExBN * P.rpad * 2;
  P.idesc_e = lora::make_idesc_f16(dt == LORA_BF16 ? 1 : 0, lora::kExBM, lora::kExBN);
  int tiles = 0;
  for (int q = 0; q < ea.S; ++q) {
    P.tile_prefix[q] = tiles;
    tiles += (ea.slices.off[q + 1] - ea.slices.off[q] + lora::kExBN - 1) / lora::kExBN;
  }
  for (int q = ea.S; q <= LORA_MAX_SLICES; ++q) P.tile_prefix[q] = tiles;
  P.tiles_total = tiles;
  // shared memory: shrink ring (also the split-K partial), rank activations,
  // base ring, B ring, tokens, barriers; one CTA per SM (the kernel holds all
  // 512 TMEM columns).  The deepest expand rings that leave room for a shrink
  // ring of at least two stages holding the partial; otherwise the pair runs
  // unfused.
  const size_t part_bytes = sizeof(float) * lora::kTcBM * (P.npad + 4);
  auto total = [&](int stages) {
    return static_cast<size_t>(stages) * P.stage_bytes +
           static_cast<size_t>(sa.S) * P.rin_bytes +
           static_cast<size_t>(P.base_stages) * lora::kExStageBytes +
           static_cast<size_t>(P.b_stages) * P.btile_bytes + 1024 + 512 +
           8 * (2 * stages + 1 + 2 * P.b_stages + 4 + 2 * 8) + 16;  // <= 8 expand stages
  };
  const int s_min = std::max<int>(2, static_cast<int>((part_bytes + P.stage_bytes - 1) /
                                                      P.stage_bytes));
  const int rings[4][2] = {{2, 6}, {2, LORA_EXPAND_B_STAGES}, {2, 2}, {1, 2}};  // {base, B}
  bool fits = false;
  for (int i = 0; i < 4 && !fits; ++i) {
    P.base_stages = rings[i][0];
    P.b_stages = rings[i][1];
    fits = s_min <= 6 && total(s_min) <= 227 * 1024;
  }
  if (!fits) return LORA_OK;
  P.stages = s_min;
  while (P.stages < 6 && total(P.stages + 1) <= 227 * 1024) ++P.stages;
  // after the shrink, its ring holds further expand stages (8 in all at most)
  P.xstages = std::min(8, P.base_stages + static_cast<int>(static_cast<size_t>(P.stages) *
                                                           P.stage_bytes / lora::kExStageBytes));
  // at least 120 KB: one CTA per SM
  const size_t smem = std::max<size_t>(total(P.stages), 120 * 1024);

  // cluster size: the largest of 16, 8, 4 CTAs for which every slot's cluster
  // (empty ones included: they leave at once, but only after being placed) is
  // resident at the same time and every CTA has at least one K block;
  // otherwise the pair runs unfused
  const long slots = lora::num_piece_slots(sa.tok, sa.nseg, lora::kTcBM);
  int cs = 0;
  for (int lg = 4; lg >= 2 && cs == 0; --lg) {
    const int c = 1 << lg;
    if (c <= dev.max_cluster && P.nkb >= c && slots <= dev.fused_clusters[lg]) cs = c;
  }
  if (cs == 0) return LORA_OK;
  P.csplit = cs;

  const int64_t n_tot = ea.slices.off[ea.S] - ea.slices.off[0];
  if (!encode_2d(&P.tmap_A, dt, sa.A, sa.K, static_cast<uint64_t>(sa.L) * sa.S * sa.rs,
                 static_cast<uint64_t>(sa.K) * 2, lora::kTcAtomK, P.npad,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&P.tmap_B, dt, ea.B, ea.r, static_cast<uint64_t>(ea.L) * n_tot,
                 static_cast<uint64_t>(ea.rs) * 2, P.rpad, lora::kExBN, swz))
    return LORA_ERR_CUDA;

  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(static_cast<unsigned>(slots * cs));
  cfg.blockDim = dim3(lora::kFuThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, lora::fused_tc_kernel<E>, P);
  ++g_launches;
  launched = true;
  g_last_path = LORA_PATH_TENSOR | LORA_PATH_FUSED | LORA_PATH_SPLITK;
  return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* lora_status_string(lora_status s) {
  switch (s) {
    case LORA_OK: return "ok";
    case LORA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case LORA_ERR_UNSUPPORTED: return "unsupported argument combination";
    case LORA_ERR_CUDA: return "CUDA error";
    case LORA_ERR_BAD_VALUES: return "tables hold invalid values";
  }
  return "unknown status";
}

uint64_t lora_launch_count(void) { return g_launches; }
void lora_reset_launch_count(void) { g_launches = 0; }
int lora_last_path(void) { return g_last_path; }

size_t lora_index64_workspace_size(int tok, int nseg) {
  if (tok < 0 || nseg < 0) return 0;
  return index64_bytes(tok, nseg);
}

size_t lora_workspace_size(int tok, int nseg, int L) {
  if (tok < 0 || nseg < 0 || L < 1) return 0;
  return workspace_ints(tok, nseg, L) * sizeof(int32_t);
}

size_t lora_validate_workspace_size(int tok) {
  if (tok < 0) return 0;
  return sizeof(uint32_t) * ((static_cast<size_t>(tok) + 31) / 32 + 1);
}

lora_status lora_device_error(int32_t* code, int clear) {
  if (!code) return LORA_ERR_INVALID_ARGUMENT;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, lora::g_lora_device_error, sizeof(int)) != cudaSuccess)
    return LORA_ERR_CUDA;
  *code = v;
  if (clear) {
    const int z = 0;
    if (cudaMemcpyToSymbol(lora::g_lora_device_error, &z, sizeof(int)) != cudaSuccess)
      return LORA_ERR_CUDA;
  }
  return LORA_OK;
}

lora_status lora_shrink(const void* x, int64_t ld_x, const void* A_stack,
                        const int32_t* seg_indptr, const int32_t* weight_indices,
                        const int32_t* permutation, void* out_r, int64_t ld_out, int tok,
                        int K, int S, int r, int rs, int nseg, int L, lora_dtype dtype,
                        void* workspace, size_t workspace_bytes, void* stream) {
  const lora_status cs = shrink_scalar_check(ld_x, ld_out, tok, K, S, r, rs, nseg, L, dtype,
                                             workspace, workspace_bytes);
  if (cs != LORA_OK) return cs;
  if (tok == 0 || nseg == 0) return LORA_OK;  // nothing to read or write
  if (!x || !A_stack || !seg_indptr || !weight_indices || !out_r)
    return LORA_ERR_INVALID_ARGUMENT;
  if (!aligned_to(x, 2) || !aligned_to(A_stack, 2) || !aligned_to(out_r, 2) ||
      !aligned_to(seg_indptr, 4) || !aligned_to(weight_indices, 4) ||
      (permutation && !aligned_to(permutation, 4)))
    return LORA_ERR_INVALID_ARGUMENT;

  lora::ShrinkArgs a{static_cast<const uint16_t*>(x), ld_x,
                     static_cast<const uint16_t*>(A_stack), seg_indptr, weight_indices,
                     permutation, static_cast<uint16_t*>(out_r), ld_out, tok, K, S, r, rs,
                     nseg, L};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const DeviceFacts* dev = device_facts();
  if (!dev) return LORA_ERR_CUDA;
  if (shrink_tc_eligible(a)) {
    Grouping g;
    const lora_status gs =
        maybe_group(seg_indptr, weight_indices, tok, nseg, L,
                    2ll * S * rs * K, workspace, workspace_bytes, st, g);
    if (gs != LORA_OK) return gs;
    return dtype == LORA_BF16 ? shrink_tc<lora::Bf16>(a, dtype, g, *dev, st)
                              : shrink_tc<lora::Fp16>(a, dtype, g, *dev, st);
  }
  return dtype == LORA_BF16 ? shrink_general<lora::Bf16>(a, st)
                            : shrink_general<lora::Fp16>(a, st);
}

lora_status lora_expand(const void* in_r, int64_t ld_in, const void* B_stack,
                        const int32_t* seg_indptr, const int32_t* weight_indices,
                        const int32_t* permutation, const int32_t* slice_offsets,
                        const float* scalings, void* base_out, int64_t ld_base, int tok, int S,
                        int r, int rs, int nseg, int L, lora_dtype dtype, void* workspace,
                        size_t workspace_bytes, void* stream) {
  lora::SliceTable tab;
  const lora_status cs = expand_scalar_check(ld_in, ld_base, tok, S, r, rs, nseg, L,
                                             slice_offsets, dtype, workspace, workspace_bytes,
                                             tab);
  if (cs != LORA_OK) return cs;
  if (tok == 0 || nseg == 0 || tab.off[S] == tab.off[0]) return LORA_OK;
  if (!in_r || !B_stack || !seg_indptr || !weight_indices || !scalings || !base_out)
    return LORA_ERR_INVALID_ARGUMENT;
  if (!aligned_to(in_r, 2) || !aligned_to(B_stack, 2) || !aligned_to(base_out, 2) ||
      !aligned_to(seg_indptr, 4) || !aligned_to(weight_indices, 4) ||
      !aligned_to(scalings, 4) || (permutation && !aligned_to(permutation, 4)))
    return LORA_ERR_INVALID_ARGUMENT;

  lora::ExpandArgs a{static_cast<const uint16_t*>(in_r), ld_in,
                     static_cast<const uint16_t*>(B_stack), seg_indptr, weight_indices,
                     permutation, scalings, static_cast<uint16_t*>(base_out), ld_base, tok, S,
                     r, rs, nseg, L, tab};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const DeviceFacts* dev = device_facts();
  if (!dev) return LORA_ERR_CUDA;
  if (expand_tc_eligible(a)) {
    Grouping g;
    const lora_status gs =
        maybe_group(seg_indptr, weight_indices, tok, nseg, L,
                    2ll * rs * (tab.off[S] - tab.off[0]), workspace, workspace_bytes, st, g);
    if (gs != LORA_OK) return gs;
    return dtype == LORA_BF16 ? expand_tc<lora::Bf16>(a, dtype, g, *dev, st)
                              : expand_tc<lora::Fp16>(a, dtype, g, *dev, st);
  }
  {
    Grouping g;
    const lora_status gs =
        maybe_group(seg_indptr, weight_indices, tok, nseg, L,
                    2ll * rs * (tab.off[S] - tab.off[0]), workspace, workspace_bytes, st, g);
    if (gs != LORA_OK) return gs;
    bool launched = false;
    const lora_status us = dtype == LORA_BF16
                               ? expand_unaligned_tc<lora::Bf16>(a, dtype, g, *dev, st, launched)
                               : expand_unaligned_tc<lora::Fp16>(a, dtype, g, *dev, st, launched);
    if (us != LORA_OK || launched) return us;
  }
  return dtype == LORA_BF16 ? expand_general<lora::Bf16>(a, st)
                            : expand_general<lora::Fp16>(a, st);
}

lora_status lora_validate(const int32_t* seg_indptr, const int32_t* weight_indices,
                          const int32_t* permutation, const int32_t* slice_offsets, int tok,
                          int nseg, int L, int S, int64_t ld_base, int32_t* d_result,
                          void* workspace, size_t workspace_bytes, void* stream) {
  if (tok < 0 || nseg < 0 || L < 1 || S < 1 || !seg_indptr || !d_result ||
      (nseg > 0 && !weight_indices))
    return LORA_ERR_INVALID_ARGUMENT;
  if (permutation && (!workspace || workspace_bytes < lora_validate_workspace_size(tok)))
    return LORA_ERR_INVALID_ARGUMENT;
  int host_bad = 0;
  if (slice_offsets) {
    if (S > LORA_MAX_SLICES) return LORA_ERR_UNSUPPORTED;
    for (int q = 0; q <= S; ++q) {
      if (slice_offsets[q] < 0 || slice_offsets[q] > ld_base) host_bad |= LORA_BAD_SLICES;
      if (q > 0 && slice_offsets[q] < slice_offsets[q - 1]) host_bad |= LORA_BAD_SLICES;
    }
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The result word starts as the host-side findings; the kernel ORs in the rest.
  lora::set_word_kernel<<<1, 1, 0, st>>>(d_result, host_bad);
  ++g_launches;
  if (permutation &&
      cudaMemsetAsync(workspace, 0, lora_validate_workspace_size(tok), st) != cudaSuccess)
    return LORA_ERR_CUDA;
  const int work = tok > nseg + 1 ? tok : nseg + 1;
  int blocks = (work + 255) / 256;
  if (blocks > 1184) blocks = 1184;
  if (blocks < 1) blocks = 1;
  lora::validate_kernel<<<blocks, 256, 0, st>>>(seg_indptr, weight_indices, permutation, tok,
                                                nseg, L, static_cast<unsigned*>(workspace),
                                                d_result);
  ++g_launches;
  return launch_status();
}

}  // extern "C"

// ------------------------------------------------------------------ identity-permutation ops
//
// The other LoRA ops of the sgl-kernel-xpu page's file table (SGEMMLoraAFwd,
// SGEMMLoraBFwd, QKVLoraBFwd, GateUpLoraBFwd, EmbeddingLoraAFwd) work on
// segments in token order.  The first four are the shrink / expand with the
// identity permutation and a fixed slice layout, so they forward to the same
// kernels; the embedding one has a gather kernel of its own.

extern "C" lora_status lora_sgemm_a(const void* x, int64_t ld_x, const void* A_stack,
                                    const int32_t* seg_indptr, const int32_t* weight_indices,
                                    void* out, int64_t ld_out, int tok, int K, int S, int r,
                                    int rs, int nseg, int L, lora_dtype dtype, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  return lora_shrink(x, ld_x, A_stack, seg_indptr, weight_indices, nullptr, out, ld_out, tok, K,
                     S, r, rs, nseg, L, dtype, workspace, workspace_bytes, stream);
}

extern "C" lora_status lora_sgemm_b(const void* in_r, int64_t ld_in, const void* B_stack,
                                    const int32_t* seg_indptr, const int32_t* weight_indices,
                                    const float* scalings, void* base_out, int64_t ld_base,
                                    int tok, int N, int r, int rs, int nseg, int L,
                                    lora_dtype dtype, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  if (N < 0) return LORA_ERR_INVALID_ARGUMENT;
  const int32_t off[2] = {0, N};
  return lora_expand(in_r, ld_in, B_stack, seg_indptr, weight_indices, nullptr, off, scalings,
                     base_out, ld_base, tok, 1, r, rs, nseg, L, dtype, workspace,
                     workspace_bytes, stream);
}

extern "C" lora_status lora_qkv_b(const void* in_r, int64_t ld_in, const void* B_stack,
                                  const int32_t* seg_indptr, const int32_t* weight_indices,
                                  const int32_t* qkv_offsets, const float* scalings,
                                  void* base_out, int64_t ld_base, int tok, int r, int rs,
                                  int nseg, int L, lora_dtype dtype, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  return lora_expand(in_r, ld_in, B_stack, seg_indptr, weight_indices, nullptr, qkv_offsets,
                     scalings, base_out, ld_base, tok, 3, r, rs, nseg, L, dtype, workspace,
                     workspace_bytes, stream);
}

extern "C" lora_status lora_gate_up_b(const void* in_r, int64_t ld_in, const void* B_stack,
                                      const int32_t* seg_indptr, const int32_t* weight_indices,
                                      const float* scalings, void* base_out, int64_t ld_base,
                                      int tok, int N, int r, int rs, int nseg, int L,
                                      lora_dtype dtype, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  if (N < 0 || N > (1 << 30)) return LORA_ERR_INVALID_ARGUMENT;
  const int32_t off[3] = {0, N, 2 * N};
  return lora_expand(in_r, ld_in, B_stack, seg_indptr, weight_indices, nullptr, off, scalings,
                     base_out, ld_base, tok, 2, r, rs, nseg, L, dtype, workspace,
                     workspace_bytes, stream);
}

extern "C" lora_status lora_embedding_a(const int32_t* ids, const void* A_emb,
                                        const int32_t* seg_indptr,
                                        const int32_t* weight_indices, void* out,
                                        int64_t ld_out, int tok, int V, int r, int rs, int nseg,
                                        int L, lora_dtype dtype, void* stream) {
  if (dtype != LORA_BF16 && dtype != LORA_FP16) return LORA_ERR_UNSUPPORTED;
  if (tok < 0 || nseg < 0 || V < 1 || r < 1 || rs < r || L < 1 || ld_out < rs)
    return LORA_ERR_INVALID_ARGUMENT;
  if (tok == 0 || nseg == 0) return LORA_OK;
  if (!ids || !A_emb || !seg_indptr || !weight_indices || !out) return LORA_ERR_INVALID_ARGUMENT;
  if (!aligned_to(ids, 4) || !aligned_to(A_emb, 2) || !aligned_to(out, 2) ||
      !aligned_to(seg_indptr, 4) || !aligned_to(weight_indices, 4))
    return LORA_ERR_INVALID_ARGUMENT;
  const long slots = lora::num_piece_slots(tok, nseg, lora::kEmbBM);
  lora::embedding_a_kernel<<<static_cast<unsigned>(slots), 128, 0,
                             static_cast<cudaStream_t>(stream)>>>(
      ids, static_cast<const uint16_t*>(A_emb), seg_indptr, weight_indices,
      static_cast<uint16_t*>(out), ld_out, tok, V, r, rs, nseg, L);
  ++g_launches;
  g_last_path = LORA_PATH_GENERAL;
  return launch_status();
}

// ------------------------------------------------------------------ scratch-free shrink
//
// lora_shrink_static_scratch serves callers that are handed only input and
// output buffers and have no way to obtain device memory of their own.  Its
// scratch (the row lists of the adapter-grouped schedule) lives in the
// file-scope array below instead of a caller workspace.  Every GPU that loads
// the library keeps this array until the process exits.

static __device__ __align__(256) int32_t
    g_lora_static_scratch[LORA_STATIC_SCRATCH_BYTES / sizeof(int32_t)];

namespace {

struct StaticScratchAddr {
  std::atomic<int> ready{0};
  void* ptr = nullptr;
};
StaticScratchAddr g_static_scratch_addr[kMaxDevices];
std::mutex g_static_scratch_mu;

// Device address of the static scratch on the current device.  The host-side
// name of the array is only a stand-in, so the address is looked up once per
// device, with that device current, and cached.  Null on failure.
void* static_scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  StaticScratchAddr& s = g_static_scratch_addr[dev];
  if (s.ready.load(std::memory_order_acquire)) return s.ptr;
  std::lock_guard<std::mutex> lk(g_static_scratch_mu);
  if (!s.ready.load(std::memory_order_relaxed)) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lora_static_scratch) != cudaSuccess || p == nullptr)
      return nullptr;
    s.ptr = p;
    s.ready.store(1, std::memory_order_release);
  }
  return s.ptr;
}

}  // namespace

extern "C" lora_status lora_shrink_static_scratch(
    const void* x, int64_t ld_x, const void* A_stack, const int32_t* seg_indptr,
    const int32_t* weight_indices, const int32_t* permutation, void* out_r, int64_t ld_out,
    int tok, int K, int S, int r, int rs, int nseg, int L, lora_dtype dtype, void* stream) {
  // Only the adapter-grouping pass uses scratch, and it runs only with more
  // segments than adapters and enough weight reads to save; any other call
  // needs none, so it has no size limit.
  if (!grouping_pays(nseg, L, 2ll * S * rs * K))
    return lora_shrink(x, ld_x, A_stack, seg_indptr, weight_indices, permutation, out_r,
                       ld_out, tok, K, S, r, rs, nseg, L, dtype, nullptr, 0, stream);
  // the grouping pass writes every word of the scratch it later reads, so
  // nothing has to be cleared between calls
  if (lora_workspace_size(tok, nseg, L) > LORA_STATIC_SCRATCH_BYTES) return LORA_ERR_UNSUPPORTED;
  void* ws = static_scratch_on_current_device();
  if (ws == nullptr) return LORA_ERR_CUDA;
  return lora_shrink(x, ld_x, A_stack, seg_indptr, weight_indices, permutation, out_r, ld_out,
                     tok, K, S, r, rs, nseg, L, dtype, ws, LORA_STATIC_SCRATCH_BYTES, stream);
}

// ------------------------------------------------------------------ int64 index tables

extern "C" lora_status lora_shrink_i64(const void* x, int64_t ld_x, const void* A_stack,
                                       const int64_t* seg_indptr,
                                       const int64_t* weight_indices,
                                       const int64_t* permutation, void* out_r, int64_t ld_out,
                                       int tok, int K, int S, int r, int rs, int nseg, int L,
                                       lora_dtype dtype, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  const lora_status cs = shrink_scalar_check(ld_x, ld_out, tok, K, S, r, rs, nseg, L, dtype,
                                             workspace, workspace_bytes);
  if (cs != LORA_OK) return cs;
  if (tok == 0 || nseg == 0) return LORA_OK;
  // every argument error is reported before the narrowing is enqueued
  if (!x || !A_stack || !out_r || !aligned_to(x, 2) || !aligned_to(A_stack, 2) ||
      !aligned_to(out_r, 2))
    return LORA_ERR_INVALID_ARGUMENT;
  if (!seg_indptr || !weight_indices || !aligned_to(seg_indptr, 8) ||
      !aligned_to(weight_indices, 8) || (permutation && !aligned_to(permutation, 8)))
    return LORA_ERR_INVALID_ARGUMENT;
  const size_t need = index64_bytes(tok, nseg);
  if (!workspace || !aligned_to(workspace, 16) || workspace_bytes < need)
    return LORA_ERR_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* w = static_cast<int32_t*>(workspace);
  const lora_status ns = narrow_tables(seg_indptr, weight_indices, permutation, tok, nseg, w, st);
  if (ns != LORA_OK) return ns;
  const int32_t* seg32 = w;
  const int32_t* wid32 = seg32 + a16(static_cast<size_t>(nseg) + 1);
  const int32_t* perm32 = permutation ? wid32 + a16(static_cast<size_t>(nseg)) : nullptr;
  return lora_shrink(x, ld_x, A_stack, seg32, wid32, perm32, out_r, ld_out, tok, K, S, r, rs,
                     nseg, L, dtype, static_cast<uint8_t*>(workspace) + need,
                     workspace_bytes - need, stream);
}

extern "C" lora_status lora_expand_i64(const void* in_r, int64_t ld_in, const void* B_stack,
                                       const int64_t* seg_indptr,
                                       const int64_t* weight_indices,
                                       const int64_t* permutation, const int32_t* slice_offsets,
                                       const float* scalings, void* base_out, int64_t ld_base,
                                       int tok, int S, int r, int rs, int nseg, int L,
                                       lora_dtype dtype, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  lora::SliceTable tab;
  const lora_status cs = expand_scalar_check(ld_in, ld_base, tok, S, r, rs, nseg, L,
                                             slice_offsets, dtype, workspace, workspace_bytes,
                                             tab);
  if (cs != LORA_OK) return cs;
  if (tok == 0 || nseg == 0 || tab.off[S] == tab.off[0]) return LORA_OK;
  // every argument error is reported before the narrowing is enqueued
  if (!in_r || !B_stack || !scalings || !base_out || !aligned_to(in_r, 2) ||
      !aligned_to(B_stack, 2) || !aligned_to(scalings, 4) || !aligned_to(base_out, 2))
    return LORA_ERR_INVALID_ARGUMENT;
  if (!seg_indptr || !weight_indices || !aligned_to(seg_indptr, 8) ||
      !aligned_to(weight_indices, 8) || (permutation && !aligned_to(permutation, 8)))
    return LORA_ERR_INVALID_ARGUMENT;
  const size_t need = index64_bytes(tok, nseg);
  if (!workspace || !aligned_to(workspace, 16) || workspace_bytes < need)
    return LORA_ERR_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* w = static_cast<int32_t*>(workspace);
  const lora_status ns = narrow_tables(seg_indptr, weight_indices, permutation, tok, nseg, w, st);
  if (ns != LORA_OK) return ns;
  const int32_t* seg32 = w;
  const int32_t* wid32 = seg32 + a16(static_cast<size_t>(nseg) + 1);
  const int32_t* perm32 = permutation ? wid32 + a16(static_cast<size_t>(nseg)) : nullptr;
  return lora_expand(in_r, ld_in, B_stack, seg32, wid32, perm32, slice_offsets, scalings,
                     base_out, ld_base, tok, S, r, rs, nseg, L, dtype,
                     static_cast<uint8_t*>(workspace) + need, workspace_bytes - need, stream);
}

// ------------------------------------------------------------------ fused pair

extern "C" lora_status lora_shrink_expand(
    const void* x, int64_t ld_x, const void* A_stack, const void* B_stack,
    const int32_t* seg_indptr, const int32_t* weight_indices, const int32_t* permutation,
    const int32_t* slice_offsets, const float* scalings, void* out_r, int64_t ld_out,
    void* base_out, int64_t ld_base, int tok, int K, int S, int r, int rs, int nseg, int L,
    lora_dtype dtype, void* workspace, size_t workspace_bytes, void* stream) {
  const lora_status cs = shrink_scalar_check(ld_x, ld_out, tok, K, S, r, rs, nseg, L, dtype,
                                             workspace, workspace_bytes);
  if (cs != LORA_OK) return cs;
  lora::SliceTable tab;
  const lora_status ce = expand_scalar_check(ld_out, ld_base, tok, S, r, rs, nseg, L,
                                             slice_offsets, dtype, workspace, workspace_bytes,
                                             tab);
  if (ce != LORA_OK) return ce;
  if (tok == 0 || nseg == 0) return LORA_OK;
  if (!x || !A_stack || !B_stack || !seg_indptr || !weight_indices || !scalings || !out_r ||
      !base_out)
    return LORA_ERR_INVALID_ARGUMENT;
  if (!aligned_to(x, 2) || !aligned_to(A_stack, 2) || !aligned_to(B_stack, 2) ||
      !aligned_to(out_r, 2) || !aligned_to(base_out, 2) || !aligned_to(seg_indptr, 4) ||
      !aligned_to(weight_indices, 4) || !aligned_to(scalings, 4) ||
      (permutation && !aligned_to(permutation, 4)))
    return LORA_ERR_INVALID_ARGUMENT;

  const lora::ShrinkArgs sa{static_cast<const uint16_t*>(x), ld_x,
                            static_cast<const uint16_t*>(A_stack), seg_indptr, weight_indices,
                            permutation, static_cast<uint16_t*>(out_r), ld_out, tok, K, S, r,
                            rs, nseg, L};
  const lora::ExpandArgs ea{static_cast<const uint16_t*>(out_r), ld_out,
                            static_cast<const uint16_t*>(B_stack), seg_indptr, weight_indices,
                            permutation, scalings, static_cast<uint16_t*>(base_out), ld_base,
                            tok, S, r, rs, nseg, L, tab};
  const DeviceFacts* dev = device_facts();
  if (!dev) return LORA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (shrink_tc_eligible(sa) && shrink_tc_aligned(sa) && expand_tc_eligible(ea) &&
      tab.off[S] > tab.off[0]) {
    bool launched = false;
    const lora_status fs = dtype == LORA_BF16
                               ? fused_tc<lora::Bf16>(sa, ea, dtype, *dev, st, launched)
                               : fused_tc<lora::Fp16>(sa, ea, dtype, *dev, st, launched);
    if (fs != LORA_OK || launched) return fs;
  }
  // the composition: the shrink's rounded output is the expand's input
  const lora_status s1 = lora_shrink(x, ld_x, A_stack, seg_indptr, weight_indices, permutation,
                                     out_r, ld_out, tok, K, S, r, rs, nseg, L, dtype, workspace,
                                     workspace_bytes, stream);
  if (s1 != LORA_OK) return s1;
  const int path = g_last_path;
  const lora_status s2 = lora_expand(out_r, ld_out, B_stack, seg_indptr, weight_indices,
                                     permutation, slice_offsets, scalings, base_out, ld_base,
                                     tok, S, r, rs, nseg, L, dtype, workspace, workspace_bytes,
                                     stream);
  g_last_path |= path;
  return s2;
}

// ------------------------------------------------------------------ base projection + expand

namespace {

template <class E>
lora_status base_expand_tc(const lora::BaseExpandArgs& a, const void* W, int64_t ld_w,
                           const void* B_stack, lora_dtype dt, cudaStream_t st) {
  lora::BaseExpandTcParams P;
  std::memset(&P, 0, sizeof(P));
  P.a = a;
  P.rpad = a.r <= 16 ? 16 : (a.r <= 32 ? 32 : 64);
  P.sw_layout = P.rpad == 16 ? 6u : (P.rpad == 32 ? 4u : 2u);
  const CUtensorMapSwizzle swz = P.rpad == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                 : P.rpad == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_128B;
  P.rin_bytes = lora::kTcBM * P.rpad * 2;
  P.btile_bytes = lora::kBeBN * P.rpad * 2;
  P.idesc = lora::make_idesc_f16(dt == LORA_BF16 ? 1 : 0, lora::kTcBM, lora::kBeBN);
  P.nkb = (a.K + lora::kTcAtomK - 1) / lora::kTcAtomK;
  int tiles = 0;
  for (int q = 0; q < a.S; ++q) {
    P.tile_prefix[q] = tiles;
    tiles += (a.slices.off[q + 1] - a.slices.off[q] + lora::kBeBN - 1) / lora::kBeBN;
  }
  for (int q = a.S; q <= LORA_MAX_SLICES; ++q) P.tile_prefix[q] = tiles;
  if (tiles == 0) return LORA_OK;
  P.tiles_total = tiles;

  // K ring of 32 KB stages; two CTAs per SM when three stages fit in 113 KB
  constexpr size_t kStage = lora::kTcBM * 128 + lora::kBeBN * 128;
  auto total = [&](int stages) {
    return static_cast<size_t>(stages) * kStage + P.rin_bytes + P.btile_bytes + 1024 + 512 +
           8 * (2 * stages + 3) + 16;
  };
  const bool two = LORA_BASE_EXPAND_CTAS_PER_SM >= 2 && total(3) <= 113 * 1024;
  const size_t cap = (two ? 113 : 225) * 1024;
  P.stages = 2;
  while (P.stages < 6 && total(P.stages + 1) <= cap) ++P.stages;
  if (total(P.stages) > 225 * 1024) return LORA_ERR_UNSUPPORTED;
  // never more than two CTAs (2 x 256 TMEM columns) on an SM
  const size_t smem = std::max<size_t>(total(P.stages), kTmemCtaMinSmem);

  const int64_t n_tot = a.slices.off[a.S] - a.slices.off[0];
  if (!encode_2d(&P.tmap_W, dt, W, a.K, static_cast<uint64_t>(n_tot),
                 static_cast<uint64_t>(ld_w) * 2, lora::kTcAtomK, lora::kBeBN,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&P.tmap_B, dt, B_stack, a.r, static_cast<uint64_t>(a.L) * n_tot,
                 static_cast<uint64_t>(a.rs) * 2, P.rpad, lora::kBeBN, swz))
    return LORA_ERR_CUDA;

  const long slots = lora::num_piece_slots(a.tok, a.nseg, lora::kTcBM);
  if (slots * tiles >= (1L << 31)) return LORA_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(slots * tiles));
  cfg.blockDim = dim3(lora::kBeThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, lora::base_expand_tc_kernel<E>, P);
  ++g_launches;
  g_last_path = LORA_PATH_TENSOR | LORA_PATH_FUSED;
  return e == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

}  // namespace

extern "C" lora_status lora_base_expand(
    const void* x, int64_t ld_x, const void* W, int64_t ld_w, const void* in_r, int64_t ld_in,
    const void* B_stack, const int32_t* seg_indptr, const int32_t* weight_indices,
    const int32_t* permutation, const int32_t* slice_offsets, const float* scalings, void* out,
    int64_t ld_out, int tok, int K, int S, int r, int rs, int nseg, int L, lora_dtype dtype,
    void* stream) {
  if (dtype != LORA_BF16 && dtype != LORA_FP16) return LORA_ERR_UNSUPPORTED;
  if (tok < 0 || nseg < 0 || K < 1 || S < 1 || r < 1 || rs < r || L < 1)
    return LORA_ERR_INVALID_ARGUMENT;
  if (S > LORA_MAX_SLICES) return LORA_ERR_UNSUPPORTED;
  if (!slice_offsets) return LORA_ERR_INVALID_ARGUMENT;
  if (ld_x < K || ld_w < K || ld_in < static_cast<int64_t>(S) * rs)
    return LORA_ERR_INVALID_ARGUMENT;
  lora::SliceTable tab{};
  tab.S = S;
  for (int q = 0; q <= S; ++q) {
    tab.off[q] = slice_offsets[q];
    if (slice_offsets[q] < 0 || slice_offsets[q] > ld_out) return LORA_ERR_INVALID_ARGUMENT;
    if (q > 0 && slice_offsets[q] < slice_offsets[q - 1]) return LORA_ERR_INVALID_ARGUMENT;
  }
  if (tok == 0 || nseg == 0 || tab.off[S] == tab.off[0]) return LORA_OK;
  if (!x || !W || !in_r || !B_stack || !seg_indptr || !weight_indices || !scalings || !out)
    return LORA_ERR_INVALID_ARGUMENT;
  if (!aligned_to(seg_indptr, 4) || !aligned_to(weight_indices, 4) ||
      !aligned_to(scalings, 4) || (permutation && !aligned_to(permutation, 4)))
    return LORA_ERR_INVALID_ARGUMENT;
  // tensor-core layout: 16-byte rows and slice starts (no element-aligned path)
  if (!aligned_to(x, 16) || !aligned_to(W, 16) || !aligned_to(in_r, 16) ||
      !aligned_to(B_stack, 16) || !aligned_to(out, 16) || (ld_x % 8) || (ld_w % 8) ||
      (ld_in % 8) || (ld_out % 8) || (K % 8) || (rs % 8) || r > 64)
    return LORA_ERR_UNSUPPORTED;
  for (int q = 0; q <= S; ++q)
    if (tab.off[q] % 8) return LORA_ERR_UNSUPPORTED;
  const int64_t n_tot = tab.off[S] - tab.off[0];
  if (static_cast<int64_t>(L) * n_tot >= (int64_t(1) << 31) || tok >= (1 << 30))
    return LORA_ERR_UNSUPPORTED;

  const lora::BaseExpandArgs a{static_cast<const uint16_t*>(x), ld_x,
                               static_cast<const uint16_t*>(in_r), ld_in, seg_indptr,
                               weight_indices, permutation, scalings,
                               static_cast<uint16_t*>(out), ld_out, tok, K, S, r, rs, nseg, L,
                               tab};
  const DeviceFacts* dev = device_facts();
  if (!dev) return LORA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dtype == LORA_BF16 ? base_expand_tc<lora::Bf16>(a, W, ld_w, B_stack, dtype, st)
                            : base_expand_tc<lora::Fp16>(a, W, ld_w, B_stack, dtype, st);
}
