// C ABI of the In-Place TTT fast-weight MLP forward: validation, workspace
// layout, tensor-map construction and kernel dispatch.  Every step of the
// computation runs in the kernels of simt.cuh and tc_gemm.cuh; this file
// only launches them.
#include <math.h>
#include <stdio.h>

#include <algorithm>
#include <atomic>
#include <type_traits>
#include <initializer_list>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "simt.cuh"
#include "tc_gemm.cuh"
#include "tc_recur.cuh"
#include "tc_tconv.cuh"

#include <nvtx3/nvToolsExt.h>

using namespace ittt;

namespace {

constexpr int kMaxDevices = 64;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::atomic<unsigned long long> g_wait_ns{4000000000ull};

// Bytes of the problem's tensors (element size of the problem's dtype).
struct Sizes {
  size_t es, BTd, BTf, df, dd, dk, Bdf32, Tx;
  explicit Sizes(const ittt_problem* p) {
    es = p->dtype == ITTT_BF16 ? 2 : 4;
    const size_t B = size_t(p->B), T = size_t(p->T), d = size_t(p->d), f = size_t(p->f);
    Tx = T + ((p->flags & ITTT_FLAG_X0_LOOKAHEAD) ? size_t(p->k - 1) : 0);
    BTd = B * T * d * es;
    BTf = B * T * f * es;
    df = d * f * es;
    dd = d * d * es;
    dk = d * size_t(p->k) * es;
    Bdf32 = B * d * f * 4;
  }
};

// ---------------------------------------------------------- buffer checks

// ittt_set_checks level: 1 = every compute entry point verifies its device
// buffers against their allocations before it launches.
std::atomic<int> g_checks{0};

typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(ptr);
  });
  return fn;
}

struct Buf {
  const void* ptr;
  size_t bytes;
};

// [ptr, ptr + bytes) inside one device allocation known to the driver.
bool buffer_in_allocation(AddressRangeFn range, const void* ptr, size_t bytes) {
  CUdeviceptr base = 0;
  size_t size = 0;
  const CUdeviceptr q = reinterpret_cast<CUdeviceptr>(ptr);
  if (range(&base, &size, q) != CUDA_SUCCESS) return false;
  return q >= base && bytes <= size && q - base <= size - bytes;
}

// With checks on: every non-null buffer must lie inside one device allocation
// from its start to start + bytes (ITTT_ERR_INVALID_ARG otherwise, before any
// launch).  Buffers the driver does not know (e.g. host memory) fail too.
ittt_status check_buffers(std::initializer_list<Buf> bufs) {
  if (g_checks.load(std::memory_order_relaxed) == 0) return ITTT_OK;
  AddressRangeFn range = address_range_fn();
  if (!range) return ITTT_ERR_CUDA;
  for (const Buf& b : bufs) {
    if (!b.ptr || b.bytes == 0) continue;
    if (!buffer_in_allocation(range, b.ptr, b.bytes)) return ITTT_ERR_INVALID_ARG;
  }
  return ITTT_OK;
}

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [outer, inner] matrix whose rows are
// row_elems elements apart; 128-byte swizzle; out-of-range boxes read zeros.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t row_elems,
              uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_elems * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per-device values cached on first use; atomics, as any host thread may call
// the library (a race only repeats an idempotent query).
int num_sms() {
  static std::atomic<int> cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline ittt_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? ITTT_OK : ITTT_ERR_CUDA;
}

inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

// 3-D tensor map over a row-major [outer2, outer1, inner] array of 2- or
// 4-byte elements, for TMA stores (128-byte swizzle; nothing is written
// outside the array).
bool make_map_3d(CUtensorMap* m, const void* ptr, bool f32, uint64_t inner, uint64_t outer1,
                 uint64_t outer2, uint32_t box_inner, uint32_t box_outer1) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const uint64_t es = f32 ? 4 : 2;
  const cuuint64_t dims[3] = {inner, outer1, outer2};
  const cuuint64_t strides[2] = {inner * es, inner * outer1 * es};
  const cuuint32_t box[3] = {box_inner, box_outer1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// MN-major operand (rows of `inner` contiguous values, `outer` rows, leading
// dimension ld) viewed as [inner/64 blocks][outer rows][64 values]: one box of
// 64 rows x `blocks` blocks lands in shared memory as `blocks` 64 x 64 tiles
// 8 KB apart, the image of `blocks` 2-D boxes.  inner must be a multiple of 64.
bool make_map_mn3(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld,
                  uint32_t blocks) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || inner % 64 != 0) return false;
  const cuuint64_t dims[3] = {64, outer, inner / 64};
  const cuuint64_t strides[2] = {ld * 2, 128};
  const cuuint32_t box[3] = {64, 64, blocks};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scan (tensor-core pairs, d and f multiples of 64): 1 = Vhat and Z tiles are
// loaded as one 3-D box each per k-block (two TMA instructions instead of four;
// measured on B200: scan 0.413 -> 0.403 ms at qwen3-4b widths, 8.75 -> 8.57 ms
// at T = 131072, C = 256).
#ifndef ITTT_SCAN_MN3D
#define ITTT_SCAN_MN3D 1
#endif

// 1 = the prefix forward computes chunks 0 and 1 with the dual-form kernels on
// the caller's stream while the scan and the apply of the other chunks run on
// a higher-priority side stream (the dual kernels fill the SMs that the scan's
// last, partial round leaves idle); 0 = one stream, apply of every chunk.
#ifndef ITTT_TAIL_DUAL
#define ITTT_TAIL_DUAL 1
#endif

// 1 = the prefix forward runs the fused scan and the apply of every chunk in
// one persistent launch (tc_recur_kernel: one work queue, readiness flags per
// d-tile and chunk); 0 = two launches (with ITTT_TAIL_DUAL as set), which
// measured faster on B200 (qwen3-4b: forward 1.284 vs 1.358 ms; the one-launch
// kernel's apply units run about a quarter slower than the apply kernel's).
// ittt_chunk_recurrence always runs the one-launch kernel.
#ifndef ITTT_FUSED_RECUR
#define ITTT_FUSED_RECUR 0
#endif
#ifndef ITTT_STAGES_RECUR
#define ITTT_STAGES_RECUR 6
#endif
// 1 = the one-launch recurrence also computes Vhat = Y W_target (target units
// ahead of the scan in its work queue; not with clipping, which rescales
// Vhat between the target and the recurrence); 0 = target GEMM launch first.
#ifndef ITTT_RECUR_TARGET
#define ITTT_RECUR_TARGET 0
#endif

// One high-priority side stream and two events per host thread and device,
// created on first use and kept for the life of the thread; `low` is a second
// side stream at the lowest priority with its own two events.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  cudaStream_t low = nullptr;
  cudaEvent_t low_fork = nullptr, low_join = nullptr;
};
thread_local SideStream g_side[kMaxDevices];

ittt_status side_stream(SideStream** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ITTT_ERR_CUDA;
  SideStream& ss = g_side[dev];
  if (!ss.stream || !ss.fork || !ss.join) {
    int least = 0, greatest = 0;
    SideStream fresh;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&fresh.stream, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaEventCreateWithFlags(&fresh.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&fresh.join, cudaEventDisableTiming) != cudaSuccess ||
        cudaStreamCreateWithPriority(&fresh.low, cudaStreamNonBlocking, least) != cudaSuccess ||
        cudaEventCreateWithFlags(&fresh.low_fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&fresh.low_join, cudaEventDisableTiming) != cudaSuccess) {
      // keep nothing half made: the next call tries again from scratch
      if (fresh.low_join) cudaEventDestroy(fresh.low_join);
      if (fresh.low_fork) cudaEventDestroy(fresh.low_fork);
      if (fresh.low) cudaStreamDestroy(fresh.low);
      if (fresh.join) cudaEventDestroy(fresh.join);
      if (fresh.fork) cudaEventDestroy(fresh.fork);
      if (fresh.stream) cudaStreamDestroy(fresh.stream);
      return ITTT_ERR_CUDA;
    }
    ss = fresh;
  }
  *out = &ss;
  return ITTT_OK;
}

// Orders the caller's stream after the side stream's work on every return
// path of a forked section: an error after the fork still makes the caller's
// stream wait for what was launched there (it writes the caller's buffers).
// Normal use: record() after the side stream's launches, wait() at the end.
struct SideJoin {
  SideStream* ss;
  cudaStream_t st;
  bool recorded = false, waited = false;
  SideJoin(SideStream* side, cudaStream_t caller) : ss(side), st(caller) {}
  SideJoin(const SideJoin&) = delete;
  SideJoin& operator=(const SideJoin&) = delete;
  ittt_status record() {
    recorded = true;
    return cudaEventRecord(ss->join, ss->stream) == cudaSuccess ? ITTT_OK : ITTT_ERR_CUDA;
  }
  ittt_status wait() {
    waited = true;
    return cudaStreamWaitEvent(st, ss->join, 0) == cudaSuccess ? ITTT_OK : ITTT_ERR_CUDA;
  }
  ~SideJoin() {
    if (waited) return;
    if (!recorded) cudaEventRecord(ss->join, ss->stream);
    cudaStreamWaitEvent(st, ss->join, 0);
  }
};

// 1 = the forward runs the look-ahead conv on a low-priority side stream
// beside the gate/up GEMM (which it does not depend on): its CTAs fill the
// threads and registers the persistent GEMM leaves free on each SM, and the
// target GEMM waits for both.
#ifndef ITTT_CONV_SIDE
#define ITTT_CONV_SIDE 1
#endif

// With ITTT_CONV_SIDE: 1 = the target GEMM follows the conv on the side stream
// (it needs only Y): its CTAs take each SM as the gate/up GEMM's CTA there
// finishes, filling the GEMM's last partial round.  Measured on B200 (builds
// alternated launch by launch): forward 0.2% faster at qwen3-4b, 0.5-0.8% at
// the long shapes.
#ifndef ITTT_TARGET_SIDE
#define ITTT_TARGET_SIDE 1
#endif

// 1 = the bf16 forward stores eta * Vhat (the target GEMM's epilogue scales the
// accumulator) and runs every later step with eta = 1: the scan's accumulator
// starts at W_down0 and its snapshots need no multiply, the gram is Z Z^T, the
// clip factor compares the norm of eta * delta directly.  The step entry points
// take Vhat and eta as before.  Measured on B200 (the two builds alternated
// launch by launch): forward 0.7% faster at qwen3-4b, 0.5-1% at the long shapes.
#ifndef ITTT_ETA_IN_VHAT
#define ITTT_ETA_IN_VHAT 1
#endif

// 1 = the forward computes Vhat with the conv in the target GEMM's prologue
// (tc_tconv_kernel, k <= 8; Y is never stored); 0 = conv, then target GEMM.
#ifndef ITTT_TARGET_CONV
#define ITTT_TARGET_CONV 0
#endif

// 1 = the forward computes the look-ahead conv (k <= 8) inside the gate/up
// GEMM kernel, in two extra warps per CTA that run beside the tensor-core
// pipeline; 0 = its own kernel between the gate/up and the target GEMM.  The
// two measured equal on B200 (qwen3-4b: 1.3594 vs 1.3555 ms and 1.4954 vs
// 1.4921 ms per forward: the warps cost the GEMM what the kernel costs).
#ifndef ITTT_CONV_IN_GATED
#define ITTT_CONV_IN_GATED 0
#endif

// Tokens per thread of the bf16 look-ahead conv.
#ifndef ITTT_CONV_RUN
#define ITTT_CONV_RUN 8
#endif

// 1 = kernels are launched with programmatic stream serialization: a kernel's
// prologue (barriers, TMEM, descriptor prefetch) overlaps the previous
// kernel's tail and it waits on the GPU (griddepcontrol.wait) before touching
// global memory.  0 = plain stream order.
#ifndef ITTT_PDL
#define ITTT_PDL 1
#endif

// Pair (two-SM, cta_group::2) tensor-core tiles: 1 = on (default), 0 = off.
#ifndef ITTT_PAIR
#define ITTT_PAIR 1
#endif
// Shared-memory pipeline depth (stages of 64-deep k-blocks) of the N = 256
// pair instances of each kind (measured best: 6); build-time tunables.
#ifndef ITTT_STAGES_GATED
#define ITTT_STAGES_GATED 6
#endif
#ifndef ITTT_STAGES_TARGET
#define ITTT_STAGES_TARGET 6
#endif
#ifndef ITTT_STAGES_SCAN
#define ITTT_STAGES_SCAN 6
#endif
#ifndef ITTT_STAGES_APPLY
#define ITTT_STAGES_APPLY 6
#endif
#ifndef ITTT_STAGES_NORM
#define ITTT_STAGES_NORM 6
#endif
// Decode: hidden units per warp of the gated GEMV for 5..8 sequences (1: fewer
// registers, more warps in flight; measured 0.132 -> 0.116 ms per step at 8).
#ifndef ITTT_GEMV_MMA_MIN_B  // decode batches from this size run the gated GEMV on warp MMAs
#define ITTT_GEMV_MMA_MIN_B 3
#endif
#ifndef ITTT_GEMV_U_WIDE
#define ITTT_GEMV_U_WIDE 1
#endif

// Store map over a bf16 [outer2, outer1, inner] view with explicit element
// strides of dims 1 and 2 (32-row x 64-column boxes, 128-byte swizzle).
bool make_store_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer1,
                    uint64_t outer2, uint64_t stride1, uint64_t stride2) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {inner, outer1, outer2};
  const cuuint64_t strides[2] = {stride1 * 2, stride2 * 2};
  const cuuint32_t box[3] = {64, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KIND, int BN, int STAGES, bool PAIR>
ittt_status launch_tc(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b2,
                      const TcParams& p, int work_items, cudaStream_t st,
                      const CUtensorMap* s_map = nullptr, const CUtensorMap* f_map = nullptr) {
  constexpr int smem = tc_smem_bytes<KIND, BN, STAGES, PAIR>();
  static_assert(smem <= 232448, "shared memory of a tc_gemm_kernel instance exceeds 227 KB");
  auto kern = tc_gemm_kernel<KIND, BN, STAGES, PAIR>;
  static std::atomic<bool> attr_done[kMaxDevices] = {};
  static std::atomic<int> max_clusters[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ITTT_ERR_CUDA;
  if (!attr_done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return ITTT_ERR_CUDA;
    attr_done[dev] = true;
  }
  const int sms = num_sms();
  if (sms <= 0) return ITTT_ERR_CUDA;
  if (work_items <= 0) return ITTT_OK;
  const CUtensorMap& sm_ = s_map ? *s_map : a;
  const CUtensorMap& fm_ = f_map ? *f_map : a;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = ITTT_PDL;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  // the gate/up kernel's two conv warps only when it runs the conv
  cfg.blockDim = dim3((KIND == TC_GATED && p.conv_y == nullptr) ? 192 : tc_threads(KIND), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  if (!PAIR) {
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(work_items < sms ? work_items : sms, 1, 1);
    if (cudaLaunchKernelEx(&cfg, kern, a, b, b2, sm_, fm_, p) != cudaSuccess) return ITTT_ERR_CUDA;
    return launch_status();
  }
  cfg.numAttrs = 2;
  if (!max_clusters[dev]) {
    cudaLaunchConfig_t q = cfg;
    q.gridDim = dim3(2 * (sms / 2), 1, 1);
    q.attrs = attr + 1;  // cluster shape only
    q.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess || n <= 0) return ITTT_ERR_CUDA;
    max_clusters[dev] = n;
  }
  const int maxc = max_clusters[dev].load();
  const int clusters = work_items < maxc ? work_items : maxc;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, a, b, b2, sm_, fm_, p) != cudaSuccess) return ITTT_ERR_CUDA;
  return launch_status();
}

// Rasterisation groups of the gate/up and target GEMMs: m-tiles (256 rows of
// A = H or Y) per group, so that a group's A rows (about ITTT_GROUP_MB MiB)
// stay in L2 while every column tile of the weights passes over them; without
// groups A is read from DRAM once per column tile when it exceeds L2 (at
// qwen3-4b-128k, 671 MB of H 76 times).
#ifndef ITTT_GROUP_MB
#define ITTT_GROUP_MB 24
#endif
// m_rows: rows of A.  0 (no groups) when all of A fits in twice the group
// size (then it stays in L2 anyway, and groups would only re-read the weights
// once per group: qwen3-4b's 42 MB of H read the 100 MB of weights twice).
int group_m_tiles(long long m_rows, long long d) {
  const long long group_bytes = (long long)ITTT_GROUP_MB * 1024 * 1024;
  if (m_rows * d * 2 <= 2 * group_bytes) return 0;
  const long long g = group_bytes / (256ll * d * 2);
  return g < 1 ? 1 : int(g);
}

// Tile width policy of the target / apply / scan GEMMs: 0 = by wave
// efficiency, 128 or 256 = fixed (build-time tunables).
#ifndef ITTT_TARGET_BN
#define ITTT_TARGET_BN 0
#endif
#ifndef ITTT_APPLY_BN
#define ITTT_APPLY_BN 0
#endif
#ifndef ITTT_SCAN_BN
#define ITTT_SCAN_BN 0
#endif

// N = 256 tiles halve the shared-memory operand traffic per flop of N = 128
// tiles and measured faster on B200 even where their last wave is emptier
// (qwen3-4b: apply 357 vs 452 us, target 96 vs 131 us); N = 128 is kept for
// problems too small to fill the GPU with N = 256 tiles.
bool choose_wide(int policy, double eff256, double eff128, long long units256, int sms) {
  if (policy == 256) return true;
  if (policy == 128) return false;
  (void)eff256;
  (void)eff128;
  return units256 >= sms / 2;
}

// Fraction of the last wave that is busy, for choosing a tile width.
double wave_efficiency(long long units, int sms) {
  if (units <= 0 || sms <= 0) return 1.0;
  const long long waves = cdiv(units, sms);
  return double(units) / double(waves * sms);
}

// -------------------------------------------------------------- validation

bool is_bf16(const ittt_problem* p) { return p->dtype == ITTT_BF16; }

ittt_status validate(const ittt_problem* p) {
  if (!p) return ITTT_ERR_INVALID_ARG;
  if (p->B <= 0 || p->T <= 0 || p->d <= 0 || p->f <= 0 || p->C <= 0 || p->k <= 0)
    return ITTT_ERR_INVALID_ARG;
  if (p->k > 16) return ITTT_ERR_UNSUPPORTED;
  if (p->dtype != ITTT_F32 && p->dtype != ITTT_BF16) return ITTT_ERR_INVALID_ARG;
  if (p->form < ITTT_FORM_AUTO || p->form > ITTT_FORM_HYBRID) return ITTT_ERR_INVALID_ARG;
  if ((p->flags & ~(ITTT_FLAG_PAD_CHUNK_END | ITTT_FLAG_X0_LOOKAHEAD)) != 0 || p->reserved != 0)
    return ITTT_ERR_INVALID_ARG;
  if (!isfinite(p->eta)) return ITTT_ERR_INVALID_ARG;
  if (!isfinite(p->clip) || p->clip < 0.f) return ITTT_ERR_INVALID_ARG;
  if (p->T % p->C != 0) return ITTT_ERR_UNSUPPORTED;
  // 32-bit row coordinates in the kernels
  const long long n = p->T / p->C;
  if (p->B * p->T >= (1ll << 31) || p->d >= (1ll << 30) || p->f >= (1ll << 30)) return ITTT_ERR_UNSUPPORTED;
  if (p->B * n * p->d >= (1ll << 31)) return ITTT_ERR_UNSUPPORTED;
  if (is_bf16(p)) {
    if (p->d % 8 || p->f % 8 || p->C % 128) return ITTT_ERR_UNSUPPORTED;
    // the fused scan keeps W_down0 / eta in the accumulator
    if (p->eta != 0.f && fabsf(p->eta) < 1e-30f) return ITTT_ERR_UNSUPPORTED;
  } else {
    if (p->B * p->T * (p->d > p->f ? p->d : p->f) >= (1ll << 31)) return ITTT_ERR_UNSUPPORTED;
  }
  return ITTT_OK;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// The form that computes the chunk recurrence for problem p.  The fp32 path
// always runs the prefix form.  AUTO picks the dual or the hybrid form by the
// rules fitted to the measured crossovers (dual_is_faster, hybrid_is_faster).
bool dual_is_faster(const ittt_problem* p);

// Chunks per group of the hybrid form: groups of about ITTT_HYBRID_TOKENS
// tokens, at least two chunks.
#ifndef ITTT_HYBRID_TOKENS
#define ITTT_HYBRID_TOKENS 1024
#endif
int hybrid_group(const ittt_problem* p) {
  return p->C * 2 >= ITTT_HYBRID_TOKENS ? 2 : ITTT_HYBRID_TOKENS / p->C;
}

// The hybrid form needs whole groups and at least two of them (one group is
// the dual form), and chunks of a multiple of 256 tokens (the chunk sizes it
// has been checked at; others run the prefix form).
bool hybrid_fits(const ittt_problem* p) {
  const long long n = p->T / p->C, m = hybrid_group(p);
  return p->C % 256 == 0 && n % m == 0 && n / m >= 2;
}

// AUTO's second rule: the hybrid form for chunks of 256 tokens when T d >= 2^24
// (and the hybrid fits).  At C = 256 a chunk is four k-blocks of the scan's
// MMA, so the prefix form's per-chunk snapshot epilogue bounds its scan; the
// hybrid stores one weight per group of four chunks and adds in-group Gram
// work.  Measured on B200 with the forms alternated forward by forward
// (bench.py --compare-forms prefix,hybrid --paired): hybrid/prefix time
// 1.038 at (d, T) = (2560, 2048), 1.004 at (2560, 4096), 0.92-0.93 at
// (2560, 8192 ... 131072), 0.91 at (4096, 4096), 0.92 at (4096, 32768),
// 0.94-0.96 at (5120, 4096 ... 16384), 0.95 at B = 2; at C = 512 the two are
// equal at T = 131072 and the hybrid is 4% slower at T = 8192, so the rule is
// C = 256 only.
bool hybrid_is_faster(const ittt_problem* p) {
  return p->C == 256 && hybrid_fits(p) && double(p->T) * double(p->d) >= 16777216.0;
}

int resolve_form(const ittt_problem* p) {
  if (!is_bf16(p)) return ITTT_FORM_PREFIX;
  if (p->form == ITTT_FORM_HYBRID) return hybrid_fits(p) ? ITTT_FORM_HYBRID : ITTT_FORM_PREFIX;
  if (p->form != ITTT_FORM_AUTO) return p->form;
  if (dual_is_faster(p)) return ITTT_FORM_DUAL;
  return hybrid_is_faster(p) ? ITTT_FORM_HYBRID : ITTT_FORM_PREFIX;
}

struct Layout {
  size_t z, y, v, stack, gram, norm2, sched, total;
  int form;
  bool tail_dual;     // prefix form: chunks 0..1 by the dual kernels (P of [B, 2C, C] at gram)
  bool one_launch;    // prefix form, bf16, n >= 2, eta != 0: the one-launch recurrence can
                      // run (its work counter and flags are at sched)
  bool fused;         // ... and the forward runs it
  bool fused_target;  // ... which also computes Vhat (target units first in its queue)
};

// Target units of the one-launch recurrence: 256-token x 256-column tiles of Vhat.
long long recur_target_units(const ittt_problem* p) {
  return ((p->B * p->T + 255) / 256) * ((p->d + 255) / 256);
}

// Readiness flags of the fused recurrence: one per (sequence, 256-row d-tile,
// chunk but the last), and one per target unit when it computes Vhat, after a
// 256-byte word for the work counter.
size_t recur_sched_bytes(const ittt_problem* p, bool with_target) {
  const size_t n = size_t(p->T / p->C);
  const size_t dtiles = size_t((p->d + 255) / 256);
  return 256 + (size_t(p->B) * dtiles * (n - 1) + (with_target ? size_t(recur_target_units(p)) : 0)) *
                   sizeof(uint32_t);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

Layout plan(const ittt_problem* p) {
  const size_t es = is_bf16(p) ? 2 : 4;
  const size_t BT = size_t(p->B) * size_t(p->T);
  const size_t n = size_t(p->T / p->C);
  Layout L{};
  L.form = resolve_form(p);
  size_t off = 0;
  L.z = off;
  off += align256(BT * p->f * es);
  L.y = off;
  off += align256(BT * p->d * es);
  L.v = off;
  off += align256(BT * p->d * es);
  L.stack = off;
  if (L.form == ITTT_FORM_PREFIX)
    off += align256(size_t(p->B) * (n - 1) * size_t(p->d) * size_t(p->f) * es);
  if (L.form == ITTT_FORM_HYBRID)  // every group's starting weight, W_down0 included
    off += align256(size_t(p->B) * (n / hybrid_group(p)) * size_t(p->d) * size_t(p->f) * es);
  L.gram = off;
  L.one_launch = is_bf16(p) && L.form == ITTT_FORM_PREFIX && ITTT_PAIR && n >= 2 && p->eta != 0.f;
  L.fused = L.one_launch && ITTT_FUSED_RECUR;
  L.fused_target = L.fused && ITTT_RECUR_TARGET && p->clip == 0.f;
  L.tail_dual = !L.fused && is_bf16(p) && L.form == ITTT_FORM_PREFIX && ITTT_TAIL_DUAL && ITTT_PAIR &&
                n >= 3 && p->C % 256 == 0 && p->eta != 0.f;
  if (L.form == ITTT_FORM_DUAL) off += align256(BT * size_t(p->T) * es);
  if (L.form == ITTT_FORM_HYBRID)  // eta Z_t Z_s inside each group: [B*T, G - C]
    off += align256(BT * size_t(hybrid_group(p) - 1) * size_t(p->C) * es);
  if (L.tail_dual) off += align256(size_t(p->B) * 2 * size_t(p->C) * size_t(p->C) * es);
  L.norm2 = off;  // clipping: [B, n] sums of squares of the chunk deltas / eta^2
  if (p->clip > 0.f) off += align256(size_t(p->B) * n * sizeof(float));
  L.sched = off;
  if (L.one_launch) off += align256(recur_sched_bytes(p, L.fused_target));
  L.total = off;
  return L;
}

// ------------------------------------------------------------- bf16 steps

typedef __nv_bfloat16 bf16;

ConvGeom conv_geom(const ittt_problem* p);

// conv_Y != nullptr: the gate/up kernel also computes the look-ahead conv of
// X0 into conv_Y (k <= 8), in two extra warps per CTA.
ittt_status gated_bf16(const ittt_problem* p, const void* H, const void* Wg, const void* Wu,
                       void* Z, cudaStream_t st, const void* conv_X0 = nullptr,
                       const void* conv_K = nullptr, void* conv_Y = nullptr) {
  const long long M = p->B * p->T;
  CUtensorMap a, b, b2;
  if (!make_map(&a, H, p->d, M, p->d, 64, 128) || !make_map(&b, Wg, p->d, p->f, p->d, 64, 128) ||
      !make_map(&b2, Wu, p->d, p->f, p->d, 64, 128))
    return ITTT_ERR_CUDA;
  constexpr bool PAIR = ITTT_PAIR != 0;
  TcParams tp{};
  tp.m_tiles = int(cdiv(M, PAIR ? 256 : 128));
  tp.n_tiles = int(cdiv(p->f, 128));
  tp.num_units = tp.m_tiles * tp.n_tiles;
  tp.M = int(M);
  tp.N = int(p->f);
  tp.num_kb = int(cdiv(p->d, 64));
  tp.out = static_cast<bf16*>(Z);
  tp.ldo = p->f;
  tp.wait_ns = g_wait_ns.load();
  tp.group_m = ITTT_GROUP_MB > 0 ? group_m_tiles(M, p->d) : 0;
  if (conv_Y != nullptr) {
    if (p->k > 8) return ITTT_ERR_UNSUPPORTED;
    tp.conv_x0 = static_cast<const bf16*>(conv_X0);
    tp.conv_k = static_cast<const bf16*>(conv_K);
    tp.conv_y = static_cast<bf16*>(conv_Y);
    tp.conv_g = conv_geom(p);
    tp.conv_d = int(p->d);
    tp.conv_taps = p->k;
    tp.conv_B = int(p->B);
  }
  CUtensorMap zm;  // Z store map: [1, B*T, f]
  if (!make_store_map(&zm, Z, p->f, M, 1, p->f, M * p->f)) return ITTT_ERR_CUDA;
  return launch_tc<TC_GATED, 256, PAIR ? ITTT_STAGES_GATED : 4, PAIR>(a, b, b2, tp, tp.num_units, st,
                                                                     nullptr, &zm);
}

ConvGeom conv_geom(const ittt_problem* p) {
  ConvGeom g;
  g.T = int(p->T);
  g.Tx = int(p->T) + ((p->flags & ITTT_FLAG_X0_LOOKAHEAD) ? p->k - 1 : 0);
  g.C = p->C;
  g.chunk_pad = (p->flags & ITTT_FLAG_PAD_CHUNK_END) ? 1 : 0;
  return g;
}

ittt_status conv_bf16(const ittt_problem* p, const void* X0, const void* Kc, void* Y,
                      cudaStream_t st) {
  const int groups = int(p->d / 8);
  // a block width (multiple of 32, <= 256) that divides the channel groups,
  // so no thread idles (d = 2560: 320 groups = 2 blocks of 160)
  int threads = 0;
  for (int t = 256; t >= 32; t -= 32)
    if (groups % t == 0) {
      threads = t;
      break;
    }
  if (threads == 0) threads = groups < 128 ? ((groups + 31) / 32) * 32 : 128;
  constexpr int RUN = ITTT_CONV_RUN;
  const long long runs = p->B * cdiv(p->T, RUN);
  if (runs >= 65536 * 1024ll) return ITTT_ERR_UNSUPPORTED;
  dim3 grid(unsigned(cdiv(groups, threads)), unsigned(runs));
  const bf16* x = static_cast<const bf16*>(X0);
  const bf16* kc = static_cast<const bf16*>(Kc);
  bf16* y = static_cast<bf16*>(Y);
  const int d = int(p->d);
  const ConvGeom g = conv_geom(p);
  if (grid.y > 65535) {
    // very long batches: fall back to the element-wise kernel
    const long long rows = p->B * p->T;
    conv_bf16_generic_kernel<<<unsigned(cdiv(rows * d, 256)), 256, 0, st>>>(x, kc, y, g, d, p->k, rows);
    return launch_status();
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = ITTT_PDL;
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaSuccess;
  switch (p->k) {
    case 1: e = cudaLaunchKernelEx(&cfg, conv_bf16_kernel<1, RUN>, x, kc, y, g, d); break;
    case 2: e = cudaLaunchKernelEx(&cfg, conv_bf16_kernel<2, RUN>, x, kc, y, g, d); break;
    case 3: e = cudaLaunchKernelEx(&cfg, conv_bf16_kernel<3, RUN>, x, kc, y, g, d); break;
    case 4: e = cudaLaunchKernelEx(&cfg, conv_bf16_kernel<4, RUN>, x, kc, y, g, d); break;
    case 5: e = cudaLaunchKernelEx(&cfg, conv_bf16_kernel<5, RUN>, x, kc, y, g, d); break;
    case 6: e = cudaLaunchKernelEx(&cfg, conv_bf16_kernel<6, RUN>, x, kc, y, g, d); break;
    case 7: e = cudaLaunchKernelEx(&cfg, conv_bf16_kernel<7, RUN>, x, kc, y, g, d); break;
    case 8: e = cudaLaunchKernelEx(&cfg, conv_bf16_kernel<8, RUN>, x, kc, y, g, d); break;
    default: {
      const long long rows = p->B * p->T;
      conv_bf16_generic_kernel<<<unsigned(cdiv(rows * d, 256)), 256, 0, st>>>(x, kc, y, g, d, p->k, rows);
    }
  }
  if (e != cudaSuccess) return ITTT_ERR_CUDA;
  return launch_status();
}

ittt_status target_gemm_bf16(const ittt_problem* p, const void* Y, const void* Wt, void* V,
                             cudaStream_t st, float scale = 1.0f) {
  const long long M = p->B * p->T;
  constexpr bool PAIR = ITTT_PAIR != 0;
  const int sms = num_sms() / (PAIR ? 2 : 1);
  const long long mt = cdiv(M, PAIR ? 256 : 128);
  const bool wide = choose_wide(ITTT_TARGET_BN, wave_efficiency(mt * cdiv(p->d, 256), sms),
                                wave_efficiency(mt * cdiv(p->d, 128), sms), mt * cdiv(p->d, 256), sms);
  const int BN = wide ? 256 : 128;
  CUtensorMap a, b;
  if (!make_map(&a, Y, p->d, M, p->d, 64, 128) || !make_map(&b, Wt, p->d, p->d, p->d, 64, 64))
    return ITTT_ERR_CUDA;
  TcParams tp{};
  tp.m_tiles = int(mt);
  tp.n_tiles = int(cdiv(p->d, BN));
  tp.num_units = tp.m_tiles * tp.n_tiles;
  tp.M = int(M);
  tp.N = int(p->d);
  tp.num_kb = int(cdiv(p->d, 64));
  tp.out = static_cast<bf16*>(V);
  tp.ldo = p->d;
  tp.v_scale = scale;
  tp.wait_ns = g_wait_ns.load();
  tp.group_m = ITTT_GROUP_MB > 0 ? group_m_tiles(M, p->d) : 0;
  CUtensorMap vm;  // Vhat store map: [1, B*T, d]
  if (!make_store_map(&vm, V, p->d, M, 1, p->d, M * p->d)) return ITTT_ERR_CUDA;
  if (wide)
    return launch_tc<TC_TARGET, 256, PAIR ? ITTT_STAGES_TARGET : 4, PAIR>(a, b, b, tp, tp.num_units, st,
                                                                         nullptr, &vm);
  return launch_tc<TC_TARGET, 128, 6, PAIR>(a, b, b, tp, tp.num_units, st, nullptr, &vm);
}

// Vhat = Conv1D(X0) W_target with the conv computed in the GEMM's prologue
// (tc_tconv_kernel): Y is never stored.  k <= 8.
ittt_status target_conv_bf16(const ittt_problem* p, const void* X0, const void* Kc, const void* Wt,
                             void* V, cudaStream_t st) {
  constexpr int STAGES = 4;
  constexpr int smem = tconv_smem_bytes<STAGES>();
  static_assert(smem <= 232448, "shared memory of the conv-target kernel exceeds 227 KB");
  if (p->k > 8) return ITTT_ERR_UNSUPPORTED;
  const long long M = p->B * p->T;
  const ConvGeom g = conv_geom(p);
  CUtensorMap mx, mb, mv;
  if (!make_map(&mx, X0, p->d, uint64_t(p->B) * g.Tx, p->d, 64, TconvShape::WROWS) ||
      !make_map(&mb, Wt, p->d, p->d, p->d, 64, 64) ||
      !make_store_map(&mv, V, p->d, M, 1, p->d, M * p->d))
    return ITTT_ERR_CUDA;
  TconvParams tp{};
  tp.m_tiles = int(cdiv(M, 256));
  tp.n_tiles = int(cdiv(p->d, 256));
  tp.num_units = tp.m_tiles * tp.n_tiles;
  tp.M = int(M);
  tp.N = int(p->d);
  tp.num_kb = int(cdiv(p->d, 64));
  tp.d = int(p->d);
  tp.k = p->k;
  tp.g = g;
  tp.conv_k = static_cast<const bf16*>(Kc);
  tp.wait_ns = g_wait_ns.load();
  auto kern = p->k == 4 ? tc_tconv_kernel<STAGES, 4> : tc_tconv_kernel<STAGES, 0>;
  static std::atomic<bool> attr_done[kMaxDevices][2] = {};
  static std::atomic<int> max_clusters[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ITTT_ERR_CUDA;
  const int inst = p->k == 4 ? 0 : 1;
  if (!attr_done[dev][inst]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return ITTT_ERR_CUDA;
    attr_done[dev][inst] = true;
  }
  const int sms = num_sms();
  if (sms <= 0) return ITTT_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = ITTT_PDL;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.blockDim = dim3(448, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (!max_clusters[dev]) {
    cudaLaunchConfig_t q = cfg;
    q.gridDim = dim3(2 * (sms / 2), 1, 1);
    q.attrs = attr + 1;
    q.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, kern, &q) != cudaSuccess || nc <= 0) return ITTT_ERR_CUDA;
    max_clusters[dev] = nc;
  }
  const int clusters = tp.num_units < max_clusters[dev].load() ? tp.num_units : max_clusters[dev].load();
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, mx, mb, mv, tp) != cudaSuccess) return ITTT_ERR_CUDA;
  return launch_status();
}

// snap_from: W^(i) for i < snap_from are not stored (their stack slices are
// left unwritten).  snap_every > 1 (the hybrid form): only W^(i) with i a
// multiple of snap_every are stored, W^(snap_every * j) in slice
// snap_first + j - 1 of the sequence's snap_per_seq slices.
ittt_status scan_bf16(const ittt_problem* p, const void* V, const void* Z, const void* W0,
                      void* stack, float* Wf, cudaStream_t st, int snap_from = 0,
                      const float* W0_f32 = nullptr, int snap_every = 1, int snap_per_seq = 0,
                      int snap_first = 0) {
  const long long BT = p->B * p->T;
  const int n = int(p->T / p->C);
  if (n > 1 && !stack) return ITTT_ERR_INVALID_ARG;
  constexpr bool PAIR = ITTT_PAIR != 0;
  const int sms = num_sms() / (PAIR ? 2 : 1);
  const long long mt = cdiv(p->d, PAIR ? 256 : 128);
  const long long t256 = p->B * mt * cdiv(p->f, 256), t128 = p->B * mt * cdiv(p->f, 128);
  const bool wide = choose_wide(ITTT_SCAN_BN, wave_efficiency(cdiv(t256, 2), sms),
                                wave_efficiency(cdiv(t128, 2), sms), cdiv(t256, 2), sms);
  const int BN = wide ? 256 : 128;
  CUtensorMap a, b;
  // (a driver that refuses the 3-D view gets the 2-D boxes)
  const bool mn3d = ITTT_SCAN_MN3D && PAIR && wide && p->d % 64 == 0 && p->f % 64 == 0 &&
                    make_map_mn3(&a, V, p->d, BT, p->d, 2) && make_map_mn3(&b, Z, p->f, BT, p->f, 2);
  if (!mn3d && (!make_map(&a, V, p->d, BT, p->d, 64, 64) || !make_map(&b, Z, p->f, BT, p->f, 64, 64)))
    return ITTT_ERR_CUDA;
  TcParams tp{};
  tp.mn3d = mn3d ? 1 : 0;
  tp.m_tiles = int(mt);
  tp.n_tiles = int(cdiv(p->f, BN));
  tp.num_units = int(p->B) * tp.m_tiles * tp.n_tiles;
  tp.M = int(p->d);
  tp.N = int(p->f);
  tp.num_kb = p->C / 64;
  tp.T = int(p->T);
  tp.C = p->C;
  tp.nchunk = n;
  tp.eta = p->eta;
  tp.inv_eta = 1.0f / p->eta;
  tp.out = static_cast<bf16*>(stack);
  tp.ldo = p->f;
  tp.out_f32 = Wf;
  tp.w0 = static_cast<const bf16*>(W0);
  tp.w0_f32 = W0_f32;
  tp.wait_ns = g_wait_ns.load();
  tp.snap_from = snap_from;
  tp.snap_every = snap_every;
  tp.snap_per_seq = snap_per_seq;
  tp.snap_first = snap_first;
  const uint64_t slices = uint64_t(p->B) * uint64_t(snap_per_seq > 0 ? snap_per_seq : n - 1);
  tp.stack_slices = n > 1 ? int(slices) : 0;
  CUtensorMap sm, fm;
  // the stack may be absent (one chunk): any valid map stands in, it is never stored to
  // store boxes: one epilogue warp's 32 rows, or (ITTT_SCAN_STORE128 builds)
  // the CTA's 128 from pooled staging, only for C >= 512: at C = 256 the
  // snapshot epilogue is the bottleneck and the four warps' hand-offs add to it
  tp.store128 = (ITTT_SCAN_STORE128 && p->C >= 512) ? 1 : 0;
  const uint32_t srows = tp.store128 ? 128 : 32;
  if (!make_map_3d(&sm, n > 1 ? stack : static_cast<const void*>(Wf), false, p->f, p->d,
                   n > 1 ? slices : 1, 64, srows) ||
      !make_map_3d(&fm, Wf, true, p->f, p->d, p->B, 32, srows))
    return ITTT_ERR_CUDA;
  const int pairs = (tp.num_units + 1) / 2;
  if (wide) return launch_tc<TC_SCAN, 256, PAIR ? ITTT_STAGES_SCAN : 4, PAIR>(a, b, b, tp, pairs, st, &sm, &fm);
  return launch_tc<TC_SCAN, 128, 5, PAIR>(a, b, b, tp, pairs, st, &sm, &fm);
}

// all_w0: every chunk uses W_down0 (eta == 0).  first_chunk: chunks before it
// are left to another kernel.
// stack_slices: slices the stack holds (default B (n - 1)); a smaller value
// makes the kernel refuse the units past it (the device-check self-test).
ittt_status apply_bf16(const ittt_problem* p, const void* Z, const void* W0, const void* stack,
                       void* O, bool all_w0, cudaStream_t st, int first_chunk = 0,
                       long long stack_slices = -1) {
  const long long BT = p->B * p->T;
  const int n = all_w0 ? 1 : int(p->T / p->C);
  const int Cc = all_w0 ? int(p->T) : p->C;
  if (n > 1 && !stack) return ITTT_ERR_INVALID_ARG;
  constexpr bool PAIR = ITTT_PAIR != 0;
  const int sms = num_sms() / (PAIR ? 2 : 1);
  const long long per = p->B * (n - first_chunk) * cdiv(Cc, PAIR ? 256 : 128);
  // tile width: N = 256 unless set at build time (128).  N = 160 would fill 7
  // full rounds where N = 256 leaves 4.3 of 5 at qwen3-4b, but measured slower
  // on B200 (385 vs 331 us): the narrower tile costs more than the idle tail.
  int BN = ITTT_APPLY_BN == 128 ? 128 : 256;
  if (ITTT_APPLY_BN == 0 && per * cdiv(p->d, 256) < sms / 2) BN = 128;
  const int brows = PAIR ? BN / 2 : BN;  // B rows loaded by each CTA
  CUtensorMap a, b, b2;
  if (!make_map(&a, Z, p->f, BT, p->f, 64, 128) ||
      !make_map(&b2, W0, p->f, p->d, p->f, 64, brows))
    return ITTT_ERR_CUDA;
  const long long slices = stack_slices >= 0 ? stack_slices : p->B * (n - 1);
  if (n > 1) {
    if (slices <= 0 || !make_map(&b, stack, p->f, uint64_t(slices) * p->d, p->f, 64, brows))
      return ITTT_ERR_CUDA;
  } else {
    b = b2;
  }
  TcParams tp{};
  tp.m_tiles = int(cdiv(Cc, PAIR ? 256 : 128));
  tp.n_tiles = int(cdiv(p->d, BN));
  tp.num_units = int(per) * tp.n_tiles;
  tp.M = Cc;
  tp.N = int(p->d);
  tp.num_kb = int(cdiv(p->f, 64));
  tp.T = int(p->T);
  tp.C = Cc;
  tp.nchunk = n;
  tp.chunk_base = first_chunk;
  tp.chunk_count = n - first_chunk;
  tp.stack_slices = n > 1 ? int(slices) : 0;
  tp.out = static_cast<bf16*>(O);
  tp.ldo = p->d;
  tp.wait_ns = g_wait_ns.load();
  // O store map: [B*n, C, d] so that a tile never writes past its chunk
  CUtensorMap om;
  if (!make_store_map(&om, O, p->d, Cc, uint64_t(p->B) * n, p->d, uint64_t(Cc) * p->d))
    return ITTT_ERR_CUDA;
  if (BN == 256)
    return launch_tc<TC_APPLY, 256, PAIR ? ITTT_STAGES_APPLY : 4, PAIR>(a, b, b2, tp, tp.num_units, st,
                                                                       nullptr, &om);
  return launch_tc<TC_APPLY, 128, PAIR ? 6 : 5, PAIR>(a, b, b2, tp, tp.num_units, st, nullptr, &om);
}

// Dual form, part 1: P[b, t, s] = eta Z_t . Z_s for chunk(s) < chunk(t), else 0.
// rows: the first `rows` tokens of every sequence (a multiple of C); P is
// [B, rows, rows - C] (token s < rows - C is the only one a row can use).
ittt_status gram_bf16(const ittt_problem* p, const void* Z, void* P, long long rows,
                      cudaStream_t st) {
  constexpr bool PAIR = ITTT_PAIR != 0;
  constexpr int BN = 256;
  const long long BT = p->B * p->T;
  const long long cols = rows - p->C;
  if (cols <= 0) return ITTT_OK;
  CUtensorMap a, b;
  if (!make_map(&a, Z, p->f, BT, p->f, 64, 128) ||
      !make_map(&b, Z, p->f, BT, p->f, 64, PAIR ? BN / 2 : BN))
    return ITTT_ERR_CUDA;
  TcParams tp{};
  tp.m_tiles = int(cdiv(rows, PAIR ? 256 : 128));
  tp.n_tiles = int(cdiv(cols, BN));
  tp.num_units = int(p->B) * tp.m_tiles * tp.n_tiles;
  tp.M = int(rows);
  tp.N = int(cols);
  tp.prow = int(rows);
  tp.num_kb = int(cdiv(p->f, 64));
  tp.T = int(p->T);
  tp.C = p->C;
  tp.eta = p->eta;
  tp.bn = BN;
  tp.out = static_cast<bf16*>(P);
  tp.ldo = cols;
  tp.wait_ns = g_wait_ns.load();
  return launch_tc<TC_GRAM, BN, PAIR ? 6 : 4, PAIR>(a, b, b, tp, tp.num_units, st);
}

// Dual form, part 2: O = Z W_down0^T + P Vhat.
// rows: output rows computed per sequence (the first `rows` tokens, a multiple
// of C); P as written by gram_bf16 with the same `rows`.
// per_seq_w0: W0 holds one first operand [d, f] per sequence ([B, d, f]: the
// hybrid form's group-start weights, a "sequence" being a group) instead of
// one shared W_down0.
ittt_status dualo_bf16(const ittt_problem* p, const void* Z, const void* W0, const void* P,
                       const void* V, void* O, long long rows, cudaStream_t st,
                       bool per_seq_w0 = false) {
  constexpr bool PAIR = ITTT_PAIR != 0;
  constexpr int BN = 256;
  const long long BT = p->B * p->T;
  const long long cols = rows - p->C;
  const uint64_t w0_rows = uint64_t(per_seq_w0 ? p->B : 1) * uint64_t(p->d);
  CUtensorMap a, b, b2, pm;
  if (!make_map(&a, Z, p->f, BT, p->f, 64, 128) ||
      !make_map(&b, W0, p->f, w0_rows, p->f, 64, PAIR ? BN / 2 : BN) ||
      !make_map(&b2, V, p->d, BT, p->d, 64, 64))
    return ITTT_ERR_CUDA;
  if (cols > 0) {
    if (!make_map(&pm, P, cols, uint64_t(p->B) * rows, cols, 64, 128)) return ITTT_ERR_CUDA;
  } else {
    pm = a;  // never read: no row of the first chunk has earlier tokens
  }
  TcParams tp{};
  tp.m_tiles = int(cdiv(rows, PAIR ? 256 : 128));
  tp.n_tiles = int(cdiv(p->d, BN));
  tp.num_units = int(p->B) * tp.m_tiles * tp.n_tiles;
  tp.M = int(rows);
  tp.prow = int(rows);
  tp.N = int(p->d);
  tp.num_kb = int(cdiv(p->f, 64));
  tp.T = int(p->T);
  tp.C = p->C;
  tp.out = static_cast<bf16*>(O);
  tp.ldo = p->d;
  tp.group_count = per_seq_w0 ? int(p->B) : 0;
  tp.wait_ns = g_wait_ns.load();
  CUtensorMap om;  // O store map: [B, rows, d] inside the [B, T, d] output
  if (!make_store_map(&om, O, p->d, rows, p->B, p->d, uint64_t(p->T) * p->d)) return ITTT_ERR_CUDA;
  return launch_tc<TC_DUALO, BN, PAIR ? 6 : 4, PAIR>(a, b, b2, tp, tp.num_units, st, &pm, &om);
}

// Update-norm clipping, bf16: norm2[b, i] += ||Vhat_i^T Z_i||_F^2 (norm2 zeroed
// here), then the rows of every chunk whose delta exceeds p->clip are scaled.
ittt_status clip_targets_bf16(const ittt_problem* p, const void* Z, void* V, float* norm2,
                              cudaStream_t st) {
  constexpr bool PAIR = ITTT_PAIR != 0;
  constexpr int BN = 256;
  const long long BT = p->B * p->T;
  const long long n = p->T / p->C;
  if (cudaMemsetAsync(norm2, 0, size_t(p->B * n) * sizeof(float), st) != cudaSuccess)
    return ITTT_ERR_CUDA;
  const int brows = PAIR ? BN / 2 : BN;
  CUtensorMap za, zb, va, vb;
  if (!make_map(&za, Z, p->f, BT, p->f, 64, 128) || !make_map(&zb, Z, p->f, BT, p->f, 64, brows) ||
      !make_map(&va, V, p->d, BT, p->d, 64, 128) || !make_map(&vb, V, p->d, BT, p->d, 64, brows))
    return ITTT_ERR_CUDA;
  const int tile = PAIR ? 256 : 128;
  TcParams tp{};
  tp.m_tiles = int(cdiv(p->T, tile));
  tp.dt_count = int(cdiv(p->C, tile)) + 1;
  tp.n_tiles = 1;
  tp.num_units = int(p->B) * tp.m_tiles * tp.dt_count;
  tp.M = int(p->T);
  tp.N = int(p->T);
  tp.num_kb = int(cdiv(p->f, 64));
  tp.num_kb2 = int(cdiv(p->d, 64));
  tp.T = int(p->T);
  tp.C = p->C;
  tp.nchunk = int(n);
  tp.norm2 = norm2;
  tp.wait_ns = g_wait_ns.load();
  ittt_status s = launch_tc<TC_NORM, BN, PAIR ? ITTT_STAGES_NORM : 4, PAIR>(za, zb, va, tp, tp.num_units, st, &vb);
  if (s != ITTT_OK) return s;
  const long long items = BT * (p->d / 8);
  clip_scale_rows_bf16<<<unsigned(cdiv(items, 256)), 256, 0, st>>>(
      static_cast<bf16*>(V), norm2, p->eta, p->clip, int(p->T), p->C, int(p->d), BT);
  return launch_status();
}

// AUTO's rule: the dual form when the chunks are short (C <= 256) and
// T C (d + f) <= 170 d f, else the prefix form.  Per sequence the dual form
// adds about T^2 (d + f) tensor FLOP (the Gram blocks and their products with
// Vhat) and the prefix form stores and reads back n - 1 = T / C - 1 weights of
// d x f, so the dual form's extra cost over the prefix form's grows as
// T C (d + f) / (d f); short chunks also leave the fused scan's snapshot
// epilogue too little time per chunk.  The constant 170 and the C <= 256 cut
// are fitted to bench.py --sweep-forms on B200 (whole forward, L2 flushed,
// median of 5): three widths (d, f) = (2560, 9728), (4096, 14336),
// (5120, 17408) x B in {1, 2, 4} x T in {1024, 1536, 2048, 3072, 4096, 8192}
// x C in {256, 512, 1024, 2048}, 162 points.  Over those points the rule's
// picks are 0.34% slower than the faster form on average (always the prefix
// form: 0.99%); it misses 16 points, 8 of them by more than 3% (all where the
// dual form won at C = 256 somewhat beyond the threshold, up to 10%).  The
// batch size B multiplies both forms' costs and does not enter the rule.
bool dual_is_faster(const ittt_problem* p) {
  if (p->C > 256) return false;
  return double(p->T) * double(p->C) * double(p->d + p->f) <= 170.0 * double(p->d) * double(p->f);
}

// The prefix form's recurrence in one persistent launch (tc_recur_kernel):
// the fused scan writes W^(1..n-1) into the stack and W_down_final, the apply
// units compute O of every chunk as soon as their d-tile's W^(i) is stored.
// sched: recur_sched_bytes() bytes, zero on entry (the work counter and the
// readiness flags).  With Y and Wt given, the launch also computes Vhat = Y Wt
// into V first (target units ahead of the scan in the queue).
ittt_status recur_fused_bf16(const ittt_problem* p, const void* V, const void* Z, const void* W0,
                             void* stack, void* O, float* Wf, uint32_t* sched, cudaStream_t st,
                             const void* Y = nullptr, const void* Wt = nullptr) {
  constexpr int STAGES = ITTT_STAGES_RECUR;
  constexpr int smem = recur_smem_bytes<STAGES>();
  static_assert(smem <= 232448, "shared memory of the fused recurrence exceeds 227 KB");
  const long long BT = p->B * p->T;
  const int n = int(p->T / p->C);
  if (n < 2 || !stack || !sched) return ITTT_ERR_INVALID_ARG;
  RecurParams rp{};
  rp.B = int(p->B);
  rp.T = int(p->T);
  rp.C = p->C;
  rp.n = n;
  rp.d = int(p->d);
  rp.f = int(p->f);
  rp.eta = p->eta;
  rp.inv_eta = 1.0f / p->eta;
  rp.s_mtiles = int(cdiv(p->d, 256));
  rp.s_ntiles = int(cdiv(p->f, kRecurBN));
  rp.s_tiles = rp.B * rp.s_mtiles * rp.s_ntiles;
  rp.s_pairs = (rp.s_tiles + 1) / 2;
  rp.s_kb = p->C / 64;
  rp.a_mtiles = int(cdiv(p->C, 256));
  rp.a_ntiles = int(cdiv(p->d, 256));
  rp.a_units = rp.B * n * rp.a_mtiles * rp.a_ntiles;
  rp.a_kb = int(cdiv(p->f, 64));
  rp.stack_slices = rp.B * (n - 1);
  rp.flag_count = rp.B * rp.s_mtiles * (n - 1);
  rp.flag_target = uint32_t(rp.s_ntiles) * 8u;
  rp.w0 = static_cast<const bf16*>(W0);
  rp.sched = sched;
  rp.wait_ns = g_wait_ns.load();
  const bool with_target = Y != nullptr && Wt != nullptr;
  if (with_target) {
    rp.t_units = int(recur_target_units(p));
    rp.t_ntiles = int(cdiv(p->d, 256));
    rp.t_kb = int(cdiv(p->d, 64));
  }
  const uint64_t slices = uint64_t(p->B) * uint64_t(n - 1);
  CUtensorMap mv, mzm, mzk, mw, mw0, ms, mf, mo;
  if (!make_map(&mv, V, p->d, BT, p->d, 64, 64) || !make_map(&mzm, Z, p->f, BT, p->f, 64, 64) ||
      !make_map(&mzk, Z, p->f, BT, p->f, 64, 128) ||
      !make_map(&mw, stack, p->f, slices * p->d, p->f, 64, 128) ||
      !make_map(&mw0, W0, p->f, p->d, p->f, 64, 128) ||
      !make_map_3d(&ms, stack, false, p->f, p->d, slices, 64, 32) ||
      !make_map_3d(&mf, Wf, true, p->f, p->d, p->B, 32, 32) ||
      !make_store_map(&mo, O, p->d, p->C, uint64_t(p->B) * n, p->d, uint64_t(p->C) * p->d))
    return ITTT_ERR_CUDA;
  CUtensorMap my = mv, mwt = mv, mvs = mo;  // stand-ins, never used without target units
  if (with_target && (!make_map(&my, Y, p->d, BT, p->d, 64, 128) ||
                      !make_map(&mwt, Wt, p->d, p->d, p->d, 64, 64) ||
                      !make_store_map(&mvs, V, p->d, BT, 1, p->d, BT * p->d)))
    return ITTT_ERR_CUDA;
  auto kern = tc_recur_kernel<STAGES>;
  static std::atomic<bool> attr_done[kMaxDevices] = {};
  static std::atomic<int> max_clusters[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ITTT_ERR_CUDA;
  if (!attr_done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return ITTT_ERR_CUDA;
    attr_done[dev] = true;
  }
  const int sms = num_sms();
  if (sms <= 0) return ITTT_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = ITTT_PDL;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.blockDim = dim3(192, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (!max_clusters[dev]) {
    cudaLaunchConfig_t q = cfg;
    q.gridDim = dim3(2 * (sms / 2), 1, 1);
    q.attrs = attr + 1;
    q.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, kern, &q) != cudaSuccess || nc <= 0) return ITTT_ERR_CUDA;
    max_clusters[dev] = nc;
  }
  const long long items = (long long)rp.t_units + rp.s_pairs + rp.a_units;
  const int clusters = int(items < max_clusters[dev].load() ? items : max_clusters[dev].load());
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, mv, mzm, mzk, mw, mw0, ms, mf, mo, my, mwt, mvs, rp) != cudaSuccess)
    return ITTT_ERR_CUDA;
  return launch_status();
}

// The chunk recurrence of a bf16 problem once Z and Vhat (clipped if asked)
// are in the workspace laid out by L: O and W_down_final from W_down0.
// Yt, Wt: with L.fused_target, the one-launch recurrence computes V = Yt Wt first.
ittt_status recurrence_bf16(const ittt_problem* p, const Layout& L, char* ws, const void* Z,
                            const void* V, const void* W0, void* O, float* Wf, cudaStream_t st,
                            const void* Yt = nullptr, const void* Wt = nullptr) {
  ittt_status s;
  void* stack = (p->T / p->C > 1 && L.form == ITTT_FORM_PREFIX) ? static_cast<void*>(ws + L.stack)
                                                                 : nullptr;
  if (p->eta == 0.f) {
    const long long df = p->d * p->f;
    broadcast_w0_kernel<<<unsigned(cdiv(df, 256)), 256, 0, st>>>(static_cast<const bf16*>(W0), Wf,
                                                                 df, int(p->B));
    if ((s = launch_status()) != ITTT_OK) return s;
    return apply_bf16(p, Z, W0, nullptr, O, true, st);
  }
  if (L.form == ITTT_FORM_HYBRID) {
    // groups of m chunks: the scan stores each group's starting weight (slice
    // g of the sequence's stack; slice 0 = W_down0), and the dual form runs
    // inside every group, a group being a sequence of G = m C tokens of the
    // same rows (Z, Vhat and O are contiguous per group)
    const int m = hybrid_group(p);
    const long long groups = (p->T / p->C) / m;
    const long long df = p->d * p->f;
    char* stack = ws + L.stack;
    ittt_problem g = *p;
    g.B = p->B * groups;
    g.T = p->T / groups;
    SideStream* ss = nullptr;
    if ((s = side_stream(&ss)) != ITTT_OK) return s;
    if (cudaEventRecord(ss->fork, st) != cudaSuccess ||
        cudaStreamWaitEvent(ss->stream, ss->fork, 0) != cudaSuccess)
      return ITTT_ERR_CUDA;
    SideJoin join(ss, st);
    // high priority: the scan with a snapshot at every group boundary
    if ((s = scan_bf16(p, V, Z, W0, stack, Wf, ss->stream, 0, nullptr, m, int(groups), 1)) != ITTT_OK)
      return s;
    if ((s = join.record()) != ITTT_OK) return s;
    // caller's stream, beside the scan: W_down0 into slice 0 of every sequence
    // and the Gram blocks inside the groups
    for (long long b = 0; b < p->B; ++b)
      if (cudaMemcpyAsync(stack + size_t(b * groups) * size_t(df) * 2, W0, size_t(df) * 2,
                          cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return ITTT_ERR_CUDA;
    void* P = ws + L.gram;
    if ((s = gram_bf16(&g, Z, P, g.T, st)) != ITTT_OK) return s;
    if ((s = join.wait()) != ITTT_OK) return s;
    return dualo_bf16(&g, Z, stack, P, V, O, g.T, st, true);
  }
  if (L.form == ITTT_FORM_DUAL) {
    void* P = ws + L.gram;
    if ((s = gram_bf16(p, Z, P, p->T, st)) != ITTT_OK) return s;
    if ((s = dualo_bf16(p, Z, W0, P, V, O, p->T, st)) != ITTT_OK) return s;
    // W_down_final = W_down0 + eta Vhat^T Z over the whole sequence: the
    // fused scan with one chunk of T tokens
    ittt_problem whole = *p;
    whole.C = static_cast<int32_t>(p->T);
    return scan_bf16(&whole, V, Z, W0, nullptr, Wf, st);
  }
  if (L.fused)  // the work counter and flags were zeroed at the start of the forward
    return recur_fused_bf16(p, V, Z, W0, stack, O, Wf, reinterpret_cast<uint32_t*>(ws + L.sched), st,
                            L.fused_target ? Yt : nullptr, L.fused_target ? Wt : nullptr);
  if (!L.tail_dual) {
    if ((s = scan_bf16(p, V, Z, W0, stack, Wf, st)) != ITTT_OK) return s;
    return apply_bf16(p, Z, W0, stack, O, false, st);
  }
  SideStream* ss = nullptr;
  if ((s = side_stream(&ss)) != ITTT_OK) return s;
  if (cudaEventRecord(ss->fork, st) != cudaSuccess ||
      cudaStreamWaitEvent(ss->stream, ss->fork, 0) != cudaSuccess)
    return ITTT_ERR_CUDA;
  SideJoin join(ss, st);
  // high priority: the fused scan, then the apply of chunks 2..n-1
  // W^(1) is used by no one: chunk 1's output comes from the dual kernels
  if ((s = scan_bf16(p, V, Z, W0, stack, Wf, ss->stream, 2)) != ITTT_OK) return s;
  if ((s = apply_bf16(p, Z, W0, stack, O, false, ss->stream, 2)) != ITTT_OK) return s;
  if ((s = join.record()) != ITTT_OK) return s;
  // caller's stream: O of chunks 0 and 1 by the dual form (needs only Z, Vhat
  // and W_down0), on the SMs the scan's last round leaves free
  void* P = ws + L.gram;
  if ((s = gram_bf16(p, Z, P, 2ll * p->C, st)) != ITTT_OK) return s;
  if ((s = dualo_bf16(p, Z, W0, P, V, O, 2ll * p->C, st)) != ITTT_OK) return s;
  return join.wait();
}

// -------------------------------------------------------------- f32 steps

ittt_status gemm_f32(const GemmF32Args& g, int nz, bool gated, cudaStream_t st) {
  if (nz <= 0 || g.M <= 0 || g.N <= 0) return ITTT_OK;
  dim3 grid(unsigned(cdiv(g.N, F32_TILE)), unsigned(cdiv(g.M, F32_TILE)), unsigned(nz));
  if (grid.y > 65535 || grid.z > 65535) return ITTT_ERR_UNSUPPORTED;
  if (gated)
    gemm_f32_kernel<true><<<grid, 256, 0, st>>>(g);
  else
    gemm_f32_kernel<false><<<grid, 256, 0, st>>>(g);
  return launch_status();
}

ittt_status gated_f32(const ittt_problem* p, const float* H, const float* Wg, const float* Wu,
                      float* Z, cudaStream_t st) {
  GemmF32Args g{};
  g.A = H; g.sAm = p->d; g.sAk = 1;
  g.B = Wg; g.B2 = Wu; g.sBn = p->d; g.sBk = 1;
  g.C = Z; g.sCm = p->f; g.sCn = 1;
  g.M = int(p->B * p->T); g.N = int(p->f); g.K = int(p->d); g.nz2 = 1; g.alpha = 1.f;
  return gemm_f32(g, 1, true, st);
}

ittt_status conv_f32(const ittt_problem* p, const float* X0, const float* Kc, float* Y,
                     cudaStream_t st) {
  const long long rows = p->B * p->T;
  conv_f32_kernel<<<unsigned(cdiv(rows * p->d, 256)), 256, 0, st>>>(X0, Kc, Y, conv_geom(p), int(p->d),
                                                                      p->k, rows);
  return launch_status();
}

ittt_status target_f32(const ittt_problem* p, const float* Y, const float* Wt, float* V,
                       cudaStream_t st) {
  GemmF32Args g{};
  g.A = Y; g.sAm = p->d; g.sAk = 1;
  g.B = Wt; g.sBn = 1; g.sBk = p->d;
  g.C = V; g.sCm = p->d; g.sCn = 1;
  g.M = int(p->B * p->T); g.N = int(p->d); g.K = int(p->d); g.nz2 = 1; g.alpha = 1.f;
  return gemm_f32(g, 1, false, st);
}

ittt_status scan_f32(const ittt_problem* p, const float* V, const float* Z, const float* W0,
                     float* stack, float* Wf, cudaStream_t st) {
  const int n = int(p->T / p->C);
  if (n > 1 && !stack) return ITTT_ERR_INVALID_ARG;
  const long long d = p->d, f = p->f, T = p->T, C = p->C;
  ittt_status s;
  GemmF32Args g{};
  g.sAm = 1; g.sAk = d; g.sBn = 1; g.sBk = f; g.sCm = f; g.sCn = 1;
  g.M = int(d); g.N = int(f); g.K = int(C); g.alpha = p->eta;
  g.sA1 = T * d; g.sB1 = T * f;
  if (n > 1) {  // deltas of chunks 0..n-2 into the stack
    g.A = V; g.B = Z; g.C = stack;
    g.sA2 = C * d; g.sB2 = C * f;
    g.sC1 = (n - 1) * d * f; g.sC2 = d * f;
    g.nz2 = n - 1;
    if ((s = gemm_f32(g, int(p->B) * (n - 1), false, st)) != ITTT_OK) return s;
  }
  // delta of the last chunk into W_final
  g.A = V + (n - 1) * C * d; g.B = Z + (n - 1) * C * f; g.C = Wf;
  g.sA2 = 0; g.sB2 = 0; g.sC1 = d * f; g.sC2 = 0; g.nz2 = 1;
  if ((s = gemm_f32(g, int(p->B), false, st)) != ITTT_OK) return s;
  if (p->clip > 0.f) {  // update-norm clipping of the materialised deltas
    clip_deltas_f32<<<unsigned(p->B * n), 256, 0, st>>>(stack, Wf, d * f, n, p->clip);
    if ((s = launch_status()) != ITTT_OK) return s;
  }
  dim3 grid(unsigned(cdiv(d * f, 256)), unsigned(p->B));
  scan_f32_kernel<<<grid, 256, 0, st>>>(W0, stack, Wf, d * f, n, int(p->B));
  return launch_status();
}

ittt_status apply_f32(const ittt_problem* p, const float* Z, const float* W0, const float* stack,
                      float* O, cudaStream_t st) {
  const int n = int(p->T / p->C);
  if (n > 1 && !stack) return ITTT_ERR_INVALID_ARG;
  const long long d = p->d, f = p->f, T = p->T, C = p->C;
  ittt_status s;
  GemmF32Args g{};
  g.sAm = f; g.sAk = 1; g.sBn = f; g.sBk = 1; g.sCm = d; g.sCn = 1;
  g.M = int(C); g.N = int(d); g.K = int(f); g.alpha = 1.f;
  // chunk 0 of every sequence: W_down0
  g.A = Z; g.sA1 = T * f; g.B = W0; g.sB1 = 0; g.C = O; g.sC1 = T * d; g.nz2 = 1;
  if ((s = gemm_f32(g, int(p->B), false, st)) != ITTT_OK) return s;
  if (n > 1) {
    g.A = Z + C * f; g.sA2 = C * f;
    g.B = stack; g.sB1 = (n - 1) * d * f; g.sB2 = d * f;
    g.C = O + C * d; g.sC2 = C * d;
    g.nz2 = n - 1;
    if ((s = gemm_f32(g, int(p->B) * (n - 1), false, st)) != ITTT_OK) return s;
  }
  return ITTT_OK;
}

// Scratch of ittt_lm_target_noalloc: a file-scope device array instead of a
// caller workspace.  Host code must not pass its name to a kernel (on the host
// it only stands for the symbol); every call looks up the device address with
// cudaGetSymbolAddress on the current device.  The lookup is not cached, so a
// primary context that the application reset and recreated is never handed an
// address of the context before it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ITTT_NOALLOC_SCRATCH_BYTES];

ittt_status noalloc_scratch(void** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return ITTT_ERR_CUDA;
  *out = ptr;
  return ITTT_OK;
}

// ------------------------------------------------------------------ decode

struct DecodeLayout {
  size_t y, v, norm2, delta, wlp, total;
};

DecodeLayout plan_decode(const ittt_problem* p) {
  const size_t es = is_bf16(p) ? 2 : 4;
  const size_t rows = size_t(p->B) * size_t(p->C);
  DecodeLayout L{};
  size_t off = 0;
  L.y = off;
  off += align256(rows * p->d * es);
  L.v = off;
  off += align256(rows * p->d * es);
  L.norm2 = off;
  off += align256(size_t(p->B) * sizeof(float));
  L.delta = off;  // fp32 path: the chunk's delta before it is added
  if (!is_bf16(p)) off += align256(size_t(p->B) * size_t(p->d) * size_t(p->f) * 4);
  L.wlp = off;    // bf16 path: the state rounded to bf16, read by the per-token apply
  if (is_bf16(p)) off += align256(size_t(p->B) * size_t(p->d) * size_t(p->f) * 2);
  L.total = off;
  return L;
}

ittt_status validate_decode(const ittt_problem* p) {
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  if (p->T != p->C || p->B > DECODE_MAX_B) return ITTT_ERR_UNSUPPORTED;
  if (!(p->flags & ITTT_FLAG_PAD_CHUNK_END) || (p->flags & ITTT_FLAG_X0_LOOKAHEAD))
    return ITTT_ERR_UNSUPPORTED;
  return ITTT_OK;
}

// A kernel launch with programmatic stream serialization: its prologue may
// overlap the previous kernel's tail (the kernel waits on griddepcontrol
// before it touches global memory).
template <typename... KArgs, typename... Args>
ittt_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = ITTT_PDL;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) != cudaSuccess)
    return ITTT_ERR_CUDA;
  return launch_status();
}

// Arguments of the vectorised gated GEMV of one decode token.
template <typename T_>
struct GemvArgs {
  const T_ *H, *Wg, *Wu, *X0_tok;
  T_ *z, *X0_dst;
  long long zs, x0s;
  int d, f;
};

// The gated GEMV with the batch size as a template argument.  U hidden units
// per warp: 2 for one or two sequences and 4 for three or four (the token rows
// are read once for every 4 to 8 weight rows), 1 above (the token rows of 5 to
// 8 sequences take enough registers already).
template <typename T_, int NB>
ittt_status gated_gemv_launch(const GemvArgs<T_>& a, cudaStream_t st) {
  constexpr int U = NB <= 2 ? 2 : (NB <= 4 ? 4 : ITTT_GEMV_U_WIDE);
  constexpr int E = Pack16<T_>::E;
  if constexpr (std::is_same<T_, bf16>::value && NB >= ITTT_GEMV_MMA_MIN_B) {
    if (a.d % 32 == 0) {  // the warp-MMA form: 16 hidden units per block of S warps
      constexpr int S = 4;
      const long long blocks = std::max<long long>(cdiv(a.f, 16), cdiv((long long)NB * (a.d / 8), 32 * S));
      return launch_pdl(gated_gemv_mma_kernel<NB, S>, dim3(unsigned(blocks)), dim3(32 * S), st, a.H,
                        a.Wg, a.Wu, a.z, a.zs, a.X0_tok, a.X0_dst, a.x0s, a.d, a.f);
    }
  }
  // enough threads for the hidden units (one warp per U) and the X0 copy
  const long long threads = std::max<long long>(cdiv(a.f, U) * 32, (long long)NB * (a.d / E));
  return launch_pdl(gated_gemv_vec_kernel<T_, NB, U>, dim3(unsigned(cdiv(threads, 64))), dim3(64),
                    st, a.H, a.Wg, a.Wu, a.z, a.zs, a.X0_tok, a.X0_dst, a.x0s, a.d, a.f);
}

template <typename T_>
ittt_status gated_gemv_vec(int nb, const GemvArgs<T_>& a, cudaStream_t st) {
  switch (nb) {
    case 1: return gated_gemv_launch<T_, 1>(a, st);
    case 2: return gated_gemv_launch<T_, 2>(a, st);
    case 3: return gated_gemv_launch<T_, 3>(a, st);
    case 4: return gated_gemv_launch<T_, 4>(a, st);
    case 5: return gated_gemv_launch<T_, 5>(a, st);
    case 6: return gated_gemv_launch<T_, 6>(a, st);
    case 7: return gated_gemv_launch<T_, 7>(a, st);
    case 8: return gated_gemv_launch<T_, 8>(a, st);
  }
  return ITTT_ERR_UNSUPPORTED;
}

template <typename T_, typename WT>
ittt_status decode_token(const ittt_problem* p, int slot, const T_* H_tok, const T_* X0_tok,
                         const T_* Wg, const T_* Wu, const WT* W_state, T_* Z_buf, T_* X0_buf,
                         T_* O_tok, cudaStream_t st) {
  const int nb = int(p->B), d = int(p->d), f = int(p->f), C = p->C;
  T_* z = Z_buf + size_t(slot) * f;
  const long long zs = (long long)C * f;
  constexpr int E = Pack16<T_>::E;
  ittt_status s;
  if (d % E == 0 && aligned16(H_tok) && aligned16(Wg) && aligned16(Wu) && aligned16(X0_tok) &&
      aligned16(X0_buf)) {
    const GemvArgs<T_> a{H_tok, Wg, Wu, X0_tok, z, X0_buf + size_t(slot) * d, zs, (long long)C * d,
                         d, f};
    if ((s = gated_gemv_vec<T_>(nb, a, st)) != ITTT_OK) return s;
  } else {
    // the token's row of the X0 chunk buffer, then the scalar GEMV
    if (cudaMemcpy2DAsync(X0_buf + size_t(slot) * d, size_t(C) * d * sizeof(T_), X0_tok,
                          size_t(d) * sizeof(T_), size_t(d) * sizeof(T_), nb,
                          cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return ITTT_ERR_CUDA;
    gated_gemv_kernel<T_><<<unsigned(cdiv(f, 8)), 256, 0, st>>>(H_tok, Wg, Wu, z, zs, nb, d, f);
    if ((s = launch_status()) != ITTT_OK) return s;
  }
  constexpr int KW = 16 / int(sizeof(WT));  // state elements per 16-byte load
  if (f % KW == 0 && aligned16(W_state) && aligned16(Z_buf)) {
    if (nb == 1)
      return launch_pdl(apply_gemv_vec_kernel<T_, WT, 1>, dim3(unsigned(cdiv(d, 2))), dim3(64), st,
                        static_cast<const T_*>(z), zs, W_state, O_tok, nb, d, f);
    return launch_pdl(apply_gemv_vec_kernel<T_, WT, 4>,
                      dim3(unsigned(cdiv((long long)nb * cdiv(d, 4), 2))), dim3(64), st,
                      static_cast<const T_*>(z), zs, W_state, O_tok, nb, d, f);
  }
  apply_gemv_kernel<T_, WT><<<unsigned(cdiv((long long)nb * d, 8)), 256, 0, st>>>(z, zs, W_state,
                                                                                 O_tok, nb, d, f);
  return launch_status();
}

// After a chunk's last token: W_state += clip(eta Vhat^T Z) of that chunk.
ittt_status decode_update(const ittt_problem* p, const void* conv_kernel, const void* W_target,
                          float* W_state, void* Z_buf, void* X0_buf, char* ws, cudaStream_t st) {
  const DecodeLayout L = plan_decode(p);
  ittt_status s;
  // the chunk as a batch of B one-chunk sequences of C tokens
  ittt_problem q = *p;
  q.T = p->C;
  if (is_bf16(p)) {
    if ((s = conv_bf16(&q, X0_buf, conv_kernel, ws + L.y, st)) != ITTT_OK) return s;
    if ((s = target_gemm_bf16(&q, ws + L.y, W_target, ws + L.v, st)) != ITTT_OK) return s;
    if (q.clip > 0.f && (s = clip_targets_bf16(&q, Z_buf, ws + L.v,
                                               reinterpret_cast<float*>(ws + L.norm2), st)) != ITTT_OK)
      return s;
    // fused scan with one chunk, started from and written back to the fp32 state
    return scan_bf16(&q, ws + L.v, Z_buf, nullptr, nullptr, W_state, st, 0, W_state);
  }
  float* Y = reinterpret_cast<float*>(ws + L.y);
  float* V = reinterpret_cast<float*>(ws + L.v);
  float* D = reinterpret_cast<float*>(ws + L.delta);
  if ((s = conv_f32(&q, static_cast<const float*>(X0_buf), static_cast<const float*>(conv_kernel), Y,
                    st)) != ITTT_OK)
    return s;
  if ((s = target_f32(&q, Y, static_cast<const float*>(W_target), V, st)) != ITTT_OK) return s;
  const long long d = p->d, f = p->f, C = p->C;
  GemmF32Args g{};
  g.A = V; g.sA1 = C * d; g.sAm = 1; g.sAk = d;
  g.B = static_cast<const float*>(Z_buf); g.sB1 = C * f; g.sBn = 1; g.sBk = f;
  g.C = D; g.sC1 = d * f; g.sCm = f; g.sCn = 1;
  g.M = int(d); g.N = int(f); g.K = int(C); g.nz2 = 1; g.alpha = p->eta;
  if ((s = gemm_f32(g, int(p->B), false, st)) != ITTT_OK) return s;
  if (p->clip > 0.f) {
    clip_deltas_f32<<<unsigned(p->B), 256, 0, st>>>(nullptr, D, d * f, 1, p->clip);
    if ((s = launch_status()) != ITTT_OK) return s;
  }
  add_f32_kernel<<<unsigned(cdiv(p->B * d * f, 256)), 256, 0, st>>>(W_state, D, p->B * d * f);
  return launch_status();
}

// -------------------------------------------------------- context parallel

// The forward's workspace (prefix form: Z, Y, Vhat, the segment's weight
// stack) plus the segment's starting fast weight [B, d, f] in the dtype.
struct CpLayout {
  Layout base;
  size_t wstart, total;
};

CpLayout plan_cp(const ittt_problem* p) {
  ittt_problem q = *p;
  q.form = ITTT_FORM_PREFIX;
  CpLayout c{};
  c.base = plan(&q);
  const size_t bdf = size_t(p->B) * size_t(p->d) * size_t(p->f);
  c.wstart = c.base.total;
  c.total = c.wstart + align256(bdf * (is_bf16(p) ? 2 : 4));
  return c;
}

// Z and Vhat of the segment into the workspace; the (clipped) chunk deltas
// summed from zero: S = their total, the weight stack = the running sums
// L_1 .. L_{n-1} before chunks 1 .. n-1.
ittt_status cp_delta(const ittt_problem* p, const void* H, const void* X0, const void* Wg,
                     const void* Wu, const void* Kc, const void* Wt, float* S, char* ws,
                     cudaStream_t st) {
  const CpLayout C = plan_cp(p);
  const Layout& L = C.base;
  ittt_status s;
  const size_t bdf = size_t(p->B) * size_t(p->d) * size_t(p->f);
  const long long n = p->T / p->C;
  void* Z = ws + L.z;
  void* Y = ws + L.y;
  void* V = ws + L.v;
  void* stack = n > 1 ? static_cast<void*>(ws + L.stack) : nullptr;
  if (is_bf16(p)) {
    if ((s = gated_bf16(p, H, Wg, Wu, Z, st)) != ITTT_OK) return s;
    if ((s = conv_bf16(p, X0, Kc, Y, st)) != ITTT_OK) return s;
    if ((s = target_gemm_bf16(p, Y, Wt, V, st)) != ITTT_OK) return s;
    if (p->clip > 0.f && p->eta != 0.f &&
        (s = clip_targets_bf16(p, Z, V, reinterpret_cast<float*>(ws + L.norm2), st)) != ITTT_OK)
      return s;
    if (cudaMemsetAsync(S, 0, bdf * sizeof(float), st) != cudaSuccess) return ITTT_ERR_CUDA;
    if (p->eta == 0.f) {  // no deltas: every running sum is zero
      if (stack && cudaMemsetAsync(stack, 0, bdf * size_t(n - 1) * 2, st) != cudaSuccess)
        return ITTT_ERR_CUDA;
      return ITTT_OK;
    }
    // the fused scan started from the fp32 zeros in S, which it overwrites
    // with the total; the targets already carry the clipping
    return scan_bf16(p, V, Z, nullptr, stack, S, st, 0, S);
  }
  float* fZ = static_cast<float*>(Z);
  float* fY = static_cast<float*>(Y);
  float* fV = static_cast<float*>(V);
  if ((s = gated_f32(p, static_cast<const float*>(H), static_cast<const float*>(Wg),
                     static_cast<const float*>(Wu), fZ, st)) != ITTT_OK)
    return s;
  if ((s = conv_f32(p, static_cast<const float*>(X0), static_cast<const float*>(Kc), fY, st)) != ITTT_OK)
    return s;
  if ((s = target_f32(p, fY, static_cast<const float*>(Wt), fV, st)) != ITTT_OK) return s;
  // the materialised deltas, clipped one by one, summed from zero
  return scan_f32(p, fV, fZ, nullptr, static_cast<float*>(stack), S, st);
}

// O and W_end of the segment from W^start = W_down0 + P: the segment's
// effective weights W^start + L_i in place of the running sums, then the
// apply of every chunk, one sequence at a time (each has its own start).
ittt_status cp_apply(const ittt_problem* p, const void* W0, const float* P, const float* S,
                     void* O, float* W_end, char* ws, cudaStream_t st) {
  const CpLayout L = plan_cp(p);
  ittt_status s;
  const long long df = p->d * p->f;
  const int n = int(p->T / p->C);
  const size_t es = is_bf16(p) ? 2 : 4;
  char* Wst = ws + L.wstart;
  char* stack = n > 1 ? ws + L.base.stack : nullptr;
  if (is_bf16(p)) {
    cp_weights_kernel<bf16, 8><<<unsigned(cdiv(df / 8, 256)), 256, 0, st>>>(
        static_cast<const bf16*>(W0), P, S, reinterpret_cast<bf16*>(Wst), W_end,
        reinterpret_cast<bf16*>(stack), n - 1, df, int(p->B));
  } else {
    cp_weights_kernel<float, 1><<<unsigned(cdiv(df, 256)), 256, 0, st>>>(
        static_cast<const float*>(W0), P, S, reinterpret_cast<float*>(Wst), W_end,
        reinterpret_cast<float*>(stack), n - 1, df, int(p->B));
  }
  if ((s = launch_status()) != ITTT_OK) return s;
  ittt_problem one = *p;
  one.B = 1;
  for (long long b = 0; b < p->B; ++b) {
    const char* Zb = ws + L.base.z + size_t(b) * size_t(p->T) * size_t(p->f) * es;
    const char* Wb = Wst + size_t(b) * size_t(df) * es;
    const char* Sb = stack ? stack + size_t(b) * size_t(n - 1) * size_t(df) * es : nullptr;
    char* Ob = static_cast<char*>(O) + size_t(b) * size_t(p->T) * size_t(p->d) * es;
    if (is_bf16(p))
      s = apply_bf16(&one, Zb, Wb, Sb, Ob, false, st);
    else
      s = apply_f32(&one, reinterpret_cast<const float*>(Zb), reinterpret_cast<const float*>(Wb),
                    reinterpret_cast<const float*>(Sb), reinterpret_cast<float*>(Ob), st);
    if (s != ITTT_OK) return s;
  }
  return ITTT_OK;
}

// ------------------------------------------------------------ timing probe

struct Probe {
  // 4 per call: before and after the gate/up GEMM, before and after the
  // chunk recurrence
  std::vector<cudaEvent_t> ev;
  int calls = 0;                // forwards recorded so far
};

Probe& probe() {
  thread_local Probe pr;
  return pr;
}

void probe_clear() {
  Probe& pr = probe();
  for (cudaEvent_t e : pr.ev) cudaEventDestroy(e);
  pr.ev.clear();
  pr.calls = 0;
}

// The event of this call's `which` point (0 / 1 before / after the gate/up
// GEMM, 2 / 3 before / after the recurrence), or null when the probe is off
// or full.
cudaEvent_t probe_event(int which) {
  Probe& pr = probe();
  const int slot = 4 * pr.calls + which;
  return slot < int(pr.ev.size()) ? pr.ev[slot] : nullptr;
}

ittt_status probe_record(int which, cudaStream_t st) {
  cudaEvent_t e = probe_event(which);
  if (!e) return ITTT_OK;
  if (cudaEventRecord(e, st) != cudaSuccess) return ITTT_ERR_CUDA;
  if (which == 3) probe().calls++;
  return ITTT_OK;
}

// A named NVTX range over a host scope: the launches inside it appear under
// this name in profilers that read NVTX.  With no tool attached a range costs
// a few nanoseconds.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace

// ================================================================= C ABI

extern "C" {

int ittt_version(void) { return 100; }

const char* ittt_status_string(ittt_status s) {
  switch (s) {
    case ITTT_OK: return "ok";
    case ITTT_ERR_INVALID_ARG: return "invalid argument";
    case ITTT_ERR_UNSUPPORTED: return "unsupported problem";
    case ITTT_ERR_WORKSPACE: return "workspace missing or too small";
    case ITTT_ERR_CUDA: return "CUDA error";
    case ITTT_ERR_TIMEOUT: return "device-side wait timed out";
    case ITTT_ERR_DEVICE_FAULT: return "device-side check failed";
  }
  return "unknown status";
}

ittt_status ittt_workspace_size(const ittt_problem* p, size_t* bytes) {
  if (!bytes) return ITTT_ERR_INVALID_ARG;
  const ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  *bytes = plan(p).total;
  return ITTT_OK;
}

ittt_status ittt_resolve_form(const ittt_problem* p, int32_t* form) {
  if (!form) return ITTT_ERR_INVALID_ARG;
  const ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  *form = resolve_form(p);
  return ITTT_OK;
}

ittt_status ittt_gated_activations(const ittt_problem* p, const void* H, const void* W_gate,
                                   const void* W_up, void* Z, void* stream) {
  const NvtxRange nvtx_range("ittt_gated_activations");
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  if (!H || !W_gate || !W_up || !Z) return ITTT_ERR_INVALID_ARG;
  const Sizes z(p);
  if ((s = check_buffers({{H, z.BTd}, {W_gate, z.df}, {W_up, z.df}, {Z, z.BTf}})) != ITTT_OK) return s;
  if (is_bf16(p)) {
    if (!aligned16(H) || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(Z)) return ITTT_ERR_UNSUPPORTED;
    return gated_bf16(p, H, W_gate, W_up, Z, as_stream(stream));
  }
  return gated_f32(p, static_cast<const float*>(H), static_cast<const float*>(W_gate),
                   static_cast<const float*>(W_up), static_cast<float*>(Z), as_stream(stream));
}

ittt_status ittt_lookahead_conv(const ittt_problem* p, const void* X0, const void* conv_kernel,
                                void* Y, void* stream) {
  const NvtxRange nvtx_range("ittt_lookahead_conv");
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  if (!X0 || !conv_kernel || !Y) return ITTT_ERR_INVALID_ARG;
  const Sizes z(p);
  if ((s = check_buffers({{X0, z.BTd / size_t(p->T) * z.Tx}, {conv_kernel, z.dk}, {Y, z.BTd}})) != ITTT_OK)
    return s;
  if (is_bf16(p)) {
    if (!aligned16(X0) || !aligned16(Y) || !aligned16(conv_kernel)) return ITTT_ERR_UNSUPPORTED;
    return conv_bf16(p, X0, conv_kernel, Y, as_stream(stream));
  }
  return conv_f32(p, static_cast<const float*>(X0), static_cast<const float*>(conv_kernel),
                  static_cast<float*>(Y), as_stream(stream));
}

ittt_status ittt_lm_target(const ittt_problem* p, const void* X0, const void* conv_kernel,
                           const void* W_target, void* Vhat, void* workspace,
                           size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("ittt_lm_target");
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  if (!X0 || !conv_kernel || !W_target || !Vhat) return ITTT_ERR_INVALID_ARG;
  const Layout L = plan(p);
  if (!workspace || workspace_bytes < L.total) return ITTT_ERR_WORKSPACE;
  {
    const Sizes z(p);
    if ((s = check_buffers({{X0, z.BTd / size_t(p->T) * z.Tx}, {conv_kernel, z.dk}, {W_target, z.dd},
                            {Vhat, z.BTd}, {workspace, workspace_bytes}})) != ITTT_OK)
      return s;
  }
  char* ws = static_cast<char*>(workspace);
  cudaStream_t st = as_stream(stream);
  if (is_bf16(p)) {
    if (!aligned16(X0) || !aligned16(W_target) || !aligned16(Vhat) || !aligned16(workspace) ||
        !aligned16(conv_kernel))
      return ITTT_ERR_UNSUPPORTED;
    if ((s = conv_bf16(p, X0, conv_kernel, ws + L.y, st)) != ITTT_OK) return s;
    return target_gemm_bf16(p, ws + L.y, W_target, Vhat, st);
  }
  float* Y = reinterpret_cast<float*>(ws + L.y);
  if ((s = conv_f32(p, static_cast<const float*>(X0), static_cast<const float*>(conv_kernel), Y, st)) != ITTT_OK)
    return s;
  return target_f32(p, Y, static_cast<const float*>(W_target), static_cast<float*>(Vhat), st);
}

ittt_status ittt_lm_target_noalloc(const ittt_problem* p, const void* X0, const void* conv_kernel,
                                   const void* W_target, void* Vhat, void* stream) {
  const NvtxRange nvtx_range("ittt_lm_target_noalloc");
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  if (!X0 || !conv_kernel || !W_target || !Vhat) return ITTT_ERR_INVALID_ARG;
  const size_t es = is_bf16(p) ? 2 : 4;
  {
    const Sizes z(p);
    if ((s = check_buffers({{X0, z.BTd / size_t(p->T) * z.Tx}, {conv_kernel, z.dk}, {W_target, z.dd},
                            {Vhat, z.BTd}})) != ITTT_OK)
      return s;
  }
  if (size_t(p->B) * size_t(p->T) * size_t(p->d) * es > size_t(ITTT_NOALLOC_SCRATCH_BYTES))
    return ITTT_ERR_WORKSPACE;
  if (is_bf16(p) && (!aligned16(X0) || !aligned16(W_target) || !aligned16(Vhat) ||
                     !aligned16(conv_kernel)))
    return ITTT_ERR_UNSUPPORTED;
  void* Y = nullptr;
  if ((s = noalloc_scratch(&Y)) != ITTT_OK) return s;
  cudaStream_t st = as_stream(stream);
  if (is_bf16(p)) {
    if ((s = conv_bf16(p, X0, conv_kernel, Y, st)) != ITTT_OK) return s;
    return target_gemm_bf16(p, Y, W_target, Vhat, st);
  }
  float* fY = static_cast<float*>(Y);
  if ((s = conv_f32(p, static_cast<const float*>(X0), static_cast<const float*>(conv_kernel), fY, st)) != ITTT_OK)
    return s;
  return target_f32(p, fY, static_cast<const float*>(W_target), static_cast<float*>(Vhat), st);
}

ittt_status ittt_clip_update_targets(const ittt_problem* p, const void* Z, void* Vhat,
                                     float* norms, void* stream) {
  const NvtxRange nvtx_range("ittt_clip_update_targets");
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  if (!Z || !Vhat || !norms) return ITTT_ERR_INVALID_ARG;
  const long long n = p->T / p->C;
  {
    const Sizes z(p);
    if ((s = check_buffers({{Z, z.BTf}, {Vhat, z.BTd}, {norms, size_t(p->B * n) * 4}})) != ITTT_OK)
      return s;
  }
  cudaStream_t st = as_stream(stream);
  if (is_bf16(p)) {
    if (!aligned16(Z) || !aligned16(Vhat)) return ITTT_ERR_UNSUPPORTED;
    if ((s = clip_targets_bf16(p, Z, Vhat, norms, st)) != ITTT_OK) return s;
  } else {
    if (cudaMemsetAsync(norms, 0, size_t(p->B * n) * sizeof(float), st) != cudaSuccess)
      return ITTT_ERR_CUDA;
    clip_norms_f32<<<unsigned(p->B * n * p->C), 256, 0, st>>>(
        static_cast<const float*>(Z), static_cast<const float*>(Vhat), norms, int(p->T), p->C,
        int(p->d), int(p->f));
    if ((s = launch_status()) != ITTT_OK) return s;
    const long long rows = p->B * p->T;
    clip_scale_rows_f32<<<unsigned(cdiv(rows * p->d, 256)), 256, 0, st>>>(
        static_cast<float*>(Vhat), norms, p->eta, p->clip, int(p->T), p->C, int(p->d), rows);
    if ((s = launch_status()) != ITTT_OK) return s;
  }
  clip_finish_norms<<<unsigned(cdiv(p->B * n, 256)), 256, 0, st>>>(norms, p->eta, int(p->B * n));
  return launch_status();
}

ittt_status ittt_fast_weight_scan(const ittt_problem* p, const void* Vhat, const void* Z,
                                  const void* W_down0, void* W_stack, float* W_down_final,
                                  void* stream) {
  const NvtxRange nvtx_range("ittt_fast_weight_scan");
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  const long long n = p->T / p->C;
  if (!Vhat || !Z || !W_down0 || !W_down_final || (n > 1 && !W_stack)) return ITTT_ERR_INVALID_ARG;
  {
    const Sizes z(p);
    if ((s = check_buffers({{Vhat, z.BTd}, {Z, z.BTf}, {W_down0, z.df},
                            {W_stack, size_t(p->B) * size_t(n - 1) * z.df}, {W_down_final, z.Bdf32}})) !=
        ITTT_OK)
      return s;
  }
  cudaStream_t st = as_stream(stream);
  if (is_bf16(p)) {
    if (!aligned16(Vhat) || !aligned16(Z) || !aligned16(W_down0) || !aligned16(W_down_final) ||
        (W_stack && !aligned16(W_stack)))
      return ITTT_ERR_UNSUPPORTED;
    if (p->eta == 0.f) {
      // no update: every W^(i) is W_down0
      const long long df = p->d * p->f;
      broadcast_w0_kernel<<<unsigned(cdiv(df, 256)), 256, 0, st>>>(
          static_cast<const bf16*>(W_down0), W_down_final, df, int(p->B));
      if ((s = launch_status()) != ITTT_OK) return s;
      for (long long i = 0; i < p->B * (n - 1); ++i)
        if (cudaMemcpyAsync(static_cast<bf16*>(W_stack) + i * df, W_down0, size_t(df) * 2,
                            cudaMemcpyDeviceToDevice, st) != cudaSuccess)
          return ITTT_ERR_CUDA;
      return ITTT_OK;
    }
    return scan_bf16(p, Vhat, Z, W_down0, W_stack, W_down_final, st);
  }
  return scan_f32(p, static_cast<const float*>(Vhat), static_cast<const float*>(Z),
                  static_cast<const float*>(W_down0), static_cast<float*>(W_stack), W_down_final, st);
}

ittt_status ittt_apply(const ittt_problem* p, const void* Z, const void* W_down0,
                       const void* W_stack, void* O, void* stream) {
  const NvtxRange nvtx_range("ittt_apply");
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  const long long n = p->T / p->C;
  if (!Z || !W_down0 || !O || (n > 1 && !W_stack)) return ITTT_ERR_INVALID_ARG;
  {
    const Sizes z(p);
    if ((s = check_buffers({{Z, z.BTf}, {W_down0, z.df},
                            {W_stack, size_t(p->B) * size_t(n - 1) * z.df}, {O, z.BTd}})) != ITTT_OK)
      return s;
  }
  cudaStream_t st = as_stream(stream);
  if (is_bf16(p)) {
    if (!aligned16(Z) || !aligned16(W_down0) || !aligned16(O) || (W_stack && !aligned16(W_stack)))
      return ITTT_ERR_UNSUPPORTED;
    return apply_bf16(p, Z, W_down0, W_stack, O, false, st);
  }
  return apply_f32(p, static_cast<const float*>(Z), static_cast<const float*>(W_down0),
                   static_cast<const float*>(W_stack), static_cast<float*>(O), st);
}

ittt_status ittt_chunk_recurrence(const ittt_problem* p, const void* Z, const void* Vhat,
                                  const void* W_down0, void* O, float* W_down_final,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("ittt_chunk_recurrence");
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  if (!Z || !Vhat || !W_down0 || !O || !W_down_final) return ITTT_ERR_INVALID_ARG;
  const Layout L = plan(p);
  if (!workspace || workspace_bytes < L.total) return ITTT_ERR_WORKSPACE;
  {
    const Sizes z(p);
    if ((s = check_buffers({{Z, z.BTf}, {Vhat, z.BTd}, {W_down0, z.df}, {O, z.BTd},
                            {W_down_final, z.Bdf32}, {workspace, workspace_bytes}})) != ITTT_OK)
      return s;
  }
  char* ws = static_cast<char*>(workspace);
  cudaStream_t st = as_stream(stream);
  if (is_bf16(p)) {
    if (!aligned16(Z) || !aligned16(Vhat) || !aligned16(W_down0) || !aligned16(O) ||
        !aligned16(W_down_final) || !aligned16(workspace))
      return ITTT_ERR_UNSUPPORTED;
    // the step runs the one-launch recurrence whenever it applies, and takes
    // Vhat as given (no target units)
    Layout Ls = L;
    Ls.fused = L.one_launch;
    Ls.tail_dual = L.tail_dual && !Ls.fused;
    Ls.fused_target = false;
    if (Ls.fused && cudaMemsetAsync(ws + L.sched, 0, recur_sched_bytes(p, false), st) != cudaSuccess)
      return ITTT_ERR_CUDA;
    return recurrence_bf16(p, Ls, ws, Z, Vhat, W_down0, O, W_down_final, st);
  }
  float* fS = reinterpret_cast<float*>(ws + L.stack);
  if ((s = scan_f32(p, static_cast<const float*>(Vhat), static_cast<const float*>(Z),
                    static_cast<const float*>(W_down0), fS, W_down_final, st)) != ITTT_OK)
    return s;
  return apply_f32(p, static_cast<const float*>(Z), static_cast<const float*>(W_down0), fS,
                   static_cast<float*>(O), st);
}

ittt_status ittt_fast_mlp_forward(const ittt_problem* p, const void* H, const void* X0,
                                  const void* W_gate, const void* W_up, const void* W_down0,
                                  const void* conv_kernel, const void* W_target, void* O,
                                  float* W_down_final, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  const NvtxRange nvtx_range("ittt_fast_mlp_forward");
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  if (!H || !X0 || !W_gate || !W_up || !W_down0 || !conv_kernel || !W_target || !O || !W_down_final)
    return ITTT_ERR_INVALID_ARG;
  const Layout L = plan(p);
  if (!workspace || workspace_bytes < L.total) return ITTT_ERR_WORKSPACE;
  {
    const Sizes z(p);
    if ((s = check_buffers({{H, z.BTd}, {X0, z.BTd / size_t(p->T) * z.Tx}, {W_gate, z.df},
                            {W_up, z.df}, {W_down0, z.df}, {conv_kernel, z.dk}, {W_target, z.dd},
                            {O, z.BTd}, {W_down_final, z.Bdf32}, {workspace, workspace_bytes}})) !=
        ITTT_OK)
      return s;
  }
  char* ws = static_cast<char*>(workspace);
  void* Z = ws + L.z;
  void* Y = ws + L.y;
  void* V = ws + L.v;
  void* stack = (p->T / p->C > 1 && L.form == ITTT_FORM_PREFIX) ? static_cast<void*>(ws + L.stack)
                                                                 : nullptr;
  cudaStream_t st = as_stream(stream);

  if (is_bf16(p)) {
    const void* ptrs[] = {H, X0, W_gate, W_up, W_down0, conv_kernel, W_target, O, W_down_final,
                          workspace};
    for (const void* q : ptrs)
      if (!aligned16(q)) return ITTT_ERR_UNSUPPORTED;
    // the fused recurrence's work counter and readiness flags start at zero;
    // cleared here, ahead of the kernels, so that the launches from the gate/up
    // GEMM on keep their programmatic overlap
    if (L.fused && cudaMemsetAsync(ws + L.sched, 0, recur_sched_bytes(p, L.fused_target), st) != cudaSuccess)
      return ITTT_ERR_CUDA;
    // the look-ahead conv runs inside the target GEMM's prologue, or inside the
    // gate/up kernel (two extra warps per CTA), for k <= 8; else as its own kernel
    const bool conv_prologue = ITTT_TARGET_CONV && p->k <= 8 && !L.fused_target;
    const bool conv_beside = !conv_prologue && ITTT_CONV_IN_GATED && p->k <= 8;
    const bool conv_side = ITTT_CONV_SIDE && !conv_prologue && !conv_beside;
    // eta folded into Vhat: the steps after the target GEMM see eta = 1
    const bool fold = ITTT_ETA_IN_VHAT && p->eta != 0.f && !conv_prologue && !L.fused_target;
    ittt_problem p_unit = *p;
    if (fold) p_unit.eta = 1.0f;
    const ittt_problem* pe = &p_unit;
    SideStream* cs = nullptr;
    if (conv_side) {
      // forked before the gate/up launch, launched after it: the GEMM's CTAs
      // are placed first, the conv's (lowest priority) go around them
      if ((s = side_stream(&cs)) != ITTT_OK) return s;
      if (cudaEventRecord(cs->low_fork, st) != cudaSuccess ||
          cudaStreamWaitEvent(cs->low, cs->low_fork, 0) != cudaSuccess)
        return ITTT_ERR_CUDA;
    }
    {
      const NvtxRange r("gate_up");
      if ((s = probe_record(0, st)) != ITTT_OK) return s;
      if ((s = conv_beside ? gated_bf16(p, H, W_gate, W_up, Z, st, X0, conv_kernel, Y)
                           : gated_bf16(p, H, W_gate, W_up, Z, st)) != ITTT_OK) {
        if (conv_side) {  // the caller's stream stays ordered after the fork
          cudaEventRecord(cs->low_join, cs->low);
          cudaStreamWaitEvent(st, cs->low_join, 0);
        }
        return s;
      }
      if ((s = probe_record(1, st)) != ITTT_OK) return s;
    }
    const bool target_side = conv_side && ITTT_TARGET_SIDE && !L.fused_target;
    if (conv_side) {
      const NvtxRange r("lookahead_conv");
      const ittt_status cst = conv_bf16(p, X0, conv_kernel, Y, cs->low);
      ittt_status tst = ITTT_OK;
      if (cst == ITTT_OK && target_side)
        tst = target_gemm_bf16(p, Y, W_target, V, cs->low, fold ? p->eta : 1.0f);
      if (cudaEventRecord(cs->low_join, cs->low) != cudaSuccess ||
          cudaStreamWaitEvent(st, cs->low_join, 0) != cudaSuccess)
        return ITTT_ERR_CUDA;
      if (cst != ITTT_OK) return cst;
      if (tst != ITTT_OK) return tst;
    }
    {
      const NvtxRange r("lm_target");
      if (conv_prologue) {
        if ((s = target_conv_bf16(p, X0, conv_kernel, W_target, V, st)) != ITTT_OK) return s;
      } else {
        if (!conv_beside && !conv_side && (s = conv_bf16(p, X0, conv_kernel, Y, st)) != ITTT_OK) return s;
        // with L.fused_target the recurrence's launch computes Vhat
        if (!L.fused_target && !target_side &&
            (s = target_gemm_bf16(p, Y, W_target, V, st, fold ? p->eta : 1.0f)) != ITTT_OK)
          return s;
      }
    }
    if (p->clip > 0.f && p->eta != 0.f) {
      const NvtxRange r("clip");
      if ((s = clip_targets_bf16(pe, Z, V, reinterpret_cast<float*>(ws + L.norm2), st)) != ITTT_OK)
        return s;
    }
    const NvtxRange r("recurrence");
    if ((s = probe_record(2, st)) != ITTT_OK) return s;
    if ((s = recurrence_bf16(pe, L, ws, Z, V, W_down0, O, W_down_final, st,
                             L.fused_target ? Y : nullptr, L.fused_target ? W_target : nullptr)) != ITTT_OK)
      return s;
    return probe_record(3, st);
  }

  const float* f_H = static_cast<const float*>(H);
  float* fZ = static_cast<float*>(Z);
  float* fY = static_cast<float*>(Y);
  float* fV = static_cast<float*>(V);
  float* fS = static_cast<float*>(stack);
  if ((s = probe_record(0, st)) != ITTT_OK) return s;
  if ((s = gated_f32(p, f_H, static_cast<const float*>(W_gate), static_cast<const float*>(W_up), fZ, st)) != ITTT_OK)
    return s;
  if ((s = probe_record(1, st)) != ITTT_OK) return s;
  if ((s = conv_f32(p, static_cast<const float*>(X0), static_cast<const float*>(conv_kernel), fY, st)) != ITTT_OK)
    return s;
  if ((s = target_f32(p, fY, static_cast<const float*>(W_target), fV, st)) != ITTT_OK) return s;
  if ((s = probe_record(2, st)) != ITTT_OK) return s;
  if ((s = scan_f32(p, fV, fZ, static_cast<const float*>(W_down0), fS, W_down_final, st)) != ITTT_OK)
    return s;
  if ((s = apply_f32(p, fZ, static_cast<const float*>(W_down0), fS, static_cast<float*>(O), st)) != ITTT_OK)
    return s;
  return probe_record(3, st);
}

ittt_status ittt_decode_workspace_size(const ittt_problem* p, size_t* bytes) {
  if (!bytes) return ITTT_ERR_INVALID_ARG;
  const ittt_status s = validate_decode(p);
  if (s != ITTT_OK) return s;
  *bytes = plan_decode(p).total;
  return ITTT_OK;
}

ittt_status ittt_decode_step(const ittt_problem* p, int64_t pos, const void* H_tok,
                             const void* X0_tok, const void* W_gate, const void* W_up,
                             const void* conv_kernel, const void* W_target, float* W_state,
                             void* Z_buf, void* X0_buf, void* O_tok, void* workspace,
                             size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("ittt_decode_step");
  ittt_status s = validate_decode(p);
  if (s != ITTT_OK) return s;
  if (pos < 0) return ITTT_ERR_INVALID_ARG;
  if (!H_tok || !X0_tok || !W_gate || !W_up || !conv_kernel || !W_target || !W_state || !Z_buf ||
      !X0_buf || !O_tok)
    return ITTT_ERR_INVALID_ARG;
  const DecodeLayout L = plan_decode(p);
  if (!workspace || workspace_bytes < L.total) return ITTT_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  {
    const Sizes z(p);
    const size_t row = size_t(p->B) * size_t(p->d) * z.es;  // one token of every sequence
    if ((s = check_buffers({{H_tok, row}, {X0_tok, row}, {W_gate, z.df}, {W_up, z.df},
                            {conv_kernel, z.dk}, {W_target, z.dd}, {W_state, z.Bdf32},
                            {Z_buf, z.BTf}, {X0_buf, z.BTd}, {O_tok, row},
                            {workspace, workspace_bytes}})) != ITTT_OK)
      return s;
  }
  const int slot = int(pos % p->C);
  if (is_bf16(p)) {
    const void* ptrs[] = {H_tok, X0_tok, W_gate, W_up, conv_kernel, W_target, W_state, Z_buf, X0_buf,
                          O_tok, workspace};
    for (const void* q : ptrs)
      if (!aligned16(q)) return ITTT_ERR_UNSUPPORTED;
    // the state's bf16 rounding, refreshed at the first token of every chunk
    bf16* wlp = reinterpret_cast<bf16*>(static_cast<char*>(workspace) + L.wlp);
    if (slot == 0) {
      const long long n = p->B * p->d * p->f;
      if ((s = launch_pdl(round_bf16_kernel, dim3(unsigned(cdiv(n / 8, 256))), dim3(256), st,
                          static_cast<const float*>(W_state), wlp, n)) != ITTT_OK)
        return s;
    }
    s = decode_token<bf16, bf16>(p, slot, static_cast<const bf16*>(H_tok),
                                 static_cast<const bf16*>(X0_tok), static_cast<const bf16*>(W_gate),
                                 static_cast<const bf16*>(W_up), wlp, static_cast<bf16*>(Z_buf),
                                 static_cast<bf16*>(X0_buf), static_cast<bf16*>(O_tok), st);
  } else {
    s = decode_token<float, float>(p, slot, static_cast<const float*>(H_tok),
                            static_cast<const float*>(X0_tok), static_cast<const float*>(W_gate),
                            static_cast<const float*>(W_up), W_state, static_cast<float*>(Z_buf),
                            static_cast<float*>(X0_buf), static_cast<float*>(O_tok), st);
  }
  if (s != ITTT_OK) return s;
  if (slot != p->C - 1 || p->eta == 0.f) return ITTT_OK;
  return decode_update(p, conv_kernel, W_target, W_state, Z_buf, X0_buf,
                       static_cast<char*>(workspace), st);
}

ittt_status ittt_cp_workspace_size(const ittt_problem* p, size_t* bytes) {
  if (!bytes) return ITTT_ERR_INVALID_ARG;
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  *bytes = plan_cp(p).total;
  return ITTT_OK;
}

ittt_status ittt_cp_delta(const ittt_problem* p, const void* H, const void* X0,
                          const void* W_gate, const void* W_up, const void* conv_kernel,
                          const void* W_target, float* S, void* workspace,
                          size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("ittt_cp_delta");
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  if (!H || !X0 || !W_gate || !W_up || !conv_kernel || !W_target || !S) return ITTT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < plan_cp(p).total) return ITTT_ERR_WORKSPACE;
  {
    const Sizes z(p);
    if ((s = check_buffers({{H, z.BTd}, {X0, z.BTd / size_t(p->T) * z.Tx}, {W_gate, z.df},
                            {W_up, z.df}, {conv_kernel, z.dk}, {W_target, z.dd}, {S, z.Bdf32},
                            {workspace, workspace_bytes}})) != ITTT_OK)
      return s;
  }
  if (is_bf16(p)) {
    const void* ptrs[] = {H, X0, W_gate, W_up, conv_kernel, W_target, S, workspace};
    for (const void* q : ptrs)
      if (!aligned16(q)) return ITTT_ERR_UNSUPPORTED;
  }
  return cp_delta(p, H, X0, W_gate, W_up, conv_kernel, W_target, S, static_cast<char*>(workspace),
                  as_stream(stream));
}

ittt_status ittt_cp_apply(const ittt_problem* p, const void* W_down0, const float* P,
                          const float* S, void* O, float* W_end, void* workspace,
                          size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx_range("ittt_cp_apply");
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  if (!W_down0 || !P || !S || !O || !W_end) return ITTT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < plan_cp(p).total) return ITTT_ERR_WORKSPACE;
  {
    const Sizes z(p);
    if ((s = check_buffers({{W_down0, z.df}, {P, z.Bdf32}, {S, z.Bdf32}, {O, z.BTd},
                            {W_end, z.Bdf32}, {workspace, workspace_bytes}})) != ITTT_OK)
      return s;
  }
  if (is_bf16(p)) {
    const void* ptrs[] = {W_down0, P, S, O, W_end, workspace};
    for (const void* q : ptrs)
      if (!aligned16(q)) return ITTT_ERR_UNSUPPORTED;
  }
  return cp_apply(p, W_down0, P, S, O, W_end, static_cast<char*>(workspace), as_stream(stream));
}

ittt_status ittt_cp_prefix(const float* S_all, int64_t G, int64_t n, float* P_all, void* stream) {
  const NvtxRange nvtx_range("ittt_cp_prefix");
  if (G < 1 || G > (1ll << 30) || n < 0) return ITTT_ERR_INVALID_ARG;
  if (n == 0) return ITTT_OK;
  if (!S_all || !P_all) return ITTT_ERR_INVALID_ARG;
  const uintptr_t s0 = reinterpret_cast<uintptr_t>(S_all), p0 = reinterpret_cast<uintptr_t>(P_all);
  const uintptr_t bytes = uintptr_t(G) * uintptr_t(n) * sizeof(float);
  if (s0 < p0 + bytes && p0 < s0 + bytes) return ITTT_ERR_INVALID_ARG;  // overlapping
  if (const ittt_status s = check_buffers({{S_all, size_t(bytes)}, {P_all, size_t(bytes)}});
      s != ITTT_OK)
    return s;
  const bool vec = (n % 4 == 0) && aligned16(S_all) && aligned16(P_all);
  const long long threads = vec ? n / 4 : n;
  cp_prefix_kernel<<<unsigned(cdiv(threads, 256)), 256, 0, as_stream(stream)>>>(S_all, P_all, int(G),
                                                                               n, vec);
  return launch_status();
}

ittt_status ittt_check_buffer(const void* ptr, size_t bytes) {
  if (!ptr) return ITTT_ERR_INVALID_ARG;
  AddressRangeFn range = address_range_fn();
  if (!range) return ITTT_ERR_CUDA;
  return buffer_in_allocation(range, ptr, bytes) ? ITTT_OK : ITTT_ERR_INVALID_ARG;
}

ittt_status ittt_set_checks(int level) {
  if (level < 0 || level > 1) return ITTT_ERR_INVALID_ARG;
  g_checks.store(level);
  return ITTT_OK;
}

ittt_status ittt_probe_start(int n) {
  if (n < 1 || n > 65536) return ITTT_ERR_INVALID_ARG;
  probe_clear();
  Probe& pr = probe();
  pr.ev.resize(size_t(4) * n, nullptr);
  for (cudaEvent_t& e : pr.ev)
    if (cudaEventCreate(&e) != cudaSuccess) {
      e = nullptr;
      probe_clear();
      return ITTT_ERR_CUDA;
    }
  return ITTT_OK;
}

ittt_status ittt_probe_read2(float* gate_up_ms, float* recurrence_ms, int capacity, int* got) {
  if (!got || capacity < 0 || (capacity > 0 && (!gate_up_ms && !recurrence_ms)))
    return ITTT_ERR_INVALID_ARG;
  Probe& pr = probe();
  const int n = std::min(pr.calls, capacity);
  ittt_status s = ITTT_OK;
  for (int i = 0; i < n && s == ITTT_OK; ++i) {
    if (cudaEventSynchronize(pr.ev[4 * i + 3]) != cudaSuccess ||
        (gate_up_ms &&
         cudaEventElapsedTime(&gate_up_ms[i], pr.ev[4 * i], pr.ev[4 * i + 1]) != cudaSuccess) ||
        (recurrence_ms &&
         cudaEventElapsedTime(&recurrence_ms[i], pr.ev[4 * i + 2], pr.ev[4 * i + 3]) != cudaSuccess))
      s = ITTT_ERR_CUDA;
  }
  *got = s == ITTT_OK ? n : 0;
  probe_clear();
  return s;
}

ittt_status ittt_probe_read(float* ms, int capacity, int* got) {
  if (!got || capacity < 0 || (capacity > 0 && !ms)) return ITTT_ERR_INVALID_ARG;
  return ittt_probe_read2(ms, nullptr, capacity, got);
}

ittt_status ittt_get_last_error(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return ITTT_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return ITTT_ERR_CUDA;
  int flag = 0;
  if (cudaMemcpyFromSymbol(&flag, g_device_status, sizeof(int)) != cudaSuccess) return ITTT_ERR_CUDA;
  if (flag != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return ITTT_ERR_CUDA;
    return static_cast<ittt_status>(flag);
  }
  return ITTT_OK;
}

ittt_status ittt_set_wait_limit_ns(uint64_t ns) {
  if (ns == 0) return ITTT_ERR_INVALID_ARG;
  g_wait_ns.store(ns);
  return ITTT_OK;
}

ittt_status ittt_selftest_device_check(const ittt_problem* p, const void* Z, const void* W_down0,
                                       const void* W_stack, void* O, void* stream) {
  const NvtxRange nvtx_range("ittt_selftest_device_check");
  ittt_status s = validate(p);
  if (s != ITTT_OK) return s;
  const long long n = p->T / p->C;
  if (!is_bf16(p) || p->B * (n - 1) < 2) return ITTT_ERR_UNSUPPORTED;
  if (!Z || !W_down0 || !W_stack || !O) return ITTT_ERR_INVALID_ARG;
  if (!aligned16(Z) || !aligned16(W_down0) || !aligned16(W_stack) || !aligned16(O))
    return ITTT_ERR_UNSUPPORTED;
  {
    const Sizes z(p);
    if ((s = check_buffers({{Z, z.BTf}, {W_down0, z.df}, {W_stack, size_t(p->B) * size_t(n - 1) * z.df},
                            {O, z.BTd}})) != ITTT_OK)
      return s;
  }
  // the kernel is told the stack holds one slice fewer than it does: the
  // units of the last sequence's last chunk find their slice outside it
  return apply_bf16(p, Z, W_down0, W_stack, O, false, as_stream(stream), 0, p->B * (n - 1) - 1);
}

ittt_status ittt_selftest_wait_timeout(uint64_t ns, void* stream) {
  if (ns == 0 || ns > 10000000000ull) return ITTT_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(ns);
  return launch_status();
}

}  // extern "C"
