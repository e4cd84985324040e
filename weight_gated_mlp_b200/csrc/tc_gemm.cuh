// Warp-specialised, persistent tcgen05 GEMM kernels of the bf16 path.
//
// One CTA per SM (192 threads):
//   warp 0      TMA producer: 128-byte-swizzled tiles into a STAGES-deep
//               shared-memory ring (full/empty mbarriers per stage)
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//               (M = 128, N = BN, K = 16 per instruction, fp32 in TMEM)
//   warps 2..5  epilogue: tcgen05.ld from TMEM, fused elementwise work,
//               global stores; warp w reads TMEM lanes 32*(w%4)..+31
// Two TMEM accumulator slots of BN fp32 columns let the epilogue of one
// work unit overlap the main loop of the next.
//
// Kinds (one template instance each):
//   TC_GATED   Z = silu(H W_gate^T) * (H W_up^T): the B tile stacks 128 rows
//              of W_gate over 128 rows of W_up, one N = 256 MMA fills a gate
//              and an up accumulator side by side, the epilogue gates them
//              and writes Z once, in bf16.  (Gated MLP of the deep-read notes,
//              "In-Place 设计".)
//   TC_TARGET  Vhat = Y W_target with W_target read N-major ([K, N] rows).
//              (LM-aligned target, deep-read notes "LM-Aligned 目标函数".)
//   TC_APPLY   O_i = Z_i W^(i)^T for every chunk i with that chunk's weight:
//              W_down0 for i = 0, else slice i-1 of the W stack.  (Apply
//              step, iplexlaw review sections 3 and 6.)
//   TC_SCAN    the update deltas and their exclusive prefix sum fused: for an
//              output tile of W (d-rows x f-cols) the accumulator starts at
//              W_down0 / eta and accumulates Vhat_i^T Z_i chunk after chunk
//              (K = tokens, both operands read M/N-major straight from the
//              row-major Vhat and Z); after chunk i the epilogue writes
//              W^(i+1) = eta * acc (bf16) into the stack, after the last chunk
//              W_down_final (fp32).  Two output tiles are interleaved chunk by
//              chunk so that one tile's snapshot overlaps the other's MMAs.
//              (Algorithm 1 of the iplexlaw review, section 6; update
//              equation of the deep-read notes, "Chunk-Wise 更新机制".)
//   TC_GRAM    dual form, part 1: P[t, s] = eta * (Z_t . Z_s) where the chunk
//              of s precedes the chunk of t, else 0 (bf16, [B, T, T], only
//              the blocks the output GEMM reads are computed and stored).
//   TC_NORM    update-norm clipping: ||Vhat_i^T Z_i||_F^2 of every chunk as
//              sum((Z_i Z_i^T) * (Vhat_i Vhat_i^T)) over pairs of 256-token
//              tiles: slot 0 accumulates a Z gram tile (K = f), slot 1 the
//              matching Vhat gram tile (K = d); the epilogue multiplies them,
//              keeps the entries whose two tokens share a chunk and adds the
//              sums into the chunk's fp32 norm^2 (the review's section 6).
//   TC_DUALO   dual form, part 2: O = Z W_down0^T + P Vhat as one GEMM whose K
//              runs first over f (B = W_down0, K-major) and then over the
//              tokens before the tile's chunk (B = Vhat, N-major).
//              The dual form is the exact rewrite O_i = Z_i W0^T +
//              eta sum_{j<i} (Z_i Z_j^T) Vhat_j of the chunk recurrence.
#pragma once

#include "common.cuh"
#include "simt.cuh"

// L2 prefetch distances (k-blocks) of the streamed operands; build-time
// tunables.  Measured on B200 (qwen3-4b shapes) the prefetch slowed both the
// apply and the scan kernel, so it is off by default.
#ifndef ITTT_APPLY_PREFETCH
#define ITTT_APPLY_PREFETCH 0
#endif
#ifndef ITTT_SCAN_PREFETCH
#define ITTT_SCAN_PREFETCH 0
#endif
// Scan: L2 prefetch of the next chunk's tiles (bit 0: Z, bit 1: Vhat).
#ifndef ITTT_SCAN_PREFETCH_NEXT
#define ITTT_SCAN_PREFETCH_NEXT 0
#endif
// Scan snapshot epilogue: 1 = the whole accumulator slot is read (as bf16,
// into registers) and handed back before any staging or store; 0 = the slot
// is handed back after its last 64-column read, between stores.  Measured on
// B200 (interleaved A/B): 0 is faster, 0.399 vs 0.412 ms at T = 8192, C = 512
// (d = 2560, f = 9728) and 8.67 vs 9.84 ms at T = 131072, C = 256.
#ifndef ITTT_SCAN_DRAIN_FIRST
#define ITTT_SCAN_DRAIN_FIRST 0
#endif
// Scan: 1 = the epilogue loads a CTA's next tile pair's starting values into
// each accumulator slot as soon as the current pair's last chunk has left it;
// 0 = both at the start of the next pair.  Measured with the builds alternated
// launch by launch: 0 is 1% faster for the scan alone at T = 8192, C = 512
// (d = 2560, f = 9728) and the same within noise in whole forwards.
#ifndef ITTT_SCAN_EARLY_INIT
#define ITTT_SCAN_EARLY_INIT 0
#endif
// Scan: 1 = the launch may stage a 64-column piece of a snapshot from all four
// epilogue warps into one 128-row buffer and store it with one TMA instruction
// (instead of four 32-row stores); the host turns it on per launch
// (TcParams::store128, C >= 512).  Off: with the builds alternated launch by
// launch the kernel without this path compiled in was as fast at C = 512 and
// 1024 and 8% faster at C = 256.
#ifndef ITTT_SCAN_STORE128
#define ITTT_SCAN_STORE128 0
#endif
// Staging buffers per epilogue warp of the scan kernel (2 or 4).
#ifndef ITTT_SCAN_STAGING_BUFS
#define ITTT_SCAN_STAGING_BUFS 2
#endif
// 1 = a pair MMA's completion is signalled to the barriers of both CTAs by one
// multicast commit; 0 = two commits, one per CTA.
#ifndef ITTT_MCAST_COMMIT
#define ITTT_MCAST_COMMIT 1
#endif
// Clipping norms: L2 prefetch distance (k-blocks) of the Z and Vhat rows, and
// whether a diagonal tile pair (ti == tj) loads its rows once and feeds them
// to the tensor cores as both operands.
#ifndef ITTT_NORM_PREFETCH
#define ITTT_NORM_PREFETCH 0
#endif
#ifndef ITTT_NORM_SHARE_AB
#define ITTT_NORM_SHARE_AB 1
#endif

namespace ittt {

enum TcKind {
  TC_GATED = 0, TC_TARGET = 1, TC_APPLY = 2, TC_SCAN = 3, TC_GRAM = 4, TC_DUALO = 5, TC_NORM = 6
};

struct TcParams {
  int num_units;   // GATED/TARGET/APPLY: work units; SCAN: output tiles
  int m_tiles;     // 128-row tiles along M
  int n_tiles;     // tiles along N (128 Z columns for GATED, BN otherwise)
  int M, N;        // output extents (APPLY: M = C rows per chunk; SCAN: d x f)
  int num_kb;      // 64-wide k-blocks per unit (SCAN: per chunk)
  int T, C, nchunk;
  float eta, inv_eta;
  int bn;               // GRAM: tile width (s-columns per unit)
  int chunk_base;       // APPLY: first chunk handled
  int chunk_count;      // APPLY: number of chunks handled
  int prow;             // GRAM/DUALO: rows of P per sequence
  int mn3d;             // SCAN: Vhat and Z tiles come as one 3-D box of 64-column blocks each
  float v_scale;        // TARGET: factor applied to the accumulator before the bf16 store
  int store128;         // SCAN: stores of 128-row boxes from pooled staging (ITTT_SCAN_STORE128)
  int snap_from;        // SCAN: snapshots W^(i) with i < snap_from are not stored
  int snap_every;       // SCAN: store W^(i) only for i a multiple of this (0: every i)
  int snap_per_seq;     // SCAN: stack slices per sequence (0: nchunk - 1)
  int snap_first;       // SCAN: stack slice of W^(snap_every) within a sequence
  int group_count;      // DUALO: 0 = first operand W_down0 [d, f]; else the
                        // per-sequence operands [B, d, f] (sequence = group)
  int num_kb2;          // NORM: k-blocks of the Vhat gram (d / 64)
  int group_m;          // GATED / TARGET: m-tiles per rasterisation group (0 = all): the
                        // units of a group (its m-tiles x every n-tile) run together, so
                        // the group's A rows stay in L2 while the column tiles pass
  int stack_slices;     // SCAN / APPLY: d x f slices the W stack holds (its tensor
                        // maps' extent); a unit whose slice index falls outside is
                        // skipped and reported as ITTT_ERR_DEVICE_FAULT
  int dt_count;         // NORM: tile offsets tj - ti tried per tile ti
  float* norm2;         // NORM: [B, n] sums of squares (accumulated)
  __nv_bfloat16* out;   // GATED: Z, TARGET: Vhat, APPLY/DUALO: O, SCAN: W stack, GRAM: P
  long long ldo;        // row stride of `out` in elements
  float* out_f32;       // SCAN: W_down_final [B, d, f]
  const __nv_bfloat16* w0;  // SCAN: W_down0 [d, f]
  const float* w0_f32;      // SCAN: per-sequence fp32 start [B, d, f] instead of w0 (decode)
  unsigned long long wait_ns;
  // GATED: the look-ahead conv Y = Conv1D(X0) computed by two extra warps per
  // CTA beside the GEMM (conv_y == nullptr: none); k <= 8
  const __nv_bfloat16* conv_x0;
  const __nv_bfloat16* conv_k;
  __nv_bfloat16* conv_y;
  ConvGeom conv_g;
  int conv_d, conv_taps, conv_B;
};

// Threads per CTA (at most): producer, MMA issuer and four epilogue warps;
// the gate/up GEMM adds two warps when it runs the look-ahead conv beside it
// (it is launched with 192 threads otherwise).
__host__ __device__ constexpr int tc_threads(int kind) { return kind == TC_GATED ? 256 : 192; }

struct TcUnit {
  int slot;    // TMEM accumulator slot (0/1)
  int b, mt, nt, chunk;
  int kb2;     // DUALO: k-blocks of the P * Vhat segment
  int pair_start;  // SCAN: first unit of a tile pair
  int pair_tiles;  // SCAN: tiles in this pair (1 or 2)
  int pair_tile0;  // SCAN: first tile index of the pair
};

template <int KIND>
__device__ __forceinline__ void tc_decode(const TcParams& p, int u, TcUnit& x) {
  if (KIND == TC_GATED || KIND == TC_TARGET) {
    x.b = 0;
    x.chunk = 0;
    const int gm = (p.group_m > 0 && p.group_m < p.m_tiles) ? p.group_m : p.m_tiles;
    const int per_group = gm * p.n_tiles;
    const int g = u / per_group;
    const int r = u - g * per_group;
    const int rows = min(gm, p.m_tiles - g * gm);  // m-tiles in this group (the last may be short)
    x.mt = g * gm + r % rows;
    x.nt = r / rows;
  } else if (KIND == TC_APPLY) {
    x.mt = u % p.m_tiles;
    int r = u / p.m_tiles;
    x.nt = r % p.n_tiles;
    r /= p.n_tiles;
    x.chunk = p.chunk_base + r % p.chunk_count;
    x.b = r / p.chunk_count;
  } else if (KIND == TC_NORM) {  // mt = tile ti, nt = tile tj = ti + offset
    x.mt = u % p.m_tiles;
    const int r = u / p.m_tiles;
    x.nt = x.mt + r % p.dt_count;
    x.b = r / p.dt_count;
    x.chunk = 0;
  } else {  // SCAN: an output tile; GRAM: nt = s-tile; DUALO: nt = d-tile
    x.mt = u % p.m_tiles;
    int r = u / p.m_tiles;
    x.nt = r % p.n_tiles;
    x.b = r / p.n_tiles;
    x.chunk = 0;
  }
}

// Dual form: tokens [0, s_end) of the sequence precede the chunk of every row
// of the output tile mt, i.e. the start of the chunk of the tile's last row.
__device__ __forceinline__ int dual_s_end(const TcParams& p, int mt, int tile_m) {
  const int last = min(mt * tile_m + tile_m, p.T) - 1;
  return (last / p.C) * p.C;
}

// Calls fn(unit) for every work unit of this CTA (of this CTA pair when
// PAIR), in the one order all roles follow.  fn returns false to stop early.
template <int KIND, bool PAIR, typename Fn>
__device__ __forceinline__ void tc_for_units(const TcParams& p, Fn&& fn) {
  const int worker = PAIR ? (blockIdx.x >> 1) : blockIdx.x;
  const int workers = PAIR ? (gridDim.x >> 1) : gridDim.x;
  constexpr int TILE_M = PAIR ? 256 : 128;
  if (KIND != TC_SCAN) {
    int it = 0;
    for (int u = worker; u < p.num_units; u += workers) {
      TcUnit x;
      tc_decode<KIND>(p, u, x);
      x.kb2 = 0;
      if (KIND == TC_GRAM && x.nt * p.bn >= dual_s_end(p, x.mt, TILE_M)) continue;  // not read
      if (KIND == TC_NORM) {
        // tiles ti <= tj must exist and share a chunk
        if (x.nt >= p.m_tiles) continue;
        const int last_i = min(x.mt * TILE_M + TILE_M, p.T) - 1;
        if ((x.nt * TILE_M) / p.C > last_i / p.C) continue;
        x.kb2 = p.num_kb2;
      }
      if (KIND == TC_DUALO) x.kb2 = dual_s_end(p, x.mt, TILE_M) / 64;
      if (KIND == TC_APPLY && x.chunk > 0 && x.b * (p.nchunk - 1) + x.chunk - 1 >= p.stack_slices) {
        // the unit's weight slice lies outside the stack: no role touches it
        set_device_status(ITTT_ERR_DEVICE_FAULT);
        continue;
      }
      x.slot = it & 1;
      ++it;
      x.pair_start = 0;
      x.pair_tiles = 1;
      x.pair_tile0 = u;
      if (!fn(x)) return;
    }
  } else {
    const int npairs = (p.num_units + 1) >> 1;
    for (int pr = worker; pr < npairs; pr += workers) {
      const int t0 = 2 * pr;
      const int nt = min(2, p.num_units - t0);
      for (int i = 0; i < p.nchunk; ++i) {
        for (int s = 0; s < nt; ++s) {
          TcUnit x;
          tc_decode<KIND>(p, t0 + s, x);
          x.kb2 = 0;
          x.chunk = i;
          x.slot = s;
          x.pair_start = (i == 0 && s == 0);
          x.pair_tiles = nt;
          x.pair_tile0 = t0;
          if (!fn(x)) return;
        }
      }
    }
  }
}

// SCAN: 64 accumulator columns (two 32-column TMEM loads) as 32 packed bf16
// pairs, times eta unless eta is folded into Vhat (SCALE = false).
template <bool SCALE>
__device__ __forceinline__ void scan_pack64(uint32_t (&pk)[32], const uint32_t (&a0)[32],
                                            const uint32_t (&a1)[32], float eta) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float x0 = __uint_as_float(a0[2 * j]), x1 = __uint_as_float(a0[2 * j + 1]);
    const float y0 = __uint_as_float(a1[2 * j]), y1 = __uint_as_float(a1[2 * j + 1]);
    pk[j] = SCALE ? pack_bf16x2(x0 * eta, x1 * eta) : pack_bf16x2(x0, x1);
    pk[16 + j] = SCALE ? pack_bf16x2(y0 * eta, y1 * eta) : pack_bf16x2(y0, y1);
  }
}

// Tile geometry.  A CTA holds 128 rows of A; with PAIR two CTAs (one cluster
// of 2, one tensor-core pair) compute a 256 x BN tile, each CTA holding its
// 128 A rows and half (BN/2) of the B rows.
template <int KIND, int BN, bool PAIR>
struct TcShape {
  static constexpr int BM = 128;                  // A rows per CTA
  static constexpr int TILE_M = PAIR ? 256 : 128; // output rows per tile
  static constexpr int BK = 64;
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // B rows (N extent) per CTA
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TX_BYTES = STAGE_BYTES * (PAIR ? 2 : 1);
  static constexpr bool A_MN = (KIND == TC_SCAN);
  static constexpr bool B_MN = (KIND == TC_SCAN || KIND == TC_TARGET);
  // two accumulator slots of BN fp32 columns, allocated as a power of two
  static constexpr int TMEM_COLS = (2 * BN <= 256) ? 256 : 512;
  // SCAN: per epilogue warp STAGING_BUFS 4 KB staging buffers (32 rows x 128
  // bytes, 128-byte swizzle) feeding TMA stores of the snapshots
  static constexpr int STAGING_BUFS = ITTT_SCAN_STAGING_BUFS;
  // staged TMA stores in the epilogue (every kind but GRAM and NORM)
  static constexpr bool TMA_EPI = (KIND != TC_GRAM && KIND != TC_NORM);
  static_assert(!TMA_EPI || BN % 64 == 0, "TMA-store epilogues work in 64-column pieces");
  static constexpr int STAGING_BYTES = TMA_EPI ? 4 * STAGING_BUFS * 4096 : 0;
  // SCAN with ITTT_SCAN_STORE128 pools the staging space into two 16 KB buffers
  static_assert(KIND != TC_SCAN || !ITTT_SCAN_STORE128 || STAGING_BYTES >= 2 * 128 * 128,
                "two 128-row staging buffers");
  // L2 prefetch distance of the producer, in k-blocks (0 = none)
  static constexpr int PREFETCH = (KIND == TC_APPLY)  ? ITTT_APPLY_PREFETCH
                                  : (KIND == TC_SCAN) ? ITTT_SCAN_PREFETCH
                                  : (KIND == TC_NORM) ? ITTT_NORM_PREFETCH
                                                      : 0;
  // epilogue arrivals that free an accumulator slot: 4 warps per CTA
  static constexpr int EPI_ARRIVALS = PAIR ? 8 : 4;
};

template <int KIND, int BN, int STAGES, bool PAIR>
constexpr int tc_smem_bytes() {
  return STAGES * TcShape<KIND, BN, PAIR>::STAGE_BYTES + TcShape<KIND, BN, PAIR>::STAGING_BYTES +
         1024 /* alignment slack */ + 256;
}

// Bounded wait that ignores the CTA's abort flag (teardown only).
__device__ __forceinline__ bool mbar_wait_teardown(uint64_t* bar, uint32_t parity,
                                                   uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > limit_ns) {
      set_device_status(ITTT_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// ------------------------------------------------------------ epilogue stores

__device__ __forceinline__ void store_bf16_row32(__nv_bfloat16* dst, const float (&v)[32],
                                                 int valid) {
  if (valid >= 32) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 w;
      w.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
      w.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
      w.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
      w.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
      d4[j] = w;
    }
  } else {
    for (int j = 0; j < valid; ++j) dst[j] = __float2bfloat16_rn(v[j]);
  }
}

template <int KIND, int BN, int STAGES, bool PAIR>
__global__ void __launch_bounds__(tc_threads(KIND), 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2,
                   const __grid_constant__ CUtensorMap tmS,   // SCAN: W stack store; DUALO: P
                   const __grid_constant__ CUtensorMap tmF,   // output store map (SCAN: W_down_final)
                   const TcParams p) {
  using S = TcShape<KIND, BN, PAIR>;
  constexpr uint32_t IDESC = make_idesc_bf16(S::TILE_M, BN, S::A_MN, S::B_MN);
  constexpr uint32_t IDESC_BMN = make_idesc_bf16(S::TILE_M, BN, S::A_MN, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* staging = smem + STAGES * S::STAGE_BYTES;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(staging + S::STAGING_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull = empty_bar + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* done_bar = tempty + 2;
  uint64_t* staged_bar = done_bar + 1;  // SCAN, 128-row stores: buffer written by all 4 warps
  uint64_t* sfree_bar = staged_bar + 2;  // SCAN, 128-row stores: buffer read by its TMA store
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sfree_bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // rank inside the tensor-core pair (0 = the CTA that issues the MMAs)
  const uint32_t rank = PAIR ? cluster_cta_rank() : 0u;
  const bool leader = (rank == 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], S::EPI_ARRIVALS);
    }
    mbar_init(done_bar, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&staged_bar[s], 4);
      mbar_init(&sfree_bar[s], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (KIND == TC_GATED || KIND == TC_APPLY || KIND == TC_DUALO || KIND == TC_NORM)
      prefetch_tmap(&tmB2);
    if (KIND == TC_DUALO || KIND == TC_SCAN || KIND == TC_NORM) prefetch_tmap(&tmS);
    if (S::TMA_EPI) prefetch_tmap(&tmF);
  }
  if (warp == 1) {
    tmem_alloc<PAIR>(tmem_slot, S::TMEM_COLS);
    tmem_relinquish<PAIR>();
  }
  tc_fence_before_sync();
  __syncthreads();
  if (PAIR) cluster_sync_all();  // the peer's barriers exist before anyone signals them
  tc_fence_after_sync();
  // everything above overlaps the previous kernel's tail; nothing below reads
  // or writes global memory before that kernel has finished
  grid_dependency_wait();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl wc{abort_flag, p.wait_ns};
  // cluster addresses of the leader's and this CTA's barriers (PAIR)
  auto leader_bar = [&](uint64_t* bar) { return cluster_addr(smem_u32(bar), 0u); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[STAGES];
      for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
      const int arow = static_cast<int>(rank) * S::BM;      // this CTA's A rows in the tile
      const int brow = static_cast<int>(rank) * S::B_ROWS;  // this CTA's B rows in the tile
      tc_for_units<KIND, PAIR>(p, [&](const TcUnit& x) -> bool {
        const int nkb = p.num_kb + x.kb2;
        // NORM, diagonal tile pair: the B rows are the A rows, loaded once
        const bool share_ab = KIND == TC_NORM && ITTT_NORM_SHARE_AB && x.nt == x.mt;
        const uint32_t tx = share_ab ? uint32_t(S::A_BYTES * (PAIR ? 2 : 1)) : uint32_t(S::TX_BYTES);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, wc)) return false;
          uint64_t* fb = &full_bar[stage];
          if (leader) mbar_arrive_expect_tx(fb, tx);
          last_parity[stage] = static_cast<int>(phase);
          uint8_t* sa = smem + stage * S::STAGE_BYTES;
          uint8_t* sb = sa + S::A_BYTES;
          const int kx = kb * S::BK;
          const uint32_t fbc = PAIR ? leader_bar(fb) : 0u;
          auto load = [&](void* dst, const CUtensorMap* m, int cx, int cy) {
            if (PAIR)
              tma_load_2d_pair(dst, m, fbc, cx, cy);
            else
              tma_load_2d(dst, m, fb, cx, cy);
          };
          const int m0 = x.mt * S::TILE_M + arow;
          if (KIND == TC_GATED) {
            load(sa, &tmA, kx, m0);
            if (!PAIR) {
              load(sb, &tmB, kx, x.nt * 128);
              load(sb + 128 * S::BK * 2, &tmB2, kx, x.nt * 128);
            } else {
              // the pair's N = 256: gate rows in the even CTA, up rows in the odd one
              load(sb, leader ? &tmB : &tmB2, kx, x.nt * 128);
            }
          } else if (KIND == TC_TARGET) {
            load(sa, &tmA, kx, m0);
#pragma unroll
            for (int j = 0; j < S::B_ROWS / 64; ++j) load(sb + j * 8192, &tmB, x.nt * BN + brow + 64 * j, kx);
          } else if (KIND == TC_APPLY) {
            load(sa, &tmA, kx, x.b * p.T + x.chunk * p.C + m0);
            if (x.chunk == 0) {
              load(sb, &tmB2, kx, x.nt * BN + brow);
            } else {
              const int slice = x.b * (p.nchunk - 1) + (x.chunk - 1);
              load(sb, &tmB, kx, slice * p.N + x.nt * BN + brow);
            }
          } else if (KIND == TC_GRAM) {
            load(sa, &tmA, kx, x.b * p.T + m0);
            load(sb, &tmB, kx, x.b * p.T + x.nt * BN + brow);
          } else if (KIND == TC_NORM) {
            if (kb < p.num_kb) {  // Z rows of tiles ti (A) and tj (B), K = f
              load(sa, &tmA, kx, x.b * p.T + m0);
              if (!share_ab) load(sb, &tmB, kx, x.b * p.T + x.nt * S::TILE_M + brow);
            } else {              // Vhat rows, K = d
              const int k2 = (kb - p.num_kb) * S::BK;
              load(sa, &tmB2, k2, x.b * p.T + m0);
              if (!share_ab) load(sb, &tmS, k2, x.b * p.T + x.nt * S::TILE_M + brow);
            }
          } else if (KIND == TC_DUALO) {
            if (kb < p.num_kb) {  // Z_tile * W_start^T (W_down0, or the group's start)
              load(sa, &tmA, kx, x.b * p.T + m0);
              load(sb, &tmB, kx, (p.group_count ? x.b * p.N : 0) + x.nt * BN + brow);
            } else {              // P_tile * Vhat (Vhat read N-major)
              const int k2 = (kb - p.num_kb) * S::BK;
              load(sa, &tmS, k2, x.b * p.prow + m0);
#pragma unroll
              for (int j = 0; j < S::B_ROWS / 64; ++j)
                load(sb + j * 8192, &tmB2, x.nt * BN + brow + 64 * j, x.b * p.T + k2);
            }
          } else {  // SCAN
            const int krow = x.b * p.T + x.chunk * p.C + kx;
            if (PAIR && p.mn3d) {
              // [64-column block][64 tokens][64 columns] boxes: the same
              // shared-memory image as the 2-D loads below, in two instructions
              tma_load_3d_pair(sa, &tmA, fbc, 0, krow, m0 >> 6);
              tma_load_3d_pair(sb, &tmB, fbc, 0, krow, (x.nt * BN + brow) >> 6);
            } else {
              load(sa, &tmA, m0, krow);
              load(sa + 8192, &tmA, m0 + 64, krow);
#pragma unroll
              for (int j = 0; j < S::B_ROWS / 64; ++j) load(sb + j * 8192, &tmB, x.nt * BN + brow + 64 * j, krow);
            }
          }
          if (S::PREFETCH > 0 && kb + S::PREFETCH < nkb) {
            const int kp = (kb + S::PREFETCH) * S::BK;
            if (KIND == TC_APPLY) {
              tma_prefetch_l2_2d(&tmA, kp, x.b * p.T + x.chunk * p.C + m0);
              if (x.chunk > 0)
                tma_prefetch_l2_2d(&tmB, kp, (x.b * (p.nchunk - 1) + x.chunk - 1) * p.N + x.nt * BN + brow);
            } else if (KIND == TC_SCAN) {
              const int krow = x.b * p.T + x.chunk * p.C + kp;
              tma_prefetch_l2_2d(&tmA, m0, krow);
              tma_prefetch_l2_2d(&tmA, m0 + 64, krow);
#pragma unroll
              for (int j = 0; j < S::B_ROWS / 64; ++j) tma_prefetch_l2_2d(&tmB, x.nt * BN + brow + 64 * j, krow);
            } else if (KIND == TC_NORM) {
              const int kbp = kb + S::PREFETCH;
              const CUtensorMap* ma = kbp < p.num_kb ? &tmA : &tmB2;
              const CUtensorMap* mb = kbp < p.num_kb ? &tmB : &tmS;
              const int kc = (kbp < p.num_kb ? kbp : kbp - p.num_kb) * S::BK;
              tma_prefetch_l2_2d(ma, kc, x.b * p.T + m0);
              if (!share_ab) tma_prefetch_l2_2d(mb, kc, x.b * p.T + x.nt * S::TILE_M + brow);
            }
          }
          if (KIND == TC_SCAN && ITTT_SCAN_PREFETCH_NEXT && x.chunk + 1 < p.nchunk) {
            // the same k-block of this tile's next chunk, about two units ahead
            const int krow = x.b * p.T + (x.chunk + 1) * p.C + kx;
            if (ITTT_SCAN_PREFETCH_NEXT & 1) {
#pragma unroll
              for (int j = 0; j < S::B_ROWS / 64; ++j) tma_prefetch_l2_2d(&tmB, x.nt * BN + brow + 64 * j, krow);
            }
            if (ITTT_SCAN_PREFETCH_NEXT & 2) {
              tma_prefetch_l2_2d(&tmA, m0, krow);
              tma_prefetch_l2_2d(&tmA, m0 + 64, krow);
            }
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        return true;
      });
      if (*abort_flag && leader) {
        // let loads already issued land before the CTA's shared memory goes away
        for (int s = 0; s < STAGES; ++s)
          if (last_parity[s] >= 0) mbar_wait_teardown(&full_bar[s], last_parity[s], p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t ecount[2] = {0, 0};
      tc_for_units<KIND, PAIR>(p, [&](const TcUnit& x) -> bool {
        // NORM units fill both slots (Z gram in 0, Vhat gram in 1)
        for (int sl = (KIND == TC_NORM ? 0 : x.slot); sl <= (KIND == TC_NORM ? 1 : x.slot); ++sl) {
          if (!mbar_wait(&tempty[sl], ecount[sl] & 1, wc)) return false;
          ecount[sl]++;
        }
        tc_fence_after_sync();
        const int nkb = p.num_kb + x.kb2;
        for (int kb = 0; kb < nkb; ++kb) {
          const bool second = (KIND == TC_NORM && kb >= p.num_kb);
          const uint32_t dtm = tmem_base + static_cast<uint32_t>((KIND == TC_NORM ? (second ? 1 : 0) : x.slot) * BN);
          const int kb_local = second ? kb - p.num_kb : kb;
          if (!mbar_wait(&full_bar[stage], phase, wc)) return false;
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(smem + stage * S::STAGE_BYTES);
          const bool share_ab = KIND == TC_NORM && ITTT_NORM_SHARE_AB && x.nt == x.mt;
          const uint32_t b_addr = share_ab ? a_addr : a_addr + S::A_BYTES;
          // DUALO switches B from K-major (W_down0) to N-major (Vhat) after f
          const bool b_mn = S::B_MN || (KIND == TC_DUALO && kb >= p.num_kb);
          const uint32_t idesc = b_mn ? IDESC_BMN : IDESC;
#pragma unroll
          for (int kk = 0; kk < S::BK / 16; ++kk) {
            const uint64_t ad = S::A_MN ? make_sdesc_sw128(a_addr + kk * 2048, 8192, 1024)
                                        : make_sdesc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = b_mn ? make_sdesc_sw128(b_addr + kk * 2048, 8192, 1024)
                                     : make_sdesc_sw128(b_addr + kk * 32, 16, 1024);
            const uint32_t acc = (KIND == TC_SCAN || kb_local > 0 || kk > 0) ? 1u : 0u;
            if (PAIR)
              umma_bf16_pair(dtm, ad, bd, idesc, acc);
            else
              umma_bf16(dtm, ad, bd, idesc, acc);
          }
          if (PAIR) {
            // both CTAs' stages are free once these MMAs complete
            if (ITTT_MCAST_COMMIT) {
              umma_commit_pair_both(smem_u32(&empty_bar[stage]));
            } else {
              umma_commit_pair(cluster_addr(smem_u32(&empty_bar[stage]), 0u));
              umma_commit_pair(cluster_addr(smem_u32(&empty_bar[stage]), 1u));
            }
          } else {
            umma_commit(&empty_bar[stage]);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
          if (KIND == TC_NORM && kb == p.num_kb - 1) {  // the Z gram tile is complete
            if (PAIR) {
              umma_commit_pair(cluster_addr(smem_u32(&tfull[0]), 0u));
              umma_commit_pair(cluster_addr(smem_u32(&tfull[0]), 1u));
            } else {
              umma_commit(&tfull[0]);
            }
          }
        }
        const int done_slot = KIND == TC_NORM ? 1 : x.slot;
        if (PAIR) {
          umma_commit_pair(cluster_addr(smem_u32(&tfull[done_slot]), 0u));
          umma_commit_pair(cluster_addr(smem_u32(&tfull[done_slot]), 1u));
        } else {
          umma_commit(&tfull[done_slot]);
        }
        return true;
      });
      // every MMA issued above has completed once done_bar flips
      if (PAIR)
        umma_commit_pair(cluster_addr(smem_u32(done_bar), 0u));
      else
        umma_commit(done_bar);
      mbar_wait_teardown(done_bar, 0, p.wait_ns);
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------ conv (GATED)
    // Y = Conv1D(X0) in pieces of 8 tokens x 8 channels, spread over every
    // CTA's two conv warps; it needs nothing the GEMM makes and the target GEMM
    // that reads Y runs after this kernel
    if (KIND == TC_GATED && p.conv_y != nullptr) {
      const int nthreads = static_cast<int>(gridDim.x) * 64;
      const int tid = static_cast<int>(blockIdx.x) * 64 + (warp - 6) * 32 + lane;
      const int groups = p.conv_d / 8;
      const int runs = (p.conv_g.T + 7) / 8;
      const long long tasks = (long long)p.conv_B * runs * groups;
      for (long long task = tid; task < tasks; task += nthreads) {
        const int grp = static_cast<int>(task % groups);
        const long long r = task / groups;
        conv_piece_bf16<8, 8>(p.conv_x0, p.conv_k, p.conv_y, p.conv_g, p.conv_d, p.conv_taps,
                              static_cast<int>(r / runs), static_cast<int>(r % runs) * 8, grp);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;  // accumulator row of this thread within this CTA
    const int row_in_tile = static_cast<int>(rank) * S::BM + r;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    uint32_t fcount[2] = {0, 0};
    // free an accumulator slot: one arrival per warp on the MMA-issuing CTA's barrier
    auto release_slot = [&](int slot) {
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (PAIR)
          mbar_arrive_cluster(leader_bar(&tempty[slot]));
        else
          mbar_arrive(&tempty[slot]);
      }
    };

    if (KIND != TC_SCAN) {
      release_slot(0);
      release_slot(1);
    }

    // SCAN: write one 32-row x 128-byte piece (this thread's row = lane) into
    // the warp's next staging buffer in the 128-byte-swizzled layout and store
    // it with TMA at (x, y, z).  The warp's buffers are used round robin; a
    // buffer is rewritten only after the TMA store issued from it has read it.
    uint8_t* my_staging = staging + (warp - 2) * (S::STAGING_BUFS * 4096);
    int staging_idx = 0;
    auto stage_and_store = [&](const uint32_t (&pk)[32], const CUtensorMap* map, int x, int y,
                               int z) {
      uint8_t* buf = my_staging + (staging_idx % S::STAGING_BUFS) * 4096;
      if (lane == 0) bulk_wait_group_read<S::STAGING_BUFS - 1>();
      __syncwarp();
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint4 v = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        *reinterpret_cast<uint4*>(buf + lane * 128 + ((ch ^ (lane & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(map, buf, x, y, z);
        bulk_commit_group();
      }
      ++staging_idx;
    };

    // SCAN with ITTT_SCAN_STORE128: the four epilogue warps write their 32 rows
    // of a piece into one 128-row staging buffer (two buffers, the warps'
    // staging space pooled) and warp 2's lane 0 stores it with one TMA
    // instruction.  Per buffer, staged_bar counts the four warps' writes and
    // sfree_bar the read of its previous store; every wait is bounded, and a
    // failed one ends the epilogue (the CTA's abort path).
    int piece_idx = 0;
    auto stage_and_store128 = [&](const uint32_t (&pk)[32], const CUtensorMap* map, int x, int y,
                                  int z) -> bool {
      const int k = piece_idx & 1;
      const uint32_t use = static_cast<uint32_t>(piece_idx >> 1);  // uses of buffer k before this one
      uint8_t* buf = staging + k * (128 * 128);
      const bool issuer = (warp == 2);
      // the store issued from this buffer two pieces ago has read it
      bool ok = mbar_wait(&sfree_bar[k], (use & 1u) ^ 1u, wc);
      __syncwarp();
      if (!ok) return false;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint4 v = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        *reinterpret_cast<uint4*>(buf + r * 128 + ((ch ^ (r & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&staged_bar[k]);
      if (issuer) {
        ok = mbar_wait(&staged_bar[k], use & 1u, wc);
        __syncwarp();
        if (!ok) return false;
        if (lane == 0) {
          tma_store_3d(map, buf, x, y, z);
          bulk_commit_group();
          // all but this store have read their buffers: the other buffer is free
          bulk_wait_group_read<1>();
          if (piece_idx > 0) mbar_arrive(&sfree_bar[k ^ 1]);
        }
        __syncwarp();
      }
      ++piece_idx;
      return true;
    };

    // SCAN: every store of the kernel (snapshots and W_down_final) goes one way
    // or the other, so the two staging schemes never share a buffer.
    // y_warp: first row of this warp's 32; y_cta: first row of the CTA's 128.
    auto scan_store = [&](const uint32_t (&pk)[32], const CUtensorMap* map, int x, int y_warp,
                          int y_cta, int z) -> bool {
      if (ITTT_SCAN_STORE128 && p.store128) return stage_and_store128(pk, map, x, y_cta, z);
      stage_and_store(pk, map, x, y_warp, z);
      return true;
    };

    // SCAN: load W_down0 / eta of `tile` into accumulator slot `slot`.
    auto scan_init = [&](int tile, int slot) {
      TcUnit t;
      tc_decode<KIND>(p, tile, t);
      const int row = t.mt * S::TILE_M + row_in_tile;
      const int col0 = t.nt * BN;
      const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(slot * BN);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        if (p.w0_f32 != nullptr) {  // per-sequence fp32 start (decode state)
          const float* src = p.w0_f32 + ((size_t)t.b * p.M + row) * (size_t)p.N + col0 + c0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float w = (row < p.M && col0 + c0 + j < p.N) ? src[j] : 0.f;
            v[j] = __float_as_uint(w * p.inv_eta);
          }
        } else if (row < p.M && col0 + c0 + 32 <= p.N) {
          const uint4* src = reinterpret_cast<const uint4*>(p.w0 + (size_t)row * p.N + col0 + c0);
          uint4 wv[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) wv[j] = __ldg(src + j);  // all four loads in flight
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 w = wv[j];
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&ww[h]);
              const float2 f2 = __bfloat1622float2(b2);
              v[8 * j + 2 * h] = __float_as_uint(f2.x * p.inv_eta);
              v[8 * j + 2 * h + 1] = __float_as_uint(f2.y * p.inv_eta);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int c = col0 + c0 + j;
            float w = 0.f;
            if (row < p.M && c < p.N) w = __bfloat162float(p.w0[(size_t)row * p.N + c]);
            v[j] = __float_as_uint(w * p.inv_eta);
          }
        }
        __syncwarp();
        tmem_st32(tbase + c0, v);
      }
      tmem_st_wait();
      release_slot(slot);
    };

    tc_for_units<KIND, PAIR>(p, [&](const TcUnit& x) -> bool {
      if (KIND == TC_SCAN && x.pair_start) {
        // (with ITTT_SCAN_EARLY_INIT the slots of every pair but a CTA's first
        // were loaded as the previous pair's last chunk left them)
        const bool first_pair = x.pair_tile0 / 2 < (PAIR ? (gridDim.x >> 1) : gridDim.x);
        if (!ITTT_SCAN_EARLY_INIT || first_pair)
          for (int s = 0; s < x.pair_tiles; ++s) scan_init(x.pair_tile0 + s, s);
      }
      if (KIND == TC_NORM) {
        bool ok = true;
        for (int sl = 0; sl < 2; ++sl) {
          ok = ok && mbar_wait(&tfull[sl], fcount[sl] & 1, wc);
          fcount[sl]++;
        }
        __syncwarp();
        if (!ok) return false;
        tc_fence_after_sync();
        const int t = x.mt * S::TILE_M + row_in_tile;  // token of this row (tile ti)
        const int tchunk = t / p.C;
        // columns (tokens of tile tj) in this row's chunk and in the sequence
        const int col_lo = tchunk * p.C - x.nt * S::TILE_M;
        const int col_hi = min(tchunk * p.C + p.C, p.T) - x.nt * S::TILE_M;
        float part = 0.f;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t gz[32], gv[32];
          __syncwarp();
          tmem_ld32(tmem_base + lane_addr + c0, gz);
          tmem_ld32(tmem_base + lane_addr + BN + c0, gv);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int c = c0 + j;
            const float g = __uint_as_float(gz[j]) * __uint_as_float(gv[j]);
            part += (c >= col_lo && c < col_hi) ? g : 0.f;
          }
        }
        release_slot(0);
        release_slot(1);
        // off-diagonal tile pairs stand for both (ti, tj) and (tj, ti)
        if (t < p.T && part != 0.f)
          atomicAdd(p.norm2 + (size_t)x.b * p.nchunk + tchunk, (x.nt == x.mt ? 1.f : 2.f) * part);
        return true;
      }
      const bool ok = mbar_wait(&tfull[x.slot], fcount[x.slot] & 1, wc);
      __syncwarp();
      if (!ok) return false;
      fcount[x.slot]++;
      tc_fence_after_sync();
      const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(x.slot * BN);

      if (KIND == TC_GATED) {
        // Z = silu(gate) * up of this warp's 32 rows, 64 columns at a time,
        // through the staging buffers and TMA stores (rows and columns past
        // the end of Z are not written)
        const int y = x.mt * S::TILE_M + static_cast<int>(rank) * S::BM + q * 32;
        const int col0 = x.nt * 128;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 64) {
          uint32_t pk[32];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t g[32], u[32];
            __syncwarp();
            tmem_ld32(tbase + c0 + 32 * h, g);
            tmem_ld32(tbase + 128 + c0 + 32 * h, u);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pk[16 * h + j] = pack_bf16x2(silu_f32(__uint_as_float(g[2 * j])) * __uint_as_float(u[2 * j]),
                                           silu_f32(__uint_as_float(g[2 * j + 1])) * __uint_as_float(u[2 * j + 1]));
          }
          if (c0 + 64 == 128) release_slot(x.slot);  // every TMEM read of the unit is done
          stage_and_store(pk, &tmF, col0 + c0, y, 0);
        }
      } else if (KIND == TC_GRAM) {
        const int t = x.mt * S::TILE_M + row_in_tile;  // token of this row
        const int tchunk = t / p.C;
        const int col0 = x.nt * BN;
        __nv_bfloat16* dst = p.out + ((size_t)x.b * p.prow + t) * (size_t)p.ldo + col0;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t a[32];
          __syncwarp();
          tmem_ld32(tbase + c0, a);
          tmem_ld_wait();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int s_tok = col0 + c0 + j;
            v[j] = (s_tok / p.C < tchunk) ? __uint_as_float(a[j]) * p.eta : 0.f;
          }
          const int valid = min(32, p.N - (col0 + c0));
          if (t < p.M && valid > 0) store_bf16_row32(dst + c0, v, valid);
        }
      } else if (KIND == TC_TARGET || KIND == TC_APPLY || KIND == TC_DUALO) {
        // bf16 store of the tile through staging + TMA; the store map clips
        // rows outside the tile's chunk / sequence and columns past N
        const int y = x.mt * S::TILE_M + static_cast<int>(rank) * S::BM + q * 32;
        const int z = KIND == TC_APPLY ? x.b * p.nchunk + x.chunk : (KIND == TC_DUALO ? x.b : 0);
        const int col0 = x.nt * BN;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 64) {
          uint32_t a0[32], a1[32];
          __syncwarp();
          tmem_ld32(tbase + c0, a0);
          tmem_ld32(tbase + c0 + 32, a1);
          tmem_ld_wait();
          if (c0 + 64 == BN) release_slot(x.slot);
          uint32_t pk[32];
          if (KIND == TC_TARGET) {
            scan_pack64<true>(pk, a0, a1, p.v_scale);  // Vhat, times eta when the forward folds it in
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              pk[j] = pack_bf16x2(__uint_as_float(a0[2 * j]), __uint_as_float(a0[2 * j + 1]));
              pk[16 + j] = pack_bf16x2(__uint_as_float(a1[2 * j]), __uint_as_float(a1[2 * j + 1]));
            }
          }
          stage_and_store(pk, &tmF, col0 + c0, y, z);
        }
      } else {  // SCAN snapshot after chunk x.chunk, stored through smem by TMA
        const int y = x.mt * S::TILE_M + static_cast<int>(rank) * S::BM + q * 32;  // first d-row of the slab
        const int y128 = x.mt * S::TILE_M + static_cast<int>(rank) * S::BM;       // first d-row of the CTA
        const int col0 = x.nt * BN;                                               // first f-column
        const int every = p.snap_every > 0 ? p.snap_every : 1;
        if (x.chunk + 1 < p.snap_from || (x.chunk + 1) % every != 0) {
          // nobody reads this W^(chunk+1): nothing to store, just free the slot
          release_slot(x.slot);
        } else if (x.chunk != p.nchunk - 1) {
          // stack slice of W^(chunk+1)
          const int per_seq = p.snap_per_seq > 0 ? p.snap_per_seq : p.nchunk - 1;
          const int z = x.b * per_seq + p.snap_first + (x.chunk + 1) / every - 1;
          const bool in_stack = z >= 0 && z < p.stack_slices;
          if (!in_stack && lane == 0) set_device_status(ITTT_ERR_DEVICE_FAULT);
          if (ITTT_SCAN_DRAIN_FIRST) {
            // read the whole slot into registers as bf16 first and hand it back to
            // the MMA issuer, then stage and store: the next chunk's MMAs on this
            // slot do not wait for the stores
            constexpr int NP = BN / 64;
            uint32_t pk[NP][32];
#pragma unroll
            for (int c = 0; c < NP; ++c) {
              uint32_t a0[32], a1[32];
              __syncwarp();
              tmem_ld32(tbase + 64 * c, a0);
              tmem_ld32(tbase + 64 * c + 32, a1);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                pk[c][j] = pack_bf16x2(__uint_as_float(a0[2 * j]) * p.eta, __uint_as_float(a0[2 * j + 1]) * p.eta);
                pk[c][16 + j] = pack_bf16x2(__uint_as_float(a1[2 * j]) * p.eta, __uint_as_float(a1[2 * j + 1]) * p.eta);
              }
            }
            release_slot(x.slot);
#pragma unroll
            for (int c = 0; c < NP; ++c)
              if (in_stack && !scan_store(pk[c], &tmS, col0 + 64 * c, y, y128, z)) return false;
          } else {
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 64) {
              uint32_t a0[32], a1[32];
              __syncwarp();
              tmem_ld32(tbase + c0, a0);
              tmem_ld32(tbase + c0 + 32, a1);
              tmem_ld_wait();
              // every TMEM read of this snapshot is done: the slot can take the next chunk
              if (c0 + 64 == BN) release_slot(x.slot);
              uint32_t pk[32];
              // eta == 1: Vhat came scaled by eta (the forward), the multiply is skipped
              if (p.eta == 1.0f)
                scan_pack64<false>(pk, a0, a1, p.eta);
              else
                scan_pack64<true>(pk, a0, a1, p.eta);
              if (in_stack && !scan_store(pk, &tmS, col0 + c0, y, y128, z)) return false;
            }
          }
        } else {
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 32) {
            uint32_t a[32];
            __syncwarp();
            tmem_ld32(tbase + c0, a);
            tmem_ld_wait();
            uint32_t pk[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) pk[j] = __float_as_uint(__uint_as_float(a[j]) * p.eta);
            if (!scan_store(pk, &tmF, col0 + c0, y, y128, x.b)) return false;
          }
          if (ITTT_SCAN_EARLY_INIT) {
            // the slot is drained for good: load the CTA's next pair's tile of
            // this slot now (the MMA issuer can start on it while the other
            // slot's last chunk is still being drained)
            const int next_t0 = x.pair_tile0 + 2 * (PAIR ? (gridDim.x >> 1) : gridDim.x);
            if (next_t0 + x.slot < p.num_units) scan_init(next_t0 + x.slot, x.slot);
          }
        }
      }
      // accumulator slot drained: hand it back to the MMA issuer
      if (!S::TMA_EPI) release_slot(x.slot);
      return true;
    });
    if (S::TMA_EPI && lane == 0) bulk_wait_group_all();
  }

  tc_fence_before_sync();
  __syncthreads();
  if (PAIR) cluster_sync_all();  // no CTA leaves while its peer may still signal it
  tc_fence_after_sync();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc<PAIR>(tmem_base, S::TMEM_COLS);
  }
}

}  // namespace ittt
