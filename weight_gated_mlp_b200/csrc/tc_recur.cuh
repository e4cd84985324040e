// The chunk recurrence of the prefix form in one persistent launch: the fused
// update scan (deltas and their exclusive prefix sum, as TC_SCAN) and the
// apply GEMM (as TC_APPLY) share the GPU through one work queue.
//
// Work items, in queue order:
//   target units (optional) Vhat = Y W_target, 256 tokens x 256 columns
//                (deep-read notes "LM-Aligned 目标函数"), ordered token tile by
//                token tile so that the first chunks' targets are done first;
//   scan pairs   two 256 x 256 output tiles of W (consecutive f-tiles of one
//                d-tile); for every chunk i the accumulator, started at
//                W_down0 / eta, takes Vhat_i^T Z_i, and the epilogue stores
//                W^(i+1) = eta * acc (bf16) into the stack, or W_down_final
//                (fp32) after the last chunk (iplexlaw review, section 6,
//                Algorithm 1 steps 1-3; deep-read notes "Chunk-Wise 更新机制").
//   apply units  O rows of 256 tokens of one chunk i times one 256-wide d-tile:
//                O_i = Z_i W^(i)^T with W^(0) = W_down0 (review sections 3 and
//                6, step 4), ordered d-tile by d-tile, chunks ascending.
// A CTA pair takes the next item from a global counter when it is ready for
// one, so the scan's last, partial round and the apply's tail fill each
// other's idle SMs.  An apply unit of chunk i >= 1 needs W^(i) of its d-tile:
// every epilogue warp of a scan tile raises the flag of (sequence, d-tile,
// chunk) once its TMA stores of that snapshot have completed, and the apply
// producer waits (bounded) until the flag counts every warp of every f-tile.
// Likewise a scan tile's chunk waits for the target units of its rows.
//
// Deadlock freedom: items only wait on flags of items earlier in the queue
// (apply on scan, scan on target; target units wait on nothing), so every
// flag waited on belongs to an item some running CTA has already taken and
// whose loads it has issued (a producer takes its next item only after
// issuing every load of the current one), and that item's own waits are on
// still earlier items.  Residency of the whole grid is not needed.
//
// Roles per CTA (192 threads, one CTA per SM, two CTAs per tensor-core pair):
//   warp 0      producer: takes items (the pair's even CTA) and issues TMA loads
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer (even CTA)
//   warps 2..5  epilogue: accumulator drains, snapshot and output stores
#pragma once

#include "tc_gemm.cuh"

// A scan warp counts a snapshot for the apply this many snapshots after it,
// once its stores have completed (the bulk groups of the D newer snapshots may
// still be in flight), so it never waits on stores issued just before; 0 =
// right after issuing them (the warp waits for their completion).
#ifndef ITTT_RECUR_FLAG_DEPTH
#define ITTT_RECUR_FLAG_DEPTH 4
#endif
// Queue orders (build-time tunables).  Apply units: 0 = d-tile by d-tile,
// chunks ascending within each; 1 = chunk by chunk, all d-tiles of a chunk
// together (a chunk's Z rows are read by all its units while in L2).  Scan
// tiles: 0 = f-tiles fastest (a pair = two f-tiles of one d-tile, a d-tile's
// tiles consecutive); 1 = d-tiles fastest (a pair = two d-tiles of one f-tile).
// 1 = the epilogue loads a following scan pair's accumulators as soon as the
// current pair's last chunk has left each slot (it reads the next item ahead).
#ifndef ITTT_RECUR_EARLY_INIT
#define ITTT_RECUR_EARLY_INIT 1
#endif
#ifndef ITTT_RECUR_APPLY_ORDER
#define ITTT_RECUR_APPLY_ORDER 1
#endif
#ifndef ITTT_RECUR_SCAN_ORDER
#define ITTT_RECUR_SCAN_ORDER 1
#endif

namespace ittt {

struct RecurParams {
  int B, T, C, n;          // n = T / C >= 2
  int d, f;
  float eta, inv_eta;
  int s_mtiles, s_ntiles;  // scan output tiles over d and f (256 each)
  int s_tiles, s_pairs;    // B * s_mtiles * s_ntiles; pairs of consecutive tiles
  int s_kb;                // k-blocks per chunk (C / 64)
  int a_mtiles, a_ntiles;  // apply: 256-row tiles per chunk, 256-wide d-tiles
  int a_units;             // B * n * a_mtiles * a_ntiles
  int a_kb;                // k-blocks over f
  int stack_slices;        // B * (n - 1)
  int flag_count;          // B * s_mtiles * (n - 1)
  uint32_t flag_target;    // epilogue warps that store one d-tile's snapshot
  int t_units;             // target units in the queue (0: Vhat is an input)
  int t_ntiles, t_kb;      // target: 256-wide column tiles over d, k-blocks over d
  const __nv_bfloat16* w0; // W_down0 [d, f]
  uint32_t* sched;         // [0]: item counter; flags from word 64: (b, d-tile, chunk),
                           // then one per target unit
  unsigned long long wait_ns;
};

constexpr int kRecurItemRing = 8;   // items published ahead to the pair's roles
constexpr int kRecurFlagBase = 64;  // first flag word (the counter has its own 256 bytes)
constexpr int kRecurBN = 256;

struct RecurShape {
  static constexpr int BM = 128, BK = 64, B_ROWS = 128;
  static constexpr int A_BYTES = BM * BK * 2;      // 16 KB
  static constexpr int B_BYTES = B_ROWS * BK * 2;  // 16 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TX_BYTES = 2 * STAGE_BYTES;  // both CTAs of the pair
  static constexpr int STAGING_BUFS = 2;
  static constexpr int STAGING_BYTES = 4 * STAGING_BUFS * 4096;
  static constexpr int CTRL_BYTES = 512;
};

template <int STAGES>
constexpr int recur_smem_bytes() {
  return STAGES * RecurShape::STAGE_BYTES + RecurShape::STAGING_BYTES + 1024 + RecurShape::CTRL_BYTES;
}

enum RecurKind { RI_TARGET = 0, RI_SCAN = 1, RI_APPLY = 2 };

struct RecurItem {
  int kind;
  bool scan;
  int t0, ntiles;            // scan: first tile and tiles in the pair (1 or 2)
  int b, chunk, mt, dt;      // apply: sequence, chunk, 256-row tile, d-tile;
                             // target: mt = token tile of B*T, dt = column tile
};

__device__ __forceinline__ RecurItem recur_item(const RecurParams& p, int q) {
  RecurItem it{};
  if (q < p.t_units) {
    it.kind = RI_TARGET;
    it.scan = false;
    it.mt = q / p.t_ntiles;
    it.dt = q % p.t_ntiles;
    return it;
  }
  q -= p.t_units;
  if (q < p.s_pairs) {
    it.kind = RI_SCAN;
    it.scan = true;
    it.t0 = 2 * q;
    it.ntiles = min(2, p.s_tiles - it.t0);
  } else {
    int a = q - p.s_pairs;
    it.kind = RI_APPLY;
    it.scan = false;
    it.mt = a % p.a_mtiles;
    a /= p.a_mtiles;
    if (ITTT_RECUR_APPLY_ORDER == 1) {
      it.dt = a % p.a_ntiles;
      a /= p.a_ntiles;
      it.chunk = a % p.n;
      it.b = a / p.n;
    } else {
      it.chunk = a % p.n;
      a /= p.n;
      it.dt = a % p.a_ntiles;
      it.b = a / p.a_ntiles;
    }
  }
  return it;
}

// scan tile u -> (sequence, d-tile, f-tile); f-tiles fastest so a d-tile's
// tiles are consecutive in the queue
__device__ __forceinline__ void recur_scan_tile(const RecurParams& p, int u, int& b, int& mt, int& nt) {
  if (ITTT_RECUR_SCAN_ORDER == 1) {
    mt = u % p.s_mtiles;
    const int r = u / p.s_mtiles;
    nt = r % p.s_ntiles;
    b = r / p.s_ntiles;
  } else {
    nt = u % p.s_ntiles;
    const int r = u / p.s_ntiles;
    mt = r % p.s_mtiles;
    b = r / p.s_mtiles;
  }
}

template <int STAGES>
__global__ void __launch_bounds__(192, 1)
    tc_recur_kernel(const __grid_constant__ CUtensorMap tmV,    // Vhat [B*T, d], 64 x 64 boxes
                    const __grid_constant__ CUtensorMap tmZm,   // Z [B*T, f], 64 x 64 boxes (scan)
                    const __grid_constant__ CUtensorMap tmZk,   // Z [B*T, f], 64 x 128 boxes (apply)
                    const __grid_constant__ CUtensorMap tmW,    // stack [B(n-1) d, f], 64 x 128 boxes
                    const __grid_constant__ CUtensorMap tmW0,   // W_down0 [d, f], 64 x 128 boxes
                    const __grid_constant__ CUtensorMap tmS,    // stack store [B(n-1), d, f], 64 x 32
                    const __grid_constant__ CUtensorMap tmF,    // W_down_final store [B, d, f] fp32
                    const __grid_constant__ CUtensorMap tmO,    // O store [B n, C, d], 64 x 32
                    const __grid_constant__ CUtensorMap tmY,    // Y [B*T, d], 64 x 128 boxes (target)
                    const __grid_constant__ CUtensorMap tmWt,   // W_target [d, d], 64 x 64 boxes
                    const __grid_constant__ CUtensorMap tmVs,   // Vhat store [1, B*T, d], 64 x 32
                    const RecurParams p) {
  using S = RecurShape;
  constexpr int BN = kRecurBN;
  constexpr uint32_t IDESC_SCAN = make_idesc_bf16(256, BN, true, true);
  constexpr uint32_t IDESC_APPLY = make_idesc_bf16(256, BN, false, false);
  constexpr uint32_t IDESC_TARGET = make_idesc_bf16(256, BN, false, true);
  constexpr int R = kRecurItemRing;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* staging = smem + STAGES * S::STAGE_BYTES;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(staging + S::STAGING_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull = empty_bar + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* tinit = tempty + 2;
  uint64_t* item_full = tinit + 2;
  uint64_t* item_empty = item_full + R;
  uint64_t* done_bar = item_empty + R;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* item_val = const_cast<int*>(abort_flag) + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_cta_rank();
  const bool leader = (rank == 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], 8);
      mbar_init(&tinit[s], 8);
    }
    for (int s = 0; s < R; ++s) {
      mbar_init(&item_full[s], 1);
      // readers of an item: the even CTA's MMA issuer and 4 epilogue warps, the
      // odd CTA's producer and 4 epilogue warps
      mbar_init(&item_empty[s], 10);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmZm);
    prefetch_tmap(&tmZk);
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmW0);
    prefetch_tmap(&tmS);
    prefetch_tmap(&tmF);
    prefetch_tmap(&tmO);
    if (p.t_units > 0) {
      prefetch_tmap(&tmY);
      prefetch_tmap(&tmWt);
      prefetch_tmap(&tmVs);
    }
  }
  if (warp == 1) {
    tmem_alloc<true>(tmem_slot, 512);
    tmem_relinquish<true>();
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after_sync();
  grid_dependency_wait();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl wc{abort_flag, p.wait_ns};
  auto leader_bar = [&](uint64_t* bar) { return cluster_addr(smem_u32(bar), 0u); };
  const int total_items = p.t_units + p.s_pairs + p.a_units;
  uint32_t* flags = p.sched + kRecurFlagBase;
  uint32_t* vflags = flags + p.flag_count;  // one per target unit

  // Reads item number k of this pair from the ring (every role but the even
  // CTA's producer), then frees the ring slot on the even CTA.  Returns false
  // when a wait gave up.
  auto read_item = [&](int k, int& q) -> bool {
    const int slot = k % R;
    if (!mbar_wait_cluster(&item_full[slot], (k / R) & 1, wc)) return false;
    q = *reinterpret_cast<volatile int*>(&item_val[slot]);
    return true;
  };
  auto free_item = [&](int k) {
    const int slot = k % R;
    mbar_arrive_release_cluster(leader_bar(&item_empty[slot]));
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[STAGES];
      for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
      const int arow = static_cast<int>(rank) * S::BM;
      const int brow = static_cast<int>(rank) * S::B_ROWS;
      auto next_stage = [&]() -> uint8_t* {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1, wc)) return nullptr;
        if (leader) mbar_arrive_expect_tx(&full_bar[stage], S::TX_BYTES);
        last_parity[stage] = static_cast<int>(phase);
        return smem + stage * S::STAGE_BYTES;
      };
      auto advance = [&]() {
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      };
      auto load = [&](void* dst, const CUtensorMap* m, int cx, int cy) {
        tma_load_2d_pair(dst, m, leader_bar(&full_bar[stage]), cx, cy);
      };
      bool ok = true;
      for (int k = 0; ok; ++k) {
        int q;
        if (leader) {
          // take the next item and publish it to both CTAs of the pair
          const int slot = k % R;
          if (!mbar_wait_cluster(&item_empty[slot], ((k / R) & 1) ^ 1, wc)) break;
          q = static_cast<int>(atomicAdd(p.sched, 1u));
          if (q > total_items) q = total_items;
          item_val[slot] = q;
          st_shared_cluster_u32(cluster_addr(smem_u32(&item_val[slot]), 1u), static_cast<uint32_t>(q));
          mbar_arrive_release_cluster(cluster_addr(smem_u32(&item_full[slot]), 0u));
          mbar_arrive_release_cluster(cluster_addr(smem_u32(&item_full[slot]), 1u));
        } else {
          if (!read_item(k, q)) break;
          free_item(k);
        }
        if (q >= total_items) break;
        const RecurItem it = recur_item(p, q);
        if (it.scan) {
          for (int i = 0; i < p.n && ok; ++i) {
            for (int s = 0; s < it.ntiles && ok; ++s) {
              int b, mt, nt;
              recur_scan_tile(p, it.t0 + s, b, mt, nt);
              const int m0 = mt * 256 + arow;
              if (p.t_units > 0) {
                // Vhat of this chunk's rows and d-tile: every target unit covering them
                const int r0 = b * p.T + i * p.C, r1 = r0 + p.C - 1;
                for (int tm = r0 / 256; tm <= r1 / 256 && ok; ++tm) {
                  const int vi = tm * p.t_ntiles + mt;
                  if (vi >= p.t_units) {
                    set_device_status(ITTT_ERR_DEVICE_FAULT);
                    *abort_flag = 1;
                    ok = false;
                  } else {
                    ok = flag_wait_geq(vflags + vi, 8u, wc);
                  }
                }
                if (!ok) break;
              }
              for (int kb = 0; kb < p.s_kb; ++kb) {
                uint8_t* sa = next_stage();
                if (!sa) {
                  ok = false;
                  break;
                }
                uint8_t* sb = sa + S::A_BYTES;
                const int krow = b * p.T + i * p.C + kb * S::BK;
                load(sa, &tmV, m0, krow);
                load(sa + 8192, &tmV, m0 + 64, krow);
                load(sb, &tmZm, nt * BN + brow, krow);
                load(sb + 8192, &tmZm, nt * BN + brow + 64, krow);
                advance();
              }
            }
          }
        } else if (it.kind == RI_TARGET) {
          const int m0 = it.mt * 256 + arow;
          for (int kb = 0; kb < p.t_kb; ++kb) {
            uint8_t* sa = next_stage();
            if (!sa) {
              ok = false;
              break;
            }
            uint8_t* sb = sa + S::A_BYTES;
            const int kx = kb * S::BK;
            load(sa, &tmY, kx, m0);
            load(sb, &tmWt, it.dt * BN + brow, kx);
            load(sb + 8192, &tmWt, it.dt * BN + brow + 64, kx);
            advance();
          }
        } else {
          const int m0 = it.mt * 256 + arow;
          int slice = -1;
          if (it.chunk > 0) {
            slice = it.b * (p.n - 1) + it.chunk - 1;
            const int fi = (it.b * p.s_mtiles + it.dt) * (p.n - 1) + it.chunk - 1;
            if (slice >= p.stack_slices || fi >= p.flag_count) {
              // an index outside the stack or the flags: report, load nothing
              set_device_status(ITTT_ERR_DEVICE_FAULT);
              *abort_flag = 1;
              ok = false;
              break;
            }
            // W^(chunk) of this d-tile: every warp of every f-tile has stored it
            if (!flag_wait_geq(flags + fi, p.flag_target, wc)) {
              ok = false;
              break;
            }
          }
          for (int kb = 0; kb < p.a_kb; ++kb) {
            uint8_t* sa = next_stage();
            if (!sa) {
              ok = false;
              break;
            }
            uint8_t* sb = sa + S::A_BYTES;
            const int kx = kb * S::BK;
            load(sa, &tmZk, kx, it.b * p.T + it.chunk * p.C + m0);
            if (slice < 0)
              load(sb, &tmW0, kx, it.dt * BN + brow);
            else
              load(sb, &tmW, kx, slice * p.d + it.dt * BN + brow);
            advance();
          }
        }
      }
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
      uint32_t ecount[2] = {0, 0}, icount[2] = {0, 0};
      int acount = 0;
      bool ok = true;
      auto run = [&](int slot, int nkb, int kind) -> bool {
        const uint32_t dtm = tmem_base + static_cast<uint32_t>(slot * BN);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, wc)) return false;
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(smem + stage * S::STAGE_BYTES);
          const uint32_t b_addr = a_addr + S::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < S::BK / 16; ++kk) {
            if (kind == RI_SCAN) {
              umma_bf16_pair(dtm, make_sdesc_sw128(a_addr + kk * 2048, 8192, 1024),
                             make_sdesc_sw128(b_addr + kk * 2048, 8192, 1024), IDESC_SCAN, 1u);
            } else if (kind == RI_TARGET) {
              umma_bf16_pair(dtm, make_sdesc_sw128(a_addr + kk * 32, 16, 1024),
                             make_sdesc_sw128(b_addr + kk * 2048, 8192, 1024), IDESC_TARGET,
                             (kb > 0 || kk > 0) ? 1u : 0u);
            } else {
              umma_bf16_pair(dtm, make_sdesc_sw128(a_addr + kk * 32, 16, 1024),
                             make_sdesc_sw128(b_addr + kk * 32, 16, 1024), IDESC_APPLY,
                             (kb > 0 || kk > 0) ? 1u : 0u);
            }
          }
          if (ITTT_MCAST_COMMIT) {
            umma_commit_pair_both(smem_u32(&empty_bar[stage]));
          } else {
            umma_commit_pair(cluster_addr(smem_u32(&empty_bar[stage]), 0u));
            umma_commit_pair(cluster_addr(smem_u32(&empty_bar[stage]), 1u));
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        umma_commit_pair(cluster_addr(smem_u32(&tfull[slot]), 0u));
        umma_commit_pair(cluster_addr(smem_u32(&tfull[slot]), 1u));
        return true;
      };
      for (int k = 0; ok; ++k) {
        int q;
        if (!read_item(k, q)) break;
        free_item(k);
        if (q >= total_items) break;
        const RecurItem it = recur_item(p, q);
        if (it.scan) {
          for (int i = 0; i < p.n && ok; ++i) {
            for (int s = 0; s < it.ntiles && ok; ++s) {
              if (!mbar_wait(&tempty[s], ecount[s] & 1, wc)) {
                ok = false;
                break;
              }
              ecount[s]++;
              if (i == 0) {  // the epilogue has loaded W_down0 / eta into the slot
                if (!mbar_wait(&tinit[s], icount[s] & 1, wc)) {
                  ok = false;
                  break;
                }
                icount[s]++;
              }
              tc_fence_after_sync();
              ok = run(s, p.s_kb, RI_SCAN);
            }
          }
        } else {
          const int slot = acount & 1;
          ++acount;
          if (!mbar_wait(&tempty[slot], ecount[slot] & 1, wc)) break;
          ecount[slot]++;
          tc_fence_after_sync();
          ok = run(slot, it.kind == RI_TARGET ? p.t_kb : p.a_kb, it.kind);
        }
      }
      umma_commit_pair(cluster_addr(smem_u32(done_bar), 0u));
      mbar_wait_teardown(done_bar, 0, p.wait_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int row_in_tile = static_cast<int>(rank) * S::BM + r;
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    uint32_t fcount[2] = {0, 0};
    int acount = 0;
    auto release_slot = [&](int slot) {
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_bar(&tempty[slot]));
    };
    release_slot(0);
    release_slot(1);

    uint8_t* my_staging = staging + (warp - 2) * (S::STAGING_BUFS * 4096);
    int staging_idx = 0;
    auto stage_and_store = [&](const uint32_t (&pk)[32], const CUtensorMap* map, int x, int y, int z) {
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

    // W_down0 / eta of scan tile u into accumulator slot `slot`
    auto scan_init = [&](int u, int slot) {
      int b, mt, nt;
      recur_scan_tile(p, u, b, mt, nt);
      (void)b;
      const int row = mt * 256 + row_in_tile;
      const int col0 = nt * BN;
      const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(slot * BN);
      // 128 columns at a time: all sixteen 16-byte loads of a group are in flight
      // together before the first conversion.  The path is chosen for the whole
      // warp (tcgen05.st is a warp-collective instruction: every lane must reach
      // the same one), the edge path masks row by row.
#pragma unroll 1
      for (int g0 = 0; g0 < BN; g0 += 128) {
        if (__all_sync(0xffffffffu, row < p.d && col0 + g0 + 128 <= p.f)) {
          const uint4* src = reinterpret_cast<const uint4*>(p.w0 + (size_t)row * p.f + col0 + g0);
          uint4 w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) w[j] = __ldg(src + j);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t v[32];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t ww[4] = {w[4 * c + j].x, w[4 * c + j].y, w[4 * c + j].z, w[4 * c + j].w};
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ww[h]));
                v[8 * j + 2 * h] = __float_as_uint(f2.x * p.inv_eta);
                v[8 * j + 2 * h + 1] = __float_as_uint(f2.y * p.inv_eta);
              }
            }
            __syncwarp();
            tmem_st32(tbase + g0 + 32 * c, v);
          }
        } else {
#pragma unroll 1
          for (int c0 = g0; c0 < g0 + 128; c0 += 32) {
            uint32_t v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int c = col0 + c0 + j;
              float w = 0.f;
              if (row < p.d && c < p.f) w = __bfloat162float(p.w0[(size_t)row * p.f + c]);
              v[j] = __float_as_uint(w * p.inv_eta);
            }
            __syncwarp();
            tmem_st32(tbase + c0, v);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_bar(&tinit[slot]));
    };

    auto wait_full = [&](int slot) -> bool {
      const bool ok = mbar_wait(&tfull[slot], fcount[slot] & 1, wc);
      __syncwarp();
      if (!ok) return false;
      fcount[slot]++;
      tc_fence_after_sync();
      return true;
    };

    // (lane 0) flags of the last stored snapshots not yet counted, oldest first
    constexpr int FD = ITTT_RECUR_FLAG_DEPTH > 0 ? ITTT_RECUR_FLAG_DEPTH : 1;
    int pending[FD];
    int npend = 0;
    auto signal_flag = [&](int fi) {
      fence_proxy_async_all();
      red_release_gpu_add(flags + fi, 1u);
    };
    auto flush_flag = [&]() {
      if (npend > 0) {
        bulk_wait_group_all();
        for (int j = 0; j < npend; ++j) signal_flag(pending[j]);
        npend = 0;
      }
    };
    const int ywarp = static_cast<int>(rank) * S::BM + q4 * 32;  // first row of this warp's slab
    // the next item, read ahead during a scan pair's last chunk so that a next
    // scan pair's accumulators are loaded as soon as each slot is drained
    int ahead_q = -1;
    bool ahead = false;
    int inited = 0;  // slots of the current item already holding W_down0 / eta
    auto read_next = [&](int k, int& q) -> bool {
      bool ok = true;
      if (lane == 0) {
        ok = read_item(k, q);
        if (ok) free_item(k);
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      q = __shfl_sync(0xffffffffu, q, 0);
      return ok;
    };
    for (int k = 0;; ++k) {
      int q = 0;
      bool ok = true;
      if (ahead) {
        q = ahead_q;
        ahead = false;
      } else {
        ok = read_next(k, q);
        inited = 0;
      }
      if (!ok || q >= total_items) break;
      const RecurItem it = recur_item(p, q);
      if (it.scan) {
        for (int s = 0; s < it.ntiles; ++s)
          if (!(inited & (1 << s))) scan_init(it.t0 + s, s);
        inited = 0;
        for (int i = 0; i < p.n && ok; ++i) {
          for (int s = 0; s < it.ntiles && ok; ++s) {
            int b, mt, nt;
            recur_scan_tile(p, it.t0 + s, b, mt, nt);
            if (!wait_full(s)) {
              ok = false;
              break;
            }
            const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(s * BN);
            const int y = mt * 256 + ywarp;
            const int col0 = nt * BN;
            if (i < p.n - 1) {
              // stack slice of W^(i+1)
              const int z = b * (p.n - 1) + i;
              const bool in_stack = z < p.stack_slices;
              if (!in_stack && lane == 0) set_device_status(ITTT_ERR_DEVICE_FAULT);
              {
                // the whole slot into registers as bf16, handed back before the stores
                uint32_t pk[BN / 64][32];
#pragma unroll
                for (int c = 0; c < BN / 64; ++c) {
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
                release_slot(s);
#pragma unroll
                for (int c = 0; c < BN / 64; ++c)
                  if (in_stack) stage_and_store(pk[c], &tmS, col0 + 64 * c, y, z);
              }
              // count this warp's rows of W^(i+1) for the apply once they are in
              // memory, ITTT_RECUR_FLAG_DEPTH snapshots later (when the stores of
              // the snapshots since then may still be in flight), so the warp never
              // waits on stores it has just issued
              if (lane == 0) {
                const int fi = (b * p.s_mtiles + mt) * (p.n - 1) + i;
                if (fi >= p.flag_count) set_device_status(ITTT_ERR_DEVICE_FAULT);
                if (ITTT_RECUR_FLAG_DEPTH > 0 && in_stack && fi < p.flag_count) {
                  if (npend == FD) {
                    // each snapshot is 4 bulk groups: at most 4 FD pending means
                    // the oldest pending snapshot's stores have completed
                    bulk_wait_group<4 * FD>();
                    signal_flag(pending[0]);
                    for (int j = 1; j < FD; ++j) pending[j - 1] = pending[j];
                    --npend;
                  }
                  pending[npend++] = fi;
                } else {
                  flush_flag();
                  bulk_wait_group_all();
                  if (fi < p.flag_count) signal_flag(fi);
                }
              }
              __syncwarp();
            } else {
              if (lane == 0) flush_flag();  // the last snapshot of the item
#pragma unroll 1
              for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t a[32];
                __syncwarp();
                tmem_ld32(tbase + c0, a);
                tmem_ld_wait();
                if (c0 + 32 == BN) release_slot(s);
                uint32_t pk[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) pk[j] = __float_as_uint(__uint_as_float(a[j]) * p.eta);
                stage_and_store(pk, &tmF, col0 + c0, y, b);
              }
              // slot s is drained for the last time in this item: if the next item
              // is a scan pair, load its tile s's starting value now
              if (ITTT_RECUR_EARLY_INIT) {
                if (!ahead) {
                  if (!read_next(k + 1, ahead_q)) {
                    ok = false;
                    break;
                  }
                  ahead = true;
                }
                if (ahead_q < total_items) {
                  const RecurItem nx = recur_item(p, ahead_q);
                  if (nx.scan && s < nx.ntiles) {
                    scan_init(nx.t0 + s, s);
                    inited |= 1 << s;
                  }
                }
              }
            }
          }
        }
        if (!ok) break;
      } else {
        const int slot = acount & 1;
        ++acount;
        if (!wait_full(slot)) break;
        const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(slot * BN);
        const bool target = it.kind == RI_TARGET;
        const int y = it.mt * 256 + ywarp;
        const int z = target ? 0 : it.b * p.n + it.chunk;
        const int col0 = it.dt * BN;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 64) {
          uint32_t a0[32], a1[32];
          __syncwarp();
          tmem_ld32(tbase + c0, a0);
          tmem_ld32(tbase + c0 + 32, a1);
          tmem_ld_wait();
          if (c0 + 64 == BN) release_slot(slot);
          uint32_t pk[32];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            pk[j] = pack_bf16x2(__uint_as_float(a0[2 * j]), __uint_as_float(a0[2 * j + 1]));
            pk[16 + j] = pack_bf16x2(__uint_as_float(a1[2 * j]), __uint_as_float(a1[2 * j + 1]));
          }
          stage_and_store(pk, target ? &tmVs : &tmO, col0 + c0, y, z);
        }
        if (target && lane == 0) {
          // this warp's rows of the Vhat tile are in memory: count them for the scan
          flush_flag();
          bulk_wait_group_all();
          const int vi = it.mt * p.t_ntiles + it.dt;
          if (vi < p.t_units) {
            fence_proxy_async_all();
            red_release_gpu_add(vflags + vi, 1u);
          } else {
            set_device_status(ITTT_ERR_DEVICE_FAULT);
          }
        }
        __syncwarp();
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }

  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still signal it
  tc_fence_after_sync();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc<true>(tmem_base, 512);
  }
}

}  // namespace ittt
