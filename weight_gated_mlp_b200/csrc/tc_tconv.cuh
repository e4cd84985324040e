// The LM-aligned target with the look-ahead conv in the GEMM's prologue:
// Vhat = Conv1D(X0) W_target without storing Y (forum summary "Three Core
// Designs" item 3; iplexlaw review section 4).
//
// Same tiles as the target GEMM (TC_TARGET: 256 x 256 output tiles on a
// tensor-core pair, W_target read N-major), but the A operand of every
// 64-channel k-block is made on chip: the producer loads the X0 window of the
// CTA's 128 rows plus the k - 1 rows after them (one TMA box of 136 rows, k <= 9), and
// four converter warps compute the conv of the block into the stage's A tile
// in the 128-byte-swizzled K-major layout the MMA reads.  A tile's Y block is
// an operand of every one of the d / 256 output-column tiles, so the conv is
// recomputed once per column tile.
//
// Roles per CTA (448 threads):
//   warp 0      producer: X0 windows into a 3-deep raw ring, W_target tiles
//               into the STAGES-deep operand ring
//   warp 1      TMEM allocator and MMA issuer (even CTA)
//   warps 2..5  epilogue: Vhat tiles through staging buffers and TMA stores
//   warps 6..13 converters: raw X0 window -> conv -> A tile of the stage
#pragma once

#include "tc_gemm.cuh"

namespace ittt {

struct TconvParams {
  int m_tiles, n_tiles, num_units;
  int M, N;            // B*T rows, d columns
  int num_kb;          // d / 64
  int d, k;
  ConvGeom g;
  const __nv_bfloat16* conv_k;  // [d, k]
  unsigned long long wait_ns;
};

struct TconvShape {
  static constexpr int BM = 128, BK = 64, B_ROWS = 128;
  static constexpr int WROWS = 136;                  // 128 rows + up to 8 look-ahead rows
  static constexpr int A_BYTES = BM * BK * 2;        // 16 KB (converter output)
  static constexpr int B_BYTES = B_ROWS * BK * 2;    // 16 KB (TMA)
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int RAW_BYTES = WROWS * 128;      // 17 KB (TMA)
  static constexpr int RAW_STAGES = 3;
  static constexpr int STAGING_BYTES = 4 * 2 * 4096;
  static constexpr int CTRL_BYTES = 512;
};

template <int STAGES>
constexpr int tconv_smem_bytes() {
  return STAGES * TconvShape::STAGE_BYTES + TconvShape::RAW_STAGES * TconvShape::RAW_BYTES +
         TconvShape::STAGING_BYTES + 1024 + TconvShape::CTRL_BYTES;
}

// KT: conv taps as a compile-time constant (static register indexing of the
// taps), or 0 for any k <= 8 read from the parameters.
template <int STAGES, int KT>
__global__ void __launch_bounds__(448, 1)
    tc_tconv_kernel(const __grid_constant__ CUtensorMap tmX,   // X0 [B*Tx, d], 64 x 144 boxes
                    const __grid_constant__ CUtensorMap tmB,   // W_target [d, d], 64 x 64 boxes
                    const __grid_constant__ CUtensorMap tmF,   // Vhat store [1, B*T, d], 64 x 32
                    const TconvParams p) {
  using S = TconvShape;
  constexpr int BN = 256;
  constexpr uint32_t IDESC = make_idesc_bf16(256, BN, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* raw = smem + STAGES * S::STAGE_BYTES;
  uint8_t* staging = raw + S::RAW_STAGES * S::RAW_BYTES;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(staging + S::STAGING_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* raw_full = empty_bar + STAGES;
  uint64_t* raw_empty = raw_full + S::RAW_STAGES;
  uint64_t* tfull = raw_empty + S::RAW_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* done_bar = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_cta_rank();
  const bool leader = (rank == 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // the producer's expected bytes (W_target tiles of both CTAs) and one
      // arrival from the converters of each CTA (their A tiles are written)
      mbar_init(&full_bar[s], 3);
      mbar_init(&empty_bar[s], 1);
    }
    for (int r = 0; r < S::RAW_STAGES; ++r) {
      mbar_init(&raw_full[r], 1);
      mbar_init(&raw_empty[r], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], 8);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmF);
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
  const int worker = blockIdx.x >> 1, workers = gridDim.x >> 1;
  const int arow = static_cast<int>(rank) * S::BM;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0, rs = 0;
      uint32_t phase = 0, rphase = 0;
      int last_parity[STAGES];
      for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
      int last_rparity[S::RAW_STAGES];
      for (int r = 0; r < S::RAW_STAGES; ++r) last_rparity[r] = -1;
      const int brow = static_cast<int>(rank) * S::B_ROWS;
      bool ok = true;
      for (int u = worker; u < p.num_units && ok; u += workers) {
        const int mt = u % p.m_tiles, nt = u / p.m_tiles;
        const int m0 = mt * 256 + arow;               // first row of this CTA in B*T
        const int b = m0 / p.g.T, t0 = m0 % p.g.T;
        const int xrow = b * p.g.Tx + t0;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          const int kx = kb * S::BK;
          // X0 window of this CTA's rows into the raw ring (this CTA's barrier)
          if (!mbar_wait(&raw_empty[rs], rphase ^ 1, wc)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&raw_full[rs], S::RAW_BYTES);
          last_rparity[rs] = static_cast<int>(rphase);
          tma_load_2d(raw + rs * S::RAW_BYTES, &tmX, &raw_full[rs], kx, xrow);
          if (++rs == S::RAW_STAGES) {
            rs = 0;
            rphase ^= 1;
          }
          // W_target tile into the operand ring (the pair's barrier)
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, wc)) {
            ok = false;
            break;
          }
          uint64_t* fb = &full_bar[stage];
          if (leader) mbar_arrive_expect_tx(fb, 2 * S::B_BYTES);
          last_parity[stage] = static_cast<int>(phase);
          uint8_t* sb = smem + stage * S::STAGE_BYTES + S::A_BYTES;
#pragma unroll
          for (int j = 0; j < S::B_ROWS / 64; ++j)
            tma_load_2d_pair(sb + j * 8192, &tmB, leader_bar(fb), nt * BN + brow + 64 * j, kx);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag) {
        for (int r = 0; r < S::RAW_STAGES; ++r)
          if (last_rparity[r] >= 0) mbar_wait_teardown(&raw_full[r], last_rparity[r], p.wait_ns);
        if (leader)
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
      int it = 0;
      bool ok = true;
      for (int u = worker; u < p.num_units && ok; u += workers) {
        const int slot = it & 1;
        ++it;
        if (!mbar_wait(&tempty[slot], ecount[slot] & 1, wc)) break;
        ecount[slot]++;
        tc_fence_after_sync();
        const uint32_t dtm = tmem_base + static_cast<uint32_t>(slot * BN);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          // the W_target bytes and both CTAs' converted A tiles
          if (!mbar_wait_cluster(&full_bar[stage], phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(smem + stage * S::STAGE_BYTES);
          const uint32_t b_addr = a_addr + S::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < S::BK / 16; ++kk)
            umma_bf16_pair(dtm, make_sdesc_sw128(a_addr + kk * 32, 16, 1024),
                           make_sdesc_sw128(b_addr + kk * 2048, 8192, 1024), IDESC,
                           (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair(cluster_addr(smem_u32(&empty_bar[stage]), 0u));
          umma_commit_pair(cluster_addr(smem_u32(&empty_bar[stage]), 1u));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair(cluster_addr(smem_u32(&tfull[slot]), 0u));
        umma_commit_pair(cluster_addr(smem_u32(&tfull[slot]), 1u));
      }
      umma_commit_pair(cluster_addr(smem_u32(done_bar), 0u));
      mbar_wait_teardown(done_bar, 0, p.wait_ns);
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------ converters
    // thread: 8 channels (chunk g of the k-block) of 4 consecutive rows
    constexpr int RR = 4;
    const int ct = threadIdx.x - 192;           // 0..255
    const int g = ct & 7, rb = ct >> 3;         // channel chunk, row block
    const int r0 = rb * RR;                     // first output row (of 128)
    int stage = 0, rs = 0;
    uint32_t phase = 0, rphase = 0;
    bool ok = true;
    for (int u = worker; u < p.num_units && ok; u += workers) {
      const int mt = u % p.m_tiles;
      const int m0 = mt * 256 + arow;
      const int t0 = m0 % p.g.T;               // token of the CTA's first row
      for (int kb = 0; kb < p.num_kb; ++kb) {
        const int c0 = kb * S::BK + g * 8;     // first channel of this thread
        const int k = KT > 0 ? KT : p.k;
        // taps of channels c0..c0+7: 8k contiguous bf16, k 16-byte loads
        float w[8][8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q >= k) break;
          const uint4 v = c0 < p.d ? __ldg(reinterpret_cast<const uint4*>(p.conv_k + (size_t)c0 * k) + q)
                                   : make_uint4(0u, 0u, 0u, 0u);
          const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv[h]));
            const int e0 = q * 8 + 2 * h;  // element index = channel * k + tap
            w[e0 % k][e0 / k] = f2.x;
            w[(e0 + 1) % k][(e0 + 1) / k] = f2.y;
          }
        }
        bool got = mbar_wait(&raw_full[rs], rphase, wc);
        got = got && mbar_wait(&empty_bar[stage], phase ^ 1, wc);
        if (!got) {
          ok = false;
          break;
        }
        const uint8_t* win = raw + rs * S::RAW_BYTES;
        uint8_t* a_tile = smem + stage * S::STAGE_BYTES;
        uint4 x[RR + 7];
#pragma unroll
        for (int i = 0; i < RR + 7; ++i) {
          const int row = r0 + i;  // window row (128-byte swizzled)
          x[i] = (i < RR + k - 1)
                     ? *reinterpret_cast<const uint4*>(win + row * 128 + ((g ^ (row & 7)) << 4))
                     : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int t = 0; t < RR; ++t) {
          const int row = r0 + t;
          const int tok = t0 + row;
          const int lim = conv_limit(p.g, tok);
          float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (j >= k || tok + j >= lim) break;
            const uint32_t vv[4] = {x[t + j].x, x[t + j].y, x[t + j].z, x[t + j].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv[h]));
              y[2 * h] = fmaf(w[j][2 * h], f2.x, y[2 * h]);
              y[2 * h + 1] = fmaf(w[j][2 * h + 1], f2.y, y[2 * h + 1]);
            }
          }
          uint4 o;
          o.x = pack_bf16x2(y[0], y[1]);
          o.y = pack_bf16x2(y[2], y[3]);
          o.z = pack_bf16x2(y[4], y[5]);
          o.w = pack_bf16x2(y[6], y[7]);
          *reinterpret_cast<uint4*>(a_tile + row * 128 + ((g ^ (row & 7)) << 4)) = o;
        }
        fence_proxy_async_smem();  // the A tile is read by the tensor cores (async proxy)
        asm volatile("bar.sync 1, 256;" ::: "memory");  // the eight converter warps
        if (ct == 0) {
          mbar_arrive_release_cluster(leader_bar(&full_bar[stage]));
          mbar_arrive(&raw_empty[rs]);
        }
        if (++rs == S::RAW_STAGES) {
          rs = 0;
          rphase ^= 1;
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    uint32_t fcount[2] = {0, 0};
    auto release_slot = [&](int slot) {
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_bar(&tempty[slot]));
    };
    release_slot(0);
    release_slot(1);
    uint8_t* my_staging = staging + (warp - 2) * 2 * 4096;
    int staging_idx = 0;
    int it = 0;
    for (int u = worker; u < p.num_units; u += workers) {
      const int mt = u % p.m_tiles, nt = u / p.m_tiles;
      const int slot = it & 1;
      ++it;
      const bool ok = mbar_wait(&tfull[slot], fcount[slot] & 1, wc);
      __syncwarp();
      if (!ok) break;
      fcount[slot]++;
      tc_fence_after_sync();
      const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(slot * BN);
      const int y = mt * 256 + arow + q * 32;
      const int col0 = nt * BN;
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
        uint8_t* buf = my_staging + (staging_idx & 1) * 4096;
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint4 v = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
          *reinterpret_cast<uint4*>(buf + lane * 128 + ((ch ^ (lane & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmF, buf, col0 + c0, y, 0);
          bulk_commit_group();
        }
        ++staging_idx;
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }

  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after_sync();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc<true>(tmem_base, 512);
  }
}

}  // namespace ittt
