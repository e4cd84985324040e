// CUDA-core kernels: the fp32 path (FFMA GEMMs, for the 1e-5 tolerance that
// tensor-core TF32 cannot meet), the depthwise look-ahead convolution in
// bf16 and fp32, and small elementwise helpers.
#pragma once

#include "common.cuh"

namespace ittt {

// ----------------------------------------------------------------------------
// fp32 tiled GEMM with two-level batching and arbitrary element strides:
//   C(z, m, n) = alpha * sum_k A(z, m, k) * B(z, n, k)
// z = z1 * nz2 + z2; operand offsets are z1 * s1 + z2 * s2.
// GATED = true computes C = silu(A Bg^T) * (A Bu^T) with B2 as the up weight.
// ----------------------------------------------------------------------------
struct GemmF32Args {
  const float* A;
  long long sA1, sA2, sAm, sAk;
  const float* B;
  const float* B2;
  long long sB1, sB2, sBn, sBk;
  float* C;
  long long sC1, sC2, sCm, sCn;
  int M, N, K, nz2;
  float alpha;
  int accumulate;  // 1: C += alpha * acc, 0: C = alpha * acc
};

constexpr int F32_TILE = 64;
constexpr int F32_KT = 16;

template <bool GATED>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const GemmF32Args g) {
  __shared__ float As[F32_KT][F32_TILE + 4];
  __shared__ float Bs[F32_KT][F32_TILE + 4];
  __shared__ float Us[GATED ? F32_KT : 1][F32_TILE + 4];

  const int z = blockIdx.z;
  const int z1 = z / g.nz2, z2 = z % g.nz2;
  const float* A = g.A + z1 * g.sA1 + z2 * g.sA2;
  const float* B = g.B + z1 * g.sB1 + z2 * g.sB2;
  const float* B2 = GATED ? g.B2 + z1 * g.sB1 + z2 * g.sB2 : nullptr;
  float* C = g.C + z1 * g.sC1 + z2 * g.sC2;

  const int m0 = blockIdx.y * F32_TILE, n0 = blockIdx.x * F32_TILE;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  float accu[GATED ? 4 : 1][GATED ? 4 : 1] = {};

  for (int k0 = 0; k0 < g.K; k0 += F32_KT) {
    for (int e = threadIdx.x; e < F32_KT * F32_TILE; e += 256) {
      const int kk = e / F32_TILE, mm = e % F32_TILE;
      const int m = m0 + mm, n = n0 + mm, k = k0 + kk;
      As[kk][mm] = (m < g.M && k < g.K) ? A[m * g.sAm + k * g.sAk] : 0.f;
      Bs[kk][mm] = (n < g.N && k < g.K) ? B[n * g.sBn + k * g.sBk] : 0.f;
      if (GATED) Us[kk][mm] = (n < g.N && k < g.K) ? B2[n * g.sBn + k * g.sBk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < F32_KT; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      if (GATED) {
        float u[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) u[j] = Us[kk][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) accu[i][j] = fmaf(a[i], u[j], accu[i][j]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < g.M && n < g.N) {
        float v;
        if (GATED) {
          const float x = acc[i][j];
          v = (x / (1.0f + expf(-x))) * accu[i][j];
        } else {
          v = g.alpha * acc[i][j];
          if (g.accumulate) v += C[m * g.sCm + n * g.sCn];
        }
        C[m * g.sCm + n * g.sCn] = v;
      }
    }
}

// ----------------------------------------------------------------------------
// Exclusive prefix sum over chunks (fp32 path), in place.
// On entry stack[b][j] holds delta_j for j = 0..n-2 and W_final[b] holds
// delta_{n-1}; on exit stack[b][i-1] = W0 + sum_{j<i} delta_j (i = 1..n-1)
// and W_final[b] = W0 + sum_{j<n} delta_j.
// ----------------------------------------------------------------------------
__global__ void scan_f32_kernel(const float* __restrict__ W0, float* __restrict__ stack,
                                float* __restrict__ W_final, long long df, int nchunk, int nb) {
  const long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  if (e >= df || b >= nb) return;
  float acc = W0 ? W0[e] : 0.f;  // no W0: the sum of the deltas alone
  float* s = stack + (long long)b * (nchunk - 1) * df + e;
  for (int i = 0; i < nchunk - 1; ++i) {
    acc += s[i * df];
    s[i * df] = acc;
  }
  W_final[(long long)b * df + e] = acc + W_final[(long long)b * df + e];
}

// ----------------------------------------------------------------------------
// Depthwise look-ahead convolution, Y[t, c] = sum_j K[c, j] * X0[t + j, c].
// ConvGeom: output row (b, t) = b * T + t reads X0 rows b * Tx + t + j for
// t + j < limit(t), X0 being zero beyond: limit = Tx (sequence-end padding;
// Tx = T, or T + k - 1 when X0 carries the next segment's first k - 1 rows)
// or the end of t's chunk (chunk-end padding).
// ----------------------------------------------------------------------------
struct ConvGeom {
  int T, Tx, C, chunk_pad;
};

__device__ __forceinline__ int conv_limit(const ConvGeom& g, int t) {
  return g.chunk_pad ? (t / g.C + 1) * g.C : g.Tx;
}

__global__ void conv_f32_kernel(const float* __restrict__ X0, const float* __restrict__ Kc,
                                float* __restrict__ Y, ConvGeom g, int d, int k, long long rows) {
  const long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (e >= rows * d) return;
  const long long row = e / d;
  const int c = static_cast<int>(e % d);
  const int t = static_cast<int>(row % g.T);
  const long long xrow = (row / g.T) * g.Tx + t;
  const int lim = conv_limit(g, t);
  float acc = 0.f;
  for (int j = 0; j < k && t + j < lim; ++j) acc = fmaf(Kc[c * k + j], X0[(xrow + j) * d + c], acc);
  Y[e] = acc;
}

// bf16 version: one thread owns 8 consecutive channels (16-byte loads and
// stores, coalesced along the channel axis) over a run of RUN tokens.  All
// RUN + KT - 1 input rows of the run are loaded before any arithmetic so that
// every thread keeps that many independent loads in flight; X0 is read once
// plus a (KT-1)-row halo per run.
template <int KT, int RUN>
__global__ void __launch_bounds__(256) conv_bf16_kernel(const __nv_bfloat16* __restrict__ X0,
                                                        const __nv_bfloat16* __restrict__ Kc,
                                                        __nv_bfloat16* __restrict__ Y, ConvGeom g,
                                                        int d) {
  grid_dependency_wait();
  const int groups = d >> 3;
  const int gi = blockIdx.x * blockDim.x + threadIdx.x;
  if (gi >= groups) return;
  const int runs_per_seq = (g.T + RUN - 1) / RUN;
  const int b = blockIdx.y / runs_per_seq;
  const int t0 = (blockIdx.y % runs_per_seq) * RUN;
  const int c0 = gi * 8;
  const long long xbase = (long long)b * g.Tx;
  const long long ybase = (long long)b * g.T;

  uint4 rows[RUN + KT - 1];
#pragma unroll
  for (int i = 0; i < RUN + KT - 1; ++i)
    rows[i] = (t0 + i < g.Tx) ? __ldg(reinterpret_cast<const uint4*>(X0 + (xbase + t0 + i) * d + c0))
                              : make_uint4(0u, 0u, 0u, 0u);

  // the taps of channels c0..c0+7 are 8*KT contiguous bf16: KT 16-byte loads
  float w[KT][8];
  const uint4* kp = reinterpret_cast<const uint4*>(Kc + c0 * KT);
#pragma unroll
  for (int q = 0; q < KT; ++q) {
    const uint4 v = __ldg(kp + q);
    const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv[h]));
      const int e0 = q * 8 + 2 * h, e1 = e0 + 1;  // element index = channel * KT + tap
      w[e0 % KT][e0 / KT] = f2.x;
      w[e1 % KT][e1 / KT] = f2.y;
    }
  }

#pragma unroll
  for (int t = 0; t < RUN; ++t) {
    if (t0 + t >= g.T) break;
    const int lim = conv_limit(g, t0 + t);
    float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < KT; ++j) {
      if (t0 + t + j >= lim) break;
      const uint32_t vv[4] = {rows[t + j].x, rows[t + j].y, rows[t + j].z, rows[t + j].w};
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
    *reinterpret_cast<uint4*>(Y + (ybase + t0 + t) * d + c0) = o;
  }
}

// Generic bf16 fallback for any k (<= 16), one element per thread.
// One piece of the bf16 look-ahead conv for threads that run it beside other
// work: RUN tokens x 8 channels (channel group `grp`) of sequence b from token
// t0, any k <= KMAX taps, the same arithmetic as conv_bf16_kernel (fp32 taps
// and products, one rounding to bf16).
template <int KMAX, int RUN>
__device__ __forceinline__ void conv_piece_bf16(const __nv_bfloat16* __restrict__ X0,
                                                const __nv_bfloat16* __restrict__ Kc,
                                                __nv_bfloat16* __restrict__ Y, const ConvGeom& g,
                                                int d, int k, int b, int t0, int grp) {
  const int c0 = grp * 8;
  const long long xbase = (long long)b * g.Tx;
  const long long ybase = (long long)b * g.T;
  uint4 rows[RUN + KMAX - 1];
#pragma unroll
  for (int i = 0; i < RUN + KMAX - 1; ++i)
    rows[i] = (i < RUN + k - 1 && t0 + i < g.Tx)
                  ? __ldg(reinterpret_cast<const uint4*>(X0 + (xbase + t0 + i) * d + c0))
                  : make_uint4(0u, 0u, 0u, 0u);
  float w[KMAX][8];
#pragma unroll
  for (int j = 0; j < KMAX; ++j)
#pragma unroll
    for (int c = 0; c < 8; ++c)
      w[j][c] = j < k ? __bfloat162float(Kc[(c0 + c) * k + j]) : 0.f;
#pragma unroll
  for (int t = 0; t < RUN; ++t) {
    if (t0 + t >= g.T) break;
    const int lim = conv_limit(g, t0 + t);
    float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j >= k || t0 + t + j >= lim) break;
      const uint32_t vv[4] = {rows[t + j].x, rows[t + j].y, rows[t + j].z, rows[t + j].w};
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
    *reinterpret_cast<uint4*>(Y + (ybase + t0 + t) * d + c0) = o;
  }
}

__global__ void conv_bf16_generic_kernel(const __nv_bfloat16* __restrict__ X0,
                                         const __nv_bfloat16* __restrict__ Kc,
                                         __nv_bfloat16* __restrict__ Y, ConvGeom g, int d, int k,
                                         long long rows) {
  const long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (e >= rows * d) return;
  const long long row = e / d;
  const int c = static_cast<int>(e % d);
  const int t = static_cast<int>(row % g.T);
  const long long xrow = (row / g.T) * g.Tx + t;
  const int lim = conv_limit(g, t);
  float acc = 0.f;
  for (int j = 0; j < k && t + j < lim; ++j)
    acc = fmaf(__bfloat162float(Kc[c * k + j]), __bfloat162float(X0[(xrow + j) * d + c]), acc);
  Y[e] = __float2bfloat16_rn(acc);
}

// ----------------------------------------------------------------------------
// Update-norm clipping helpers.  norm2[b * n + i] holds ||Vhat_i^T Z_i||_F^2
// of sequence b's chunk i; the delta's norm is |eta| sqrt(norm2).
// ----------------------------------------------------------------------------
__device__ __forceinline__ float clip_scale(float norm2, float eta, float tau) {
  const float nrm = fabsf(eta) * sqrtf(norm2);
  return (tau > 0.f && nrm > tau) ? tau / nrm : 1.f;
}

// Rescale the rows of Vhat [rows, d] whose chunk's delta exceeds tau (bf16,
// 8 channels per thread, 16-byte accesses; rows of unclipped chunks are not
// touched).
__global__ void clip_scale_rows_bf16(__nv_bfloat16* __restrict__ V, const float* __restrict__ norm2,
                                     float eta, float tau, int T, int C, int d, long long rows) {
  grid_dependency_wait();
  const int groups = d >> 3;
  const long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (e >= rows * groups) return;
  const long long row = e / groups;
  const int c0 = static_cast<int>(e % groups) * 8;
  const int n = T / C;
  const long long b = row / T;
  const int chunk = static_cast<int>(row % T) / C;
  const float sc = clip_scale(norm2[b * n + chunk], eta, tau);
  if (sc == 1.f) return;
  uint4* ptr = reinterpret_cast<uint4*>(V + row * d + c0);
  uint4 v = *ptr;
  uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv[h]));
    vv[h] = pack_bf16x2(f2.x * sc, f2.y * sc);
  }
  *ptr = make_uint4(vv[0], vv[1], vv[2], vv[3]);
}

// fp32 version, one element per thread.
__global__ void clip_scale_rows_f32(float* __restrict__ V, const float* __restrict__ norm2,
                                    float eta, float tau, int T, int C, int d, long long rows) {
  const long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (e >= rows * d) return;
  const long long row = e / d;
  const int n = T / C;
  const float sc = clip_scale(norm2[(row / T) * n + static_cast<int>(row % T) / C], eta, tau);
  if (sc != 1.f) V[e] *= sc;
}

// norms[i] = |eta| sqrt(norm2[i]) in place.
__global__ void clip_finish_norms(float* __restrict__ norms, float eta, int count) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < count) norms[i] = fabsf(eta) * sqrtf(norms[i]);
}

// fp32 norm^2 of each chunk by the gram identity, one block per (b, chunk, s):
// sum_t (Z_s . Z_t)(V_s . V_t) over the chunk's tokens t, added to norm2.
__global__ void clip_norms_f32(const float* __restrict__ Z, const float* __restrict__ V,
                               float* __restrict__ norm2, int T, int C, int d, int f) {
  const int n = T / C;
  const int s_local = blockIdx.x % C;
  const int chunk = (blockIdx.x / C) % n;
  const int b = blockIdx.x / (C * n);
  const long long s = (long long)b * T + (long long)chunk * C + s_local;
  float part = 0.f;
  for (int t_local = threadIdx.x; t_local < C; t_local += blockDim.x) {
    const long long t = (long long)b * T + (long long)chunk * C + t_local;
    float zz = 0.f, vv = 0.f;
    for (int j = 0; j < f; ++j) zz = fmaf(Z[s * f + j], Z[t * f + j], zz);
    for (int j = 0; j < d; ++j) vv = fmaf(V[s * d + j], V[t * d + j], vv);
    part = fmaf(zz, vv, part);
  }
  __shared__ float red[256];
  red[threadIdx.x] = part;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) atomicAdd(norm2 + b * n + chunk, red[0]);
}

// fp32 path of the forward: clip the materialised deltas in place.  Slice j of
// sequence b: stack[b][j] for j < n-1, W_final[b] for j = n-1.  One block per
// slice: sum of squares, then rescale.
__global__ void clip_deltas_f32(float* __restrict__ stack, float* __restrict__ W_final,
                                long long df, int nchunk, float tau) {
  const int b = blockIdx.x / nchunk, j = blockIdx.x % nchunk;
  float* x = (j < nchunk - 1) ? stack + ((long long)b * (nchunk - 1) + j) * df
                              : W_final + (long long)b * df;
  float part = 0.f;
  for (long long e = threadIdx.x; e < df; e += blockDim.x) part = fmaf(x[e], x[e], part);
  __shared__ float red[256];
  red[threadIdx.x] = part;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  const float nrm = sqrtf(red[0]);
  if (!(tau > 0.f && nrm > tau)) return;
  const float sc = tau / nrm;
  for (long long e = threadIdx.x; e < df; e += blockDim.x) x[e] *= sc;
}

// ----------------------------------------------------------------------------
// Decode GEMVs (memory-bound: every weight byte is read once per step).
// ----------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float& o, float x) { o = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16& o, float x) { o = __float2bfloat16_rn(x); }

constexpr int DECODE_MAX_B = 8;

// Z[b * zstride + j] = silu(H[b] . W_gate[j]) * (H[b] . W_up[j]) for b < nb
// (nb <= DECODE_MAX_B): one warp per hidden unit j, lanes striding over d so
// that a warp reads contiguous pieces of the two weight rows.
template <typename T_>
__global__ void gated_gemv_kernel(const T_* __restrict__ H, const T_* __restrict__ Wg,
                                  const T_* __restrict__ Wu, T_* __restrict__ Z, long long zstride,
                                  int nb, int d, int f) {
  grid_dependency_wait();
  const int j = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (j >= f) return;
  float g[DECODE_MAX_B], u[DECODE_MAX_B];
#pragma unroll
  for (int b = 0; b < DECODE_MAX_B; ++b) g[b] = u[b] = 0.f;
  const T_* wg = Wg + (long long)j * d;
  const T_* wu = Wu + (long long)j * d;
  for (int c = lane; c < d; c += 32) {
    const float a = to_f(wg[c]), bb = to_f(wu[c]);
#pragma unroll
    for (int b = 0; b < DECODE_MAX_B; ++b) {
      if (b < nb) {
        const float h = to_f(H[(long long)b * d + c]);
        g[b] = fmaf(h, a, g[b]);
        u[b] = fmaf(h, bb, u[b]);
      }
    }
  }
#pragma unroll
  for (int b = 0; b < DECODE_MAX_B; ++b) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      g[b] += __shfl_xor_sync(0xffffffffu, g[b], o);
      u[b] += __shfl_xor_sync(0xffffffffu, u[b], o);
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int b = 0; b < DECODE_MAX_B; ++b)
      if (b < nb) from_f(Z[(long long)b * zstride + j], (g[b] / (1.0f + expf(-g[b]))) * u[b]);
  }
}

// O[b, a] = Z[b] . W[b, a, :] with a per-sequence fast weight W [nb, d, f] (fp32 or bf16):
// one warp per output (b, a), lanes striding over f.
template <typename T_, typename WT>
__global__ void apply_gemv_kernel(const T_* __restrict__ Z, long long zstride,
                                  const WT* __restrict__ W, T_* __restrict__ O, int nb, int d,
                                  int f) {
  grid_dependency_wait();
  const long long w = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= (long long)nb * d) return;
  const int b = static_cast<int>(w / d), a = static_cast<int>(w % d);
  const WT* row = W + ((long long)b * d + a) * f;
  const T_* z = Z + (long long)b * zstride;
  float acc = 0.f;
  for (int j = lane; j < f; j += 32) acc = fmaf(to_f(z[j]), to_f(row[j]), acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) from_f(O[(long long)b * d + a], acc);
}

// 16-byte packs of T_ unpacked to fp32: 8 bf16 or 4 floats.
template <typename T_>
struct Pack16;
template <>
struct Pack16<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ __forceinline__ static void unpack(const uint4& v, float* o) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      o[2 * i] = f2.x;
      o[2 * i + 1] = f2.y;
    }
  }
};
template <>
struct Pack16<float> {
  static constexpr int E = 4;
  __device__ __forceinline__ static void unpack(const uint4& v, float* o) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
  }
};

// Decode: steps of loads issued together by the gated GEMV for 3..8 sequences.
#ifndef ITTT_GEMV_BATCH_WIDE
#define ITTT_GEMV_BATCH_WIDE 1
#endif

// Vectorised gated GEMV of the decode step: NB tokens (one per sequence), one
// warp per U consecutive hidden units, two warps per block (many small blocks
// spread the equal work items evenly over the SMs).  The first threads also
// copy the token's X0 rows into the chunk buffer.  Every lane reads 16 bytes of each
// weight row per step (a warp covers 32 x 16 bytes of a row), the token rows
// once for all U units; needs d % E == 0 and 16-byte aligned rows.
template <typename T_, int NB, int U>
__global__ void __launch_bounds__(64) gated_gemv_vec_kernel(
    const T_* __restrict__ H, const T_* __restrict__ Wg, const T_* __restrict__ Wu,
    T_* __restrict__ Z, long long zstride, const T_* __restrict__ X0_tok, T_* __restrict__ X0_dst,
    long long x0stride, int d, int f) {
  grid_dependency_wait();
  grid_launch_dependents();  // the apply GEMV may start; it waits for Z itself
  constexpr int E = Pack16<T_>::E;
  constexpr int BATCH = NB <= 2 ? 4 : ITTT_GEMV_BATCH_WIDE;  // steps whose loads are issued together
  const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  // the token's X0 rows into the chunk buffer (16 bytes per thread)
  if (gtid < (long long)NB * (d / E)) {
    const int b = static_cast<int>(gtid / (d / E));
    const int c = static_cast<int>(gtid % (d / E)) * E;
    *reinterpret_cast<uint4*>(X0_dst + b * x0stride + c) =
        __ldg(reinterpret_cast<const uint4*>(X0_tok + (long long)b * d + c));
  }
  const int j0 = static_cast<int>(gtid >> 5) * U;
  const int lane = threadIdx.x & 31;
  if (j0 >= f) return;
  float g[NB][U], u[NB][U];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int q = 0; q < U; ++q) g[b][q] = u[b][q] = 0.f;
#pragma unroll (BATCH == 1 ? 2 : 1)
  for (int c0 = lane * E; c0 < d; c0 += 32 * E * BATCH) {
    uint4 hr[BATCH][NB], ga[BATCH][U], ua[BATCH][U];
#pragma unroll
    for (int i = 0; i < BATCH; ++i) {
      const int c = c0 + i * 32 * E;
      if (c < d) {
#pragma unroll
        for (int b = 0; b < NB; ++b) hr[i][b] = __ldg(reinterpret_cast<const uint4*>(H + (long long)b * d + c));
#pragma unroll
        for (int q = 0; q < U; ++q) {
          if (j0 + q < f) {
            ga[i][q] = __ldg(reinterpret_cast<const uint4*>(Wg + (long long)(j0 + q) * d + c));
            ua[i][q] = __ldg(reinterpret_cast<const uint4*>(Wu + (long long)(j0 + q) * d + c));
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < BATCH; ++i) {
      if (c0 + i * 32 * E < d) {
        float h[NB][E];
#pragma unroll
        for (int b = 0; b < NB; ++b) Pack16<T_>::unpack(hr[i][b], h[b]);
#pragma unroll
        for (int q = 0; q < U; ++q) {
          if (j0 + q < f) {
            float a[E], e2[E];
            Pack16<T_>::unpack(ga[i][q], a);
            Pack16<T_>::unpack(ua[i][q], e2);
#pragma unroll
            for (int b = 0; b < NB; ++b)
#pragma unroll
              for (int e = 0; e < E; ++e) {
                g[b][q] = fmaf(h[b][e], a[e], g[b][q]);
                u[b][q] = fmaf(h[b][e], e2[e], u[b][q]);
              }
          }
        }
      }
    }
  }
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int q = 0; q < U; ++q)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        g[b][q] += __shfl_xor_sync(0xffffffffu, g[b][q], o);
        u[b][q] += __shfl_xor_sync(0xffffffffu, u[b][q], o);
      }
  if (lane == 0) {
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int q = 0; q < U; ++q)
        if (j0 + q < f) from_f(Z[(long long)b * zstride + j0 + q], silu_f32(g[b][q]) * u[b][q]);
  }
}

// Warp-level tensor-core MMA m16n8k16 (bf16 in, fp32 accumulate), c += a * b.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Gated GEMV of the decode step for bf16 on warp-level MMAs: the NB <= 8 token
// rows are the n = 8 columns (missing ones zero), 16 hidden units the m = 16
// rows, so the weights are read once for all tokens and the products leave the
// FMA pipe.  Block = S warps on the units j0 .. j0+15; warp w takes the w-th of
// S ranges of the d inputs, and the partial sums meet in shared memory, where
// the first warp adds them in warp order and writes silu(g) * u.  Lane (r, c)
// (r = lane / 4, c = lane % 4) loads 16 contiguous bytes of weight rows j0+r
// and j0+r+8 and of token row r per 32 inputs; its 8 inputs fill the k-slots
// the fragment layout gives that lane in two MMAs (2c, 2c+1, 2c+8, 2c+9 of
// each), in the same order for the weights and the tokens, which a dot product
// does not see.  Needs d % 32 == 0 and 16-byte aligned rows.  The first
// threads also copy the token's X0 rows into the chunk buffer.
template <int NB, int S>
__global__ void __launch_bounds__(32 * S) gated_gemv_mma_kernel(
    const __nv_bfloat16* __restrict__ H, const __nv_bfloat16* __restrict__ Wg,
    const __nv_bfloat16* __restrict__ Wu, __nv_bfloat16* __restrict__ Z, long long zstride,
    const __nv_bfloat16* __restrict__ X0_tok, __nv_bfloat16* __restrict__ X0_dst,
    long long x0stride, int d, int f) {
  static_assert(NB >= 1 && NB <= 8, "the tokens are the 8 columns of one MMA");
  constexpr int UNR = 4;  // 32-input steps whose loads are issued together
  grid_dependency_wait();
  grid_launch_dependents();  // the apply GEMV may start; it waits for Z itself
  const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gtid < (long long)NB * (d / 8)) {
    const int b = static_cast<int>(gtid / (d / 8));
    const int c = static_cast<int>(gtid % (d / 8)) * 8;
    *reinterpret_cast<uint4*>(X0_dst + b * x0stride + c) =
        __ldg(reinterpret_cast<const uint4*>(X0_tok + (long long)b * d + c));
  }
  const int j0 = blockIdx.x * 16;
  if (j0 >= f) return;  // whole block: j0 depends on the block only
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 2, c4 = lane & 3;
  const bool va = j0 + r < f, vb = j0 + r + 8 < f, vt = r < NB;
  const __nv_bfloat16* ga = Wg + (long long)(va ? j0 + r : 0) * d + c4 * 8;
  const __nv_bfloat16* gb = Wg + (long long)(vb ? j0 + r + 8 : 0) * d + c4 * 8;
  const __nv_bfloat16* ua = Wu + (long long)(va ? j0 + r : 0) * d + c4 * 8;
  const __nv_bfloat16* ub = Wu + (long long)(vb ? j0 + r + 8 : 0) * d + c4 * 8;
  const __nv_bfloat16* hx = H + (long long)(vt ? r : 0) * d + c4 * 8;
  const int steps = d / 32;
  const int s0 = warp * steps / S, s1 = (warp + 1) * steps / S;
  // Rows past f and tokens past NB read row 0 instead: they feed only
  // accumulator entries that are never written.
  float cg[4] = {0.f, 0.f, 0.f, 0.f}, cu[4] = {0.f, 0.f, 0.f, 0.f};
  auto ld = [](const __nv_bfloat16* ptr) { return __ldg(reinterpret_cast<const uint4*>(ptr)); };
  auto step = [&](const uint4& wa, const uint4& wb, const uint4& xa, const uint4& xb, const uint4& x) {
    mma_bf16_16816(cg, wa.x, wb.x, wa.y, wb.y, x.x, x.y);
    mma_bf16_16816(cg, wa.z, wb.z, wa.w, wb.w, x.z, x.w);
    mma_bf16_16816(cu, xa.x, xb.x, xa.y, xb.y, x.x, x.y);
    mma_bf16_16816(cu, xa.z, xb.z, xa.w, xb.w, x.z, x.w);
  };
  int s = s0;
  for (; s + UNR <= s1; s += UNR) {
    uint4 wa[UNR], wb[UNR], xa[UNR], xb[UNR], x[UNR];
#pragma unroll
    for (int i = 0; i < UNR; ++i) {
      const long long o = (long long)(s + i) * 32;
      wa[i] = ld(ga + o);
      wb[i] = ld(gb + o);
      xa[i] = ld(ua + o);
      xb[i] = ld(ub + o);
      x[i] = ld(hx + o);
    }
#pragma unroll
    for (int i = 0; i < UNR; ++i) step(wa[i], wb[i], xa[i], xb[i], x[i]);
  }
  for (; s < s1; ++s) {
    const long long o = (long long)s * 32;
    step(ld(ga + o), ld(gb + o), ld(ua + o), ld(ub + o), ld(hx + o));
  }
  if constexpr (S > 1) {
    __shared__ float part[S - 1][8][32];
    if (warp > 0) {
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        part[warp - 1][v][lane] = cg[v];
        part[warp - 1][4 + v][lane] = cu[v];
      }
    }
    __syncthreads();
    if (warp > 0) return;
#pragma unroll
    for (int w = 0; w < S - 1; ++w)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        cg[v] += part[w][v][lane];
        cu[v] += part[w][4 + v][lane];
      }
  }
  // accumulator (row j0+r, tokens 2c, 2c+1) in [0], [1]; row j0+r+8 in [2], [3]
  const int t0 = 2 * c4, t1 = 2 * c4 + 1;
  if (va && t0 < NB) from_f(Z[(long long)t0 * zstride + j0 + r], silu_f32(cg[0]) * cu[0]);
  if (va && t1 < NB) from_f(Z[(long long)t1 * zstride + j0 + r], silu_f32(cg[1]) * cu[1]);
  if (vb && t0 < NB) from_f(Z[(long long)t0 * zstride + j0 + r + 8], silu_f32(cg[2]) * cu[2]);
  if (vb && t1 < NB) from_f(Z[(long long)t1 * zstride + j0 + r + 8], silu_f32(cg[3]) * cu[3]);
}

// Vectorised apply GEMV of the decode step: O[b, a] = Z[b] . W[b, a, :] with
// the per-sequence state W [nb, d, f] of type WT (fp32, or its bf16 rounding),
// one warp per U consecutive rows a of one sequence; a lane reads 16 bytes of
// each state row and of Z per step, and issues the loads of BATCH steps before
// it uses any (the kernel is bound by memory latency, not by issue).  Needs
// f % (16 / sizeof(WT)) == 0 (aligned state rows and Z pieces).
template <typename T_, typename WT, int U>
__global__ void __launch_bounds__(64) apply_gemv_vec_kernel(
    const T_* __restrict__ Z, long long zstride, const WT* __restrict__ W, T_* __restrict__ O,
    int nb, int d, int f) {
  static_assert(sizeof(T_) == sizeof(WT), "Z and the state are read in equal 16-byte pieces");
  constexpr int K = 16 / int(sizeof(WT));
  constexpr int BATCH = U == 1 ? 8 : 4;  // steps whose loads are issued together
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long row_groups = (d + U - 1) / U;
  const bool active = w < (long long)nb * row_groups;
  const int b = active ? static_cast<int>(w / row_groups) : 0;
  const int a0 = active ? static_cast<int>(w % row_groups) * U : 0;
  const T_* z = Z + (long long)b * zstride;
  const WT* rows = W + ((long long)b * d + a0) * f;
  // The state is not written by the kernel this one may overlap (the gated
  // GEMV, which writes Z): its first pieces go to L2 before the wait.
  if (active) {
#pragma unroll
    for (int i = 0; i < BATCH; ++i) {
      const int j = lane * K + i * 32 * K;
      if (j < f) {
#pragma unroll
        for (int q = 0; q < U; ++q)
          if (a0 + q < d) prefetch_l2(rows + (long long)q * f + j);
      }
    }
  }
  grid_dependency_wait();
  if (!active) return;
  float acc[U];
#pragma unroll
  for (int q = 0; q < U; ++q) acc[q] = 0.f;
  for (int j0 = lane * K; j0 < f; j0 += 32 * K * BATCH) {
    uint4 zr[BATCH], wr[BATCH][U];
#pragma unroll
    for (int i = 0; i < BATCH; ++i) {
      const int j = j0 + i * 32 * K;
      if (j < f) {
        zr[i] = __ldg(reinterpret_cast<const uint4*>(z + j));
#pragma unroll
        for (int q = 0; q < U; ++q)
          if (a0 + q < d) wr[i][q] = __ldg(reinterpret_cast<const uint4*>(rows + (long long)q * f + j));
      }
    }
#pragma unroll
    for (int i = 0; i < BATCH; ++i) {
      if (j0 + i * 32 * K < f) {
        float zz[K];
        Pack16<T_>::unpack(zr[i], zz);
#pragma unroll
        for (int q = 0; q < U; ++q) {
          if (a0 + q < d) {
            float wv[K];
            Pack16<WT>::unpack(wr[i][q], wv);
#pragma unroll
            for (int e = 0; e < K; ++e) acc[q] = fmaf(zz[e], wv[e], acc[q]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < U; ++q)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], o);
  if (lane == 0) {
#pragma unroll
    for (int q = 0; q < U; ++q)
      if (a0 + q < d) from_f(O[(long long)b * d + a0 + q], acc[q]);
  }
}

// dst = bf16(src), 8 elements per thread (n % 8 == 0, 16-byte aligned).
__global__ void round_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                  long long n) {
  grid_dependency_wait();
  const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (i >= n) return;
  const float4 a = __ldg(reinterpret_cast<const float4*>(src + i));
  const float4 c = __ldg(reinterpret_cast<const float4*>(src + i + 4));
  *reinterpret_cast<uint4*>(dst + i) = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w),
                                                  pack_bf16x2(c.x, c.y), pack_bf16x2(c.z, c.w));
}

// dst[i] += src[i] (fp32).
__global__ void add_f32_kernel(float* __restrict__ dst, const float* __restrict__ src, long long n) {
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i < n) dst[i] += src[i];
}

// ----------------------------------------------------------------------------
// Context parallelism.
//
// Exclusive prefix over the leading axis: P[g, e] = S[0, e] + ... + S[g-1, e]
// (row 0 zeros), accumulated in that order in fp32.  One thread per 4 (vec:
// n % 4 == 0 and 16-byte aligned rows) or 1 column walks the G rows; every row
// access is coalesced across the warp.
__global__ void cp_prefix_kernel(const float* __restrict__ S, float* __restrict__ P, int G,
                                 long long n, bool vec) {
  const long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (vec) {
    const long long e = 4 * t;
    if (e >= n) return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int g = 0; g < G; ++g) {
      *reinterpret_cast<float4*>(P + (long long)g * n + e) = acc;
      const float4 v = __ldg(reinterpret_cast<const float4*>(S + (long long)g * n + e));
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
  } else {
    if (t >= n) return;
    float acc = 0.f;
    for (int g = 0; g < G; ++g) {
      P[(long long)g * n + t] = acc;
      acc += __ldg(S + (long long)g * n + t);
    }
  }
}

// The weights of one segment once its prefix P (sum of the earlier segments'
// deltas) is known.  cp_delta left in `stack` the segment's own running sums
// L_1 .. L_{n-1} (started from zero); here, per sequence b and element e,
// with w = W0[e] + P[b, e] in fp32:
//   W_start[b, e] = w              (the apply's operand for the first chunk)
//   stack[b, i, e] = w + L_{i+1}   (the effective weight of chunk i + 1)
//   W_end[b, e]   = w + S[b, e]    (the state after the segment)
// each rounded once to T_.  VEC elements per thread (16-byte stack accesses
// for bf16 when df % 8 == 0, else 1).
template <typename T_, int VEC>
__global__ void cp_weights_kernel(const T_* __restrict__ W0, const float* __restrict__ P,
                                  const float* __restrict__ S, T_* __restrict__ W_start,
                                  float* __restrict__ W_end, T_* __restrict__ stack, int n_snap,
                                  long long df, int nb) {
  static_assert(VEC == 1 || (VEC == 8 && sizeof(T_) == 2), "8-wide only for bf16");
  const long long e0 = (blockIdx.x * (long long)blockDim.x + threadIdx.x) * VEC;
  if (e0 >= df) return;
  float w0[VEC];
  if constexpr (VEC == 8) {
    Pack16<T_>::unpack(__ldg(reinterpret_cast<const uint4*>(W0 + e0)), w0);
  } else {
    w0[0] = to_f(W0[e0]);
  }
  for (int b = 0; b < nb; ++b) {
    const long long be = (long long)b * df + e0;
    float w[VEC];
    T_* st = stack + (long long)b * n_snap * df + e0;
    if constexpr (VEC == 8) {
      const float4 p0 = *reinterpret_cast<const float4*>(P + be);
      const float4 p1 = *reinterpret_cast<const float4*>(P + be + 4);
      const float4 s0 = *reinterpret_cast<const float4*>(S + be);
      const float4 s1 = *reinterpret_cast<const float4*>(S + be + 4);
      const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
      const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      uint32_t o[4];
      float e[8];
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        w[v] = w0[v] + pv[v];
        e[v] = w[v] + sv[v];
      }
#pragma unroll
      for (int h = 0; h < 4; ++h) o[h] = pack_bf16x2(w[2 * h], w[2 * h + 1]);
      *reinterpret_cast<uint4*>(W_start + be) = make_uint4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<float4*>(W_end + be) = make_float4(e[0], e[1], e[2], e[3]);
      *reinterpret_cast<float4*>(W_end + be + 4) = make_float4(e[4], e[5], e[6], e[7]);
      for (int i = 0; i < n_snap; ++i, st += df) {
        float l[8];
        Pack16<T_>::unpack(*reinterpret_cast<const uint4*>(st), l);
#pragma unroll
        for (int h = 0; h < 4; ++h) o[h] = pack_bf16x2(w[2 * h] + l[2 * h], w[2 * h + 1] + l[2 * h + 1]);
        *reinterpret_cast<uint4*>(st) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    } else {
      w[0] = w0[0] + P[be];
      from_f(W_start[be], w[0]);
      W_end[be] = w[0] + S[be];
      for (int i = 0; i < n_snap; ++i, st += df) from_f(*st, w[0] + to_f(*st));
    }
  }
}

// W_final[b] = float(W0) for every sequence (eta = 0: no update happens).
__global__ void broadcast_w0_kernel(const __nv_bfloat16* __restrict__ W0, float* __restrict__ Wf,
                                    long long df, int nb) {
  const long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (e >= df) return;
  const float v = __bfloat162float(W0[e]);
  for (int b = 0; b < nb; ++b) Wf[(long long)b * df + e] = v;
}

// Bounded-wait self test: waits on a barrier nobody arrives on.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl wc{&abort_flag, limit_ns};
    mbar_wait(&bar, 0, wc);
  }
}

}  // namespace ittt
