// poem_pooled.cu -- pooled block-score estimates for the practical POEM selector
// (sm_100a, CUDA cores).
//
// The practical variant of the method (reading note "Attention deletion error",
// the paragraph on Equation (6) and Appendix B) ranks blocks from cheap estimates
// of the dense reference output and of the block outputs instead of exact
// per-query scores.  The estimators are not printed; this library pools by mean:
//   q~_{h,i}          mean of the B queries of tile i, head h
//   k~_{g,b}, v~_{g,b} means of the B keys / values of block b, KV head g
//   m~_b = softmax over b <= i of scale * <q~_{h,i}, k~_{g,b}>   (pooled mass)
//   o~   = sum_b m~_b v~_b                                       (estimated o)
//   d~_b = || v~_b - o~ ||                                       (estimated deviation)
// so that m~_b d~_b estimates the proxy I_b = m_b ||v_b - o|| of Equation (4).
//
// Kernels (caller's stream):
//   pool_mean      grid (tile, channel groups, tensor): each thread sums the B
//                  rows of one (head, 8-channel group) of one tile with 16-byte
//                  streaming loads, in fp32, and writes the mean -- row-major for
//                  q~ and v~, channel-major ([D][T]) for k~ and v~.  HBM-bound:
//                  reads Q, K and V once.
//   pooled_scores  one CTA per (R_t adjacent tiles x R_h query heads of one KV
//                  head), largest tiles first; its R = R_h * R_t <= 8 rows share
//                  every k~ / v~ value they load:
//                    logits  lane per block, channel-major k~ (coalesced), q~
//                            broadcast from shared memory, packed f32x2 FMAs
//                    softmax warp per row -> m~ (shared memory and m_pool)
//                    o~      thread per (channel, block slice), 4 blocks a step
//                    d~      lane per block like the logits, v~ - o~ squared
//                  The k~ / v~ of a KV head (T * D * 4 bytes each) stay in L2
//                  across its CTAs; no warp shuffles on the per-block paths.
// With a query offset (chunked prefill) q~ covers the Tq query tiles, k~ / v~
// all q_tile0 + Tq key blocks, and local tile i sees blocks 0 .. q_tile0 + i.
#include "common.cuh"

namespace poem {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;
constexpr int kMaxRows = 8;
constexpr size_t kPooledSmemCap = 200 * 1024;

template <int D>
__global__ void __launch_bounds__(kPoolThreads) pool_mean_kernel(const PoolParams p) {
  constexpr int C8 = D / 8;
  const int which = blockIdx.z;  // 0: q, 1: k, 2: v
  const int heads = which == 0 ? p.n_q_heads : p.n_kv_heads;
  const int u = blockIdx.y * kPoolThreads + threadIdx.x;
  const int i = blockIdx.x;                            // query tile (q) or key block (k, v)
  const int T = which == 0 ? p.n_tiles : p.n_kv_tiles;
  if (u >= heads * C8 || i >= T) return;
  const int h = u / C8;
  const int c8 = u - h * C8;
  const __nv_bfloat16* src = which == 0 ? p.q : (which == 1 ? p.k : p.v);
  const int64_t st_tok = which == 0 ? p.q_stride_tok : p.kv_stride_tok;
  const int64_t st_head = which == 0 ? p.q_stride_head : p.kv_stride_head;
  const __nv_bfloat16* base = src + (int64_t)i * p.block * st_tok + (int64_t)h * st_head + c8 * 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 8
  for (int t = 0; t < p.block; ++t) {
    const uint4 w = __ldcs(reinterpret_cast<const uint4*>(base + (int64_t)t * st_tok));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += bf16lo_to_f32(ws[e]);
      acc[2 * e + 1] += bf16hi_to_f32(ws[e]);
    }
  }
  const float inv = 1.0f / (float)p.block;
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] *= inv;
  if (which != 1) {  // row-major [H, T, D]
    float* dst = (which == 0 ? p.q_bar : p.v_bar) + ((int64_t)h * T + i) * D + c8 * 8;
    reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    reinterpret_cast<float4*>(dst)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  if (which != 0) {  // channel-major [H, D, T]
    float* dst = (which == 1 ? p.k_bar_t : p.v_bar_t) + ((int64_t)h * D + c8 * 8) * T + i;
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[(int64_t)e * T] = acc[e];
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

template <int D, int R>
__global__ void __launch_bounds__(kScoreThreads) pooled_scores_kernel(const PoolParams p) {
  constexpr int S = kScoreThreads / D;  // block slices of the o~ pass
  extern __shared__ __align__(16) float smf[];
  const int T = p.n_tiles;      // query tiles
  const int Tk = p.n_kv_tiles;  // key blocks
  const int t0 = p.q_tile0;
  const int ld = (Tk + 3) & ~3;
  float* qb = smf;                // [R][D]
  float* ob = qb + R * D;         // [R][D]
  float* part = ob + R * D;       // [S][R][D]
  float* buf = part + S * R * D;  // [R][ld]: logits -> m~ -> d~
  __shared__ int s_head[R], s_tile[R];

  const int Rh = p.heads_per_cta, Rt = p.tiles_per_cta;
  const int n_hchunks = p.n_q_heads / Rh;
  const int tg = blockIdx.x / n_hchunks;
  const int h0 = (blockIdx.x - tg * n_hchunks) * Rh;
  const int i_top = T - 1 - tg * Rt;  // local tiles i_top, i_top - 1, ..., i_top - Rt + 1 (those >= 0)
  const int g = h0 / p.group;
  const int nbmax = i_top + t0 + 1;   // key blocks of the longest row
  const int nb4 = (nbmax + 3) & ~3;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* kT = p.k_bar_t + (int64_t)g * D * Tk;
  const float* vT = p.v_bar_t + (int64_t)g * D * Tk;
  const float* vb = p.v_bar + (int64_t)g * Tk * D;

  // Row r: head h0 + r % Rh, local tile i_top - r / Rh (invalid when the tile is
  // < 0 or r >= Rh * Rt); nb_r = t0 + tile + 1 visible blocks, 0 for invalid rows.
  int nb[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int tile = (r < Rh * Rt) ? i_top - r / Rh : -1;
    nb[r] = tile >= 0 ? t0 + tile + 1 : 0;
  }
  if (threadIdx.x < R) {
    const int r = threadIdx.x;
    s_head[r] = h0 + r % Rh;
    s_tile[r] = (r < Rh * Rt) ? i_top - r / Rh : -1;
  }
  for (int x = threadIdx.x; x < R * D; x += kScoreThreads) {
    const int r = x / D, c = x - r * D;
    const int tile = (r < Rh * Rt) ? i_top - r / Rh : -1;
    qb[x] = tile >= 0 ? p.q_bar[((int64_t)(h0 + r % Rh) * T + tile) * D + c] : 0.f;
  }
  __syncthreads();

  // Logits: lane per block; channel-major k~ makes each channel one coalesced load.
  for (int b0 = warp * 32; b0 < nbmax; b0 += kScoreThreads) {
    const int b = b0 + lane;
    const bool ok = b < nbmax;
    uint64_t acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0ull;
#pragma unroll 4
    for (int c = 0; c < D; c += 4) {
      float kv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) kv[e] = ok ? kT[(int64_t)(c + e) * Tk + b] : 0.f;
      const uint64_t k01 = f2_pack(kv[0], kv[1]), k23 = f2_pack(kv[2], kv[3]);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float4 qv = *reinterpret_cast<const float4*>(qb + r * D + c);
        acc[r] = f2_fma(f2_pack(qv.x, qv.y), k01, acc[r]);
        acc[r] = f2_fma(f2_pack(qv.z, qv.w), k23, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (b < nb[r]) {
        float lo, hi;
        f2_unpack(acc[r], lo, hi);
        buf[r * ld + b] = (lo + hi) * p.scale;
      }
    }
  }
  __syncthreads();

  // Softmax per row (warp per row): m~ to shared memory and to m_pool; entries
  // from nb_r up to the 4-block boundary of the longest row are zeroed.
  for (int r = warp; r < R; r += kScoreWarps) {
    float* row = buf + r * ld;
    const int n = (s_tile[r] >= 0) ? t0 + s_tile[r] + 1 : 0;
    if (n > 0) {
      float mx = -INFINITY;
      for (int b = lane; b < n; b += 32) mx = fmaxf(mx, row[b]);
      mx = warp_max(mx);
      float den = 0.f;
      for (int b = lane; b < n; b += 32) {
        const float e = expf(row[b] - mx);
        row[b] = e;
        den += e;
      }
      den = warp_sum(den);
      const float inv = 1.0f / den;
      float* dst = p.m_pool + row_off(T, t0, s_head[r], s_tile[r]);
      for (int b = lane; b < n; b += 32) {
        const float m = row[b] * inv;
        row[b] = m;
        dst[b] = m;
      }
    }
    for (int b = n + lane; b < nb4; b += 32) row[b] = 0.f;
  }
  __syncthreads();

  // o~ = sum_b m~_b v~_b: thread per (slice, channel), four blocks per step.
  {
    const int c = threadIdx.x % D;
    const int sl = threadIdx.x / D;
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    for (int b4 = sl * 4; b4 < nb4; b4 += 4 * S) {
      float vv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) vv[e] = (b4 + e < nbmax) ? vb[(int64_t)(b4 + e) * D + c] : 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float4 m = *reinterpret_cast<const float4*>(buf + r * ld + b4);
        acc[r] = fmaf(m.x, vv[0], acc[r]);
        acc[r] = fmaf(m.y, vv[1], acc[r]);
        acc[r] = fmaf(m.z, vv[2], acc[r]);
        acc[r] = fmaf(m.w, vv[3], acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) part[(sl * R + r) * D + c] = acc[r];
  }
  __syncthreads();
  for (int x = threadIdx.x; x < R * D; x += kScoreThreads) {
    float a = 0.f;
#pragma unroll
    for (int sl = 0; sl < S; ++sl) a += part[sl * R * D + x];
    ob[x] = a;
  }
  __syncthreads();

  // d~_b = || v~_b - o~ ||: lane per block like the logits; overwrites m~.
  const uint64_t neg1 = f2_pack(-1.f, -1.f);
  for (int b0 = warp * 32; b0 < nbmax; b0 += kScoreThreads) {
    const int b = b0 + lane;
    const bool ok = b < nbmax;
    uint64_t acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0ull;
#pragma unroll 4
    for (int c = 0; c < D; c += 4) {
      float vv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) vv[e] = ok ? vT[(int64_t)(c + e) * Tk + b] : 0.f;
      const uint64_t v01 = f2_pack(vv[0], vv[1]), v23 = f2_pack(vv[2], vv[3]);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float4 ov = *reinterpret_cast<const float4*>(ob + r * D + c);
        const uint64_t d01 = f2_fma(f2_pack(ov.x, ov.y), neg1, v01);  // v~ - o~, exactly rounded
        const uint64_t d23 = f2_fma(f2_pack(ov.z, ov.w), neg1, v23);
        acc[r] = f2_fma(d01, d01, acc[r]);
        acc[r] = f2_fma(d23, d23, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (b < nb[r]) {
        float lo, hi;
        f2_unpack(acc[r], lo, hi);
        buf[r * ld + b] = sqrtf(lo + hi);
      }
    }
  }
  __syncthreads();
  for (int r = 0; r < R; ++r) {
    if (s_tile[r] < 0) continue;
    const int n = t0 + s_tile[r] + 1;
    float* dst = p.d_pool + row_off(T, t0, s_head[r], s_tile[r]);
    for (int b = threadIdx.x; b < n; b += kScoreThreads) dst[b] = buf[r * ld + b];
  }
}

size_t pooled_smem(int R, int T, int D) {
  const int S = kScoreThreads / D;
  const int ld = (T + 3) & ~3;
  return sizeof(float) * ((size_t)(2 + S) * R * D + (size_t)R * ld);
}

template <int D, int R>
cudaError_t launch_scores_r(const PoolParams& p, cudaStream_t stream) {
  cudaError_t e = ensure_smem_limit(pooled_scores_kernel<D, R>, kPooledSmemCap);
  if (e != cudaSuccess) return e;
  const int n_tgroups = (p.n_tiles + p.tiles_per_cta - 1) / p.tiles_per_cta;
  const int grid = n_tgroups * (p.n_q_heads / p.heads_per_cta);
  pooled_scores_kernel<D, R><<<grid, kScoreThreads, pooled_smem(R, p.n_kv_tiles, D), stream>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_scores(const PoolParams& p, cudaStream_t stream) {
  switch (p.heads_per_cta * p.tiles_per_cta) {
    case 1: return launch_scores_r<D, 1>(p, stream);
    case 2: return launch_scores_r<D, 2>(p, stream);
    case 3: return launch_scores_r<D, 3>(p, stream);
    case 4: return launch_scores_r<D, 4>(p, stream);
    case 5: return launch_scores_r<D, 5>(p, stream);
    case 6: return launch_scores_r<D, 6>(p, stream);
    case 7: return launch_scores_r<D, 7>(p, stream);
    case 8: return launch_scores_r<D, 8>(p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

// Work unit of pooled_scores: the largest divisor R_h <= 8 of the group size,
// then the most adjacent tiles R_t with R_h * R_t <= 8, both within the shared
// memory cap (R_h = R_t = 1 fits up to 8192 tiles).
cudaError_t launch_pooled(int head_dim, PoolParams p, cudaStream_t stream) {
  if (p.n_tiles <= 0) return cudaSuccess;
  int rh = 1;
  for (int r = kMaxRows; r >= 1; --r)
    if (p.group % r == 0 && pooled_smem(r, p.n_kv_tiles, head_dim) <= kPooledSmemCap) {
      rh = r;
      break;
    }
  int rt = 1;
  for (int t = kMaxRows / rh; t >= 1; --t)
    if (pooled_smem(rh * t, p.n_kv_tiles, head_dim) <= kPooledSmemCap) {
      rt = t;
      break;
    }
  p.heads_per_cta = rh;
  p.tiles_per_cta = rt;
  const dim3 pg(p.n_kv_tiles, (p.n_q_heads * (head_dim / 8) + kPoolThreads - 1) / kPoolThreads, 3);
  if (head_dim == 128) {
    pool_mean_kernel<128><<<pg, kPoolThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_scores<128>(p, stream);
  }
  pool_mean_kernel<64><<<pg, kPoolThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_scores<64>(p, stream);
}

}  // namespace poem
