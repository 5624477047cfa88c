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
//                  streaming loads, in fp32, and writes the mean.  HBM-bound:
//                  reads Q, K and V once.
//   pooled_scores  one CTA per (tile i, R query heads sharing a KV head), large
//                  tiles first: logits by warp-per-block dot products (lane slices
//                  of the channels, butterfly reduction), softmax per row, o~ with
//                  threads over channels, then d~ like the logits.  k~ and v~ of a
//                  KV head (T * D * 4 bytes each) stay in L2 across its CTAs.
#include "common.cuh"

namespace poem {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kScoreThreads = 256;
constexpr int kMaxRows = 8;
constexpr size_t kPooledSmemCap = 200 * 1024;

__device__ __forceinline__ int64_t tri_off(int n_tiles, int h, int i) {
  return (int64_t)h * ((int64_t)n_tiles * (n_tiles + 1) / 2) + (int64_t)i * (i + 1) / 2;
}

template <int D>
__global__ void __launch_bounds__(kPoolThreads) pool_mean_kernel(const PoolParams p) {
  constexpr int C8 = D / 8;
  const int which = blockIdx.z;  // 0: q, 1: k, 2: v
  const int heads = which == 0 ? p.n_q_heads : p.n_kv_heads;
  const int u = blockIdx.y * kPoolThreads + threadIdx.x;
  if (u >= heads * C8) return;
  const int h = u / C8;
  const int c8 = u - h * C8;
  const int i = blockIdx.x;
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
      acc[2 * e] += __uint_as_float(ws[e] << 16);
      acc[2 * e + 1] += __uint_as_float(ws[e] & 0xffff0000u);
    }
  }
  const float inv = 1.0f / (float)p.block;
  float* dst = (which == 0 ? p.q_bar : (which == 1 ? p.k_bar : p.v_bar)) + ((int64_t)h * p.n_tiles + i) * D + c8 * 8;
  reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  reinterpret_cast<float4*>(dst)[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
}

// Lane slice of a D-channel fp32 row: E = D / 32 consecutive channels per lane.
template <int E>
struct Slice {
  float x[E];
};

template <int E>
__device__ __forceinline__ Slice<E> load_slice(const float* row, int lane) {
  Slice<E> s;
  if constexpr (E == 4) {
    const float4 v = *reinterpret_cast<const float4*>(row + lane * 4);
    s.x[0] = v.x; s.x[1] = v.y; s.x[2] = v.z; s.x[3] = v.w;
  } else {
    const float2 v = *reinterpret_cast<const float2*>(row + lane * 2);
    s.x[0] = v.x; s.x[1] = v.y;
  }
  return s;
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
  constexpr int E = D / 32;
  constexpr int S = kScoreThreads / D;  // channel-parallel slices of the o~ pass
  constexpr int W = kScoreThreads / 32;
  extern __shared__ __align__(16) float smf[];
  const int T = p.n_tiles;
  const int ld = (T + 3) & ~3;
  float* qb = smf;             // [R][D]
  float* ob = qb + R * D;      // [R][D]
  float* part = ob + R * D;    // [S][R][D]
  float* buf = part + S * R * D;  // [R][ld]: logits -> m~ -> d~

  const int n_chunks = p.n_q_heads / R;
  const int u = blockIdx.x;
  const int i = T - 1 - u / n_chunks;
  const int h0 = (u - (u / n_chunks) * n_chunks) * R;
  const int g = h0 / p.group;
  const int nb = i + 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* kbar = p.k_bar + (int64_t)g * T * D;
  const float* vbar = p.v_bar + (int64_t)g * T * D;

  for (int x = threadIdx.x; x < R * D; x += kScoreThreads) {
    const int r = x / D, c = x - r * D;
    qb[x] = p.q_bar[((int64_t)(h0 + r) * T + i) * D + c];
  }
  __syncthreads();

  // Logits: warp per block, lane slices of the channels.
  {
    Slice<E> qs[R];
#pragma unroll
    for (int r = 0; r < R; ++r) qs[r] = load_slice<E>(qb + r * D, lane);
    for (int b = warp; b < nb; b += W) {
      const Slice<E> ks = load_slice<E>(kbar + (int64_t)b * D, lane);
      float s[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) a = fmaf(qs[r].x[e], ks.x[e], a);
        s[r] = warp_sum(a);
      }
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (lane == r) buf[r * ld + b] = s[r] * p.scale;
    }
  }
  __syncthreads();

  // Softmax per row (warp per row): m~ to shared memory and to m_pool.
  for (int r = warp; r < R; r += W) {
    float* row = buf + r * ld;
    float mx = -INFINITY;
    for (int b = lane; b < nb; b += 32) mx = fmaxf(mx, row[b]);
    mx = warp_max(mx);
    float den = 0.f;
    for (int b = lane; b < nb; b += 32) {
      const float e = expf(row[b] - mx);
      row[b] = e;
      den += e;
    }
    den = warp_sum(den);
    const float inv = 1.0f / den;
    float* dst = p.m_pool + tri_off(T, h0 + r, i);
    for (int b = lane; b < nb; b += 32) {
      const float m = row[b] * inv;
      row[b] = m;
      dst[b] = m;
    }
  }
  __syncthreads();

  // o~ = sum_b m~_b v~_b: thread per (slice, channel), slices interleave blocks.
  {
    const int c = threadIdx.x % D;
    const int sl = threadIdx.x / D;
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    for (int b = sl; b < nb; b += S) {
      const float vv = vbar[(int64_t)b * D + c];
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = fmaf(buf[r * ld + b], vv, acc[r]);
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

  // d~_b = || v~_b - o~ ||, like the logits; overwrites m~ in shared memory.
  {
    Slice<E> os[R];
#pragma unroll
    for (int r = 0; r < R; ++r) os[r] = load_slice<E>(ob + r * D, lane);
    for (int b = warp; b < nb; b += W) {
      const Slice<E> vs = load_slice<E>(vbar + (int64_t)b * D, lane);
      float s[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const float df = vs.x[e] - os[r].x[e];
          a = fmaf(df, df, a);
        }
        s[r] = warp_sum(a);
      }
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (lane == r) buf[r * ld + b] = sqrtf(s[r]);
    }
  }
  __syncthreads();
  for (int r = 0; r < R; ++r) {
    float* dst = p.d_pool + tri_off(T, h0 + r, i);
    for (int b = threadIdx.x; b < nb; b += kScoreThreads) dst[b] = buf[r * ld + b];
  }
}

size_t pooled_smem(int R, int T, int D) {
  const int S = kScoreThreads / D;
  const int ld = (T + 3) & ~3;
  return sizeof(float) * ((size_t)(2 + S) * R * D + (size_t)R * ld);
}

template <int D, int R>
cudaError_t launch_scores_r(const PoolParams& p, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(pooled_scores_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kPooledSmemCap);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int grid = p.n_tiles * (p.n_q_heads / R);
  pooled_scores_kernel<D, R><<<grid, kScoreThreads, pooled_smem(R, p.n_tiles, D), stream>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_scores(const PoolParams& p, cudaStream_t stream) {
  switch (p.rows_per_cta) {
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

// Rows per CTA: the largest divisor of the group size that is <= 8 and whose
// shared-memory footprint fits the cap (R = 1 always fits up to 8192 tiles).
int pooled_rows_per_cta(int group, int n_tiles, int head_dim) {
  for (int r = kMaxRows; r >= 1; --r)
    if (group % r == 0 && pooled_smem(r, n_tiles, head_dim) <= kPooledSmemCap) return r;
  return 1;
}

cudaError_t launch_pooled(int head_dim, const PoolParams& p, cudaStream_t stream) {
  if (p.n_tiles <= 0) return cudaSuccess;
  const dim3 pg(p.n_tiles, (p.n_q_heads * (head_dim / 8) + kPoolThreads - 1) / kPoolThreads, 3);
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
