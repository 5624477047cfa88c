// common.cuh -- parameter blocks shared by the host entry points and the kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <utility>

#include "sm100.cuh"

namespace poem {

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the current
// device.  The attribute is per device, so the setting is remembered per (kernel,
// device); thread-safe.  Sizes up to the 48 KB default need no call.
template <typename F>
inline cudaError_t ensure_smem_limit(F* func, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(reinterpret_cast<const void*>(func), dev);
  const auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done[key] = bytes;
  return e;
}

constexpr int kWsHeader = 256;          // bytes reserved at the start of every workspace
constexpr int kThreadsFwd = 192;        // 4 softmax warps + 1 TMA warp + 1 MMA warp
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Launch order of the (head, tile) rows of a layer when no explicit order is
// given: KV-head-major (so the CTAs that run together share one KV head's keys
// and values in L2), last tile first (longest causal rows first), and the query
// heads of a group next to each other.
__host__ __device__ __forceinline__ int default_row_of_unit(int u, int n_tiles, int group) {
  const int per_g = n_tiles * group;
  const int g = u / per_g;
  const int rem = u - g * per_g;
  const int i = n_tiles - 1 - rem / group;
  const int h = g * group + rem % group;
  return h * n_tiles + i;
}

// Offset of row (head h, local query tile i) in the packed per-(head, tile, block)
// arrays (scores, estimates, per-row scratch lists).  Local tile i is global tile
// t0 + i (t0 = query offset / block) and has t0 + i + 1 visible key blocks, so
// each head holds E = Tq t0 + Tq (Tq + 1) / 2 entries; t0 = 0 gives the plain
// lower-triangular layout h T (T + 1) / 2 + i (i + 1) / 2.
__host__ __device__ __forceinline__ int64_t row_entries(int n_q_tiles, int t0) {
  return (int64_t)n_q_tiles * t0 + (int64_t)n_q_tiles * (n_q_tiles + 1) / 2;
}
__host__ __device__ __forceinline__ int64_t row_off(int n_q_tiles, int t0, int h, int i) {
  return (int64_t)h * row_entries(n_q_tiles, t0) + (int64_t)i * t0 + (int64_t)i * (i + 1) / 2;
}

struct FwdParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int32_t* order;
  __nv_bfloat16* o;
  float* lse;
  int64_t o_stride_tok;
  int64_t o_stride_head;
  int n_tokens;       // query tokens (rows of q, o and lse)
  int n_q_heads;
  int n_tiles;        // query tiles
  int q_tile0;        // global tile of the first query tile (query offset / block)
  int group;          // query heads per KV head
  float scale_log2;   // softmax_scale * log2(e)
  DevErr err;
};

struct ScoreParams {
  float* I_hat;        // packed lower-triangular [Hq, T(T+1)/2]
  float* m_hat;
  float* ws_o;         // [Hq, T, S, D] fp32 dense outputs of the sampled queries
  float* ws_lse;       // [Hq, T, S] fp32 log2-domain log-sum-exp (scaled logits)
  int n_tokens;
  int n_q_heads;
  int n_kv_heads;
  int n_tiles;         // query tiles
  int q_tile0;         // global tile of the first query tile
  int group;
  int n_sample;        // S
  int sample_stride;   // B / S
  float scale_log2;
  DevErr err;
  int64_t n_entries;     // entries of I_hat / m_hat (bounds of the debug build)
  // Pass 1 runs the P V contraction of CTAs whose tiles are all >= 32 with one fp16
  // P on a dense fp16 copy of V; a finite |v| outside the fp16 range sets
  // *v_overflow and every CTA takes the bf16 hi/lo contraction instead.
  const __nv_bfloat16* v_src;
  int64_t v_stride_tok, v_stride_head;
  __half* v_half;        // [n_kv, Hkv, D]
  uint32_t* v_overflow;  // in the workspace header (byte 8)
  int n_kv;              // key / value tokens (q_offset + n_tokens)
};

struct SelectParams {
  const float* I_hat;
  const float* m_hat;
  const int32_t* ref_row_ptr;  // mass-only: budget source (nullable)
  int32_t* counts;             // [rows] list lengths
  int32_t* scratch;            // [Hq * T(T+1)/2] ids at each row's triangular offset
  int32_t* row_ptr;
  int32_t* col_idx;
  int32_t* order;
  int64_t col_capacity;
  int n_q_heads;
  int n_tiles;   // query tiles
  int q_tile0;   // global tile of the first query tile
  int group;
  double tau;
  const float* tau_heads;  // nullable: per-query-head tau (device, [n_q_heads]) instead of tau
  int mass_only;
  // Practical selector (pooled estimates): m_hat holds m~, d_pool holds d~.
  const float* d_pool;
  double w;      // weight of log d~ in the rerank key
  double gamma;  // pooled-mass retention threshold
  const float* gamma_heads;  // nullable: per-query-head gamma (device, [n_q_heads]) instead of gamma
  double rho;    // stage-1 shortlist fraction of the candidates
  int practical;
  DevErr err;
  int64_t n_entries;  // entries of the per-row scratch (bounds of the debug build)
};

// Mean pooling and pooled score estimates for the practical selector.
struct PoolParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  int64_t q_stride_tok, q_stride_head;
  int64_t kv_stride_tok, kv_stride_head;
  float* q_bar;    // [Hq, Tq, D] fp32 tile means of the queries
  float* k_bar_t;  // [Hkv, D, Tk] fp32 block means of the keys, channel-major
  float* v_bar;    // [Hkv, Tk, D] fp32 block means of the values
  float* v_bar_t;  // [Hkv, D, Tk] the same, channel-major
  float* m_pool;   // packed per (head, query tile) rows (row_off): m~
  float* d_pool;   //                                                d~
  int n_q_heads;
  int n_kv_heads;
  int n_tiles;     // query tiles Tq
  int n_kv_tiles;  // key blocks Tk = q_tile0 + Tq
  int q_tile0;
  int block;
  int group;
  int heads_per_cta;  // query heads of one KV head per CTA (divides group)
  int tiles_per_cta;  // adjacent query tiles per CTA; heads * tiles <= 8
  float scale;        // softmax scale (natural-log domain)
  DevErr err;
};

// Launchers (defined in the kernel translation units).
cudaError_t launch_bsa_fwd(int head_dim, int block, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const FwdParams& p, int n_units, cudaStream_t stream);
cudaError_t launch_bsa_fwd_grouped(int head_dim, int block, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                   const CUtensorMap& tmV, const FwdParams& p, int n_kv_heads, cudaStream_t stream);
cudaError_t launch_score(int head_dim, int block, const CUtensorMap& tmQs, const CUtensorMap& tmK,
                         const CUtensorMap& tmV, const CUtensorMap& tmVh, const ScoreParams& p, cudaStream_t stream);
cudaError_t launch_score_pass1(int head_dim, int block, const CUtensorMap& tmQs, const CUtensorMap& tmK,
                               const CUtensorMap& tmV, const CUtensorMap& tmVh, const ScoreParams& p, int grid,
                               cudaStream_t stream);
cudaError_t launch_v_to_half(const ScoreParams& p, int head_dim, cudaStream_t stream);
cudaError_t launch_select(const SelectParams& p, cudaStream_t stream);
cudaError_t launch_pooled(int head_dim, PoolParams p, cudaStream_t stream);

}  // namespace poem
