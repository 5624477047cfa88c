// poem_api.cu -- host side of the C ABI declared in include/poem.h: argument
// validation, workspace layout, TMA descriptor encoding and kernel launches.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/poem.h"
#include "common.cuh"

namespace {

thread_local char g_last_error[512] = {0};
uint64_t g_wait_limit_ns = 2000000000ull;

poem_status cuda_fail(cudaError_t e, const char* where) {
  std::snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
  return POEM_ERR_CUDA;
}

poem_status arg_fail(poem_status s, const char* what) {
  std::snprintf(g_last_error, sizeof g_last_error, "%s", what);
  return s;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Layout {
  int T;       // query tiles
  int t0;      // global tile of the first query tile (q_offset / block)
  int Tk;      // key blocks (t0 + T)
  int n_kv;    // key / value tokens (q_offset + n_tokens)
  int G;       // query heads per KV head
  float scale; // softmax scale
};

constexpr int kMaxTiles = 8192;

// Shape checks shared by every entry point.
poem_status check_shape(const poem_shape* s, Layout* out) {
  if (!s) return arg_fail(POEM_ERR_INVALID_ARG, "shape is NULL");
  if (s->n_tokens <= 0 || s->n_q_heads <= 0 || s->n_kv_heads <= 0 || s->head_dim <= 0 || s->block <= 0)
    return arg_fail(POEM_ERR_INVALID_ARG, "sizes must be positive");
  if (s->n_q_heads % s->n_kv_heads) return arg_fail(POEM_ERR_INVALID_ARG, "n_q_heads % n_kv_heads != 0");
  if (s->n_tokens % s->block) return arg_fail(POEM_ERR_INVALID_ARG, "n_tokens % block != 0");
  if (s->q_offset < 0 || s->q_offset % s->block)
    return arg_fail(POEM_ERR_INVALID_ARG, "q_offset must be >= 0 and a multiple of block");
  if ((int64_t)s->q_offset + s->n_tokens > (int64_t)INT32_MAX)
    return arg_fail(POEM_ERR_INVALID_ARG, "q_offset + n_tokens overflows int32");
  if (!(s->softmax_scale >= 0.f) || !std::isfinite(s->softmax_scale))
    return arg_fail(POEM_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  if (s->head_dim != 64 && s->head_dim != 128) return arg_fail(POEM_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (s->block != 64 && s->block != 128) return arg_fail(POEM_ERR_UNSUPPORTED, "block must be 64 or 128");
  if ((s->q_offset + s->n_tokens) / s->block > kMaxTiles)
    return arg_fail(POEM_ERR_UNSUPPORTED, "more than 8192 key blocks");
  const int64_t strides[6] = {s->q_stride_tok, s->q_stride_head, s->kv_stride_tok,
                              s->kv_stride_head, s->o_stride_tok, s->o_stride_head};
  for (int64_t st : strides)
    if (st <= 0 || (st % 8) != 0 || st >= (int64_t(1) << 38))
      return arg_fail(POEM_ERR_INVALID_ARG, "strides must be positive multiples of 8 elements");
  out->T = s->n_tokens / s->block;
  out->t0 = s->q_offset / s->block;
  out->Tk = out->t0 + out->T;
  out->n_kv = s->q_offset + s->n_tokens;
  out->G = s->n_q_heads / s->n_kv_heads;
  out->scale = s->softmax_scale > 0.f ? s->softmax_scale : 1.0f / std::sqrt((float)s->head_dim);
  return POEM_OK;
}

// Entries of the per-(head, query tile, visible block) arrays (row_off layout).
size_t tri_entries(const poem_shape* s, const Layout& L) {
  return (size_t)s->n_q_heads * (size_t)poem::row_entries(L.T, L.t0);
}

// Score workspace: header (error word; the fp16-range flag of V at byte 8), the dense
// outputs o [rows, D] fp32 and log-sum-exps [rows] of the sampled queries (pass 1 ->
// pass 2), then the fp16 copy of V [n_kv, Hkv, D] for pass 1's fp16 P V contraction.
size_t score_ws_bytes(const poem_shape* s, int T) {
  const size_t rows = (size_t)s->n_q_heads * T * s->n_sample;
  const size_t vh = (size_t)(s->q_offset + s->n_tokens) * s->n_kv_heads * s->head_dim * 2;
  return poem::kWsHeader + round_up(rows * s->head_dim * sizeof(float), 256) + round_up(rows * sizeof(float), 256) +
         round_up(vh, 256);
}

size_t select_ws_bytes(const poem_shape* s, const Layout& L) {
  const size_t rows = (size_t)s->n_q_heads * L.T;
  return poem::kWsHeader + round_up(rows * sizeof(int32_t), 256) + round_up(tri_entries(s, L) * sizeof(int32_t), 256);
}

size_t fwd_ws_bytes(const poem_shape*, int) { return poem::kWsHeader; }

// Pooled means (fp32) after the header: q~ [Hq, Tq, D], then k~ channel-major
// [Hkv, D, Tk], v~ [Hkv, Tk, D] and v~ channel-major [Hkv, D, Tk].
size_t pooled_ws_bytes(const poem_shape* s, const Layout& L) {
  const size_t qn = (size_t)s->n_q_heads * L.T * s->head_dim, kn = (size_t)s->n_kv_heads * L.Tk * s->head_dim;
  return poem::kWsHeader + round_up(qn * sizeof(float), 256) + 3 * round_up(kn * sizeof(float), 256);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [n_tokens, n_heads, head_dim] bf16 viewed as a 3-D tensor (head_dim, head, token);
// box = 64 elements x 1 head x box_rows tokens, 128-byte swizzle.
poem_status make_map_3d(CUtensorMap* m, const void* base, int head_dim, int n_heads, int n_tokens, int64_t st_head,
                        int64_t st_tok, int box_rows,
                        CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto fn = encode_fn();
  if (!fn) return arg_fail(POEM_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)n_heads, (cuuint64_t)n_tokens};
  cuuint64_t strides[2] = {(cuuint64_t)st_head * 2, (cuuint64_t)st_tok * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, dtype, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled (3d) failed: %d", (int)r);
    return POEM_ERR_CUDA;
  }
  return POEM_OK;
}

// Sampled queries of q viewed as (head_dim, head, sample j, tile i): token iB + j*stride.
poem_status make_map_sampled(CUtensorMap* m, const void* base, const poem_shape* s, int T) {
  auto fn = encode_fn();
  if (!fn) return arg_fail(POEM_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  const int stride = s->block / s->n_sample;
  cuuint64_t dims[4] = {(cuuint64_t)s->head_dim, (cuuint64_t)s->n_q_heads, (cuuint64_t)s->n_sample, (cuuint64_t)T};
  cuuint64_t strides[3] = {(cuuint64_t)s->q_stride_head * 2, (cuuint64_t)s->q_stride_tok * 2 * stride,
                           (cuuint64_t)s->q_stride_tok * 2 * s->block};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)s->n_sample, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled (4d) failed: %d", (int)r);
    return POEM_ERR_CUDA;
  }
  return POEM_OK;
}

poem::DevErr dev_err(void* ws) { return poem::DevErr{reinterpret_cast<uint32_t*>(ws), g_wait_limit_ns}; }

}  // namespace

namespace poem {
void set_last_error(const char* msg) { std::snprintf(g_last_error, sizeof g_last_error, "%s", msg); }
}  // namespace poem

extern "C" {

poem_status poem_workspace_size(const poem_shape* shape, size_t* score_bytes, size_t* select_bytes,
                                size_t* fwd_bytes) {
  Layout L;
  poem_status st = check_shape(shape, &L);
  if (st != POEM_OK) return st;
  if (score_bytes) *score_bytes = score_ws_bytes(shape, L.T);
  if (select_bytes) *select_bytes = select_ws_bytes(shape, L);
  if (fwd_bytes) *fwd_bytes = fwd_ws_bytes(shape, L.T);
  return POEM_OK;
}

poem_status poem_score(const poem_shape* shape, const poem_bf16* q, const poem_bf16* k, const poem_bf16* v,
                       float* I_hat, float* m_hat, void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  poem_status st = check_shape(shape, &L);
  if (st != POEM_OK) return st;
  if (shape->n_sample != 16 || shape->block % shape->n_sample)
    return arg_fail(POEM_ERR_UNSUPPORTED, "n_sample must be 16");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(I_hat) || !aligned16(m_hat) || !aligned16(ws))
    return arg_fail(POEM_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  if (ws_bytes < score_ws_bytes(shape, L.T)) return arg_fail(POEM_ERR_WORKSPACE, "score workspace too small");
  CUtensorMap tmQs, tmK, tmV;
  if ((st = make_map_sampled(&tmQs, q, shape, L.T)) != POEM_OK) return st;
  if ((st = make_map_3d(&tmK, k, shape->head_dim, shape->n_kv_heads, L.n_kv, shape->kv_stride_head,
                        shape->kv_stride_tok, shape->block)) != POEM_OK)
    return st;
  if ((st = make_map_3d(&tmV, v, shape->head_dim, shape->n_kv_heads, L.n_kv, shape->kv_stride_head,
                        shape->kv_stride_tok, shape->block)) != POEM_OK)
    return st;
  const size_t rows = (size_t)shape->n_q_heads * L.T * shape->n_sample;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  const size_t off_o = poem::kWsHeader;
  const size_t off_lse = off_o + round_up(rows * shape->head_dim * sizeof(float), 256);
  const size_t off_vh = off_lse + round_up(rows * sizeof(float), 256);
  // dense fp16 copy of V for pass 1: [n_kv, Hkv, D], head stride D, token stride Hkv D
  CUtensorMap tmVh;
  if ((st = make_map_3d(&tmVh, base + off_vh, shape->head_dim, shape->n_kv_heads, L.n_kv, shape->head_dim,
                        (int64_t)shape->n_kv_heads * shape->head_dim, shape->block,
                        CU_TENSOR_MAP_DATA_TYPE_FLOAT16)) != POEM_OK)
    return st;
  poem::ScoreParams p{};
  p.I_hat = I_hat;
  p.m_hat = m_hat;
  p.ws_o = reinterpret_cast<float*>(base + off_o);
  p.ws_lse = reinterpret_cast<float*>(base + off_lse);
  p.v_src = reinterpret_cast<const __nv_bfloat16*>(v);
  p.v_stride_tok = shape->kv_stride_tok;
  p.v_stride_head = shape->kv_stride_head;
  p.v_half = reinterpret_cast<__half*>(base + off_vh);
  p.v_overflow = reinterpret_cast<uint32_t*>(base + 8);
  p.n_kv = L.n_kv;
  p.n_tokens = shape->n_tokens;
  p.n_q_heads = shape->n_q_heads;
  p.n_kv_heads = shape->n_kv_heads;
  p.n_tiles = L.T;
  p.q_tile0 = L.t0;
  p.group = L.G;
  p.n_sample = shape->n_sample;
  p.sample_stride = shape->block / shape->n_sample;
  p.scale_log2 = L.scale * poem::kLog2e;
  p.err = dev_err(ws);
  p.n_entries = (int64_t)tri_entries(shape, L);
  cudaError_t e = poem::launch_score(shape->head_dim, shape->block, tmQs, tmK, tmV, tmVh, p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "poem_score launch");
  return POEM_OK;
}

struct PracticalArgs {
  const float* d_pool;
  double w, gamma, rho;
  const float* gamma_heads;  // nullable
};

static poem_status select_common(const poem_shape* shape, const float* I_hat, const float* m_hat,
                                 const int32_t* ref_row_ptr, double tau, int mass_only, int32_t* row_ptr,
                                 int32_t* col_idx, int64_t col_capacity, int32_t* order, void* ws, size_t ws_bytes,
                                 void* stream, const PracticalArgs* practical = nullptr,
                                 const float* tau_heads = nullptr) {
  Layout L;
  poem_status st = check_shape(shape, &L);
  if (st != POEM_OK) return st;
  if (practical && !aligned16(practical->d_pool))
    return arg_fail(POEM_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  if ((practical && practical->gamma_heads && !aligned16(practical->gamma_heads)))
    return arg_fail(POEM_ERR_INVALID_ARG, "gamma_per_head must be 16-byte aligned");
  if ((!mass_only && !practical && !aligned16(I_hat)) || !aligned16(m_hat) || !aligned16(row_ptr) || !aligned16(ws) ||
      (col_capacity > 0 && !aligned16(col_idx)) || (order && !aligned16(order)) ||
      (mass_only && !aligned16(ref_row_ptr)))
    return arg_fail(POEM_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  if (col_capacity < 0) return arg_fail(POEM_ERR_INVALID_ARG, "col_capacity < 0");
  if (tri_entries(shape, L) > (size_t)INT32_MAX)
    return arg_fail(POEM_ERR_UNSUPPORTED, "the block lists could exceed int32 row_ptr offsets (too many heads x tiles)");
  if (!mass_only && (!std::isfinite(tau) || tau < 0.0)) return arg_fail(POEM_ERR_INVALID_ARG, "tau must be finite and >= 0");
  if (ws_bytes < select_ws_bytes(shape, L)) return arg_fail(POEM_ERR_WORKSPACE, "select workspace too small");
  if (order && L.G * L.T > (1 << 14)) return arg_fail(POEM_ERR_UNSUPPORTED, "work order needs group*tiles <= 16384");
  const size_t rows = (size_t)shape->n_q_heads * L.T;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  poem::SelectParams p{};
  p.I_hat = I_hat;
  p.m_hat = m_hat;
  p.ref_row_ptr = ref_row_ptr;
  p.counts = reinterpret_cast<int32_t*>(base + poem::kWsHeader);
  p.scratch = reinterpret_cast<int32_t*>(base + poem::kWsHeader + round_up(rows * sizeof(int32_t), 256));
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.order = order;
  p.col_capacity = col_capacity;
  p.n_q_heads = shape->n_q_heads;
  p.n_tiles = L.T;
  p.q_tile0 = L.t0;
  p.group = L.G;
  p.tau = tau;
  p.tau_heads = tau_heads;
  p.mass_only = mass_only;
  if (practical) {
    p.practical = 1;
    p.d_pool = practical->d_pool;
    p.w = practical->w;
    p.gamma = practical->gamma;
    p.gamma_heads = practical->gamma_heads;
    p.rho = practical->rho;
  }
  p.err = dev_err(ws);
  p.n_entries = (int64_t)tri_entries(shape, L);
  cudaError_t e = poem::launch_select(p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "poem_select launch");
  return POEM_OK;
}

poem_status poem_select(const poem_shape* shape, const float* I_hat, const float* m_hat, float tau,
                        int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int32_t* order, void* ws,
                        size_t ws_bytes, void* stream) {
  if (!std::isfinite(tau) || tau < 0.f) return arg_fail(POEM_ERR_INVALID_ARG, "tau must be finite and >= 0");
  return select_common(shape, I_hat, m_hat, nullptr, (double)tau, 0, row_ptr, col_idx, col_capacity, order, ws,
                       ws_bytes, stream);
}

poem_status poem_select_per_head(const poem_shape* shape, const float* I_hat, const float* m_hat,
                                 const float* tau_per_head, int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                 int32_t* order, void* ws, size_t ws_bytes, void* stream) {
  if (!aligned16(tau_per_head)) return arg_fail(POEM_ERR_INVALID_ARG, "tau_per_head must be non-NULL and 16-byte aligned");
  return select_common(shape, I_hat, m_hat, nullptr, 0.0, 0, row_ptr, col_idx, col_capacity, order, ws, ws_bytes,
                       stream, nullptr, tau_per_head);
}

poem_status poem_select_mass_only(const poem_shape* shape, const float* m_hat, const int32_t* ref_row_ptr,
                                  int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int32_t* order,
                                  void* ws, size_t ws_bytes, void* stream) {
  return select_common(shape, nullptr, m_hat, ref_row_ptr, 0.0, 1, row_ptr, col_idx, col_capacity, order, ws,
                       ws_bytes, stream);
}

poem_status poem_select_ranked_budget(const poem_shape* shape, const float* score, const int32_t* ref_row_ptr,
                                      int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int32_t* order,
                                      void* ws, size_t ws_bytes, void* stream) {
  return select_common(shape, nullptr, score, ref_row_ptr, 0.0, 1, row_ptr, col_idx, col_capacity, order, ws,
                       ws_bytes, stream);
}

poem_status poem_pooled_workspace_size(const poem_shape* shape, size_t* pooled_bytes) {
  Layout L;
  poem_status st = check_shape(shape, &L);
  if (st != POEM_OK) return st;
  if (pooled_bytes) *pooled_bytes = pooled_ws_bytes(shape, L);
  return POEM_OK;
}

poem_status poem_score_pooled(const poem_shape* shape, const poem_bf16* q, const poem_bf16* k, const poem_bf16* v,
                              float* m_pool, float* d_pool, void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  poem_status st = check_shape(shape, &L);
  if (st != POEM_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(m_pool) || !aligned16(d_pool) || !aligned16(ws))
    return arg_fail(POEM_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  if (ws_bytes < pooled_ws_bytes(shape, L)) return arg_fail(POEM_ERR_WORKSPACE, "pooled workspace too small");
  const size_t qn = (size_t)shape->n_q_heads * L.T * shape->head_dim;
  const size_t kn = (size_t)shape->n_kv_heads * L.Tk * shape->head_dim;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws) + poem::kWsHeader;
  poem::PoolParams p{};
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.k = reinterpret_cast<const __nv_bfloat16*>(k);
  p.v = reinterpret_cast<const __nv_bfloat16*>(v);
  p.q_stride_tok = shape->q_stride_tok;
  p.q_stride_head = shape->q_stride_head;
  p.kv_stride_tok = shape->kv_stride_tok;
  p.kv_stride_head = shape->kv_stride_head;
  const size_t qb = round_up(qn * sizeof(float), 256), kb = round_up(kn * sizeof(float), 256);
  p.q_bar = reinterpret_cast<float*>(base);
  p.k_bar_t = reinterpret_cast<float*>(base + qb);
  p.v_bar = reinterpret_cast<float*>(base + qb + kb);
  p.v_bar_t = reinterpret_cast<float*>(base + qb + 2 * kb);
  p.m_pool = m_pool;
  p.d_pool = d_pool;
  p.n_q_heads = shape->n_q_heads;
  p.n_kv_heads = shape->n_kv_heads;
  p.n_tiles = L.T;
  p.n_kv_tiles = L.Tk;
  p.q_tile0 = L.t0;
  p.block = shape->block;
  p.group = L.G;
  p.scale = L.scale;
  p.err = dev_err(ws);
  cudaError_t e = poem::launch_pooled(shape->head_dim, p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "poem_score_pooled launch");
  return POEM_OK;
}

poem_status poem_select_practical(const poem_shape* shape, const float* m_pool, const float* d_pool, double w,
                                  double gamma, double rho, int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                  int32_t* order, void* ws, size_t ws_bytes, void* stream) {
  if (!std::isfinite(w) || w < 0.0) return arg_fail(POEM_ERR_INVALID_ARG, "w must be finite and >= 0");
  if (std::isnan(gamma)) return arg_fail(POEM_ERR_INVALID_ARG, "gamma is NaN");
  if (!(rho >= 0.0 && rho <= 1.0)) return arg_fail(POEM_ERR_INVALID_ARG, "rho must lie in [0, 1]");
  PracticalArgs pa{d_pool, w, gamma, rho, nullptr};
  return select_common(shape, nullptr, m_pool, nullptr, 0.0, 0, row_ptr, col_idx, col_capacity, order, ws, ws_bytes,
                       stream, &pa);
}

poem_status poem_select_practical_per_head(const poem_shape* shape, const float* m_pool, const float* d_pool, double w,
                                           const float* gamma_per_head, double rho, int32_t* row_ptr,
                                           int32_t* col_idx, int64_t col_capacity, int32_t* order, void* ws,
                                           size_t ws_bytes, void* stream) {
  if (!std::isfinite(w) || w < 0.0) return arg_fail(POEM_ERR_INVALID_ARG, "w must be finite and >= 0");
  if (!(rho >= 0.0 && rho <= 1.0)) return arg_fail(POEM_ERR_INVALID_ARG, "rho must lie in [0, 1]");
  if (!aligned16(gamma_per_head))
    return arg_fail(POEM_ERR_INVALID_ARG, "gamma_per_head must be non-NULL and 16-byte aligned");
  PracticalArgs pa{d_pool, w, 0.0, rho, gamma_per_head};
  return select_common(shape, nullptr, m_pool, nullptr, 0.0, 0, row_ptr, col_idx, col_capacity, order, ws, ws_bytes,
                       stream, &pa);
}

// Checks, tensor maps and parameter block shared by bsa_fwd and bsa_fwd_grouped.
static poem_status fwd_setup(const poem_shape* shape, const void* q, const void* k, const void* v,
                             const int32_t* row_ptr, const int32_t* col_idx, const int32_t* order, void* o,
                             float* lse, void* ws, size_t ws_bytes, Layout* L, CUtensorMap* tmQ, CUtensorMap* tmK,
                             CUtensorMap* tmV, poem::FwdParams* p) {
  poem_status st = check_shape(shape, L);
  if (st != POEM_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(row_ptr) || !aligned16(o) || !aligned16(ws) ||
      (col_idx && !aligned16(col_idx)) || (order && !aligned16(order)) || (lse && !aligned16(lse)))
    return arg_fail(POEM_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  if (ws_bytes < fwd_ws_bytes(shape, L->T)) return arg_fail(POEM_ERR_WORKSPACE, "fwd workspace too small");
  if ((st = make_map_3d(tmQ, q, shape->head_dim, shape->n_q_heads, shape->n_tokens, shape->q_stride_head,
                        shape->q_stride_tok, 128)) != POEM_OK)
    return st;
  if ((st = make_map_3d(tmK, k, shape->head_dim, shape->n_kv_heads, L->n_kv, shape->kv_stride_head,
                        shape->kv_stride_tok, shape->block)) != POEM_OK)
    return st;
  if ((st = make_map_3d(tmV, v, shape->head_dim, shape->n_kv_heads, L->n_kv, shape->kv_stride_head,
                        shape->kv_stride_tok, shape->block)) != POEM_OK)
    return st;
  *p = poem::FwdParams{};
  p->row_ptr = row_ptr;
  p->col_idx = col_idx;
  p->order = order;
  p->o = reinterpret_cast<__nv_bfloat16*>(o);
  p->lse = lse;
  p->o_stride_tok = shape->o_stride_tok;
  p->o_stride_head = shape->o_stride_head;
  p->n_tokens = shape->n_tokens;
  p->n_q_heads = shape->n_q_heads;
  p->n_tiles = L->T;
  p->q_tile0 = L->t0;
  p->group = L->G;
  p->scale_log2 = L->scale * poem::kLog2e;
  p->err = dev_err(ws);
  return POEM_OK;
}

poem_status bsa_fwd(const poem_shape* shape, const poem_bf16* q, const poem_bf16* k, const poem_bf16* v,
                    const int32_t* row_ptr, const int32_t* col_idx, const int32_t* order, poem_bf16* o, float* lse,
                    void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  CUtensorMap tmQ, tmK, tmV;
  poem::FwdParams p;
  poem_status st = fwd_setup(shape, q, k, v, row_ptr, col_idx, order, o, lse, ws, ws_bytes, &L, &tmQ, &tmK, &tmV, &p);
  if (st != POEM_OK) return st;
  cudaError_t e = poem::launch_bsa_fwd(shape->head_dim, shape->block, tmQ, tmK, tmV, p, shape->n_q_heads * L.T,
                                       (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "bsa_fwd launch");
  return POEM_OK;
}

poem_status bsa_fwd_grouped(const poem_shape* shape, const poem_bf16* q, const poem_bf16* k, const poem_bf16* v,
                            const int32_t* row_ptr, const int32_t* col_idx, poem_bf16* o, float* lse, void* ws,
                            size_t ws_bytes, void* stream) {
  Layout L;
  CUtensorMap tmQ, tmK, tmV;
  poem::FwdParams p;
  poem_status st = fwd_setup(shape, q, k, v, row_ptr, col_idx, nullptr, o, lse, ws, ws_bytes, &L, &tmQ, &tmK, &tmV, &p);
  if (st != POEM_OK) return st;
  cudaError_t e = poem::launch_bsa_fwd_grouped(shape->head_dim, shape->block, tmQ, tmK, tmV, p, shape->n_kv_heads,
                                               (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "bsa_fwd_grouped launch");
  return POEM_OK;
}

poem_status poem_check(void* stream, void* ws) {
  if (!aligned16(ws)) return arg_fail(POEM_ERR_INVALID_ARG, "ws must be non-NULL and 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof word, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "poem_check");
  if (word) {
    e = cudaMemsetAsync(ws, 0, sizeof word, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "poem_check reset");
  }
  if (word & poem::kErrTimeout) return POEM_ERR_TIMEOUT;
  if (word & poem::kErrBadList) return POEM_ERR_BAD_LIST;
  if (word & poem::kErrCapacity) return POEM_ERR_CAPACITY;
  if (word & poem::kErrBadParam) return POEM_ERR_INVALID_ARG;
  if (word & poem::kErrBounds)
    return arg_fail(POEM_ERR_BOUNDS, "a device bounds check of the debug build failed (the access was skipped)");
  return POEM_OK;
}

void poem_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns; }

const char* poem_status_string(poem_status s) {
  switch (s) {
    case POEM_OK: return "POEM_OK";
    case POEM_ERR_INVALID_ARG: return "POEM_ERR_INVALID_ARG";
    case POEM_ERR_UNSUPPORTED: return "POEM_ERR_UNSUPPORTED";
    case POEM_ERR_CUDA: return "POEM_ERR_CUDA";
    case POEM_ERR_TIMEOUT: return "POEM_ERR_TIMEOUT";
    case POEM_ERR_CAPACITY: return "POEM_ERR_CAPACITY";
    case POEM_ERR_WORKSPACE: return "POEM_ERR_WORKSPACE";
    case POEM_ERR_BAD_LIST: return "POEM_ERR_BAD_LIST";
    case POEM_ERR_BOUNDS: return "POEM_ERR_BOUNDS";
  }
  return "POEM_ERR_UNKNOWN";
}

const char* poem_last_error(void) { return g_last_error; }

}  // extern "C"
