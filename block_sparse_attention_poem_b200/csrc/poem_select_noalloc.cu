// poem_select_noalloc.cu -- block selection for callers that cannot allocate device
// memory: the same selection kernels as poem_select, with their scratch (list
// lengths, per-row candidate lists and the error word) in a fixed array that is
// part of the library's device image instead of a caller-provided workspace.
//
// Some callers own no allocator: a serving runtime that reserves all of HBM at
// start-up and forbids libraries from growing their footprint while requests run,
// or a plug-in that is only ever handed pointers by its host process.  They can
// still pass inputs and outputs; the scratch comes from here.
//
// The array is kStaticScratchBytes (8 MiB) of device memory held by every GPU that
// loads the library, until the process exits.  All calls share it, so calls whose
// kernels overlap on the GPU (different streams, or different host threads) race
// on it: serialise them.  The first call on a device resolves the array's device
// address (once per device, with that device current) -- make that first call
// before any stream capture.
#include <cmath>
#include <cstdio>
#include <mutex>

#include "../../include/poem.h"
#include "common.cuh"

namespace poem {
void set_last_error(const char* msg);  // poem_api.cu
}  // namespace poem

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB

// In host code this name is only a host-side stand-in for the array; the device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_select_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the scratch array on the current device (resolved once).
cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_select_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" poem_status poem_select_noalloc(const poem_shape* shape, const float* I_hat, const float* m_hat,
                                           float tau, int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                           int32_t* order, void* stream) {
  size_t need = 0;
  poem_status st = poem_workspace_size(shape, nullptr, &need, nullptr);  // validates the shape
  if (st != POEM_OK) return st;
  if (need > kStaticScratchBytes) {
    char msg[200];
    std::snprintf(msg, sizeof msg,
                  "poem_select_noalloc: this shape needs %zu bytes of scratch; the static maximum is %zu bytes",
                  need, kStaticScratchBytes);
    poem::set_last_error(msg);
    return POEM_ERR_WORKSPACE;
  }
  if (!std::isfinite(tau) || tau < 0.f) return POEM_ERR_INVALID_ARG;
  if (!aligned16(I_hat) || !aligned16(m_hat) || !aligned16(row_ptr) || (col_capacity > 0 && !aligned16(col_idx)) ||
      (order && !aligned16(order)) || col_capacity < 0)
    return POEM_ERR_INVALID_ARG;
  const int T = shape->n_tokens / shape->block;
  const int G = shape->n_q_heads / shape->n_kv_heads;
  if (order && G * T > (1 << 14)) return POEM_ERR_UNSUPPORTED;

  void* base = nullptr;
  cudaError_t e = scratch_on_current_device(&base);
  if (e != cudaSuccess) return POEM_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The error word is the only part read before it is written; the list lengths
  // and per-row lists are fully rewritten by every call.
  e = cudaMemsetAsync(base, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return POEM_ERR_CUDA;

  const size_t rows = (size_t)shape->n_q_heads * T;
  uint8_t* b = static_cast<uint8_t*>(base);
  poem::SelectParams p{};
  p.I_hat = I_hat;
  p.m_hat = m_hat;
  p.ref_row_ptr = nullptr;
  p.counts = reinterpret_cast<int32_t*>(b + poem::kWsHeader);
  p.scratch = reinterpret_cast<int32_t*>(b + poem::kWsHeader + round_up(rows * sizeof(int32_t), 256));
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.order = order;
  p.col_capacity = col_capacity;
  p.n_q_heads = shape->n_q_heads;
  p.n_tiles = T;
  p.q_tile0 = shape->q_offset / shape->block;
  p.group = G;
  p.tau = (double)tau;
  p.mass_only = 0;
  p.err = poem::DevErr{reinterpret_cast<uint32_t*>(base), 0};
  e = poem::launch_select(p, s);
  return e == cudaSuccess ? POEM_OK : POEM_ERR_CUDA;
}
