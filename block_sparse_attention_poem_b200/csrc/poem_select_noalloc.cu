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
// The array is kStaticScratchBytes (8 MiB) of device memory.  It belongs to this
// file's device module, which CUDA (lazy module loading, the default) loads on a
// device the first time the array's address is asked for there -- the first call
// of poem_select_noalloc on that device.  That call commits the 8 MiB, which the
// device then holds until the process exits; a caller that reserves device memory
// up front makes this first call before the reservation.  All calls share the
// array, so calls whose kernels overlap on the GPU (different streams, or different
// host threads) race on it: serialise them.  The address is resolved once per
// device, with that device current; make the first call before any stream capture.
// A cached address that no longer names device memory (after cudaDeviceReset) is
// detected on the host and resolved again.
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

poem_status fail(poem_status s, const char* what) {
  poem::set_last_error(what);
  return s;
}

poem_status cuda_fail(cudaError_t e, const char* where) {
  char msg[256];
  std::snprintf(msg, sizeof msg, "poem_select_noalloc: %s: %s (%s)", where, cudaGetErrorName(e),
                cudaGetErrorString(e));
  poem::set_last_error(msg);
  return POEM_ERR_CUDA;
}

// True when `ptr` still names device memory of device `dev` (a host-side query; it
// enqueues no work).
bool still_device_memory(void* ptr, int dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
    (void)cudaGetLastError();  // the query's failure is not the caller's error
    return false;
  }
  return a.type == cudaMemoryTypeDevice && a.device == dev;
}

// Device address of the scratch array on the current device (resolved once per
// device; resolved again if the cached address no longer names device memory).
cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_addr[dev] && !still_device_memory(g_scratch_addr[dev], dev)) g_scratch_addr[dev] = nullptr;
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_select_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

void forget_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_scratch_addr[dev] = nullptr;
}

}  // namespace

extern "C" poem_status poem_select_noalloc(const poem_shape* shape, const float* I_hat, const float* m_hat,
                                           float tau, int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                           int32_t* order, void* stream) {
  size_t need = 0;
  poem_status st = poem_workspace_size(shape, nullptr, &need, nullptr);  // validates the shape, sets the message
  if (st != POEM_OK) return st;
  if (need > kStaticScratchBytes) {
    char msg[200];
    std::snprintf(msg, sizeof msg,
                  "poem_select_noalloc: this shape needs %zu bytes of scratch; the static maximum is %zu bytes",
                  need, kStaticScratchBytes);
    return fail(POEM_ERR_WORKSPACE, msg);
  }
  if (!std::isfinite(tau) || tau < 0.f) return fail(POEM_ERR_INVALID_ARG, "poem_select_noalloc: tau must be finite and >= 0");
  if (col_capacity < 0) return fail(POEM_ERR_INVALID_ARG, "poem_select_noalloc: col_capacity < 0");
  if (!aligned16(I_hat) || !aligned16(m_hat) || !aligned16(row_ptr) || (col_capacity > 0 && !aligned16(col_idx)) ||
      (order && !aligned16(order)))
    return fail(POEM_ERR_INVALID_ARG, "poem_select_noalloc: pointers must be non-NULL and 16-byte aligned");
  const int T = shape->n_tokens / shape->block;
  const int G = shape->n_q_heads / shape->n_kv_heads;
  if (order && G * T > (1 << 14))
    return fail(POEM_ERR_UNSUPPORTED, "poem_select_noalloc: work order needs group*tiles <= 16384");

  void* base = nullptr;
  cudaError_t e = scratch_on_current_device(&base);
  if (e != cudaSuccess) return cuda_fail(e, "resolving the scratch array");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The error word is the only part read before it is written; the list lengths
  // and per-row lists are fully rewritten by every call.
  e = cudaMemsetAsync(base, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) {
    forget_current_device();
    return cuda_fail(e, "clearing the error word");
  }

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
  p.n_entries = (int64_t)shape->n_q_heads * poem::row_entries(T, p.q_tile0);
  e = poem::launch_select(p, s);
  if (e != cudaSuccess) {
    forget_current_device();
    return cuda_fail(e, "selection launch");
  }
  return POEM_OK;
}
