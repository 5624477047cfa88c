// fwd_common.cuh -- device helpers shared by the attention-forward kernels
// (bsa_fwd.cu, bsa_fwd_grouped.cu): the visible-block test, the bounded mbarrier wait
// that also gives up once another role has aborted, and the exponentials of one S row
// (online softmax of the reading note "Attention deletion error", Section 4.1).
#pragma once
#include "common.cuh"

namespace poem {
namespace fwd {

__device__ __forceinline__ bool block_ok(int id, int tile) { return id >= 0 && id <= tile; }

// Bounded wait that also gives up as soon as another role has aborted.
template <typename Barriers>  // any barrier block with a volatile int abort_flag
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Barriers* sb, const DevErr& e) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (sb->abort_flag) return false;
    if (globaltimer_ns() - t0 > e.timeout_ns) {
      sb->abort_flag = 1;
      raise_err(e, kErrTimeout);
      return false;
    }
  }
}

// The same wait made by a whole warp, with a warp-uniform result.
template <typename Barriers>
__device__ __forceinline__ bool warp_wait_or_abort(uint64_t* bar, uint32_t parity, Barriers* sb, const DevErr& e) {
  return __all_sync(0xffffffffu, wait_or_abort(bar, parity, sb, e));
}

constexpr uint64_t kDrainNs = 2000000000ull;  // waits for already-issued async work

// Exponentials of one S row (re-read from TMEM in 64-column halves), the bf16 P
// written over the first BN/2 TMEM columns of S, and the row sum added to *l.
// On the diagonal block the masked columns get weight exactly zero.
template <int BN, bool DIAG>
__device__ __forceinline__ void exp_pack_store(uint32_t tS, float sl2, float m_use, int lim, float* l,
                                               uint64_t* p_half) {
  const uint64_t scale2 = f2_pack(sl2, sl2);
  const uint64_t negm2 = f2_pack(-m_use, -m_use);
  uint64_t acc = f2_pack(0.f, 0.f);
#pragma unroll
  for (int hf = 0; hf < BN / 64; ++hf) {
    // re-read 64 S columns; the P words of this half go to columns [32 hf, 32 hf + 32),
    // which hold S values already read
    uint32_t a[2][32];
    tmem_ld32(tS + hf * 64, a[0]);
    tmem_ld32(tS + hf * 64 + 32, a[1]);
    tmem_ld_wait();
    tmem_reg_fence(a[0]);
    tmem_reg_fence(a[1]);
    uint32_t packed[32];
#pragma unroll
    for (int x = 0; x < 32; ++x) {
      const uint32_t* src = a[x >> 4];
      const int k = (2 * x) & 31;
      const uint64_t xv = f2_fma(f2_pack(__uint_as_float(src[k]), __uint_as_float(src[k + 1])), scale2, negm2);
      float x0, x1, y0, y1;
      f2_unpack(xv, x0, x1);
      if (DIAG) {
        y0 = (hf * 64 + 2 * x <= lim) ? ex2_approx(x0) : 0.f;
        y1 = (hf * 64 + 2 * x + 1 <= lim) ? ex2_approx(x1) : 0.f;
      } else {
        y0 = ex2_approx(x0);
        y1 = ex2_approx(x1);
      }
      acc = f2_add(acc, f2_pack(y0, y1));
      packed[x] = pack_bf16x2(y0, y1);
    }
    tmem_st32(tS + hf * 32, packed);
    // this half of P (and any O rescale before it) is in TMEM: its P V MMAs may start
    tmem_st_wait();
    tc_fence_before();
    warp_arrive(&p_half[hf]);
  }
  float a0, a1;
  f2_unpack(acc, a0, a1);
  *l += a0 + a1;
}

}  // namespace fwd
}  // namespace poem
