// score_common.cuh -- device helpers shared by the two score passes (poem_score.cu,
// poem_score_pass1.cu): the exponentials of one sampled-query row of S written back
// as a bf16 hi/lo pair or as one fp16 P for the P V contraction, and the row maximum
// of S.
#pragma once
#include "common.cuh"

namespace poem {
namespace score {

// A CTA whose smallest global query tile is at least this takes the single fp16 P
// (with V in fp16) in both passes; earlier tiles take the bf16 hi/lo pair.  On the
// first tiles one or a few blocks carry nearly all of a query's mass, r_b cancels
// almost exactly against m_b o, and the fp16 rounding of P would dominate I_b.
constexpr int kHalfMinTile = 32;

// p = 2^(s * scale * log2e - m) for one row's BN scores (re-read from TMEM in 64-column
// halves; masked columns > lim exactly 0 when MASKED), written back over S as
// interleaved bf16 P_hi / P_lo words (per 16-key k-step: 8 words P_hi, then 8 words
// P_lo = p - P_hi rounded to bf16).  Returns sum p.  (Summing the unrounded p instead
// of P_hi + P_lo changes the sum by an unbiased ~2^-18 relative error per weight.)
template <int BN, bool MASKED>
__device__ __forceinline__ float exp_split_store(uint32_t tS, float sl2, float m_use, int lim) {
  const uint64_t scale2 = f2_pack(sl2, sl2);
  const uint64_t negm2 = f2_pack(-m_use, -m_use);
  uint64_t acc = f2_pack(0.f, 0.f);
#pragma unroll
  for (int cp = 0; cp < BN / 64; ++cp) {
    uint32_t a[2][32];
    tmem_ld32(tS + cp * 64, a[0]);
    tmem_ld32(tS + cp * 64 + 32, a[1]);
    tmem_ld_wait();
    tmem_reg_fence(a[0]);
    tmem_reg_fence(a[1]);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {  // the four 16-key k-steps of this half
      const uint32_t* src = a[ks >> 1] + (ks & 1) * 16;
      uint32_t out[16];
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const int col = cp * 64 + ks * 16 + 2 * x;
        const uint64_t xv = f2_fma(f2_pack(__uint_as_float(src[2 * x]), __uint_as_float(src[2 * x + 1])), scale2, negm2);
        float x0, x1;
        f2_unpack(xv, x0, x1);
        float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        if (MASKED) {
          if (col > lim) p0 = 0.f;
          if (col + 1 > lim) p1 = 0.f;
        }
        acc = f2_add(acc, f2_pack(p0, p1));
        const uint32_t wh = pack_bf16x2(p0, p1);
        out[x] = wh;
        out[8 + x] = pack_bf16x2(p0 - bf16lo_to_f32(wh), p1 - bf16hi_to_f32(wh));
      }
      tmem_st16(tS + cp * 64 + ks * 16, out);
    }
  }
  float a0, a1;
  f2_unpack(acc, a0, a1);
  return a0 + a1;
}

// p = 2^(s * scale * log2e - m) for one row's BN scores as one fp16 P (re-read from
// TMEM in 64-column halves; masked columns > lim exactly 0 when MASKED): k-step kk
// (keys 16 kk .. 16 kk + 15) goes to columns [8 kk, 8 kk + 8) of the row's S buffer,
// which hold scores already read.  Returns sum p.
template <int BN, bool MASKED>
__device__ __forceinline__ float exp_f16_store(uint32_t tS, float sl2, float m_use, int lim) {
  const uint64_t scale2 = f2_pack(sl2, sl2);
  const uint64_t negm2 = f2_pack(-m_use, -m_use);
  uint64_t acc = f2_pack(0.f, 0.f);
#pragma unroll
  for (int cp = 0; cp < BN / 64; ++cp) {
    uint32_t a[2][32];
    tmem_ld32(tS + cp * 64, a[0]);
    tmem_ld32(tS + cp * 64 + 32, a[1]);
    tmem_ld_wait();
    tmem_reg_fence(a[0]);
    tmem_reg_fence(a[1]);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t out[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const int col = cp * 64 + hf * 32 + 2 * x;
        const uint64_t xv = f2_fma(f2_pack(__uint_as_float(a[hf][2 * x]), __uint_as_float(a[hf][2 * x + 1])), scale2, negm2);
        float x0, x1;
        f2_unpack(xv, x0, x1);
        float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        if (MASKED) {
          if (col > lim) p0 = 0.f;
          if (col + 1 > lim) p1 = 0.f;
        }
        acc = f2_add(acc, f2_pack(p0, p1));
        out[x] = pack_f16x2(p0, p1);
      }
      tmem_st16(tS + cp * 32 + hf * 16, out);
    }
  }
  float a0, a1;
  f2_unpack(acc, a0, a1);
  return a0 + a1;
}

// Maximum of one row's visible scores (columns <= lim when MASKED), read in 64-column halves.
template <int BN, bool MASKED>
__device__ __forceinline__ float row_max(uint32_t tS, int lim) {
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int cp = 0; cp < BN / 64; ++cp) {
    uint32_t a[2][32];
    tmem_ld32(tS + cp * 64, a[0]);
    tmem_ld32(tS + cp * 64 + 32, a[1]);
    tmem_ld_wait();
    tmem_reg_fence(a[0]);
    tmem_reg_fence(a[1]);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int x = 0; x < 32; x += 2) {
        if (MASKED) {
          const int col = cp * 64 + h * 32 + x;
          mx[h] = fmax3(mx[h], (col <= lim) ? __uint_as_float(a[h][x]) : -INFINITY,
                        (col + 1 <= lim) ? __uint_as_float(a[h][x + 1]) : -INFINITY);
        } else {
          mx[h] = fmax3(mx[h], __uint_as_float(a[h][x]), __uint_as_float(a[h][x + 1]));
        }
      }
  }
  return fmaxf(mx[0], mx[1]);
}

// The same exponentials and hi/lo words from a row already held in registers (one
// TMEM read per block instead of one per 64-column half).
template <int BN, bool MASKED>
__device__ __forceinline__ float exp_split_store_regs(uint32_t tS, const uint32_t (&a)[BN / 32][32], float sl2,
                                                      float m_use, int lim) {
  const uint64_t scale2 = f2_pack(sl2, sl2);
  const uint64_t negm2 = f2_pack(-m_use, -m_use);
  uint64_t acc = f2_pack(0.f, 0.f);
#pragma unroll
  for (int ks = 0; ks < BN / 16; ++ks) {  // 16-key k-steps
    const uint32_t* src = a[ks >> 1] + (ks & 1) * 16;
    uint32_t out[16];
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const int col = ks * 16 + 2 * x;
      const uint64_t xv = f2_fma(f2_pack(__uint_as_float(src[2 * x]), __uint_as_float(src[2 * x + 1])), scale2, negm2);
      float x0, x1;
      f2_unpack(xv, x0, x1);
      float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
      if (MASKED) {
        if (col > lim) p0 = 0.f;
        if (col + 1 > lim) p1 = 0.f;
      }
      acc = f2_add(acc, f2_pack(p0, p1));
      const uint32_t wh = pack_bf16x2(p0, p1);
      out[x] = wh;
      out[8 + x] = pack_bf16x2(p0 - bf16lo_to_f32(wh), p1 - bf16hi_to_f32(wh));
    }
    tmem_st16(tS + ks * 16, out);
  }
  float a0, a1;
  f2_unpack(acc, a0, a1);
  return a0 + a1;
}

// Load one row of S (BN fp32 columns) into registers with a single wait.
template <int BN>
__device__ __forceinline__ void load_row(uint32_t tS, uint32_t (&a)[BN / 32][32]) {
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + c * 32, a[c]);
  tmem_ld_wait();
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) tmem_reg_fence(a[c]);
}

// Maximum of a register-held row's visible scores (columns <= lim when MASKED).
template <int BN, bool MASKED>
__device__ __forceinline__ float row_max_regs(const uint32_t (&a)[BN / 32][32], int lim) {
  float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int c = 0; c < BN / 32; ++c)
#pragma unroll
    for (int x = 0; x < 32; x += 2) {
      float v0 = __uint_as_float(a[c][x]), v1 = __uint_as_float(a[c][x + 1]);
      if (MASKED) {
        if (c * 32 + x > lim) v0 = -INFINITY;
        if (c * 32 + x + 1 > lim) v1 = -INFINITY;
      }
      m[(x >> 1) & 3] = fmax3(m[(x >> 1) & 3], v0, v1);
    }
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// The exponentials of a register-held row as one fp16 P: k-step kk (keys 16 kk ..
// 16 kk + 15) in columns [8 kk, 8 kk + 8) of the row's S buffer.  Returns sum p.
template <int BN, bool MASKED>
__device__ __forceinline__ float exp_f16_store_regs(uint32_t tS, const uint32_t (&a)[BN / 32][32], float sl2,
                                                    float m_use, int lim) {
  const uint64_t scale2 = f2_pack(sl2, sl2);
  const uint64_t negm2 = f2_pack(-m_use, -m_use);
  uint64_t acc = f2_pack(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t out[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      const int col = c * 32 + 2 * x;
      const uint64_t xv = f2_fma(f2_pack(__uint_as_float(a[c][2 * x]), __uint_as_float(a[c][2 * x + 1])), scale2, negm2);
      float x0, x1;
      f2_unpack(xv, x0, x1);
      float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
      if (MASKED) {
        if (col > lim) p0 = 0.f;
        if (col + 1 > lim) p1 = 0.f;
      }
      acc = f2_add(acc, f2_pack(p0, p1));
      out[x] = pack_f16x2(p0, p1);
    }
    tmem_st16(tS + c * 16, out);
  }
  float a0, a1;
  f2_unpack(acc, a0, a1);
  return a0 + a1;
}

}  // namespace score
}  // namespace poem
