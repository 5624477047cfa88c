// poem_score.cu -- exact output-relative block scores on the sampled queries (sm_100a).
//
// What is computed (reading note "Attention deletion error", Section 4.1 and
// Equation (4)): for a query q, head h and visible key block b,
//   m_b = sum_{u in b, u <= q} p_u,      r_b = sum_{u in b, u <= q} p_u v_u - m_b o,
//   I_b = || r_b ||  (= m_b || v_b - o ||),
// with p the dense causal softmax of q and o its dense output.  The scores are
// taken on the S = 16 strided queries q_j = iB + j (B / S) of each query tile i
// and max-aggregated:  I_hat[h, i, b] = max_j I_b(q_j),  m_hat likewise.
//
// Two passes over the key blocks, both on the tensor cores:
//   pass 1: dense causal attention of the sampled queries -> o (fp32) and the
//           log-sum-exp of their scaled logits (log2 units) in the workspace.
//   pass 2: recompute S, form the exact normalised p = 2^(s log2e scale - lse),
//           per block r_b = P_b V_b - m_b o and its norm, max over the 16 queries.
//
// Packing: one CTA owns 8 groups of 16 sampled queries that share a KV head --
// groups are enumerated per KV head in (tile, query head) order, so a CTA covers
// 2 adjacent tiles x 4 heads for 4-way GQA.  The 16 rows of a group are gathered
// by one 4-D TMA box (dims: head_dim, head, sample j, tile i).  A CTA sweeps key
// blocks 0 .. (largest tile among its groups); a query masks keys after itself.
//
// Precision: P enters the P V contraction as a hi/lo pair of bf16 matrices
// (P = P_hi + P_lo, two MMAs into the same accumulator), about 16 significant
// bits, so that o, r_b and I_b keep ~1e-6 relative accuracy; a single bf16 P
// gives ~1e-3 and would move near-tied blocks across the selection cut.
#include "common.cuh"

namespace poem {
namespace {

template <int D, int BN>
struct ScoreCfg {
  static constexpr int M = 128;
  static constexpr int kGroups = 8;        // groups of 16 sampled queries per CTA
  static constexpr int kRowsPerGroup = 16;
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = M * D * 2;
  static constexpr int kKVBytes = BN * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kKVBytes;
  static constexpr int kOffBar = kOffV + kKVBytes;
  // + barriers + alignment slack; at least 80 KB so that no more than two CTAs (2 x 256
  // TMEM columns) are resident on an SM and tcgen05.alloc never has to wait.
  static constexpr int kSmemBytes = (kOffBar + 128 + 1024) > 81920 ? (kOffBar + 128 + 1024) : 81920;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kColS = 0;     // S (fp32), then P_hi / P_lo interleaved per 16-key k-step
  static constexpr uint32_t kColO = 128;   // O (pass 1) or P_b V_b (pass 2)
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(M, BN, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(M, D, 1);
};

struct ScoreBarriers {
  uint64_t q_full, k_full, k_empty, v_full, v_empty, s_full, p_full, o_full, drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

constexpr uint64_t kDrainNs = 2000000000ull;

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, ScoreBarriers* sb, const DevErr& e) {
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

// CTA -> (KV head, first group).  CTAs are launched KV-head-major and, within a
// KV head, the CTAs holding the last tiles (longest sweeps) first.
__device__ __forceinline__ void score_cta_coords(int cta, int ctas_per_g, int& g, int& z0) {
  g = cta / ctas_per_g;
  const int c = ctas_per_g - 1 - (cta - g * ctas_per_g);
  z0 = c * 8;
}

// p = 2^(s * scale * log2e - m) for one row's BN scores (masked columns > lim when
// MASKED), written back over S as interleaved bf16 P_hi / P_lo words; *msum += sum p.
// (Summing the unrounded p instead of P_hi + P_lo changes m_b by an unbiased
// ~2^-18 relative error per weight.)
template <int BN, bool MASKED>
__device__ __forceinline__ void split_chunks(uint32_t tS, float sl2, float m_use, int lim, float* msum) {
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
    for (int h = 0; h < 2; ++h) {
      uint32_t out[32];
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const int col = cp * 64 + h * 32 + 2 * x;
        const uint64_t xv = f2_fma(f2_pack(__uint_as_float(a[h][2 * x]), __uint_as_float(a[h][2 * x + 1])), scale2, negm2);
        float x0, x1;
        f2_unpack(xv, x0, x1);
        float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        if (MASKED) {
          if (col > lim) p0 = 0.f;
          if (col + 1 > lim) p1 = 0.f;
        }
        acc = f2_add(acc, f2_pack(p0, p1));
        const uint32_t wh = pack_bf16x2(p0, p1);
        const uint32_t wl = pack_bf16x2(p0 - bf16lo_to_f32(wh), p1 - bf16hi_to_f32(wh));
        // k-step (x / 8): words 0-7 P_hi, 8-15 P_lo
        out[(x >> 3) * 16 + (x & 7)] = wh;
        out[(x >> 3) * 16 + 8 + (x & 7)] = wl;
      }
      tmem_st32(tS + cp * 64 + h * 32, out);
    }
  }
  float a0, a1;
  f2_unpack(acc, a0, a1);
  *msum += a0 + a1;
}

template <int D, int BN, int PASS>
__global__ void __launch_bounds__(kThreadsFwd, 2)
    poem_score_kernel(const __grid_constant__ CUtensorMap tmQs, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const ScoreParams p) {
  using C = ScoreCfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  ScoreBarriers* sb = reinterpret_cast<ScoreBarriers*>(smem + C::kOffBar);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = p.group;
  const int n_groups = p.n_tiles * G;  // per KV head
  const int ctas_per_g = (n_groups + 7) / 8;
  int g, z0;
  score_cta_coords(blockIdx.x, ctas_per_g, g, z0);
  const int z_last = min(z0 + 7, n_groups - 1);
  const int nb = z_last / G + 1;  // key blocks 0 .. largest tile of the CTA
  const int i_lo = z0 / G;        // smallest tile of the CTA: blocks < i_lo need no mask

  if (tid == 0) {
    mbar_init(&sb->q_full, 1);
    mbar_init(&sb->k_full, 1);
    mbar_init(&sb->k_empty, 1);
    mbar_init(&sb->v_full, 1);
    mbar_init(&sb->v_empty, 1);
    mbar_init(&sb->s_full, 1);
    mbar_init(&sb->p_full, 128);
    mbar_init(&sb->o_full, 1);
    mbar_init(&sb->drain, 1);
    sb->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc<C::kTmemCols>(&sb->tmem_base);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sb->tmem_base;

  if (warp == 4) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      tma_prefetch_desc(&tmQs);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&sb->q_full, C::kQBytes);
      for (int zl = 0; zl < C::kGroups; ++zl) {
        const int z = z0 + zl;  // groups past the end read out-of-range tiles: zero-filled
        const int i = z / G;
        const int hq = g * G + (z - i * G);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sQ + c * (C::M * 128) + zl * (C::kRowsPerGroup * 128), &tmQs, &sb->q_full, c * 64, hq, 0,
                      i);
      }
      int k_issued = 0, v_issued = 0;
      for (int b = 0; b < nb && !sb->abort_flag; ++b) {
        if (!wait_or_abort(&sb->k_empty, (k_issued & 1) ^ 1, sb, p.err)) break;
        mbar_arrive_expect_tx(&sb->k_full, C::kKVBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(sK + c * (BN * 128), &tmK, &sb->k_full, c * 64, g, b * BN);
        ++k_issued;
        if (!wait_or_abort(&sb->v_empty, (v_issued & 1) ^ 1, sb, p.err)) break;
        mbar_arrive_expect_tx(&sb->v_full, C::kKVBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(sV + c * (BN * 128), &tmV, &sb->v_full, c * 64, g, b * BN);
        ++v_issued;
      }
      mbar_wait(&sb->q_full, 0, kDrainNs);
      if (k_issued) mbar_wait(&sb->k_full, (k_issued - 1) & 1, kDrainNs);
      if (v_issued) mbar_wait(&sb->v_full, (v_issued - 1) & 1, kDrainNs);
    }
  } else if (warp == 5) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      const uint32_t tS = tmem + C::kColS;
      const uint32_t tO = tmem + C::kColO;
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
      bool ok = wait_or_abort(&sb->q_full, 0, sb, p.err);
      // P V_b with P = P_hi + P_lo (both bf16, read from TMEM).  Pass 1 accumulates
      // over blocks; pass 2 starts a fresh accumulator per block.
      auto issue_pv = [&](int j) -> bool {
        if (!wait_or_abort(&sb->p_full, j & 1, sb, p.err)) return false;
        tc_fence_after();
        if (!wait_or_abort(&sb->v_full, j & 1, sb, p.err)) return false;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // P for keys [16 kk, 16 kk + 16): P_hi words at TMEM columns [16 kk, +8),
          // P_lo words at [16 kk + 8, +8)
          const uint64_t bdesc = smem_desc_sw128(aV + kk * 2048, BN * 128, 1024);
          const bool fresh = (PASS == 2 || j == 0) && kk == 0;
          mma_ts(tO, tS + kk * 16, bdesc, C::kIdescPV, fresh ? 0u : 1u);
          mma_ts(tO, tS + kk * 16 + 8, bdesc, C::kIdescPV, 1u);
        }
        mma_commit(&sb->v_empty);
        if (PASS == 2) mma_commit(&sb->o_full);  // P_b V_b of this block is ready
        return true;
      };
      int it = 0;
      for (int b = 0; b < nb && ok; ++b) {
        if (b > 0 && !issue_pv(b - 1)) { ok = false; break; }
        if (!wait_or_abort(&sb->k_full, b & 1, sb, p.err)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          const uint64_t adesc = smem_desc_sw128(aQ + (kk >> 2) * (C::M * 128) + koff, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(aK + (kk >> 2) * (BN * 128) + koff, 16, 1024);
          mma_ss(tS, adesc, bdesc, C::kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sb->s_full);
        mma_commit(&sb->k_empty);
        ++it;
      }
      if (ok && it > 0) {
        if (issue_pv(it - 1) && PASS == 1) mma_commit(&sb->o_full);
      }
      mma_commit(&sb->drain);
      mbar_wait(&sb->drain, 0, kDrainNs);
    }
  } else {
    // ============================ softmax warps ============================
    const int r = tid;
    const int zl = r >> 4;
    const int j = r & 15;
    const int z = z0 + zl;
    const bool valid = (z < n_groups);
    const int i = valid ? z / G : 0;
    const int hq = g * G + (valid ? z - i * G : 0);
    const int qpos = valid ? i * BN + j * p.sample_stride : -1;  // -1: padding row, sees nothing
    const int64_t srow = ((int64_t)hq * p.n_tiles + i) * p.n_sample + j;  // sampled-row index
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t tS = lane_base + C::kColS;
    const uint32_t tO = lane_base + C::kColO;
    float m_run = -INFINITY, l_run = 0.f;
    const float lse2 = (PASS == 2 && valid) ? p.ws_lse[srow] : 0.f;
    const float* orow = p.ws_o + srow * D;
    bool ok = true;
    const float sl2 = p.scale_log2;
    for (int b = 0; b < nb; ++b) {
      if (!__all_sync(0xffffffffu, wait_or_abort(&sb->s_full, b & 1, sb, p.err))) { ok = false; break; }
      tc_fence_after();
      const int lim = qpos - b * BN;  // columns <= lim are visible to this query
      float m_use = 0.f;
      if (PASS == 1) {
        // phase 1: row max over the visible columns (one wait for all chunks)
        float mx = -INFINITY;
        {
          uint32_t raw[BN / 32][32];
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + c * 32, raw[c]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) tmem_reg_fence(raw[c]);
          if (b < i_lo) {
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
#pragma unroll
              for (int x = 0; x < 32; x += 2)
                mx = fmax3(mx, __uint_as_float(raw[c][x]), __uint_as_float(raw[c][x + 1]));
          } else {
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
#pragma unroll
              for (int x = 0; x < 32; ++x) mx = fmaxf(mx, (c * 32 + x <= lim) ? __uint_as_float(raw[c][x]) : -INFINITY);
          }
        }
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool grow = (m_new > m_run + 8.0f);
        float alpha = 1.f;
        if (grow) {
          alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        if (b > 0 && __any_sync(0xffffffffu, grow)) {
          uint32_t ov[D / 32][32];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, ov[c]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            tmem_reg_fence(ov[c]);
#pragma unroll
            for (int x = 0; x < 32; ++x) ov[c][x] = __float_as_uint(__uint_as_float(ov[c][x]) * alpha);
            tmem_st32(tO + c * 32, ov[c]);
          }
        }
        l_run *= alpha;
        m_use = (m_run == -INFINITY) ? 0.f : m_run;
      } else {
        m_use = lse2;
      }
      // phase 2: p, split P = P_hi + P_lo in bf16, in place: the 32 S columns of a
      // chunk (two 16-key k-steps) become, per k-step, 8 P_hi words then 8 P_lo words.
      // Rows of a CTA whose tiles all lie past this block need no mask (uniform).
      float msum = 0.f;
      if (b < i_lo)
        split_chunks<BN, false>(tS, sl2, m_use, lim, &msum);
      else
        split_chunks<BN, true>(tS, sl2, m_use, lim, &msum);
      if (PASS == 1) l_run += msum;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sb->p_full);

      if (PASS == 2) {
        // r_b = P_b V_b - m_b o ;  I_b = || r_b ||
        if (!__all_sync(0xffffffffu, wait_or_abort(&sb->o_full, b & 1, sb, p.err))) { ok = false; break; }
        tc_fence_after();
        uint32_t pv[D / 32][32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, pv[c]);
        tmem_ld_wait();
        uint64_t acc2 = f2_pack(0.f, 0.f);
        const uint64_t negm2 = f2_pack(-msum, -msum);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          tmem_reg_fence(pv[c]);
          if (valid) {
            const float4* o4 = reinterpret_cast<const float4*>(orow + c * 32);
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              const float4 ov = o4[x];
              const uint64_t e01 = f2_fma(negm2, f2_pack(ov.x, ov.y),
                                          f2_pack(__uint_as_float(pv[c][4 * x]), __uint_as_float(pv[c][4 * x + 1])));
              const uint64_t e23 = f2_fma(negm2, f2_pack(ov.z, ov.w),
                                          f2_pack(__uint_as_float(pv[c][4 * x + 2]), __uint_as_float(pv[c][4 * x + 3])));
              acc2 = f2_fma(e01, e01, acc2);
              acc2 = f2_fma(e23, e23, acc2);
            }
          }
        }
        float acc0, acc1;
        f2_unpack(acc2, acc0, acc1);
        const float acc = acc0 + acc1;
        float Ib = valid ? sqrtf(acc) : 0.f;
        float mb = valid ? msum : 0.f;
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) {  // max over the 16 queries of the group
          Ib = fmaxf(Ib, __shfl_xor_sync(0xffffffffu, Ib, off));
          mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
        }
        if (j == 0 && valid && b <= i) {
          const int64_t off = (int64_t)hq * ((int64_t)p.n_tiles * (p.n_tiles + 1) / 2) + (int64_t)i * (i + 1) / 2 + b;
          p.I_hat[off] = Ib;
          p.m_hat[off] = mb;
        }
      }
    }
    if (PASS == 1 && __all_sync(0xffffffffu, ok && !sb->abort_flag)) {
      if (__all_sync(0xffffffffu, wait_or_abort(&sb->o_full, 0, sb, p.err))) {
        tc_fence_after();
        const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
        float* dst = p.ws_o + srow * D;
        uint32_t ov[D / 32][32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, ov[c]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          tmem_reg_fence(ov[c]);
          if (valid) {
            float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
            for (int x = 0; x < 8; ++x)
              d4[x] = make_float4(__uint_as_float(ov[c][4 * x]) * inv_l, __uint_as_float(ov[c][4 * x + 1]) * inv_l,
                                  __uint_as_float(ov[c][4 * x + 2]) * inv_l, __uint_as_float(ov[c][4 * x + 3]) * inv_l);
          }
        }
        if (valid) p.ws_lse[srow] = (l_run > 0.f) ? m_run + __log2f(l_run) : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) {
    __syncwarp();
    tmem_dealloc<C::kTmemCols>(tmem);
  }
}

template <int D, int BN, int PASS>
cudaError_t launch_pass(const CUtensorMap& tmQs, const CUtensorMap& tmK, const CUtensorMap& tmV,
                        const ScoreParams& p, int grid, cudaStream_t stream) {
  using C = ScoreCfg<D, BN>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(poem_score_kernel<D, BN, PASS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  poem_score_kernel<D, BN, PASS><<<grid, kThreadsFwd, C::kSmemBytes, stream>>>(tmQs, tmK, tmV, p);
  return cudaGetLastError();
}

template <int D, int BN>
cudaError_t launch_score_t(const CUtensorMap& tmQs, const CUtensorMap& tmK, const CUtensorMap& tmV,
                           const ScoreParams& p, cudaStream_t stream) {
  const int ctas_per_g = (p.n_tiles * p.group + 7) / 8;
  const int grid = p.n_kv_heads * ctas_per_g;
  cudaError_t e = launch_pass<D, BN, 1>(tmQs, tmK, tmV, p, grid, stream);
  if (e != cudaSuccess) return e;
  return launch_pass<D, BN, 2>(tmQs, tmK, tmV, p, grid, stream);
}

}  // namespace

cudaError_t launch_score(int head_dim, int block, const CUtensorMap& tmQs, const CUtensorMap& tmK,
                         const CUtensorMap& tmV, const ScoreParams& p, cudaStream_t stream) {
  if (head_dim == 128 && block == 128) return launch_score_t<128, 128>(tmQs, tmK, tmV, p, stream);
  if (head_dim == 128 && block == 64) return launch_score_t<128, 64>(tmQs, tmK, tmV, p, stream);
  if (head_dim == 64 && block == 128) return launch_score_t<64, 128>(tmQs, tmK, tmV, p, stream);
  if (head_dim == 64 && block == 64) return launch_score_t<64, 64>(tmQs, tmK, tmV, p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace poem
