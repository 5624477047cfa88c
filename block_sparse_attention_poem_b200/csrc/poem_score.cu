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
// With a query offset (chunked prefill) local query tile i is global tile
// q_tile0 + i: its sampled queries sit at key positions (q_tile0 + i) B + j (B / S)
// and its score row has q_tile0 + i + 1 entries (row_off layout).
//
// Pipeline (one CTA per SM, TMEM fully allocated):
//   TMEM  S0 [0,128)  S1 [128,256)  -- S double-buffered: S_{b+1} is computed while
//                                      the softmax of block b runs
//         O / P V [256,384)           -- pass 1: running O; pass 2: P_b V_b
//         o [384,512)                 -- pass 2: the row's dense output (from pass 1)
//   smem  Q tile, 2-stage K ring, 2-stage V ring (160 KB at d = 128)
//   warps 0-3 softmax (one sampled query per thread), warps 4-7 (pass 2 only) the
//         norm of P_b V_b - m_b o while the softmax warps move on to block b+1,
//         then one TMA warp and one MMA-issuing warp.
//   MMA order: S_0, S_1, PV_0, S_2, PV_1, ...
//
// Precision: P enters the P V contraction as a hi/lo pair of bf16 matrices
// (P = P_hi + P_lo, two MMAs into the same accumulator), about 16 significant
// bits, so that o, r_b and I_b keep ~1e-6 relative accuracy; a single bf16 P
// gives ~1e-3 and would move near-tied blocks across the selection cut.
//
// Every mbarrier wait below is made at most one phase behind the barrier (each
// wait's completion is a precondition of the barrier's next phase), so parity
// waits cannot alias.
#include "common.cuh"

namespace poem {
namespace {

template <int D, int BN, int PASS>
struct ScoreCfg {
  static constexpr int M = 128;
  static constexpr int kGroups = 8;        // groups of 16 sampled queries per CTA
  static constexpr int kRowsPerGroup = 16;
  static constexpr int kChunks = D / 64;
  static constexpr int kStages = 2;
  static constexpr int kQBytes = M * D * 2;
  static constexpr int kKVBytes = BN * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kOffBar = kOffV + kStages * kKVBytes;
  static constexpr int kOffM = kOffBar + 256;                 // m_b hand-off, [2][128] floats
  // at least 120 KB so that one CTA (holding all 512 TMEM columns) occupies an SM
  static constexpr int kSmemBytes = (kOffM + 2 * 128 * 4 + 1024) > 122880 ? (kOffM + 2 * 128 * 4 + 1024) : 122880;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;     // S buffer s at [128 s, 128 s + BN)
  static constexpr uint32_t kColO = 256;   // O (pass 1) or P_b V_b (pass 2)
  static constexpr uint32_t kColOd = 384;  // pass 2: dense output o of the row
  static constexpr int kWarpProd = (PASS == 2) ? 8 : 4;
  static constexpr int kWarpMma = kWarpProd + 1;
  static constexpr int kThreads = (kWarpMma + 1) * 32;
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(M, BN, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(M, D, 1);
};

struct ScoreBarriers {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2];
  uint64_t pv_full, pv_empty;    // P V accumulator done / released by the norm warps
  uint64_t m_ready[2], m_empty[2];
  uint64_t drain;
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

// Warp-uniform wait (tcgen05.ld/st are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, ScoreBarriers* sb, const DevErr& e) {
  return __all_sync(0xffffffffu, wait_or_abort(bar, parity, sb, e));
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
__global__ void __launch_bounds__(ScoreCfg<D, BN, PASS>::kThreads, 1)
    poem_score_kernel(const __grid_constant__ CUtensorMap tmQs, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const ScoreParams p) {
  using C = ScoreCfg<D, BN, PASS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  ScoreBarriers* sb = reinterpret_cast<ScoreBarriers*>(smem + C::kOffBar);
  float* sm_m = reinterpret_cast<float*>(smem + C::kOffM);  // [2][128]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = p.group;
  const int n_groups = p.n_tiles * G;  // per KV head
  const int ctas_per_g = (n_groups + 7) / 8;
  int g, z0;
  score_cta_coords(blockIdx.x, ctas_per_g, g, z0);
  const int z_last = min(z0 + 7, n_groups - 1);
  const int t0 = p.q_tile0;            // global index of local query tile 0
  const int nb = z_last / G + 1 + t0;  // key blocks 0 .. largest (global) tile of the CTA
  const int i_lo = z0 / G + t0;        // smallest global tile of the CTA: blocks < i_lo need no mask

  if (tid == 0) {
    mbar_init(&sb->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sb->k_full[s], 1);
      mbar_init(&sb->k_empty[s], 1);
      mbar_init(&sb->v_full[s], 1);
      mbar_init(&sb->v_empty[s], 1);
      mbar_init(&sb->s_full[s], 1);
      mbar_init(&sb->p_full[s], 128);
      mbar_init(&sb->m_ready[s], 128);
      mbar_init(&sb->m_empty[s], 128);
    }
    mbar_init(&sb->pv_full, 1);
    mbar_init(&sb->pv_empty, 128);
    mbar_init(&sb->drain, 1);
    sb->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::kWarpMma) tmem_alloc<C::kTmemCols>(&sb->tmem_base);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sb->tmem_base;

  if (warp == C::kWarpProd) {
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
        const int s = b & 1;
        const uint32_t par = ((b >> 1) & 1) ^ 1;  // completion #(b/2 - 1) of the stage's empty barrier
        if (!wait_or_abort(&sb->k_empty[s], par, sb, p.err)) break;
        mbar_arrive_expect_tx(&sb->k_full[s], C::kKVBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(sK + s * C::kKVBytes + c * (BN * 128), &tmK, &sb->k_full[s], c * 64, g, b * BN);
        ++k_issued;
        if (!wait_or_abort(&sb->v_empty[s], par, sb, p.err)) break;
        mbar_arrive_expect_tx(&sb->v_full[s], C::kKVBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(sV + s * C::kKVBytes + c * (BN * 128), &tmV, &sb->v_full[s], c * 64, g, b * BN);
        ++v_issued;
      }
      // Drain: the last load issued into each stage must have landed.
      mbar_wait(&sb->q_full, 0, kDrainNs);
      for (int b = max(0, k_issued - 2); b < k_issued; ++b) mbar_wait(&sb->k_full[b & 1], (b >> 1) & 1, kDrainNs);
      for (int b = max(0, v_issued - 2); b < v_issued; ++b) mbar_wait(&sb->v_full[b & 1], (b >> 1) & 1, kDrainNs);
    }
  } else if (warp == C::kWarpMma) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      const uint32_t tO = tmem + C::kColO;
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
      bool ok = wait_or_abort(&sb->q_full, 0, sb, p.err);
      // P V_j with P = P_hi + P_lo read from S buffer j % 2.  Pass 1 accumulates over
      // blocks; pass 2 starts a fresh accumulator per block, once the norm warps have
      // read the previous one.
      auto issue_pv = [&](int j) -> bool {
        const int s = j & 1;
        if (!wait_or_abort(&sb->p_full[s], (j >> 1) & 1, sb, p.err)) return false;
        if (!wait_or_abort(&sb->v_full[s], (j >> 1) & 1, sb, p.err)) return false;
        if (PASS == 2 && j > 0 && !wait_or_abort(&sb->pv_empty, (j - 1) & 1, sb, p.err)) return false;
        tc_fence_after();
        const uint32_t tP = tmem + C::kColS + s * 128;
        const uint32_t aVs = aV + s * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // keys [16 kk, 16 kk + 16): P_hi words at [16 kk, +8), P_lo at [16 kk + 8, +8)
          const uint64_t bdesc = smem_desc_sw128(aVs + kk * 2048, BN * 128, 1024);
          const bool fresh = (PASS == 2 || j == 0) && kk == 0;
          mma_ts(tO, tP + kk * 16, bdesc, C::kIdescPV, fresh ? 0u : 1u);
          mma_ts(tO, tP + kk * 16 + 8, bdesc, C::kIdescPV, 1u);
        }
        mma_commit(&sb->v_empty[s]);
        mma_commit(&sb->pv_full);
        return true;
      };
      for (int b = 0; b < nb && ok; ++b) {
        const int s = b & 1;
        if (!wait_or_abort(&sb->k_full[s], (b >> 1) & 1, sb, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tS = tmem + C::kColS + s * 128;
        const uint32_t aKs = aK + s * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          const uint64_t adesc = smem_desc_sw128(aQ + (kk >> 2) * (C::M * 128) + koff, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(aKs + (kk >> 2) * (BN * 128) + koff, 16, 1024);
          mma_ss(tS, adesc, bdesc, C::kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sb->s_full[s]);
        mma_commit(&sb->k_empty[s]);
        if (b > 0 && !issue_pv(b - 1)) { ok = false; break; }
      }
      if (ok && nb > 0) issue_pv(nb - 1);
      mma_commit(&sb->drain);
      mbar_wait(&sb->drain, 0, kDrainNs);
    }
  } else if (warp < 4) {
    // ============================ softmax warps ============================
    const int r = tid;
    const int zl = r >> 4;
    const int j = r & 15;
    const int z = z0 + zl;
    const bool valid = (z < n_groups);
    const int i = valid ? z / G : 0;
    const int hq = g * G + (valid ? z - i * G : 0);
    const int qpos = valid ? (i + t0) * BN + j * p.sample_stride : -1;  // key position; -1: padding row
    const int64_t srow = ((int64_t)hq * p.n_tiles + i) * p.n_sample + j;  // sampled-row index
    const uint32_t lane_off = ((uint32_t)(warp * 32) << 16);
    const uint32_t tO = tmem + lane_off + C::kColO;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    const float lse2 = (PASS == 2 && valid) ? p.ws_lse[srow] : 0.f;
    bool ok = true;
    for (int b = 0; b < nb; ++b) {
      const int s = b & 1;
      const uint32_t tS = tmem + lane_off + C::kColS + s * 128;
      if (!warp_wait(&sb->s_full[s], (b >> 1) & 1, sb, p.err)) { ok = false; break; }
      tc_fence_after();
      const int lim = qpos - b * BN;  // columns <= lim are visible to this query
      float m_use;
      if (PASS == 1) {
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
        // Rescaling O needs P V_{b-1} complete (S_b may finish before it).
        if (b > 0 && __any_sync(0xffffffffu, grow)) {
          if (!warp_wait(&sb->pv_full, (b - 1) & 1, sb, p.err)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(tO + c * 32, ov);
            tmem_ld_wait();
            tmem_reg_fence(ov);
#pragma unroll
            for (int x = 0; x < 32; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * alpha);
            tmem_st32(tO + c * 32, ov);
          }
        }
        l_run *= alpha;
        m_use = (m_run == -INFINITY) ? 0.f : m_run;
      } else {
        m_use = lse2;
      }
      float msum = 0.f;
      if (b < i_lo)
        split_chunks<BN, false>(tS, sl2, m_use, lim, &msum);
      else
        split_chunks<BN, true>(tS, sl2, m_use, lim, &msum);
      if (PASS == 1) {
        l_run += msum;
      } else {
        // hand m_b to the norm warps (slot s is free once block b-2's norm read it)
        if (b >= 2 && !wait_or_abort(&sb->m_empty[s], ((b >> 1) & 1) ^ 1, sb, p.err)) ok = false;
        sm_m[s * 128 + r] = valid ? msum : 0.f;
        mbar_arrive(&sb->m_ready[s]);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sb->p_full[s]);
      if (!__all_sync(0xffffffffu, ok)) break;
    }
    if (PASS == 1 && __all_sync(0xffffffffu, ok && !sb->abort_flag)) {
      // P V_{nb-2} may still be in flight: observe its completion first, so the wait for
      // P V_{nb-1} is never two phases behind the barrier.
      const bool prev_ok = (nb < 2) || warp_wait(&sb->pv_full, (nb - 2) & 1, sb, p.err);
      if (prev_ok && warp_wait(&sb->pv_full, (nb - 1) & 1, sb, p.err)) {
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
  } else if (PASS == 2) {
    // ====================== norm warps (pass 2, warps 4-7) ======================
    const int r = tid - 128;                 // TMEM lane = row
    const int zl = r >> 4;
    const int j = r & 15;
    const int z = z0 + zl;
    const bool valid = (z < n_groups);
    const int i = valid ? z / G : 0;
    const int hq = g * G + (valid ? z - i * G : 0);
    const int64_t srow = ((int64_t)hq * p.n_tiles + i) * p.n_sample + j;
    const uint32_t lane_off = ((uint32_t)((warp - 4) * 32) << 16);
    const uint32_t tPV = tmem + lane_off + C::kColO;
    const uint32_t tOd = tmem + lane_off + C::kColOd;
    // the row's dense output o (pass 1) into TMEM columns [384, 384 + D)
    {
      const float4* o4 = reinterpret_cast<const float4*>(p.ws_o + srow * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t w[32];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float4 v = valid ? o4[c * 8 + x] : make_float4(0.f, 0.f, 0.f, 0.f);
          w[4 * x] = __float_as_uint(v.x);
          w[4 * x + 1] = __float_as_uint(v.y);
          w[4 * x + 2] = __float_as_uint(v.z);
          w[4 * x + 3] = __float_as_uint(v.w);
        }
        tmem_st32(tOd + c * 32, w);
      }
      tmem_st_wait();
    }
    const int64_t tri = row_off(p.n_tiles, t0, hq, i);
    for (int b = 0; b < nb; ++b) {
      const int s = b & 1;
      if (!warp_wait(&sb->pv_full, b & 1, sb, p.err)) break;
      if (!warp_wait(&sb->m_ready[s], (b >> 1) & 1, sb, p.err)) break;
      tc_fence_after();
      const float mb_row = sm_m[s * 128 + r];
      mbar_arrive(&sb->m_empty[s]);
      const uint64_t negm2 = f2_pack(-mb_row, -mb_row);
      uint64_t acc2 = f2_pack(0.f, 0.f);
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf) {
        uint32_t pv[2][32], od[2][32];
        tmem_ld32(tPV + hf * 64, pv[0]);
        tmem_ld32(tPV + hf * 64 + 32, pv[1]);
        tmem_ld32(tOd + hf * 64, od[0]);
        tmem_ld32(tOd + hf * 64 + 32, od[1]);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tmem_reg_fence(pv[h]);
          tmem_reg_fence(od[h]);
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            const uint64_t e = f2_fma(negm2, f2_pack(__uint_as_float(od[h][x]), __uint_as_float(od[h][x + 1])),
                                      f2_pack(__uint_as_float(pv[h][x]), __uint_as_float(pv[h][x + 1])));
            acc2 = f2_fma(e, e, acc2);
          }
        }
      }
      // P V_b has been read: the accumulator may be reused for block b+1.
      tc_fence_before();
      mbar_arrive(&sb->pv_empty);
      float a0, a1;
      f2_unpack(acc2, a0, a1);
      float Ib = valid ? sqrtf(a0 + a1) : 0.f;
      float mb = valid ? mb_row : 0.f;
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) {  // max over the 16 queries of the group
        Ib = fmaxf(Ib, __shfl_xor_sync(0xffffffffu, Ib, off));
        mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
      }
      if (j == 0 && valid && b <= i + t0) {
        p.I_hat[tri + b] = Ib;
        p.m_hat[tri + b] = mb;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::kWarpMma) {
    __syncwarp();
    tmem_dealloc<C::kTmemCols>(tmem);
  }
}

template <int D, int BN, int PASS>
cudaError_t launch_pass(const CUtensorMap& tmQs, const CUtensorMap& tmK, const CUtensorMap& tmV,
                        const ScoreParams& p, int grid, cudaStream_t stream) {
  using C = ScoreCfg<D, BN, PASS>;
  cudaError_t e = ensure_smem_limit(poem_score_kernel<D, BN, PASS>, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  poem_score_kernel<D, BN, PASS><<<grid, C::kThreads, C::kSmemBytes, stream>>>(tmQs, tmK, tmV, p);
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
