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
//   pass 1 (poem_score_pass1.cu): dense causal attention of the sampled queries ->
//           o (fp32) and the log-sum-exp of their scaled logits (log2 units) in the
//           workspace.
//   pass 2 (this file): recompute S, form the exact normalised
//           p = 2^(s log2e scale - lse), per block r_b = P_b V_b - m_b o and its norm,
//           max over the 16 queries.
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
// Pass 2 pipeline (one CTA per SM, TMEM fully allocated):
//   TMEM  S buffers s = 0, 1, 2 at [128 s, 128 s + BN): the MMAs run up to two blocks
//         ahead of the softmax; the P_b V_b accumulator at [384, 384 + D), read by the
//         norm warps while the next blocks' S are computed
//   smem  Q tile, 3-stage K ring, 2-stage V ring (192 KB at d = 128)
//   warps 0-3 and 8-11 softmax (two warpgroups taking alternate key blocks: with
//   lse known the blocks are independent), warps 4-7 the norm of P_b V_b - m_b o with
//   o held in registers; warp 12 issues TMA loads (K and V rings independently);
//   warp 13 issues the MMAs, converged, from one elected lane; warps 14-15 idle.
//   Registers per thread: 128 at launch; the norm warpgroup raises its budget to
//   184 and warps 12-15 lower theirs to 72 (128 + 184 + 128 + 72 = 4 x 128).
//   MMA order: S_0, S_1, S_2, PV_0, S_3, PV_1, ...
//
// Precision: on a CTA's first query tiles (below score::kHalfMinTile) P enters the
// P V contraction as a hi/lo pair of bf16 matrices (P = P_hi + P_lo, two MMAs into
// the same accumulator), about 16 significant bits: there one or a few blocks hold
// nearly all of a query's mass and r_b cancels almost exactly.  Later CTAs take one
// fp16 P (11 significant bits, scaled by 2^6 so that small weights stay normal)
// against the fp16 copy of V: r_b's rounding error is then ~1e-5 m_b |v|, inside
// the score tolerance.  A single bf16 P (8 bits) would move near-tied blocks across
// the selection cut.  m_b always sums the unrounded fp32 weights.
//
// Every mbarrier wait below is made at most one phase behind the barrier (each
// wait's completion is a precondition of the barrier's next phase), so parity
// waits cannot alias.
#include "common.cuh"
#include "score_common.cuh"

namespace poem {
namespace {

template <int D, int BN>
struct ScoreCfg {
  static constexpr int M = 128;
  static constexpr int kGroups = 8;        // groups of 16 sampled queries per CTA
  static constexpr int kRowsPerGroup = 16;
  static constexpr int kChunks = D / 64;
  static constexpr int kStagesK = 3;       // K ring: a load is issued two blocks ahead of its use
  static constexpr int kStagesV = 2;
  static constexpr int kQBytes = M * D * 2;
  static constexpr int kKVBytes = BN * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kStagesK * kKVBytes;
  static constexpr int kOffBar = kOffV + kStagesV * kKVBytes;
  static constexpr int kOffM = kOffBar + 256;                 // [2][128] floats: m_b hand-off
  // at least 120 KB so that one CTA (holding all 512 TMEM columns) occupies an SM
  static constexpr int kSmemBytes = (kOffM + 2 * 128 * 4 + 1024) > 122880 ? (kOffM + 2 * 128 * 4 + 1024) : 122880;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;     // S buffer s (0, 1, 2) at [128 s, 128 s + BN)
  static constexpr uint32_t kColAcc = 384; // P_b V_b accumulator at [384, 384 + D)
  static constexpr int kWarpProd = 12;     // warps 0-3, 8-11 softmax, 4-7 norm, 12 TMA, 13 MMA
  static constexpr int kWarpMma = 13;
  static constexpr int kThreads = 512;
  static constexpr uint32_t kRegNorm = 184;  // per-thread registers after the reallocation
  static constexpr uint32_t kRegProd = 72;
  static_assert(128 + kRegNorm + 128 + kRegProd == 4 * 128, "register budget of the launch");
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(M, BN, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(M, D, 1);
  static constexpr uint32_t kIdescPVh = idesc_f16_f32(M, D, 1);  // fp16 P x fp16 V
  static constexpr float kHalfScaleLog2 = 6.0f;                  // fp16 P holds 2^6 p
};

struct ScoreBarriers {
  uint64_t q_full;
  uint64_t k_full[3], k_empty[3], v_full[2], v_empty[2];
  uint64_t s_full[3], p_full[3];
  uint64_t acc_full, acc_empty;  // P_b V_b complete / read by the norm warps
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

using score::exp_f16_store;
using score::exp_split_store;

template <int D, int BN>
__global__ void __launch_bounds__(ScoreCfg<D, BN>::kThreads, 1)
    poem_score_pass2_kernel(const __grid_constant__ CUtensorMap tmQs, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmVh,
                      const ScoreParams p) {
  using C = ScoreCfg<D, BN>;
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
  // the fp16 copy of V was written (and its range flag set) before pass 1 ran
  const bool half_p = (i_lo >= score::kHalfMinTile) && (*p.v_overflow == 0);

  if (tid == 0) {
    mbar_init(&sb->q_full, 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(&sb->k_full[s], 1);
      mbar_init(&sb->k_empty[s], 1);
      mbar_init(&sb->s_full[s], 1);
      mbar_init(&sb->p_full[s], 4);  // barriers signalled by 4 warps: one arrival per warp
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sb->v_full[s], 1);
      mbar_init(&sb->v_empty[s], 1);
      mbar_init(&sb->m_ready[s], 4);
      mbar_init(&sb->m_empty[s], 4);
    }
    mbar_init(&sb->acc_full, 1);
    mbar_init(&sb->acc_empty, 4);
    mbar_init(&sb->drain, 1);
    sb->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::kWarpMma) tmem_alloc<C::kTmemCols>(&sb->tmem_base);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sb->tmem_base;

  if (warp >= C::kWarpProd) {
    // warps 12-15 (one warpgroup): lower the register budget, one instruction for all four
    warpgroup_reg_dec<C::kRegProd>();
    if (warp == C::kWarpProd) {
      // ============================ TMA producer ============================
      if (lane == 0) {
        tma_prefetch_desc(&tmQs);
        tma_prefetch_desc(&tmK);
        const CUtensorMap* mapV = half_p ? &tmVh : &tmV;  // 2-byte elements either way
        tma_prefetch_desc(mapV);
        mbar_arrive_expect_tx(&sb->q_full, C::kQBytes);
        for (int zl = 0; zl < C::kGroups; ++zl) {
          const int z = z0 + zl;  // groups past the end read out-of-range tiles: zero-filled
          const int i = z / G;
          const int hq = g * G + (z - i * G);
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(sQ + c * (C::M * 128) + zl * (C::kRowsPerGroup * 128), &tmQs, &sb->q_full, c * 64, hq, 0,
                        i);
        }
        // K and V rings advance independently: K_b is loaded once S_{b-3} has released
        // its stage, V_b once P V_{b-2} has.
        int kb = 0, vb = 0;
        uint64_t t_last = globaltimer_ns();
        while ((kb < nb || vb < nb) && !sb->abort_flag) {
          bool progressed = false;
          // a fresh stage passes the parity-1 test at once; later, completion #(b/stages - 1)
          if (kb < nb && mbar_try_wait(&sb->k_empty[kb % 3], ((kb / 3) & 1) ^ 1)) {
            const int st = kb % 3;
            mbar_arrive_expect_tx(&sb->k_full[st], C::kKVBytes);
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_3d(sK + st * C::kKVBytes + c * (BN * 128), &tmK, &sb->k_full[st], c * 64, g, kb * BN);
            ++kb;
            progressed = true;
          }
          if (vb < kb && mbar_try_wait(&sb->v_empty[vb & 1], ((vb >> 1) & 1) ^ 1)) {
            const int st = vb & 1;
            mbar_arrive_expect_tx(&sb->v_full[st], C::kKVBytes);
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_3d(sV + st * C::kKVBytes + c * (BN * 128), mapV, &sb->v_full[st], c * 64, g, vb * BN);
            ++vb;
            progressed = true;
          }
          if (progressed) {
            t_last = globaltimer_ns();
          } else if (globaltimer_ns() - t_last > p.err.timeout_ns) {
            sb->abort_flag = 1;
            raise_err(p.err, kErrTimeout);
            break;
          }
        }
        // Drain: the last load issued into each stage must have landed.
        mbar_wait(&sb->q_full, 0, kDrainNs);
        for (int x = max(0, kb - 3); x < kb; ++x) mbar_wait(&sb->k_full[x % 3], (x / 3) & 1, kDrainNs);
        for (int x = max(0, vb - 2); x < vb; ++x) mbar_wait(&sb->v_full[x & 1], (x >> 1) & 1, kDrainNs);
      }
    } else if (warp == C::kWarpMma) {
      // ============================ MMA issuer ============================
      // The whole warp runs this loop converged (waits and operands are warp-uniform);
      // one elected lane issues each MMA and commit.
      // Order S_0, S_1, S_2, PV_0, S_3, PV_1, ...: S_b lands in S buffer b % 3 (free once
      // P V_{b-3}, issued just before, has read it), P_b V_b in the accumulator, started
      // fresh once the norm warps have read P V_{b-1}.
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
      const uint32_t tAcc = tmem + C::kColAcc;
      bool ok = warp_wait(&sb->q_full, 0, sb, p.err);
      // `ready`: P_j, V_j (and this step's K) were all found complete by one joint
      // test; the accumulator, which the norm warps release only shortly before it is
      // needed, is always waited for on its own.
      auto issue_pv = [&](int j, bool ready) -> bool {
        const int s = j % 3, sv = j & 1;
        if (!ready) {
          if (!warp_wait(&sb->p_full[s], (j / 3) & 1, sb, p.err)) return false;
          if (!warp_wait(&sb->v_full[sv], (j >> 1) & 1, sb, p.err)) return false;
        }
        if (j >= 1 && !warp_wait(&sb->acc_empty, (j - 1) & 1, sb, p.err)) return false;
        tc_fence_after();
        const uint32_t tP = tmem + C::kColS + s * 128;
        const uint32_t aVs = aV + sv * C::kKVBytes;
        if (half_p) {
  #pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // keys [16 kk, 16 kk + 16): fp16 P words at [8 kk, 8 kk + 8)
            const uint64_t bdesc = smem_desc_sw128(aVs + kk * 2048, BN * 128, 1024);
            mma_ts_warp(tAcc, tP + kk * 8, bdesc, C::kIdescPVh, kk > 0 ? 1u : 0u);
          }
        } else {
  #pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // keys [16 kk, 16 kk + 16): P_hi words at [16 kk, +8), P_lo at [16 kk + 8, +8)
            const uint64_t bdesc = smem_desc_sw128(aVs + kk * 2048, BN * 128, 1024);
            mma_ts_warp(tAcc, tP + kk * 16, bdesc, C::kIdescPV, kk > 0 ? 1u : 0u);
            mma_ts_warp(tAcc, tP + kk * 16 + 8, bdesc, C::kIdescPV, 1u);
          }
        }
        mma_commit_warp(&sb->v_empty[sv]);
        mma_commit_warp(&sb->acc_full);
        return true;
      };
      for (int b = 0; b < nb && ok; ++b) {
        const int s = b % 3;
        bool ready = mbar_test_wait(&sb->k_full[s], (b / 3) & 1);
        if (b >= 3) {
          const int j = b - 3;
          ready = ready & mbar_test_wait(&sb->p_full[j % 3], (j / 3) & 1) &
                  mbar_test_wait(&sb->v_full[j & 1], (j >> 1) & 1);
        }
        ready = __all_sync(0xffffffffu, ready);
        if (b >= 3 && !issue_pv(b - 3, ready)) { ok = false; break; }
        if (!ready && !warp_wait(&sb->k_full[s], (b / 3) & 1, sb, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tS = tmem + C::kColS + s * 128;
        const uint32_t aKs = aK + s * C::kKVBytes;
  #pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          const uint64_t adesc = smem_desc_sw128(aQ + (kk >> 2) * (C::M * 128) + koff, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(aKs + (kk >> 2) * (BN * 128) + koff, 16, 1024);
          mma_ss_warp(tS, adesc, bdesc, C::kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit_warp(&sb->s_full[s]);
        mma_commit_warp(&sb->k_empty[s]);
      }
      for (int j = max(0, nb - 3); j < nb && ok; ++j)
        if (!issue_pv(j, false)) ok = false;
      mma_commit_warp(&sb->drain);
      mbar_wait(&sb->drain, 0, kDrainNs);
    }  // warps 14-15 idle
  } else if (warp < 4 || warp >= 8) {
    // ================= pass 2: softmax warps 0-3 (even blocks), 8-11 (odd) =================
    const int wg = warp >> 3;
    const int r = tid & 127;
    const int zl = r >> 4;
    const int j = r & 15;
    const int z = z0 + zl;
    const bool valid = (z < n_groups);
    const int i = valid ? z / G : 0;
    const int hq = g * G + (valid ? z - i * G : 0);
    const int qpos = valid ? (i + t0) * BN + j * p.sample_stride : -1;
    const int64_t srow = ((int64_t)hq * p.n_tiles + i) * p.n_sample + j;
    const uint32_t lane_off = ((uint32_t)((warp & 3) * 32) << 16);
    const float sl2 = p.scale_log2;
    const bool in_ws = POEM_IN_BOUNDS(p.err, srow, (int64_t)p.n_q_heads * p.n_tiles * p.n_sample);
    const float lse2 = (valid && in_ws) ? p.ws_lse[srow] : 0.f;
    bool ok = true;
    // Block b's wait on s_full[b % 3] is at most one phase behind: S_{b+3} needs
    // P V_b, which needs this warpgroup's P_b.  m_b goes to slot b & 1 = wg.
    for (int b = wg; b < nb; b += 2) {
      const int s = b % 3, sm = b & 1;
      const uint32_t tS = tmem + lane_off + C::kColS + s * 128;
      if (!warp_wait(&sb->s_full[s], (b / 3) & 1, sb, p.err)) { ok = false; break; }
      tc_fence_after();
      const int lim = qpos - b * BN;
      float msum;
      if (half_p) {
        // 2^6 p in fp16; m_b is the sum of the unscaled fp32 weights
        const float m16 = lse2 - C::kHalfScaleLog2;
        msum = ((b < i_lo) ? exp_f16_store<BN, false>(tS, sl2, m16, lim)
                           : exp_f16_store<BN, true>(tS, sl2, m16, lim)) *
               (1.0f / 64.0f);
      } else {
        msum = (b < i_lo) ? exp_split_store<BN, false>(tS, sl2, lse2, lim)
                          : exp_split_store<BN, true>(tS, sl2, lse2, lim);
      }
      // hand m_b to the norm warps (slot b % 2 is free once block b-2's norm read it)
      if (b >= 2 && !warp_wait(&sb->m_empty[sm], ((b >> 1) & 1) ^ 1, sb, p.err)) ok = false;
      sm_m[sm * 128 + r] = valid ? msum : 0.f;
      warp_arrive(&sb->m_ready[sm]);
      tmem_st_wait();
      tc_fence_before();
      warp_arrive(&sb->p_full[s]);
      if (!__all_sync(0xffffffffu, ok)) break;
    }
  } else {
    // ====================== pass 2: norm warps 4-7 ======================
    // The row's dense output o (pass 1) stays in registers; per block b the
    // accumulator holds P_b V_b (2^6 P_b V_b with the fp16 P), and
    // I_b = || P_b V_b - m_b o ||.
    warpgroup_reg_inc<C::kRegNorm>();
    const int r = tid - 128;                 // TMEM lane = row
    const int zl = r >> 4;
    const int j = r & 15;
    const int z = z0 + zl;
    const bool valid = (z < n_groups);
    const int i = valid ? z / G : 0;
    const int hq = g * G + (valid ? z - i * G : 0);
    const int64_t srow = ((int64_t)hq * p.n_tiles + i) * p.n_sample + j;
    const uint32_t lane_off = ((uint32_t)((warp - 4) * 32) << 16);
    float od[D];
    {
      const float4* o4 = reinterpret_cast<const float4*>(p.ws_o + srow * D);
      const bool in_ws = POEM_IN_BOUNDS(p.err, srow, (int64_t)p.n_q_heads * p.n_tiles * p.n_sample);
#pragma unroll
      for (int x = 0; x < D / 4; ++x) {
        const float4 v = (valid && in_ws) ? o4[x] : make_float4(0.f, 0.f, 0.f, 0.f);
        od[4 * x] = v.x;
        od[4 * x + 1] = v.y;
        od[4 * x + 2] = v.z;
        od[4 * x + 3] = v.w;
      }
    }
    const int64_t tri = row_off(p.n_tiles, t0, hq, i);
    for (int b = 0; b < nb; ++b) {
      const int s = b & 1;
      if (!warp_wait(&sb->acc_full, b & 1, sb, p.err)) break;
      if (!warp_wait(&sb->m_ready[s], (b >> 1) & 1, sb, p.err)) break;
      tc_fence_after();
      const float mb_row = sm_m[s * 128 + r];
      warp_arrive(&sb->m_empty[s]);
      const uint32_t tAcc = tmem + lane_off + C::kColAcc;
      const float acc_scale = half_p ? 64.0f : 1.0f;  // the accumulator holds acc_scale P_b V_b
      const uint64_t negm2 = f2_pack(-mb_row * acc_scale, -mb_row * acc_scale);
      uint64_t acc2 = f2_pack(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint32_t pv[16];
        tmem_ld16(tAcc + c * 16, pv);
        tmem_ld_wait();
        tmem_reg_fence16(pv);
#pragma unroll
        for (int x = 0; x < 16; x += 2) {
          const uint64_t e = f2_fma(negm2, f2_pack(od[c * 16 + x], od[c * 16 + x + 1]),
                                    f2_pack(__uint_as_float(pv[x]), __uint_as_float(pv[x + 1])));
          acc2 = f2_fma(e, e, acc2);
        }
      }
      // P V_b has been read: the accumulator may take block b + 1.
      tc_fence_before();
      warp_arrive(&sb->acc_empty);
      float a0, a1;
      f2_unpack(acc2, a0, a1);
      float Ib = valid ? sqrtf(a0 + a1) * (1.0f / acc_scale) : 0.f;
      float mb = valid ? mb_row : 0.f;
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) {  // max over the 16 queries of the group
        Ib = fmaxf(Ib, __shfl_xor_sync(0xffffffffu, Ib, off));
        mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
      }
      if (j == 0 && valid && b <= i + t0 && POEM_IN_BOUNDS(p.err, tri + b, p.n_entries)) {
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

template <int D, int BN>
cudaError_t launch_pass2(const CUtensorMap& tmQs, const CUtensorMap& tmK, const CUtensorMap& tmV,
                         const CUtensorMap& tmVh, const ScoreParams& p, int grid, cudaStream_t stream) {
  using C = ScoreCfg<D, BN>;
  cudaError_t e = ensure_smem_limit(poem_score_pass2_kernel<D, BN>, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  poem_score_pass2_kernel<D, BN><<<grid, C::kThreads, C::kSmemBytes, stream>>>(tmQs, tmK, tmV, tmVh, p);
  return cudaGetLastError();
}

// The fp16 copy of V, pass 1 (poem_score_pass1.cu: o and lse of the sampled
// queries), then pass 2.
template <int D, int BN>
cudaError_t launch_score_t(const CUtensorMap& tmQs, const CUtensorMap& tmK, const CUtensorMap& tmV,
                           const CUtensorMap& tmVh, const ScoreParams& p, cudaStream_t stream) {
  const int ctas_per_g = (p.n_tiles * p.group + 7) / 8;
  const int grid = p.n_kv_heads * ctas_per_g;
  cudaError_t e = launch_v_to_half(p, D, stream);
  if (e != cudaSuccess) return e;
  e = launch_score_pass1(D, BN, tmQs, tmK, tmV, tmVh, p, grid, stream);
  if (e != cudaSuccess) return e;
  return launch_pass2<D, BN>(tmQs, tmK, tmV, tmVh, p, grid, stream);
}

}  // namespace

cudaError_t launch_score(int head_dim, int block, const CUtensorMap& tmQs, const CUtensorMap& tmK,
                         const CUtensorMap& tmV, const CUtensorMap& tmVh, const ScoreParams& p, cudaStream_t stream) {
  if (head_dim == 128 && block == 128) return launch_score_t<128, 128>(tmQs, tmK, tmV, tmVh, p, stream);
  if (head_dim == 128 && block == 64) return launch_score_t<128, 64>(tmQs, tmK, tmV, tmVh, p, stream);
  if (head_dim == 64 && block == 128) return launch_score_t<64, 128>(tmQs, tmK, tmV, tmVh, p, stream);
  if (head_dim == 64 && block == 64) return launch_score_t<64, 64>(tmQs, tmK, tmV, tmVh, p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace poem
