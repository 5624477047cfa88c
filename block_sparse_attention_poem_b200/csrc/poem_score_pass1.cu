// poem_score_pass1.cu -- pass 1 of the exact block scores (sm_100a): the dense causal
// attention of the sampled queries.
//
// For the 16 strided sampled queries q_j = iB + j (B / 16) of every (head, query tile)
// this pass computes the dense softmax output o and the log-sum-exp of the scaled
// logits (log2 units) -- o is the dense reference output of the reading note
// "Attention deletion error", Section 4.1, against which pass 2 (poem_score.cu)
// measures every block's deviation I_b = || P_b V_b - m_b o || (Equation (4)).
// I_b can cancel, so o is needed to ~1e-6 relative.  P enters the P V contraction
//   - as one fp16 matrix (11 significant bits, one MMA) on an fp16 copy of V, in the
//     CTAs whose query tiles are all >= 32: o averages over >= 32 blocks of keys and
//     its error stays far inside the score tolerance (a simulation against the fp64
//     oracle on the Llama-shaped 32K layer: 3% of the tolerance for tiles >= 32);
//     P is scaled by 2^6 (reference max - 6) so it stays in fp16's normal range;
//   - as a bf16 hi/lo pair (two MMAs into one accumulator, ~16 significant bits) in
//     the CTAs with earlier tiles, where few keys are visible (tile 0's one block
//     cancels exactly), and everywhere when a finite |v| exceeds the fp16 range
//     (the V copy then raises a flag in the workspace).
//
// Packing as in pass 2: one CTA per SM holds 8 groups of 16 sampled queries of one KV
// head (2 adjacent tiles x 4 query heads for 4-way GQA), gathered by one 4-D TMA box
// per group, and sweeps key blocks 0 .. (largest tile of the CTA).
//
// Pipeline:
//   TMEM  S buffers s = 0, 1, 2 at [128 s, 128 s + BN); O at [384, 384 + D).  With
//         three S buffers the MMAs run up to two blocks ahead of the softmax.
//   smem  Q tile, 3-stage K ring, 2-stage V ring (192 KB at d = 128).
//   warps 0-3 / 4-7: online softmax of the even / odd key blocks, one sampled query
//         per thread.  The running state passes between the two warpgroups through
//         shared memory: block b's reference max (published right after its row max)
//         and the row sum through b (published after its exponentials).  The
//         reference moves only when the max grows by more than 2^8, and O is then
//         rescaled once P V_{b-1} has completed.  The warpgroup of the last block
//         writes o and lse.  Warp 8: TMA, K and V rings advancing independently;
//         warp 9: MMAs, converged, issued by one elected lane; warps 10-11 idle.
//   Registers per thread: 168 at launch; warps 8-11 lower theirs to 56 and the two
//   softmax warpgroups raise theirs to 224 (224 + 224 + 56 = 3 x 168).
//   MMA order: S_0, S_1, S_2, PV_0, S_3, PV_1, ...  (S_b follows P V_{b-3}, which
//   freed its S buffer).
//
// Every mbarrier wait is made at most one phase behind its barrier.  A rescale of O at
// block b waits for P V_{b-1} on accumulator barrier (b - 1) % 2: P V_{b+1} cannot
// start before this block's P, so that barrier is within one phase of the wait; the
// hand-off barriers of block b - 1 likewise cannot move on before block b has
// published its own state.  The end of the sweep waits on its own
// barrier (o_full), committed once after the last P V.
#include "common.cuh"
#include "fwd_common.cuh"
#include "score_common.cuh"

namespace poem {
namespace {

template <int D, int BN>
struct P1Cfg {
  static constexpr int M = 128;
  static constexpr int kGroups = 8;
  static constexpr int kRowsPerGroup = 16;
  static constexpr int kChunks = D / 64;
  static constexpr int kStagesK = 3;
  static constexpr int kStagesV = 2;
  static constexpr int kQBytes = M * D * 2;
  static constexpr int kKVBytes = BN * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kStagesK * kKVBytes;
  static constexpr int kOffBar = kOffV + kStagesV * kKVBytes;
  static constexpr int kOffX = kOffBar + 256;  // [2][128] reference maxima, [2][128] row sums
  // at least 120 KB so that one CTA (holding all 512 TMEM columns) occupies an SM
  static constexpr int kSmemBytes =
      (kOffX + 4 * 128 * 4 + 1024) > 122880 ? (kOffX + 4 * 128 * 4 + 1024) : 122880;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 384;
  static constexpr int kWarpProd = 8;
  static constexpr int kWarpMma = 9;
  static constexpr int kThreads = 384;
  static constexpr uint32_t kRegSoftmax = 224;  // per-thread registers after the reallocation
  static constexpr uint32_t kRegProd = 56;
  static_assert(2 * kRegSoftmax + kRegProd == 3 * 168, "register budget of the launch");
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(M, BN, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(M, D, 1);
  static constexpr uint32_t kIdescPVh = idesc_f16_f32(M, D, 1);  // fp16 P x fp16 V
};

struct P1Barriers {
  uint64_t q_full;
  uint64_t k_full[3], k_empty[3];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[3], p_full[3];
  uint64_t acc_full[2];  // P V_j complete, on barrier j % 2
  uint64_t o_full;       // the last P V complete
  uint64_t ref_ready[2], l_ready[2];  // block b's reference max / row sum, slot b % 2
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

using fwd::kDrainNs;
using fwd::wait_or_abort;
using score::exp_f16_store_regs;
using score::exp_split_store_regs;

// ---- V -> fp16 -----------------------------------------------------------------
// One thread converts 8 consecutive channels of one (token, KV head) row of V into the
// dense fp16 copy [n_kv, Hkv, D] (exact for every bf16 value in fp16's range); a finite
// |v| above the fp16 maximum sets the flag.
__global__ void __launch_bounds__(256) v_to_half_kernel(const ScoreParams p, int head_dim) {
  const int per_row = head_dim / 8;
  const int64_t n_items = (int64_t)p.n_kv * p.n_kv_heads * per_row;
  bool over = false;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < n_items;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = it / per_row;
    const int c8 = (int)(it - row * per_row) * 8;
    const int64_t t = row / p.n_kv_heads;
    const int h = (int)(row - t * p.n_kv_heads);
    const uint4 raw = *reinterpret_cast<const uint4*>(p.v_src + t * p.v_stride_tok + h * p.v_stride_head + c8);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t o[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float lo = bf16lo_to_f32(w[x]), hi = bf16hi_to_f32(w[x]);
      over |= (fabsf(lo) > 65504.f && fabsf(lo) <= 3.402823466e38f) ||
              (fabsf(hi) > 65504.f && fabsf(hi) <= 3.402823466e38f);
      o[x] = pack_f16x2(lo, hi);
    }
    *reinterpret_cast<uint4*>(p.v_half + row * head_dim + c8) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (__any_sync(0xffffffffu, over) && (threadIdx.x & 31) == 0) atomicOr(p.v_overflow, 1u);
}
using score::load_row;
using score::row_max_regs;

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, P1Barriers* sb, const DevErr& e) {
  return __all_sync(0xffffffffu, wait_or_abort(bar, parity, sb, e));
}

// CTA -> (KV head, first group): KV-head-major, the CTAs holding the last tiles first.
__device__ __forceinline__ void p1_cta_coords(int cta, int ctas_per_g, int& g, int& z0) {
  g = cta / ctas_per_g;
  const int c = ctas_per_g - 1 - (cta - g * ctas_per_g);
  z0 = c * 8;
}

template <int D, int BN>
__global__ void __launch_bounds__(P1Cfg<D, BN>::kThreads, 1)
    poem_score_pass1_kernel(const __grid_constant__ CUtensorMap tmQs, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmVh,
                            const ScoreParams p) {
  using C = P1Cfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  P1Barriers* sb = reinterpret_cast<P1Barriers*>(smem + C::kOffBar);
  float* x_ref = reinterpret_cast<float*>(smem + C::kOffX);  // [2][128]
  float* x_l = x_ref + 2 * 128;                               // [2][128]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = p.group;
  const int n_groups = p.n_tiles * G;  // per KV head
  const int ctas_per_g = (n_groups + 7) / 8;
  int g, z0;
  p1_cta_coords(blockIdx.x, ctas_per_g, g, z0);
  const int z_last = min(z0 + 7, n_groups - 1);
  const int t0 = p.q_tile0;
  const int nb = z_last / G + 1 + t0;  // key blocks 0 .. largest (global) tile of the CTA
  const int i_lo = z0 / G + t0;        // blocks < i_lo need no causal mask
  // fp16 P for this CTA (uniform): all its tiles >= 32 and V inside fp16's range
  const bool half_p = (i_lo >= score::kHalfMinTile) && (*p.v_overflow == 0);

  if (tid == 0) {
    mbar_init(&sb->q_full, 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(&sb->k_full[s], 1);
      mbar_init(&sb->k_empty[s], 1);
      mbar_init(&sb->s_full[s], 1);
      mbar_init(&sb->p_full[s], 4);  // one arrival per softmax warp
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sb->v_full[s], 1);
      mbar_init(&sb->v_empty[s], 1);
      mbar_init(&sb->acc_full[s], 1);
      mbar_init(&sb->ref_ready[s], 4);  // one arrival per softmax warp
      mbar_init(&sb->l_ready[s], 4);
    }
    mbar_init(&sb->o_full, 1);
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
    // warps 8-11 (one warpgroup): lower the register budget, one instruction for all four
    warpgroup_reg_dec<C::kRegProd>();
    if (warp == C::kWarpProd) {
      // ============================ TMA producer ============================
      // K and V rings advance independently: K_b is loaded once S_{b-3} has released its
      // stage, V_b once P V_{b-2} has.
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
        int kb = 0, vb = 0;
        uint64_t t_last = globaltimer_ns();
        while ((kb < nb || vb < nb) && !sb->abort_flag) {
          bool progressed = false;
          // a fresh stage passes the parity-1 test at once; later, completion #(b/stages - 1)
          if (kb < nb && mbar_try_wait(&sb->k_empty[kb % 3], ((kb / 3) & 1) ^ 1)) {
            const int s = kb % 3;
            mbar_arrive_expect_tx(&sb->k_full[s], C::kKVBytes);
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_3d(sK + s * C::kKVBytes + c * (BN * 128), &tmK, &sb->k_full[s], c * 64, g, kb * BN);
            ++kb;
            progressed = true;
          }
          if (vb < kb && mbar_try_wait(&sb->v_empty[vb & 1], ((vb >> 1) & 1) ^ 1)) {
            const int s = vb & 1;
            mbar_arrive_expect_tx(&sb->v_full[s], C::kKVBytes);
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_3d(sV + s * C::kKVBytes + c * (BN * 128), mapV, &sb->v_full[s], c * 64, g, vb * BN);
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
        for (int b = max(0, kb - 3); b < kb; ++b) mbar_wait(&sb->k_full[b % 3], (b / 3) & 1, kDrainNs);
        for (int b = max(0, vb - 2); b < vb; ++b) mbar_wait(&sb->v_full[b & 1], (b >> 1) & 1, kDrainNs);
      }
    } else if (warp == C::kWarpMma) {
      // ============================ MMA issuer ============================
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
      const uint32_t tO = tmem + C::kColO;
      bool ok = warp_wait(&sb->q_full, 0, sb, p.err);
      // `ready`: the step's barriers were all found complete by one joint test.
      auto issue_pv = [&](int j, bool ready) -> bool {
        const int s = j % 3, sv = j & 1;
        if (!ready) {
          if (!warp_wait(&sb->p_full[s], (j / 3) & 1, sb, p.err)) return false;
          if (!warp_wait(&sb->v_full[sv], (j >> 1) & 1, sb, p.err)) return false;
        }
        tc_fence_after();
        const uint32_t tP = tmem + s * 128;
        const uint32_t aVs = aV + sv * C::kKVBytes;
        if (half_p) {
  #pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // keys [16 kk, 16 kk + 16): fp16 P words at [8 kk, +8)
            const uint64_t bdesc = smem_desc_sw128(aVs + kk * 2048, BN * 128, 1024);
            mma_ts_warp(tO, tP + kk * 8, bdesc, C::kIdescPVh, (j > 0 || kk > 0) ? 1u : 0u);
          }
        } else {
  #pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // keys [16 kk, 16 kk + 16): P_hi words at [16 kk, +8), P_lo at [16 kk + 8, +8)
            const uint64_t bdesc = smem_desc_sw128(aVs + kk * 2048, BN * 128, 1024);
            mma_ts_warp(tO, tP + kk * 16, bdesc, C::kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
            mma_ts_warp(tO, tP + kk * 16 + 8, bdesc, C::kIdescPV, 1u);
          }
        }
        mma_commit_warp(&sb->v_empty[sv]);
        mma_commit_warp(&sb->acc_full[j & 1]);
        if (j == nb - 1) mma_commit_warp(&sb->o_full);
        return true;
      };
      for (int b = 0; b < nb && ok; ++b) {
        const int s = b % 3;
        // Every barrier of this step (P V_{b-3}'s P and V, S_b's K) tested at once:
        // normally all are complete, and one test latency replaces three successive
        // waits.  Otherwise each is waited for in turn, bounded.
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
        const uint32_t tS = tmem + s * 128;
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
    }  // warps 10-11 idle
  } else {
    // ============================ softmax warps ============================
    warpgroup_reg_inc<C::kRegSoftmax>();
    const int wg = warp >> 2;                // 0: even blocks, 1: odd blocks
    const int r = tid & 127;                 // TMEM lane = sampled row
    const int zl = r >> 4;
    const int j = r & 15;
    const int z = z0 + zl;
    const bool valid = (z < n_groups);
    const int i = valid ? z / G : 0;
    const int hq = g * G + (valid ? z - i * G : 0);
    const int qpos = valid ? (i + t0) * BN + j * p.sample_stride : -1;  // key position; -1: padding row
    const int64_t srow = ((int64_t)hq * p.n_tiles + i) * p.n_sample + j;
    const uint32_t lane_off = ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t tO = tmem + lane_off + C::kColO;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;                 // reference max after this warpgroup's last block
    float l_run = 0.f;                       // row sum through that block
    bool ok = true;
    for (int b = wg; b < nb; b += 2) {
      const int s = b % 3;
      const uint32_t tS = tmem + lane_off + s * 128;
      // S_b ready (S_{b+3} needs P V_b, hence this warpgroup's P_b)
      if (!warp_wait(&sb->s_full[s], (b / 3) & 1, sb, p.err)) { ok = false; break; }
      tc_fence_after();
      const int lim = qpos - b * BN;  // columns <= lim are visible to this query
      uint32_t a[BN / 32][32];        // the row of S, read once
      load_row<BN>(tS, a);
      const float mx = (b < i_lo) ? row_max_regs<BN, false>(a, lim) : row_max_regs<BN, true>(a, lim);
      // the reference through block b - 1 (the other warpgroup's)
      float m_prev = -INFINITY;
      if (b > 0) {
        if (!warp_wait(&sb->ref_ready[(b - 1) & 1], ((b - 1) >> 1) & 1, sb, p.err)) { ok = false; break; }
        m_prev = x_ref[((b - 1) & 1) * 128 + r];
      }
      const float m_new = fmaxf(m_prev, mx * sl2);
      const bool grow = (m_new > m_prev + 8.0f);
      float alpha = 1.f, m_cur = m_prev;
      if (grow) {
        alpha = (m_prev == -INFINITY) ? 0.f : ex2_approx(m_prev - m_new);
        m_cur = m_new;
      }
      x_ref[(b & 1) * 128 + r] = m_cur;
      warp_arrive(&sb->ref_ready[b & 1]);
      if (b >= 1 && __any_sync(0xffffffffu, grow)) {
        // O holds P V_0 .. P V_{b-1} (against m_prev) once P V_{b-1} is complete; P V_b
        // waits for this block's P, so O may then be rescaled in place.
        if (!warp_wait(&sb->acc_full[(b - 1) & 1], ((b - 1) >> 1) & 1, sb, p.err)) { ok = false; break; }
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
      // reference of the weights: the running max, lowered by 6 for fp16 P so that
      // P <= 2^14 and weights down to 2^-20 of the reference keep full fp16 precision
      const float m_use = (m_cur == -INFINITY) ? 0.f : (half_p ? m_cur - 6.0f : m_cur);
      float bsum;
      if (half_p)
        bsum = (b < i_lo) ? exp_f16_store_regs<BN, false>(tS, a, sl2, m_use, lim)
                          : exp_f16_store_regs<BN, true>(tS, a, sl2, m_use, lim);
      else
        bsum = (b < i_lo) ? exp_split_store_regs<BN, false>(tS, a, sl2, m_use, lim)
                          : exp_split_store_regs<BN, true>(tS, a, sl2, m_use, lim);
      tmem_st_wait();
      tc_fence_before();
      warp_arrive(&sb->p_full[s]);
      // the row sum through b - 1, then through b
      float l_prev = 0.f;
      if (b > 0) {
        if (!warp_wait(&sb->l_ready[(b - 1) & 1], ((b - 1) >> 1) & 1, sb, p.err)) { ok = false; break; }
        l_prev = x_l[((b - 1) & 1) * 128 + r];
      }
      l_run = l_prev * alpha + bsum;
      m_run = m_cur;
      x_l[(b & 1) * 128 + r] = l_run;
      warp_arrive(&sb->l_ready[b & 1]);
    }
    // ---- epilogue (the warpgroup of the last block): o = O / l, lse = m + log2(l) ----
    if (((nb - 1) & 1) == wg && __all_sync(0xffffffffu, ok && !sb->abort_flag) &&
        warp_wait(&sb->o_full, 0, sb, p.err)) {
      tc_fence_after();
      const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
      float* dst = p.ws_o + srow * D;
      const bool in_ws = POEM_IN_BOUNDS(p.err, srow, (int64_t)p.n_q_heads * p.n_tiles * p.n_sample);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32(tO + c * 32, ov);
        tmem_ld_wait();
        tmem_reg_fence(ov);
        if (valid && in_ws) {
          float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
          for (int x = 0; x < 8; ++x)
            d4[x] = make_float4(__uint_as_float(ov[4 * x]) * inv_l, __uint_as_float(ov[4 * x + 1]) * inv_l,
                                __uint_as_float(ov[4 * x + 2]) * inv_l, __uint_as_float(ov[4 * x + 3]) * inv_l);
        }
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : (half_p ? m_run - 6.0f : m_run);
      if (valid && in_ws) p.ws_lse[srow] = (l_run > 0.f) ? m_use + __log2f(l_run) : -INFINITY;
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
cudaError_t launch_p1_t(const CUtensorMap& tmQs, const CUtensorMap& tmK, const CUtensorMap& tmV,
                        const CUtensorMap& tmVh, const ScoreParams& p, int grid, cudaStream_t stream) {
  using C = P1Cfg<D, BN>;
  cudaError_t e = ensure_smem_limit(poem_score_pass1_kernel<D, BN>, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  poem_score_pass1_kernel<D, BN><<<grid, C::kThreads, C::kSmemBytes, stream>>>(tmQs, tmK, tmV, tmVh, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_v_to_half(const ScoreParams& p, int head_dim, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(p.v_overflow, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return e;
  const int64_t items = (int64_t)p.n_kv * p.n_kv_heads * (head_dim / 8);
  const int64_t want = (items + 255) / 256;
  const int grid = (int)(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
  v_to_half_kernel<<<grid, 256, 0, stream>>>(p, head_dim);
  return cudaGetLastError();
}

cudaError_t launch_score_pass1(int head_dim, int block, const CUtensorMap& tmQs, const CUtensorMap& tmK,
                               const CUtensorMap& tmV, const CUtensorMap& tmVh, const ScoreParams& p, int grid,
                               cudaStream_t stream) {
  if (head_dim == 128 && block == 128) return launch_p1_t<128, 128>(tmQs, tmK, tmV, tmVh, p, grid, stream);
  if (head_dim == 128 && block == 64) return launch_p1_t<128, 64>(tmQs, tmK, tmV, tmVh, p, grid, stream);
  if (head_dim == 64 && block == 128) return launch_p1_t<64, 128>(tmQs, tmK, tmV, tmVh, p, grid, stream);
  if (head_dim == 64 && block == 64) return launch_p1_t<64, 64>(tmQs, tmK, tmV, tmVh, p, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace poem
