// bsa_fwd.cu -- causal GQA block-sparse attention forward on sm_100a.
//
// Computes, for every listed (head h, query tile i) row, the renormalised sparse
// output of the reading note "Attention deletion error", Section 4.1: softmax
// attention of each query over only the keys of the kept blocks (and, on the
// diagonal block, only keys at or before the query).
//
// One CTA per (head, tile) row, 128 query rows (M = 128; with 64-token blocks the
// upper 64 rows are padding and are not stored).  With a query offset (chunked
// prefill) local query tile i is global tile q_tile0 + i: it sees key blocks
// 0 .. q_tile0 + i and its diagonal block is q_tile0 + i.  Roles:
//   warps 0-3  softmax: one query row per thread; reads S from TMEM, keeps the
//              running max / sum, writes P (bf16) back into the S columns, rescales
//              O in TMEM only when the max grows by more than 2^8, and runs the
//              epilogue (O / l -> bf16, lse).
//   warp 4     TMA producer: Q once, then K_j and V_j of every listed block.
//   warp 5     MMA issuer (converged warp; one elected lane issues): S = Q K_j^T
//              (SS form), O += P V_j (P read from TMEM) in two 64-key halves, each
//              started as soon as the softmax warps have written that half of P;
//              completion tracked with tcgen05.commit -> mbarriers.
// TMEM: 256 columns per CTA -- S/P at [0, BN), O at [128, 128 + D).  Shared
// memory holds one Q, one K and one V tile (96 KB at D = BN = 128), so two CTAs
// run per SM and their softmax / MMA phases interleave on the tensor cores.
#include "common.cuh"
#include "fwd_common.cuh"

namespace poem {
namespace {

template <int D, int BN>
struct FwdCfg {
  static constexpr int M = 128;
  static constexpr int kChunks = D / 64;              // 128-byte column chunks per row
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
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColO = 128;
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(M, BN, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(M, D, 1);
};

struct FwdBarriers {
  uint64_t q_full, k_full, k_empty, v_full, v_empty, s_full, p_half[2], o_full, drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

using fwd::block_ok;
using fwd::exp_pack_store;
using fwd::kDrainNs;
using fwd::wait_or_abort;
using fwd::warp_wait_or_abort;

template <int D, int BN>
__global__ void __launch_bounds__(kThreadsFwd, 2)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  FwdBarriers* sb = reinterpret_cast<FwdBarriers*>(smem + C::kOffBar);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---- which (head, tile) row this CTA computes ----
  const int unit = blockIdx.x;
  const int row = p.order ? p.order[unit] : default_row_of_unit(unit, p.n_tiles, p.group);
  if (row < 0 || row >= p.n_q_heads * p.n_tiles) {  // uniform for the whole CTA
    if (tid == 0) raise_err(p.err, kErrBadList);
    return;
  }
  const int h = row / p.n_tiles;
  const int tile = row - h * p.n_tiles;   // local query tile (row of Q / O)
  const int gtile = tile + p.q_tile0;     // its global index: key blocks 0 .. gtile are visible
  const int hk = h / p.group;
  const int beg = p.row_ptr[row];
  int end = p.row_ptr[row + 1];
  if (end < beg) {
    if (tid == 0) raise_err(p.err, kErrBadList);
    end = beg;
  }

  if (tid == 0) {
    mbar_init(&sb->q_full, 1);
    mbar_init(&sb->k_full, 1);
    mbar_init(&sb->k_empty, 1);
    mbar_init(&sb->v_full, 1);
    mbar_init(&sb->v_empty, 1);
    mbar_init(&sb->s_full, 1);
    mbar_init(&sb->p_half[0], 4);  // one arrival per softmax warp
    mbar_init(&sb->p_half[1], 4);
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
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int q_issued = 0, k_issued = 0, v_issued = 0;
      bool have_any = false;
      for (int e = beg; e < end; ++e) {
        if (block_ok(p.col_idx[e], gtile)) { have_any = true; break; }
      }
      if (have_any) {
        mbar_arrive_expect_tx(&sb->q_full, C::kQBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(sQ + c * (C::M * 128), &tmQ, &sb->q_full, c * 64, h, tile * BN);
        q_issued = 1;
      }
      for (int e = beg; e < end && !sb->abort_flag; ++e) {
        const int id = p.col_idx[e];
        if (!block_ok(id, gtile)) {
          raise_err(p.err, kErrBadList);
          continue;
        }
        if (!wait_or_abort(&sb->k_empty, (k_issued & 1) ^ 1, sb, p.err)) break;
        mbar_arrive_expect_tx(&sb->k_full, C::kKVBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(sK + c * (BN * 128), &tmK, &sb->k_full, c * 64, hk, id * BN);
        ++k_issued;
        if (!wait_or_abort(&sb->v_empty, (v_issued & 1) ^ 1, sb, p.err)) break;
        mbar_arrive_expect_tx(&sb->v_full, C::kKVBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(sV + c * (BN * 128), &tmV, &sb->v_full, c * 64, hk, id * BN);
        ++v_issued;
      }
      // Drain: the last issued loads must have landed before the CTA may exit
      // (each barrier has at most one load in flight).
      if (q_issued) mbar_wait(&sb->q_full, 0, kDrainNs);
      if (k_issued) mbar_wait(&sb->k_full, (k_issued - 1) & 1, kDrainNs);
      if (v_issued) mbar_wait(&sb->v_full, (v_issued - 1) & 1, kDrainNs);
    }
  } else if (warp == 5) {
    // ============================ MMA issuer ============================
    // The whole warp runs the loop converged (list entries, waits and operands are
    // warp-uniform); one elected lane issues each MMA and commit.
    const uint32_t tS = tmem + C::kColS;
    const uint32_t tO = tmem + C::kColO;
    const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
    int it = 0;
    bool ok = true;
    bool q_ready = false;
    // O += P_j V_j in two 64-key halves, each issued as soon as the softmax warps
    // have written that half of P_j.
    auto issue_pv = [&](int j) -> bool {
      if (!warp_wait_or_abort(&sb->v_full, j & 1, sb, p.err)) return false;
#pragma unroll
      for (int hv = 0; hv < BN / 64; ++hv) {
        if (!warp_wait_or_abort(&sb->p_half[hv], j & 1, sb, p.err)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = hv * 4; kk < hv * 4 + 4; ++kk) {
          // V tile is MN-major (d contiguous): LBO = stride between 64-wide d chunks,
          // SBO = stride between 8-key groups; a k-step covers 16 keys = 2 groups.
          const uint64_t bdesc = smem_desc_sw128(aV + kk * 2048, BN * 128, 1024);
          mma_ts_warp(tO, tS + kk * 8, bdesc, C::kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
        }
      }
      mma_commit_warp(&sb->v_empty);
      return true;
    };
    for (int e = beg; e < end && ok; ++e) {
      if (!block_ok(p.col_idx[e], gtile)) continue;
      if (!q_ready) {
        if (!warp_wait_or_abort(&sb->q_full, 0, sb, p.err)) { ok = false; break; }
        q_ready = true;
      }
      if (it > 0 && !issue_pv(it - 1)) { ok = false; break; }
      if (!warp_wait_or_abort(&sb->k_full, it & 1, sb, p.err)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        // Q and K tiles are K-major, 128-byte swizzled; a k-step is 16 elements (32 B)
        // inside a 64-element chunk; chunks are whole row-blocks apart.
        const uint32_t koff = (kk & 3) * 32;
        const uint64_t adesc = smem_desc_sw128(aQ + (kk >> 2) * (C::M * 128) + koff, 16, 1024);
        const uint64_t bdesc = smem_desc_sw128(aK + (kk >> 2) * (BN * 128) + koff, 16, 1024);
        mma_ss_warp(tS, adesc, bdesc, C::kIdescQK, kk > 0 ? 1u : 0u);
      }
      mma_commit_warp(&sb->s_full);
      mma_commit_warp(&sb->k_empty);
      ++it;
    }
    if (ok && it > 0) {
      if (issue_pv(it - 1)) mma_commit_warp(&sb->o_full);
    }
    // Drain every MMA this warp issued before TMEM is released.
    mma_commit_warp(&sb->drain);
    mbar_wait(&sb->drain, 0, kDrainNs);
  } else {
    // ============================ softmax warps ============================
    const int r = tid;                       // query row within the tile (TMEM lane)
    const int qpos = tile * BN + r;          // query token index of this row (row of O / lse)
    const int kpos = gtile * BN + r;         // its position among the keys
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t tS = lane_base + C::kColS;
    const uint32_t tO = lane_base + C::kColO;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;                 // running max, log2 units of scaled logits
    float l_run = 0.f;                       // running sum of the weights
    int it = 0;
    bool ok = true;
    int id = (beg < end) ? p.col_idx[beg] : -1;
    for (int e = beg; e < end; ++e) {
      const int id_next = (e + 1 < end) ? p.col_idx[e + 1] : -1;  // prefetched a block ahead
      if (block_ok(id, gtile)) {
        // tcgen05.ld is warp-collective: every lane of the warp takes the same branch.
        if (!__all_sync(0xffffffffu, wait_or_abort(&sb->s_full, it & 1, sb, p.err))) { ok = false; break; }
        tc_fence_after();
        const bool diag = (id == gtile);
        const int lim = kpos - id * BN;  // on the diagonal block, columns <= lim are visible
        // row max of S_j (all column chunks, one wait)
        float mx = -INFINITY;
        {
          uint32_t sv[BN / 32][32];
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + c * 32, sv[c]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) tmem_reg_fence(sv[c]);
          // four independent partial maxima (short dependency chains)
          float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          if (diag) {  // uniform branch
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
#pragma unroll
              for (int x = 0; x < 32; ++x)
                pm[x & 3] = fmaxf(pm[x & 3], (c * 32 + x <= lim) ? __uint_as_float(sv[c][x]) : -INFINITY);
          } else {
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
#pragma unroll
              for (int x = 0; x < 32; x += 2)
                pm[(x >> 1) & 3] = fmax3(pm[(x >> 1) & 3], __uint_as_float(sv[c][x]), __uint_as_float(sv[c][x + 1]));
          }
          mx = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3]));
        }
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool grow = (m_new > m_run + 8.0f);
        float alpha = 1.f;
        if (grow) {
          alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        // O must be rescaled when this row's reference max moved (S_j complete implies
        // the previous P V_{j-1} is complete: the MMAs run in issue order).
        if (it > 0 && __any_sync(0xffffffffu, grow)) {
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
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        if (diag)
          exp_pack_store<BN, true>(tS, sl2, m_use, lim, &l_run, sb->p_half);
        else
          exp_pack_store<BN, false>(tS, sl2, m_use, lim, &l_run, sb->p_half);
        ++it;
      }
      id = id_next;
    }
    // ---- epilogue ----
    if (__all_sync(0xffffffffu, ok && !sb->abort_flag)) {
      const bool store = (r < BN);
      __nv_bfloat16* orow = p.o + (int64_t)qpos * p.o_stride_tok + (int64_t)h * p.o_stride_head;
      if (it > 0) {
        if (__all_sync(0xffffffffu, wait_or_abort(&sb->o_full, 0, sb, p.err))) {
          tc_fence_after();
          const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
          uint32_t ov[D / 32][32];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, ov[c]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            tmem_reg_fence(ov[c]);
            if (store) {
              uint32_t w[16];
#pragma unroll
              for (int x = 0; x < 16; ++x)
                w[x] = pack_bf16x2(__uint_as_float(ov[c][2 * x]) * inv_l, __uint_as_float(ov[c][2 * x + 1]) * inv_l);
              uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
              for (int x = 0; x < 4; ++x) dst[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
            }
          }
          if (store && p.lse)
            p.lse[(int64_t)h * p.n_tokens + qpos] =
                (l_run > 0.f) ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
        }
      } else if (store) {
        uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
        for (int x = 0; x < D / 8; ++x) dst[x] = make_uint4(0, 0, 0, 0);
        if (p.lse) p.lse[(int64_t)h * p.n_tokens + qpos] = -INFINITY;
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

template <int D, int BN>
cudaError_t launch_fwd_t(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                         const FwdParams& p, int n_units, cudaStream_t stream) {
  using C = FwdCfg<D, BN>;
  cudaError_t e = ensure_smem_limit(bsa_fwd_kernel<D, BN>, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  bsa_fwd_kernel<D, BN><<<n_units, kThreadsFwd, C::kSmemBytes, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bsa_fwd(int head_dim, int block, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const FwdParams& p, int n_units, cudaStream_t stream) {
  if (n_units <= 0) return cudaSuccess;
  if (head_dim == 128 && block == 128) return launch_fwd_t<128, 128>(tmQ, tmK, tmV, p, n_units, stream);
  if (head_dim == 128 && block == 64) return launch_fwd_t<128, 64>(tmQ, tmK, tmV, p, n_units, stream);
  if (head_dim == 64 && block == 128) return launch_fwd_t<64, 128>(tmQ, tmK, tmV, p, n_units, stream);
  if (head_dim == 64 && block == 64) return launch_fwd_t<64, 64>(tmQ, tmK, tmV, p, n_units, stream);
  return cudaErrorInvalidValue;
}

}  // namespace poem
