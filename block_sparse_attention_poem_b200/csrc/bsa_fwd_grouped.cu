// bsa_fwd_grouped.cu -- causal GQA block-sparse attention forward with K/V tiles
// shared by two query heads of one KV group (sm_100a).
//
// Computes exactly what bsa_fwd computes -- for every (head h, query tile i) row the
// renormalised sparse output of the reading note "Attention deletion error",
// Section 4.1, over the blocks listed for that row -- but one CTA takes the rows of
// two query heads h, h + 1 of one KV group at the same tile i and walks the UNION of
// their two lists: each block's K and V tiles are loaded into shared memory once and
// serve both heads, while each head computes S, its softmax and P V only on the
// blocks of its own list.  One CTA per SM (512 TMEM columns).
//
// Work order: KV head major, last tile first, pairs of adjacent query heads (with an
// odd group size the last pair has one head).  With a query offset (chunked prefill)
// local query tile i is global tile q_tile0 + i, as in bsa_fwd.
//
// Roles (320 threads):
//   warps 0-3 / 4-7  softmax of head A / head B: one query row per thread, as in
//              bsa_fwd (running max, P over the S columns, O rescaled only when the
//              max grows by more than 2^8, epilogue).
//   warp 8     TMA producer: Q_A and Q_B once, then K_b, V_b for every block b of the
//              union, in ascending order, into a ring of shared-memory slots.
//   warp 9     MMA issuer (converged warp; one elected lane issues).  At each union block b, for head x = A, B:
//              first O_x += P_x V_x for x's previous block (if one is pending), then,
//              if b is in x's list, S_x = Q_x K_b^T.  A head's P V therefore waits at
//              most one union step, so each V tile is released one step after its
//              block and the ring never needs more than two blocks' tiles; a K tile is
//              released after its last S, a V tile after its last P V.
// TMEM: head x has S/P at [256x, 256x + BN) and O at [256x + 128, 256x + 128 + D).
#include <climits>

#include "common.cuh"
#include "fwd_common.cuh"

namespace poem {
namespace {

constexpr int kMaxSlots = 8;
constexpr int kThreadsGrouped = 320;
constexpr int kSmemCap = 232448;  // opt-in maximum of dynamic shared memory per CTA

template <int D, int BN>
struct GrpCfg {
  static constexpr int M = 128;
  static constexpr int kChunks = D / 64;              // 128-byte column chunks per row
  static constexpr int kQBytes = M * D * 2;
  static constexpr int kKVBytes = BN * D * 2;
  static constexpr int kOffQ = 0;                     // Q_A, then Q_B
  static constexpr int kOffRing = 2 * kQBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kSlotsFit = (kSmemCap - 1024 - kOffRing - kBarBytes) / kKVBytes;
  static constexpr int kSlots = kSlotsFit < kMaxSlots ? kSlotsFit : kMaxSlots;
  static constexpr int kOffBar = kOffRing + kSlots * kKVBytes;
  // above half the SM's shared memory so that one CTA (512 TMEM columns) is resident
  // per SM and tcgen05.alloc never has to wait
  static constexpr int kSmemBytes = (kOffBar + kBarBytes + 1024) > 120 * 1024 ? (kOffBar + kBarBytes + 1024)
                                                                              : 120 * 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(M, BN, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(M, D, 1);
  static_assert(kSlots >= 4, "the K/V ring needs four slots (two blocks)");
  static_assert(kSmemBytes <= kSmemCap, "shared memory");
};

struct FwdBarriers {
  uint64_t slot_full[kMaxSlots], slot_empty[kMaxSlots];
  uint64_t q_full[2], s_full[2], p_half[2][2], o_full[2], drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

using fwd::block_ok;
using fwd::exp_pack_store;
using fwd::kDrainNs;
using fwd::wait_or_abort;
using fwd::warp_wait_or_abort;

// The two rows of a CTA: query heads 2p and 2p + 1 of KV group g at local tile i.
struct PairRow {
  int h, tile, gtile, beg, end;
  bool live;
};

__host__ __device__ __forceinline__ int grouped_units(int n_kv_heads, int n_tiles, int group) {
  return n_kv_heads * n_tiles * ((group + 1) / 2);
}

__device__ __forceinline__ PairRow pair_row(const FwdParams& p, int unit, int x, int* hk, bool report) {
  PairRow R{0, 0, 0, 0, 0, false};
  const int pairs = (p.group + 1) / 2;
  const int per_g = p.n_tiles * pairs;
  const int g = unit / per_g;
  const int rem = unit - g * per_g;
  const int i = p.n_tiles - 1 - rem / pairs;
  const int j = 2 * (rem % pairs) + x;  // head within the group
  *hk = g;
  if (j >= p.group) return R;           // odd group size: the last pair has one head
  R.h = g * p.group + j;
  R.tile = i;
  R.gtile = i + p.q_tile0;
  const int row = R.h * p.n_tiles + i;
  R.beg = p.row_ptr[row];
  R.end = p.row_ptr[row + 1];
  if (R.end < R.beg) {
    if (report) raise_err(p.err, kErrBadList);
    R.end = R.beg;
  }
  R.live = true;
  return R;
}

// First entry at or after e whose id is visible to the row (ids outside 0..gtile
// are skipped; the producer reports them).
__device__ __forceinline__ int next_valid(const FwdParams& p, const PairRow& R, int e, bool report) {
  for (; e < R.end; ++e) {
    if (block_ok(p.col_idx[e], R.gtile)) return e;
    if (report) raise_err(p.err, kErrBadList);
  }
  return R.end;
}

__device__ __forceinline__ int id_at(const FwdParams& p, const PairRow& R, int e) {
  return e < R.end ? p.col_idx[e] : INT_MAX;
}

template <int D, int BN>
__global__ void __launch_bounds__(kThreadsGrouped, 1)
    bsa_fwd_grouped_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = GrpCfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sRing = smem + C::kOffRing;
  FwdBarriers* sb = reinterpret_cast<FwdBarriers*>(smem + C::kOffBar);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int unit = blockIdx.x;

  if (tid == 0) {
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&sb->slot_full[s], 1);
      mbar_init(&sb->slot_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sb->q_full[x], 1);
      mbar_init(&sb->s_full[x], 1);
      mbar_init(&sb->p_half[x][0], 4);  // one arrival per softmax warp
      mbar_init(&sb->p_half[x][1], 4);
      mbar_init(&sb->o_full[x], 1);
    }
    mbar_init(&sb->drain, 1);
    sb->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) tmem_alloc<C::kTmemCols>(&sb->tmem_base);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sb->tmem_base;

  if (warp == 8) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int hk = 0;
      const PairRow R[2] = {pair_row(p, unit, 0, &hk, true), pair_row(p, unit, 1, &hk, true)};
      int e[2], q_issued[2] = {0, 0};
      for (int x = 0; x < 2; ++x) {
        e[x] = R[x].live ? next_valid(p, R[x], R[x].beg, true) : R[x].end;
        if (e[x] < R[x].end) {
          mbar_arrive_expect_tx(&sb->q_full[x], C::kQBytes);
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(smem + C::kOffQ + x * C::kQBytes + c * (C::M * 128), &tmQ, &sb->q_full[x], c * 64,
                        R[x].h, R[x].tile * BN);
          q_issued[x] = 1;
        }
      }
      int n = 0;  // tiles loaded so far; tile n goes to slot n % kSlots
      bool ok = true;
      auto load = [&](const CUtensorMap* map, int id) -> bool {
        const int s = n % C::kSlots;
        if (!wait_or_abort(&sb->slot_empty[s], ((n / C::kSlots) & 1) ^ 1, sb, p.err)) return false;
        mbar_arrive_expect_tx(&sb->slot_full[s], C::kKVBytes);
        uint8_t* dst = sRing + s * C::kKVBytes;
        for (int c = 0; c < C::kChunks; ++c) tma_load_3d(dst + c * (BN * 128), map, &sb->slot_full[s], c * 64, hk, id * BN);
        ++n;
        return true;
      };
      // the union of the two lists, ascending: K_b then V_b for each block
      while (ok && (e[0] < R[0].end || e[1] < R[1].end) && !sb->abort_flag) {
        const int b0 = id_at(p, R[0], e[0]), b1 = id_at(p, R[1], e[1]);
        const int b = b0 < b1 ? b0 : b1;
        ok = load(&tmK, b) && load(&tmV, b);
        if (b0 == b) e[0] = next_valid(p, R[0], e[0] + 1, true);
        if (b1 == b) e[1] = next_valid(p, R[1], e[1] + 1, true);
      }
      // Drain: every issued load must have landed before the CTA may exit (the last
      // load of each slot completes the phase waited for here).
      for (int x = 0; x < 2; ++x)
        if (q_issued[x]) mbar_wait(&sb->q_full[x], 0, kDrainNs);
      for (int s = 0; s < C::kSlots && s < n; ++s) mbar_wait(&sb->slot_full[s], ((n - 1 - s) / C::kSlots) & 1, kDrainNs);
    }
  } else if (warp == 9) {
    // ============================ MMA issuer ============================
    // The whole warp runs the schedule converged (list entries, waits and operands are
    // warp-uniform); one elected lane issues each MMA and commit.
    {
      int hk = 0;
      const PairRow R[2] = {pair_row(p, unit, 0, &hk, false), pair_row(p, unit, 1, &hk, false)};
      const uint32_t aRing = smem_u32(sRing);
      int e[2] = {0, 0};
      int k[2] = {0, 0};            // P V products issued per head
      int nq[2] = {0, 0};           // S products issued per head
      bool pend[2] = {false, false};  // a P V waiting for the next union step
      int pend_v[2] = {0, 0};       // its V tile (load index)
      bool pend_rel[2] = {false, false};  // whether that P V is the V tile's last use
      bool ok = true;
      auto wait_tile = [&](int n) -> bool {
        return warp_wait_or_abort(&sb->slot_full[n % C::kSlots], (n / C::kSlots) & 1, sb, p.err);
      };
      // O_x += P_x V (in two 64-key halves, each as soon as that half of P_x is written)
      auto issue_pv = [&](int x) -> bool {
        const int n = pend_v[x];
        if (!wait_tile(n)) return false;
        const uint32_t aV = aRing + (n % C::kSlots) * C::kKVBytes;
        const uint32_t tS = tmem + 256u * x;
        const uint32_t tO = tS + 128u;
#pragma unroll
        for (int hv = 0; hv < BN / 64; ++hv) {
          if (!warp_wait_or_abort(&sb->p_half[x][hv], k[x] & 1, sb, p.err)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = hv * 4; kk < hv * 4 + 4; ++kk) {
            // V tile is MN-major (d contiguous): LBO = stride between 64-wide d chunks,
            // SBO = stride between 8-key groups; a k-step covers 16 keys = 2 groups.
            const uint64_t bdesc = smem_desc_sw128(aV + kk * 2048, BN * 128, 1024);
            mma_ts_warp(tO, tS + kk * 8, bdesc, C::kIdescPV, (k[x] > 0 || kk > 0) ? 1u : 0u);
          }
        }
        if (pend_rel[x]) mma_commit_warp(&sb->slot_empty[n % C::kSlots]);
        ++k[x];
        pend[x] = false;
        if (e[x] >= R[x].end) mma_commit_warp(&sb->o_full[x]);  // that was the head's last block
        return true;
      };
      // S_x = Q_x K^T with the K tile of load index n
      auto issue_qk = [&](int x, int n, bool release) -> bool {
        if (nq[x] == 0 && !warp_wait_or_abort(&sb->q_full[x], 0, sb, p.err)) return false;
        if (!wait_tile(n)) return false;
        tc_fence_after();
        const uint32_t aQ = smem_u32(smem + C::kOffQ + x * C::kQBytes);
        const uint32_t aK = aRing + (n % C::kSlots) * C::kKVBytes;
        const uint32_t tS = tmem + 256u * x;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // Q and K tiles are K-major, 128-byte swizzled; a k-step is 16 elements (32 B)
          // inside a 64-element chunk; chunks are whole row-blocks apart.
          const uint32_t koff = (kk & 3) * 32;
          const uint64_t adesc = smem_desc_sw128(aQ + (kk >> 2) * (C::M * 128) + koff, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(aK + (kk >> 2) * (BN * 128) + koff, 16, 1024);
          mma_ss_warp(tS, adesc, bdesc, C::kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit_warp(&sb->s_full[x]);
        if (release) mma_commit_warp(&sb->slot_empty[n % C::kSlots]);
        ++nq[x];
        return true;
      };
      for (int x = 0; x < 2; ++x) e[x] = R[x].live ? next_valid(p, R[x], R[x].beg, false) : R[x].end;
      int n = 0;  // load index of the current union block's K tile (its V tile is n + 1)
      while (ok && (e[0] < R[0].end || e[1] < R[1].end)) {
        const int b0 = id_at(p, R[0], e[0]), b1 = id_at(p, R[1], e[1]);
        const int b = b0 < b1 ? b0 : b1;
        const bool in[2] = {b0 == b, b1 == b};
        for (int x = 0; x < 2 && ok; ++x) {
          if (pend[x]) ok = issue_pv(x);  // the previous block of head x
          if (ok && in[x]) {
            // K_b's last use is head B's S when b is in B's list, else head A's
            ok = issue_qk(x, n, x == 1 || !in[1]);
            e[x] = next_valid(p, R[x], e[x] + 1, false);
            pend[x] = true;
            pend_v[x] = n + 1;
            pend_rel[x] = (x == 1 || !in[1]);  // V_b's last use: B's P V, else A's
          }
        }
        n += 2;
      }
      for (int x = 0; x < 2 && ok; ++x)
        if (pend[x]) ok = issue_pv(x);
      // Drain every MMA this warp issued before TMEM is released.
      mma_commit_warp(&sb->drain);
      mbar_wait(&sb->drain, 0, kDrainNs);
    }
  } else {
    // ============================ softmax warps ============================
    const int rx = warp >> 2;                // 0: head A, 1: head B
    int hk_unused = 0;
    const PairRow R = pair_row(p, unit, rx, &hk_unused, false);
    const int r = tid & 127;                 // query row within the tile (TMEM lane)
    const int qpos = R.tile * BN + r;        // query token index of this row (row of O / lse)
    const int kpos = R.gtile * BN + r;       // its position among the keys
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t tS = lane_base + 256u * rx;
    const uint32_t tO = tS + 128u;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;                 // running max, log2 units of scaled logits
    float l_run = 0.f;                       // running sum of the weights
    int it = 0;
    bool ok = true;
    int id = (R.beg < R.end) ? p.col_idx[R.beg] : -1;
    for (int e = R.beg; e < R.end; ++e) {
      const int id_next = (e + 1 < R.end) ? p.col_idx[e + 1] : -1;  // prefetched a block ahead
      if (block_ok(id, R.gtile)) {
        // tcgen05.ld is warp-collective: every lane of the warp takes the same branch.
        if (!__all_sync(0xffffffffu, wait_or_abort(&sb->s_full[rx], it & 1, sb, p.err))) { ok = false; break; }
        tc_fence_after();
        const bool diag = (id == R.gtile);
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
          exp_pack_store<BN, true>(tS, sl2, m_use, lim, &l_run, sb->p_half[rx]);
        else
          exp_pack_store<BN, false>(tS, sl2, m_use, lim, &l_run, sb->p_half[rx]);
        ++it;
      }
      id = id_next;
    }
    // ---- epilogue ----
    if (R.live && __all_sync(0xffffffffu, ok && !sb->abort_flag)) {
      const bool store = (r < BN);
      __nv_bfloat16* orow = p.o + (int64_t)qpos * p.o_stride_tok + (int64_t)R.h * p.o_stride_head;
      if (it > 0) {
        if (__all_sync(0xffffffffu, wait_or_abort(&sb->o_full[rx], 0, sb, p.err))) {
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
            p.lse[(int64_t)R.h * p.n_tokens + qpos] =
                (l_run > 0.f) ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
        }
      } else if (store) {
        uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
        for (int x = 0; x < D / 8; ++x) dst[x] = make_uint4(0, 0, 0, 0);
        if (p.lse) p.lse[(int64_t)R.h * p.n_tokens + qpos] = -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) {
    __syncwarp();
    tmem_dealloc<C::kTmemCols>(tmem);
  }
}

template <int D, int BN>
cudaError_t launch_grouped_t(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                             const FwdParams& p, int n_kv_heads, cudaStream_t stream) {
  using C = GrpCfg<D, BN>;
  cudaError_t e = ensure_smem_limit(bsa_fwd_grouped_kernel<D, BN>, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int units = grouped_units(n_kv_heads, p.n_tiles, p.group);
  bsa_fwd_grouped_kernel<D, BN><<<units, kThreadsGrouped, C::kSmemBytes, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bsa_fwd_grouped(int head_dim, int block, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                   const CUtensorMap& tmV, const FwdParams& p, int n_kv_heads, cudaStream_t stream) {
  if (n_kv_heads <= 0 || p.n_tiles <= 0) return cudaSuccess;
  if (head_dim == 128 && block == 128) return launch_grouped_t<128, 128>(tmQ, tmK, tmV, p, n_kv_heads, stream);
  if (head_dim == 128 && block == 64) return launch_grouped_t<128, 64>(tmQ, tmK, tmV, p, n_kv_heads, stream);
  if (head_dim == 64 && block == 128) return launch_grouped_t<64, 128>(tmQ, tmK, tmV, p, n_kv_heads, stream);
  if (head_dim == 64 && block == 64) return launch_grouped_t<64, 64>(tmQ, tmK, tmV, p, n_kv_heads, stream);
  return cudaErrorInvalidValue;
}

}  // namespace poem
