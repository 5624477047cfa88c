// poem_select.cu -- threshold block selection and CSR emission (sm_100a, CUDA cores).
//
// Per (head h, query tile i) row, from the aggregated scores I_hat[h, i, 0..i] and
// masses m_hat[h, i, 0..i]:
//   mandatory  {0, i-1, i}       (sink, local and diagonal blocks)
//   candidates {1, .., i-2}, ranked by (I_hat desc, id asc)
//   D_k        the candidates ranked k, k+1, ..  (dropped when the top k are kept)
//   keep the top k for the smallest k with  S_m(k) < 1  and  S_I(k) <= tau (1 - S_m(k)),
//   S_I(k) = sum_{D_k} I_hat,  S_m(k) = sum_{D_k} m_hat   (fp64 suffix sums),
// which makes the triangle bound of the reading note "Attention deletion error",
// Equation (4), hold with the max-aggregated scores.  Equal scores favour the
// smaller id and lists are emitted in ascending id order, as in the appendix
// "Block ordering" of the "Block-Filtered Long-Context Attention" page.
//
// The practical selector (pooled estimates m~, d~ of the reading note's
// Equation (6) paragraph) keeps, per row, the mandatory blocks and the shortest
// prefix of a two-stage ranking whose pooled mass reaches gamma:
//   stage 1    candidates ranked by (m~ desc, id asc); the first ceil(rho |Cand|)
//   stage 2    that shortlist reranked by (log m~ + w log d~ desc, id asc), fp64
//   threshold  sum_{mandatory} m~ + sum_{prefix} m~ >= gamma (fp64), else the
//              whole shortlist.
//
// Kernels (all on the caller's stream):
//   select_rows   one CTA per row: bitonic sort of 64-bit keys (~bits(score) : id)
//                 in shared memory, fp64 suffix scan, min-reduce of the cut,
//                 ascending compaction into the row's triangular scratch slot.
//   select_practical_rows  one CTA per row: the stage-1 sort as above, a sort of
//                 (order-mapped fp64 key, id) pairs, an fp64 prefix scan of the
//                 masses and a min-reduce of the cut; same compaction.
//   scan_counts   one CTA: exclusive scan of the list lengths -> row_ptr.
//   gather_lists  one CTA per row: scratch -> col_idx (bounded by the capacity).
//   work_order    one CTA per KV head: rows of the head group by list length desc.
#include "common.cuh"

namespace poem {
namespace {

constexpr int kSelThreads = 128;

// Ascending bitonic sort of n (power of two) 64-bit keys in shared memory.
__device__ void bitonic_sort_u64(uint64_t* a, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int t = threadIdx.x; t < n; t += blockDim.x) {
        const int partner = t ^ jj;
        if (partner > t) {
          const bool up = ((t & k) == 0);
          const uint64_t x = a[t], y = a[partner];
          if ((x > y) == up) {
            a[t] = y;
            a[partner] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

__device__ void bitonic_sort_u32(uint32_t* a, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int t = threadIdx.x; t < n; t += blockDim.x) {
        const int partner = t ^ jj;
        if (partner > t) {
          const bool up = ((t & k) == 0);
          const uint32_t x = a[t], y = a[partner];
          if ((x > y) == up) {
            a[t] = y;
            a[partner] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Ascending bitonic sort of n (power of two) (key, id) pairs, lexicographic.
__device__ void bitonic_sort_pairs(uint64_t* a, uint32_t* id, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int t = threadIdx.x; t < n; t += blockDim.x) {
        const int partner = t ^ jj;
        if (partner > t) {
          const bool up = ((t & k) == 0);
          const uint64_t x = a[t], y = a[partner];
          const uint32_t ix = id[t], iy = id[partner];
          const bool gt = (x > y) || (x == y && ix > iy);
          if (gt == up) {
            a[t] = y;
            a[partner] = x;
            id[t] = iy;
            id[partner] = ix;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Unsigned keys whose ascending order is the DESCENDING order of the value
// (finite or infinite, not NaN); -0 and +0 map to the same key.
__device__ __forceinline__ uint32_t desc_key_f32(float x) {
  if (x == 0.f) x = 0.f;
  const uint32_t b = __float_as_uint(x);
  const uint32_t asc = (b >> 31) ? ~b : (b | 0x80000000u);
  return ~asc;
}

__device__ __forceinline__ uint64_t desc_key_f64(double x) {
  if (x == 0.0) x = 0.0;
  const uint64_t b = (uint64_t)__double_as_longlong(x);
  const uint64_t asc = (b >> 63) ? ~b : (b | 0x8000000000000000ull);
  return ~asc;
}

// Stage-2 rank key log m~ + w log d~ in fp64, with log 0 = -inf; a block of zero
// mass, or of zero deviation when w > 0, ranks last.
__device__ __forceinline__ double practical_rank_key(float m, float d, double w) {
  const double lm = (m > 0.f) ? log((double)m) : -INFINITY;
  const double ld = (d > 0.f) ? log((double)d) : -INFINITY;
  if (lm == -INFINITY || (w > 0.0 && ld == -INFINITY)) return -INFINITY;
  return (w == 0.0) ? lm : lm + w * ld;
}

// Block-wide exclusive prefix scan (sum over lower thread ids) of one double.
__device__ double block_excl_scan_d(double a, double* tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double x = a;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  double ex = __shfl_up_sync(0xffffffffu, x, 1);
  if (lane == 0) ex = 0.0;
  __syncthreads();
  double wsum = 0.0;
  for (int w = 0; w < warp; ++w) wsum += tmp[w];
  __syncthreads();
  return wsum + ex;
}

// Block-wide exclusive scan of one int per thread (blockDim.x == kSelThreads).
__device__ int block_excl_scan_int(int v, int* tmp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < kSelThreads / 32) ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kSelThreads / 32) tmp[lane] = w;
  }
  __syncthreads();
  const int base = (warp > 0) ? tmp[warp - 1] : 0;
  *total = tmp[kSelThreads / 32 - 1];
  __syncthreads();
  return base + x - v;
}

// Block-wide exclusive *suffix* scan (sum over higher thread ids) of a double pair.
__device__ void block_suffix_scan_d2(double a, double b, double* tmpa, double* tmpb, double& ea, double& eb) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double xa = a, xb = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double ya = __shfl_down_sync(0xffffffffu, xa, o);
    const double yb = __shfl_down_sync(0xffffffffu, xb, o);
    if (lane + o < 32) {
      xa += ya;
      xb += yb;
    }
  }
  // xa: inclusive suffix within the warp; the exclusive one is the next lane's.
  double na = __shfl_down_sync(0xffffffffu, xa, 1);
  double nb = __shfl_down_sync(0xffffffffu, xb, 1);
  if (lane == 31) {
    na = 0.0;
    nb = 0.0;
  }
  if (lane == 0) {
    tmpa[warp] = xa;
    tmpb[warp] = xb;
  }
  __syncthreads();
  double wa = 0.0, wb = 0.0;
  for (int w = kSelThreads / 32 - 1; w > warp; --w) {
    wa += tmpa[w];
    wb += tmpb[w];
  }
  ea = na + wa;
  eb = nb + wb;
  __syncthreads();
}

// Ascending compaction of the kept flags of block ids 0..i (i: the row's global
// tile) into the row's scratch slot at offset off; the length goes to counts[row].
__device__ void emit_row(const SelectParams& p, const int* keep, int row, int i, int64_t off, int* tmpi) {
  const int n = i + 1;
  const int E2 = (n + kSelThreads - 1) / kSelThreads;
  const int b0 = threadIdx.x * E2;
  const int b1 = min(n, b0 + E2);
  int cnt = 0;
  for (int b = b0; b < b1; ++b) cnt += keep[b];
  int total;
  int pos = block_excl_scan_int(cnt, tmpi, &total);
  int32_t* dst = p.scratch + off;
  for (int b = b0; b < b1; ++b)
    if (keep[b]) {
      if (POEM_IN_BOUNDS(p.err, off + pos, p.n_entries)) dst[pos] = b;
      ++pos;
    }
  if (threadIdx.x == 0 && POEM_IN_BOUNDS(p.err, row, (int64_t)p.n_q_heads * p.n_tiles)) p.counts[row] = total;
}

__global__ void __launch_bounds__(kSelThreads) select_rows_kernel(const SelectParams p) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int row = blockIdx.x;
  const int T = p.n_tiles;
  const int h = row / T;
  const int il = row - h * T;       // local query tile
  const int i = il + p.q_tile0;     // global tile: blocks 0..i visible
  const int nc = max(0, i - 2);
  int P = 1;
  while (P < nc) P <<= 1;
  uint64_t* keys = reinterpret_cast<uint64_t*>(sm);                      // [P]
  int* keep = reinterpret_cast<int*>(sm + sizeof(uint64_t) * (size_t)max(P, 1));  // [i + 1]
  __shared__ double tmpa[kSelThreads / 32], tmpb[kSelThreads / 32];
  __shared__ int tmpi[kSelThreads / 32];
  __shared__ int s_kcut;

  const int64_t off = row_off(T, p.q_tile0, h, il);
  const float* Ih = p.I_hat + off;
  const float* mh = p.m_hat + off;
  const float* rank_src = p.mass_only ? mh : Ih;

  for (int t = threadIdx.x; t < P; t += blockDim.x) {
    uint64_t key = ~0ull;
    if (t < nc) {
      const int id = t + 1;
      const float sc = fmaxf(rank_src[id], 0.f);  // canonical +0 for zero scores
      key = ((uint64_t)(~__float_as_uint(sc)) << 32) | (uint32_t)id;
    }
    keys[t] = key;
  }
  for (int b = threadIdx.x; b <= i; b += blockDim.x) keep[b] = 0;
  if (threadIdx.x == 0) s_kcut = nc;
  __syncthreads();
  if (nc > 1) bitonic_sort_u64(keys, P);

  int kcut = nc;
  if (p.mass_only) {
    const int ref = p.ref_row_ptr[row + 1] - p.ref_row_ptr[row];
    const int n_mand = (i == 0) ? 1 : (i == 1 ? 2 : 3);
    kcut = min(max(ref - n_mand, 0), nc);
  } else if (nc > 0) {
    // Threshold of this row: the call's tau, or its head's entry of tau_heads (a
    // NaN, negative or infinite entry keeps every candidate and is reported).
    double tau = p.tau;
    bool keep_all = false;  // uniform over the CTA
    if (p.tau_heads) {
      const float th = p.tau_heads[h];
      if (!(th >= 0.f) || isinf(th)) {
        if (threadIdx.x == 0) raise_err(p.err, kErrBadParam);
        keep_all = true;
      } else {
        tau = (double)th;
      }
    }
    // Each thread owns a contiguous run of ranks; suffix sums inside the run, then
    // a block suffix scan of the run totals.
    const int E = (nc + kSelThreads - 1) / kSelThreads;
    const int r0 = threadIdx.x * E;
    const int r1 = min(nc, r0 + E);
    double ta = 0.0, tb = 0.0;
    for (int r = r1 - 1; r >= r0; --r) {
      const int id = (int)(keys[r] & 0xffffffffu);
      ta += (double)Ih[id];
      tb += (double)mh[id];
    }
    double ca, cb;
    block_suffix_scan_d2(ta, tb, tmpa, tmpb, ca, cb);
    // Walk the run from its end toward its start, accumulating onto the carry.
    int best = nc;
    double sa = ca, sb2 = cb;
    for (int r = r1 - 1; r >= r0; --r) {
      const int id = (int)(keys[r] & 0xffffffffu);
      sa += (double)Ih[id];
      sb2 += (double)mh[id];
      if (sb2 < 1.0 && sa <= tau * (1.0 - sb2)) best = r;
    }
    if (best < nc && !keep_all) atomicMin(&s_kcut, best);
    __syncthreads();
    kcut = s_kcut;
  }
  // Mark kept blocks: mandatory + top kcut candidates.
  for (int r = threadIdx.x; r < kcut; r += blockDim.x) keep[(int)(keys[r] & 0xffffffffu)] = 1;
  if (threadIdx.x == 0) {
    keep[0] = 1;
    keep[i] = 1;
    if (i >= 1) keep[i - 1] = 1;
  }
  __syncthreads();
  emit_row(p, keep, row, i, off, tmpi);
}

__global__ void __launch_bounds__(kSelThreads) select_practical_rows_kernel(const SelectParams p) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int row = blockIdx.x;
  const int T = p.n_tiles;
  const int h = row / T;
  const int il = row - h * T;       // local query tile
  const int i = il + p.q_tile0;     // global tile: blocks 0..i visible
  const int nc = max(0, i - 2);
  int P = 1;
  while (P < nc) P <<= 1;
  uint64_t* keys = reinterpret_cast<uint64_t*>(sm);                    // [P]
  uint32_t* ids = reinterpret_cast<uint32_t*>(sm + sizeof(uint64_t) * (size_t)P);  // [P]
  int* keep = reinterpret_cast<int*>(sm + (sizeof(uint64_t) + sizeof(uint32_t)) * (size_t)P);  // [i + 1]
  __shared__ double tmpd[kSelThreads / 32];
  __shared__ int tmpi[kSelThreads / 32];
  __shared__ int s_kcut;

  const int64_t off = row_off(T, p.q_tile0, h, il);
  const float* mp = p.m_hat + off;
  const float* dp = p.d_pool + off;

  // Stage 1: candidates by (m~ desc, id asc).
  for (int t = threadIdx.x; t < P; t += blockDim.x)
    keys[t] = (t < nc) ? (((uint64_t)desc_key_f32(mp[t + 1]) << 32) | (uint32_t)(t + 1)) : ~0ull;
  for (int b = threadIdx.x; b <= i; b += blockDim.x) keep[b] = 0;
  if (nc > 1) {
    __syncthreads();
    bitonic_sort_u64(keys, P);
  }
  const int n1 = min(nc, max(0, (int)ceil(p.rho * (double)nc)));
  if (threadIdx.x == 0) s_kcut = n1;
  int P2 = 1;
  while (P2 < n1) P2 <<= 1;
  __syncthreads();
  // Stage 2: the shortlist by (log m~ + w log d~ desc, id asc); each thread
  // rewrites only the entries it reads.
  for (int t = threadIdx.x; t < P2; t += blockDim.x) {
    if (t < n1) {
      const uint32_t id = (uint32_t)(keys[t] & 0xffffffffu);
      ids[t] = id;
      keys[t] = desc_key_f64(practical_rank_key(mp[id], dp[id], p.w));
    } else {
      ids[t] = 0xffffffffu;
      keys[t] = ~0ull;
    }
  }
  __syncthreads();
  if (n1 > 1) bitonic_sort_pairs(keys, ids, P2);

  // Threshold of this row: the call's gamma, or its head's entry of gamma_heads
  // (a NaN or infinite entry keeps the whole shortlist and is reported).
  double gamma = p.gamma;
  if (p.gamma_heads) {
    const float gh = p.gamma_heads[h];
    if (isnan(gh) || isinf(gh)) {
      if (threadIdx.x == 0) raise_err(p.err, kErrBadParam);
      gamma = INFINITY;  // never reached: the whole shortlist is kept
    } else {
      gamma = (double)gh;
    }
  }
  // Threshold: mandatory mass (ascending ids), then the reranked prefix, in fp64.
  double acc0 = (double)mp[0];
  if (i >= 2) acc0 += (double)mp[i - 1];
  if (i >= 1) acc0 += (double)mp[i];
  const int E = (n1 + kSelThreads - 1) / kSelThreads;
  const int r0 = min(n1, threadIdx.x * E);
  const int r1 = min(n1, r0 + E);
  double loc = 0.0;
  for (int r = r0; r < r1; ++r) loc += (double)mp[ids[r]];
  const double carry = block_excl_scan_d(loc, tmpd);
  double run = acc0 + carry;
  for (int r = r0; r < r1; ++r) {
    run += (double)mp[ids[r]];
    if (run >= gamma) {
      atomicMin(&s_kcut, r + 1);
      break;
    }
  }
  if (threadIdx.x == 0 && acc0 >= gamma) atomicMin(&s_kcut, 0);
  __syncthreads();
  const int kcut = s_kcut;
  for (int r = threadIdx.x; r < kcut; r += blockDim.x) keep[ids[r]] = 1;
  if (threadIdx.x == 0) {
    keep[0] = 1;
    keep[i] = 1;
    if (i >= 1) keep[i - 1] = 1;
  }
  __syncthreads();
  emit_row(p, keep, row, i, off, tmpi);
}

// Exclusive scan of counts[0..rows) into row_ptr[0..rows] (single CTA).
__global__ void __launch_bounds__(1024) scan_counts_kernel(const int32_t* counts, int32_t* row_ptr, int rows) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = 0; base < rows; base += 1024) {
    const int idx = base + threadIdx.x;
    const int v = (idx < rows) ? counts[idx] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;
    }
    __syncthreads();
    const int excl = carry + ((warp > 0) ? warp_tot[warp - 1] : 0) + x - v;
    if (idx < rows) row_ptr[idx] = excl;
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_tot[31];
    __syncthreads();
  }
  if (threadIdx.x == 0) row_ptr[rows] = carry;
}

__global__ void __launch_bounds__(128) gather_lists_kernel(const SelectParams p) {
  const int row = blockIdx.x;
  const int T = p.n_tiles;
  const int h = row / T;
  const int i = row - h * T;
  const int64_t start = p.row_ptr[row];
  const int n = p.counts[row];
  const int64_t off = row_off(T, p.q_tile0, h, i);
  const int32_t* src = p.scratch + off;
  const int64_t cap = p.col_capacity;
  for (int x = threadIdx.x; x < n; x += blockDim.x) {
    const int64_t d = start + x;
    if (d < cap && POEM_IN_BOUNDS(p.err, off + x, p.n_entries)) p.col_idx[d] = src[x];
  }
  if (threadIdx.x == 0 && start + n > cap) raise_err(p.err, kErrCapacity);
}

// Rows of one KV head's query-head group, by list length descending, ties by row id.
__global__ void __launch_bounds__(1024) work_order_kernel(const SelectParams p, int seg_pow2) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm);
  const int seg = p.group * p.n_tiles;
  const int base = blockIdx.x * seg;
  for (int t = threadIdx.x; t < seg_pow2; t += blockDim.x) {
    uint32_t key = 0xffffffffu;
    if (t < seg) {
      const int len = min(p.row_ptr[base + t + 1] - p.row_ptr[base + t], 4095);
      key = ((uint32_t)(4095 - len) << 20) | (uint32_t)t;
    }
    keys[t] = key;
  }
  __syncthreads();
  bitonic_sort_u32(keys, seg_pow2);
  for (int t = threadIdx.x; t < seg; t += blockDim.x) p.order[base + t] = base + (int)(keys[t] & 0xfffffu);
}

}  // namespace

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) {
  const int rows = p.n_q_heads * p.n_tiles;
  if (rows <= 0) return cudaSuccess;
  const int n_blocks = p.n_tiles + p.q_tile0;  // key blocks of the longest row
  int P = 1;
  while (P < n_blocks) P <<= 1;
  if (p.practical) {
    const size_t smem = (sizeof(uint64_t) + sizeof(uint32_t)) * (size_t)P + sizeof(int) * (size_t)n_blocks + 16;
    cudaError_t e = ensure_smem_limit(select_practical_rows_kernel, smem);
    if (e != cudaSuccess) return e;
    select_practical_rows_kernel<<<rows, kSelThreads, smem, stream>>>(p);
  } else {
    const size_t smem = sizeof(uint64_t) * (size_t)P + sizeof(int) * (size_t)n_blocks + 16;
    cudaError_t e = ensure_smem_limit(select_rows_kernel, smem);
    if (e != cudaSuccess) return e;
    select_rows_kernel<<<rows, kSelThreads, smem, stream>>>(p);
  }
  scan_counts_kernel<<<1, 1024, 0, stream>>>(p.counts, p.row_ptr, rows);
  gather_lists_kernel<<<rows, 128, 0, stream>>>(p);
  if (p.order) {
    const int seg = p.group * p.n_tiles;
    int sp = 1;
    while (sp < seg) sp <<= 1;
    const size_t osmem = sizeof(uint32_t) * (size_t)sp;
    cudaError_t e = ensure_smem_limit(work_order_kernel, osmem);
    if (e != cudaSuccess) return e;
    work_order_kernel<<<p.n_q_heads / p.group, 1024, osmem, stream>>>(p, sp);
  }
  return cudaGetLastError();
}

}  // namespace poem
