// Decode-time selection in one launch: the column scores q_j = sum_i x[i, j]^2
// of a short activation matrix x (n <= 32 rows), the TopK index set I of the
// k = ceil(rho d) largest (lower index on ties, ascending), and the packed
// activations x[:, I] ("Algorithm Deep-Dive: RMM", Core Approach: s_j =
// ||A[:, j]||_2, keep the TopK-largest; the reduced product then reads x[:, I]).
//
// At decode sizes each of the three steps is a latency-bound launch of a few
// microseconds, and one CTA selecting over d = 8192 keys is issue-bound, so the
// work is spread over one cluster of C CTAs of 256 threads (C <= 8):
//   * each thread owns KPT consecutive columns (4 while 8 CTAs of 1024 columns
//     cover d, i.e. d <= 8192; else 8, d <= 16384); CTA r owns columns
//     [256 KPT r, 256 KPT (r + 1)).  The thread copies its chunk of every row
//     into shared memory with cp.async (all rows in flight at once, where
//     batches of eight register loads cost one round trip each), computes the
//     fp64 scores from there with the arithmetic of the short-matrix
//     column-score kernel (bit-identical keys), and packs x[:, I] from the same
//     copy at the end;
//   * the k-th largest key is found by an MSB-first radix select over the
//     64-bit key patterns (non-negative doubles order like their bits): leading
//     bits shared by every key are skipped (cluster-wide AND / OR), each pass
//     resolves 8 bits with per-warp histograms merged per CTA and then across
//     the cluster through distributed shared memory (each thread reads its bin
//     from every CTA with independent loads), one cluster barrier per pass; the same barrier carries each pass's AND / OR of the bucket's
//     members, so bits the bucket shares are skipped and a bucket of identical
//     keys (squares of a single bf16 row) ends the passes at once;
//   * the compaction takes every key above the threshold and the lowest-index
//     keys equal to it, in index order: counts are exchanged once across the
//     cluster (CTA order is column order; warp 0 reads the lower CTAs' counts
//     in parallel and scans them), then two block scans give each
//     thread its positions; the thread writes I and, for its kept columns,
//     x[:, I] (zero-padded to the packed row length).
// Every count is an integer, so the result does not depend on atomic order.
#pragma once
#include "ptx.cuh"
#include "colsq.cuh"
#include "select.cuh"

namespace rmm {

struct DecodeSelParams {
  const uint16_t* x;  // bf16 [n][ldx]
  int64_t ldx;
  int n;              // 1..32
  int d;              // 1..kDecSelMaxD
  int k;              // 1..d
  int32_t* idx;       // [k]
  uint16_t* xpack;    // [n][ld_pack] or nullptr: x[:, I], columns [k, ld_pack) zeroed
  int64_t ld_pack;
};

constexpr int kDecSelThreads = 256;
constexpr int kDecSelMaxCtas = 8;                // portable cluster size
// KPT columns per thread: 4 for d <= 8192 (clusters of up to 8 CTAs of 1024
// columns: half the per-thread work of 8), 8 up to d = 16384
constexpr int kDecSelMaxD = kDecSelThreads * 8 * kDecSelMaxCtas;
__host__ __device__ constexpr int decsel_cols_per_cta(int kpt) { return kDecSelThreads * kpt; }
constexpr int kDecSelMaxRows = 32;
// shared memory for the staged rows: n rows x 256 threads x KPT bf16
__host__ __device__ constexpr int decsel_stage_bytes(int n, int kpt) { return n * kDecSelThreads * kpt * 2; }

// The two halves of a cluster barrier, for work that can overlap its latency.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

__device__ __forceinline__ uint64_t ld_shared_cluster_u64(uint32_t addr) {
  uint64_t v;
  asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_shared_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// AND and OR of v over the whole cluster.  Each CTA stages its block result in
// `slot` (two words), the cluster barrier publishes them, lanes q < C of warp 0
// read CTA q's pair, and the combined result is broadcast through `res`.  No
// CTA rewrites `slot` before every CTA has passed the next cluster barrier.
__device__ __forceinline__ void decsel_cluster_andor(uint64_t& a, uint64_t& o, uint64_t* s_warp_and,
                                                     uint64_t* s_warp_or, uint64_t* slot, uint64_t* res, int C) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    a &= __shfl_xor_sync(0xffffffffu, a, off);
    o |= __shfl_xor_sync(0xffffffffu, o, off);
  }
  if (lane == 0) {
    s_warp_and[warp] = a;
    s_warp_or[warp] = o;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t ba = ~0ull, bo = 0ull;
    for (int w = 0; w < kDecSelThreads / 32; ++w) {
      ba &= s_warp_and[w];
      bo |= s_warp_or[w];
    }
    slot[0] = ba;
    slot[1] = bo;
  }
  cluster_sync();
  if (warp == 0) {
    uint64_t ra = ~0ull, ro = 0ull;
    if (lane < C) {
      const uint32_t base = smem_u32(slot);
      ra = ld_shared_cluster_u64(map_shared_rank(base, static_cast<uint32_t>(lane)));
      ro = ld_shared_cluster_u64(map_shared_rank(base + 8, static_cast<uint32_t>(lane)));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      ra &= __shfl_xor_sync(0xffffffffu, ra, off);
      ro |= __shfl_xor_sync(0xffffffffu, ro, off);
    }
    if (lane == 0) {
      res[0] = ra;
      res[1] = ro;
    }
  }
  __syncthreads();
  a = res[0];
  o = res[1];
}

template <int KPT>
__global__ void __launch_bounds__(kDecSelThreads) decode_select_kernel(const DecodeSelParams p) {
  __shared__ uint32_t whist[kDecSelThreads / 32][256];
  __shared__ uint32_t hist[2][256];
  __shared__ uint64_t s_wand[kDecSelThreads / 32], s_wor[kDecSelThreads / 32];
  __shared__ uint64_t s_andor[2], s_andor_res[2];
  __shared__ uint64_t s_pass_andor[2][2];  // the bucket's AND / OR per pass (read by the cluster), double-buffered
  __shared__ int s_warp[32];
  __shared__ int s_total;
  __shared__ int s_digit, s_above, s_cnt;
  __shared__ int s_counts[2];  // this CTA's keys above the threshold / equal to it (read by the cluster)
  __shared__ int s_sel_base, s_eq_before;
  extern __shared__ __align__(16) uint8_t s_rows[];  // [n][kDecSelThreads][KPT] bf16

  wait_prior_kernels();
  const int C = static_cast<int>(gridDim.x);  // the grid is one cluster
  const int rank = static_cast<int>(cluster_ctarank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t col0 = static_cast<int64_t>(rank) * decsel_cols_per_cta(KPT) + tid * KPT;

  // ---- this thread's chunk of every row, staged in shared memory
  constexpr int WPR = KPT / 2;  // 32-bit words per row chunk
  const bool full = col0 + KPT <= p.d;
  uint8_t* my_rows = s_rows + tid * (KPT * 2);
  constexpr int kRowStride = kDecSelThreads * KPT * 2;
  if (col0 < p.d) {
    if (full) {
      // x is 16-byte aligned with a row pitch of a multiple of 8 elements, so
      // each chunk (8 or 16 bytes) is aligned
      for (int r = 0; r < p.n; ++r) {
        const uint16_t* src = p.x + static_cast<int64_t>(r) * p.ldx + col0;
        const uint32_t dst = smem_u32(my_rows + r * kRowStride);
        if constexpr (KPT == 8)
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
        else
          asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
    } else {
      for (int r = 0; r < p.n; ++r) {
        const uint16_t* src = p.x + static_cast<int64_t>(r) * p.ldx + col0;
        uint32_t* dst = reinterpret_cast<uint32_t*>(my_rows + r * kRowStride);
        for (int q = 0; q < WPR; ++q) {
          uint32_t v = 0u;
          for (int e = 2 * q; e < 2 * q + 2; ++e)
            if (col0 + e < p.d) v |= static_cast<uint32_t>(__ldg(src + e)) << (16 * (e & 1));
          dst[q] = v;
        }
      }
    }
  }
  // each thread reads back only what it copied itself
  auto row_words = [&](int64_t r, uint32_t(&w)[WPR]) {
    const uint8_t* src = my_rows + r * kRowStride;
    if constexpr (KPT == 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(src);
      w[0] = v.x;
      w[1] = v.y;
      w[2] = v.z;
      w[3] = v.w;
    } else {
      const uint2 v = *reinterpret_cast<const uint2*>(src);
      w[0] = v.x;
      w[1] = v.y;
    }
  };

  // ---- scores (fp64, bit-identical to colsq_short_kernel) and their key patterns
  uint64_t key[KPT];
  uint32_t valid = 0;
  {
    double acc[KPT];
    if (col0 < p.d) {
      colsq_short_sum<KPT>(p.n, row_words, acc);
    } else {
#pragma unroll
      for (int e = 0; e < KPT; ++e) acc[e] = 0.0;
    }
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
      key[e] = static_cast<uint64_t>(__double_as_longlong(acc[e]));
      if (col0 + e < p.d) valid |= 1u << e;
    }
  }

  // ---- radix select of the k-th largest key
  uint64_t pre = 0, msk = 0;
  int need = p.k;
  bool take = (p.k == p.d);
  int cursor = 0;  // bits [0, cursor) of the key are unresolved
  {
    uint64_t a = ~0ull, o = 0ull;
#pragma unroll
    for (int e = 0; e < KPT; ++e)
      if ((valid >> e) & 1u) {
        a &= key[e];
        o |= key[e];
      }
    decsel_cluster_andor(a, o, s_wand, s_wor, s_andor, s_andor_res, C);
    const uint64_t differ = a ^ o;
    if (!take) {
      if (differ == 0ull) {  // every key is the same: the lower indices win
        pre = a;
        msk = ~0ull;
      } else {
        const int top = 63 - __clzll(static_cast<long long>(differ));
        msk = (top == 63) ? 0ull : (~0ull << (top + 1));
        pre = a & msk;
        cursor = top + 1;
      }
    }
  }
  int pass = 0;
  while (!take && cursor > 0) {
    const int width = cursor >= 8 ? 8 : cursor;
    const int shift = cursor - width;
    const uint32_t dmask = (1u << width) - 1u;
    for (int i = lane; i < 256; i += 32) whist[warp][i] = 0u;
    __syncwarp();
    // the bucket's histogram of the next digit, and the AND / OR of its members
    uint64_t ba = ~0ull, bo = 0ull;
#pragma unroll
    for (int e = 0; e < KPT; ++e)
      if (((valid >> e) & 1u) && (key[e] & msk) == pre) {
        ba &= key[e];
        bo |= key[e];
        atomicAdd(&whist[warp][static_cast<uint32_t>(key[e] >> shift) & dmask], 1u);
      }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      ba &= __shfl_xor_sync(0xffffffffu, ba, off);
      bo |= __shfl_xor_sync(0xffffffffu, bo, off);
    }
    if (lane == 0) {
      s_wand[warp] = ba;
      s_wor[warp] = bo;
    }
    __syncthreads();
    uint32_t c = 0;
#pragma unroll
    for (int w = 0; w < kDecSelThreads / 32; ++w) c += whist[w][tid];
    uint32_t* hb = hist[pass & 1];
    hb[tid] = c;
    uint64_t* ab = s_pass_andor[pass & 1];
    if (tid == 0) {
      uint64_t xa = ~0ull, xo = 0ull;
      for (int w = 0; w < kDecSelThreads / 32; ++w) {
        xa &= s_wand[w];
        xo |= s_wor[w];
      }
      ab[0] = xa;
      ab[1] = xo;
    }
    // every CTA's histogram and AND / OR of this pass are visible (and the ones
    // two passes back are no longer read)
    cluster_sync();
    if (warp == 0) {
      uint64_t ra = ~0ull, ro = 0ull;
      if (lane < C) {
        const uint32_t aaddr = smem_u32(ab);
        ra = ld_shared_cluster_u64(map_shared_rank(aaddr, static_cast<uint32_t>(lane)));
        ro = ld_shared_cluster_u64(map_shared_rank(aaddr + 8, static_cast<uint32_t>(lane)));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        ra &= __shfl_xor_sync(0xffffffffu, ra, off);
        ro |= __shfl_xor_sync(0xffffffffu, ro, off);
      }
      if (lane == 0) {
        s_andor_res[0] = ra;
        s_andor_res[1] = ro;
      }
    }
    // thread t takes digit 255 - t, so the exclusive scan in thread order counts the larger digits
    const int bin = 255 - tid;
    const uint32_t haddr = smem_u32(hb + bin);
    uint32_t hv[kDecSelMaxCtas];
#pragma unroll
    for (int q = 0; q < kDecSelMaxCtas; ++q)
      hv[q] = q < C ? ld_shared_cluster_u32(map_shared_rank(haddr, static_cast<uint32_t>(q))) : 0u;
    uint32_t cnt = 0;
#pragma unroll
    for (int q = 0; q < kDecSelMaxCtas; ++q) cnt += hv[q];
    const int above = block_exclusive_scan<kDecSelThreads>(static_cast<int>(cnt), s_warp, &s_total);
    if (bin <= static_cast<int>(dmask) && above < need && need <= above + static_cast<int>(cnt)) {
      s_digit = bin;
      s_above = above;
      s_cnt = static_cast<int>(cnt);
    }
    __syncthreads();
    const uint64_t ga = s_andor_res[0], go = s_andor_res[1];
    const uint64_t open = (cursor >= 64) ? ~0ull : ((1ull << cursor) - 1ull);  // unresolved bits
    ++pass;
    if (((ga ^ go) & open) == 0ull) {
      // every member of the bucket has the same key: the lower indices win
      pre |= ga & open;
      msk = ~0ull;
      cursor = 0;
      __syncthreads();
      break;
    }
    need -= s_above;
    pre |= static_cast<uint64_t>(s_digit) << shift;
    msk |= static_cast<uint64_t>(dmask) << shift;
    cursor = shift;
    if (s_cnt == need) {
      take = true;
    } else if (cursor > 0) {
      // bits below the digit that the whole bucket shares are shared by the
      // digit's sub-bucket too: skip them (all of them for exact ties)
      const uint64_t below = (1ull << cursor) - 1ull;
      const uint64_t dl = (ga ^ go) & below;
      if (dl == 0ull) {
        pre |= ga & below;
        msk = ~0ull;
        cursor = 0;
      } else {
        const int top = 63 - __clzll(static_cast<long long>(dl));
        const uint64_t shared = below & ~((1ull << (top + 1)) - 1ull);
        pre |= ga & shared;
        msk |= shared;
        cursor = top + 1;
      }
    }
    __syncthreads();
  }

  // ---- classify: above the threshold, or equal to it
  uint32_t gt = 0, eq = 0;
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    if (!((valid >> e) & 1u)) continue;
    const uint64_t km = key[e] & msk;
    if (km > pre) gt |= 1u << e;
    else if (km == pre) eq |= 1u << e;
  }
  // this CTA's counts, exchanged across the cluster (column order = CTA order)
  const int eq_rank = block_exclusive_scan<kDecSelThreads>(__popc(eq), s_warp, &s_total);
  const int eq_cta = s_total;
  const int gt_rank = block_exclusive_scan<kDecSelThreads>(__popc(gt), s_warp, &s_total);
  (void)gt_rank;
  const int gt_cta = s_total;
  if (tid == 0) {
    s_counts[0] = gt_cta;
    s_counts[1] = eq_cta;
  }
  cluster_sync();
  if (warp == 0) {
    // lane q < rank holds CTA q's counts; the keys equal to the threshold that
    // CTA q takes depend on those of the CTAs before it (an exclusive scan)
    int g = 0, e = 0;
    if (lane < rank) {
      const uint32_t base = smem_u32(s_counts);
      g = static_cast<int>(ld_shared_cluster_u32(map_shared_rank(base, static_cast<uint32_t>(lane))));
      e = static_cast<int>(ld_shared_cluster_u32(map_shared_rank(base + 4, static_cast<uint32_t>(lane))));
    }
    int e_incl = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, e_incl, o);
      if (lane >= o) e_incl += y;
    }
    int taken = take ? e : need - (e_incl - e);
    taken = taken < 0 ? 0 : (taken > e ? e : taken);
    int sel_before = g + taken;  // 0 for lanes at or past rank
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sel_before += __shfl_xor_sync(0xffffffffu, sel_before, o);
    const int eq_before = __shfl_sync(0xffffffffu, e_incl, 31);
    if (lane == 0) {
      s_sel_base = sel_before;
      s_eq_before = eq_before;
    }
  }
  __syncthreads();
  // no CTA reads another's shared memory past this point: arrive now, and wait
  // (so that no CTA exits while another may still read it) only at the end
  cluster_arrive();
  uint32_t sel = gt;
  {
    int r = s_eq_before + eq_rank;
#pragma unroll
    for (int e = 0; e < KPT; ++e)
      if ((eq >> e) & 1u) {
        if (take || r < need) sel |= 1u << e;
        ++r;
      }
  }
  const int pos0 = s_sel_base + block_exclusive_scan<kDecSelThreads>(__popc(sel), s_warp, &s_total);
  {
    int pos = pos0;
#pragma unroll
    for (int e = 0; e < KPT; ++e)
      if ((sel >> e) & 1u) p.idx[pos++] = static_cast<int32_t>(col0 + e);
  }
  if (p.xpack != nullptr) {
    if (sel != 0u) {
      // from the staged copy of the thread's columns
      for (int r = 0; r < p.n; ++r) {
        uint32_t w[WPR];
        row_words(r, w);
        uint16_t* dst = p.xpack + static_cast<int64_t>(r) * p.ld_pack;
        int pos = pos0;
#pragma unroll
        for (int e = 0; e < KPT; ++e)
          if ((sel >> e) & 1u) dst[pos++] = static_cast<uint16_t>(w[e >> 1] >> (16 * (e & 1)));
      }
    }
    if (rank == C - 1 && tid < p.n)
      for (int64_t t = p.k; t < p.ld_pack; ++t) p.xpack[static_cast<int64_t>(tid) * p.ld_pack + t] = 0;
  }
  cluster_wait();
}

}  // namespace rmm
