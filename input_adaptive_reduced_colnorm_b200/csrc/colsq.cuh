// Column sum of squares q_j = sum_i A[i, j]^2 (the squared importance score
// s_j = ||A[:, j]||_2 of "Algorithm Deep-Dive: RMM", Core Approach).
//
// HBM-bound: every element of A is read once with 16-byte loads (8 bf16
// columns per thread).  Squares of bf16 values are exact in fp32; each thread
// adds four rows in fp32 and then folds that into an fp64 accumulator, so the
// result carries ~1e-7 relative error at most, far inside the 1e-5 near-tie
// band the parity tests use.
//
// Cross-row reduction: the CTAs of one thread-block cluster split the rows of
// one column strip; each CTA reduces its rows in shared memory, then CTA rank 0
// sums the partials of ranks 0..C-1 in that fixed order through distributed
// shared memory.  No atomics, no global partials, bitwise deterministic.
#pragma once
#include "ptx.cuh"

namespace rmm {

struct ColsqParams {
  const uint16_t* A;      // bf16 bits, [batch][n][lda]
  int64_t batch_stride;   // elements between batch items
  int64_t n, d, lda;
  int64_t causal_off;     // with CAUSAL: element (i, j) counts iff j <= i + causal_off
  double* colsq;          // [batch][d]
  int64_t rows_per_cta;   // rows handled by one CTA of a cluster
  int csize;              // cluster size along rows (1, 2, 4 or 8)
};

template <int TX, bool CAUSAL>
__global__ void __launch_bounds__(256, 2) colsq_kernel(const ColsqParams p) {
  wait_prior_kernels();
  constexpr int TY = 256 / TX;
  constexpr int W = TX * 8;  // columns per strip
  __shared__ double red[TY][W + 1];
  __shared__ double part[W];

  const int tx = threadIdx.x % TX;
  const int ty = threadIdx.x / TX;
  const int C = p.csize;
  const uint32_t rank = (C > 1) ? cluster_ctarank() : 0u;
  const int64_t strip = blockIdx.x / C;
  const int64_t b = blockIdx.y;
  const int64_t col0 = strip * W + tx * 8;
  const uint16_t* A = p.A + b * p.batch_stride;

  int64_t r_begin = static_cast<int64_t>(rank) * p.rows_per_cta;
  int64_t r_end = r_begin + p.rows_per_cta;
  if (r_end > p.n) r_end = p.n;
  if (CAUSAL) {
    // rows i < strip_start - off see none of this strip's columns
    const int64_t first = strip * W - p.causal_off;
    if (first > r_begin) r_begin = first;
  }

  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;

  if (col0 < p.d) {
    const bool full = (col0 + 8 <= p.d);
    // bursts of U rows: all U 16-byte loads are in flight before any is used
    constexpr int U = 16;
    for (int64_t i = r_begin + ty; i < r_end; i += U * TY) {
      uint32_t w[U][4];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t row = i + u * TY;
        w[u][0] = w[u][1] = w[u][2] = w[u][3] = 0u;
        if (row < r_end) {
          const uint16_t* src = A + row * p.lda + col0;
          if (full) {
            const uint4 v = ldg_nc_v4(src);
            w[u][0] = v.x; w[u][1] = v.y; w[u][2] = v.z; w[u][3] = v.w;
          } else {
            for (int e = 0; e < 8; ++e)
              if (col0 + e < p.d) w[u][e >> 1] |= static_cast<uint32_t>(__ldg(src + e)) << (16 * (e & 1));
          }
        }
      }
      // four rows at a time in fp32 (bf16 squares are exact in fp32), then fp64
#pragma unroll
      for (int g = 0; g < U; g += 4) {
        float a32[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) a32[e] = 0.f;
#pragma unroll
        for (int u = g; u < g + 4; ++u) {
          const int64_t lim = CAUSAL ? (i + u * TY + p.causal_off) : 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float x = (e & 1) ? bf16hi(w[u][e >> 1]) : bf16lo(w[u][e >> 1]);
            if (CAUSAL && col0 + e > lim) x = 0.f;
            a32[e] = fmaf(x, x, a32[e]);
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += static_cast<double>(a32[e]);
      }
    }
  }

#pragma unroll
  for (int e = 0; e < 8; ++e) red[ty][tx * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < W) {
    double s = 0.0;
    for (int y = 0; y < TY; ++y) s += red[y][threadIdx.x];
    part[threadIdx.x] = s;
  }
  if (C > 1) {
    cluster_sync();  // every CTA's partial is now visible to the cluster
    if (rank == 0 && threadIdx.x < W) {
      const int64_t col = strip * W + threadIdx.x;
      const uint32_t a = smem_u32(&part[threadIdx.x]);
      double s = 0.0;
      for (int r = 0; r < C; ++r) s += ld_shared_cluster_f64(map_shared_rank(a, static_cast<uint32_t>(r)));
      if (col < p.d) p.colsq[b * p.d + col] = s;
    }
    cluster_sync();  // keep every CTA's shared memory alive until rank 0 has read it
  } else {
    if (threadIdx.x < W) {
      const int64_t col = strip * W + threadIdx.x;
      if (col < p.d) p.colsq[b * p.d + col] = part[threadIdx.x];
    }
  }
}

}  // namespace rmm

namespace rmm {

// ---------------------------------------------------------------- TMA-staged variant
// Same sums, for matrices with at least a few dozen rows.  A strip of W columns
// is streamed through shared memory in 16 KB tiles of R = 8192 / W rows by one
// producer thread issuing 3-D TMA loads (x = column, y = row, z = batch item)
// into a ring of kColsqStages buffers; eight consumer warps square and sum each
// tile straight out of shared memory.  Keeping ~96 KB of loads in flight per
// CTA costs no registers, so the kernel holds HBM busy with two CTAs per SM.
//
// Work split: the CTAs of a cluster share one strip.  With CAUSAL the rows of
// a strip that see none of its columns are skipped first and only the visible
// rows are dealt out in whole tiles, so every CTA of the cluster has the same
// amount of work (the triangle of a causal matrix no longer leaves half of
// each cluster idle at the cluster barrier).  Rows past n and columns past d
// are outside the tensor map and arrive as zeros.
//
// Summation order per column: each thread adds 4 rows in fp32 (exact bf16
// squares, ~1e-7 relative rounding), folds them into fp64, then the warps'
// partials are added in a fixed order and the cluster's CTAs in rank order.
// Deterministic.
constexpr int kColsqStages = 6;
constexpr uint32_t kColsqTileBytes = 16384;
constexpr int kColsqThreads = 288;  // 8 consumer warps + 1 producer warp

struct ColsqTmaParams {
  int64_t n, d;
  int64_t causal_off;  // with CAUSAL: element (i, j) counts iff j <= i + causal_off
  double* colsq;       // [batch][d]
  int csize;           // CTAs of a cluster sharing one strip (1, 2, 4 or 8)
};

template <int W>
struct ColsqShape {
  static constexpr int TX = W / 8;                          // threads across a row (8 columns each)
  static constexpr int TY = 256 / TX;                       // rows covered by one pass of the consumers
  static constexpr int R = kColsqTileBytes / (2 * W);       // rows per tile
  static constexpr int RPT = R / TY;                        // rows per thread per tile
  static_assert(RPT == 4, "each thread adds four rows of a tile in fp32");
};

template <int W, bool CAUSAL>
__global__ void __launch_bounds__(kColsqThreads, 2)
    colsq_tma_kernel(const __grid_constant__ CUtensorMap tmA, const ColsqTmaParams p) {
  using S = ColsqShape<W>;
  extern __shared__ __align__(128) uint8_t smem[];  // kColsqStages tiles, reused for the final reduction
  __shared__ uint64_t full[kColsqStages], empty[kColsqStages];
  __shared__ double part[W];
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int C = p.csize;
  const uint32_t rank = (C > 1) ? cluster_ctarank() : 0u;
  const int64_t strip = blockIdx.x / C;
  const int b = blockIdx.y;
  const int64_t c0 = strip * W;

  // the strip's visible rows, in whole tiles, split evenly over the cluster
  int64_t first = 0;
  if (CAUSAL) {
    first = c0 - p.causal_off;
    if (first < 0) first = 0;
    first = first / S::R * S::R;
  }
  const int64_t tiles = first < p.n ? (p.n - first + S::R - 1) / S::R : 0;
  const int64_t per = (tiles + C - 1) / C;
  const int64_t t_begin = static_cast<int64_t>(rank) * per;
  const int64_t t_end = t_begin + per < tiles ? t_begin + per : tiles;
  const int nt = t_end > t_begin ? static_cast<int>(t_end - t_begin) : 0;
  const int64_t row0 = first + t_begin * S::R;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kColsqStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8 && lane == 0) prefetch_tensormap(&tmA);
  __syncthreads();
  wait_prior_kernels();

  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
  const int tx = threadIdx.x % S::TX;
  const int ty = threadIdx.x / S::TX;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0;
      bool ok = true;
      for (int t = 0; t < nt; ++t) {
        const int stage = t % kColsqStages;
        const int use = t / kColsqStages;
        if (use > 0 && !mbar_wait(&empty[stage], (use - 1) & 1, abort_flag, kDevErrTimeoutProducer)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], kColsqTileBytes);
        tma_load_3d(smem + stage * kColsqTileBytes, &tmA, &full[stage], static_cast<int32_t>(c0),
                    static_cast<int32_t>(row0 + static_cast<int64_t>(t) * S::R), b);
        ++issued;
      }
      if (!ok) {
        // wait (bounded) for the loads already issued so none lands after exit
        for (int s = 0; s < kColsqStages; ++s) {
          const uint32_t uses = (issued + kColsqStages - 1 - s) / kColsqStages;
          if (uses == 0) continue;
          const uint32_t a = smem_u32(&full[s]);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(a, (uses - 1) & 1u) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const uint32_t base = smem_u32(smem) + static_cast<uint32_t>((ty * W + tx * 8) * 2);
    for (int t = 0; t < nt; ++t) {
      const int stage = t % kColsqStages;
      if (!mbar_wait(&full[stage], (t / kColsqStages) & 1, abort_flag, kDevErrTimeoutEpilogue)) break;
      uint4 v[S::RPT];
#pragma unroll
      for (int u = 0; u < S::RPT; ++u) v[u] = lds_v4(base + stage * kColsqTileBytes + u * S::TY * W * 2);
      const uint32_t* w = reinterpret_cast<const uint32_t*>(v);
      float a32[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) a32[e] = 0.f;
      const int64_t r = row0 + static_cast<int64_t>(t) * S::R;
      if (CAUSAL && c0 + W - 1 > r + p.causal_off) {
        // this tile crosses the diagonal: drop (i, j) with j > i + off
#pragma unroll
        for (int u = 0; u < S::RPT; ++u) {
          const int64_t lim = r + ty + u * S::TY + p.causal_off - (c0 + tx * 8);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float x = (e & 1) ? bf16hi(w[u * 4 + (e >> 1)]) : bf16lo(w[u * 4 + (e >> 1)]);
            if (e > lim) x = 0.f;
            a32[e] = fmaf(x, x, a32[e]);
          }
        }
      } else {
#pragma unroll
        for (int u = 0; u < S::RPT; ++u) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float x = (e & 1) ? bf16hi(w[u * 4 + (e >> 1)]) : bf16lo(w[u * 4 + (e >> 1)]);
            a32[e] = fmaf(x, x, a32[e]);
          }
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += static_cast<double>(a32[e]);
      // release the stage only once its values are consumed, with the warp's
      // reads ordered before the producer's next TMA write into it
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
    }
  }

  // ------------------------------------------------------------ reduction
  __syncthreads();  // every tile consumed (or abandoned): the ring can hold the partials
  double* red = reinterpret_cast<double*>(smem);  // [TY][W]
  if (warp < 8) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red[ty * W + tx * 8 + e] = acc[e];
  }
  __syncthreads();
  if (threadIdx.x < W) {
    double s = 0.0;
    for (int y = 0; y < S::TY; ++y) s += red[y * W + threadIdx.x];
    part[threadIdx.x] = s;
  }
  if (C > 1) {
    cluster_sync();
    if (rank == 0 && threadIdx.x < W) {
      const int64_t col = c0 + threadIdx.x;
      const uint32_t a = smem_u32(&part[threadIdx.x]);
      double s = 0.0;
      for (int q = 0; q < C; ++q) s += ld_shared_cluster_f64(map_shared_rank(a, static_cast<uint32_t>(q)));
      if (col < p.d) p.colsq[static_cast<int64_t>(b) * p.d + col] = s;
    }
    cluster_sync();
  } else if (threadIdx.x < W) {
    const int64_t col = c0 + threadIdx.x;
    if (col < p.d) p.colsq[static_cast<int64_t>(b) * p.d + col] = part[threadIdx.x];
  }
}

}  // namespace rmm

namespace rmm {

// ---------------------------------------------------------------- short matrices
// Column sums of squares of a matrix of at most 32 rows (decode activations,
// the query rows of one key/value group): one thread per 8 columns reads all n
// rows of its columns, so no reduction between threads is needed and a grid of
// ceil(d / 1024) x batch CTAs of 128 threads covers the matrix once.  Rows are
// summed 4 at a time in fp32 (exact bf16 squares) and folded into fp64, in row
// order.  Non-causal only.
constexpr int kColsqShortMaxRows = 32;

// Sums of squares of columns [col0, col0 + CPT) (CPT = 4 or 8) of an n-row
// matrix (n may be anything; used for n <= 32): rows summed 4 at a time in fp32
// (exact bf16 squares) and folded into fp64, in row order.  Columns at or past d
// read as 0.  Each column's arithmetic does not depend on CPT, and the decode
// selection kernel computes its scores with this same summation (reading its
// rows from shared memory), so its keys are bit-identical to colsq_short_kernel's.
//
// The summation itself, over row chunks that ``row_words(r, w)`` supplies (the
// CPT bf16 values of row r as CPT / 2 packed words): rows in batches of eight
// (all eight fetched before any is used), four squares added in fp32, then each
// group of four added to the fp64 total in row order.
template <int CPT, typename RowWords>
__device__ __forceinline__ void colsq_short_sum(int64_t n, RowWords&& row_words, double (&acc)[CPT]) {
  static_assert(CPT == 4 || CPT == 8, "four or eight columns per thread");
  constexpr int WPR = CPT / 2;  // 32-bit words per row chunk
#pragma unroll
  for (int e = 0; e < CPT; ++e) acc[e] = 0.0;
  for (int64_t r0 = 0; r0 < n; r0 += 8) {
    uint32_t w[8][WPR];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
#pragma unroll
      for (int q = 0; q < WPR; ++q) w[u][q] = 0u;
      if (r0 + u < n) row_words(r0 + u, w[u]);
    }
#pragma unroll
    for (int g = 0; g < 8; g += 4) {
      float a32[CPT];
#pragma unroll
      for (int e = 0; e < CPT; ++e) a32[e] = 0.f;
#pragma unroll
      for (int u = g; u < g + 4; ++u) {
#pragma unroll
        for (int e = 0; e < CPT; ++e) {
          const float x = (e & 1) ? bf16hi(w[u][e >> 1]) : bf16lo(w[u][e >> 1]);
          a32[e] = fmaf(x, x, a32[e]);
        }
      }
#pragma unroll
      for (int e = 0; e < CPT; ++e) acc[e] += static_cast<double>(a32[e]);
    }
  }
}

// Columns col0 .. col0 + CPT - 1 of A read from global memory.
template <int CPT>
__device__ __forceinline__ void colsq_short_cols(const uint16_t* A, int64_t lda, int64_t n, int64_t col0, int64_t d,
                                                 double (&acc)[CPT]) {
  constexpr int WPR = CPT / 2;
  const bool full = col0 + CPT <= d;
  colsq_short_sum<CPT>(
      n,
      [&](int64_t r, uint32_t(&w)[WPR]) {
        const uint16_t* src = A + r * lda + col0;
        if (full) {
          if constexpr (CPT == 8) {
            const uint4 v = ldg_nc_v4(src);
            w[0] = v.x;
            w[1] = v.y;
            w[2] = v.z;
            w[3] = v.w;
          } else {
            const uint2 v = ldg_nc_v2(src);
            w[0] = v.x;
            w[1] = v.y;
          }
        } else {
          for (int e = 0; e < CPT; ++e)
            if (col0 + e < d) w[e >> 1] |= static_cast<uint32_t>(__ldg(src + e)) << (16 * (e & 1));
        }
      },
      acc);
}

__global__ void __launch_bounds__(128) colsq_short_kernel(const ColsqParams p) {
  wait_prior_kernels();
  const int64_t b = blockIdx.y;
  const int64_t col0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (col0 >= p.d) return;
  double acc[8];
  colsq_short_cols<8>(p.A + b * p.batch_stride, p.lda, p.n, col0, p.d, acc);
  double* out = p.colsq + b * p.d + col0;
#pragma unroll
  for (int e = 0; e < 8; ++e)
    if (col0 + e < p.d) out[e] = acc[e];
}

}  // namespace rmm
