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
