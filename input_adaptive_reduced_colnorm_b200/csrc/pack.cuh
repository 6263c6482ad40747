// Compact pack of the kept contraction columns: dst[r, t] = src[r, I[t]] for
// t < k, zero for k <= t < k_pad ("Algorithm Deep-Dive: RMM", Core Approach:
// RMM_rho(A, B) = A[:, I] B[I, :]; the gathered A[:, I] is stored K-major so the
// tensor-core GEMM can stream it with plain TMA tiles).
//
// A column gather of a row-major matrix touches nearly every 32-byte sector of
// a row, so each row is first staged in shared memory with coalesced 16-byte
// loads and the gather runs out of shared memory; writes are 16-byte vectors.
// Rows of at most 1024 columns are handled one per warp; longer rows one per CTA.
// With ``causal`` the entry (i, t) is kept only if I[t] <= i + causal_off (the
// masked upper triangle of an attention-probability matrix reads as zero), and
// only the visible prefix of the row is read.
#pragma once
#include "ptx.cuh"

namespace rmm {

struct PackParams {
  const uint16_t* src;   // bf16 bits
  int64_t src_ld;        // elements between rows of one source item
  int64_t rows;          // rows per batch item
  int64_t d;             // columns of the source
  // source item of batch item b: (b / g_outer) * s_outer + ((b % g_outer) / g_inner) * s_inner
  int64_t g_outer, g_inner, s_outer, s_inner;
  const int32_t* idx;    // [batch][k]
  int64_t k, k_pad;
  uint16_t* dst;         // [batch * rows][k_pad]
  int64_t batch;
  int causal;
  int64_t causal_off;
};

__device__ __forceinline__ const uint16_t* pack_src_row(const PackParams& p, int64_t r, int64_t& b, int64_t& i) {
  b = r / p.rows;
  i = r - b * p.rows;
  const int64_t item = (b / p.g_outer) * p.s_outer + ((b % p.g_outer) / p.g_inner) * p.s_inner;
  return p.src + item + i * p.src_ld;
}

__device__ __forceinline__ uint4 pack_gather8(const PackParams& p, const uint16_t* row, const int32_t* idx, int64_t t0,
                                              int64_t lim) {
  uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int64_t t = t0 + e;
    if (t < p.k) {
      const int32_t j = __ldg(idx + t);
      if (j < lim) w[e >> 1] |= static_cast<uint32_t>(row[j]) << (16 * (e & 1));
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void pack_stage(uint16_t* buf, const uint16_t* src, int64_t lim, int64_t d, int t,
                                           int nt) {
  // copy the first `lim` columns; vector loads where 8 columns fit inside d
  const int64_t nvec = (lim + 7) / 8;
  for (int64_t v = t; v < nvec; v += nt) {
    const int64_t c = v * 8;
    if (c + 8 <= d) {
      *reinterpret_cast<uint4*>(buf + c) = ldg_nc_v4(src + c);
    } else {
      for (int e = 0; e < 8; ++e) buf[c + e] = (c + e < d) ? __ldg(src + c + e) : uint16_t(0);
    }
  }
}

// one row per warp; dynamic shared memory: 8 warps x d_round bf16
__global__ void __launch_bounds__(256) pack_rows_warp_kernel(const PackParams p, int64_t d_round) {
  extern __shared__ __align__(16) uint16_t pk_smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint16_t* buf = pk_smem + warp * d_round;
  const int64_t total = p.batch * p.rows;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + warp; r < total; r += static_cast<int64_t>(gridDim.x) * 8) {
    int64_t b, i;
    const uint16_t* src = pack_src_row(p, r, b, i);
    int64_t lim = p.d;
    if (p.causal) {
      lim = i + p.causal_off + 1;
      if (lim > p.d) lim = p.d;
      if (lim < 0) lim = 0;
    }
    pack_stage(buf, src, lim, p.d, lane, 32);
    __syncwarp();
    const int32_t* idx = p.idx + b * p.k;
    uint16_t* dst = p.dst + r * p.k_pad;
    for (int64_t t0 = static_cast<int64_t>(lane) * 8; t0 < p.k_pad; t0 += 256) {
      const uint4 v = pack_gather8(p, buf, idx, t0, lim);
      if (t0 + 8 <= p.k_pad) {
        *reinterpret_cast<uint4*>(dst + t0) = v;
      } else {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        for (int e = 0; t0 + e < p.k_pad; ++e) dst[t0 + e] = static_cast<uint16_t>(w[e >> 1] >> (16 * (e & 1)));
      }
    }
    __syncwarp();
  }
}

// one row per CTA; dynamic shared memory: d_round bf16
__global__ void __launch_bounds__(256) pack_rows_cta_kernel(const PackParams p) {
  extern __shared__ __align__(16) uint16_t pk_smem[];
  const int64_t total = p.batch * p.rows;
  for (int64_t r = blockIdx.x; r < total; r += gridDim.x) {
    int64_t b, i;
    const uint16_t* src = pack_src_row(p, r, b, i);
    int64_t lim = p.d;
    if (p.causal) {
      lim = i + p.causal_off + 1;
      if (lim > p.d) lim = p.d;
      if (lim < 0) lim = 0;
    }
    pack_stage(pk_smem, src, lim, p.d, threadIdx.x, 256);
    __syncthreads();
    const int32_t* idx = p.idx + b * p.k;
    uint16_t* dst = p.dst + r * p.k_pad;
    for (int64_t t0 = static_cast<int64_t>(threadIdx.x) * 8; t0 < p.k_pad; t0 += 2048) {
      const uint4 v = pack_gather8(p, pk_smem, idx, t0, lim);
      if (t0 + 8 <= p.k_pad) {
        *reinterpret_cast<uint4*>(dst + t0) = v;
      } else {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        for (int e = 0; t0 + e < p.k_pad; ++e) dst[t0 + e] = static_cast<uint16_t>(w[e >> 1] >> (16 * (e & 1)));
      }
    }
    __syncthreads();
  }
}

// Row pack of the kept contraction rows of the second operand:
// dst[b][t, :] = src_item(b)[I_b[t], :] for t < k, zero rows for k <= t < rows_out
// ("Algorithm Deep-Dive: RMM", Core Approach: B[I, :]).  Whole rows are
// contiguous, so this is a fully coalesced 16-byte copy at HBM speed; the
// tensor-core GEMM then streams B[I, :] with large TMA tiles.
struct RowPackParams {
  const uint16_t* src;
  int64_t src_ld;                             // elements between source rows
  int64_t cols;                               // columns copied per row
  const int32_t* idx;                         // [batch][k]
  int64_t k;
  int64_t rows_out;                           // rows per batch item in dst (>= k)
  uint16_t* dst;
  int64_t dst_ld;                             // multiple of 8, >= cols
  int64_t batch;
  int64_t g_outer, g_inner, s_outer, s_inner; // source item of b (as in PackParams)
};

__global__ void __launch_bounds__(256) pack_rows_gather_kernel(const RowPackParams p) {
  constexpr int ILP = 4;
  const int64_t vpr = (p.cols + 7) / 8;  // 16-byte vectors per row
  const int64_t total = p.batch * p.rows_out * vpr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t v0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v0 < total; v0 += ILP * stride) {
    uint4 val[ILP];
    int64_t out_off[ILP];
#pragma unroll
    for (int u = 0; u < ILP; ++u) {
      const int64_t v = v0 + u * stride;
      val[u] = make_uint4(0u, 0u, 0u, 0u);
      out_off[u] = -1;
      if (v < total) {
        const int64_t row = v / vpr;
        const int64_t c = v - row * vpr;
        const int64_t b = row / p.rows_out;
        const int64_t t = row - b * p.rows_out;
        out_off[u] = row * p.dst_ld + c * 8;
        if (t < p.k) {
          const int64_t j = __ldg(p.idx + b * p.k + t);
          const int64_t item = (b / p.g_outer) * p.s_outer + ((b % p.g_outer) / p.g_inner) * p.s_inner;
          const uint16_t* src = p.src + item + j * p.src_ld + c * 8;
          if (c * 8 + 8 <= p.cols) {
            val[u] = ldg_nc_v4(src);
          } else {
            uint32_t w[4] = {0u, 0u, 0u, 0u};
            for (int e = 0; c * 8 + e < p.cols; ++e) w[e >> 1] |= static_cast<uint32_t>(__ldg(src + e)) << (16 * (e & 1));
            val[u] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < ILP; ++u)
      if (out_off[u] >= 0) *reinterpret_cast<uint4*>(p.dst + out_off[u]) = val[u];
  }
}

}  // namespace rmm
