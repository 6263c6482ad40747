// Compact pack of the kept contraction columns: dst[r, t] = src[r, I[t]] for
// t < k, zero for k <= t < k_pad ("Algorithm Deep-Dive: RMM", Core Approach:
// RMM_rho(A, B) = A[:, I] B[I, :]; the gathered A[:, I] is stored K-major so the
// tensor-core GEMM can stream it with plain TMA tiles).
//
// A column gather of a row-major matrix touches nearly every 32-byte sector of
// a row, so each row is first staged in shared memory with coalesced 16-byte
// loads and the gather runs out of shared memory; writes are 16-byte vectors.
// Rows of at most 1024 columns are handled one per warp; longer rows one per
// CTA, with the next row's cp.async copy in flight while the current row is
// gathered and the index set held in shared memory as 16-bit offsets.
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

// first element of batch item b's source matrix (32-bit division when it fits)
__device__ __forceinline__ const uint16_t* pack_item_base(const PackParams& p, int64_t b) {
  if (b < (1LL << 31) && p.g_outer < (1LL << 31) && p.g_inner < (1LL << 31)) {
    const uint32_t b32 = static_cast<uint32_t>(b), go = static_cast<uint32_t>(p.g_outer);
    const uint32_t outer = b32 / go, inner = (b32 - outer * go) / static_cast<uint32_t>(p.g_inner);
    return p.src + static_cast<int64_t>(outer) * p.s_outer + static_cast<int64_t>(inner) * p.s_inner;
  }
  return p.src + (b / p.g_outer) * p.s_outer + ((b % p.g_outer) / p.g_inner) * p.s_inner;
}

__device__ __forceinline__ const uint16_t* pack_src_row(const PackParams& p, int64_t r, int64_t& b, int64_t& i) {
  if (r < (1LL << 31) && p.rows < (1LL << 31))
    b = static_cast<uint32_t>(r) / static_cast<uint32_t>(p.rows);
  else
    b = r / p.rows;
  i = r - b * p.rows;
  return pack_item_base(p, b) + i * p.src_ld;
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
  wait_prior_kernels();
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

__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ int64_t pack_visible(const PackParams& p, int64_t i) {
  if (!p.causal) return p.d;
  int64_t lim = i + p.causal_off + 1;
  return lim > p.d ? p.d : (lim < 0 ? 0 : lim);
}

// async copy of the first `lim` columns of one row into shared memory
__device__ __forceinline__ void pack_stage_async(uint16_t* buf, const uint16_t* src, int64_t lim, int64_t d) {
  const int64_t nvec = (lim + 7) / 8;
  for (int64_t v = threadIdx.x; v < nvec; v += blockDim.x) {
    const int64_t c = v * 8;
    const int64_t rem = d - c;
    cp_async16_zfill(buf + c, src + c, rem >= 8 ? 16u : static_cast<uint32_t>(rem * 2));
  }
}

// Contiguous row range per CTA; NBUF row buffers, so NBUF - 1 rows are being
// copied (cp.async) while the current row is gathered.  Dynamic shared memory:
// 16-bit index offsets [k_pad] (0xFFFF marks padding) + NBUF row buffers
// [d_round].  The batch item of a row is tracked incrementally (integer
// divisions only when the item changes).
struct PackCursor {
  int64_t b, i;          // batch item, row within it
  const uint16_t* base;  // source item base
  __device__ void init(const PackParams& p, int64_t r) {
    b = r / p.rows;
    i = r - b * p.rows;
    set_base(p);
  }
  __device__ void set_base(const PackParams& p) {
    base = p.src + (b / p.g_outer) * p.s_outer + ((b % p.g_outer) / p.g_inner) * p.s_inner;
  }
  __device__ void next(const PackParams& p) {
    if (++i == p.rows) {
      i = 0;
      ++b;
      set_base(p);
    }
  }
};

template <int NBUF>
__global__ void __launch_bounds__(256) pack_rows_cta_kernel(const PackParams p, int64_t d_round, int64_t idx_elems) {
  wait_prior_kernels();
  extern __shared__ __align__(16) uint16_t pk_smem[];
  uint16_t* s_idx = pk_smem;
  uint16_t* bufs = pk_smem + idx_elems;
  const int64_t total = p.batch * p.rows;
  const int64_t per = (total + gridDim.x - 1) / gridDim.x;
  const int64_t r_begin = static_cast<int64_t>(blockIdx.x) * per;
  int64_t r_end = r_begin + per;
  if (r_end > total) r_end = total;
  if (r_begin >= r_end) return;
  const int nrows = static_cast<int>(r_end - r_begin);
  const int k_pad = static_cast<int>(p.k_pad);

  PackCursor stage_at, gather_at;
  stage_at.init(p, r_begin);
  gather_at = stage_at;
  // prologue: the first NBUF - 1 rows (one commit group each, empty groups past the end)
#pragma unroll
  for (int q = 0; q < NBUF - 1; ++q) {
    if (q < nrows) {
      pack_stage_async(bufs + q * d_round, stage_at.base + stage_at.i * p.src_ld, pack_visible(p, stage_at.i), p.d);
      stage_at.next(p);
    }
    cp_async_commit();
  }
  int64_t cur_b = -1;
  for (int q = 0; q < nrows; ++q) {
    {  // copy row q + NBUF - 1 into the buffer freed by row q - 1
      const int qn = q + NBUF - 1;
      if (qn < nrows) {
        pack_stage_async(bufs + (qn % NBUF) * d_round, stage_at.base + stage_at.i * p.src_ld,
                         pack_visible(p, stage_at.i), p.d);
        stage_at.next(p);
      }
      cp_async_commit();
      cp_async_wait<NBUF - 1>();  // row q's group has landed
    }
    if (gather_at.b != cur_b) {  // (re)load this batch item's index set as 16-bit offsets
      const int32_t* I = p.idx + gather_at.b * p.k;
      const int k = static_cast<int>(p.k);
      for (int t0 = threadIdx.x; t0 < k_pad; t0 += 8 * blockDim.x) {
        int32_t v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {  // eight loads in flight per thread
          const int t = t0 + e * blockDim.x;
          v[e] = (t < k) ? __ldg(I + t) : 0xFFFF;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int t = t0 + e * blockDim.x;
          if (t < k_pad) s_idx[t] = static_cast<uint16_t>(v[e]);
        }
      }
      cur_b = gather_at.b;
    }
    __syncthreads();
    const uint16_t* row = bufs + (q % NBUF) * d_round;
    const uint32_t lim = static_cast<uint32_t>(pack_visible(p, gather_at.i));
    uint16_t* dst = p.dst + (r_begin + q) * p.k_pad;
    for (int t0 = threadIdx.x * 8; t0 < k_pad; t0 += 8 * blockDim.x) {
      const uint4 iv = *reinterpret_cast<const uint4*>(s_idx + t0);
      const uint32_t iw[4] = {iv.x, iv.y, iv.z, iv.w};
      uint32_t w[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const uint32_t j0 = iw[h] & 0xFFFFu, j1 = iw[h] >> 16;
        const uint32_t v0 = (j0 < lim) ? row[j0] : 0u;  // 0xFFFF padding is never < lim (d <= 32768)
        const uint32_t v1 = (j1 < lim) ? row[j1] : 0u;
        w[h] = v0 | (v1 << 16);
      }
      *reinterpret_cast<uint4*>(dst + t0) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    gather_at.next(p);
    __syncthreads();
  }
}

// Short rows (d <= 512): one warp per row, no shared-memory staging.  Lane l
// produces the column pairs l, l + 32, ... of the packed row from two 2-byte
// loads of the source row (its few 128-byte lines stay in L1 while the warp
// gathers them) and the warp writes 128 contiguous bytes per pair group.  Four
// rows are in flight per warp; the kept-index pairs of the current batch item
// stay in registers (lanes x pair groups <= 32 x 4, so k_pad <= 256).
__global__ void __launch_bounds__(256) pack_short_rows_kernel(const PackParams p) {
  wait_prior_kernels();
  constexpr int R = 4;   // rows in flight per warp
  constexpr int PG = 4;  // pair groups per lane: k_pad <= 2 * 32 * PG
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t total = p.batch * p.rows;
  const int pairs = static_cast<int>(p.k_pad / 2);
  int64_t cur_b = -1;
  int j0[PG], j1[PG];
  for (int64_t r0 = (static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) * R; r0 < total;
       r0 += warps * R) {
    uint32_t out[R][PG];
    // batch item and row of r0 (the divisions once per R rows, 32-bit when the
    // sizes allow); the next rows step through them
    int64_t b, i;
    if (total < (1LL << 31)) {
      b = static_cast<uint32_t>(r0) / static_cast<uint32_t>(p.rows);
      i = r0 - b * p.rows;
    } else {
      b = r0 / p.rows;
      i = r0 - b * p.rows;
    }
    const uint16_t* item_base = pack_item_base(p, b);
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const int64_t row = r0 + u;
#pragma unroll
      for (int q = 0; q < PG; ++q) out[u][q] = 0u;
      if (row >= total) continue;
      if (u > 0 && ++i == p.rows) {
        ++b;
        i = 0;
        item_base = pack_item_base(p, b);
      }
      const uint16_t* src = item_base + i * p.src_ld;
      if (b != cur_b) {  // this batch item's kept columns (0xFFFF past k: padding)
#pragma unroll
        for (int q = 0; q < PG; ++q) {
          const int t = 2 * (q * 32 + lane);
          j0[q] = (t < p.k) ? __ldg(p.idx + b * p.k + t) : 0xFFFF;
          j1[q] = (t + 1 < p.k) ? __ldg(p.idx + b * p.k + t + 1) : 0xFFFF;
        }
        cur_b = b;
      }
      const int64_t lim = pack_visible(p, i);
#pragma unroll
      for (int q = 0; q < PG; ++q) {
        const uint32_t v0 = (j0[q] < lim) ? __ldg(src + j0[q]) : 0u;
        const uint32_t v1 = (j1[q] < lim) ? __ldg(src + j1[q]) : 0u;
        out[u][q] = v0 | (v1 << 16);
      }
    }
#pragma unroll
    for (int u = 0; u < R; ++u) {
      const int64_t row = r0 + u;
      if (row >= total) continue;
      uint32_t* dst = reinterpret_cast<uint32_t*>(p.dst + row * p.k_pad);
#pragma unroll
      for (int q = 0; q < PG; ++q) {
        const int t2 = q * 32 + lane;
        if (t2 < pairs) dst[t2] = out[u][q];
      }
    }
  }
}

// Narrow rows (d a power of two from 64 to 256, no causal mask, rows per batch
// item a multiple of 8): each warp stages 8 consecutive rows with 16-byte loads,
// all in flight at once, into its shared-memory slice, then lane l writes the
// column pairs l, l + 32, ... of each packed row from there.  (One row in flight
// per warp left the 131072-row packs of the attention's 64-dim score product
// latency-bound.)  The kept-index pairs of the current batch item stay in
// registers (k_pad <= 256).
template <int D>
__global__ void __launch_bounds__(256) pack_narrow_rows_kernel(const PackParams p) {
  wait_prior_kernels();
  constexpr int RW = 8;            // rows per warp step
  constexpr int VPR = D / 8;       // 16-byte vectors per row
  constexpr int VPL = RW * VPR / 32;  // vectors per lane per step
  constexpr int PG = 4;            // pair groups per lane: k_pad <= 256
  __shared__ __align__(16) uint16_t pn_buf[8][RW][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint16_t (*buf)[D] = pn_buf[warp];
  const int64_t steps = p.batch * p.rows / RW;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * 8;
  const int pairs = static_cast<int>(p.k_pad / 2);
  int64_t cur_b = -1;
  uint32_t j0[PG], j1[PG];
  for (int64_t st = static_cast<int64_t>(blockIdx.x) * 8 + warp; st < steps; st += wstride) {
    const int64_t r0 = st * RW;
    int64_t b, i;
    const uint16_t* src = pack_src_row(p, r0, b, i);  // the step's 8 rows share their batch item
    uint4 v[VPL];
#pragma unroll
    for (int q = 0; q < VPL; ++q) {
      const int vi = q * 32 + lane;
      v[q] = ldg_nc_v4(src + static_cast<int64_t>(vi / VPR) * p.src_ld + (vi % VPR) * 8);
    }
    if (b != cur_b) {  // this batch item's kept columns (0xFFFF past k: padding)
#pragma unroll
      for (int q = 0; q < PG; ++q) {
        const int t = 2 * (q * 32 + lane);
        j0[q] = (t < p.k) ? static_cast<uint32_t>(__ldg(p.idx + b * p.k + t)) : 0xFFFFu;
        j1[q] = (t + 1 < p.k) ? static_cast<uint32_t>(__ldg(p.idx + b * p.k + t + 1)) : 0xFFFFu;
      }
      cur_b = b;
    }
    __syncwarp();  // the previous step's gathers from buf are done
#pragma unroll
    for (int q = 0; q < VPL; ++q) {
      const int vi = q * 32 + lane;
      *reinterpret_cast<uint4*>(&buf[vi / VPR][(vi % VPR) * 8]) = v[q];
    }
    __syncwarp();
#pragma unroll
    for (int u = 0; u < RW; ++u) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(p.dst + (r0 + u) * p.k_pad);
#pragma unroll
      for (int q = 0; q < PG; ++q) {
        const int t2 = q * 32 + lane;
        if (t2 < pairs) {
          const uint32_t a = (j0[q] < static_cast<uint32_t>(D)) ? buf[u][j0[q]] : 0u;
          const uint32_t c = (j1[q] < static_cast<uint32_t>(D)) ? buf[u][j1[q]] : 0u;
          dst[t2] = a | (c << 16);
        }
      }
    }
  }
}

// Same pack, with each source row staged by one 1-D bulk copy (TMA) instead
// of 16-byte cp.async by every thread.  Thread 0 keeps NBUF - 1 rows in
// flight; the CTA gathers one staged row per step with a single barrier.
// Each thread produces column PAIRS: lanes read consecutive entries of the
// index set, so the 32 gathers of one warp instruction fall within a few
// hundred bytes of the row (no 8-way bank conflicts) and the warp writes 128
// contiguous bytes.  Dynamic shared memory: NBUF row buffers of ``buf_bytes``,
// then the index set as 16-bit offsets [k_pad] (0xFFFF marks padding).
// Requires 16-byte aligned source rows and an even k_pad.
template <int NBUF>
__global__ void __launch_bounds__(256) pack_rows_bulk_kernel(const PackParams p, uint32_t buf_bytes) {
  extern __shared__ __align__(128) uint8_t pk_bulk_smem[];
  __shared__ uint64_t full[NBUF];
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;
  uint8_t* bufs = pk_bulk_smem;
  uint16_t* s_idx = reinterpret_cast<uint16_t*>(pk_bulk_smem + static_cast<size_t>(NBUF) * buf_bytes);

  const int64_t total = p.batch * p.rows;
  const int64_t per = (total + gridDim.x - 1) / gridDim.x;
  const int64_t r_begin = static_cast<int64_t>(blockIdx.x) * per;
  int64_t r_end = r_begin + per;
  if (r_end > total) r_end = total;
  if (r_begin >= r_end) return;  // uniform over the CTA
  const int nrows = static_cast<int>(r_end - r_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NBUF; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  wait_prior_kernels();

  PackCursor stage_at, gather_at;
  stage_at.init(p, r_begin);
  gather_at = stage_at;
  uint32_t issued = 0;
  auto issue_next = [&]() {  // thread 0: stage row `issued` into buffer issued % NBUF
    const int64_t lim = pack_visible(p, stage_at.i);
    const uint32_t bytes = static_cast<uint32_t>((lim + 7) / 8 * 16);
    uint64_t* bar = &full[issued % NBUF];
    if (bytes > 0) {
      mbar_arrive_expect_tx(bar, bytes);
      bulk_load_1d(bufs + (issued % NBUF) * buf_bytes, stage_at.base + stage_at.i * p.src_ld, bytes, bar);
    } else {
      mbar_arrive(bar);  // nothing visible in this row
    }
    stage_at.next(p);
    ++issued;
  };
  if (threadIdx.x == 0)
    while (issued < static_cast<uint32_t>(NBUF - 1) && issued < static_cast<uint32_t>(nrows)) issue_next();

  const int pairs = static_cast<int>(p.k_pad / 2);
  const uint32_t* idx2 = reinterpret_cast<const uint32_t*>(s_idx);
  int64_t cur_b = -1;
  for (int q = 0; q < nrows; ++q) {
    if (gather_at.b != cur_b) {  // (re)load this batch item's index set
      __syncthreads();
      const int32_t* I = p.idx + gather_at.b * p.k;
      const int k = static_cast<int>(p.k);
      const int k_pad = static_cast<int>(p.k_pad);
      for (int t0 = threadIdx.x; t0 < k_pad; t0 += 8 * blockDim.x) {
        int32_t v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int t = t0 + e * blockDim.x;
          v[e] = (t < k) ? __ldg(I + t) : 0xFFFF;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int t = t0 + e * blockDim.x;
          if (t < k_pad) s_idx[t] = static_cast<uint16_t>(v[e]);
        }
      }
      cur_b = gather_at.b;
    }
    const bool got = mbar_wait(&full[q % NBUF], (q / NBUF) & 1, abort_flag, kDevErrTimeoutProducer);
    // row q has landed everywhere and every thread is done with row q - 1
    if (!__syncthreads_and(got)) break;
    if (threadIdx.x == 0 && issued < static_cast<uint32_t>(nrows)) {
      // every thread's reads of row q - 1's buffer (ordered before this point by
      // the barrier) before the bulk copy into it: the issuing thread fences
      fence_proxy_async_smem();
      issue_next();  // into row q - 1's buffer
    }

    const uint16_t* row = reinterpret_cast<const uint16_t*>(bufs + (q % NBUF) * buf_bytes);
    const uint32_t lim = static_cast<uint32_t>(pack_visible(p, gather_at.i));
    uint32_t* dst = reinterpret_cast<uint32_t*>(p.dst + (r_begin + q) * p.k_pad);
#pragma unroll 4
    for (int t = threadIdx.x; t < pairs; t += 256) {
      const uint32_t w = idx2[t];
      const uint32_t j0 = w & 0xFFFFu, j1 = w >> 16;
      const uint32_t v0 = (j0 < lim) ? row[j0] : 0u;  // 0xFFFF padding is never < lim (d <= 32768)
      const uint32_t v1 = (j1 < lim) ? row[j1] : 0u;
      dst[t] = v0 | (v1 << 16);
    }
    gather_at.next(p);
  }
  if (threadIdx.x == 0 && *abort_flag) {
    // wait (bounded) for the copies already issued so none lands after exit
    for (int s = 0; s < NBUF; ++s) {
      const uint32_t uses = (issued + NBUF - 1 - s) / NBUF;
      if (uses == 0) continue;
      const uint32_t a = smem_u32(&full[s]);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(a, (uses - 1) & 1u) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
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

// 2-D layout: 2^tpr_log2 threads per output row, 256 >> tpr_log2 rows per CTA
// pass, grid-stride over row groups; each thread copies every (2^tpr_log2)-th
// 16-byte vector of its row, up to eight loads in flight.
__global__ void __launch_bounds__(256) pack_rows_gather_kernel(const RowPackParams p, int tpr_log2) {
  wait_prior_kernels();
  constexpr int ILP = 8;
  const int tpr = 1 << tpr_log2;
  const int rpg = 256 >> tpr_log2;
  const int tx = threadIdx.x & (tpr - 1);
  const int64_t total = p.batch * p.rows_out;
  const int vpr = static_cast<int>((p.cols + 7) / 8);
  const bool full_tail = (p.cols % 8) == 0;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * rpg + (threadIdx.x >> tpr_log2); row < total;
       row += static_cast<int64_t>(gridDim.x) * rpg) {
    const int64_t b = row / p.rows_out;
    const int64_t t = row - b * p.rows_out;
    uint16_t* dst = p.dst + row * p.dst_ld;
    const uint16_t* src = nullptr;
    if (t < p.k) {
      const int64_t j = __ldg(p.idx + b * p.k + t);
      const int64_t item = (b / p.g_outer) * p.s_outer + ((b % p.g_outer) / p.g_inner) * p.s_inner;
      src = p.src + item + j * p.src_ld;
    }
    for (int c0 = tx; c0 < vpr; c0 += tpr * ILP) {
      uint4 v[ILP];
#pragma unroll
      for (int u = 0; u < ILP; ++u) {
        const int c = c0 + u * tpr;
        v[u] = make_uint4(0u, 0u, 0u, 0u);
        if (src != nullptr && c < vpr) {
          if (full_tail || c + 1 < vpr) {
            v[u] = ldg_nc_v4(src + c * 8);
          } else {
            uint32_t w[4] = {0u, 0u, 0u, 0u};
            for (int e = 0; c * 8 + e < p.cols; ++e)
              w[e >> 1] |= static_cast<uint32_t>(__ldg(src + c * 8 + e)) << (16 * (e & 1));
            v[u] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < ILP; ++u) {
        const int c = c0 + u * tpr;
        if (c < vpr) *reinterpret_cast<uint4*>(dst + c * 8) = v[u];
      }
    }
  }
}

// Row pack by bulk copies: rows of 16-byte multiples, every row kept
// (rows_out == k).  Each CTA owns a contiguous range of at most
// kRowpackMaxRows packed rows and copies them in chunks of at most
// kRowpackChunk bytes: a 1-D bulk load into a ring slot of shared memory, then
// a 1-D bulk store from that slot to the packed matrix, kRowpackStages - 1
// loads in flight while the stores drain.  The CTA's row indices are staged in
// shared memory first and one thread walks the chunks with an incremental
// cursor, so issuing a copy costs a few instructions and no memory round trip.
constexpr int kRowpackStages = 6;
constexpr uint32_t kRowpackChunk = 16384;
constexpr int64_t kRowpackMaxRows = 2048;

struct RowpackCursor {
  int64_t local;   // packed row within this CTA's range
  int64_t b, t;    // batch item, row within it
  int c;           // chunk within the row
  const uint16_t* item;
  __device__ void set_item(const RowPackParams& p) {
    item = p.src + (b / p.g_outer) * p.s_outer + ((b % p.g_outer) / p.g_inner) * p.s_inner;
  }
  __device__ void next(const RowPackParams& p, int chunks) {
    if (++c < chunks) return;
    c = 0;
    ++local;
    if (++t == p.k) {
      t = 0;
      ++b;
      set_item(p);
    }
  }
};

__global__ void __launch_bounds__(32) pack_rows_bulk_copy_kernel(const RowPackParams p, int chunks) {
  extern __shared__ __align__(128) uint8_t rp_smem[];
  __shared__ uint64_t full[kRowpackStages];
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;
  int32_t* s_rows = reinterpret_cast<int32_t*>(rp_smem + kRowpackStages * kRowpackChunk);
  const int64_t total = p.batch * p.k;
  const int64_t per = (total + gridDim.x - 1) / gridDim.x;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * per;
  int64_t r1 = r0 + per;
  if (r1 > total) r1 = total;
  if (r0 >= r1) return;  // uniform over the CTA
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRowpackStages; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  wait_prior_kernels();
  for (int64_t r = threadIdx.x; r < r1 - r0; r += 32) s_rows[r] = __ldg(p.idx + r0 + r);
  __syncthreads();
  if (threadIdx.x != 0) return;

  const int64_t n = (r1 - r0) * chunks;
  const int64_t chunk_elems = kRowpackChunk / 2;
  const uint32_t last_bytes = static_cast<uint32_t>(p.cols * 2 - static_cast<int64_t>(chunks - 1) * kRowpackChunk);
  RowpackCursor ld{0, r0 / p.k, r0 % p.k, 0, nullptr};
  ld.set_item(p);
  RowpackCursor st = ld;
  auto load = [&](int64_t q) {
    const uint32_t bytes = (ld.c == chunks - 1) ? last_bytes : kRowpackChunk;
    const uint16_t* src = ld.item + static_cast<int64_t>(s_rows[ld.local]) * p.src_ld + ld.c * chunk_elems;
    uint64_t* bar = &full[q % kRowpackStages];
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load_1d(rp_smem + (q % kRowpackStages) * kRowpackChunk, src, bytes, bar);
    ld.next(p, chunks);
  };
  int64_t loaded = 0;
  while (loaded < kRowpackStages && loaded < n) load(loaded++);
  for (int64_t q = 0; q < n; ++q) {
    const int s = static_cast<int>(q % kRowpackStages);
    if (!mbar_wait(&full[s], static_cast<uint32_t>((q / kRowpackStages) & 1), abort_flag, kDevErrTimeoutProducer)) break;
    const uint32_t bytes = (st.c == chunks - 1) ? last_bytes : kRowpackChunk;
    uint16_t* dst = p.dst + (st.b * p.rows_out + st.t) * p.dst_ld + st.c * chunk_elems;
    bulk_store_1d(dst, rp_smem + s * kRowpackChunk, bytes);
    bulk_commit_group();
    st.next(p, chunks);
    if (q >= 1 && loaded < n) {
      bulk_wait_group_read<1>();  // the store of chunk q - 1 has left its slot
      load(loaded++);             // chunk q - 1 + kRowpackStages into that slot
    }
  }
  bulk_wait_group<0>();
  if (*abort_flag) {
    // wait (bounded) for the loads already issued so none lands after exit
    for (int s = 0; s < kRowpackStages; ++s) {
      const int64_t uses = (loaded + kRowpackStages - 1 - s) / kRowpackStages;
      if (uses == 0) continue;
      const uint32_t a = smem_u32(&full[s]);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(a, static_cast<uint32_t>((uses - 1) & 1)) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  }
}

// Masked copy: the dropped contraction terms set to zero instead of skipped.
// For QK^T (keep indexes the columns of Q_h: head-feature dims) and PV (keep
// indexes the rows of V_g(h): token positions) the product is bound by writing
// S or reading P, so skipping the dropped terms saves no time; zeroing them
// gives exactly sum_{j in I} A[:, j] B[j, :] with no packed copies.
//   dst[b][r, c] = keep_b[by_rows ? r : c] ? src_item(b)[r, c] : 0
struct MaskParams {
  const uint16_t* src;
  uint16_t* dst;
  int64_t rows, cols;                          // per batch item (cols % 8 == 0)
  const uint8_t* keep;                         // [batch][by_rows ? rows : cols]
  int by_rows;
  int64_t batch;
  int64_t g_outer, g_inner, s_outer, s_inner;  // source item of b (as in PackParams)
};

// One batch item per blockIdx.y; inside an item each thread walks the 16-byte
// vectors v, v + stride, ... with an incremental (row, column) cursor, so the
// loop carries no divisions.
__global__ void __launch_bounds__(256) mask_copy_kernel(const MaskParams p) {
  wait_prior_kernels();
  constexpr int ILP = 4;
  const int64_t b = blockIdx.y;
  const int64_t vpr = p.cols / 8;
  const int64_t per_item = p.rows * vpr;
  const uint8_t* kb = p.keep + b * (p.by_rows ? p.rows : p.cols);
  const uint16_t* src = p.src + (b / p.g_outer) * p.s_outer + ((b % p.g_outer) / p.g_inner) * p.s_inner;
  uint16_t* dst = p.dst + b * per_item * 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t srow = stride / vpr;
  const int64_t scol = stride - srow * vpr;
  int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  int64_t row = v / vpr;
  int64_t col = v - row * vpr;
  while (v < per_item) {
    uint4 val[ILP];
    int64_t off[ILP];
#pragma unroll
    for (int u = 0; u < ILP; ++u) {
      off[u] = -1;
      val[u] = make_uint4(0u, 0u, 0u, 0u);
      if (v < per_item) {
        off[u] = v * 8;
        const uint16_t* sp = src + row * p.cols + col * 8;
        if (p.by_rows) {
          if (__ldg(kb + row)) val[u] = ldg_nc_v4(sp);
        } else {
          const uint2 kk = *reinterpret_cast<const uint2*>(kb + col * 8);  // eight keep bytes
          if (kk.x | kk.y) {
            const uint4 x = ldg_nc_v4(sp);
            const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
            const uint32_t ks[2] = {kk.x, kk.y};
            uint32_t o[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const uint32_t kw = ks[h >> 1] >> (16 * (h & 1));  // keep bytes of elements 2h, 2h+1
              const uint32_t m = ((kw & 0xFFu) ? 0x0000FFFFu : 0u) | ((kw & 0xFF00u) ? 0xFFFF0000u : 0u);
              o[h] = xs[h] & m;
            }
            val[u] = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
      v += stride;
      row += srow;
      col += scol;
      if (col >= vpr) {
        col -= vpr;
        ++row;
      }
    }
#pragma unroll
    for (int u = 0; u < ILP; ++u)
      if (off[u] >= 0) *reinterpret_cast<uint4*>(dst + off[u]) = val[u];
  }
}

}  // namespace rmm
