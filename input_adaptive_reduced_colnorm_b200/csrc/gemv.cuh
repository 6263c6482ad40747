// Decode-shaped reduced product (n <= 32 activation rows):
//   Y[n x m] = x[:, I] . W[I, :]        ("Algorithm Deep-Dive: RMM", Core
//   Approach, applied to a linear projection at decode time)
// It is bound by HBM reads of the k kept weight rows (k * m * 2 bytes), so only
// those rows are read, once, straight from W -- no packed copy of W[I, :].
//
// Tensor cores with the operands swapped: D[128 weight columns x N rows] =
// W_I^T (M = 128, MN-major) . x_I^T (N = 16 or 32, K-major), fp32 accumulators
// in tensor memory, four of them (one per 128-column tile of a super tile).
//   warps 0-3  producers: each CTA works on a 512-column super tile, so every
//              kept row contributes one contiguous 1 KB run per stage (runs of
//              256 B per row reached only ~40% of HBM bandwidth); the runs are
//              loaded with 16-byte cp.async straight into the 128-byte-swizzled
//              MN-major operand layout (a TMA row gather stages only ~7 B/clk/SM
//              on B200, 16-byte cp.async ~35 B/clk/SM); two threads per kept
//              row, the next row number prefetched one stage ahead; thread 0
//              also brings the packed activations x_I with a TMA tile.  A
//              producer never waits for its own copies: cp.async.mbarrier.arrive
//              counts the thread on the stage's full barrier once its copies have
//              landed, so all three 64 KB stages can be in flight, and the MMA
//              thread fences the async proxy after its wait.  (The first version
//              waited for its copies two stages back and fenced in the producers;
//              the fence also waits for the copies still in flight, and the
//              kernel streamed 0.79 of the copy bandwidth instead of 0.92.)
//   warp 4     allocates TMEM; one thread issues tcgen05.mma (M=128, N, K=16).
//   warps 5-8  epilogue: tcgen05.ld -> fp32 partial sums in global memory.
// Work split (stream-K): the (super tile, 64-row k-block) units are cut into
// one contiguous range per CTA; a CTA writes one partial super tile per super
// tile it touches, into slot (super tile + cta), and gemv_fixup_kernel adds the
// partials of each column in CTA order, so the result is deterministic.  (Adding
// them in the last CTA of each super tile, behind an arrival counter, was
// measured slower: 128 epilogue threads cannot keep enough partial loads in
// flight once n >= 8.)
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace rmm {

struct GemvParams {
  const uint16_t* W;   // [d][ldw] bf16
  int64_t ldw;
  const int32_t* idx;  // [k] kept rows, ascending, or null for rows [0, k)
  int k;
  int m;               // columns of W and Y
  int n;               // rows of x and Y (<= N)
  int m_super;         // ceil(m / 512): 512-column super tiles (four 128-column MMA tiles)
  int kb_total;        // ceil(k / 64)
  int64_t units;       // m_super * kb_total
  float* partial;      // [m_super + gridDim.x][4][n][128]
};

// Owners of the units of super tile `sup`: CTAs c_lo..c_hi (each with at least
// one unit when the grid does not exceed the unit count).  ``fn(c)`` is called
// for every CTA that touched the super tile, in increasing c.
template <typename F>
__device__ __forceinline__ void gemv_for_each_owner(const GemvParams& p, int64_t G, int sup, F&& fn) {
  const int64_t U = p.units;
  const int64_t u_lo = static_cast<int64_t>(sup) * p.kb_total;
  const int64_t u_hi = u_lo + p.kb_total - 1;
  if ((U + 1) * G < (1LL << 32)) {
    // the unit split in 32-bit unsigned arithmetic (the usual case; much cheaper
    // than 64-bit division)
    const uint32_t u32 = static_cast<uint32_t>(U), g32 = static_cast<uint32_t>(G);
    const uint32_t c_lo = (static_cast<uint32_t>(u_lo + 1) * g32 - 1u) / u32;  // owner of unit u_lo
    const uint32_t c_hi = (static_cast<uint32_t>(u_hi + 1) * g32 - 1u) / u32;  // owner of unit u_hi
    uint32_t start_c = (c_lo * u32) / g32;
    for (uint32_t c = c_lo; c <= c_hi; ++c) {
      const uint32_t start_next = ((c + 1u) * u32) / g32;
      if (start_next > start_c) fn(static_cast<int64_t>(c));  // CTA c had at least one unit
      start_c = start_next;
    }
  } else {
    const int64_t c_lo = ((u_lo + 1) * G - 1) / U;
    const int64_t c_hi = ((u_hi + 1) * G - 1) / U;
    int64_t start_c = (c_lo * U) / G;
    for (int64_t c = c_lo; c <= c_hi; ++c) {
      const int64_t start_next = ((c + 1) * U) / G;
      if (start_next > start_c) fn(c);
      start_c = start_next;
    }
  }
}

constexpr int kGemvTiles = 4;                  // 128-column MMA tiles per super tile
constexpr int kGemvCols = 128 * kGemvTiles;    // 512 columns = 1 KB of each kept row per stage
constexpr int kGemvStages = 3;

__device__ __forceinline__ int64_t gemv_unit_begin(int64_t c, int64_t units, int64_t G) { return (c * units) / G; }

__device__ __forceinline__ void cp_async16_z(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
// arrive on `bar` once every cp.async this thread issued so far has landed (the
// arrival is one of the barrier's expected count)
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns (thread t: row lane_base + t).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// exactly N (16 or 32) accumulator columns of this warp's 32 lanes
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[N]) {
  static_assert(N == 16 || N == 32, "N must be 16 or 32");
  if constexpr (N == 16) {
    uint32_t r[16];
    tmem_ld16(taddr, r);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
  } else {
    uint32_t r[32];
    tmem_ld32(taddr, r);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  }
}

__device__ __forceinline__ int gemv_row_of(const GemvParams& p, int t) {
  if (t >= p.k) return -1;
  return (p.idx != nullptr) ? __ldg(p.idx + t) : t;
}

template <int N>
__global__ void __launch_bounds__(288, 1) gemv_kernel(const __grid_constant__ CUtensorMap tmX, const GemvParams p) {
  constexpr int A_BYTES = kGemvCols * 64 * 2;  // 64 kept rows x 512 columns
  constexpr int X_BYTES = N * 64 * 2;
  constexpr uint32_t IDESC = make_idesc_bf16(128, N, 1, 0);
  constexpr uint32_t ACC_COLS = kGemvTiles * N;  // one accumulator = four N-column tiles
  constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;   // double-buffered (128 or 256 columns)

  extern __shared__ uint8_t gv_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gv_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sX = smem + kGemvStages * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sX + kGemvStages * X_BYTES);
  uint64_t* empty = full + kGemvStages;
  uint64_t* tfull = empty + kGemvStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemvStages; ++s) {
      mbar_init(&full[s], 128 + 1);  // 128 producer arrivals + the TMA issuer's expect_tx
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmX);
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  wait_prior_kernels();  // operands and partials are touched only after this

  const int64_t G = gridDim.x;
  const int64_t u_begin = gemv_unit_begin(blockIdx.x, p.units, G);
  const int64_t u_end = gemv_unit_begin(blockIdx.x + 1, p.units, G);

  if (warp < 4) {
    // ------------------------------------------------------------ producers
    // warp w copies kept rows 16w .. 16w+15 of the k-block; each warp instruction
    // moves 512 contiguous bytes of one row (lane = 16-byte chunk).  Every lane
    // holds the warp's 16 row numbers in registers, loaded one stage ahead
    // (same-address loads, no cross-lane traffic between the copies).
    const int tid = threadIdx.x;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int rows_next[16];
    if (u_begin < u_end) {
      const int t0 = static_cast<int>(u_begin % p.kb_total) * 64 + warp * 16;
#pragma unroll
      for (int q = 0; q < 16; ++q) rows_next[q] = gemv_row_of(p, t0 + q);
    }
    for (int64_t u = u_begin; u < u_end; ++u) {
      const int sup = static_cast<int>(u / p.kb_total);
      const int kb = static_cast<int>(u - static_cast<int64_t>(sup) * p.kb_total);
      int rows[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) rows[q] = rows_next[q];
      if (u + 1 < u_end) {
        const int t0 = static_cast<int>((u + 1) % p.kb_total) * 64 + warp * 16;
#pragma unroll
        for (int q = 0; q < 16; ++q) rows_next[q] = gemv_row_of(p, t0 + q);
      }
      // one lane per warp waits, so the warp leaves the loop together
      int go = 1;
      if (lane == 0) go = mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kDevErrTimeoutProducer) ? 1 : 0;
      go = __shfl_sync(0xffffffffu, go, 0);
      if (!go) {
        ok = false;
        break;
      }
      if (tid == 0) {
        mbar_arrive_expect_tx(&full[stage], X_BYTES);
        tma_load_2d(sX + stage * X_BYTES, &tmX, &full[stage], kb * 64, 0);
      }
      uint8_t* dstA = sA + stage * A_BYTES;
      const int col_base = sup * kGemvCols;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int r = warp * 16 + (j >> 1);   // kept row within the k-block
        const int64_t row = rows[j >> 1];
        const int c16 = (j & 1) * 32 + lane;  // 16-byte chunk within the 1 KB row segment
        const int tile = c16 >> 4;            // 128-column MMA tile
        const int a = (c16 >> 3) & 1;         // 64-column atom within the tile
        const int cw = c16 & 7;               // 16-byte column within the atom
        const int col = col_base + c16 * 8;
        const uint16_t* src = p.W;
        uint32_t bytes = 0;
        if (row >= 0 && col < p.m) {
          src = p.W + row * p.ldw + col;
          bytes = (col + 8 <= p.m) ? 16u : static_cast<uint32_t>((p.m - col) * 2);
        }
        cp_async16_z(dstA + tile * 16384 + a * 8192 + r * 128 + ((cw ^ (r & 7)) << 4), src, bytes);
      }
      cp_async_arrive_noinc(&full[stage]);
      if (++stage == kGemvStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    // nothing may land after exit (the abort path leaves copies in flight)
    cp_async_wait_all();
    (void)ok;
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int seg = 0;
      bool ok = true;
      int64_t u = u_begin;
      while (u < u_end && ok) {
        const int sup = static_cast<int>(u / p.kb_total);
        const int64_t sup_end = static_cast<int64_t>(sup + 1) * p.kb_total;
        const int64_t seg_end = u_end < sup_end ? u_end : sup_end;
        const int acc = seg & 1;
        if (!mbar_wait(&tempty[acc], ((seg >> 1) & 1) ^ 1u, abort_flag, kDevErrTimeoutMma)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * ACC_COLS;
        for (int64_t v = u; v < seg_end; ++v) {
          if (!mbar_wait(&full[stage], phase, abort_flag, kDevErrTimeoutMma)) {
            ok = false;
            break;
          }
          // the stage's cp.async writes (acquired through the barrier) are ordered
          // before the MMA's async-proxy reads
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
          const uint32_t x0 = smem_u32(sX + stage * X_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = make_sw128_desc(x0 + kk * 32, 16, 1024);
#pragma unroll
            for (int tl = 0; tl < kGemvTiles; ++tl) {
              const uint64_t ad = make_sw128_desc(a0 + tl * 16384 + kk * 2048, 8192, 1024);
              umma_bf16(d_tmem + static_cast<uint32_t>(tl * N), ad, bd, IDESC, (v != u || kk != 0) ? 1u : 0u);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == kGemvStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        ++seg;
        u = seg_end;
      }
      umma_commit(drain);
      const uint32_t a = smem_u32(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int col_in_tile = quarter * 32 + lane;
    int seg = 0;
    int64_t u = u_begin;
    while (u < u_end) {
      const int sup = static_cast<int>(u / p.kb_total);
      const int64_t sup_end = static_cast<int64_t>(sup + 1) * p.kb_total;
      const int64_t seg_end = u_end < sup_end ? u_end : sup_end;
      const int acc = seg & 1;
      if (!mbar_wait(&tfull[acc], (seg >> 1) & 1, abort_flag, kDevErrTimeoutEpilogue, 256)) break;
      tc_fence_after();
      float v[kGemvTiles][N];
#pragma unroll
      for (int tl = 0; tl < kGemvTiles; ++tl)
        tmem_ld_cols<N>(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc) * ACC_COLS +
                            static_cast<uint32_t>(tl * N),
                        v[tl]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      float* part = p.partial + (static_cast<int64_t>(sup) + blockIdx.x) * kGemvTiles * p.n * 128;
#pragma unroll
      for (int tl = 0; tl < kGemvTiles; ++tl)
#pragma unroll
        for (int rr = 0; rr < N; ++rr)
          if (rr < p.n) part[(tl * p.n + rr) * 128 + col_in_tile] = v[tl][rr];
      ++seg;
      u = seg_end;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// Y[r, col] = bf16( sum over the CTAs c that touched the column's super tile, in
// increasing c, of their partial sums ).  One CTA per (128-column MMA tile of a
// super tile, 4 rows): thread 0 lists the owning CTAs in shared memory once (at
// most grid + 1 of them: dynamic shared memory of (grid + 1) ints), then each
// thread adds the float4 partials of 4 columns of one row over the list
// (independent loads, summed in CTA order), times scale[col] when scale is given.
__global__ void __launch_bounds__(128) gemv_fixup_kernel(const GemvParams p, int grid, uint16_t* Y, int64_t ldy,
                                                         const float* scale) {
  extern __shared__ int s_own[];
  __shared__ int s_count;
  const int sup = blockIdx.x / kGemvTiles;
  const int tl = blockIdx.x % kGemvTiles;
  // the owner list depends only on the launch shape: built before the wait, while
  // the product kernel is still running
  if (threadIdx.x == 0) {
    int c_count = 0;
    gemv_for_each_owner(p, grid, sup, [&](int64_t c) { s_own[c_count++] = static_cast<int>(c); });
    s_count = c_count;
  }
  __syncthreads();
  wait_prior_kernels();
  const int count = s_count;
  const int i4 = (threadIdx.x & 31) * 4;
  const int r = blockIdx.y * 4 + (threadIdx.x >> 5);
  if (r >= p.n) return;
  const int64_t slot = static_cast<int64_t>(kGemvTiles) * p.n * 128;  // floats per partial super tile
  const float* src = p.partial + static_cast<int64_t>(sup) * slot + (static_cast<int64_t>(tl) * p.n + r) * 128 + i4;
  float ax = 0.f, ay = 0.f, az = 0.f, aw = 0.f;
  int q = 0;
  for (; q + 4 <= count; q += 4) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = *reinterpret_cast<const float4*>(src + static_cast<int64_t>(s_own[q + u]) * slot);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      ax += v[u].x;
      ay += v[u].y;
      az += v[u].z;
      aw += v[u].w;
    }
  }
  for (; q < count; ++q) {
    const float4 v = *reinterpret_cast<const float4*>(src + static_cast<int64_t>(s_own[q]) * slot);
    ax += v.x;
    ay += v.y;
    az += v.z;
    aw += v.w;
  }
  const int col = sup * kGemvCols + tl * 128 + i4;
  float a[4] = {ax, ay, az, aw};
  if (scale != nullptr) {  // int8 weights: one fp32 scale per output column
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (col + e < p.m) a[e] *= __ldg(scale + col + e);
  }
  uint16_t* y = Y + static_cast<int64_t>(r) * ldy + col;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (col + e < p.m) {
      const __nv_bfloat16 h = __float2bfloat16_rn(a[e]);
      y[e] = *reinterpret_cast<const uint16_t*>(&h);
    }
}

}  // namespace rmm
