// Decode-shaped reduced product with int8 weights (n <= 8 activation rows):
//   Y[n x m] = (x[:, I] . Wq[I, :]) * scale[None, :]
// ("Reduced Matrix Multiplication ... Technical Summary", Compatibility: the
// method works with INT8 weight quantization; "Algorithm Deep-Dive: RMM",
// Compatibility & generalization: INT8 + RMM stack).  Only the k kept rows of
// Wq are read, one byte per weight: half the bytes of the bf16 path again.
//
// CUDA cores: each thread owns 8 consecutive output columns and streams the
// 8-byte int8 run of every kept row of its CTA's row chunk (the CTA's 256
// threads read 2 KB contiguous of each row), 16 rows in flight per thread.
// An int8 value b becomes float exactly as (2^23 + (b + 128)) - (2^23 + 128):
// the byte b ^ 0x80 is placed in the low mantissa byte of 2^23 with one byte
// permute, then one subtraction.  Conversion and products run on packed fp32
// pairs (two columns per instruction); accumulation is fp32.  CTAs split
// the kept rows into chunks and write fp32 partial sums, which
// gemv_i8_fixup_kernel adds in chunk order and scales (deterministic).  The
// kept activations x[:, I] are read through the index set while a CTA stages
// its row chunk, so the call needs no separate pack of x.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "gemv.cuh"

namespace rmm {

constexpr int kI8MaxChunk = 512;  // kept rows per CTA (a multiple of 16)
constexpr int kI8MaxRows = 8;     // activation rows

struct GemvI8Params {
  const int8_t* W;     // [d][ldw] int8
  int64_t ldw;
  const uint16_t* x;   // bf16 [n][ldx], all d columns: the kept ones are read through idx
  int64_t ldx;
  const int32_t* idx;  // [k] kept rows, or null for rows [0, k)
  int k, m, n;
  int chunk, chunks;
  float* partial;      // [chunks][n][m]
};

__device__ __forceinline__ uint2 ldg_nc_u2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// Packed fp32 pairs (sm_100): two columns per 64-bit register, one instruction.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  return static_cast<uint64_t>(__float_as_uint(lo)) | (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ void f2_fma(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// eight signed bytes -> four exact float pairs: the biased byte b ^ 0x80 goes
// into the low mantissa byte of 2^23, then 2^23 + 128 is subtracted from both
// halves of a pair at once
__device__ __forceinline__ void i8x8_to_f2(uint2 v, uint64_t (&f)[4]) {
  const uint64_t bias = f2_pack(-8388736.0f, -8388736.0f);
  const uint32_t w[2] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t u = w[i >> 1];
    const uint32_t sel = 0x7540u + static_cast<uint32_t>((i & 1) * 2);
    const uint32_t lo = __byte_perm(u, 0x4B000000u, sel);
    const uint32_t hi = __byte_perm(u, 0x4B000000u, sel + 1);
    f[i] = f2_add(static_cast<uint64_t>(lo) | (static_cast<uint64_t>(hi) << 32), bias);
  }
}

// grid (ceil(m / 2048), chunks), 256 threads
template <int NR>
__global__ void __launch_bounds__(256, (NR == 1) ? 4 : ((NR == 2) ? 3 : 2)) gemv_i8_kernel(const GemvI8Params p) {
  constexpr int U = (NR >= 8) ? 8 : 16;  // kept rows in flight per thread
  __shared__ uint64_t xs[NR][kI8MaxChunk];  // x value of row r at kept row i, duplicated into a pair
  __shared__ int rows[kI8MaxChunk];
  wait_prior_kernels();
  const int t0 = blockIdx.y * p.chunk;
  const int cnt = (p.k - t0) < p.chunk ? (p.k - t0) : p.chunk;
  const int cnt16 = (cnt + 15) & ~15;  // <= chunk <= kI8MaxChunk: the tail reads zeros
  for (int i = threadIdx.x; i < cnt16; i += blockDim.x) {
    const bool in = i < cnt;
    const int row = in ? (p.idx ? __ldg(p.idx + t0 + i) : t0 + i) : 0;
    rows[i] = row;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const float xv = (in && r < p.n) ? bf16lo(static_cast<uint32_t>(__ldg(p.x + r * p.ldx + row))) : 0.f;
      xs[r][i] = f2_pack(xv, xv);
    }
  }
  __syncthreads();
  const int64_t col0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (col0 >= p.m) return;
  uint64_t acc[NR][4];
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[r][e] = 0ull;
  const int8_t* wb = p.W + col0;
  for (int i0 = 0; i0 < cnt; i0 += U) {
    uint2 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      v[u] = (i0 + u < cnt) ? ldg_nc_u2(wb + static_cast<int64_t>(rows[i0 + u]) * p.ldw) : make_uint2(0u, 0u);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      uint64_t f[4];
      i8x8_to_f2(v[u], f);
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        const uint64_t xv = xs[r][i0 + u];
#pragma unroll
        for (int e = 0; e < 4; ++e) f2_fma(acc[r][e], xv, f[e]);
      }
    }
  }
  float* out = p.partial + static_cast<int64_t>(blockIdx.y) * p.n * p.m + col0;
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    if (r >= p.n) break;
    uint4* o = reinterpret_cast<uint4*>(out + static_cast<int64_t>(r) * p.m);
    o[0] = make_uint4(static_cast<uint32_t>(acc[r][0]), static_cast<uint32_t>(acc[r][0] >> 32),
                      static_cast<uint32_t>(acc[r][1]), static_cast<uint32_t>(acc[r][1] >> 32));
    o[1] = make_uint4(static_cast<uint32_t>(acc[r][2]), static_cast<uint32_t>(acc[r][2] >> 32),
                      static_cast<uint32_t>(acc[r][3]), static_cast<uint32_t>(acc[r][3] >> 32));
  }
}

// Y[r][c] = bf16(scale[c] * sum over chunks, in order, of the partials); grid
// (ceil(m / 256), n).
__global__ void __launch_bounds__(256) gemv_i8_fixup_kernel(const float* partial, const float* scale, int chunks, int n,
                                                           int m, uint16_t* Y, int64_t ldy) {
  wait_prior_kernels();
  const int col = blockIdx.x * blockDim.x + threadIdx.x;
  const int r = blockIdx.y;
  if (col >= m) return;
  float s = 0.f;
  for (int c = 0; c < chunks; ++c) s += partial[(static_cast<int64_t>(c) * n + r) * m + col];
  const __nv_bfloat16 b = __float2bfloat16_rn(s * __ldg(scale + col));
  Y[static_cast<int64_t>(r) * ldy + col] = *reinterpret_cast<const uint16_t*>(&b);
}

// ---------------------------------------------------------------- tensor cores
// The same reduced product for up to 32 activation rows on the tensor cores:
// the bf16 decode product's structure (gemv_kernel: stream-K over 512-column
// super tiles x 64-row k-blocks, swapped operands, M = 128 weight columns and N =
// 16 / 32 activation rows, fp32 partials added in CTA order by gemv_fixup_kernel,
// which also applies the per-column scale), with a dequantising producer: eight
// warps load the kept int8 rows with 16-byte loads into registers (a warp
// instruction covers one row's 512-byte run), one k-block ahead, convert them
// exactly to bf16 (an int8 value has at most 8 significant bits; the float trick
// above, then the upper halves of two floats packed as a bf16 pair) and store
// them into the 128-byte-swizzled MN-major stage of the bf16 kernel.  The kept
// activations x[:, I] (packed, bf16) come by TMA as in the bf16 kernel.
// 416 threads: warps 0-7 producers, warp 8 MMA, warps 9-12 epilogue.
struct GemvI8TcParams {
  const int8_t* W;     // [d][ldw] int8
  int64_t ldw;
  const int32_t* idx;  // [k] kept rows, ascending, or null for rows [0, k)
  int k, m, n;
  int m_super, kb_total;
  int64_t units;
  float* partial;      // [m_super + gridDim.x][4][n][128]
};

constexpr int kI8TcProducerWarps = 16;
constexpr int kI8TcThreads = (kI8TcProducerWarps + 5) * 32;

// sixteen int8 (one 16-byte load) -> sixteen bf16 (two 16-byte words)
__device__ __forceinline__ void i8x16_to_bf16(uint4 v, uint4& lo, uint4& hi) {
  uint64_t f0[4], f1[4];
  i8x8_to_f2(make_uint2(v.x, v.y), f0);
  i8x8_to_f2(make_uint2(v.z, v.w), f1);
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // bf16 = the upper half of the (exact) float
    b[i] = __byte_perm(static_cast<uint32_t>(f0[i]), static_cast<uint32_t>(f0[i] >> 32), 0x7632);
    b[4 + i] = __byte_perm(static_cast<uint32_t>(f1[i]), static_cast<uint32_t>(f1[i] >> 32), 0x7632);
  }
  lo = make_uint4(b[0], b[1], b[2], b[3]);
  hi = make_uint4(b[4], b[5], b[6], b[7]);
}

template <int N>
__global__ void __launch_bounds__(kI8TcThreads, 1)
    gemv_i8tc_kernel(const __grid_constant__ CUtensorMap tmX, const GemvI8TcParams p) {
  constexpr int A_BYTES = kGemvCols * 64 * 2;  // 64 kept rows x 512 columns, bf16
  constexpr int X_BYTES = N * 64 * 2;
  constexpr uint32_t IDESC = make_idesc_bf16(128, N, 1, 0);
  constexpr uint32_t ACC_COLS = kGemvTiles * N;
  constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
  constexpr int PW = kI8TcProducerWarps;
  constexpr int RPW = 64 / PW;  // kept rows per producer warp and k-block

  extern __shared__ uint8_t gvi_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gvi_raw) + 1023) & ~uintptr_t(1023));
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
      mbar_init(&full[s], PW + 1);  // the producer warps + the x tile's expect_tx
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
  if (warp == PW) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  wait_prior_kernels();

  const int64_t G = gridDim.x;
  const int64_t u_begin = gemv_unit_begin(blockIdx.x, p.units, G);
  const int64_t u_end = gemv_unit_begin(blockIdx.x + 1, p.units, G);

  if (warp < PW) {
    // ------------------------------------------------------------ producers
    // lane l covers columns [16 l, 16 l + 16) of the super tile: MMA tile l / 8,
    // 64-column atom (l / 4) % 2, 16-byte bf16 chunks 2 (l % 4) and 2 (l % 4) + 1.
    // Lanes of the odd atom store their two chunks in the other order, so each
    // group of 8 lanes writes 8 different 16-byte bank groups per store.
    const int c16 = lane * 16;
    const int tile = lane >> 3, atom = (lane >> 2) & 1, cw = (lane & 3) * 2;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    auto rows_of = [&](int64_t u, int (&dst)[RPW]) {
      const int kb = static_cast<int>(u % p.kb_total);
#pragma unroll
      for (int j = 0; j < RPW; ++j) {
        const int t = kb * 64 + warp * RPW + j;
        dst[j] = (u < u_end && t < p.k) ? (p.idx != nullptr ? __ldg(p.idx + t) : t) : -1;
      }
    };
    // a row starts 16-byte aligned only when the row stride is a multiple of 16
    // bytes (the interface promises 8): otherwise two 8-byte loads per chunk
    const bool rows16 = (p.ldw & 15) == 0;
    auto load_row = [&](int64_t u, int row) -> uint4 {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      const int col = static_cast<int>(u / p.kb_total) * kGemvCols + c16;
      if (u < u_end && row >= 0 && col < p.m) {
        const int8_t* src = p.W + static_cast<int64_t>(row) * p.ldw + col;
        if (col + 16 <= p.m) {
          if (rows16) {
            v = ldg_nc_v4(src);
          } else {
            const uint2 a = ldg_nc_u2(src), b = ldg_nc_u2(src + 8);
            v = make_uint4(a.x, a.y, b.x, b.y);
          }
        } else {  // m is a multiple of 8: the last chunk may hold 8 columns
          const uint2 h = ldg_nc_u2(src);
          v = make_uint4(h.x, h.y, 0u, 0u);
        }
      }
      return v;
    };
    // Two units of kept rows in flight per thread (buf[0] and buf[1], 64 KB of
    // int8 per CTA): a row is converted and stored, then its register is
    // reloaded at once with the same row of the unit two ahead.  Row numbers are
    // loaded one unit before their data.
    uint4 buf[2][RPW];
    int rows_next[RPW];
    rows_of(u_begin, rows_next);
#pragma unroll
    for (int j = 0; j < RPW; ++j) buf[0][j] = load_row(u_begin, rows_next[j]);
    rows_of(u_begin + 1, rows_next);
#pragma unroll
    for (int j = 0; j < RPW; ++j) buf[1][j] = load_row(u_begin + 1, rows_next[j]);
    rows_of(u_begin + 2, rows_next);
    for (int64_t u0 = u_begin; u0 < u_end && ok; u0 += 2) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int64_t u = u0 + hh;
        if (u >= u_end) break;
        const int kb = static_cast<int>(u % p.kb_total);
        int go = 1;
        if (lane == 0) go = mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kDevErrTimeoutProducer) ? 1 : 0;
        go = __shfl_sync(0xffffffffu, go, 0);
        if (!go) {
          ok = false;
          break;
        }
        if (threadIdx.x == 0) {
          mbar_arrive_expect_tx(&full[stage], X_BYTES);
          tma_load_2d(sX + stage * X_BYTES, &tmX, &full[stage], kb * 64, 0);
        }
        uint8_t* dst = sA + stage * A_BYTES + tile * 16384 + atom * 8192;
#pragma unroll
        for (int j = 0; j < RPW; ++j) {
          const int r = warp * RPW + j;  // kept row within the k-block
          uint4 lo, hi;
          i8x16_to_bf16(buf[hh][j], lo, hi);
          buf[hh][j] = load_row(u + 2, rows_next[j]);
          const uint4 first = atom ? hi : lo, second = atom ? lo : hi;
          *reinterpret_cast<uint4*>(dst + r * 128 + (((cw + atom) ^ (r & 7)) << 4)) = first;
          *reinterpret_cast<uint4*>(dst + r * 128 + (((cw + 1 - atom) ^ (r & 7)) << 4)) = second;
        }
        rows_of(u + 3, rows_next);
        // no proxy fence here: it would wait for this thread's loads still in flight
        // (two units ahead); the MMA thread fences after its wait instead
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);  // release: the warp's stores, ordered by the syncwarp
        if (++stage == kGemvStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    (void)ok;
  } else if (warp == PW) {
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
          // the producers' generic-proxy stores (acquired through the barrier) are
          // ordered before the MMA's async-proxy reads of the stage
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
    // ------------------------------------------------------------ epilogue (one MMA tile at a time)
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
      float* part = p.partial + (static_cast<int64_t>(sup) + blockIdx.x) * kGemvTiles * p.n * 128;
#pragma unroll 1
      for (int tl = 0; tl < kGemvTiles; ++tl) {
        float v[N];
        tmem_ld_cols<N>(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc) * ACC_COLS +
                            static_cast<uint32_t>(tl * N),
                        v);
        tmem_ld_wait();
#pragma unroll
        for (int rr = 0; rr < N; ++rr)
          if (rr < p.n) part[(tl * p.n + rr) * 128 + col_in_tile] = v[rr];
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      ++seg;
      u = seg_end;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == PW) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace rmm
