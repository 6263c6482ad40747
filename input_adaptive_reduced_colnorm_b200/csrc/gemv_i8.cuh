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

}  // namespace rmm
