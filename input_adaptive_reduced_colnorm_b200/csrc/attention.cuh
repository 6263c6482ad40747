// Attention with a reduced score product, fused so that the scores S and the
// probabilities P never leave the SM ("Algorithm Deep-Dive: RMM", Component
// mapping: QK^T selects head dims by the Q column norm, K gathers them under
// GQA; Attention vs MLP, Table 16: attention-internal reduction):
//   S_h = scale * Q_h[:, I_h] K_g(h)[:, I_h]^T   (-inf above the causal diagonal)
//   O_h = softmax_rows(S_h) V_g(h)
// The index sets come from the column-norm and selection kernels.  For k <= 64
// the score product runs over 64 dims on Q[:, I_h] and K_g(h)[:, I_h] packed per
// query head (zero past k, kp = 64); otherwise it reads Q with the dropped dims of
// its head zeroed and K as it is (kp = 128).  Either way it is exactly
// sum_{t in I_h} Q_h[:, t] K_g(h)[:, t]^T.  The value product is the ordinary one
// (selecting P's columns would need all of P first).
//
// One CTA per (query head, pair of 128-row query tiles), see attn_pp_kernel:
//   warp 0       TMA: both Q tiles once, then 128-key blocks of K (K-major) and V
//                (MN-major, 128 dims) into two-stage rings.
//   warp 1       tensor memory (512 columns: S_A, S_B, O_A, O_B); lane 0 issues
//                S_t(j) = Q_t K(j)^T (M = N = 128, K = kp) and O_t += P_t(j) V(j)
//                (A = P_t from tensor memory, K = 128), alternating the tiles.
//   warps 2..17  softmax, two threads per query row (warps 2-9 tile A, 10-17
//                tile B; in each tile the first four warps take keys 0-63 of a
//                block, the next four keys 64-127): running max m and sum l in
//                log2 units, weights by ex2.approx (in the masked diagonal
//                blocks half of them by a fitted polynomial on the FMA pipe), P
//                written back as bf16 pairs into tensor memory, O rescaled there
//                when a row's maximum jumped; at the end O / l.
// Every wait is bounded (about one second); on a timeout the CTA records an
// error code, drains its copies, lets the MMA finish and returns.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace rmm {

struct AttnParams {
  int nq, nk;          // query / key rows of one head
  int kp;              // score dims staged per tile: 128 (Q with the dropped dims zeroed) or 64 (packed)
  int k_per_item;      // 1: K holds one packed copy per query head (rows item * nk ..), 0: per key head
  int hq, hkv;         // heads (GQA: query head h reads key/value head h / (hq / hkv))
  int items;           // batch * hq
  int m_tiles;         // ceil(nq / 128)
  int causal;
  int64_t causal_off;  // key j is visible to query i iff j <= i + causal_off
  float scale_log2;    // scale * log2(e)
  uint16_t* O;         // bf16 [items][nq][128]
};

constexpr int kAttnTile = 128;
constexpr uint32_t kAttnQBytes = 128 * 128 * 2;  // Q tile, up to 128 dims (two 64-dim atoms)
constexpr uint32_t kAttnKBytes = 128 * 128 * 2;  // one K block, up to 128 dims
constexpr uint32_t kAttnVBytes = 128 * 128 * 2;  // one V block: 2 key halves x 2 column atoms of 64 x 64

// 2^x with the hardware approximation (relative error ~2^-22; exp2(-inf) = 0).
__device__ __forceinline__ float attn_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (sm_100): two keys of a row per instruction.
__device__ __forceinline__ uint64_t attn_f2(float lo, float hi) {
  return static_cast<uint64_t>(__float_as_uint(lo)) | (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ float attn_lo(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float attn_hi(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ uint64_t attn_fma2(uint64_t a, uint64_t b, uint64_t c) {  // a * b + c
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t attn_add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t attn_sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// max(a, b, c) in one instruction (sm_100)
__device__ __forceinline__ float attn_max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// bf16 pair (lo in the low half), round to nearest
__device__ __forceinline__ uint32_t attn_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// 2^x on the FMA pipe for two arguments at once, for the share of the weights
// that does not go to the special-function unit.  x = n + f with n the nearest
// integer (x + 1.5 * 2^23 rounds it into the low mantissa bits) and f in
// [-1/2, 1/2]; 2^f from a cubic fitted here (relative-error minimax on
// [-1/2, 1/2], Remez exchange) with maximum relative error 7.49e-5, far below
// the bf16 rounding of P; n is added to the exponent field (one shift-add per
// value).  The bound holds for x in [-125, 0] (the fp32 evaluation adds a few
// 1e-7).  On [-126, -125) the sum can land in the subnormal range where n = -126
// and the cubic is below 1, and the relative error there reaches 1.5e-4.
// Arguments are clamped at -126, so anything smaller gives about 2^-126 (weights
// that small are 2^-125 of the row's largest weight, 1, and vanish next to it).
constexpr float kAttnExp2C0 = 0.99992805719f;
constexpr float kAttnExp2C1 = 0.69326096773f;
constexpr float kAttnExp2C2 = 0.24261112511f;
constexpr float kAttnExp2C3 = 0.05517166853f;

__device__ __forceinline__ uint64_t attn_exp2_poly2(uint64_t x) {
  const uint64_t xc = attn_f2(fmaxf(attn_lo(x), -126.f), fmaxf(attn_hi(x), -126.f));
  const uint64_t magic = attn_f2(12582912.f, 12582912.f);
  const uint64_t r = attn_add2(xc, magic);              // 1.5 * 2^23 + n
  const uint64_t f = attn_sub2(xc, attn_sub2(r, magic));  // x - n, exact
  uint64_t q = attn_fma2(attn_f2(kAttnExp2C3, kAttnExp2C3), f, attn_f2(kAttnExp2C2, kAttnExp2C2));
  q = attn_fma2(q, f, attn_f2(kAttnExp2C1, kAttnExp2C1));
  q = attn_fma2(q, f, attn_f2(kAttnExp2C0, kAttnExp2C0));
  // the low 9 bits of r hold n (two's complement): shifted into the exponent field
  const uint32_t lo = static_cast<uint32_t>(q) + (static_cast<uint32_t>(r) << 23);
  const uint32_t hi = static_cast<uint32_t>(q >> 32) + (static_cast<uint32_t>(r >> 32) << 23);
  return static_cast<uint64_t>(lo) | (static_cast<uint64_t>(hi) << 32);
}

// one argument (the masked blocks): the same arithmetic, the same result
__device__ __forceinline__ float attn_exp2_poly(float x) { return attn_lo(attn_exp2_poly2(attn_f2(x, x))); }

// Elementwise attn_exp2_poly and CUDA's exp2f, for the unit test of the fit
// (rmm_debug_exp2_poly).
__global__ void attn_exp2_probe_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                       float* __restrict__ y_ref, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = x[i];
    y_poly[i] = attn_exp2_poly(v);
    y_ref[i] = exp2f(v);
  }
}

// The softmax's reference maximum of a row moves only when the row's maximum
// exceeds it by more than this (log2 units), so the unnormalised weights stay
// below 2^8 = 256 (exact range for fp32 sums and bf16 P) and O is rescaled only
// on such jumps.  The result is the same softmax: O and l share the reference.
constexpr float kAttnRescaleLog2 = 8.f;

// Visible key blocks of the query tile starting at row m0.
__device__ __forceinline__ int attn_key_blocks(const AttnParams& p, int m0) {
  const int all = (p.nk + kAttnTile - 1) / kAttnTile;
  if (!p.causal) return all;
  int64_t last = static_cast<int64_t>(m0) + kAttnTile - 1;
  if (last > p.nq - 1) last = p.nq - 1;
  const int64_t lim = last + p.causal_off;  // last visible key of the tile
  const int nb = static_cast<int>(lim / kAttnTile) + 1;
  return nb < all ? nb : all;
}

}  // namespace rmm

namespace rmm {

// ---------------------------------------------------------------- two query tiles per CTA
// The same attention with two 128-row query tiles A and B of one head per CTA
// and two softmax warpgroups, so one tile's softmax runs while the tensor cores
// work on the other tile (320 threads: TMA warp, MMA warp, softmax warps 2-5 for
// A and 6-9 for B).  Tensor memory: S_A, S_B, O_A, O_B (128 columns each).  P(j)
// of a tile is written as packed bf16 pairs over the first 64 columns of its S
// region and the value MMA reads it from tensor memory (A operand in tensor
// memory), so shared memory holds only Q_A, Q_B and the K / V rings.  The MMAs of
// one thread execute in issue order: S_X(j+1) is issued after PV_X(j), so it
// cannot overwrite P_X(j) early, and the commit that signals S_X(j) also covers
// PV_X(j-1), which makes O_X safe to rescale.
constexpr int kAttnPPThreads = 18 * 32;  // TMA warp, MMA warp, 16 softmax warps
// row-max / row-sum exchange [2 bufs][tile][quarter][half][lane] floats, then the
// wait results [2 bufs][tile][quarter] ints (two per quarter, the first used)
constexpr int kAttnXchBytes = 2 * 2 * 4 * 2 * 32 * 4 + 2 * 2 * 4 * 2 * 4;
constexpr int kAttnPPSmem = 2 * kAttnQBytes + 2 * kAttnKBytes + 2 * kAttnVBytes + kAttnXchBytes + 1024 + 256;

// named barrier of the two warps that share a row quarter of a tile (64 threads)
__device__ __forceinline__ void attn_pair_sync(int id) { asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory"); }

__global__ void __launch_bounds__(kAttnPPThreads, 1)
    attn_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  extern __shared__ uint8_t app_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(app_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                    // [2 tiles][kAttnQBytes]
  uint8_t* sK = sQ + 2 * kAttnQBytes;    // [2 stages]
  uint8_t* sV = sK + 2 * kAttnKBytes;    // [2 stages]
  float* s_xch = reinterpret_cast<float*>(sV + 2 * kAttnVBytes);  // kAttnXchBytes
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + 2 * kAttnVBytes + kAttnXchBytes);
  uint64_t* q_full = bars;        // 1
  uint64_t* k_full = bars + 1;    // 2 (stages)
  uint64_t* k_empty = bars + 3;   // 2
  uint64_t* v_full = bars + 5;    // 2
  uint64_t* v_empty = bars + 7;   // 2
  uint64_t* s_full = bars + 9;    // 2 (tiles)
  uint64_t* p_full = bars + 11;   // 2 (tiles)
  uint64_t* pv_done = bars + 13;  // 2 (tiles): the last value product
  uint64_t* drain = bars + 15;    // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pairs = (p.m_tiles + 1) / 2;
  const int item = static_cast<int>(blockIdx.x % p.items);
  const int pt = pairs - 1 - static_cast<int>(blockIdx.x / p.items);  // heaviest causal pairs first
  const int m0 = pt * 2 * kAttnTile;
  const int b = item / p.hq, h = item % p.hq;
  const int g = h / (p.hq / p.hkv);
  int nkb_t[2];
  nkb_t[0] = attn_key_blocks(p, m0);
  nkb_t[1] = attn_key_blocks(p, m0 + kAttnTile < p.nq ? m0 + kAttnTile : m0);
  const int nkb = nkb_t[0] > nkb_t[1] ? nkb_t[0] : nkb_t[1];
  const int qrow0 = item * p.nq + m0;
  const int krow0 = (p.k_per_item ? item : b * p.hkv + g) * p.nk;
  const int vrow0 = (b * p.hkv + g) * p.nk;
  const uint32_t k_bytes = static_cast<uint32_t>(p.kp) * kAttnTile * 2;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 256);  // both softmax warpgroups of the tile
      mbar_init(&pv_done[s], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  wait_prior_kernels();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t k_issued = 0, v_issued = 0;
      bool ok = true;
      mbar_arrive_expect_tx(q_full, 2 * k_bytes);
      for (int t = 0; t < 2; ++t)
        for (int a = 0; a < p.kp / 64; ++a)
          tma_load_2d(sQ + t * kAttnQBytes + a * 16384, &tmQ, q_full, a * 64, qrow0 + t * kAttnTile);
      for (int j = 0; j < nkb && ok; ++j) {
        const int s = j & 1;
        const uint32_t use = static_cast<uint32_t>(j >> 1);
        if (!mbar_wait(&k_empty[s], (use & 1u) ^ 1u, abort_flag, kDevErrTimeoutProducer)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&k_full[s], k_bytes);
        for (int a = 0; a < p.kp / 64; ++a)
          tma_load_2d(sK + s * kAttnKBytes + a * 16384, &tmK, &k_full[s], a * 64, krow0 + j * kAttnTile);
        ++k_issued;
        if (!mbar_wait(&v_empty[s], (use & 1u) ^ 1u, abort_flag, kDevErrTimeoutProducer)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], kAttnVBytes);
        for (int kh = 0; kh < 2; ++kh)
          for (int a = 0; a < 2; ++a)
            tma_load_2d(sV + s * kAttnVBytes + kh * 16384 + a * 8192, &tmV, &v_full[s], a * 64,
                        vrow0 + j * kAttnTile + kh * 64);
        ++v_issued;
      }
      if (!ok) {
        // wait (bounded) for the copies this CTA issued so none lands after exit
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(smem_u32(q_full), 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
        }
        for (int s = 0; s < 2; ++s) {
          const uint32_t ku = (k_issued + 1 - s) / 2, vu = (v_issued + 1 - s) / 2;
          const uint64_t t1 = globaltimer_ns();
          if (ku)
            while (!mbar_try_wait(smem_u32(&k_full[s]), (ku - 1) & 1u) && globaltimer_ns() - t1 < kWaitTimeoutNs) {
            }
          const uint64_t t2 = globaltimer_ns();
          if (vu)
            while (!mbar_try_wait(smem_u32(&v_full[s]), (vu - 1) & 1u) && globaltimer_ns() - t2 < kWaitTimeoutNs) {
            }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, abort_flag, kDevErrTimeoutMma);
      const uint32_t idesc_s = make_idesc_bf16(128, 128, 0, 0);  // Q and K both K-major
      const uint32_t idesc_o = make_idesc_bf16(128, 128, 0, 1);  // P (tensor memory, K-major), V MN-major
      // S_t(j) = Q_t K(j)^T; the first user of K(j) waits for it, tile B (the last user) releases it
      auto issue_s = [&](int t, int j) -> bool {
        const int s = j & 1;
        const uint32_t use = static_cast<uint32_t>(j >> 1);
        const bool first = (t == 0) || (j >= nkb_t[0]);
        if (first && !mbar_wait(&k_full[s], use & 1u, abort_flag, kDevErrTimeoutMma)) return false;
        tc_fence_after();
        const uint32_t q0 = smem_u32(sQ + t * kAttnQBytes);
        const uint32_t k0 = smem_u32(sK + s * kAttnKBytes);
        for (int kk = 0; kk < p.kp / 16; ++kk) {
          const uint32_t off = static_cast<uint32_t>((kk >> 2) * 16384 + (kk & 3) * 32);
          umma_bf16(tmem_base + static_cast<uint32_t>(t * 128), make_sw128_desc(q0 + off, 16, 1024),
                    make_sw128_desc(k0 + off, 16, 1024), idesc_s, kk != 0 ? 1u : 0u);
        }
        if (t == 1) umma_commit(&k_empty[s]);
        umma_commit(&s_full[t]);
        return true;
      };
      // O_t += P_t(j) V(j), P_t(j) in columns [0, 32) (keys 0-63) and [64, 96) (keys 64-127) of S_t
      auto issue_pv = [&](int t, int j) -> bool {
        const int s = j & 1;
        const uint32_t use = static_cast<uint32_t>(j >> 1);
        if (!mbar_wait(&p_full[t], static_cast<uint32_t>(j) & 1u, abort_flag, kDevErrTimeoutMma)) return false;
        const bool first = (t == 0) || (j >= nkb_t[0]);
        if (first && !mbar_wait(&v_full[s], use & 1u, abort_flag, kDevErrTimeoutMma)) return false;
        tc_fence_after();
        const uint32_t v0 = smem_u32(sV + s * kAttnVBytes);
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t boff = static_cast<uint32_t>((kk >> 2) * 16384 + (kk & 3) * 2048);
          umma_bf16_ts(tmem_base + 256u + static_cast<uint32_t>(t * 128),
                       tmem_base + static_cast<uint32_t>(t * 128 + (kk >> 2) * 64 + (kk & 3) * 8),
                       make_sw128_desc(v0 + boff, 8192, 1024),
                       idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        if (t == 1) umma_commit(&v_empty[s]);
        if (j == (t ? nkb_t[1] : nkb_t[0]) - 1) umma_commit(&pv_done[t]);
        return true;
      };
      if (ok && nkb_t[0] > 0) ok = issue_s(0, 0);
      if (ok && nkb_t[1] > 0) ok = issue_s(1, 0);
      for (int j = 0; j < nkb && ok; ++j) {
        if (j < nkb_t[0]) {
          ok = issue_pv(0, j);
          if (ok && j + 1 < nkb_t[0]) ok = issue_s(0, j + 1);
        }
        if (ok && j < nkb_t[1]) {
          ok = issue_pv(1, j);
          if (ok && j + 1 < nkb_t[1]) ok = issue_s(1, j + 1);
        }
      }
      // every MMA issued by this thread is complete once `drain` flips
      umma_commit(drain);
      const uint32_t a = smem_u32(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (tile X) + epilogue
    // Two threads per query row: warps 2-9 serve tile A, 10-17 tile B; within a
    // tile the first four warps take keys 0-63 of every block (hw = 0), the next
    // four keys 64-127 (hw = 1).  Warp w reads tensor-memory lanes 32 (w % 4) ..
    // 32 (w % 4) + 31, so the two warps of a row quarter share their rows; they
    // exchange the block's row maximum (and at the end the row sum) through
    // shared memory at a 64-thread named barrier.
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      int got = 1;
      if (lane == 0) got = mbar_wait(bar, parity, abort_flag, kDevErrTimeoutEpilogue, 32) ? 1 : 0;
      return __shfl_sync(0xffffffffu, got, 0) != 0;
    };
    const int w = warp - 2;
    const int X = w >> 3;         // tile
    const int hw = (w >> 2) & 1;  // key half of each block
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int pair_bar = 1 + X * 4 + quarter;  // named barrier 1..8
    float* xch = s_xch + (X * 4 + quarter) * 64 + lane;  // + buf * 512 + half * 32
    volatile int* got_flag = reinterpret_cast<volatile int*>(s_xch + 1024) + (X * 4 + quarter) * 2;  // + buf * 16 + half
    const int64_t qi = static_cast<int64_t>(m0) + X * kAttnTile + r;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t s_col = lane_base + static_cast<uint32_t>(X * 128 + hw * 64);  // this thread's 64 scores
    const uint32_t o_col = lane_base + 256u + static_cast<uint32_t>(X * 128 + hw * 64);  // its 64 columns of O
    // the row's last visible key, clamped to [-1, nk - 1] (32-bit from here on)
    int64_t last64 = p.causal ? qi + p.causal_off : static_cast<int64_t>(p.nk) - 1;
    last64 = last64 < -1 ? -1 : (last64 > p.nk - 1 ? p.nk - 1 : last64);
    const int last_key = static_cast<int>(last64);
    const int my_nkb = X ? nkb_t[1] : nkb_t[0];
    float m_run = -INFINITY, l_half = 0.f;
    bool ok = true;
    for (int j = 0; j < my_nkb && ok; ++j) {
      // The hw = 0 warp waits (bounded) for S(j) and passes the outcome to its
      // partner at a named barrier, so both warps of the pair take the same path
      // and meet at every named barrier the same number of times (a bar.sync has
      // no time limit).  The flag of a block is rewritten only two blocks later,
      // after barriers the partner passes only once it has read it.
      volatile int* gf = got_flag + (j & 1) * 16;
      if (hw == 0) {
        const bool got = warp_wait(&s_full[X], static_cast<uint32_t>(j) & 1u);
        if (lane == 0) gf[0] = got ? 1 : 0;
      }
      attn_pair_sync(pair_bar);
      if (gf[0] == 0) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int key0 = j * kAttnTile + hw * 64;  // this thread's first key of the block
      // every one of this thread's keys visible to the row: no masking work
      const bool full = key0 + 63 <= last_key;
      // pass 1: the maximum of this thread's 64 scores (scaled, masked), eight
      // independent chains.  tcgen05.ld is warp-collective (.sync.aligned): every
      // lane executes the same loads, outside any branch on row-dependent values.
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
      const bool fast = full && p.scale_log2 > 0.f;
      {
        uint32_t v[2][32];
        tmem_ld32(s_col, v[0]);
        tmem_ld32(s_col + 32u, v[1]);
        tmem_ld_wait();
        if (fast) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            mx8[e & 7] = attn_max3(mx8[e & 7], __uint_as_float(v[0][e]), __uint_as_float(v[1][e]));
        } else {
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (key0 + e <= last_key)
              mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(v[e >> 5][e & 31]) * p.scale_log2);
        }
      }
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      if (fast) mx *= p.scale_log2;
      // the row maximum: exchange with the other half (double-buffered by block
      // parity, so a value is never overwritten before the partner has read it).
      // The barrier also orders the partner's score loads before this thread's
      // stores of P below.
      float* xb = xch + (j & 1) * 512;
      xb[hw * 32] = mx;
      tc_fence_before();
      attn_pair_sync(pair_bar);
      tc_fence_after();
      mx = fmaxf(mx, xb[(hw ^ 1) * 32]);
      // the reference maximum moves only when the row's maximum grows by more than
      // kAttnRescaleLog2 (log2 units): the weights exp2(s - m) then stay below 2^8,
      // and O and l are rescaled rarely instead of at almost every block.  Both
      // halves of a row compute the same m and corr.
      const bool grow = (m_run == -INFINITY) || (mx > m_run + kAttnRescaleLog2);
      const float m_new = grow ? fmaxf(m_run, mx) : m_run;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float corr = grow ? attn_exp2(m_run - m_use) : 1.f;  // 0 for the first block
      // pass 2: P = exp2(s * scale_log2 - m) as bf16 pairs; keys 64 hw .. 64 hw + 63
      // go to columns 64 hw .. 64 hw + 31 of S (this thread's own scores, read)
      uint64_t sum2[2];  // fp32 pairs: four independent partial sums
      sum2[0] = sum2[1] = 0ull;
      const uint64_t sc2 = attn_f2(p.scale_log2, p.scale_log2), nm2 = attn_f2(-m_use, -m_use);
      for (int h = 0; h < 2; ++h) {
        uint32_t vc[32];
        tmem_ld32(s_col + static_cast<uint32_t>(h * 32), vc);
        tmem_ld_wait();
        uint32_t pk[16];
        if (full) {
          // every key on the special-function unit (one instruction per key; the
          // packed cubic takes ~2.5, and the unit has room at this rate)
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t xq = attn_fma2(attn_f2(__uint_as_float(vc[2 * e]), __uint_as_float(vc[2 * e + 1])), sc2, nm2);
            const float y0 = attn_exp2(attn_lo(xq)), y1 = attn_exp2(attn_hi(xq));
            sum2[e & 1] = attn_add2(sum2[e & 1], attn_f2(y0, y1));
            pk[e] = attn_bf16x2(y0, y1);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int ka = key0 + h * 32 + 2 * e;
            const float x0 =
                (ka <= last_key) ? attn_exp2_poly(fmaf(__uint_as_float(vc[2 * e]), p.scale_log2, -m_use)) : 0.f;
            const float x1 =
                (ka + 1 <= last_key) ? attn_exp2(fmaf(__uint_as_float(vc[2 * e + 1]), p.scale_log2, -m_use)) : 0.f;
            sum2[e & 1] = attn_add2(sum2[e & 1], attn_f2(x0, x1));
            pk[e] = attn_bf16x2(x0, x1);
          }
        }
        tmem_st16(s_col + static_cast<uint32_t>(h * 16), pk);
      }
      const uint64_t s01 = attn_add2(sum2[0], sum2[1]);
      l_half = l_half * corr + (attn_lo(s01) + attn_hi(s01));
      m_run = m_new;
      // O *= corr where some row's reference maximum moved (this thread's 64
      // columns); PV(j-1) is complete (it was issued before S(j))
      if (j > 0 && __any_sync(0xffffffffu, corr != 1.f)) {
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          tmem_ld32(o_col + static_cast<uint32_t>(c * 32), o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
          tmem_st32(o_col + static_cast<uint32_t>(c * 32), o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[X]);
    }
    // epilogue: O / l as bf16, l = the sum of both halves of the row (both warps of
    // the pair leave the loop after the same block, see the wait flag)
    xch[(my_nkb & 1) * 512 + hw * 32] = l_half;
    attn_pair_sync(pair_bar);
    const float l_row = l_half + xch[(my_nkb & 1) * 512 + (hw ^ 1) * 32];
    if (ok && my_nkb > 0 && warp_wait(&pv_done[X], 0u)) {
      tc_fence_after();
      const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
      uint16_t* orow = p.O + (static_cast<int64_t>(item) * p.nq + qi) * 128 + hw * 64;
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tmem_ld32(o_col + static_cast<uint32_t>(c * 32), v);
        tmem_ld_wait();
        uint32_t o[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const __nv_bfloat162 t2 =
              __floats2bfloat162_rn(__uint_as_float(v[2 * e]) * inv, __uint_as_float(v[2 * e + 1]) * inv);
          o[e] = *reinterpret_cast<const uint32_t*>(&t2);
        }
        if (qi < p.nq) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            reinterpret_cast<uint4*>(orow + c * 32)[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace rmm
