// Attention with a reduced score product, fused so that the scores S and the
// probabilities P never leave the SM ("Algorithm Deep-Dive: RMM", Component
// mapping: QK^T selects head dims by the Q column norm, K gathers them under
// GQA; Attention vs MLP, Table 16: attention-internal reduction):
//   S_h = scale * Q_h[:, I_h] K_g(h)[:, I_h]^T   (-inf above the causal diagonal)
//   O_h = softmax_rows(S_h) V_g(h)
// The index sets come from the column-norm and selection kernels; Q[:, I_h] and
// K_g(h)[:, I_h] are packed per query head, zero-padded to KP = 64 or 128 dims, so
// the score product contracts over KP instead of 128.  The value product is the
// ordinary one (selecting P's columns would need all of P first).
//
// One CTA per (query head, 128-row query tile), 192 threads:
//   warp 0      TMA: the Q tile once, then 128-key blocks of K (K-major, KP
//               dims) and V (MN-major, 128 dims) into two-stage rings.
//   warp 1      tensor memory (512 columns: S double buffer 2 x 128, O 128);
//               lane 0 issues S(j) = Q K(j)^T (M = 128, N = 128, K = KP) into
//               S buffer j % 2, and O += P(j) V(j) (M = 128, N = 128, K = 128),
//               S(j+1) ahead of PV(j) so the score MMA overlaps softmax(j).
//   warps 2..5  online softmax, one query row per thread: read S(j) from tensor
//               memory, scale and mask, running max m and sum l (exp2 with the
//               scale folded in log2 units), rescale the row of O in tensor
//               memory when m grows, write P(j) as bf16 into the 128-byte-
//               swizzled K-major layout the PV MMA reads; at the end O / l.
// Every wait is bounded (about one second); on a timeout the CTA records an
// error code, drains its copies, lets the MMA finish and returns.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace rmm {

struct AttnParams {
  int nq, nk;          // query / key rows of one head
  int kp;              // packed score dims: 64 or 128
  int hq, hkv;         // heads (GQA: query head h reads key/value head h / (hq / hkv))
  int items;           // batch * hq
  int m_tiles;         // ceil(nq / 128)
  int k_per_item;      // 1: K rows are packed per query head (item * nk); 0: K as given ((b * hkv + g) * nk)
  int causal;
  int64_t causal_off;  // key j is visible to query i iff j <= i + causal_off
  float scale_log2;    // scale * log2(e)
  uint16_t* O;         // bf16 [items][nq][128]
};

constexpr int kAttnTile = 128;
constexpr uint32_t kAttnQBytes = 128 * 128 * 2;  // Q tile, up to 128 dims (two 64-dim atoms)
constexpr uint32_t kAttnKBytes = 128 * 128 * 2;  // one K block, up to 128 dims
constexpr uint32_t kAttnVBytes = 128 * 128 * 2;  // one V block: 2 key halves x 2 column atoms of 64 x 64
constexpr uint32_t kAttnPBytes = 128 * 128 * 2;  // P tile, K-major over 128 keys (two atoms)
constexpr int kAttnSmem = kAttnQBytes + 2 * kAttnKBytes + 2 * kAttnVBytes + kAttnPBytes + 1024 + 256;

// 2^x with the hardware approximation (relative error ~2^-22; exp2(-inf) = 0).
__device__ __forceinline__ float attn_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

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

__global__ void __launch_bounds__(192, 1)
    attn_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  extern __shared__ uint8_t attn_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kAttnQBytes;
  uint8_t* sV = sK + 2 * kAttnKBytes;
  uint8_t* sP = sV + 2 * kAttnVBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + kAttnPBytes);
  uint64_t* q_full = bars;           // 1
  uint64_t* k_full = bars + 1;       // 2
  uint64_t* k_empty = bars + 3;      // 2
  uint64_t* v_full = bars + 5;       // 2
  uint64_t* v_empty = bars + 7;      // 2
  uint64_t* s_full = bars + 9;       // 2
  uint64_t* s_empty = bars + 11;     // 2
  uint64_t* p_full = bars + 13;      // 1
  uint64_t* pv_done = bars + 14;     // 1
  uint64_t* drain = bars + 15;       // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // heaviest causal tiles first: the last query tiles of every head lead the grid
  const int item = static_cast<int>(blockIdx.x % p.items);
  const int mt = p.m_tiles - 1 - static_cast<int>(blockIdx.x / p.items);
  const int m0 = mt * kAttnTile;
  const int b = item / p.hq, h = item % p.hq;
  const int g = h / (p.hq / p.hkv);
  const int nkb = attn_key_blocks(p, m0);
  const int qrow0 = item * p.nq + m0;
  const int krow0 = p.k_per_item ? item * p.nk : (b * p.hkv + g) * p.nk;
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
      mbar_init(&s_empty[s], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
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
      mbar_arrive_expect_tx(q_full, k_bytes);
      for (int a = 0; a < p.kp / 64; ++a) tma_load_2d(sQ + a * 16384, &tmQ, q_full, a * 64, qrow0);
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
      const uint32_t idesc_o = make_idesc_bf16(128, 128, 0, 1);  // P K-major, V MN-major
      const uint32_t q0 = smem_u32(sQ), p0 = smem_u32(sP);
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        const uint32_t use = static_cast<uint32_t>(j >> 1);
        if (!mbar_wait(&k_full[s], use & 1u, abort_flag, kDevErrTimeoutMma)) return false;
        if (!mbar_wait(&s_empty[s], (use & 1u) ^ 1u, abort_flag, kDevErrTimeoutMma)) return false;
        tc_fence_after();
        const uint32_t k0 = smem_u32(sK + s * kAttnKBytes);
        for (int kk = 0; kk < p.kp / 16; ++kk) {
          const uint32_t off = static_cast<uint32_t>((kk >> 2) * 16384 + (kk & 3) * 32);
          umma_bf16(tmem_base + static_cast<uint32_t>(s * 128), make_sw128_desc(q0 + off, 16, 1024),
                    make_sw128_desc(k0 + off, 16, 1024), idesc_s, kk != 0 ? 1u : 0u);
        }
        umma_commit(&k_empty[s]);
        umma_commit(&s_full[s]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int s = j & 1;
        const uint32_t use = static_cast<uint32_t>(j >> 1);
        if (!mbar_wait(p_full, static_cast<uint32_t>(j) & 1u, abort_flag, kDevErrTimeoutMma)) return false;
        if (!mbar_wait(&v_full[s], use & 1u, abort_flag, kDevErrTimeoutMma)) return false;
        tc_fence_after();
        const uint32_t v0 = smem_u32(sV + s * kAttnVBytes);
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = static_cast<uint32_t>((kk >> 2) * 16384 + (kk & 3) * 32);
          const uint32_t boff = static_cast<uint32_t>((kk >> 2) * 16384 + (kk & 3) * 2048);
          umma_bf16(tmem_base + 256, make_sw128_desc(p0 + aoff, 16, 1024), make_sw128_desc(v0 + boff, 8192, 1024),
                    idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&v_empty[s]);
        umma_commit(pv_done);
        return true;
      };
      if (ok && nkb > 0) ok = issue_s(0);
      for (int j = 0; j < nkb && ok; ++j) {
        if (j + 1 < nkb) ok = issue_s(j + 1);
        if (ok) ok = issue_pv(j);
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
    // ------------------------------------------------------------ softmax + epilogue
    // tcgen05.ld / st are warp-collective: lane 0 waits and the warp follows
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      int got = 1;
      if (lane == 0) got = mbar_wait(bar, parity, abort_flag, kDevErrTimeoutEpilogue, 32) ? 1 : 0;
      return __shfl_sync(0xffffffffu, got, 0) != 0;
    };
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row of the tile (tensor-memory lane)
    const int64_t qi = static_cast<int64_t>(m0) + r;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const int64_t last_key = p.causal ? qi + p.causal_off : static_cast<int64_t>(p.nk) - 1;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkb && ok; ++j) {
      const int s = j & 1;
      const uint32_t use = static_cast<uint32_t>(j >> 1);
      if (!warp_wait(&s_full[s], use & 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int64_t key0 = static_cast<int64_t>(j) * kAttnTile;
      const uint32_t s_col = lane_base + static_cast<uint32_t>(s * 128);
      // the whole row of S(j) in registers: scaled, masked, row maximum
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(s_col + static_cast<uint32_t>(c * 32), v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(v[e]);
      }
      tc_fence_before();
      mbar_arrive(&s_empty[s]);  // S buffer s may be overwritten by S(j + 2)
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < 128; ++e) {
        const int64_t key = key0 + e;
        x[e] = (key < p.nk && key <= last_key) ? x[e] * p.scale_log2 : -INFINITY;
        mx = fmaxf(mx, x[e]);
      }
      const float m_new = fmaxf(m_run, mx);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float corr = attn_exp2(m_run - m_use);  // 0 for the first block
      // the previous PV product must be done before O is rescaled and P overwritten
      if (j > 0 && !warp_wait(pv_done, static_cast<uint32_t>(j - 1) & 1u)) {
        ok = false;
        break;
      }
      // P = exp2(x - m) as bf16 into the swizzled K-major tile
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const __nv_bfloat162 t2 =
              __floats2bfloat162_rn(attn_exp2(x[c * 32 + 2 * e] - m_use), attn_exp2(x[c * 32 + 2 * e + 1] - m_use));
          sum += __low2float(t2) + __high2float(t2);  // the row sum of the rounded weights that multiply V
          pk[e] = *reinterpret_cast<const uint32_t*>(&t2);
        }
        // keys c*32 .. c*32+31 = 16-byte chunks 4c .. 4c+3 of the row (atom = chunk / 8)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = c * 4 + q;
          const int atom = chunk >> 3, cw = chunk & 7;
          *reinterpret_cast<uint4*>(sP + atom * 16384 + r * 128 + ((cw ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      l_run = l_run * corr + sum;
      m_run = m_new;
      // O *= corr, only in warps where some row's maximum grew (tcgen05.ld / st are warp-wide)
      if (j > 0 && __any_sync(0xffffffffu, corr != 1.f)) {
        tc_fence_after();
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(lane_base + 256u + static_cast<uint32_t>(c * 32), v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * corr);
          tmem_st32(lane_base + 256u + static_cast<uint32_t>(c * 32), v);
        }
        tmem_st_wait();
      }
      fence_proxy_async_smem();  // P (generic-proxy stores) is read by the MMA (async proxy)
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // epilogue: O / l as bf16
    if (ok && nkb > 0 && warp_wait(pv_done, static_cast<uint32_t>(nkb - 1) & 1u)) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      uint16_t* orow = p.O + (static_cast<int64_t>(item) * p.nq + qi) * 128;
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(lane_base + 256u + static_cast<uint32_t>(c * 32), v);
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
