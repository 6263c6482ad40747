// Reduced product on the 5th-generation tensor cores:
//   Y[M x N] = A_I[M x k] . B[I, :][k x N]      ("Algorithm Deep-Dive: RMM",
//   Core Approach: RMM_rho(A, B) = A[:, I] B[I, :]; the reduced product is still
//   a dense contraction over the k kept indices).
//
// Persistent, warp-specialised tcgen05 kernel, one CTA per SM:
//   warp 0      TMA producer: A tile (K-major, 128 x 64 bf16, 128-byte swizzle)
//               and B tile, either MN-major (64 contraction rows x BN columns,
//               B[I, :] packed row-contiguous beforehand, or B itself on the
//               rho = 1 path) or K-major (per-head Q K^T, K packed like Q).
//               Kept rows are packed before the GEMM rather than gathered per
//               tile: on B200 a TMA row gather (tile::gather4, 4 rows x 128 B per
//               copy) or a 512-byte bulk copy per row stages only ~7-8 B/clk/SM,
//               while 64 x 64 tiles stage ~44 B/clk/SM, so the per-copy cost of
//               small TMA copies, not DRAM, would bound the product.
//   warp 1      allocates tensor memory; lane 0 issues tcgen05.mma (M=128,
//               N=BN, K=16 per instruction) into a double-buffered fp32
//               accumulator in TMEM and commits to mbarriers.
//   warps 2..5  epilogue: tcgen05.ld TMEM -> registers -> bf16/fp32 -> a
//               128-byte-swizzled 32-row chunk in shared memory (two per warp,
//               alternating) -> one TMA tensor store per chunk, clipped to the
//               batch item's rows and columns.  (Stores from registers, one row
//               per lane, left the fp32 score writes at ~26% of HBM bandwidth.)
// Work split: tiles are dealt to the CTAs round-robin.  When the tile count is
// not a multiple of the grid, the last wave holds fewer tiles than there are
// CTAs and most SMs would idle for a whole tile time; instead each of those
// tail_tiles trailing tiles is cut along N into tail_split pieces of BN /
// tail_split columns (a narrower UMMA, N = 128 or 64), one piece per CTA, so
// the last wave takes about 1 / tail_split of a tile time.  Nothing is added
// across CTAs: every output element is still produced by one accumulator.
// Every wait is bounded (about one second); on a timeout the CTA records an
// error code, drains its own copies in flight, frees its TMEM and returns.
// There is no cluster multicast anywhere: each CTA fetches its own tiles and
// L2 absorbs the reuse between CTAs.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace rmm {

enum BMode : int { kBTileMN = 1, kBTileK = 2 };
enum EpiMode : int { kEpiBf16 = 0, kEpiF32 = 1 };
enum CausalMode : int { kCausalNone = 0, kCausalMaskScores = 1, kCausalLimitK = 2 };

struct GemmParams {
  int M, N;              // rows / columns of one batch item's output
  int k;                 // kept contraction length (true k, not padded)
  int num_kb;            // ceil(k / 64)
  int batch;
  int m_tiles, n_tiles;
  int a_rows_per_batch;  // A tensor-map row of (b, m) = b * a_rows_per_batch + m
  // B tensor-map row of batch item b: b_row_base(b) + t (MN tile, contraction
  // row t) or + n (K-major tile), b_row_base(b) = (b / b_g_outer) * b_s_outer +
  // ((b % b_g_outer) / b_g_inner) * b_s_inner
  const int32_t* idx;    // [batch][k] ascending kept indices (causal k-limit), or null for I = [0, k)
  int64_t idx_bstride;
  int b_g_outer, b_g_inner;
  int64_t b_s_outer, b_s_inner;
  // output
  void* out;
  int64_t ldo;           // elements between output rows
  int64_t out_bstride;   // elements between batch items
  float scale;
  int64_t causal_off;    // key/position j is visible to row i iff j <= i + causal_off
  // narrow last wave (MN-major B only): the last tail_tiles tiles are cut into
  // tail_split pieces of BN / tail_split (>= 64) columns; 0 / 1 = no cut
  int tail_tiles, tail_split;
  // gathered B (CTA-pair kernel only): the kept rows B[I[t], :] are read straight
  // from the weights through the index set instead of from a packed copy
  const uint16_t* gw0;   // [d][gldw] bf16 (gate weights with SWIGLU)
  const uint16_t* gw1;   // up weights (SWIGLU), else unused
  int64_t gldw;
  const int32_t* gidx;   // [k] ascending kept rows
  // test hook (0 in every product call): 1 makes the producer, once the stage
  // ring is full, wait on a barrier that nothing arrives on, with a 1 ms limit,
  // so that its bounded wait runs out and the kernel takes its timeout path
  int expire_producer_waits;
};

// wait limit of the test hook's producer wait: far below the ~1 s of every other
// wait, far above the polling granularity
constexpr uint64_t kGemmHookWaitNs = 1000ull * 1000ull;

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGES = (BN >= 256) ? 4 : (BN >= 128 ? 6 : 8);
  static constexpr int TMEM_COLS = 2 * BN;  // two accumulators
  static constexpr int EPI_BYTES = 4 * 2 * 4096;  // 4 epilogue warps x 2 chunks of 32 rows x 128 bytes
  static constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES) + EPI_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(8 * (3 * STAGES + 6) + 8 <= 256, "barrier area");
};

__device__ __forceinline__ int64_t gemm_b_row_base(const GemmParams& p, int b) {
  return static_cast<int64_t>(b / p.b_g_outer) * p.b_s_outer +
         static_cast<int64_t>((b % p.b_g_outer) / p.b_g_inner) * p.b_s_inner;
}

// Number of 64-wide k-blocks a tile needs.
template <int BN, int CAUSAL>
__device__ __forceinline__ int gemm_tile_kb(const GemmParams& p, int b, int m0, int n0) {
  if (CAUSAL == kCausalMaskScores) {
    // a tile whose first key lies beyond every row's horizon is fully masked
    if (static_cast<int64_t>(n0) > static_cast<int64_t>(m0) + 127 + p.causal_off) return 0;
    return p.num_kb;
  } else if (CAUSAL == kCausalLimitK) {
    // kept positions I[t] <= last row + off contribute; I is ascending
    const int64_t hz = static_cast<int64_t>(m0) + 127 + p.causal_off;
    if (p.idx == nullptr) {  // identity index set
      const int64_t lim = hz + 1 < 0 ? 0 : (hz + 1 > p.k ? p.k : hz + 1);
      return static_cast<int>((lim + 63) >> 6);
    }
    const int32_t* I = p.idx + static_cast<int64_t>(b) * p.idx_bstride;
    int lo = 0, hi = p.k;  // first t with I[t] > hz
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (static_cast<int64_t>(__ldg(I + mid)) <= hz) lo = mid + 1;
      else hi = mid;
    }
    return (lo + 63) >> 6;
  }
  return p.num_kb;
}

// Causal PV: does k-block kb of the M tile at m0 hold entries above the
// diagonal (key j > row i + causal_off) for some row?  Those A tiles are masked
// in shared memory before the MMA reads them.
template <int CAUSAL>
__device__ __forceinline__ bool gemm_diag_block(const GemmParams& p, int m0, int kb) {
  return CAUSAL == kCausalLimitK &&
         static_cast<int64_t>(kb) * 64 + 63 > static_cast<int64_t>(m0) + p.causal_off;
}

// Zero A-tile entries (row r, column c) with 64 kb + c > m0 + r + causal_off;
// 32 lanes, four rows each, 128-byte-swizzled K-major layout.
__device__ __forceinline__ void gemm_mask_diag(uint8_t* tileA, const GemmParams& p, int m0, int kb, int lane) {
  for (int r = lane; r < 128; r += 32) {
    const int64_t lim = static_cast<int64_t>(m0) + r + p.causal_off - static_cast<int64_t>(kb) * 64;  // last visible column
    if (lim >= 63) continue;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c_lo = u * 8;
      if (c_lo + 7 <= lim) continue;
      uint4* ptr = reinterpret_cast<uint4*>(tileA + r * 128 + ((u ^ (r & 7)) << 4));
      if (c_lo > lim) {
        *ptr = make_uint4(0u, 0u, 0u, 0u);
      } else {
        uint4 v = *ptr;
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (c_lo + e > lim) w[e >> 1] &= (e & 1) ? 0x0000FFFFu : 0xFFFF0000u;
        *ptr = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

// Tile order: batch item, then N tile, then M tile fastest, so CTAs running at
// the same time share B column blocks in L2.
__device__ __forceinline__ void gemm_tile_coords(const GemmParams& p, int tile, int& b, int& m0, int& nt) {
  const int per_b = p.m_tiles * p.n_tiles;
  b = tile / per_b;
  const int r = tile - b * per_b;
  nt = r / p.m_tiles;
  m0 = (r - nt * p.m_tiles) * 128;
}

// One unit of a CTA's work: output columns [nt * BN + n_off, + w) of one tile.
struct GemmWork {
  int tile, n_off, w;
};

// The it-th work unit of this CTA, or false when it has none left: whole tiles
// blockIdx.x, + P, ... first, then at most one piece of the narrow last wave.
// (P workers, this one is bx: CTAs, or CTA pairs in the pair kernel)
template <int BN>
__device__ __forceinline__ bool gemm_work(const GemmParams& p, int total_tiles, int it, GemmWork& wk, int P = -1,
                                          int bx = -1) {
  if (P < 0) {
    P = gridDim.x;
    bx = blockIdx.x;
  }
  const int whole = total_tiles - p.tail_tiles;
  const int n_whole = whole > bx ? (whole - bx + P - 1) / P : 0;
  if (it < n_whole) {
    wk.tile = bx + it * P;
    wk.n_off = 0;
    wk.w = BN;
    return true;
  }
  if (p.tail_tiles == 0) return false;
  const int q = bx + (it - n_whole) * P;  // piece of the last wave
  if (q >= p.tail_tiles * p.tail_split) return false;
  wk.tile = whole + q / p.tail_split;
  wk.w = BN / p.tail_split;
  wk.n_off = (q % p.tail_split) * wk.w;
  return true;
}

template <int BN, int BMODE, int EPI, int CAUSAL>
__global__ void __launch_bounds__(192, 1)
    rmm_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmO, const GemmParams p) {
  using C = GemmCfg<BN>;
  constexpr int STAGES = C::STAGES;
  constexpr uint32_t IDESC = make_idesc_bf16(128, BN, 0, (BMODE == kBTileK) ? 0 : 1);

  extern __shared__ uint8_t gemm_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::A_BYTES;
  uint8_t* sE = sB + STAGES * C::B_BYTES;  // epilogue staging, 1024-byte aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(sE + C::EPI_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* ready = drain + 1;  // [STAGES]: diagonal A tiles masked (causal PV)
  uint64_t* never = ready + STAGES;  // test hook only: no thread ever arrives on it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    for (int st = 0; st < STAGES; ++st) mbar_init(&ready[st], 1);
    mbar_init(never, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = p.batch * p.m_tiles * p.n_tiles;
  wait_prior_kernels();  // operands and the output buffer are touched only after this

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0;
    bool ok = true;
    GemmWork wk;
    for (int it = 0; ok && gemm_work<BN>(p, total_tiles, it, wk); ++it) {
      int b, m0, nt;
      gemm_tile_coords(p, wk.tile, b, m0, nt);
      const int n0 = nt * BN + wk.n_off;
      const int nkb = gemm_tile_kb<BN, CAUSAL>(p, b, m0, nt * BN);
      const uint32_t b_bytes = static_cast<uint32_t>(wk.w) * 64 * 2;
      const int a_row = b * p.a_rows_per_batch + m0;
      const int64_t brow0 = gemm_b_row_base(p, b);
      for (int kb = 0; kb < nkb; ++kb) {
        int w = 1;
        if (lane == 0) {
          if (p.expire_producer_waits && issued == static_cast<uint32_t>(STAGES))
            w = mbar_wait(never, 0u, abort_flag, kDevErrTimeoutProducer, 0, false, kGemmHookWaitNs) ? 1 : 0;
          else
            w = mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kDevErrTimeoutProducer) ? 1 : 0;
        }
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[stage], C::A_BYTES + b_bytes);
          tma_load_2d(sA + stage * C::A_BYTES, &tmA, &full[stage], kb * 64, a_row);
        }
        __syncwarp();
        uint8_t* dstB = sB + stage * C::B_BYTES;
        if (BMODE == kBTileMN) {
          if (lane < wk.w / 64)
            tma_load_2d(dstB + lane * 8192, &tmB, &full[stage], n0 + lane * 64, static_cast<int32_t>(brow0 + kb * 64));
        } else {
          if (lane == 0) tma_load_2d(dstB, &tmB, &full[stage], kb * 64, static_cast<int32_t>(brow0 + n0));
        }
        __syncwarp();
        if (gemm_diag_block<CAUSAL>(p, m0, kb)) {
          // let this stage land, zero its entries above the diagonal, then release it to the MMA
          int landed = 1;
          if (lane == 0) landed = mbar_wait(&full[stage], phase, abort_flag, kDevErrTimeoutProducer) ? 1 : 0;
          landed = __shfl_sync(0xffffffffu, landed, 0);
          if (!landed) {
            ok = false;
            break;
          }
          gemm_mask_diag(sA + stage * C::A_BYTES, p, m0, kb, lane);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ready[stage]);
        }
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      // drain: wait for the copies this CTA issued so no TMA writes land after exit
      for (int s = 0; s < STAGES; ++s) {
        const uint32_t uses = (issued + STAGES - 1 - s) / STAGES;  // loads issued into stage s
        if (uses == 0) continue;
        const uint32_t par = (uses - 1) & 1u;
        const uint32_t a = smem_u32(&full[s]);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(a, par) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t ready_phase = 0;  // one parity bit per stage for the `ready` barriers
      int acc_i = 0;
      bool ok = true;
      GemmWork wk;
      for (int it = 0; ok && gemm_work<BN>(p, total_tiles, it, wk); ++it) {
        int b, m0, nt;
        gemm_tile_coords(p, wk.tile, b, m0, nt);
        const int nkb = gemm_tile_kb<BN, CAUSAL>(p, b, m0, nt * BN);
        if (nkb == 0) continue;
        const uint32_t idesc = (wk.w == BN) ? IDESC : make_idesc_bf16(128, wk.w, 0, (BMODE == kBTileK) ? 0 : 1);
        const int acc = acc_i & 1;
        const uint32_t acc_par = (acc_i >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_par ^ 1u, abort_flag, kDevErrTimeoutMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < nkb; ++kb) {
          bool got;
          if (gemm_diag_block<CAUSAL>(p, m0, kb)) {
            got = mbar_wait(&ready[stage], (ready_phase >> stage) & 1u, abort_flag, kDevErrTimeoutMma);
            ready_phase ^= 1u << stage;
          } else {
            got = mbar_wait(&full[stage], phase, abort_flag, kDevErrTimeoutMma);
          }
          if (!got) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = make_sw128_desc(a0 + kk * 32, 16, 1024);
            const uint64_t bd = (BMODE == kBTileK) ? make_sw128_desc(b0 + kk * 32, 16, 1024)
                                                   : make_sw128_desc(b0 + kk * 2048, 8192, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        ++acc_i;
      }
      // all MMAs issued by this thread are complete once `drain` flips
      umma_commit(drain);
      const uint32_t a = smem_u32(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    uint8_t* ebuf = sE + (warp - 2) * 8192;
    constexpr int CW = (EPI == kEpiF32) ? 32 : 64;  // columns per 128-byte chunk row
    int acc_i = 0;
    int seq = 0;  // chunks staged by this warp so far (buffer alternation)
    GemmWork wk;
    for (int it = 0; gemm_work<BN>(p, total_tiles, it, wk); ++it) {
      int b, m0, nt;
      gemm_tile_coords(p, wk.tile, b, m0, nt);
      const int n0 = nt * BN + wk.n_off;
      const int nkb = gemm_tile_kb<BN, CAUSAL>(p, b, m0, nt * BN);
      const int row0 = m0 + quarter * 32;  // this warp's 32-row slab
      const int row = row0 + lane;
      if (nkb > 0) {
        const int acc = acc_i & 1;
        const uint32_t acc_par = (acc_i >> 1) & 1;
        if (!mbar_wait(&tfull[acc], acc_par, abort_flag, kDevErrTimeoutEpilogue, 64)) break;
        tc_fence_after();
      }
      for (int c = 0; c < wk.w / CW; ++c) {
        float v[CW];
        if (nkb > 0) {
          uint32_t r[32];
#pragma unroll
          for (int h = 0; h < CW / 32; ++h) {
            tmem_ld32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                          static_cast<uint32_t>((acc_i & 1) * BN + c * CW + h * 32),
                      r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[h * 32 + e] = __uint_as_float(r[e]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < CW; ++e) v[e] = 0.f;
        }
        const int col0 = n0 + c * CW;
        uint8_t* buf = ebuf + (seq & 1) * 4096;
        // the store issued two chunks ago read this buffer; let it finish reading
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        uint32_t w[32];
        if (EPI == kEpiF32) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            float x = v[e] * p.scale;
            if (CAUSAL == kCausalMaskScores && static_cast<int64_t>(col0 + e) > static_cast<int64_t>(row) + p.causal_off)
              x = -__int_as_float(0x7f800000);
            w[e] = __float_as_uint(x);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const __nv_bfloat162 t2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
            w[e] = *reinterpret_cast<const uint32_t*>(&t2);
          }
        }
        // row `lane` of the chunk, 16-byte unit j at position j ^ (row & 7) (128-byte swizzle)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
              make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < p.M && col0 < p.N) {
          tma_store_3d(&tmO, buf, col0, row0, b);
          bulk_commit_group();
        }
        ++seq;
      }
      if (nkb > 0) {
        tc_fence_before();
        mbar_arrive(&tempty[acc_i & 1]);
        ++acc_i;
      }
    }
    if (lane == 0) bulk_wait_group<0>();  // every store has finished before the CTA exits
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace rmm
