// Reduced product of the linear path on CTA pairs (tcgen05 .cta_group::2):
//   Y[M x N] = A_I[M x k] . B[I, :][k x N]      ("Algorithm Deep-Dive: RMM",
//   Core Approach: RMM_rho(A, B) = A[:, I] B[I, :]).
//
// Why pairs: a one-CTA 128 x 256 tile needs 48 KB of operands in shared memory
// per 64-deep k-block, about 96 bytes per tensor cycle per SM, which L2 cannot
// feed at full tensor rate (the one-CTA kernel keeps the tensor pipe ~64 % busy).
// Two CTAs of a cluster compute one 256 x 256 tile with a single M = 256 MMA:
// each CTA stages its own 128 rows of A and HALF of the B tile (128 columns),
// 32 KB per k-block, and the tensor cores read the peer's half through the
// pair.  Each CTA's tensor memory holds its 128 rows x 256 fp32 columns.
//
// Roles (192 threads per CTA, both CTAs):
//   warp 0      TMA producer: waits for its own free stage, loads its A rows and
//               B columns; every load counts its bytes on the EVEN CTA's full
//               barrier (the .cta_group::2 form of the tensor load, no multicast).
//   warp 1      allocates 512 tensor-memory columns in both CTAs (same warp,
//               same slot); in the even CTA lane 0 issues the M = 256 MMAs and
//               commits to the stage's empty barrier and the accumulator's full
//               barrier in BOTH CTAs (multicast commit).
//   warps 2..5  epilogue on this CTA's 128 rows (as in the one-CTA kernel);
//               when an accumulator is drained each warp arrives on the even
//               CTA's accumulator-empty barrier (8 arrivals per use).
// SWIGLU (the gate and up projections of an MLP block, "Algorithm Deep-Dive:
// RMM", Attention vs MLP): the two B halves of a pair tile come from two
// tensor maps, the even CTA loading gate columns [c, c+128) and the odd CTA up
// columns [c, c+128) of the same output columns, so each CTA's accumulator holds
// gate (columns 0-127) and up (128-255) for its rows; the epilogue writes
// H = SiLU(gate) * up (128 columns per 256-wide tile, bf16).  A narrow piece of
// width w holds gate in columns [0, w/2) and up in [w/2, w).
// GATHER (the reduced product without a packed copy of B[I, :]): each CTA's B
// half comes straight from the kept rows of the weights, B[I[t], :] for the 64
// kept indices t of a k-block, read through the index set by four more warps
// (warps 6-9, 320 threads per CTA).  A kept row contributes one contiguous
// 256-byte run (128 columns) per CTA and k-block; the warps copy the runs with
// 16-byte cp.async straight into the 128-byte-swizzled MN-major stage (a TMA
// copy per row or per four rows stages only ~7-8 B/clk/SM on B200, 16-byte
// cp.async ~35, and the pair needs ~22 B/clk/SM of B at full tensor rate).
// A B thread never waits for its own copies: cp.async.mbarrier.arrive counts
// it on a barrier once they have landed, so every stage of the ring can be in
// flight.  On the even CTA that barrier is the MMA's full barrier itself (it
// counts the A bytes of both CTAs, this CTA's 128 B threads and one forwarder);
// on the odd CTA it is a local one (bfull), and one thread (warp 1, idle there
// otherwise) waits on it, fences the async proxy and arrives on the even CTA's
// full barrier with cluster-scope release.  The MMA thread waits with
// cluster-scope acquire and fences the async proxy for its own CTA's copies.
// (A proxy fence in the copying threads themselves waits for their copies still
// in flight: the first version fenced there and kept about one stage in
// flight.)  Kept indices t >= k and columns past N read as zeros.
// Work split as in the one-CTA kernel, with pairs as the workers: whole tiles
// round-robin, then the tiles of a partial last wave cut into two 256 x 128
// pieces.  Every wait is bounded; the CTAs meet at a cluster barrier before
// either frees tensor memory or exits, so no CTA's shared memory goes away
// while the pair's MMA or the peer's copies may still use it.
#pragma once
#include "gemm.cuh"

namespace rmm {

struct PairCfg {
  static constexpr int A_BYTES = 128 * 64 * 2;  // this CTA's 128 rows x 64 k
  static constexpr int B_BYTES = 128 * 64 * 2;  // this CTA's 128 of the 256 columns x 64 k
  static constexpr int STAGES = 6;
  static constexpr int EPI_BYTES = 4 * 2 * 4096;
  static constexpr int TMEM_COLS = 512;          // two 256-column accumulators
  static constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES) + EPI_BYTES + 1024 + 256;
  static_assert(8 * (3 * STAGES + 5) + 8 <= 256, "barrier area");
};

constexpr int kPairGatherWarps = 4;  // B producer warps per CTA with GATHER (warps 6-9)

__device__ __forceinline__ void pair_cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// arrive on `bar` once every cp.async this thread issued so far has landed (the
// arrival is one of the barrier's expected count)
__device__ __forceinline__ void pair_cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void pair_cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Pair tile order: batch item, then N tile, then 256-row M tile fastest.
__device__ __forceinline__ void pair_tile_coords(const GemmParams& p, int tile, int& b, int& m0, int& nt) {
  const int per_b = p.m_tiles * p.n_tiles;
  b = tile / per_b;
  const int r = tile - b * per_b;
  nt = r / p.m_tiles;
  m0 = (r - nt * p.m_tiles) * 256;
}

template <bool SWIGLU, bool GATHER>
__global__ void __launch_bounds__(GATHER ? 320 : 192, 1)
    rmm_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmO,
                         const GemmParams p) {
  using C = PairCfg;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t pair_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pair_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::A_BYTES;
  uint8_t* sE = sB + STAGES * C::B_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sE + C::EPI_BYTES);  // used in the even CTA
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;  // used in the even CTA
  uint64_t* drain = tempty + 2;
  uint64_t* bfull = drain + 1;  // GATHER, odd CTA: its B threads' copies of a stage have landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bfull + STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the MMAs
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // GATHER: the A bytes of both CTAs (one expect_tx arrival), every B thread of
      // this CTA (its copies landed) and the odd CTA's forwarding thread
      mbar_init(&full[s], GATHER ? 1 + 32 * kPairGatherWarps + 1 : 1);
      mbar_init(&empty[s], 1);
      mbar_init(&bfull[s], 32 * kPairGatherWarps);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    if (!GATHER) prefetch_tensormap(&tmB);
    if (SWIGLU && !GATHER) prefetch_tensormap(&tmB2);
    prefetch_tensormap(&tmO);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = p.batch * p.m_tiles * p.n_tiles;
  const uint32_t full_even = map_shared_rank(smem_u32(&full[0]), 0u);
  const uint32_t tempty_even = map_shared_rank(smem_u32(&tempty[0]), 0u);
  wait_prior_kernels();

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;
      bool ok = true;
      GemmWork wk;
      for (int it = 0; ok && gemm_work<256>(p, total_tiles, it, wk, npairs, pair); ++it) {
        int b, m0, nt;
        pair_tile_coords(p, wk.tile, b, m0, nt);
        const int half = wk.w / 2;
        const int a_row = b * p.a_rows_per_batch + m0 + static_cast<int>(rank) * 128;
        // B columns of this CTA's half: its 128 of the 256 columns, or (SWIGLU)
        // the same output columns of gate (even CTA) or up (odd CTA)
        const int nb = SWIGLU ? nt * 128 + wk.n_off / 2 : nt * 256 + wk.n_off + static_cast<int>(rank) * half;
        const CUtensorMap* tb = (SWIGLU && rank == 1) ? &tmB2 : &tmB;
        const int64_t brow0 = gemm_b_row_base(p, b);
        const uint32_t pair_bytes = 2u * static_cast<uint32_t>(C::A_BYTES + (GATHER ? 0 : half * 64 * 2));
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kDevErrTimeoutProducer)) {
            ok = false;
            break;
          }
          const uint32_t bar = full_even + 8u * static_cast<uint32_t>(stage);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], pair_bytes);
          tma_load_2d_pair(sA + stage * C::A_BYTES, &tmA, bar, kb * 64, a_row);
          if (!GATHER)
            for (int j = 0; j < half / 64; ++j)
              tma_load_2d_pair(sB + stage * C::B_BYTES + j * 8192, tb, bar, nb + j * 64,
                               static_cast<int32_t>(brow0 + kb * 64));
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && rank == 0) {
        // wait (bounded) for the stages this pair filled, so no copy lands after exit
        for (int s = 0; s < STAGES; ++s) {
          const uint32_t uses = (issued + STAGES - 1 - s) / STAGES;
          if (uses == 0) continue;
          const uint32_t a = smem_u32(&full[s]);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(a, (uses - 1) & 1u) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (rank == 0 && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc_i = 0;
      bool ok = true;
      GemmWork wk;
      for (int it = 0; ok && gemm_work<256>(p, total_tiles, it, wk, npairs, pair); ++it) {
        const int acc = acc_i & 1;
        const uint32_t acc_par = (acc_i >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_par ^ 1u, abort_flag, kDevErrTimeoutMma, 0, true)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = make_idesc_bf16(256, wk.w, 0, 1);
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          // GATHER: the B warps of the odd CTA arrive with cluster-scope release
          if (!mbar_wait(&full[stage], phase, abort_flag, kDevErrTimeoutMma, 0, GATHER)) {
            ok = false;
            break;
          }
          // GATHER: this CTA's cp.async writes of the stage (acquired through the
          // barrier) are ordered before the MMA's async-proxy reads
          if (GATHER) fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = make_sw128_desc(a0 + kk * 32, 16, 1024);
            const uint64_t bd = make_sw128_desc(b0 + kk * 2048, 8192, 1024);
            umma_bf16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(&tfull[acc], 0x3);
        ++acc_i;
      }
      // every MMA issued by this thread is complete once `drain` flips
      umma_commit_pair(drain, 0x1);
      const uint32_t a = smem_u32(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    } else if (GATHER && rank == 1 && lane == 0) {
      // ------------------------------------------------------------ forwarder (odd CTA)
      // The B threads of this CTA count their copies on the local bfull barrier
      // (cp.async.mbarrier.arrive reaches this CTA's barriers only); once a
      // stage's copies have all landed this thread fences the async proxy and
      // passes the stage on to the even CTA's full barrier (cluster release).
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      GemmWork wk;
      for (int it = 0; ok && gemm_work<256>(p, total_tiles, it, wk, npairs, pair); ++it) {
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&bfull[stage], phase, abort_flag, kDevErrTimeoutProducer)) {
            ok = false;
            break;
          }
          fence_proxy_async_smem();
          mbar_arrive_cluster(full_even + 8u * static_cast<uint32_t>(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (GATHER && warp >= 6) {
    // ------------------------------------------------------------ gathered B (both CTAs)
    // warp g copies kept rows 16g .. 16g+15 of each k-block: a row's run is cpr
    // 16-byte chunks (cpr = 16, or 8 for a 64-column half), rpi = 32 / cpr rows
    // per warp instruction; each lane holds the row numbers of its rows for the
    // current and the next k-block (loaded one k-block ahead, no shuffles; four
    // k-blocks ahead measured no faster).
    const int g = warp - 6;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int rows_next[8];
    auto load_rows = [&](int kb, int rpi, int (&dst)[8]) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int t = kb * 64 + g * 16 + j * rpi + lane / (32 / rpi);
        dst[j] = (j * rpi < 16 && t < p.k) ? __ldg(p.gidx + t) : -1;
      }
    };
    GemmWork wk;
    int cur_rpi = 0;
    for (int it = 0; ok && gemm_work<256>(p, total_tiles, it, wk, npairs, pair); ++it) {
      int b, m0, nt;
      pair_tile_coords(p, wk.tile, b, m0, nt);
      const int half = wk.w / 2;
      const int cpr = half / 8;   // chunks per row: 16 (128 columns) or 8 (64)
      const int rpi = 32 / cpr;   // rows per warp instruction: 2 or 4
      const int nb = SWIGLU ? nt * 128 + wk.n_off / 2 : nt * 256 + wk.n_off + static_cast<int>(rank) * half;
      const uint16_t* W = (SWIGLU && rank == 1) ? p.gw1 : p.gw0;
      const int c16 = lane % cpr;
      const int col = nb + c16 * 8;
      uint32_t col_bytes = 0;
      if (col < p.N) col_bytes = (col + 8 <= p.N) ? 16u : static_cast<uint32_t>((p.N - col) * 2);
      const int atom = c16 >> 3, cw = c16 & 7;
      if (rpi != cur_rpi) {
        load_rows(0, rpi, rows_next);
        cur_rpi = rpi;
      }
      for (int kb = 0; kb < p.num_kb; ++kb) {
        int rows[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) rows[j] = rows_next[j];
        load_rows(kb + 1 < p.num_kb ? kb + 1 : 0, rpi, rows_next);
        int go = 1;
        if (lane == 0) go = mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kDevErrTimeoutProducer) ? 1 : 0;
        go = __shfl_sync(0xffffffffu, go, 0);
        if (!go) {
          ok = false;
          break;
        }
        const uint32_t dst0 = smem_u32(sB + stage * C::B_BYTES) + static_cast<uint32_t>(atom * 8192);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j * rpi < 16) {
            const int r = g * 16 + j * rpi + lane / cpr;  // kept row within the k-block
            const uint32_t dst = dst0 + static_cast<uint32_t>(r * 128 + ((cw ^ (r & 7)) << 4));
            const int64_t src_row = rows[j];
            const uint16_t* src = W;
            uint32_t bytes = 0;
            if (src_row >= 0 && col_bytes != 0) {
              src = W + src_row * p.gldw + col;
              bytes = col_bytes;
            }
            pair_cp_async16(dst, src, bytes);
          }
        }
        // this thread is counted on the stage once its copies have landed: on the
        // even CTA straight on the MMA's full barrier, on the odd CTA on bfull (the
        // forwarder passes it on); no waits here, so every stage can be in flight
        pair_cp_async_arrive_noinc(rank == 0 ? &full[stage] : &bfull[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // nothing may land after exit (the abort path leaves copies in flight)
    pair_cp_async_wait_all();
    (void)ok;
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    uint8_t* ebuf = sE + (warp - 2) * 8192;
    int acc_i = 0;
    int seq = 0;
    GemmWork wk;
    for (int it = 0; gemm_work<256>(p, total_tiles, it, wk, npairs, pair); ++it) {
      int b, m0, nt;
      pair_tile_coords(p, wk.tile, b, m0, nt);
      const int n0 = SWIGLU ? nt * 128 + wk.n_off / 2 : nt * 256 + wk.n_off;
      const int row0 = m0 + static_cast<int>(rank) * 128 + quarter * 32;
      const int out_w = SWIGLU ? wk.w / 2 : wk.w;  // output columns of this unit
      const int acc = acc_i & 1;
      if (!mbar_wait(&tfull[acc], (acc_i >> 1) & 1, abort_flag, kDevErrTimeoutEpilogue, 64)) break;
      tc_fence_after();
      for (int c = 0; c < out_w / 64; ++c) {
        uint32_t w[32];
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t r[32];
          tmem_ld32(lane_base + static_cast<uint32_t>(acc * 256 + c * 64 + h * 32), r);
          tmem_ld_wait();
          if (SWIGLU) {
            uint32_t u[32];
            tmem_ld32(lane_base + static_cast<uint32_t>(acc * 256 + out_w + c * 64 + h * 32), u);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float g = __uint_as_float(r[e]);
              r[e] = __float_as_uint(g / (1.f + __expf(-g)) * __uint_as_float(u[e]));
            }
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const __nv_bfloat162 t2 = __floats2bfloat162_rn(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
            w[h * 16 + e] = *reinterpret_cast<const uint32_t*>(&t2);
          }
        }
        const int col0 = n0 + c * 64;
        uint8_t* buf = ebuf + (seq & 1) * 4096;
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(&tempty[acc]);
        else mbar_arrive_cluster(tempty_even + 8u * static_cast<uint32_t>(acc));
      }
      ++acc_i;
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync();  // both CTAs are done with every MMA, copy and accumulator
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace rmm
