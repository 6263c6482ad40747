// Decode attention against a key/value cache (one query row per head), reduced
// along the contraction axis ("Algorithm Deep-Dive: RMM", Component mapping and
// Engineering Notes: decode prunes attention; "RMM: 把 Transformer 矩阵乘法切到
// 刚好够用", sections on QK^T and PV).
//
// The G = Hq / Hkv query rows that share a key/value head form the rows of A, so
// each key/value group has one index set and its cache is read once for the
// whole group:
//   QK^T:  I_g = TopK over head dims of the column norms of Q_g [G, dh];
//          S[h, j] = scale * sum_{t in I_g} Q[h, t] Kt_g[t, j]   (Kt: dim-major cache)
//   PV:    I_g = TopK over token positions of the column norms of P_g [G, nk];
//          O[h, :] = sum_{j in I_g} P[h, j] V_g[j, :]            (V: token-major cache)
// With G query rows these are GEMV-shaped and bound by reading the kept cache
// rows, so they run on the CUDA cores: every kept row is read once with 16-byte
// loads, several rows in flight per thread, products accumulated in fp32.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace rmm {

constexpr int kDecodeQkMaxK = 512;  // head dims kept per group (dh <= 512)

struct DecodeQkParams {
  const uint16_t* Q;   // bf16 [groups * G][dh]
  const uint16_t* Kt;  // bf16 [groups][dh][ldk]: dim-major key cache
  float* S;            // fp32 [groups * G][lds]
  const int32_t* idx;  // [groups][k] kept dims (ascending), or null: all dims
  int64_t nk, ldk, lds;
  int dh, k;
  float scale;
};

constexpr int kDecodePvMaxChunk = 512;  // kept positions per CTA

struct DecodePvParams {
  const uint16_t* P;   // bf16 [groups * G][ldp]
  const uint16_t* V;   // bf16 [groups][cap][DH]: token-major value cache
  const int32_t* idx;  // [groups][k] kept positions (ascending), or null: positions 0..k-1
  float* partial;      // fp32 [groups][splits][G][DH]
  int64_t ldp, cap;
  int k, chunk, splits;
};

// grid (splits, groups), 256 threads: DH / 8 threads per V row, 256 / (DH / 8)
// rows in flight per pass; dynamic shared memory: [rows per pass][G][DH] fp32
// partial sums, added in a fixed order at the end (deterministic).
template <int G, int DH>
__global__ void __launch_bounds__(256) decode_pv_kernel(const DecodePvParams p) {
  constexpr int TPR = DH / 8;
  constexpr int SLOTS = 256 / TPR;
  __shared__ float ps[G][kDecodePvMaxChunk];
  __shared__ int pos[kDecodePvMaxChunk];
  extern __shared__ float red[];  // [SLOTS][G][DH]
  wait_prior_kernels();
  const int64_t grp = blockIdx.y;
  const int split = blockIdx.x;
  const int c0 = split * p.chunk;
  const int cnt = (p.k - c0) < p.chunk ? (p.k - c0) : p.chunk;
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
    const int j = p.idx ? __ldg(p.idx + grp * p.k + c0 + i) : c0 + i;
    pos[i] = j;
#pragma unroll
    for (int h = 0; h < G; ++h) ps[h][i] = bf16lo(static_cast<uint32_t>(__ldg(p.P + (grp * G + h) * p.ldp + j)));
  }
  __syncthreads();
  const int slot = threadIdx.x / TPR;
  const int cx = (threadIdx.x % TPR) * 8;
  const uint16_t* vb = p.V + grp * p.cap * DH + cx;
  float acc[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[h][e] = 0.f;
  constexpr int U = 4;
  for (int i0 = slot; i0 < cnt; i0 += U * SLOTS) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * SLOTS;
      v[u] = (i < cnt) ? ldg_nc_v4(vb + static_cast<int64_t>(pos[i]) * DH) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * SLOTS;
      if (i >= cnt) break;
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float x = (e & 1) ? bf16hi(w[e >> 1]) : bf16lo(w[e >> 1]);
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h][e] = fmaf(ps[h][i], x, acc[h][e]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) red[(slot * G + h) * DH + cx + e] = acc[h][e];
  __syncthreads();
  float* out = p.partial + ((grp * p.splits + split) * G) * DH;
  for (int o = threadIdx.x; o < G * DH; o += blockDim.x) {
    float s = 0.f;
    for (int q = 0; q < SLOTS; ++q) s += red[q * G * DH + o];
    out[o] = s;
  }
}

// O[grp * G + h][c] = bf16(sum over splits, in order, of the partials); one CTA
// per group, G * DH threads.
__global__ void __launch_bounds__(1024) decode_pv_fixup_kernel(const float* partial, uint16_t* O, int splits, int gd) {
  wait_prior_kernels();
  const int64_t grp = blockIdx.x;
  const int o = threadIdx.x;
  if (o >= gd) return;
  const float* src = partial + grp * splits * gd + o;
  float s = 0.f;
  for (int q = 0; q < splits; ++q) s += src[static_cast<int64_t>(q) * gd];
  const __nv_bfloat16 b = __float2bfloat16_rn(s);
  O[grp * gd + o] = *reinterpret_cast<const uint16_t*>(&b);
}

}  // namespace rmm

namespace rmm {

// ---------------------------------------------------------------- QK^T, staged rows
// The same scores with the kept dim-rows staged in shared memory by 1-D bulk
// copies: a CTA owns 2048 tokens of one group; one producer thread copies the
// 4 KB slice of every kept row into a ring of kDqkStages stages (two rows per
// stage), eight consumer warps (8 tokens per thread) multiply out of shared
// memory.  About 48 KB per CTA stays in flight without holding registers.
constexpr int kDqkTokens = 2048;
constexpr int kDqkRowsPerStage = 2;
constexpr int kDqkStages = 6;
constexpr uint32_t kDqkRowBytes = kDqkTokens * 2;
constexpr uint32_t kDqkStageBytes = kDqkRowsPerStage * kDqkRowBytes;

// grid (ceil(nk / 2048), groups), 288 threads; dynamic shared memory: the ring.
template <int G>
__global__ void __launch_bounds__(288) decode_qk_staged_kernel(const DecodeQkParams p) {
  extern __shared__ __align__(128) uint8_t dqk_ring[];
  __shared__ float qs[G][kDecodeQkMaxK];
  __shared__ int rows[kDecodeQkMaxK];
  __shared__ uint64_t full[kDqkStages], empty[kDqkStages];
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t grp = blockIdx.y;
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * kDqkTokens;
  const int64_t jn = (p.nk - j0) < kDqkTokens ? (p.nk - j0) : kDqkTokens;  // tokens of this CTA
  const uint32_t row_bytes = static_cast<uint32_t>((jn + 7) / 8 * 16);     // stays inside the row: ldk % 8 == 0
  const int k = p.k;
  const int nst = (k + kDqkRowsPerStage - 1) / kDqkRowsPerStage;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDqkStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  wait_prior_kernels();
  const int32_t* I = p.idx ? p.idx + grp * k : nullptr;
  for (int t = threadIdx.x; t < k; t += blockDim.x) {
    const int r = I ? __ldg(I + t) : t;
    rows[t] = r;
#pragma unroll
    for (int h = 0; h < G; ++h)
      qs[h][t] = bf16lo(static_cast<uint32_t>(__ldg(p.Q + (grp * G + h) * p.dh + r))) * p.scale;
  }
  __syncthreads();
  const uint16_t* kt = p.Kt + grp * p.dh * p.ldk + j0;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0;
      bool ok = true;
      for (int st = 0; st < nst; ++st) {
        const int s = st % kDqkStages;
        const int use = st / kDqkStages;
        if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1, abort_flag, kDevErrTimeoutProducer)) {
          ok = false;
          break;
        }
        const int r0 = st * kDqkRowsPerStage;
        const int nr = (k - r0) < kDqkRowsPerStage ? (k - r0) : kDqkRowsPerStage;
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nr) * row_bytes);
        for (int q = 0; q < nr; ++q)
          bulk_load_1d(dqk_ring + s * kDqkStageBytes + q * kDqkRowBytes, kt + static_cast<int64_t>(rows[r0 + q]) * p.ldk,
                       row_bytes, &full[s]);
        ++issued;
      }
      if (!ok) {
        // wait (bounded) for the copies already issued so none lands after exit
        for (int s = 0; s < kDqkStages; ++s) {
          const uint32_t uses = (issued + kDqkStages - 1 - s) / kDqkStages;
          if (uses == 0) continue;
          const uint32_t a = smem_u32(&full[s]);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(a, (uses - 1) & 1u) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
    return;
  }
  // -------------------------------------------------------------- consumers
  float acc[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[h][e] = 0.f;
  const uint32_t base = smem_u32(dqk_ring) + threadIdx.x * 16;
  for (int st = 0; st < nst; ++st) {
    const int s = st % kDqkStages;
    if (!mbar_wait(&full[s], (st / kDqkStages) & 1, abort_flag, kDevErrTimeoutEpilogue)) break;
    const int r0 = st * kDqkRowsPerStage;
    const int nr = (k - r0) < kDqkRowsPerStage ? (k - r0) : kDqkRowsPerStage;
    uint4 v[kDqkRowsPerStage];
#pragma unroll
    for (int q = 0; q < kDqkRowsPerStage; ++q)
      v[q] = (q < nr) ? lds_v4(base + s * kDqkStageBytes + q * kDqkRowBytes) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int q = 0; q < kDqkRowsPerStage; ++q) {
      if (q >= nr) break;
      const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float x = (e & 1) ? bf16hi(w[e >> 1]) : bf16lo(w[e >> 1]);
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h][e] = fmaf(qs[h][r0 + q], x, acc[h][e]);
      }
    }
    // release the stage only once its values are consumed, with the warp's reads
    // ordered before the producer's next bulk copy into it
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  const int64_t jt = j0 + threadIdx.x * 8;
  if (jt >= p.nk) return;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float* sp = p.S + (grp * G + h) * p.lds + jt;
    if (jt + 8 <= p.nk) {
      reinterpret_cast<float4*>(sp)[0] = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
      reinterpret_cast<float4*>(sp)[1] = make_float4(acc[h][4], acc[h][5], acc[h][6], acc[h][7]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (jt + e < p.nk) sp[e] = acc[h][e];
    }
  }
}

}  // namespace rmm
