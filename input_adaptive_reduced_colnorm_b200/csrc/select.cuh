// TopK selection of the k = ceil(rho d) largest column scores, lower index on
// ties, emitted in ascending index order ("Algorithm Deep-Dive: RMM", Core
// Approach: keep the TopK-largest ceil(rho d); tie rule and order are readings).
//
// One CTA per selection row.  Keys are the fp64 sums of squares q_j; for
// non-negative doubles the IEEE bit pattern orders like the value, so the
// k-th largest key is found by an MSB-first radix select on the 64-bit
// pattern, 8 bits per pass.  The top 32 bits of every key live in registers
// (thread t owns the contiguous indices [t*KPT, (t+1)*KPT)); the low 32 bits
// are fetched from global memory only for keys that still tie on the top 32
// bits, which happens only for (near-)exact ties.  A pass stops early as soon
// as the bucket holding the k-th key is taken whole.  The final compaction is
// two block-wide prefix scans in index order, which yields the lower-index tie
// rule and the ascending order without any sort.  All counts are integers, so
// the result does not depend on atomic ordering.
#pragma once
#include "ptx.cuh"

namespace rmm {

struct SelectParams {
  const double* colsq;  // [batch][d]
  int64_t d;
  int64_t k;
  int32_t* idx;         // [batch][k]
  double* retained;     // [batch] or nullptr: sum_{j in I} q_j / sum_j q_j
};

template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* s_total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < NW) ? s_warp[lane] : 0;
    int t = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < NW) s_warp[lane] = t - w;  // exclusive prefix of warp totals
    if (lane == NW - 1) *s_total = t;
  }
  __syncthreads();
  const int r = s_warp[warp] + x - v;
  __syncthreads();
  return r;
}

template <int NT>
__device__ __forceinline__ double block_sum_f64(double v, double* s_buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  if (lane == 0) s_buf[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < NT / 32; ++w) t += s_buf[w];
  __syncthreads();
  return t;  // valid in thread 0 only
}

template <int KPT, int NT>
__global__ void __launch_bounds__(NT) select_kernel(const SelectParams p) {
  constexpr int NW = NT / 32;
  __shared__ uint32_t whist[NW][256];
  __shared__ uint32_t hist[256];
  __shared__ int s_digit, s_above, s_cnt;
  __shared__ int s_warp[32];
  __shared__ int s_total;
  __shared__ double s_sum[32];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t b = blockIdx.x;
  const double* q = p.colsq + b * p.d;
  int32_t* out = p.idx + b * p.k;
  const int64_t j0 = static_cast<int64_t>(threadIdx.x) * KPT;

  uint32_t hi[KPT];
  uint32_t valid = 0;
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    const int64_t j = j0 + e;
    hi[e] = 0u;
    if (j < p.d) {
      hi[e] = static_cast<uint32_t>(static_cast<uint64_t>(__double_as_longlong(q[j])) >> 32);
      valid |= 1u << e;
    }
  }

  uint32_t pre_hi = 0, msk_hi = 0, pre_lo = 0, msk_lo = 0;
  int need = static_cast<int>(p.k);
  bool take_bucket = (p.k == p.d);  // everything is kept: nothing to rank

  for (int pass = 0; pass < 8 && !take_bucket; ++pass) {
    for (int i = threadIdx.x; i < NW * 256; i += NT) (&whist[0][0])[i] = 0u;
    __syncthreads();
    const int shift = 24 - 8 * (pass & 3);
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
      bool m = ((valid >> e) & 1u) && ((hi[e] & msk_hi) == pre_hi);
      uint32_t dig = 0;
      if (m) {
        if (pass < 4) {
          dig = (hi[e] >> shift) & 255u;
        } else {
          const uint32_t lo = static_cast<uint32_t>(__double_as_longlong(q[j0 + e]));
          m = (lo & msk_lo) == pre_lo;
          dig = (lo >> shift) & 255u;
        }
      }
      const uint32_t key = m ? dig : (256u + lane);
      const uint32_t grp = __match_any_sync(0xffffffffu, key);
      if (m && lane == __ffs(grp) - 1) atomicAdd(&whist[warp][dig], static_cast<uint32_t>(__popc(grp)));
    }
    __syncthreads();
    for (int bin = threadIdx.x; bin < 256; bin += NT) {
      uint32_t s = 0;
      for (int w = 0; w < NW; ++w) s += whist[w][bin];
      hist[bin] = s;
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t c[8];
      uint32_t ls = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[lane * 8 + i];
        ls += c[i];
      }
      // sum over lanes above this one (bins with larger digits)
      uint32_t incl = ls;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += y;
      }
      uint32_t above = incl - ls;
#pragma unroll
      for (int i = 7; i >= 0; --i) {
        if (above < static_cast<uint32_t>(need) && static_cast<uint32_t>(need) <= above + c[i]) {
          s_digit = lane * 8 + i;
          s_above = static_cast<int>(above);
          s_cnt = static_cast<int>(c[i]);
        }
        above += c[i];
      }
    }
    __syncthreads();
    need -= s_above;
    if (pass < 4) {
      pre_hi |= static_cast<uint32_t>(s_digit) << shift;
      msk_hi |= 255u << shift;
    } else {
      pre_lo |= static_cast<uint32_t>(s_digit) << shift;
      msk_lo |= 255u << shift;
    }
    if (s_cnt == need) take_bucket = true;
    __syncthreads();
  }

  // classify the owned keys: greater than the threshold bucket, or inside it
  uint32_t gt = 0, eq = 0;
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    if (!((valid >> e) & 1u)) continue;
    const uint32_t h = hi[e] & msk_hi;
    if (h > pre_hi) {
      gt |= 1u << e;
    } else if (h == pre_hi) {
      if (msk_lo == 0u) {
        eq |= 1u << e;
      } else {
        const uint32_t lo = static_cast<uint32_t>(__double_as_longlong(q[j0 + e])) & msk_lo;
        if (lo > pre_lo) gt |= 1u << e;
        else if (lo == pre_lo) eq |= 1u << e;
      }
    }
  }
  uint32_t sel = gt;
  if (take_bucket) {
    sel |= eq;
  } else {
    // keep the first `need` bucket members in index order
    const int before = block_exclusive_scan<NT>(__popc(eq), s_warp, &s_total);
    int r = before;
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
      if ((eq >> e) & 1u) {
        if (r < need) sel |= 1u << e;
        ++r;
      }
    }
  }
  const int pos0 = block_exclusive_scan<NT>(__popc(sel), s_warp, &s_total);
  int pos = pos0;
  double kept = 0.0, all = 0.0;
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    if ((sel >> e) & 1u) out[pos++] = static_cast<int32_t>(j0 + e);
  }
  if (p.retained != nullptr) {
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
      if ((valid >> e) & 1u) {
        const double v = q[j0 + e];
        all += v;
        if ((sel >> e) & 1u) kept += v;
      }
    }
    const double tk = block_sum_f64<NT>(kept, s_sum);
    const double ta = block_sum_f64<NT>(all, s_sum);
    if (threadIdx.x == 0) p.retained[b] = (ta > 0.0) ? tk / ta : 1.0;
  }
}

// I = [0, d) for the rho = 1 path when the caller asks for the index set.
__global__ void iota_kernel(int32_t* idx, int64_t batch, int64_t d) {
  const int64_t total = batch * d;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x)
    idx[t] = static_cast<int32_t>(t % d);
}

}  // namespace rmm
