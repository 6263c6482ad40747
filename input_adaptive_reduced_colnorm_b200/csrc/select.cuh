// TopK selection of the k = ceil(rho d) largest column scores, lower index on
// ties, emitted in ascending index order ("Algorithm Deep-Dive: RMM", Core
// Approach: keep the TopK-largest ceil(rho d); tie rule and order are readings).
//
// One CTA per selection row.  Keys are the fp64 sums of squares q_j; for
// non-negative doubles the IEEE bit pattern orders like the value, so the k-th
// largest key is found by an MSB-first radix select on the 64-bit pattern:
//   * the top 32 bits of every key are staged in shared memory with coalesced
//     loads (thread t then owns the contiguous indices [t*KPT, (t+1)*KPT) and
//     keeps them in registers);
//   * leading bits shared by all keys are skipped (block-wide AND/OR), and each
//     pass resolves the next 12 bits with one 4096-bin shared histogram;
//   * the low 32 bits are fetched from global memory only for keys that still
//     tie on the top 32 bits (exact or near-exact ties);
//   * a pass stops early as soon as the bucket holding the k-th key is taken
//     whole.
// The final compaction is two block-wide prefix scans in index order, which
// gives the lower-index tie rule and the ascending order without any sort.
// All counts are integers, so the result does not depend on atomic ordering.
#pragma once
#include "ptx.cuh"

namespace rmm {

struct SelectParams {
  const double* colsq;  // [batch][d]
  int64_t d;
  int64_t k;
  int32_t* idx;         // [batch][k]
  double* retained;     // [batch] or nullptr: sum_{j in I} q_j / sum_j q_j
  uint8_t* keep;        // [batch][d] or nullptr: 1 where j is in I, else 0
};

constexpr int kSelBits = 12;
constexpr int kSelBins = 1 << kSelBits;

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

// Shared-memory slot of key j in the staging array: one padding word per 32
// keys, so that thread t reading its KPT contiguous keys (t * KPT + e) hits 32
// different banks for every power-of-two KPT <= 32.
__device__ __forceinline__ int sel_slot(int j) { return j + (j >> 5); }

// dynamic shared memory: hi32 keys [NT * KPT + NT * KPT / 32] (uint32, padded)
template <int KPT, int NT>
__global__ void __launch_bounds__(NT) select_kernel(const SelectParams p) {
  wait_prior_kernels();
  constexpr int NW = NT / 32;
  constexpr int BPT = kSelBins / NT;  // histogram bins scanned per thread
  static_assert(kSelBins % NT == 0, "bins must split evenly");
  static_assert(KPT <= 32 && (KPT & (KPT - 1)) == 0, "a thread's keys must lie in one padded block of 32");
  extern __shared__ __align__(16) uint32_t s_keys[];
  __shared__ uint32_t hist[kSelBins];
  __shared__ int s_warp[32];
  __shared__ int s_total;
  __shared__ int s_digit, s_above, s_cnt;
  __shared__ uint32_t s_and[32], s_or[32];
  __shared__ double s_sum[32];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t b = blockIdx.x;
  const double* q = p.colsq + b * p.d;
  int32_t* out = p.idx + b * p.k;
  const int d = static_cast<int>(p.d);
  const int j0 = threadIdx.x * KPT;

  // coalesced staging of the top 32 bits of every key, eight loads in flight
  // per thread before the first store
  for (int e0 = 0; e0 < KPT; e0 += 8) {
    constexpr int B = KPT < 8 ? KPT : 8;
    uint32_t v[B];
#pragma unroll
    for (int e = 0; e < B; ++e) {
      const int j = (e0 + e) * NT + threadIdx.x;
      v[e] = (j < d) ? static_cast<uint32_t>(static_cast<uint64_t>(__double_as_longlong(__ldg(q + j))) >> 32) : 0u;
    }
#pragma unroll
    for (int e = 0; e < B; ++e) {
      const int j = (e0 + e) * NT + threadIdx.x;
      if (j < d) s_keys[sel_slot(j)] = v[e];
    }
  }
  __syncthreads();
  // this thread's keys stay in shared memory (conflict-free by the padding) and
  // are re-read by each pass instead of being held in registers
  const uint32_t* my_keys = s_keys + sel_slot(j0);
  uint32_t valid = 0;
  uint32_t kand = 0xffffffffu, kor = 0u;
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    if (j0 + e < d) {
      const uint32_t h = my_keys[e];
      valid |= 1u << e;
      kand &= h;
      kor |= h;
    }
  }
  // bits on which all keys agree need no pass
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kand &= __shfl_xor_sync(0xffffffffu, kand, o);
    kor |= __shfl_xor_sync(0xffffffffu, kor, o);
  }
  if (lane == 0) {
    s_and[warp] = kand;
    s_or[warp] = kor;
  }
  __syncthreads();
  kand = 0xffffffffu;
  kor = 0u;
  for (int w = 0; w < NW; ++w) {
    kand &= s_and[w];
    kor |= s_or[w];
  }
  const uint32_t differ = kand ^ kor;  // bits not shared by every key

  uint32_t pre_hi = 0, msk_hi = 0, pre_lo = 0, msk_lo = 0;
  int need = static_cast<int>(p.k);
  bool take_bucket = (p.k == p.d);
  if (!take_bucket && differ == 0u) {
    // all top-32 bits equal: decide on the low 32 bits
    msk_hi = 0xffffffffu;
    pre_hi = kand;
  } else if (!take_bucket) {
    const int top = 31 - __clz(differ);  // highest differing bit
    msk_hi = (top == 31) ? 0u : (0xffffffffu << (top + 1));
    pre_hi = kand & msk_hi;
  }
  // bit cursor: position (in the 64-bit key) just above the next digit
  int cursor = 32 + ((msk_hi == 0xffffffffu) ? 0 : (32 - __popc(msk_hi)));

  bool lo_checked = false;
  while (!take_bucket && cursor > 0) {
    if (cursor <= 32 && !lo_checked) {
      // the high words are resolved: one AND / OR of the low words still in the
      // bucket skips their shared leading bits, and identical keys (exact ties,
      // e.g. the squares of a single bf16 row) end the passes at once
      lo_checked = true;
      uint32_t la = 0xffffffffu, lr = 0u;
#pragma unroll
      for (int e = 0; e < KPT; ++e) {
        if (((valid >> e) & 1u) && (my_keys[e] & msk_hi) == pre_hi) {
          const uint32_t lo = static_cast<uint32_t>(__double_as_longlong(q[j0 + e]));
          if ((lo & msk_lo) == pre_lo) {
            la &= lo;
            lr |= lo;
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        la &= __shfl_xor_sync(0xffffffffu, la, o);
        lr |= __shfl_xor_sync(0xffffffffu, lr, o);
      }
      __syncthreads();  // every thread has read s_and / s_or of the earlier reduction
      if (lane == 0) {
        s_and[warp] = la;
        s_or[warp] = lr;
      }
      __syncthreads();
      la = 0xffffffffu;
      lr = 0u;
      for (int w = 0; w < NW; ++w) {
        la &= s_and[w];
        lr |= s_or[w];
      }
      const uint32_t open = (cursor == 32) ? 0xffffffffu : ((1u << cursor) - 1u);  // unresolved low bits
      const uint32_t dl = (la ^ lr) & open;
      if (dl == 0u) {  // every key left has the same value: the lower indices win
        pre_lo = (pre_lo & ~open) | (la & open);
        msk_lo = 0xffffffffu;
        break;
      }
      const int top = 31 - __clz(dl);
      const uint32_t shared = open & ((top == 31) ? 0u : (0xffffffffu << (top + 1)));
      pre_lo |= la & shared;
      msk_lo |= shared;
      cursor = top + 1;
    }
    const int width = cursor >= kSelBits ? kSelBits : cursor;
    const int shift = cursor - width;  // bit position of the digit in the 64-bit key
    const uint32_t dmask = (1u << width) - 1u;
    for (int i = threadIdx.x; i < kSelBins; i += NT) hist[i] = 0u;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
      bool m = ((valid >> e) & 1u) && (my_keys[e] & msk_hi) == pre_hi;
      uint32_t dig = 0;
      if (m) {
        if (shift >= 32) {
          dig = (my_keys[e] >> (shift - 32)) & dmask;
        } else {
          const uint32_t lo = static_cast<uint32_t>(__double_as_longlong(q[j0 + e]));
          m = (lo & msk_lo) == pre_lo;
          if (shift + width > 32) {  // digit straddles the two halves
            const uint64_t full = (static_cast<uint64_t>(my_keys[e]) << 32) | lo;
            dig = static_cast<uint32_t>(full >> shift) & dmask;
          } else {
            dig = (lo >> shift) & dmask;
          }
        }
      }
      if (m) atomicAdd(&hist[dig], 1u);
    }
    __syncthreads();
    // descending suffix sums: bin b's "above" = count of larger digits
    uint32_t c[BPT];
    uint32_t ls = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      c[i] = hist[threadIdx.x * BPT + i];
      ls += c[i];
    }
    // larger digits live in higher threads: their count is total - before - own
    const int before = block_exclusive_scan<NT>(static_cast<int>(ls), s_warp, &s_total);
    const uint32_t total = static_cast<uint32_t>(s_total);
    uint32_t above = total - static_cast<uint32_t>(before) - ls;  // digits held by higher threads
#pragma unroll
    for (int i = BPT - 1; i >= 0; --i) {
      const int bin = threadIdx.x * BPT + i;
      if (bin <= static_cast<int>(dmask) && above < static_cast<uint32_t>(need) &&
          static_cast<uint32_t>(need) <= above + c[i]) {
        s_digit = bin;
        s_above = static_cast<int>(above);
        s_cnt = static_cast<int>(c[i]);
      }
      above += c[i];
    }
    __syncthreads();
    need -= s_above;
    const uint64_t dg = static_cast<uint64_t>(s_digit) << shift;
    const uint64_t dm = static_cast<uint64_t>(dmask) << shift;
    pre_hi |= static_cast<uint32_t>(dg >> 32);
    msk_hi |= static_cast<uint32_t>(dm >> 32);
    pre_lo |= static_cast<uint32_t>(dg);
    msk_lo |= static_cast<uint32_t>(dm);
    if (s_cnt == need) take_bucket = true;
    cursor = shift;
    __syncthreads();
  }

  // classify the owned keys: above the threshold bucket, or inside it
  uint32_t gt = 0, eq = 0;
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    if (!((valid >> e) & 1u)) continue;
    const uint32_t h = my_keys[e] & msk_hi;
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
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    if ((sel >> e) & 1u) out[pos++] = j0 + e;
  }
  if (p.keep != nullptr) {
    uint8_t* kp = p.keep + b * p.d;
#pragma unroll
    for (int e = 0; e < KPT; ++e)
      if ((valid >> e) & 1u) kp[j0 + e] = static_cast<uint8_t>((sel >> e) & 1u);
  }
  if (p.retained != nullptr) {
    double kept = 0.0, all = 0.0;
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
  wait_prior_kernels();
  const int64_t total = batch * d;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x)
    idx[t] = static_cast<int32_t>(t % d);
}

}  // namespace rmm
