// C ABI of the RMM library: argument checks, workspace layout, tensor maps and
// the launch sequence of each entry point.  See include/rmm.h for the contract.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "rmm.h"
#include "ptx.cuh"
#include "colsq.cuh"
#include "select.cuh"
#include "pack.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "gemv.cuh"
#include "decode_attn.cuh"
#include "gemv_i8.cuh"
#include "attention.cuh"
#include "decode_select.cuh"

using namespace rmm;

namespace {

thread_local std::string t_last_error;

rmm_status fail(rmm_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

rmm_status cuda_fail(cudaError_t e, const char* what) {
  return fail(RMM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }
inline int64_t ceil_div(int64_t x, int64_t m) { return (x + m - 1) / m; }

constexpr int64_t kMaxSelectD = 32768;
constexpr int64_t kOneCtaMaxRows = 128;  // products of at most this many rows run on one-CTA tiles
constexpr int64_t kIntMax = 2147483647LL;

// ---------------------------------------------------------------- device facts
int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 or fp32 tensor map with 128-byte swizzle; OOB elements read as 0.
rmm_status make_tmap(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                     uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(RMM_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RMM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return RMM_OK;
}

// 3-D output map [batch][rows][cols] for the GEMM's TMA-store epilogue: boxes of
// 32 rows x 128 bytes (32 fp32 or 64 bf16 columns), 128-byte swizzle; stores are
// clipped to each batch item's rows and columns.
rmm_status make_tmap_out(CUtensorMap* tm, const void* base, bool f32, uint64_t cols, uint64_t rows, uint64_t batch,
                         uint64_t ld, uint64_t bstride) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(RMM_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const uint64_t eb = f32 ? 4 : 2;
  cuuint64_t dims[3] = {cols, rows, batch};
  cuuint64_t strides[2] = {ld * eb, (batch > 1 ? bstride : rows * ld) * eb};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / eb), 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(tm, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RMM_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d)", static_cast<int>(r));
  return RMM_OK;
}

// Launch with programmatic stream serialisation (see wait_prior_kernels()).
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                           Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- workspace carving
struct Carver {
  uint8_t* base;
  size_t cur = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <typename T>
  T* take(int64_t count) {
    cur = (cur + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + cur) : nullptr;
    cur += static_cast<size_t>(count) * sizeof(T);
    return p;
  }
  size_t bytes() const { return (cur + 255) & ~size_t(255); }
};

// ---------------------------------------------------------------- launches
// Cluster launch with programmatic stream serialisation.
template <typename... KArgs, typename... Args>
cudaError_t launch_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, int csize, cudaStream_t s,
                           Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(csize);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Column sums of squares through shared-memory tiles (colsq_tma_kernel).  The
// strip width W and the cluster size C are chosen so that one wave of two CTAs
// per SM holds as many CTAs as possible while every CTA keeps at least two
// tiles; problems larger than a wave take W = 256 and C up to 8 (at least four
// tiles per CTA) so that no single CTA is long enough to leave a tail.
template <int W, bool CAUSAL>
rmm_status launch_colsq_tma_t(const CUtensorMap& tm, const ColsqTmaParams& p, int64_t strips, int64_t batch,
                              cudaStream_t s) {
  constexpr size_t smem = static_cast<size_t>(kColsqStages) * kColsqTileBytes;
  cudaError_t e = cudaFuncSetAttribute(colsq_tma_kernel<W, CAUSAL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "column-norm attribute");
  e = launch_cluster(colsq_tma_kernel<W, CAUSAL>, dim3(static_cast<unsigned>(strips * p.csize), static_cast<unsigned>(batch)),
                     dim3(kColsqThreads), smem, p.csize, s, tm, p);
  if (e != cudaSuccess) return cuda_fail(e, "column-norm launch");
  return RMM_OK;
}

rmm_status launch_colsq_tma(const uint16_t* A, int64_t batch, int64_t bstride, int64_t n, int64_t d, int64_t lda,
                            bool causal, int64_t off, double* colsq, cudaStream_t s) {
  const int64_t wave = 2LL * num_sms();
  int W = 0, C = 0;
  int64_t best = 0;
  for (int w = 256; w >= 64; w /= 2) {
    // a strip twice as wide as the matrix stages (and sums) as many zero columns
    // as real ones: the narrower strip holds twice the rows per tile
    if (w > 64 && w >= 2 * d) continue;
    const int64_t R = kColsqTileBytes / (2 * w);
    for (int c = 1; c <= 8; c *= 2) {
      if (c > 1 && n < c * 2 * R) break;
      const int64_t ctas = ceil_div(d, w) * batch * c;
      if (ctas <= wave && ctas > best) {
        best = ctas;
        W = w;
        C = c;
      }
    }
  }
  if (best == 0) {
    W = 256;
    const int64_t R = kColsqTileBytes / (2 * W);
    C = 1;
    while (C < 8 && n >= 2 * C * 4 * R) C *= 2;
  }
  const int64_t strips = ceil_div(d, W);
  if (strips * C > kIntMax || batch > 65535 || n > kIntMax || d > kIntMax)
    return fail(RMM_ERR_UNSUPPORTED, "column-norm grid too large");

  auto fn = encode_fn();
  if (fn == nullptr) return fail(RMM_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  CUtensorMap tm;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n), static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(lda) * 2,
                           static_cast<cuuint64_t>(batch > 1 ? bstride : n * lda) * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(W), static_cast<cuuint32_t>(kColsqTileBytes / (2 * W)), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(A), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RMM_ERR_CUDA, "cuTensorMapEncodeTiled (column norms) failed (%d)", static_cast<int>(r));

  ColsqTmaParams p{};
  p.n = n;
  p.d = d;
  p.causal_off = off;
  p.colsq = colsq;
  p.csize = C;
#define RMM_COLSQ_TMA_CASE(w)                                                          \
  case w:                                                                              \
    return causal ? launch_colsq_tma_t<w, true>(tm, p, strips, batch, s)               \
                  : launch_colsq_tma_t<w, false>(tm, p, strips, batch, s);
  switch (W) {
    RMM_COLSQ_TMA_CASE(256)
    RMM_COLSQ_TMA_CASE(128)
    RMM_COLSQ_TMA_CASE(64)
  }
#undef RMM_COLSQ_TMA_CASE
  return fail(RMM_ERR_UNSUPPORTED, "column-norm strip width");
}

// Column sums of squares.  Matrices of 64 rows or more whose batch items start
// on 16-byte boundaries stream through shared memory with TMA
// (colsq_tma_kernel); short ones (decode rows) and oddly strided batches use
// the register kernel, whose 16-row bursts of direct loads finish a few rows in
// one round trip.
rmm_status launch_colsq(const uint16_t* A, int64_t batch, int64_t bstride, int64_t n, int64_t d, int64_t lda,
                        bool causal, int64_t off, double* colsq, cudaStream_t s) {
  if (n >= 64 && (batch == 1 || bstride % 8 == 0)) return launch_colsq_tma(A, batch, bstride, n, d, lda, causal, off, colsq, s);
  if (!causal && n <= kColsqShortMaxRows) {
    if (batch > 65535) return fail(RMM_ERR_UNSUPPORTED, "column-norm grid too large");
    ColsqParams p{};
    p.A = A;
    p.batch_stride = bstride;
    p.n = n;
    p.d = d;
    p.lda = lda;
    p.colsq = colsq;
    const dim3 grid(static_cast<unsigned>(ceil_div(d, 1024)), static_cast<unsigned>(batch));
    const cudaError_t e = launch_chained(colsq_short_kernel, grid, dim3(128), 0, s, p);
    if (e != cudaSuccess) return cuda_fail(e, "column-norm launch");
    return RMM_OK;
  }
  // Register kernel: pick the strip width (TX threads x 8 columns) and the
  // cluster size C (CTAs splitting a strip's rows) so that the grid fits in one
  // wave of two CTAs per SM with as many CTAs as possible; larger problems
  // simply take several waves.
  const int64_t wave = 2LL * num_sms();
  int C = 0, TX = 0;
  int64_t best = 0;
  for (int tx = 32; tx >= 4; tx /= 2) {
    for (int c = 1; c <= 8; c *= 2) {
      if (c > 1 && n / c < 64) break;  // keep at least 64 rows per CTA
      const int64_t ctas = ceil_div(d, tx * 8) * batch * c;
      if (ctas <= wave && ctas > best) {
        best = ctas;
        C = c;
        TX = tx;
      }
    }
  }
  if (best == 0) {  // even the smallest grid exceeds one wave: widest strips, full clusters
    TX = 32;
    C = 1;
    while (C < 8 && n / (2 * C) >= 128) C *= 2;
  }
  const int64_t strips = ceil_div(d, TX * 8);
  if (strips * C > kIntMax || batch > 65535) return fail(RMM_ERR_UNSUPPORTED, "column-norm grid too large");
  ColsqParams p{};
  p.A = A;
  p.batch_stride = bstride;
  p.n = n;
  p.d = d;
  p.lda = lda;
  p.causal_off = off;
  p.colsq = colsq;
  p.rows_per_cta = ceil_div(n, C);
  p.csize = C;
  const dim3 grid(static_cast<unsigned>(strips * C), static_cast<unsigned>(batch), 1);
  cudaError_t e = cudaSuccess;
#define RMM_COLSQ_CASE(tx)                                                                                  \
  case tx:                                                                                                  \
    e = causal ? launch_cluster(colsq_kernel<tx, true>, grid, dim3(256), 0, C, s, p)                        \
               : launch_cluster(colsq_kernel<tx, false>, grid, dim3(256), 0, C, s, p);                      \
    break;
  switch (TX) {
    RMM_COLSQ_CASE(32)
    RMM_COLSQ_CASE(16)
    RMM_COLSQ_CASE(8)
    RMM_COLSQ_CASE(4)
  }
#undef RMM_COLSQ_CASE
  if (e != cudaSuccess) return cuda_fail(e, "column-norm launch");
  return RMM_OK;
}

template <int KPT, int NT>
rmm_status launch_select_t(const SelectParams& p, int64_t batch, cudaStream_t s) {
  // dynamic keys plus ~17 KB of static histogram and scan space can pass 48 KB
  const size_t smem = static_cast<size_t>(NT) * KPT * sizeof(uint32_t) * 33 / 32 + sizeof(uint32_t);
  {
    const cudaError_t e = cudaFuncSetAttribute(select_kernel<KPT, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e, "select attribute");
  }
  const cudaError_t e = launch_chained(select_kernel<KPT, NT>, dim3(static_cast<unsigned>(batch)), dim3(NT), smem, s, p);
  if (e != cudaSuccess) return cuda_fail(e, "select launch");
  return RMM_OK;
}

rmm_status launch_select(const double* colsq, int64_t batch, int64_t d, int64_t k, int32_t* idx, double* retained,
                         cudaStream_t s, uint8_t* keep = nullptr) {
  SelectParams p{colsq, d, k, idx, retained, keep};
  if (d <= 128) return launch_select_t<1, 128>(p, batch, s);
  if (d <= 1024) return launch_select_t<1, 1024>(p, batch, s);
  if (d <= 2048) return launch_select_t<2, 1024>(p, batch, s);
  if (d <= 4096) return launch_select_t<4, 1024>(p, batch, s);
  if (d <= 8192) return launch_select_t<8, 1024>(p, batch, s);
  if (d <= 16384) return launch_select_t<16, 1024>(p, batch, s);
  return launch_select_t<32, 1024>(p, batch, s);
}

// Decode selection in one cluster launch (decode_select.cuh): scores, TopK,
// index set and (xpack != nullptr) x[:, I] zero-padded to ld_pack columns, for
// 1 <= n <= 32 rows and d <= kDecSelMaxD; callers use the three-kernel chain
// (scores, selection, pack) outside that range.
bool decode_select_fits(int64_t n, int64_t d) { return n >= 1 && n <= kDecSelMaxRows && d >= 1 && d <= kDecSelMaxD; }

rmm_status launch_decode_select(const uint16_t* x, int64_t n, int64_t d, int64_t ldx, int64_t k, int32_t* idx,
                                uint16_t* xpack, int64_t ld_pack, cudaStream_t s) {
  DecodeSelParams p{};
  p.x = x;
  p.ldx = ldx;
  p.n = static_cast<int>(n);
  p.d = static_cast<int>(d);
  p.k = static_cast<int>(k);
  p.idx = idx;
  p.xpack = xpack;
  p.ld_pack = ld_pack;
  // four columns per thread while a cluster of at most 8 CTAs covers d, else eight
  const bool four = d <= decsel_cols_per_cta(4) * kDecSelMaxCtas;
  const int C = static_cast<int>(ceil_div(d, decsel_cols_per_cta(four ? 4 : 8)));
  auto kern = four ? decode_select_kernel<4> : decode_select_kernel<8>;
  const int smem = decsel_stage_bytes(static_cast<int>(n), four ? 4 : 8);  // the staged rows
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "decode selection attribute");
  e = launch_cluster(kern, dim3(static_cast<unsigned>(C)), dim3(kDecSelThreads), static_cast<size_t>(smem), C, s, p);
  if (e != cudaSuccess) return cuda_fail(e, "decode selection launch");
  return RMM_OK;
}

rmm_status launch_pack(const PackParams& p, cudaStream_t s) {
  const int64_t rows = p.batch * p.rows;
  const int64_t d_round = round_up(p.d, 8);
  cudaError_t e;
  const bool narrow = (p.d == 64 || p.d == 128 || p.d == 256) && p.src_ld % 8 == 0 && p.k_pad <= 256 &&
                      p.k_pad % 2 == 0 && !p.causal && p.rows % 8 == 0 && p.d <= p.src_ld &&
                      (p.batch == 1 || (p.s_outer % 8 == 0 && p.s_inner % 8 == 0));
  if (narrow && rows >= 8192) {
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(ceil_div(rows / 8, 8), 6LL * num_sms()));
    auto kern = (p.d == 64) ? pack_narrow_rows_kernel<64> : (p.d == 128) ? pack_narrow_rows_kernel<128>
                                                                         : pack_narrow_rows_kernel<256>;
    e = launch_chained(kern, dim3(static_cast<unsigned>(grid)), dim3(256), 0, s, p);
    if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  } else if (p.d <= 512 && p.k_pad <= 256 && p.k_pad % 2 == 0) {
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(ceil_div(rows, 8 * 4), 8LL * num_sms()));
    e = launch_chained(pack_short_rows_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, s, p);
    if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  } else if (p.d <= 1024) {
    const size_t smem = static_cast<size_t>(8 * d_round * 2);
    const int64_t grid = std::min<int64_t>(ceil_div(rows, 8), 8LL * num_sms());
    e = launch_chained(pack_rows_warp_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), smem, s, p, d_round);
    if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  } else if (p.k_pad % 2 == 0 && (p.batch == 1 || (p.s_outer % 8 == 0 && p.s_inner % 8 == 0))) {
    // rows staged by bulk copies: as many row buffers (2 to 4) as fit in
    // ~110 KB, so that two CTAs share an SM even for the longest rows
    const uint32_t buf_bytes = static_cast<uint32_t>(round_up(d_round * 2, 128));
    const size_t idx_bytes = static_cast<size_t>(round_up(p.k_pad * 2, 16));
    int nbuf = 4;
    while (nbuf > 2 && nbuf * static_cast<size_t>(buf_bytes) + idx_bytes > 110 * 1024) --nbuf;
    const size_t smem = nbuf * static_cast<size_t>(buf_bytes) + idx_bytes;
    if (smem > 220 * 1024) return fail(RMM_ERR_UNSUPPORTED, "row too long for the pack kernel");
    auto kern = (nbuf == 4) ? pack_rows_bulk_kernel<4> : (nbuf == 3) ? pack_rows_bulk_kernel<3> : pack_rows_bulk_kernel<2>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e, "pack attribute");
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
    if (e != cudaSuccess || per_sm < 1) per_sm = 1;
    const int64_t grid = std::min<int64_t>(rows, static_cast<int64_t>(per_sm) * num_sms());
    e = launch_chained(kern, dim3(static_cast<unsigned>(grid)), dim3(256), smem, s, p, buf_bytes);
    if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  } else {
    // four row buffers for rows up to 8192 columns, two beyond (more CTAs per SM)
    const int64_t idx_elems = round_up(p.k_pad, 8);
    const int nbuf = (d_round <= 8192) ? 4 : 2;
    const size_t smem = static_cast<size_t>((idx_elems + nbuf * d_round) * 2);
    if (smem > 227 * 1024) return fail(RMM_ERR_UNSUPPORTED, "row too long for the pack kernel");
    auto kern = (nbuf == 4) ? pack_rows_cta_kernel<4> : pack_rows_cta_kernel<2>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e, "pack attribute");
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
    if (e != cudaSuccess || per_sm < 1) per_sm = 1;
    const int64_t grid = std::min<int64_t>(rows, static_cast<int64_t>(per_sm) * num_sms());
    e = launch_chained(kern, dim3(static_cast<unsigned>(grid)), dim3(256), smem, s, p, d_round, idx_elems);
    if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  return RMM_OK;
}

rmm_status launch_rowpack(const RowPackParams& p, cudaStream_t s) {
  if (p.rows_out == p.k && p.k > 0 && p.cols % 8 == 0 && p.src_ld % 8 == 0 && p.dst_ld % 8 == 0 &&
      (p.batch == 1 || (p.s_outer % 8 == 0 && p.s_inner % 8 == 0))) {
    // whole rows by bulk copies: two CTAs per SM, at most kRowpackMaxRows rows each
    const int64_t chunks = ceil_div(p.cols * 2, kRowpackChunk);
    const int64_t rows = p.batch * p.k;
    if (chunks > kIntMax) return fail(RMM_ERR_UNSUPPORTED, "rows too long for the row pack");
    const int64_t grid = std::min<int64_t>(rows, std::max<int64_t>(2LL * num_sms(), ceil_div(rows, kRowpackMaxRows)));
    const size_t smem = static_cast<size_t>(kRowpackStages) * kRowpackChunk + kRowpackMaxRows * sizeof(int32_t);
    cudaError_t e = cudaFuncSetAttribute(pack_rows_bulk_copy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e, "row pack attribute");
    e = launch_chained(pack_rows_bulk_copy_kernel, dim3(static_cast<unsigned>(grid)), dim3(32), smem, s, p,
                       static_cast<int>(chunks));
    if (e != cudaSuccess) return cuda_fail(e, "row pack launch");
    return RMM_OK;
  }
  // threads per row: a power of two with at least 8 vectors per thread where the
  // rows are long enough, so each thread keeps several 16-byte loads in flight
  const int64_t vpr = (p.cols + 7) / 8;
  int tpr_log2 = 0;
  while ((1LL << tpr_log2) < 256 && (1LL << (tpr_log2 + 1)) * 8 <= vpr) ++tpr_log2;
  const int64_t rows = p.batch * p.rows_out;
  const int64_t groups = ceil_div(rows, 256 >> tpr_log2);
  const int64_t grid = std::min<int64_t>(groups, 4LL * num_sms());
  const cudaError_t e = launch_chained(pack_rows_gather_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, s, p, tpr_log2);
  if (e != cudaSuccess) return cuda_fail(e, "row pack launch");
  return RMM_OK;
}

rmm_status launch_mask(const MaskParams& p, cudaStream_t s) {
  const int64_t per_item = p.rows * (p.cols / 8);
  if (p.batch > 65535) return fail(RMM_ERR_UNSUPPORTED, "too many batch items for the mask copy");
  const int64_t cap = std::max<int64_t>(1, 8LL * num_sms() / p.batch);
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(ceil_div(per_item, 256 * 4), cap));
  const cudaError_t e = launch_chained(mask_copy_kernel, dim3(static_cast<unsigned>(grid), static_cast<unsigned>(p.batch)),
                                       dim3(256), 0, s, p);
  if (e != cudaSuccess) return cuda_fail(e, "mask launch");
  return RMM_OK;
}

template <int BN, int BMODE, int EPI, int CAUSAL>
rmm_status launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p, cudaStream_t s) {
  auto kern = rmm_gemm_kernel<BN, BMODE, EPI, CAUSAL>;
  CUtensorMap to;
  if (rmm_status st = make_tmap_out(&to, p.out, EPI == kEpiF32, static_cast<uint64_t>(p.N), static_cast<uint64_t>(p.M),
                                    static_cast<uint64_t>(p.batch), static_cast<uint64_t>(p.ldo),
                                    static_cast<uint64_t>(p.out_bstride)))
    return st;
  constexpr int smem = GemmCfg<BN>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "gemm attribute");
  const int64_t tiles = static_cast<int64_t>(p.batch) * p.m_tiles * p.n_tiles;
  if (tiles > kIntMax) return fail(RMM_ERR_UNSUPPORTED, "too many output tiles");
  const int64_t units = tiles - p.tail_tiles + static_cast<int64_t>(p.tail_tiles) * std::max(p.tail_split, 1);
  const int grid = static_cast<int>(std::min<int64_t>(units, num_sms()));
  e = launch_chained(kern, dim3(grid), dim3(192), smem, s, ta, tb, to, p);
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return RMM_OK;
}

// Linear-path product on CTA pairs (256 x 256 tiles, see gemm_pair.cuh).  With
// tb2 != nullptr the gate / up variant: B halves from tb (gate) and tb2 (up),
// output H = SiLU(gate) * up with 128 output columns per tile.
// With gather, B is read through p.gidx from p.gw0 (and p.gw1) instead of tb / tb2.
rmm_status launch_gemm_pair(const CUtensorMap& ta, const CUtensorMap& tb, GemmParams p, cudaStream_t s,
                            const CUtensorMap* tb2 = nullptr, bool gather = false) {
  CUtensorMap to;
  if (rmm_status st = make_tmap_out(&to, p.out, false, static_cast<uint64_t>(p.N), static_cast<uint64_t>(p.M),
                                    static_cast<uint64_t>(p.batch), static_cast<uint64_t>(p.ldo),
                                    static_cast<uint64_t>(p.out_bstride)))
    return st;
  constexpr int smem = PairCfg::SMEM_BYTES;
  const bool swiglu = tb2 != nullptr;
  auto kern = gather ? (swiglu ? rmm_gemm_pair_kernel<true, true> : rmm_gemm_pair_kernel<false, true>)
                     : (swiglu ? rmm_gemm_pair_kernel<true, false> : rmm_gemm_pair_kernel<false, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "gemm attribute");
  const int64_t tiles = static_cast<int64_t>(p.batch) * p.m_tiles * p.n_tiles;
  if (tiles > kIntMax) return fail(RMM_ERR_UNSUPPORTED, "too many output tiles");
  // a partial last wave of pair tiles is cut into 256 x 128 pieces when twice
  // its tiles still fit one per pair
  const int64_t P = std::max(1, num_sms() / 2);
  const int64_t R = tiles > P ? tiles % P : tiles;
  if (R > 0 && 2 * R <= P) {
    p.tail_tiles = static_cast<int>(R);
    p.tail_split = 2;
  }
  const int64_t units = tiles - p.tail_tiles + static_cast<int64_t>(p.tail_tiles) * std::max(p.tail_split, 1);
  const int pairs = static_cast<int>(std::min<int64_t>(units, P));
  e = launch_cluster(kern, dim3(static_cast<unsigned>(2 * pairs)), dim3(gather ? 320 : 192), smem, 2, s, ta, tb,
                     tb2 ? *tb2 : tb, to, p);
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return RMM_OK;
}

GemmParams gemm_defaults() {
  GemmParams p{};
  p.batch = 1;
  p.b_g_outer = 1;
  p.b_g_inner = 1;
  p.b_s_outer = 0;
  p.b_s_inner = 0;
  p.scale = 1.f;
  return p;
}

rmm_status check_rho(double rho) {
  if (!(rho > 0.0 && rho <= 1.0)) return fail(RMM_ERR_INVALID_ARG, "rho must lie in (0, 1], got %g", rho);
  return RMM_OK;
}

// S3 of the linear path: A_pack = A[:, I] (zero-padded to ld_pack columns).
rmm_status pack_columns(const uint16_t* A, int64_t n, int64_t d, int64_t lda, const int32_t* idx, int64_t k,
                        uint16_t* apack, int64_t ld_pack, cudaStream_t s) {
  PackParams pk{};
  pk.src = A;
  pk.src_ld = lda;
  pk.rows = n;
  pk.d = d;
  pk.g_outer = 1;
  pk.g_inner = 1;
  pk.idx = idx;
  pk.k = k;
  pk.k_pad = ld_pack;
  pk.dst = apack;
  pk.batch = 1;
  return launch_pack(pk, s);
}

// B_pack[t, :] = B[I[t], :] (row stride ld_pack, a multiple of 8).
rmm_status gather_rows(const uint16_t* B, int64_t m, int64_t ldb, const int32_t* idx, int64_t k, uint16_t* bpack,
                       int64_t ld_pack, cudaStream_t s) {
  RowPackParams rp{};
  rp.src = B;
  rp.src_ld = ldb;
  rp.cols = m;
  rp.idx = idx;
  rp.k = k;
  rp.rows_out = k;
  rp.dst = bpack;
  rp.dst_ld = ld_pack;
  rp.batch = 1;
  rp.g_outer = 1;
  rp.g_inner = 1;
  return launch_rowpack(rp, s);
}

// Dense tensor-core product Y = A[:, :k] . B[:k, :], A K-major [n][lda], B
// MN-major [k][ldb] (rows past k and columns past the extents read as zero).
rmm_status gemm_packed(const uint16_t* A, int64_t n, int64_t k, int64_t lda, const uint16_t* B, int64_t m, int64_t ldb,
                       uint16_t* Y, int64_t ldy, cudaStream_t s) {
  CUtensorMap ta, tb;
  if (rmm_status st = make_tmap(&ta, A, k, n, lda * 2, 64, 128)) return st;
  if (rmm_status st = make_tmap(&tb, B, m, k, ldb * 2, 64, 64)) return st;
  GemmParams g = gemm_defaults();
  g.M = static_cast<int>(n);
  g.N = static_cast<int>(m);
  g.out = Y;
  g.ldo = ldy;
  g.m_tiles = static_cast<int>(ceil_div(n, 128));
  g.n_tiles = static_cast<int>(ceil_div(m, 256));
  g.k = static_cast<int>(k);
  g.num_kb = static_cast<int>(ceil_div(k, 64));
  if (n > kOneCtaMaxRows) {
    g.m_tiles = static_cast<int>(ceil_div(n, 256));
    return launch_gemm_pair(ta, tb, g, s);
  }
  // narrow last wave: cut the tiles of a partial last wave into 2 or 4 pieces
  // along N when that many pieces still fit one per SM
  const int64_t tiles = static_cast<int64_t>(g.m_tiles) * g.n_tiles;
  const int64_t P = num_sms();
  const int64_t R = tiles > P ? tiles % P : tiles;
  int split = 4;
  while (split > 1 && R * split > P) split /= 2;
  if (R > 0 && split > 1) {
    g.tail_tiles = static_cast<int>(R);
    g.tail_split = split;
  }
  return launch_gemm<256, kBTileMN, kEpiBf16, kCausalNone>(ta, tb, g, s);
}

// Y = A_pack[:, :k] . B[I, :] on CTA pairs, the kept rows of B read through the
// index set straight from B (no packed copy of B[I, :]).
rmm_status gemm_gathered(const uint16_t* A, int64_t n, int64_t k, int64_t lda, const uint16_t* B, int64_t m,
                         int64_t ldb, const int32_t* idx, uint16_t* Y, int64_t ldy, cudaStream_t s) {
  CUtensorMap ta;
  if (rmm_status st = make_tmap(&ta, A, k, n, lda * 2, 64, 128)) return st;
  GemmParams g = gemm_defaults();
  g.M = static_cast<int>(n);
  g.N = static_cast<int>(m);
  g.out = Y;
  g.ldo = ldy;
  g.m_tiles = static_cast<int>(ceil_div(n, 256));
  g.n_tiles = static_cast<int>(ceil_div(m, 256));
  g.k = static_cast<int>(k);
  g.num_kb = static_cast<int>(ceil_div(k, 64));
  g.gw0 = B;
  g.gw1 = B;
  g.gldw = ldb;
  g.gidx = idx;
  return launch_gemm_pair(ta, ta, g, s, nullptr, true);
}

// Decode path (n <= 32): Y = x[:, I] . W[I, :] streaming only the kept rows of W.
constexpr int64_t kDecodeMaxRows = 32;
// int8 weights: activation rows up to which the CUDA-core kernel runs; the tensor
// cores take more
constexpr int64_t kI8CudaCoreMaxRows = 2;

int decode_grid(int64_t units) { return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(units, num_sms()))); }

size_t decode_partial_floats(int64_t n, int64_t m, int64_t k) {
  const int64_t m_super = ceil_div(m, kGemvCols);
  const int64_t units = m_super * ceil_div(k, 64);
  return static_cast<size_t>((m_super + decode_grid(units)) * kGemvTiles * n * 128);
}

rmm_status decode_product(const uint16_t* xp, int64_t n, int64_t ldx, const uint16_t* W, int64_t k, int64_t m,
                          int64_t ldw, const int32_t* idx, float* partial, uint16_t* Y, int64_t ldy, cudaStream_t s) {
  GemvParams g{};
  g.W = W;
  g.ldw = ldw;
  g.idx = idx;
  g.k = static_cast<int>(k);
  g.m = static_cast<int>(m);
  g.n = static_cast<int>(n);
  g.m_super = static_cast<int>(ceil_div(m, kGemvCols));
  g.kb_total = static_cast<int>(ceil_div(k, 64));
  g.units = static_cast<int64_t>(g.m_super) * g.kb_total;
  g.partial = partial;
  const int grid = decode_grid(g.units);
  const int N = (n <= 16) ? 16 : 32;
  CUtensorMap tx;
  // x_I (or x itself) as the K-major operand: N rows (rows past n read zero) x 64 columns per box
  if (rmm_status st = make_tmap(&tx, xp, k, n, ldx * 2, 64, static_cast<uint32_t>(N))) return st;
  const int smem = 1024 + kGemvStages * (kGemvCols * 64 * 2 + N * 64 * 2) + 256;
  cudaError_t e;
  if (N == 16) {
    e = cudaFuncSetAttribute(gemv_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) e = launch_chained(gemv_kernel<16>, dim3(grid), dim3(288), smem, s, tx, g);
  } else {
    e = cudaFuncSetAttribute(gemv_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) e = launch_chained(gemv_kernel<32>, dim3(grid), dim3(288), smem, s, tx, g);
  }
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  e = launch_chained(gemv_fixup_kernel, dim3(static_cast<unsigned>(g.m_super * kGemvTiles), static_cast<unsigned>(ceil_div(n, 4))),
                     dim3(128), static_cast<size_t>(grid + 1) * sizeof(int), s, g, grid, Y, ldy,
                     static_cast<const float*>(nullptr));
  if (e != cudaSuccess) return cuda_fail(e, "decode fix-up launch");
  return RMM_OK;
}

}  // namespace

// ============================================================== public API
extern "C" {

int64_t rmm_k(double rho, int64_t d) {
  if (!(rho > 0.0 && rho <= 1.0) || d < 1) return -1;
  const double x = rho * static_cast<double>(d);
  int64_t k = static_cast<int64_t>(std::ceil(x - 1e-9 * x));
  if (k < 1) k = 1;
  if (k > d) k = d;
  return k;
}

// ---------------------------------------------------------------- fused reduced attention
}  // extern "C"

namespace {
// Workspace of rmm_attention (rho < 1): scores, index sets, keep bytes and Q with
// the dropped dims zeroed for 64 < k < 128; for k <= 64, Q[:, I_h] and
// K_g(h)[:, I_h] packed to 64 dims per query head, so the score MMA runs over 64
// dims instead of 128 (the kernel's MMAs are bound by their shared-memory operand
// reads, so halving the score product's K shortens it).
constexpr int64_t kAttnPackedDims = 64;
size_t attention_bytes(int64_t items, int64_t nq, int64_t nk, int64_t dh, int64_t k) {
  if (k == dh) return 0;
  Carver c(nullptr);
  c.take<double>(items * dh);
  c.take<int32_t>(items * k);
  if (k <= kAttnPackedDims) {
    c.take<uint16_t>(items * nq * kAttnPackedDims);
    c.take<uint16_t>(items * nk * kAttnPackedDims);
  } else {
    c.take<uint8_t>(items * dh);
    c.take<uint16_t>(items * nq * dh);
  }
  return c.bytes();
}
}  // namespace

extern "C" {

size_t rmm_attention_workspace_bytes(int64_t batch, int64_t hq, int64_t hkv, int64_t nq, int64_t nk, int64_t dh,
                                     double rho) {
  (void)hkv;
  const int64_t k = rmm_k(rho, dh);
  if (k < 0 || batch < 1 || hq < 1 || nq < 1 || nk < 1) return 0;
  return attention_bytes(batch * hq, nq, nk, dh, k);
}

rmm_status rmm_attention(const rmm_bf16* Q, const rmm_bf16* K, const rmm_bf16* V, rmm_bf16* O, int64_t batch,
                         int64_t hq, int64_t hkv, int64_t nq, int64_t nk, int64_t dh, int causal, float scale,
                         double rho, int32_t* idx_out, void* ws, size_t ws_bytes, rmm_stream stream) {
  t_last_error.clear();
  if (rmm_status st = check_rho(rho)) return st;
  if (Q == nullptr || K == nullptr || V == nullptr || O == nullptr)
    return fail(RMM_ERR_INVALID_ARG, "Q, K, V and O are required");
  if (batch < 1 || hq < 1 || hkv < 1 || nq < 1 || nk < 1 || dh < 1) return fail(RMM_ERR_INVALID_ARG, "sizes must be >= 1");
  if (hq % hkv) return fail(RMM_ERR_INVALID_ARG, "hq must be a multiple of hkv");
  if (causal != 0 && causal != 1) return fail(RMM_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (!std::isfinite(scale)) return fail(RMM_ERR_INVALID_ARG, "scale must be finite");
  if (dh != 128) return fail(RMM_ERR_UNSUPPORTED, "the fused attention kernel takes head dim 128");
  if (causal && nq > nk) return fail(RMM_ERR_UNSUPPORTED, "causal attention needs nq <= nk (every query sees a key)");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || (ws != nullptr && !aligned16(ws)))
    return fail(RMM_ERR_UNSUPPORTED, "pointers must be 16-byte aligned");
  const int64_t items = batch * hq;
  const int64_t m_tiles = ceil_div(nq, 128);
  if (items * nq > kIntMax - 256 || items * nk > kIntMax - 256 || batch * hkv * nk > kIntMax - 256 ||
      items * m_tiles > kIntMax)
    return fail(RMM_ERR_UNSUPPORTED, "problem too large");
  const int64_t k = rmm_k(rho, dh);
  const size_t need = attention_bytes(items, nq, nk, dh, k);
  if (need > 0 && (ws == nullptr || ws_bytes < need))
    return fail(RMM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  AttnParams ap{};
  ap.nq = static_cast<int>(nq);
  ap.nk = static_cast<int>(nk);
  ap.hq = static_cast<int>(hq);
  ap.hkv = static_cast<int>(hkv);
  ap.items = static_cast<int>(items);
  ap.m_tiles = static_cast<int>(m_tiles);
  ap.causal = causal;
  ap.causal_off = nk - nq;
  ap.scale_log2 = scale * 1.4426950408889634f;
  ap.O = O;
  const uint16_t* qsrc = Q;
  const uint16_t* ksrc = K;
  ap.kp = 128;
  ap.k_per_item = 0;
  if (k < dh && k <= kAttnPackedDims) {
    // scores and selection on Q, then Q[:, I_h] and K_g(h)[:, I_h] packed to 64
    // dims (zero past k) for every query head
    Carver c(ws);
    double* colsq = c.take<double>(items * dh);
    int32_t* idx_ws = c.take<int32_t>(items * k);
    int32_t* idx = idx_out ? idx_out : idx_ws;
    uint16_t* qp = c.take<uint16_t>(items * nq * kAttnPackedDims);
    uint16_t* kpk = c.take<uint16_t>(items * nk * kAttnPackedDims);
    if (rmm_status st = launch_colsq(Q, items, nq * dh, nq, dh, dh, false, 0, colsq, s)) return st;
    if (rmm_status st = launch_select(colsq, items, dh, k, idx, nullptr, s)) return st;
    PackParams pq{};
    pq.src = Q;
    pq.src_ld = dh;
    pq.rows = nq;
    pq.d = dh;
    pq.g_outer = 1;
    pq.g_inner = 1;
    pq.s_outer = nq * dh;
    pq.s_inner = 0;
    pq.idx = idx;
    pq.k = k;
    pq.k_pad = kAttnPackedDims;
    pq.dst = qp;
    pq.batch = items;
    if (rmm_status st = launch_pack(pq, s)) return st;
    PackParams pk = pq;  // query head b * hq + h reads key head b * hkv + h / (hq / hkv)
    pk.src = K;
    pk.rows = nk;
    pk.g_outer = hq;
    pk.s_outer = hkv * nk * dh;
    pk.g_inner = hq / hkv;
    pk.s_inner = nk * dh;
    pk.dst = kpk;
    if (rmm_status st = launch_pack(pk, s)) return st;
    qsrc = qp;
    ksrc = kpk;
    ap.kp = static_cast<int>(kAttnPackedDims);
    ap.k_per_item = 1;
  } else if (k < dh) {
    Carver c(ws);
    double* colsq = c.take<double>(items * dh);
    int32_t* idx_ws = c.take<int32_t>(items * k);
    int32_t* idx = idx_out ? idx_out : idx_ws;
    if (rmm_status st = launch_colsq(Q, items, nq * dh, nq, dh, dh, false, 0, colsq, s)) return st;
    uint8_t* keep = c.take<uint8_t>(items * dh);
    uint16_t* qm = c.take<uint16_t>(items * nq * dh);
    if (rmm_status st = launch_select(colsq, items, dh, k, idx, nullptr, s, keep)) return st;
    MaskParams mp{};
    mp.src = Q;
    mp.dst = qm;
    mp.rows = nq;
    mp.cols = dh;
    mp.keep = keep;
    mp.by_rows = 0;
    mp.batch = items;
    mp.g_outer = 1;
    mp.g_inner = 1;
    mp.s_outer = nq * dh;
    if (rmm_status st = launch_mask(mp, s)) return st;
    qsrc = qm;
  } else if (idx_out != nullptr) {
    const cudaError_t e = launch_chained(iota_kernel, dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(items * dh, 256), 1024))),
                                         dim3(256), 0, s, idx_out, items, dh);
    if (e != cudaSuccess) return cuda_fail(e, "iota launch");
  }
  CUtensorMap tq, tk, tv;
  if (rmm_status st = make_tmap(&tq, qsrc, ap.kp, items * nq, ap.kp * 2, 64, 128)) return st;
  if (rmm_status st = make_tmap(&tk, ksrc, ap.kp, (ap.k_per_item ? items : batch * hkv) * nk, ap.kp * 2, 64, 128))
    return st;
  if (rmm_status st = make_tmap(&tv, V, dh, batch * hkv * nk, dh * 2, 64, 64)) return st;
  cudaError_t e = cudaFuncSetAttribute(attn_pp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnPPSmem);
  if (e != cudaSuccess) return cuda_fail(e, "attention attribute");
  e = launch_chained(attn_pp_kernel, dim3(static_cast<unsigned>(items * ceil_div(m_tiles, 2))), dim3(kAttnPPThreads), kAttnPPSmem, s,
                     tq, tk, tv, ap);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return RMM_OK;
}

// ---------------------------------------------------------------- int8 weights
}  // extern "C"

namespace {
// Row chunks of the int8 GEMV: about four CTAs per SM over all column blocks,
// at most kI8MaxChunk rows each, and few enough chunks that the fp32 partial
// sums (chunks x n x m x 4 bytes) stay near 12 % of the kept int8 rows.
// Row chunks of the int8 GEMV: as many as one wave of co-resident CTAs holds
// (the kernel's launch bounds give 4, 3 or 2 CTAs per SM for 1, 2 or more rows),
// so that every CTA starts at once and no partial second wave follows.  A chunk
// is a multiple of 16 kept rows and at most kI8MaxChunk.
void i8_plan(int64_t n, int64_t k, int64_t m, int* chunk, int* chunks) {
  const int64_t col_blocks = ceil_div(m, 2048);
  const int64_t per_sm = (n == 1) ? 4 : ((n == 2) ? 3 : 2);
  const int64_t max_chunks = std::max<int64_t>(1, (per_sm * num_sms()) / col_blocks);
  int64_t len = round_up(ceil_div(k, max_chunks), 16);
  if (len > kI8MaxChunk) len = kI8MaxChunk;
  *chunk = static_cast<int>(len);
  *chunks = static_cast<int>(ceil_div(k, len));
}

template <int NR>
cudaError_t launch_gemv_i8_t(const GemvI8Params& p, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(ceil_div(p.m, 2048)), static_cast<unsigned>(p.chunks));
  return launch_chained(gemv_i8_kernel<NR>, grid, dim3(256), 0, s, p);
}
}  // namespace

extern "C" {

// int8 weights on the tensor cores (n > kI8CudaCoreMaxRows): dequantised in the
// producer into the bf16 UMMA stage; x[:, I] packed by the decode selection.
rmm_status int8_tc_product(const uint16_t* xp, int64_t n, int64_t ldx, const int8_t* W, int64_t k, int64_t m,
                           int64_t ldw, const int32_t* idx, const float* scale, float* partial, uint16_t* Y, int64_t ldy,
                           cudaStream_t s) {
  GemvI8TcParams g{};
  g.W = W;
  g.ldw = ldw;
  g.idx = idx;
  g.k = static_cast<int>(k);
  g.m = static_cast<int>(m);
  g.n = static_cast<int>(n);
  g.m_super = static_cast<int>(ceil_div(m, kGemvCols));
  g.kb_total = static_cast<int>(ceil_div(k, 64));
  g.units = static_cast<int64_t>(g.m_super) * g.kb_total;
  g.partial = partial;
  const int grid = decode_grid(g.units);
  const int N = (n <= 16) ? 16 : 32;
  CUtensorMap tx;
  if (rmm_status st = make_tmap(&tx, xp, k, n, ldx * 2, 64, static_cast<uint32_t>(N))) return st;
  const int smem = 1024 + kGemvStages * (kGemvCols * 64 * 2 + N * 64 * 2) + 256;
  cudaError_t e;
  if (N == 16) {
    e = cudaFuncSetAttribute(gemv_i8tc_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) e = launch_chained(gemv_i8tc_kernel<16>, dim3(grid), dim3(kI8TcThreads), smem, s, tx, g);
  } else {
    e = cudaFuncSetAttribute(gemv_i8tc_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) e = launch_chained(gemv_i8tc_kernel<32>, dim3(grid), dim3(kI8TcThreads), smem, s, tx, g);
  }
  if (e != cudaSuccess) return cuda_fail(e, "int8 tensor-core launch");
  GemvParams f{};
  f.k = g.k;
  f.m = g.m;
  f.n = g.n;
  f.m_super = g.m_super;
  f.kb_total = g.kb_total;
  f.units = g.units;
  f.partial = partial;
  e = launch_chained(gemv_fixup_kernel, dim3(static_cast<unsigned>(f.m_super * kGemvTiles), static_cast<unsigned>(ceil_div(n, 4))),
                     dim3(128), static_cast<size_t>(grid + 1) * sizeof(int), s, f, grid, Y, ldy, scale);
  if (e != cudaSuccess) return cuda_fail(e, "int8 fix-up launch");
  return RMM_OK;
}

size_t rmm_linear_int8_workspace_bytes(int64_t n, int64_t d, int64_t m, double rho) {
  const int64_t k = rmm_k(rho, d);
  if (k < 0 || n < 1 || m < 1) return 0;
  if (n > kI8CudaCoreMaxRows) {
    Carver c(nullptr);
    if (k < d) {
      c.take<double>(d);
      c.take<int32_t>(k);
      c.take<uint16_t>(n * round_up(k, 8));
    }
    c.take<float>(static_cast<int64_t>(decode_partial_floats(n, m, k)));
    return c.bytes();
  }
  int chunk = 0, chunks = 0;
  i8_plan(n, k, m, &chunk, &chunks);
  Carver c(nullptr);
  if (k < d) {
    c.take<double>(d);
    c.take<int32_t>(k);
  }
  c.take<float>(static_cast<int64_t>(chunks) * n * m);
  return c.bytes();
}

rmm_status rmm_linear_int8(const rmm_bf16* A, int64_t n, int64_t d, int64_t lda, const int8_t* Wq, int64_t m,
                           int64_t ldw, const float* scale, rmm_bf16* Y, int64_t ldy, double rho, int32_t* idx_out,
                           void* ws, size_t ws_bytes, rmm_stream stream) {
  t_last_error.clear();
  if (rmm_status st = check_rho(rho)) return st;
  if (A == nullptr || Wq == nullptr || scale == nullptr || Y == nullptr)
    return fail(RMM_ERR_INVALID_ARG, "A, Wq, scale and Y are required");
  if (n < 1 || d < 1 || m < 1) return fail(RMM_ERR_INVALID_ARG, "n, d and m must be >= 1");
  if (lda < d || ldw < m || ldy < m) return fail(RMM_ERR_INVALID_ARG, "leading dimension too small");
  if (n > kDecodeMaxRows) return fail(RMM_ERR_UNSUPPORTED, "the int8 path takes at most 32 activation rows");
  if (!aligned16(A) || !aligned16(Wq) || !aligned16(Y) || (ws != nullptr && !aligned16(ws)) || (lda % 8) ||
      (ldw % 8) || (ldy % 8) || (m % 8))
    return fail(RMM_ERR_UNSUPPORTED, "pointers 16-byte aligned; lda, ldw, ldy and m multiples of 8");
  if (d > kMaxSelectD || m > kIntMax || static_cast<int64_t>(d) * ldw > (1LL << 40))
    return fail(RMM_ERR_UNSUPPORTED, "dimension too large");
  const size_t need = rmm_linear_int8_workspace_bytes(n, d, m, rho);
  if (ws == nullptr || ws_bytes < need)
    return fail(RMM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t k = rmm_k(rho, d);
  if (n > kI8CudaCoreMaxRows) {
    // tensor cores: the decode selection (with x[:, I]), then the dequantising product
    Carver c(ws);
    if (k == d) {
      float* partial = c.take<float>(static_cast<int64_t>(decode_partial_floats(n, m, k)));
      if (idx_out != nullptr) {
        const cudaError_t e = launch_chained(iota_kernel, dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(d, 256), 1024))),
                                             dim3(256), 0, s, idx_out, 1, d);
        if (e != cudaSuccess) return cuda_fail(e, "iota launch");
      }
      return int8_tc_product(A, n, lda, Wq, d, m, ldw, nullptr, scale, partial, reinterpret_cast<uint16_t*>(Y), ldy, s);
    }
    const int64_t k_pad = round_up(k, 8);
    double* colsq = c.take<double>(d);
    int32_t* idx_ws = c.take<int32_t>(k);
    uint16_t* xpack = c.take<uint16_t>(n * k_pad);
    float* partial = c.take<float>(static_cast<int64_t>(decode_partial_floats(n, m, k)));
    int32_t* idx = idx_out ? idx_out : idx_ws;
    if (decode_select_fits(n, d)) {
      if (rmm_status st = launch_decode_select(A, n, d, lda, k, idx, xpack, k_pad, s)) return st;
    } else {
      if (rmm_status st = launch_colsq(A, 1, 0, n, d, lda, false, 0, colsq, s)) return st;
      if (rmm_status st = launch_select(colsq, 1, d, k, idx, nullptr, s)) return st;
      if (rmm_status st = pack_columns(A, n, d, lda, idx, k, xpack, k_pad, s)) return st;
    }
    return int8_tc_product(xpack, n, k_pad, Wq, k, m, ldw, idx, scale, partial, reinterpret_cast<uint16_t*>(Y), ldy, s);
  }
  int chunk = 0, chunks = 0;
  i8_plan(n, k, m, &chunk, &chunks);
  if (chunks > 65535) return fail(RMM_ERR_UNSUPPORTED, "too many row chunks");
  Carver c(ws);
  GemvI8Params p{};
  p.W = Wq;
  p.ldw = ldw;
  p.x = A;
  p.ldx = lda;
  p.k = static_cast<int>(k);
  p.m = static_cast<int>(m);
  p.n = static_cast<int>(n);
  p.chunk = chunk;
  p.chunks = chunks;
  if (k < d) {
    double* colsq = c.take<double>(d);
    int32_t* idx_ws = c.take<int32_t>(k);
    int32_t* idx = idx_out ? idx_out : idx_ws;
    if (decode_select_fits(n, d)) {
      if (rmm_status st = launch_decode_select(A, n, d, lda, k, idx, nullptr, 0, s)) return st;
    } else {
      if (rmm_status st = launch_colsq(A, 1, 0, n, d, lda, false, 0, colsq, s)) return st;
      if (rmm_status st = launch_select(colsq, 1, d, k, idx, nullptr, s)) return st;
    }
    p.idx = idx;
  } else if (idx_out != nullptr) {
    const cudaError_t e = launch_chained(iota_kernel, dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(d, 256), 1024))),
                                         dim3(256), 0, s, idx_out, 1, d);
    if (e != cudaSuccess) return cuda_fail(e, "iota launch");
  }
  float* partial = c.take<float>(static_cast<int64_t>(chunks) * n * m);
  p.partial = partial;
  cudaError_t e = cudaSuccess;
  if (n == 1) e = launch_gemv_i8_t<1>(p, s);
  else if (n == 2) e = launch_gemv_i8_t<2>(p, s);
  else if (n <= 4) e = launch_gemv_i8_t<4>(p, s);
  else e = launch_gemv_i8_t<8>(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "int8 GEMV launch");
  e = launch_chained(gemv_i8_fixup_kernel, dim3(static_cast<unsigned>(ceil_div(m, 256)), static_cast<unsigned>(n)), dim3(256),
                     0, s, static_cast<const float*>(partial), scale, chunks, static_cast<int>(n), static_cast<int>(m),
                     reinterpret_cast<uint16_t*>(Y), ldy);
  if (e != cudaSuccess) return cuda_fail(e, "int8 GEMV fix-up launch");
  return RMM_OK;
}

// ---------------------------------------------------------------- MLP block
}  // extern "C"

namespace {
// Workspace of the gate / up half of rmm_mlp (rho_gu < 1): scores, index set,
// X[:, I] and the kept rows of both weights.
size_t mlp_gate_up_bytes(int64_t n, int64_t d, int64_t f, int64_t k) {
  if (k == d) return 0;
  Carver c(nullptr);
  c.take<double>(d);
  c.take<int32_t>(k);
  c.take<uint16_t>(n * round_up(k, 8));
  c.take<uint16_t>(k * round_up(f, 8));
  c.take<uint16_t>(k * round_up(f, 8));
  return c.bytes();
}
}  // namespace

extern "C" {

size_t rmm_mlp_workspace_bytes(int64_t n, int64_t d, int64_t f, int64_t m, double rho_gu, double rho_down) {
  const int64_t k = rmm_k(rho_gu, d);
  if (k < 0 || n < 1 || f < 1 || m < 1 || rmm_k(rho_down, f) < 0) return 0;
  return mlp_gate_up_bytes(n, d, f, k) + rmm_linear_workspace_bytes(n, f, m, rho_down);
}

rmm_status rmm_mlp(const rmm_bf16* X, int64_t n, int64_t d, int64_t ldx, const rmm_bf16* Wg, const rmm_bf16* Wu,
                   int64_t f, int64_t ldw, const rmm_bf16* Wd, int64_t m, int64_t ldwd, rmm_bf16* H, int64_t ldh,
                   rmm_bf16* Y, int64_t ldy, double rho_gu, double rho_down, int32_t* idx_gu_out,
                   int32_t* idx_down_out, void* ws, size_t ws_bytes, rmm_stream stream) {
  t_last_error.clear();
  if (rmm_status st = check_rho(rho_gu)) return st;
  if (rmm_status st = check_rho(rho_down)) return st;
  if (X == nullptr || Wg == nullptr || Wu == nullptr || Wd == nullptr || H == nullptr || Y == nullptr)
    return fail(RMM_ERR_INVALID_ARG, "X, Wg, Wu, Wd, H and Y are required");
  if (n < 1 || d < 1 || f < 1 || m < 1) return fail(RMM_ERR_INVALID_ARG, "n, d, f and m must be >= 1");
  if (ldx < d || ldw < f || ldwd < m || ldh < f || ldy < m) return fail(RMM_ERR_INVALID_ARG, "leading dimension too small");
  if (!aligned16(X) || !aligned16(Wg) || !aligned16(Wu) || !aligned16(Wd) || !aligned16(H) || !aligned16(Y) ||
      (ws != nullptr && !aligned16(ws)) || (ldx % 8) || (ldw % 8) || (ldwd % 8) || (ldh % 8) || (ldy % 8))
    return fail(RMM_ERR_UNSUPPORTED, "pointers must be 16-byte aligned and leading dims multiples of 8");
  if (d > kMaxSelectD || f > kMaxSelectD) return fail(RMM_ERR_UNSUPPORTED, "d and f must be at most 32768");
  if (n > kIntMax - 256 || f > kIntMax - 256 || m > kIntMax - 256) return fail(RMM_ERR_UNSUPPORTED, "dimension too large");
  const int64_t k = rmm_k(rho_gu, d);
  const size_t gu_bytes = mlp_gate_up_bytes(n, d, f, k);
  const size_t need = gu_bytes + rmm_linear_workspace_bytes(n, f, m, rho_down);  // both parts 256-byte multiples
  if ((need > 0 && ws == nullptr) || ws_bytes < need)
    return fail(RMM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // gate and up: one selection on X, one fused product writing H = SiLU(gate) * up
  const uint16_t* A = X;
  int64_t K = d, lda = ldx;
  const uint16_t* Bg = Wg;
  const uint16_t* Bu = Wu;
  int64_t ldb = ldw;
  if (k < d) {
    Carver c(ws);
    double* colsq = c.take<double>(d);
    int32_t* idx_ws = c.take<int32_t>(k);
    const int64_t k_pad = round_up(k, 8), f_pad = round_up(f, 8);
    uint16_t* xpack = c.take<uint16_t>(n * k_pad);
    uint16_t* gpack = c.take<uint16_t>(k * f_pad);
    uint16_t* upack = c.take<uint16_t>(k * f_pad);
    int32_t* idx = idx_gu_out ? idx_gu_out : idx_ws;
    if (decode_select_fits(n, d)) {
      if (rmm_status st = launch_decode_select(X, n, d, ldx, k, idx, xpack, k_pad, s)) return st;
    } else {
      if (rmm_status st = launch_colsq(X, 1, 0, n, d, ldx, false, 0, colsq, s)) return st;
      if (rmm_status st = launch_select(colsq, 1, d, k, idx, nullptr, s)) return st;
      if (rmm_status st = pack_columns(X, n, d, ldx, idx, k, xpack, k_pad, s)) return st;
    }
    if (rmm_status st = gather_rows(Wg, f, ldw, idx, k, gpack, f_pad, s)) return st;
    if (rmm_status st = gather_rows(Wu, f, ldw, idx, k, upack, f_pad, s)) return st;
    A = xpack;
    K = k;
    lda = k_pad;
    Bg = gpack;
    Bu = upack;
    ldb = f_pad;
  } else if (idx_gu_out != nullptr) {
    const cudaError_t e = launch_chained(iota_kernel, dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(d, 256), 1024))),
                                         dim3(256), 0, s, idx_gu_out, 1, d);
    if (e != cudaSuccess) return cuda_fail(e, "iota launch");
  }
  CUtensorMap ta, tg, tu;
  if (rmm_status st = make_tmap(&ta, A, K, n, lda * 2, 64, 128)) return st;
  if (rmm_status st = make_tmap(&tg, Bg, f, K, ldb * 2, 64, 64)) return st;
  if (rmm_status st = make_tmap(&tu, Bu, f, K, ldb * 2, 64, 64)) return st;
  GemmParams g = gemm_defaults();
  g.M = static_cast<int>(n);
  g.N = static_cast<int>(f);
  g.out = H;
  g.ldo = ldh;
  g.m_tiles = static_cast<int>(ceil_div(n, 256));
  g.n_tiles = static_cast<int>(ceil_div(f, 128));
  g.k = static_cast<int>(K);
  g.num_kb = static_cast<int>(ceil_div(K, 64));
  if (rmm_status st = launch_gemm_pair(ta, tg, g, s, &tu)) return st;

  // down: RMM on H with its own rho and selection
  uint8_t* ws_down = ws ? static_cast<uint8_t*>(ws) + gu_bytes : nullptr;
  const size_t down_bytes = ws ? ws_bytes - gu_bytes : 0;
  return rmm_linear(H, n, f, ldh, Wd, m, ldwd, Y, ldy, rho_down, idx_down_out, down_bytes ? ws_down : nullptr,
                    down_bytes, stream);
}

// ---------------------------------------------------------------- decode attention
}  // extern "C"

namespace {
bool decode_group_ok(int64_t g) { return g == 1 || g == 2 || g == 4 || g == 8; }

// Kept positions per PV CTA: enough CTAs for about four per SM over all groups.
void decode_pv_plan(int64_t groups, int64_t k, int* chunk, int* splits) {
  const int64_t want = 4LL * num_sms();
  int64_t c = ceil_div(groups * k, want);
  c = round_up(std::max<int64_t>(c, 32), 32);
  if (c > kDecodePvMaxChunk) c = kDecodePvMaxChunk;
  *chunk = static_cast<int>(c);
  *splits = static_cast<int>(ceil_div(k, c));
}

template <int G>
cudaError_t launch_decode_qk_t(const DecodeQkParams& p, int64_t groups, cudaStream_t s) {
  constexpr size_t smem = static_cast<size_t>(kDqkStages) * kDqkStageBytes;
  const cudaError_t e = cudaFuncSetAttribute(decode_qk_staged_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(ceil_div(p.nk, kDqkTokens)), static_cast<unsigned>(groups));
  return launch_chained(decode_qk_staged_kernel<G>, grid, dim3(288), smem, s, p);
}

template <int G, int DH>
cudaError_t launch_decode_pv_t(const DecodePvParams& p, int64_t groups, cudaStream_t s) {
  constexpr size_t smem = static_cast<size_t>(256 / (DH / 8)) * G * DH * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(decode_pv_kernel<G, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(p.splits), static_cast<unsigned>(groups));
  return launch_chained(decode_pv_kernel<G, DH>, grid, dim3(256), smem, s, p);
}
}  // namespace

extern "C" {

size_t rmm_decode_qk_workspace_bytes(int64_t batch, int64_t hq, int64_t hkv, int64_t dh, double rho) {
  const int64_t k = rmm_k(rho, dh);
  if (k < 0 || batch < 1 || hq < 1 || hkv < 1 || k == dh) return 0;
  const int64_t groups = batch * hkv;
  Carver c(nullptr);
  c.take<double>(groups * dh);
  c.take<int32_t>(groups * k);
  return c.bytes();
}

rmm_status rmm_decode_qk(const rmm_bf16* Q, const rmm_bf16* Kt, float* S, int64_t batch, int64_t hq, int64_t hkv,
                         int64_t dh, int64_t nk, int64_t ldk, int64_t lds, float scale, double rho, int32_t* idx_out,
                         void* ws, size_t ws_bytes, rmm_stream stream) {
  t_last_error.clear();
  if (rmm_status st = check_rho(rho)) return st;
  if (Q == nullptr || Kt == nullptr || S == nullptr) return fail(RMM_ERR_INVALID_ARG, "Q, Kt and S are required");
  if (batch < 1 || hq < 1 || hkv < 1 || dh < 1 || nk < 1 || ldk < nk || lds < nk)
    return fail(RMM_ERR_INVALID_ARG, "need batch, hq, hkv, dh, nk >= 1, ldk >= nk and lds >= nk");
  if (hq % hkv) return fail(RMM_ERR_INVALID_ARG, "hq must be a multiple of hkv");
  if (!std::isfinite(scale)) return fail(RMM_ERR_INVALID_ARG, "scale must be finite");
  const int64_t G = hq / hkv;
  if (!decode_group_ok(G)) return fail(RMM_ERR_UNSUPPORTED, "hq / hkv must be 1, 2, 4 or 8");
  if (dh % 8 || dh > kDecodeQkMaxK) return fail(RMM_ERR_UNSUPPORTED, "dh must be a multiple of 8 and at most 512");
  if (!aligned16(Q) || !aligned16(Kt) || !aligned16(S) || (ldk % 8) || (lds % 4))
    return fail(RMM_ERR_UNSUPPORTED, "pointers must be 16-byte aligned, ldk a multiple of 8 and lds of 4");
  const int64_t groups = batch * hkv;
  if (groups > 65535 || nk > kIntMax) return fail(RMM_ERR_UNSUPPORTED, "too many groups or tokens");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t k = rmm_k(rho, dh);
  DecodeQkParams p{};
  p.Q = Q;
  p.Kt = Kt;
  p.S = S;
  p.nk = nk;
  p.ldk = ldk;
  p.lds = lds;
  p.dh = static_cast<int>(dh);
  p.k = static_cast<int>(k);
  p.scale = scale;
  if (k < dh) {
    const size_t need = rmm_decode_qk_workspace_bytes(batch, hq, hkv, dh, rho);
    if (ws == nullptr || ws_bytes < need)
      return fail(RMM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
    Carver c(ws);
    double* colsq = c.take<double>(groups * dh);
    int32_t* idx_ws = c.take<int32_t>(groups * k);
    int32_t* idx = idx_out ? idx_out : idx_ws;
    if (rmm_status st = launch_colsq(Q, groups, G * dh, G, dh, dh, false, 0, colsq, s)) return st;
    if (rmm_status st = launch_select(colsq, groups, dh, k, idx, nullptr, s)) return st;
    p.idx = idx;
  } else if (idx_out != nullptr) {
    const cudaError_t e = launch_chained(iota_kernel, dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(groups * dh, 256), 1024))),
                                         dim3(256), 0, s, idx_out, groups, dh);
    if (e != cudaSuccess) return cuda_fail(e, "iota launch");
  }
  cudaError_t e = cudaSuccess;
  switch (G) {
    case 1: e = launch_decode_qk_t<1>(p, groups, s); break;
    case 2: e = launch_decode_qk_t<2>(p, groups, s); break;
    case 4: e = launch_decode_qk_t<4>(p, groups, s); break;
    default: e = launch_decode_qk_t<8>(p, groups, s); break;
  }
  if (e != cudaSuccess) return cuda_fail(e, "decode QK launch");
  return RMM_OK;
}

size_t rmm_decode_pv_workspace_bytes(int64_t batch, int64_t hq, int64_t hkv, int64_t nk, int64_t dh, double rho) {
  const int64_t k = rmm_k(rho, nk);
  if (k < 0 || batch < 1 || hq < 1 || hkv < 1 || dh < 1 || hq % hkv) return 0;
  const int64_t groups = batch * hkv;
  int chunk = 0, splits = 0;
  decode_pv_plan(groups, k, &chunk, &splits);
  Carver c(nullptr);
  if (k < nk) {
    c.take<double>(groups * nk);
    c.take<int32_t>(groups * k);
  }
  c.take<float>(groups * splits * (hq / hkv) * dh);
  return c.bytes();
}

rmm_status rmm_decode_pv(const rmm_bf16* P, const rmm_bf16* V, rmm_bf16* O, int64_t batch, int64_t hq, int64_t hkv,
                         int64_t nk, int64_t ldp, int64_t cap, int64_t dh, double rho, int32_t* idx_out, void* ws,
                         size_t ws_bytes, rmm_stream stream) {
  t_last_error.clear();
  if (rmm_status st = check_rho(rho)) return st;
  if (P == nullptr || V == nullptr || O == nullptr) return fail(RMM_ERR_INVALID_ARG, "P, V and O are required");
  if (batch < 1 || hq < 1 || hkv < 1 || dh < 1 || nk < 1 || ldp < nk || cap < nk)
    return fail(RMM_ERR_INVALID_ARG, "need batch, hq, hkv, dh, nk >= 1, ldp >= nk and cap >= nk");
  if (hq % hkv) return fail(RMM_ERR_INVALID_ARG, "hq must be a multiple of hkv");
  const int64_t G = hq / hkv;
  if (!decode_group_ok(G)) return fail(RMM_ERR_UNSUPPORTED, "hq / hkv must be 1, 2, 4 or 8");
  if (dh != 64 && dh != 128 && dh != 256) return fail(RMM_ERR_UNSUPPORTED, "dh must be 64, 128 or 256");
  if (G * dh > 1024) return fail(RMM_ERR_UNSUPPORTED, "hq / hkv times dh must be at most 1024");
  if (!aligned16(P) || !aligned16(V) || !aligned16(O) || (ldp % 8))
    return fail(RMM_ERR_UNSUPPORTED, "pointers must be 16-byte aligned and ldp a multiple of 8");
  if (nk > kMaxSelectD) return fail(RMM_ERR_UNSUPPORTED, "nk above the selection limit (32768)");
  const int64_t groups = batch * hkv;
  if (groups > 65535) return fail(RMM_ERR_UNSUPPORTED, "too many groups");
  const size_t need = rmm_decode_pv_workspace_bytes(batch, hq, hkv, nk, dh, rho);
  if (ws == nullptr || ws_bytes < need)
    return fail(RMM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t k = rmm_k(rho, nk);
  int chunk = 0, splits = 0;
  decode_pv_plan(groups, k, &chunk, &splits);
  Carver c(ws);
  DecodePvParams p{};
  if (k < nk) {
    double* colsq = c.take<double>(groups * nk);
    int32_t* idx_ws = c.take<int32_t>(groups * k);
    int32_t* idx = idx_out ? idx_out : idx_ws;
    if (rmm_status st = launch_colsq(P, groups, G * ldp, G, nk, ldp, false, 0, colsq, s)) return st;
    if (rmm_status st = launch_select(colsq, groups, nk, k, idx, nullptr, s)) return st;
    p.idx = idx;
  } else if (idx_out != nullptr) {
    const cudaError_t e = launch_chained(iota_kernel, dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(groups * nk, 256), 1024))),
                                         dim3(256), 0, s, idx_out, groups, nk);
    if (e != cudaSuccess) return cuda_fail(e, "iota launch");
  }
  float* partial = c.take<float>(groups * splits * G * dh);
  p.P = P;
  p.V = V;
  p.partial = partial;
  p.ldp = ldp;
  p.cap = cap;
  p.k = static_cast<int>(k);
  p.chunk = chunk;
  p.splits = splits;
  cudaError_t e = cudaSuccess;
#define RMM_DPV(g, d) \
  if (G == g && dh == d) e = launch_decode_pv_t<g, d>(p, groups, s);
  RMM_DPV(1, 64) RMM_DPV(1, 128) RMM_DPV(1, 256) RMM_DPV(2, 64) RMM_DPV(2, 128) RMM_DPV(2, 256)
  RMM_DPV(4, 64) RMM_DPV(4, 128) RMM_DPV(4, 256) RMM_DPV(8, 64) RMM_DPV(8, 128)
#undef RMM_DPV
  if (e != cudaSuccess) return cuda_fail(e, "decode PV launch");
  e = launch_chained(decode_pv_fixup_kernel, dim3(static_cast<unsigned>(groups)), dim3(static_cast<unsigned>(G * dh)), 0, s,
                     static_cast<const float*>(partial), reinterpret_cast<uint16_t*>(O), splits, static_cast<int>(G * dh));
  if (e != cudaSuccess) return cuda_fail(e, "decode PV fix-up launch");
  return RMM_OK;
}

const char* rmm_status_string(rmm_status s) {
  switch (s) {
    case RMM_OK: return "ok";
    case RMM_ERR_INVALID_ARG: return "invalid argument";
    case RMM_ERR_UNSUPPORTED: return "unsupported layout or size";
    case RMM_ERR_WORKSPACE: return "workspace too small";
    case RMM_ERR_CUDA: return "CUDA error";
    case RMM_ERR_DEVICE_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* rmm_last_error(void) { return t_last_error.c_str(); }

const char* rmm_version(void) { return "rmm-b200 0.1"; }

rmm_status rmm_device_error(int32_t* code_out) {
  if (code_out == nullptr) return fail(RMM_ERR_INVALID_ARG, "code_out is null");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "device synchronise");
  int32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  const int32_t zero = 0;
  e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
  *code_out = v;
  return RMM_OK;
}

// ---------------------------------------------------------------- test hooks
rmm_status rmm_debug_exp2_poly(const float* x, float* y_poly, float* y_exp2f, int64_t n, rmm_stream stream) {
  t_last_error.clear();
  if (x == nullptr || y_poly == nullptr || y_exp2f == nullptr || n < 1) return fail(RMM_ERR_INVALID_ARG, "bad arguments");
  const int64_t grid = std::min<int64_t>(ceil_div(n, 256), 4LL * num_sms());
  attn_exp2_probe_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly, y_exp2f, n);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "exp2 probe launch");
  return RMM_OK;
}

rmm_status rmm_debug_gemm_expire_producer(const rmm_bf16* A_pack, int64_t n, int64_t k, int64_t lda,
                                          const rmm_bf16* B_pack, int64_t m, int64_t ldb, rmm_bf16* Y, int64_t ldy,
                                          rmm_stream stream) {
  t_last_error.clear();
  if (A_pack == nullptr || B_pack == nullptr || Y == nullptr) return fail(RMM_ERR_INVALID_ARG, "null pointer");
  if (n < 1 || k < 1 || m < 1 || lda < k || ldb < m || ldy < m)
    return fail(RMM_ERR_INVALID_ARG, "need n, k, m >= 1, lda >= k, ldb and ldy >= m");
  if (n > 128) return fail(RMM_ERR_UNSUPPORTED, "the hook runs the one-CTA product (n <= 128)");
  if (!aligned16(A_pack) || !aligned16(B_pack) || !aligned16(Y) || (lda % 8) || (ldb % 8) || (ldy % 8))
    return fail(RMM_ERR_UNSUPPORTED, "pointers must be 16-byte aligned and leading dims multiples of 8");
  if (m > kIntMax - 256 || k > kIntMax - 64) return fail(RMM_ERR_UNSUPPORTED, "dimension too large");
  CUtensorMap ta, tb;
  if (rmm_status st = make_tmap(&ta, A_pack, k, n, lda * 2, 64, 128)) return st;
  if (rmm_status st = make_tmap(&tb, B_pack, m, k, ldb * 2, 64, 64)) return st;
  GemmParams g = gemm_defaults();
  g.M = static_cast<int>(n);
  g.N = static_cast<int>(m);
  g.out = Y;
  g.ldo = ldy;
  g.m_tiles = 1;
  g.n_tiles = static_cast<int>(ceil_div(m, 256));
  g.k = static_cast<int>(k);
  g.num_kb = static_cast<int>(ceil_div(k, 64));
  g.expire_producer_waits = 1;
  return launch_gemm<256, kBTileMN, kEpiBf16, kCausalNone>(ta, tb, g, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- select
size_t rmm_select_workspace_bytes(int64_t batch, int64_t n, int64_t d) {
  (void)n;
  if (batch < 1 || d < 1) return 0;
  Carver c(nullptr);
  c.take<double>(batch * d);
  return c.bytes();
}

rmm_status rmm_select(const rmm_bf16* A, int64_t batch, int64_t batch_stride, int64_t n, int64_t d, int64_t lda,
                      int causal, double rho, int32_t* idx_out, double* colsq_out, double* retained_out, void* ws,
                      size_t ws_bytes, rmm_stream stream) {
  t_last_error.clear();
  if (rmm_status st = check_rho(rho)) return st;
  if (A == nullptr || idx_out == nullptr) return fail(RMM_ERR_INVALID_ARG, "A and idx_out are required");
  if (batch < 1 || n < 1 || d < 1) return fail(RMM_ERR_INVALID_ARG, "batch, n and d must be >= 1");
  if (lda < d) return fail(RMM_ERR_INVALID_ARG, "lda < d");
  if (batch > 1 && batch_stride < (n - 1) * lda + d) return fail(RMM_ERR_INVALID_ARG, "batch_stride too small");
  if (causal != 0 && causal != 1) return fail(RMM_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (d > kMaxSelectD) return fail(RMM_ERR_UNSUPPORTED, "d > %lld", static_cast<long long>(kMaxSelectD));
  if (n > kIntMax || batch > 65535) return fail(RMM_ERR_UNSUPPORTED, "n or batch too large");
  if (!aligned16(A) || (lda % 8) != 0 || (batch > 1 && (batch_stride % 8) != 0))
    return fail(RMM_ERR_UNSUPPORTED, "A must be 16-byte aligned with lda and batch_stride multiples of 8");
  const int64_t k = rmm_k(rho, d);
  double* colsq = colsq_out;
  if (colsq == nullptr) {
    const size_t need = rmm_select_workspace_bytes(batch, n, d);
    if (ws == nullptr || ws_bytes < need)
      return fail(RMM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
    Carver c(ws);
    colsq = c.take<double>(batch * d);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t off = d - n;
  if (rmm_status st = launch_colsq(A, batch, batch_stride, n, d, lda, causal != 0, off, colsq, s)) return st;
  return launch_select(colsq, batch, d, k, idx_out, retained_out, s);
}

// ---------------------------------------------------------------- selection without allocation
// For callers that may not allocate device memory at all: the fp64 column
// scores that rmm_select keeps in the caller's workspace live instead in one
// fixed array inside the library.  Every device that loads the library holds
// this array (2 MiB) until the process exits.
}  // extern "C"

namespace {
constexpr int64_t kNoAllocScores = RMM_SELECT_NOALLOC_MAX_SCORES;
static_assert(kNoAllocScores * sizeof(double) == 2u * 1024u * 1024u, "the header documents a 2 MiB scratch array");
static __device__ __align__(256) double g_noalloc_scores[kNoAllocScores];

// Unique id of the calling thread's current CUDA context (cuCtxGetId, resolved
// through the runtime's driver entry-point query so the library needs no link
// against libcuda).  0 if the query is unavailable.
unsigned long long current_context_id() {
  using CtxGetCurrent = CUresult (*)(CUcontext*);
  using CtxGetId = CUresult (*)(CUcontext, unsigned long long*);
  static CtxGetCurrent get_current = nullptr;
  static CtxGetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_noalloc_scores for the current device.  In host code the
// array's name only stands for the symbol, so the address is looked up with
// cudaGetSymbolAddress, with that device current, once per device and context,
// and cached.  The cache remembers the context's unique id: after a device
// reset (a new primary context) the next call looks the address up again.
rmm_status noalloc_scores(double** out) {
  static std::mutex mu;
  static double* cached[64] = {};
  static unsigned long long cached_ctx[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(RMM_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (cached[dev] == nullptr || ctx == 0 || cached_ctx[dev] != ctx) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scores);
    if (e != cudaSuccess || ptr == nullptr) return cuda_fail(e, "cudaGetSymbolAddress(score scratch)");
    cached[dev] = static_cast<double*>(ptr);
    cached_ctx[dev] = current_context_id();  // the lookup may have created the primary context
  }
  *out = cached[dev];
  return RMM_OK;
}
}  // namespace

extern "C" {

rmm_status rmm_select_noalloc(const rmm_bf16* A, int64_t batch, int64_t batch_stride, int64_t n, int64_t d,
                              int64_t lda, int causal, double rho, int32_t* idx_out, double* retained_out,
                              rmm_stream stream) {
  t_last_error.clear();
  if (rmm_status st = check_rho(rho)) return st;
  if (A == nullptr || idx_out == nullptr) return fail(RMM_ERR_INVALID_ARG, "A and idx_out are required");
  if (batch < 1 || n < 1 || d < 1) return fail(RMM_ERR_INVALID_ARG, "batch, n and d must be >= 1");
  if (lda < d) return fail(RMM_ERR_INVALID_ARG, "lda < d");
  if (batch > 1 && batch_stride < (n - 1) * lda + d) return fail(RMM_ERR_INVALID_ARG, "batch_stride too small");
  if (causal != 0 && causal != 1) return fail(RMM_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (d > kMaxSelectD) return fail(RMM_ERR_UNSUPPORTED, "d > %lld", static_cast<long long>(kMaxSelectD));
  // batch > kNoAllocScores / d  <=>  batch * d > kNoAllocScores, without forming the product
  if (batch > kNoAllocScores / d)
    return fail(RMM_ERR_UNSUPPORTED,
                "rmm_select_noalloc holds at most %lld scores (batch * d); got batch %lld x d %lld -- use rmm_select "
                "with a workspace",
                static_cast<long long>(kNoAllocScores), static_cast<long long>(batch), static_cast<long long>(d));
  if (n > kIntMax || batch > 65535) return fail(RMM_ERR_UNSUPPORTED, "n or batch too large");
  if (!aligned16(A) || (lda % 8) != 0 || (batch > 1 && (batch_stride % 8) != 0))
    return fail(RMM_ERR_UNSUPPORTED, "A must be 16-byte aligned with lda and batch_stride multiples of 8");
  double* colsq = nullptr;
  if (rmm_status st = noalloc_scores(&colsq)) return st;
  // every score of [0, batch * d) is rewritten below, so nothing needs clearing
  const int64_t k = rmm_k(rho, d);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (rmm_status st = launch_colsq(A, batch, batch_stride, n, d, lda, causal != 0, d - n, colsq, s)) return st;
  return launch_select(colsq, batch, d, k, idx_out, retained_out, s);
}

// ---------------------------------------------------------------- linear
size_t rmm_linear_workspace_bytes(int64_t n, int64_t d, int64_t m, double rho) {
  const int64_t k = rmm_k(rho, d);
  if (k < 0 || n < 1 || m < 1) return 0;
  Carver c(nullptr);
  if (n <= kDecodeMaxRows) {
    if (k < d) {
      c.take<double>(d);
      c.take<int32_t>(k);
      c.take<uint16_t>(n * round_up(k, 8));
    }
    c.take<float>(static_cast<int64_t>(decode_partial_floats(n, m, k)));
    return c.bytes();
  }
  if (k == d) return 0;
  c.take<double>(d);
  c.take<int32_t>(k);
  c.take<uint16_t>(n * round_up(k, 8));
  c.take<uint16_t>(k * round_up(m, 8));
  return c.bytes();
}

rmm_status rmm_linear(const rmm_bf16* A, int64_t n, int64_t d, int64_t lda, const rmm_bf16* B, int64_t m,
                      int64_t ldb, rmm_bf16* Y, int64_t ldy, double rho, int32_t* idx_out, void* ws, size_t ws_bytes,
                      rmm_stream stream) {
  t_last_error.clear();
  if (rmm_status st = check_rho(rho)) return st;
  if (A == nullptr || B == nullptr || Y == nullptr) return fail(RMM_ERR_INVALID_ARG, "A, B and Y are required");
  if (n < 1 || d < 1 || m < 1) return fail(RMM_ERR_INVALID_ARG, "n, d and m must be >= 1");
  if (lda < d || ldb < m || ldy < m) return fail(RMM_ERR_INVALID_ARG, "leading dimension too small");
  if (!aligned16(A) || !aligned16(B) || !aligned16(Y) || (lda % 8) || (ldb % 8) || (ldy % 8))
    return fail(RMM_ERR_UNSUPPORTED, "pointers must be 16-byte aligned and leading dims multiples of 8");
  if (n > kIntMax - 128 || m > kIntMax - 256 || d > kIntMax - 64)
    return fail(RMM_ERR_UNSUPPORTED, "dimension too large");
  const int64_t k = rmm_k(rho, d);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n <= kDecodeMaxRows) {
    // decode: stream only the kept rows of B (all rows when rho = 1)
    if (d > kMaxSelectD && k < d) return fail(RMM_ERR_UNSUPPORTED, "d > %lld", static_cast<long long>(kMaxSelectD));
    const size_t need = rmm_linear_workspace_bytes(n, d, m, rho);
    if (ws == nullptr || ws_bytes < need)
      return fail(RMM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
    Carver c(ws);
    if (k == d) {
      float* partial = c.take<float>(static_cast<int64_t>(decode_partial_floats(n, m, k)));
      if (idx_out != nullptr) {
        const cudaError_t e = launch_chained(iota_kernel, dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(d, 256), 1024))), dim3(256), 0, s, idx_out, 1, d);
        if (e != cudaSuccess) return cuda_fail(e, "iota launch");
      }
      return decode_product(A, n, lda, B, d, m, ldb, nullptr, partial, Y, ldy, s);
    }
    const int64_t k_pad = round_up(k, 8);
    double* colsq = c.take<double>(d);
    int32_t* idx_ws = c.take<int32_t>(k);
    uint16_t* xpack = c.take<uint16_t>(n * k_pad);
    float* partial = c.take<float>(static_cast<int64_t>(decode_partial_floats(n, m, k)));
    int32_t* idx = idx_out ? idx_out : idx_ws;
    if (decode_select_fits(n, d)) {
      if (rmm_status st = launch_decode_select(A, n, d, lda, k, idx, xpack, k_pad, s)) return st;
    } else {
      if (rmm_status st = launch_colsq(A, 1, 0, n, d, lda, false, 0, colsq, s)) return st;
      if (rmm_status st = launch_select(colsq, 1, d, k, idx, nullptr, s)) return st;
      if (rmm_status st = pack_columns(A, n, d, lda, idx, k, xpack, k_pad, s)) return st;
    }
    return decode_product(xpack, n, k_pad, B, k, m, ldb, idx, partial, Y, ldy, s);
  }
  if (k == d) {
    // rho = 1: the dense product, I = [0, d)
    if (idx_out != nullptr) {
      const cudaError_t e = launch_chained(iota_kernel, dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(d, 256), 1024))), dim3(256), 0, s, idx_out, 1, d);
      if (e != cudaSuccess) return cuda_fail(e, "iota launch");
    }
    return gemm_packed(A, n, d, lda, B, m, ldb, Y, ldy, s);
  }
  if (d > kMaxSelectD) return fail(RMM_ERR_UNSUPPORTED, "d > %lld", static_cast<long long>(kMaxSelectD));
  const size_t need = rmm_linear_workspace_bytes(n, d, m, rho);
  if (ws == nullptr || ws_bytes < need)
    return fail(RMM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
  const int64_t k_pad = round_up(k, 8);
  const int64_t m_pad = round_up(m, 8);
  Carver c(ws);
  double* colsq = c.take<double>(d);
  int32_t* idx_ws = c.take<int32_t>(k);
  uint16_t* apack = c.take<uint16_t>(n * k_pad);
  int32_t* idx = idx_out ? idx_out : idx_ws;

  uint16_t* bpack = c.take<uint16_t>(k * m_pad);
  if (rmm_status st = launch_colsq(A, 1, 0, n, d, lda, false, 0, colsq, s)) return st;
  if (rmm_status st = launch_select(colsq, 1, d, k, idx, nullptr, s)) return st;
  if (rmm_status st = pack_columns(A, n, d, lda, idx, k, apack, k_pad, s)) return st;
  // the kept rows of B are packed and streamed by TMA tiles: measured on B200, this
  // beats reading them through the index set inside the product (rmm_gemm_gathered)
  if (rmm_status st = gather_rows(B, m, ldb, idx, k, bpack, m_pad, s)) return st;
  return gemm_packed(apack, n, k, k_pad, bpack, m, m_pad, Y, ldy, s);
}

rmm_status rmm_gather_columns(const rmm_bf16* A, int64_t n, int64_t d, int64_t lda, const int32_t* idx, int64_t k,
                              rmm_bf16* A_pack, int64_t ld_pack, rmm_stream stream) {
  t_last_error.clear();
  if (A == nullptr || idx == nullptr || A_pack == nullptr) return fail(RMM_ERR_INVALID_ARG, "null pointer");
  if (n < 1 || d < 1 || k < 1 || k > d || lda < d || ld_pack < k)
    return fail(RMM_ERR_INVALID_ARG, "need n, d >= 1, 1 <= k <= d, lda >= d, ld_pack >= k");
  if (!aligned16(A) || !aligned16(A_pack) || (lda % 8) || (ld_pack % 8))
    return fail(RMM_ERR_UNSUPPORTED, "pointers must be 16-byte aligned and leading dims multiples of 8");
  if (d > kMaxSelectD || n > kIntMax) return fail(RMM_ERR_UNSUPPORTED, "dimension too large");
  return pack_columns(A, n, d, lda, idx, k, A_pack, ld_pack, static_cast<cudaStream_t>(stream));
}

rmm_status rmm_gather_rows(const rmm_bf16* B, int64_t d, int64_t m, int64_t ldb, const int32_t* idx, int64_t k,
                           rmm_bf16* B_pack, int64_t ld_pack, rmm_stream stream) {
  t_last_error.clear();
  if (B == nullptr || idx == nullptr || B_pack == nullptr) return fail(RMM_ERR_INVALID_ARG, "null pointer");
  if (d < 1 || m < 1 || k < 1 || k > d || ldb < m || ld_pack < m)
    return fail(RMM_ERR_INVALID_ARG, "need d, m >= 1, 1 <= k <= d, ldb and ld_pack >= m");
  if (!aligned16(B) || !aligned16(B_pack) || (ldb % 8) || (ld_pack % 8))
    return fail(RMM_ERR_UNSUPPORTED, "pointers must be 16-byte aligned and leading dims multiples of 8");
  return gather_rows(B, m, ldb, idx, k, B_pack, ld_pack, static_cast<cudaStream_t>(stream));
}

rmm_status rmm_gemm_gathered(const rmm_bf16* A_pack, int64_t n, int64_t k, int64_t lda, const rmm_bf16* B, int64_t d,
                             int64_t m, int64_t ldb, const int32_t* idx, rmm_bf16* Y, int64_t ldy, rmm_stream stream) {
  t_last_error.clear();
  if (A_pack == nullptr || B == nullptr || idx == nullptr || Y == nullptr) return fail(RMM_ERR_INVALID_ARG, "null pointer");
  if (n < 1 || k < 1 || d < 1 || k > d || m < 1 || lda < k || ldb < m || ldy < m)
    return fail(RMM_ERR_INVALID_ARG, "need n, m >= 1, 1 <= k <= d, lda >= k, ldb and ldy >= m");
  if (!aligned16(A_pack) || !aligned16(B) || !aligned16(Y) || (lda % 8) || (ldb % 8) || (ldy % 8))
    return fail(RMM_ERR_UNSUPPORTED, "pointers must be 16-byte aligned and leading dims multiples of 8");
  if (n > kIntMax - 256 || m > kIntMax - 256 || k > kIntMax - 64) return fail(RMM_ERR_UNSUPPORTED, "dimension too large");
  return gemm_gathered(A_pack, n, k, lda, B, m, ldb, idx, Y, ldy, static_cast<cudaStream_t>(stream));
}

rmm_status rmm_gemm_packed(const rmm_bf16* A_pack, int64_t n, int64_t k, int64_t lda, const rmm_bf16* B_pack,
                           int64_t m, int64_t ldb, rmm_bf16* Y, int64_t ldy, rmm_stream stream) {
  t_last_error.clear();
  if (A_pack == nullptr || B_pack == nullptr || Y == nullptr) return fail(RMM_ERR_INVALID_ARG, "null pointer");
  if (n < 1 || k < 1 || m < 1 || lda < k || ldb < m || ldy < m)
    return fail(RMM_ERR_INVALID_ARG, "need n, k, m >= 1, lda >= k, ldb and ldy >= m");
  if (!aligned16(A_pack) || !aligned16(B_pack) || !aligned16(Y) || (lda % 8) || (ldb % 8) || (ldy % 8))
    return fail(RMM_ERR_UNSUPPORTED, "pointers must be 16-byte aligned and leading dims multiples of 8");
  if (n > kIntMax - 128 || m > kIntMax - 256 || k > kIntMax - 64) return fail(RMM_ERR_UNSUPPORTED, "dimension too large");
  return gemm_packed(A_pack, n, k, lda, B_pack, m, ldb, Y, ldy, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- QK^T
size_t rmm_qk_workspace_bytes(int64_t batch, int64_t hq, int64_t hkv, int64_t nq, int64_t nk, int64_t dh,
                              double rho) {
  (void)hkv;
  (void)nk;
  const int64_t k = rmm_k(rho, dh);
  if (k < 0 || batch < 1 || hq < 1 || nq < 1) return 0;
  if (k == dh) return 0;
  const int64_t items = batch * hq;
  Carver c(nullptr);
  c.take<double>(items * dh);
  c.take<int32_t>(items * k);
  c.take<uint8_t>(items * dh);
  c.take<uint16_t>(items * nq * dh);
  return c.bytes();
}

rmm_status rmm_qk(const rmm_bf16* Q, const rmm_bf16* K, float* S, int64_t batch, int64_t hq, int64_t hkv, int64_t nq,
                  int64_t nk, int64_t dh, int causal, float scale, double rho, int32_t* idx_out, void* ws,
                  size_t ws_bytes, rmm_stream stream) {
  t_last_error.clear();
  if (rmm_status st = check_rho(rho)) return st;
  if (Q == nullptr || K == nullptr || S == nullptr) return fail(RMM_ERR_INVALID_ARG, "Q, K and S are required");
  if (batch < 1 || hq < 1 || hkv < 1 || nq < 1 || nk < 1 || dh < 1)
    return fail(RMM_ERR_INVALID_ARG, "sizes must be >= 1");
  if (hq % hkv) return fail(RMM_ERR_INVALID_ARG, "Hq (%lld) must be a multiple of Hkv (%lld)",
                            static_cast<long long>(hq), static_cast<long long>(hkv));
  if (causal != 0 && causal != 1) return fail(RMM_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (!std::isfinite(scale)) return fail(RMM_ERR_INVALID_ARG, "scale must be finite");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(S) || (dh % 8) || (nk % 4))
    return fail(RMM_ERR_UNSUPPORTED, "pointers must be 16-byte aligned, dh % 8 == 0 and nk % 4 == 0");
  if (dh > kMaxSelectD) return fail(RMM_ERR_UNSUPPORTED, "dh too large");
  const int64_t items = batch * hq;
  if (items > 65535 || items * nq > kIntMax - 128 || batch * hkv * nk > kIntMax - 256 || items * nk > kIntMax - 256)
    return fail(RMM_ERR_UNSUPPORTED, "problem too large");
  const int64_t k = rmm_k(rho, dh);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  GemmParams g = gemm_defaults();
  g.M = static_cast<int>(nq);
  g.N = static_cast<int>(nk);
  g.batch = static_cast<int>(items);
  g.m_tiles = static_cast<int>(ceil_div(nq, 128));
  g.n_tiles = static_cast<int>(ceil_div(nk, 256));
  g.a_rows_per_batch = static_cast<int>(nq);
  g.out = S;
  g.ldo = nk;
  g.out_bstride = nq * nk;
  g.scale = scale;
  g.causal_off = nk - nq;
  CUtensorMap ta, tb;
  if (k == dh) {
    if (rmm_status st = make_tmap(&ta, Q, dh, items * nq, dh * 2, 64, 128)) return st;
    if (rmm_status st = make_tmap(&tb, K, dh, batch * hkv * nk, dh * 2, 64, 256)) return st;
    g.k = static_cast<int>(dh);
    g.num_kb = static_cast<int>(ceil_div(dh, 64));
    g.b_g_outer = static_cast<int>(hq);
    g.b_g_inner = static_cast<int>(hq / hkv);
    g.b_s_outer = hkv * nk;
    g.b_s_inner = nk;
    if (idx_out != nullptr) {
      const cudaError_t e = launch_chained(iota_kernel, dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(items * dh, 256), 1024))), dim3(256), 0, s, idx_out, items, dh);
      if (e != cudaSuccess) return cuda_fail(e, "iota launch");
    }
  } else {
    // QK^T is bound by writing S: the dropped head dims of each query head are
    // zeroed (Q_m) and the dense product with K runs as is -- exactly
    // sum_{j in I_h} Q_h[:, j] K_g(h)[:, j]^T, without packed Q_I / K_I copies.
    const size_t need = rmm_qk_workspace_bytes(batch, hq, hkv, nq, nk, dh, rho);
    if (ws == nullptr || ws_bytes < need)
      return fail(RMM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
    Carver c(ws);
    double* colsq = c.take<double>(items * dh);
    int32_t* idx_ws = c.take<int32_t>(items * k);
    uint8_t* keep = c.take<uint8_t>(items * dh);
    uint16_t* qm = c.take<uint16_t>(items * nq * dh);
    int32_t* idx = idx_out ? idx_out : idx_ws;
    if (rmm_status st = launch_colsq(Q, items, nq * dh, nq, dh, dh, false, 0, colsq, s)) return st;
    if (rmm_status st = launch_select(colsq, items, dh, k, idx, nullptr, s, keep)) return st;
    MaskParams mp{};
    mp.src = Q;
    mp.dst = qm;
    mp.rows = nq;
    mp.cols = dh;
    mp.keep = keep;
    mp.by_rows = 0;
    mp.batch = items;
    mp.g_outer = 1;
    mp.g_inner = 1;
    mp.s_outer = nq * dh;
    if (rmm_status st = launch_mask(mp, s)) return st;
    if (rmm_status st = make_tmap(&ta, qm, dh, items * nq, dh * 2, 64, 128)) return st;
    if (rmm_status st = make_tmap(&tb, K, dh, batch * hkv * nk, dh * 2, 64, 256)) return st;
    g.k = static_cast<int>(dh);
    g.num_kb = static_cast<int>(ceil_div(dh, 64));
    g.b_g_outer = static_cast<int>(hq);
    g.b_g_inner = static_cast<int>(hq / hkv);
    g.b_s_outer = hkv * nk;
    g.b_s_inner = nk;
  }
  if (causal) return launch_gemm<256, kBTileK, kEpiF32, kCausalMaskScores>(ta, tb, g, s);
  return launch_gemm<256, kBTileK, kEpiF32, kCausalNone>(ta, tb, g, s);
}

// ---------------------------------------------------------------- PV
size_t rmm_pv_workspace_bytes(int64_t batch, int64_t h, int64_t hkv, int64_t nq, int64_t nk, int64_t dh, double rho) {
  (void)hkv;
  (void)nq;
  const int64_t k = rmm_k(rho, nk);
  if (k < 0 || batch < 1 || h < 1 || dh < 1) return 0;
  if (k == nk) return 0;
  const int64_t items = batch * h;
  Carver c(nullptr);
  c.take<double>(items * nk);
  c.take<int32_t>(items * k);
  c.take<uint8_t>(items * nk);
  c.take<uint16_t>(items * nk * dh);
  return c.bytes();
}

rmm_status rmm_pv(const rmm_bf16* P, const rmm_bf16* V, rmm_bf16* O, int64_t batch, int64_t h, int64_t hkv,
                  int64_t nq, int64_t nk, int64_t dh, int causal, double rho, int32_t* idx_out, void* ws,
                  size_t ws_bytes, rmm_stream stream) {
  t_last_error.clear();
  if (rmm_status st = check_rho(rho)) return st;
  if (P == nullptr || V == nullptr || O == nullptr) return fail(RMM_ERR_INVALID_ARG, "P, V and O are required");
  if (batch < 1 || h < 1 || hkv < 1 || nq < 1 || nk < 1 || dh < 1)
    return fail(RMM_ERR_INVALID_ARG, "sizes must be >= 1");
  if (h % hkv) return fail(RMM_ERR_INVALID_ARG, "H must be a multiple of Hkv");
  if (causal != 0 && causal != 1) return fail(RMM_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (!aligned16(P) || !aligned16(V) || !aligned16(O) || (nk % 8) || (dh != 64 && dh != 128))
    return fail(RMM_ERR_UNSUPPORTED, "pointers must be 16-byte aligned, nk % 8 == 0 and dh in {64, 128}");
  if (nk > kMaxSelectD) return fail(RMM_ERR_UNSUPPORTED, "nk > %lld", static_cast<long long>(kMaxSelectD));
  const int64_t items = batch * h;
  if (items > 65535 || items * nq > kIntMax - 128 || batch * hkv * nk > kIntMax - 64)
    return fail(RMM_ERR_UNSUPPORTED, "problem too large");
  const int64_t k = rmm_k(rho, nk);
  const int64_t off = nk - nq;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  GemmParams g = gemm_defaults();
  g.M = static_cast<int>(nq);
  g.N = static_cast<int>(dh);
  g.batch = static_cast<int>(items);
  g.m_tiles = static_cast<int>(ceil_div(nq, 128));
  g.n_tiles = 1;
  g.a_rows_per_batch = static_cast<int>(nq);
  g.out = O;
  g.ldo = dh;
  g.out_bstride = nq * dh;
  g.causal_off = off;
  g.b_g_outer = static_cast<int>(h);
  g.b_g_inner = static_cast<int>(h / hkv);
  g.b_s_outer = hkv * nk;
  g.b_s_inner = nk;
  CUtensorMap ta, tb;
  const bool dense = (k == nk);
  if (dense) {
    if (rmm_status st = make_tmap(&ta, P, nk, items * nq, nk * 2, 64, 128)) return st;
    if (rmm_status st = make_tmap(&tb, V, dh, batch * hkv * nk, dh * 2, 64, 64)) return st;
    g.k = static_cast<int>(nk);
    g.num_kb = static_cast<int>(ceil_div(nk, 64));
    g.idx = nullptr;
    if (idx_out != nullptr) {
      const cudaError_t e = launch_chained(iota_kernel, dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(items * nk, 256), 4096))), dim3(256), 0, s, idx_out, items, nk);
      if (e != cudaSuccess) return cuda_fail(e, "iota launch");
    }
  } else {
    // PV is bound by reading P: the V rows of dropped key positions are zeroed
    // (V_m, per query head) and the product streams P once -- exactly
    // sum_{j in I_h} P_h[:, j] V_g(h)[j, :], without a packed P_I.  With
    // causal = 1 the entries above the diagonal are masked in shared memory.
    const size_t need = rmm_pv_workspace_bytes(batch, h, hkv, nq, nk, dh, rho);
    if (ws == nullptr || ws_bytes < need)
      return fail(RMM_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
    Carver c(ws);
    double* colsq = c.take<double>(items * nk);
    int32_t* idx_ws = c.take<int32_t>(items * k);
    uint8_t* keep = c.take<uint8_t>(items * nk);
    uint16_t* vm = c.take<uint16_t>(items * nk * dh);
    int32_t* idx = idx_out ? idx_out : idx_ws;
    if (rmm_status st = launch_colsq(P, items, nq * nk, nq, nk, nk, causal != 0, off, colsq, s)) return st;
    if (rmm_status st = launch_select(colsq, items, nk, k, idx, nullptr, s, keep)) return st;
    MaskParams mp{};
    mp.src = V;
    mp.dst = vm;
    mp.rows = nk;
    mp.cols = dh;
    mp.keep = keep;
    mp.by_rows = 1;
    mp.batch = items;
    mp.g_outer = h;
    mp.g_inner = h / hkv;
    mp.s_outer = hkv * nk * dh;
    mp.s_inner = nk * dh;
    if (rmm_status st = launch_mask(mp, s)) return st;
    if (rmm_status st = make_tmap(&ta, P, nk, items * nq, nk * 2, 64, 128)) return st;
    if (rmm_status st = make_tmap(&tb, vm, dh, items * nk, dh * 2, 64, 64)) return st;
    g.k = static_cast<int>(nk);
    g.num_kb = static_cast<int>(ceil_div(nk, 64));
    g.idx = nullptr;
    g.b_g_outer = 1;
    g.b_g_inner = 1;
    g.b_s_outer = nk;
    g.b_s_inner = 0;
  }
  if (dh == 128)
    return causal ? launch_gemm<128, kBTileMN, kEpiBf16, kCausalLimitK>(ta, tb, g, s)
                  : launch_gemm<128, kBTileMN, kEpiBf16, kCausalNone>(ta, tb, g, s);
  return causal ? launch_gemm<64, kBTileMN, kEpiBf16, kCausalLimitK>(ta, tb, g, s)
                : launch_gemm<64, kBTileMN, kEpiBf16, kCausalNone>(ta, tb, g, s);
}

}  // extern "C"
