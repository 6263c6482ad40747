/*
 * rmm.h -- C ABI of the B200 (sm_100a) Reduced Matrix Multiplication library.
 *
 * Reduced Matrix Multiplication (RMM) replaces a product Y = A.B, with A (n x d)
 * the activations and B (d x m), by the reduced product over the contraction
 * indices whose activation columns carry the most energy:
 *
 *     s_j = ||A[:, j]||_2,   I = TopK_{k}(s),   k = ceil(rho * d),
 *     RMM_rho(A, B) = A[:, I] . B[I, :]
 *
 * Source: "Algorithm Deep-Dive: RMM -- TopK Column-Norm Slicing" (hackcv.com),
 * section "Core Approach (Formula Level)"; the same statement appears in
 * "RMM：把 Transformer 矩阵乘法切到刚好够用" (kaelemshawn.blog) and in the
 * gist.science technical summary of "Reduced Matrix Multiplication:
 * Input-Adaptive Matrix-Product Reduction for LLM Inference", Methodology.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Element types: activations, weights and products are bfloat16, passed as
 *    raw 16-bit patterns (rmm_bf16).  Accumulation is fp32 on the tensor cores;
 *    bf16 outputs are rounded to nearest even.  Column scores are fp64.
 *  - Layouts are row-major.  Leading dimensions (lda, ldb, ldy) count elements.
 *  - Index sets are int32, strictly ascending, of length k; ties in the column
 *    norm go to the lower index.
 *  - Ownership: the caller owns every buffer.  Device pointers must point to
 *    memory of the current CUDA device.  The library allocates nothing,
 *    keeps no state between calls and never synchronises: all work is enqueued
 *    on `stream` (an opaque cudaStream_t; NULL is the legacy default stream).
 *    Scratch memory is the caller's `ws` buffer of at least the size returned
 *    by the matching *_workspace_bytes() query (0 bytes is valid when the
 *    query returns 0).  Calls that share one workspace must be ordered.
 *  - Alignment: device pointers must be 16-byte aligned and leading dimensions
 *    multiples of 8 elements; otherwise RMM_ERR_UNSUPPORTED is returned.
 *  - Errors: argument problems are detected on the host and returned before
 *    anything is enqueued.  A failed launch returns RMM_ERR_CUDA.  Device-side
 *    faults surface on the caller's next synchronisation.  A kernel that waits
 *    on a barrier for about a second without progress gives up, records a code
 *    read by rmm_device_error(), and returns.  rmm_last_error() describes the
 *    most recent failure on the calling thread.
 *  - There is no CPU fallback: every compute step runs in the library's CUDA
 *    kernels (sm_100a only).
 */
#ifndef RMM_H_
#define RMM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t rmm_bf16; /* IEEE bfloat16 bit pattern */
typedef void* rmm_stream;  /* cudaStream_t */

typedef enum {
  RMM_OK = 0,
  RMM_ERR_INVALID_ARG = 1,    /* bad rho, negative or zero size, null pointer, Hq % Hkv != 0 ... */
  RMM_ERR_UNSUPPORTED = 2,    /* misaligned pointer / leading dim, size beyond the documented limits */
  RMM_ERR_WORKSPACE = 3,      /* ws_bytes smaller than the query's answer, or ws == NULL when needed */
  RMM_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
  RMM_ERR_DEVICE_TIMEOUT = 5  /* a kernel gave up on a bounded wait (see rmm_device_error) */
} rmm_status;

/* k = ceil(rho * d): the number of kept contraction indices.
 * ("The retention-ratio (rho) Knob": rho in (0, 1] keeps ceil(rho d) dims.)
 * Computed as ceil(x - 1e-9 x) with x = rho * d, so that products which land a
 * rounding step above an integer (0.1 * 30 = 3.0000000000000004) give the
 * intended value; clamped to [1, d].  Returns -1 if rho is not in (0, 1]
 * (NaN included) or d < 1. */
int64_t rmm_k(double rho, int64_t d);

/* ---------------------------------------------------------------- selection
 * rmm_select: column scores and TopK index set ("Core Approach": s_j =
 * ||A[:, j]||_2, keep the TopK-largest ceil(rho d)).  Batched: item b's matrix
 * starts at A + b * batch_stride (elements), n rows x d columns, leading
 * dimension lda.
 *   causal      0, or 1 to treat entries (i, j) with j > i + (d - n) as zero
 *               (bottom-right aligned causal attention probabilities; they are
 *               not read).
 *   idx_out     device int32 [batch][k], k = rmm_k(rho, d); required.
 *   colsq_out   device fp64 [batch][d] or NULL: q_j = sum_i A[i, j]^2.
 *   retained_out device fp64 [batch] or NULL: sum_{j in I} q_j / sum_j q_j.
 * Limits: d <= 32768, n < 2^31.  Workspace: rmm_select_workspace_bytes(). */
size_t rmm_select_workspace_bytes(int64_t batch, int64_t n, int64_t d);
rmm_status rmm_select(const rmm_bf16* A, int64_t batch, int64_t batch_stride, int64_t n, int64_t d, int64_t lda,
                      int causal, double rho, int32_t* idx_out, double* colsq_out, double* retained_out, void* ws,
                      size_t ws_bytes, rmm_stream stream);

/* rmm_select_noalloc: rmm_select for callers that cannot allocate device memory.
 * This entry point has no counterpart on the pages; it exists for hosts whose
 * device memory is owned by someone else (a framework allocator or a fixed
 * memory budget reserved up front) and for latency-critical paths where a
 * cudaMalloc/cudaFree, which may synchronise the device, is not acceptable.
 * It computes exactly what rmm_select computes (same kernels, same results)
 * but takes no workspace and returns no scores: the fp64 column scores live in
 * one fixed scratch array inside the library, RMM_SELECT_NOALLOC_MAX_SCORES
 * doubles (2 MiB) that every device which loads the library keeps until the
 * process exits.  Nothing is allocated by this call.
 *   - batch * d must not exceed RMM_SELECT_NOALLOC_MAX_SCORES; larger problems
 *     return RMM_ERR_UNSUPPORTED with a message naming the limit.
 *   - The first call on a device looks up the scratch array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it; make that
 *     first call before any stream capture on the device.  The cache is keyed
 *     on the current context's unique id, so a call after cudaDeviceReset (a
 *     new context) looks the address up again: make that call before any
 *     stream capture too.
 *   - Every call on a device shares the one array.  Calls whose kernels can
 *     overlap on the GPU (different streams without ordering between them)
 *     race on it and give undefined results; order them on one stream or with
 *     events.  The array keeps the last call's scores, and each call rewrites
 *     all batch * d scores it uses before reading them.
 * Arguments, layouts and error behaviour are those of rmm_select. */
#define RMM_SELECT_NOALLOC_MAX_SCORES 262144
rmm_status rmm_select_noalloc(const rmm_bf16* A, int64_t batch, int64_t batch_stride, int64_t n, int64_t d,
                              int64_t lda, int causal, double rho, int32_t* idx_out, double* retained_out,
                              rmm_stream stream);

/* ---------------------------------------------------------------- linear
 * rmm_linear: Y = A[:, I] . B[I, :] with I selected on A (linear and MLP
 * projections X.W reduce the activation hidden dim: "Core Approach",
 * component mapping).
 *   A   device bf16 [n][lda], n x d activations.
 *   B   device bf16 [d][ldb], d x m, the contraction index is the ROW (the
 *       transpose of a torch nn.Linear weight, stored once; weights are not
 *       modified, rows outside I are simply not read).
 *   Y   device bf16 [n][ldy], n x m output.
 *   idx_out  device int32 [k] or NULL: the index set used.
 * rho == 1 runs the dense product A.B (no scores, no selection, no pack).
 * n > 128 reads the kept rows of B straight from B inside the tensor-core
 * product (CTA pairs); 32 < n <= 128 packs them first (one-CTA tiles).
 * n <= 32 runs the decode path (a gathered GEMV-shaped kernel that streams only
 * the kept rows of B; the scores, the selection and x[:, I] come from one
 * cluster launch when d <= 16384).  Limits: d <= 32768, n, m < 2^31. */
size_t rmm_linear_workspace_bytes(int64_t n, int64_t d, int64_t m, double rho);
rmm_status rmm_linear(const rmm_bf16* A, int64_t n, int64_t d, int64_t lda, const rmm_bf16* B, int64_t m,
                      int64_t ldb, rmm_bf16* Y, int64_t ldy, double rho, int32_t* idx_out, void* ws, size_t ws_bytes,
                      rmm_stream stream);

/* ---------------------------------------------------------------- linear stages
 * The steps that follow the selection in rmm_linear, exposed so a caller can
 * run (or time) them on their own.  rmm_linear with rho < 1 is rmm_select's
 * kernels followed by exactly rmm_gather_columns and rmm_gemm_gathered for
 * n > 128 rows, rmm_gather_columns, rmm_gather_rows and rmm_gemm_packed for
 * 32 < n <= 128 (one-CTA tiles); with rho = 1 it is rmm_gemm_packed on A and B
 * themselves.
 *
 * rmm_gather_columns: A_pack[i, t] = A[i, idx[t]] for t < k and 0 for
 * k <= t < ld_pack -- the gathered A[:, I] of "Core Approach", stored K-major.
 *   A       device bf16 [n][lda], n x d.
 *   idx     device int32 [k], entries in [0, d) (not checked on the host).
 *   A_pack  device bf16 [n][ld_pack]; ld_pack >= k and a multiple of 8.
 * rmm_gather_rows: B_pack[t, :] = B[idx[t], :] for t < k -- the kept rows
 * B[I, :] of "Core Approach", copied row-contiguous.
 *   B       device bf16 [d][ldb], d x m;  B_pack device bf16 [k][ld_pack],
 *   ld_pack >= m and a multiple of 8.
 * rmm_gemm_packed: Y = A_pack[:, :k] . B_pack[:k, :] on the tensor cores
 * (tcgen05, fp32 accumulation in tensor memory, bf16 output).
 *   A_pack [n][lda] (lda >= k), B_pack [k][ldb] (ldb >= m), Y [n][ldy].
 * rmm_gemm_gathered: Y = A_pack[:, :k] . B[idx[0:k], :] -- the reduced product
 * of "Core Approach" with the kept rows of B read through the index set
 * straight from B (no packed copy), on pairs of CTAs (tcgen05 cta_group::2).
 *   A_pack [n][lda] (lda >= k), B [d][ldb] (ldb >= m), idx device int32 [k]
 *   with entries in [0, d) (not checked on the host), Y [n][ldy].  The result
 *   equals rmm_gemm_packed on rmm_gather_rows' copy, bit for bit.
 * None of the four needs a workspace. */
rmm_status rmm_gather_columns(const rmm_bf16* A, int64_t n, int64_t d, int64_t lda, const int32_t* idx, int64_t k,
                              rmm_bf16* A_pack, int64_t ld_pack, rmm_stream stream);
rmm_status rmm_gather_rows(const rmm_bf16* B, int64_t d, int64_t m, int64_t ldb, const int32_t* idx, int64_t k,
                           rmm_bf16* B_pack, int64_t ld_pack, rmm_stream stream);
rmm_status rmm_gemm_packed(const rmm_bf16* A_pack, int64_t n, int64_t k, int64_t lda, const rmm_bf16* B_pack,
                           int64_t m, int64_t ldb, rmm_bf16* Y, int64_t ldy, rmm_stream stream);
rmm_status rmm_gemm_gathered(const rmm_bf16* A_pack, int64_t n, int64_t k, int64_t lda, const rmm_bf16* B, int64_t d,
                             int64_t m, int64_t ldb, const int32_t* idx, rmm_bf16* Y, int64_t ldy, rmm_stream stream);

/* ---------------------------------------------------------------- attention scores
 * rmm_qk: per query head h, I_h = TopK of the column norms of Q_h over its nq
 * rows (head-feature dims), then S_h = scale * Q_h[:, I_h] . K_g(h)[:, I_h]^T
 * with g(h) = h / (Hq / Hkv) under GQA ("Core Approach", component mapping:
 * QK^T selects along the head feature dim with score = Q column norm; under GQA
 * the selection is made on Q per head and K gathers the corresponding dims).
 *   Q  device bf16 [batch][Hq][nq][dh], contiguous.
 *   K  device bf16 [batch][Hkv][nk][dh], contiguous.
 *   S  device fp32 [batch][Hq][nq][nk], contiguous.  With causal = 1, entries
 *      with key j > i + (nk - nq) are -inf (bottom-right alignment).
 *   idx_out device int32 [batch][Hq][k] or NULL, k = rmm_k(rho, dh).
 * The product is bound by writing S, so the dropped head dims are zeroed in a
 * per-head copy of Q (workspace) and the tensor-core GEMM reads K as it is:
 * the result is exactly the reduced product.
 * Requires Hq % Hkv == 0, dh % 8 == 0, nk % 4 == 0, dh <= 32768. */
size_t rmm_qk_workspace_bytes(int64_t batch, int64_t hq, int64_t hkv, int64_t nq, int64_t nk, int64_t dh,
                              double rho);
rmm_status rmm_qk(const rmm_bf16* Q, const rmm_bf16* K, float* S, int64_t batch, int64_t hq, int64_t hkv, int64_t nq,
                  int64_t nk, int64_t dh, int causal, float scale, double rho, int32_t* idx_out, void* ws,
                  size_t ws_bytes, rmm_stream stream);

/* ---------------------------------------------------------------- attention output
 * rmm_pv: per head h, I_h = TopK over key positions of the column norms of P_h
 * taken over all query rows, then O_h = P_h[:, I_h] . V_g(h)[I_h, :]
 * ("Core Approach", component mapping: PV selects along token positions).
 *   P  device bf16 [batch][H][nq][nk], contiguous (attention probabilities).
 *   V  device bf16 [batch][Hkv][nk][dh], contiguous.
 *   O  device bf16 [batch][H][nq][dh], contiguous.
 *   causal = 1 treats P[i, j] with j > i + (nk - nq) as zero: those entries are
 *   not read for the scores and are zeroed before any product uses them.
 *   idx_out device int32 [batch][H][k] or NULL, k = rmm_k(rho, nk).
 * The product is bound by reading P, so the V rows of dropped positions are
 * zeroed in a per-head copy of V (workspace) and P is streamed once by the
 * tensor-core GEMM: the result is exactly the reduced product.
 * Requires H % Hkv == 0, nk % 8 == 0, dh == 64 or 128, nk <= 32768. */
size_t rmm_pv_workspace_bytes(int64_t batch, int64_t h, int64_t hkv, int64_t nq, int64_t nk, int64_t dh, double rho);
rmm_status rmm_pv(const rmm_bf16* P, const rmm_bf16* V, rmm_bf16* O, int64_t batch, int64_t h, int64_t hkv,
                  int64_t nq, int64_t nk, int64_t dh, int causal, double rho, int32_t* idx_out, void* ws,
                  size_t ws_bytes, rmm_stream stream);

/* ---------------------------------------------------------------- fused reduced attention
 * O_h = softmax_rows(scale * Q_h[:, I_h] K_g(h)[:, I_h]^T, causal) V_g(h) in one
 * kernel, S and P kept on chip ("Algorithm Deep-Dive: RMM", Component mapping:
 * QK^T selects head dims by the Q column norm, K gathers them under GQA; Attention
 * vs MLP, Table 16: attention-internal reduction).  I_h is chosen exactly as in
 * rmm_qk; the softmax and the value product are the ordinary ones.  For
 * k <= 64 the score product runs over 64 dims: Q[:, I_h] and K_g(h)[:, I_h] are
 * packed per query head into the workspace (zero past k); for 64 < k < dh it reads
 * Q with the dropped dims of each head zeroed (workspace) and K as it is.
 *   Q  device bf16 [batch][hq][nq][dh], K / V [batch][hkv][nk][dh], contiguous.
 *   O  device bf16 [batch][hq][nq][dh].
 *   causal = 1: bottom-right aligned (key j visible to query i iff j <= i + nk - nq),
 *   requires nq <= nk.  idx_out device int32 [batch][hq][k] or NULL.
 * Requires dh == 128.  Workspace: rmm_attention_workspace_bytes (0 at rho = 1). */
size_t rmm_attention_workspace_bytes(int64_t batch, int64_t hq, int64_t hkv, int64_t nq, int64_t nk, int64_t dh,
                                     double rho);
rmm_status rmm_attention(const rmm_bf16* Q, const rmm_bf16* K, const rmm_bf16* V, rmm_bf16* O, int64_t batch,
                         int64_t hq, int64_t hkv, int64_t nq, int64_t nk, int64_t dh, int causal, float scale,
                         double rho, int32_t* idx_out, void* ws, size_t ws_bytes, rmm_stream stream);

/* ---------------------------------------------------------------- int8 weights
 * Reduced projection with int8 weights for decode (n <= 32 rows):
 *   Y = (A[:, I] . Wq[I, :]) * scale[None, :]
 * with I = TopK of A's column norms exactly as in rmm_linear ("Reduced Matrix
 * Multiplication ... Technical Summary", Compatibility: INT8 weight
 * quantization; "Algorithm Deep-Dive: RMM", Compatibility & generalization).
 * The weights are stored int8 with one fp32 scale per output column (W = Wq *
 * scale, a reading: the pages name no scheme); only the kept rows of Wq are
 * read, with fp32 accumulation: on the CUDA cores for n <= 2, on the tensor
 * cores for 3 <= n <= 32 (the kept rows dequantised exactly to bf16 in shared
 * memory, the scales applied to the fp32 sums).
 *   A      device bf16 [n][lda], n x d, n <= 32.
 *   Wq     device int8 [d][ldw], d x m (contraction index as the row), ldw % 8 == 0.
 *   scale  device fp32 [m].
 *   Y      device bf16 [n][ldy].
 *   idx_out device int32 [rmm_k(rho, d)] or NULL.
 * Requires m % 8 == 0, d <= 32768.  Workspace: scores, index set and fp32
 * partial sums (added in a fixed order); for n <= 2 the kernel reads A[:, I]
 * through the index set, for larger n the selection packs it. */
size_t rmm_linear_int8_workspace_bytes(int64_t n, int64_t d, int64_t m, double rho);
rmm_status rmm_linear_int8(const rmm_bf16* A, int64_t n, int64_t d, int64_t lda, const int8_t* Wq, int64_t m,
                           int64_t ldw, const float* scale, rmm_bf16* Y, int64_t ldy, double rho, int32_t* idx_out,
                           void* ws, size_t ws_bytes, rmm_stream stream);

/* ---------------------------------------------------------------- MLP block
 * The gate / up / down projections of a gated MLP ("Algorithm Deep-Dive: RMM",
 * Attention vs MLP: structural asymmetry, and Engineering Notes: conservative
 * MLP rho, Down can be lower).  Gate and up contract the same input X, so ONE
 * index set I (TopK of X's column norms, rho_gu) serves both, and one fused
 * tensor-core product on CTA pairs writes
 *   H = SiLU(X[:, I] Wg[I, :]) * (X[:, I] Wu[I, :]),   SiLU(x) = x / (1 + e^-x);
 * then Y = RMM_rho_down(H, Wd) exactly as rmm_linear (its own selection on H).
 *   X   device bf16 [n][ldx], n x d.
 *   Wg, Wu device bf16 [d][ldw], d x f (contraction index as the row).
 *   Wd  device bf16 [f][ldwd], f x m.
 *   H   device bf16 [n][ldh], written (the down projection's input).
 *   Y   device bf16 [n][ldy].
 *   idx_gu_out  device int32 [rmm_k(rho_gu, d)] or NULL; idx_down_out device
 *   int32 [rmm_k(rho_down, f)] or NULL.
 *   ws  rmm_mlp_workspace_bytes(n, d, f, m, rho_gu, rho_down) bytes (0 at
 *   rho_gu = rho_down = 1 with n > 32: NULL allowed).
 * Limits: d, f <= 32768; leading dims multiples of 8, pointers 16-byte aligned. */
size_t rmm_mlp_workspace_bytes(int64_t n, int64_t d, int64_t f, int64_t m, double rho_gu, double rho_down);
rmm_status rmm_mlp(const rmm_bf16* X, int64_t n, int64_t d, int64_t ldx, const rmm_bf16* Wg, const rmm_bf16* Wu,
                   int64_t f, int64_t ldw, const rmm_bf16* Wd, int64_t m, int64_t ldwd, rmm_bf16* H, int64_t ldh,
                   rmm_bf16* Y, int64_t ldy, double rho_gu, double rho_down, int32_t* idx_gu_out,
                   int32_t* idx_down_out, void* ws, size_t ws_bytes, rmm_stream stream);

/* ---------------------------------------------------------------- decode attention
 * One query row per head against a key/value cache ("Algorithm Deep-Dive: RMM",
 * Component mapping and Engineering Notes: decode prunes attention).  The
 * G = hq / hkv query rows that share a key/value head are the rows of A, so each
 * (batch item, key/value head) group gets ONE index set, chosen on the column
 * norms of its G rows, and its cache rows are read once for the whole group.
 * Query head h of batch item b belongs to group b * hkv + h / G.
 *
 * rmm_decode_qk: I_g = TopK of the column norms of Q_g over the dh head dims,
 *   S[b][h][j] = scale * sum_{t in I_g} Q[b][h][t] * Kt[b][g][t][j], j < nk.
 *   Q   device bf16 [batch][hq][dh], contiguous.
 *   Kt  device bf16 [batch][hkv][dh][ldk]: the key cache stored dim-major
 *       (token j of dim t at Kt[..][t][j]) so that a kept dim is one contiguous
 *       row; tokens j < nk are valid, ldk >= nk and a multiple of 8 (columns up
 *       to the next multiple of 8 past nk are read, and ignored).
 *   S   device fp32 [batch][hq][lds], lds >= nk and a multiple of 4.
 *   idx_out device int32 [batch][hkv][k] or NULL, k = rmm_k(rho, dh).
 *   Requires dh % 8 == 0, dh <= 512, hq / hkv in {1, 2, 4, 8}.
 * rmm_decode_pv: I_g = TopK of the column norms of P_g over the nk positions,
 *   O[b][h][:] = sum_{j in I_g} P[b][h][j] * V[b][g][j][:].
 *   P   device bf16 [batch][hq][ldp] (softmax probabilities of the one query
 *       row), ldp >= nk and a multiple of 8.
 *   V   device bf16 [batch][hkv][cap][dh]: the value cache, token-major, cap >= nk.
 *   O   device bf16 [batch][hq][dh], contiguous.
 *   idx_out device int32 [batch][hkv][k] or NULL, k = rmm_k(rho, nk).
 *   Requires dh in {64, 128, 256}, hq / hkv in {1, 2, 4, 8}, (hq / hkv) * dh
 *   <= 1024, nk <= 32768.
 * rho = 1 reads the whole cache (no scores, no selection).  Workspaces: the
 * scores and index sets (rho < 1) and, for PV, fp32 partial sums of the token
 * chunks that a fix-up kernel adds in a fixed order (deterministic). */
size_t rmm_decode_qk_workspace_bytes(int64_t batch, int64_t hq, int64_t hkv, int64_t dh, double rho);
rmm_status rmm_decode_qk(const rmm_bf16* Q, const rmm_bf16* Kt, float* S, int64_t batch, int64_t hq, int64_t hkv,
                         int64_t dh, int64_t nk, int64_t ldk, int64_t lds, float scale, double rho, int32_t* idx_out,
                         void* ws, size_t ws_bytes, rmm_stream stream);
size_t rmm_decode_pv_workspace_bytes(int64_t batch, int64_t hq, int64_t hkv, int64_t nk, int64_t dh, double rho);
rmm_status rmm_decode_pv(const rmm_bf16* P, const rmm_bf16* V, rmm_bf16* O, int64_t batch, int64_t hq, int64_t hkv,
                         int64_t nk, int64_t ldp, int64_t cap, int64_t dh, double rho, int32_t* idx_out, void* ws,
                         size_t ws_bytes, rmm_stream stream);

/* ---------------------------------------------------------------- diagnostics */
const char* rmm_status_string(rmm_status s);
/* Message of the most recent failure on the calling thread ("" if none). */
const char* rmm_last_error(void);
/* Reads and clears the device-side error word of the current device (0 = no
 * kernel gave up on a wait).  Synchronises the device.  Returns RMM_ERR_CUDA if
 * the read itself fails, else RMM_OK. */
rmm_status rmm_device_error(int32_t* code_out);
/* Library version, e.g. "rmm-b200 0.1". */
const char* rmm_version(void);

/* ---------------------------------------------------------------- test hooks
 * Two entry points that exist only so that tests can reach device code no
 * product call exposes on its own; neither is part of the method.
 *
 * rmm_debug_exp2_poly: y_poly[i] = the fused attention's FMA-pipe 2^x (x split
 * into its nearest integer n and f in [-1/2, 1/2], a cubic fitted to 2^f, the
 * packed-pair code the attention runs: relative error < 7.6e-5 for x in
 * [-125, 0], <= 1.6e-4
 * on [-126, -125) where the result can fall into the subnormal range, about
 * 2^-126 below -126) and y_exp2f[i] = CUDA's exp2f(x[i]), i < n.  All three are
 * device fp32 buffers.
 *
 * rmm_debug_gemm_expire_producer: rmm_gemm_packed's one-CTA tensor-core product
 * (n <= 128 only) in which the producer, once its ring of shared-memory stages
 * is full (k > 256), waits on a barrier that nothing arrives on, through the
 * same bounded wait as every other wait but with a 1 ms limit instead of about
 * one second.  That wait runs out and the kernel takes its timeout path: it
 * records code 1 (producer timeout) in the device error word (rmm_device_error),
 * the other roles see the abort and stop, copies in flight are drained, tensor
 * memory is freed and the kernel returns.  Y is left partly written. */
rmm_status rmm_debug_exp2_poly(const float* x, float* y_poly, float* y_exp2f, int64_t n, rmm_stream stream);
rmm_status rmm_debug_gemm_expire_producer(const rmm_bf16* A_pack, int64_t n, int64_t k, int64_t lda,
                                          const rmm_bf16* B_pack, int64_t m, int64_t ldb, rmm_bf16* Y, int64_t ldy,
                                          rmm_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* RMM_H_ */
