/*
 * gptq_b200.h — C ABI of the GPTQ layer-quantization library for NVIDIA B200 (sm_100a).
 *
 * The library quantizes one linear layer W (d_out x d_in, fp32, row-major) to a
 * b-bit group-wise integer grid with the GPTQ method:
 *
 *   1. gptq_hessian_accumulate   H (+)= 2 X^T X over calibration tokens X (n x d_in).
 *   2. gptq_prepare_hinv         lambda = damp_rel * mean(diag H), Hd = H + lambda I,
 *                                U = upper Cholesky factor of Hd^-1 (U^T U = Hd^-1).
 *   3. gptq_quantize_layer       greedy column-order rounding with OBS error compensation,
 *                                lazy 128-column blocks and one trailing update per block;
 *                                writes packed codes, fp16 scales and packed zero points.
 *   4. gptq_pack_int / gptq_dequant   packing of b-bit codes; W_hat = s * (q - z).
 *   5. gptq_dequant_gemm         Y = X W_hat^T straight from the packed arrays.
 *
 * Activation ordering (desc_act) visits the columns in another order:
 * gptq_act_sum_accumulate (beside stage 1) and gptq_act_order rank the columns,
 * gptq_prepare_hinv_permuted replaces stage 2, gptq_quantize_layer_act_order stage 3,
 * and gptq_dequant_g_idx reads the per-column group index the latter writes.
 *
 * Sources (page titles as printed; sections in quotes):
 *   - "GPTQ：基于近似二阶信息的大模型权重量化" (freeguideonline GPTQ tutorial):
 *     "对称与仿射量化" (q = round(x/s) + z, group-wise scale/zero),
 *     "阶段一：构建 Hessian 逆近似" (H = 2 X^T X + lambda I, upper Cholesky factor),
 *     "阶段二：贪婪顺序量化与懒惰批更新" (fixed column order, lazy batch updates),
 *     "阶段三：量化与反量化" (per-group scale found during the pass, INT x scale).
 *     "激活排序（desc_act）" (columns ranked by the sum of absolute input activations,
 *     the least influential quantized first).
 *   - "GPTQ/AWQ量化中Group Size的精确含义与计算" (feinterview group-size article):
 *     codes 0..2^b-1, scale and zero per group along the input dimension,
 *     group_size = -1 is one group per row, "存储代价" (16-bit scale, b-bit zero,
 *     symmetric stores no zero).
 *
 * Conventions for every entry point:
 *   - Pointers named as device pointers must point to memory of the current CUDA
 *     device; the caller owns all memory.  The library never allocates.
 *   - ``stream`` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Work is enqueued asynchronously on it; argument errors are returned at once
 *     and enqueue nothing.
 *   - Errors detected on the device (non-finite values, a non-positive pivot, a
 *     bounded wait that ran out) are recorded in a per-process device status word
 *     and returned by the next call of gptq_sync_status() on that stream
 *     (gptq_prepare_hinv synchronises by itself).
 *   - gptq_last_error() returns a thread-local text for the last failing call.
 *   - Nothing here is thread-safe against concurrent calls that share buffers.
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GPTQ_OK = 0,
    GPTQ_ERR_INVALID_ARG = 1,   /* bad pointer, size, layout or config value            */
    GPTQ_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement           */
    GPTQ_ERR_NOT_PD = 3,        /* damped Hessian not positive definite (bad_col set)    */
    GPTQ_ERR_NONFINITE = 4,     /* NaN or Inf found in an input                          */
    GPTQ_ERR_CUDA = 5,          /* a CUDA runtime or driver call failed                  */
    GPTQ_ERR_TIMEOUT = 6,       /* a bounded device-side wait ran out                    */
    GPTQ_ERR_WORKSPACE = 7      /* workspace missing or smaller than the query returned */
} gptq_status;

typedef enum { GPTQ_BF16 = 0, GPTQ_F32 = 1 } gptq_dtype;

/* Quantization settings (tutorial "代码示例" BaseQuantizeConfig: bits, group_size,
 * desc_act; group-size article: sym).
 *   bits        2, 3, 4 or 8.
 *   group_size  -1 (one group per row) or a divisor of block_size that is >= 16.
 *   sym         0 = asymmetric (zero point stored), 1 = symmetric (implicit zero 2^(bits-1)).
 *   block_size  lazy-batch width; 128 is the only value this build accepts.
 *   damp_rel    lambda = damp_rel * mean(diag H); must be >= 0 and finite.
 *   desc_act    0 = natural column order (gptq_quantize_layer); 1 = activation ordering,
 *               ascending sum of |x| (the tutorial's text: least influential columns first);
 *               2 = descending (the reading the flag's name suggests).  1 and 2 are run by
 *               gptq_quantize_layer_act_order, which rejects 0; gptq_quantize_layer rejects
 *               1 and 2.  Any other value is GPTQ_ERR_INVALID_ARG. */
typedef struct {
    int bits;
    int group_size;
    int sym;
    int block_size;
    float damp_rel;
    int desc_act;
} gptq_config;

/* Fill *cfg with bits=4, group_size=128, sym=0, block_size=128, damp_rel=0.01, desc_act=0. */
void gptq_default_config(gptq_config* cfg);

/* Static text for a status code; never NULL. */
const char* gptq_status_string(gptq_status s);

/* Text describing the last non-OK return on the calling thread ("" if none). */
const char* gptq_last_error(void);

/* Library version as major*10000 + minor*100 + patch. */
int gptq_version(void);

/* ------------------------------------------------------------------ stage 1
 * H (+)= 2 X^T X          (tutorial "阶段一", H = 2 X^T X)
 *   X        device, n x d_in row-major, bf16 (raw uint16 bit patterns) or fp32.
 *   H        device, d_in x d_in row-major fp32, written in full (both triangles).
 *   accumulate  0: H = 2 X^T X;  1: H += 2 X^T X (call once per calibration batch).
 *   ws       device workspace of at least gptq_hessian_workspace_bytes(n, d_in, xt) bytes.
 * Products are formed on the tensor cores (bf16 exact products, or fp32 split into
 * two tf32 parts with three products), accumulated in fp32.
 * Requires d_in % 8 == 0, 1 <= n, d_in <= 65536.  Non-finite X values propagate
 * into H and are reported by gptq_prepare_hinv. */
size_t gptq_hessian_workspace_bytes(int64_t n, int64_t d_in, gptq_dtype xt);
gptq_status gptq_hessian_accumulate(const void* X, gptq_dtype xt, int64_t n, int64_t d_in,
                                    float* H, int accumulate, void* ws, size_t ws_bytes,
                                    void* stream);

/* ------------------------------------------------------------------ stage 2
 * U = upper Cholesky factor of (H + lambda I)^-1, lambda = damp_rel * mean(diag H)
 * (tutorial "阶段一" steps 1-2 read as the upper factor of the inverse Hessian).
 *   H        device, d_in x d_in fp32, symmetric; only the upper triangle is read. Not modified.
 *   U        device, d_in x d_in fp32 row-major; written in full (strict lower triangle = 0).
 *   bad_col  host pointer or NULL; on GPTQ_ERR_NOT_PD receives the first failing column.
 *   lambda_out  host pointer or NULL; receives lambda.
 * Computed as Hd = R R^T with R upper (Cholesky from the bottom-right), then U = R^-1,
 * blocked by 128: fp32 diagonal blocks, every off-diagonal block product a 3xTF32
 * tensor-core tile, all in one persistent launch that takes the tiles in the dependency
 * order gptq_chol_schedule returns (one CTA per SM; waits between tiles are bounded).
 * Synchronises ``stream`` once to report NOT_PD / NONFINITE.  Returns
 * GPTQ_ERR_INVALID_ARG when mean(diag H) <= 0.  Requires d_in % 8 == 0. */
size_t gptq_prepare_hinv_workspace_bytes(int64_t d_in);
gptq_status gptq_prepare_hinv(const float* H, int64_t d_in, float damp_rel, float* U,
                              void* ws, size_t ws_bytes, int64_t* bad_col, float* lambda_out,
                              void* stream);

/* gptq_prepare_hinv without any host synchronisation: the same U, enqueued on ``stream``
 * and returned at once, so that a whole layer (stages 1-3) can be enqueued without a
 * round trip to the host.  lambda_dev (device float, or NULL) receives lambda on the
 * stream.  A non-positive pivot, a non-finite value or a zero Hessian is reported by the
 * next gptq_sync_status() (GPTQ_ERR_NOT_PD / NONFINITE / INVALID_ARG, with the column
 * in gptq_last_error()); until then U is undefined.  Arguments as gptq_prepare_hinv. */
gptq_status gptq_prepare_hinv_async(const float* H, int64_t d_in, float damp_rel, float* U,
                                    void* ws, size_t ws_bytes, float* lambda_dev, void* stream);

/* ------------------------------------------------------------------ stage 3
 * GPTQ column loop (tutorial "阶段二", "阶段三"; group-size article).
 *   W        device, d_out x d_in fp32 row-major; consumed as scratch (holds the
 *            compensated weights on return).
 *   U        device, output of gptq_prepare_hinv.
 *   qweight  device int32 [ceil(d_in*bits/32), d_out]: column o holds row o's codes as a
 *            little-endian bits-wide stream along d_in (code j at bits j*bits..).
 *   scales   device fp16 bit patterns [n_groups, d_out], n_groups = ceil(d_in/g) (1 for g=-1).
 *   qzeros   device int32 [n_groups, ceil(d_out*bits/32)], zero points packed along d_out
 *            the same way; must be NULL when cfg->sym != 0.
 *   err_sq   device fp32 [d_out] or NULL: per row sum_c e_c^2 with e_c = (w_c - w_hat_c)/U_cc,
 *            which equals (W0 - W_hat) Hd (W0 - W_hat)^T of that row.
 *   ws       device workspace of at least gptq_quantize_workspace_bytes(d_out, d_in, cfg) bytes.
 * Per group: scale = fp16(range/maxq) from the current compensated weights at the
 * group's first column (asymmetric range includes 0); zero = clamp(rint(-xmin/s));
 * code = clamp(rint(w/s) + zero, 0, maxq), ties to even.
 * Requires d_in % 8 == 0, 1 <= d_out. */
size_t gptq_quantize_workspace_bytes(int64_t d_out, int64_t d_in, const gptq_config* cfg);
gptq_status gptq_quantize_layer(float* W, const float* U, int64_t d_out, int64_t d_in,
                                const gptq_config* cfg, int32_t* qweight, uint16_t* scales,
                                int32_t* qzeros, float* err_sq, void* ws, size_t ws_bytes,
                                void* stream);

/* ------------------------------------------------------------------ packing, dequantization
 * gptq_pack_int: pack bits-wide codes (uint8, values < 2^bits) of each row into a
 * little-endian bit stream of int32 words, nwords = ceil(cols*bits/32).
 *   layout 0: packed[r * nwords + k]   (qzeros layout)
 *   layout 1: packed[k * rows + r]     (qweight layout)
 * Values >= 2^bits are masked to their low bits. */
gptq_status gptq_pack_int(const uint8_t* codes, int64_t rows, int64_t cols, int bits,
                          int layout, int32_t* packed, void* stream);

/* W_hat[o, c] = scale[g(c), o] * (q[o, c] - zero[g(c), o])   (tutorial "阶段三";
 * group-size article).  Same array layouts as gptq_quantize_layer; qzeros NULL iff sym. */
gptq_status gptq_dequant(const int32_t* qweight, const uint16_t* scales, const int32_t* qzeros,
                         int64_t d_out, int64_t d_in, const gptq_config* cfg, float* W_hat,
                         void* stream);

/* ------------------------------------------------------------------ activation ordering
 * (tutorial "激活排序（desc_act）": columns ranked by the sum of absolute input
 * activations; groups are formed in that order and a per-column group index maps each
 * column back to its group).
 *
 * gptq_act_sum_accumulate: act[c] (+)= sum_t |X[t, c]|, accumulated in fp64 in a fixed
 * order (the same bits on every run).  X as in gptq_hessian_accumulate (16-byte aligned,
 * d_in % 8 == 0); act device fp64 [d_in], 8-byte aligned; accumulate 0 overwrites.  A
 * non-finite sum is reported by the next gptq_sync_status() (GPTQ_ERR_NONFINITE). */
gptq_status gptq_act_sum_accumulate(const void* X, gptq_dtype xt, int64_t n, int64_t d_in, double* act,
                                    int accumulate, void* stream);

/* gptq_act_order: the quantization order of the columns.
 *   perm  device int32 [d_in]: perm[k] = the column quantized at position k.
 *   rank  device int32 [d_in]: its inverse, rank[perm[k]] = k.
 *   desc_act 1: act ascending; 2: act descending.  Equal values (+0 and -0 are equal) keep
 *   increasing column index in both directions; NaN sorts by its bit pattern.
 * Always writes a valid permutation.  1 <= d_in <= 65536. */
gptq_status gptq_act_order(const double* act, int64_t d_in, int desc_act, int32_t* perm, int32_t* rank,
                           void* stream);

/* gptq_prepare_hinv_permuted: gptq_prepare_hinv of the permuted Hessian
 * Hp[i][j] = H[perm[i]][perm[j]], i.e. U with U^T U = (Hp + lambda I)^-1.  lambda is that of
 * H (the diagonal is only reordered).  H must hold both triangles (gptq_hessian_accumulate
 * writes both); perm is a device int32 permutation of 0..d_in-1.  bad_col is a position
 * in quantization order.  An entry of perm outside [0, d_in) or a repeated entry returns
 * GPTQ_ERR_INVALID_ARG (index = its position) and U is then undefined.  Workspace as
 * gptq_prepare_hinv_workspace_bytes(d_in). */
gptq_status gptq_prepare_hinv_permuted(const float* H, const int32_t* perm, int64_t d_in, float damp_rel, float* U,
                                       void* ws, size_t ws_bytes, int64_t* bad_col, float* lambda_out, void* stream);
/* The same without host synchronisation (see gptq_prepare_hinv_async); an invalid perm is
 * reported by the next gptq_sync_status(). */
gptq_status gptq_prepare_hinv_permuted_async(const float* H, const int32_t* perm, int64_t d_in, float damp_rel,
                                             float* U, void* ws, size_t ws_bytes, float* lambda_dev, void* stream);

/* gptq_quantize_layer_act_order: the column loop of gptq_quantize_layer on the columns in
 * the order perm; cfg->desc_act must be 1 or 2 (the order itself is the one in perm).
 *   W        device fp32 [d_out, d_in] in the original column order; read only.
 *   U        output of gptq_prepare_hinv_permuted with the same perm.
 *   qweight  as gptq_quantize_layer, codes in the ORIGINAL column order.
 *   scales, qzeros  as gptq_quantize_layer; group k holds the columns perm[k*g .. k*g+g-1].
 *   g_idx    device int32 [d_in]: g_idx[c] = rank of c / g (0 for group_size -1).
 *   err_sq   as gptq_quantize_layer (the row's quadratic form does not depend on the order).
 *   ws       at least gptq_quantize_workspace_bytes(d_out, d_in, cfg) bytes with cfg->desc_act
 *            set (the plain loop's workspace plus a permuted copy of W and of the codes).
 * An invalid perm is reported by the next gptq_sync_status() (GPTQ_ERR_INVALID_ARG). */
gptq_status gptq_quantize_layer_act_order(const float* W, const float* U, const int32_t* perm, int64_t d_out,
                                          int64_t d_in, const gptq_config* cfg, int32_t* qweight, uint16_t* scales,
                                          int32_t* qzeros, int32_t* g_idx, float* err_sq, void* ws, size_t ws_bytes,
                                          void* stream);

/* W_hat[o, c] = scale[g_idx[c], o] * (q[o, c] - zero[g_idx[c], o]); arrays as gptq_dequant.
 * A g_idx entry outside [0, n_groups) is reported by the next gptq_sync_status(). */
gptq_status gptq_dequant_g_idx(const int32_t* qweight, const uint16_t* scales, const int32_t* qzeros,
                               const int32_t* g_idx, int64_t d_out, int64_t d_in, const gptq_config* cfg,
                               float* W_hat, void* stream);

/* ------------------------------------------------------------------ dequantizing GEMM
 * Y[m, n] = sum_k X[m, k] * W_hat[n, k] with W_hat[n, k] = scale[g(k), n] * (q[n, k] - zero[g(k), n])
 * (tutorial "阶段三": the integer times its scale; group-size article: groups along d_in),
 * straight from the packed arrays of gptq_quantize_layer: the consumer of its output.
 *   X        device bf16 (raw uint16 bit patterns) [M, d_in] row-major.
 *   qweight, scales, qzeros  as written by gptq_quantize_layer (qzeros NULL iff sym).
 *   Y        device fp32 [M, d_out] row-major, written in full.
 * Each group's partial product X (q - z)^T is formed on the tensor cores from exact
 * products (q - z is exact in bf16) with fp32 accumulation, then scaled by the group's
 * fp16 scales once per tile and summed in fp32; no rounded copy of W_hat is made.
 * Requires bits 2, 4 or 8 and group_size -1 or a multiple of 64 dividing d_in
 * (GPTQ_ERR_UNSUPPORTED otherwise, also for desc_act != 0), d_in % 64 == 0,
 * d_out % 8 == 0, all pointers 16-byte aligned. */
gptq_status gptq_dequant_gemm(const void* X, int64_t M, const int32_t* qweight, const uint16_t* scales,
                              const int32_t* qzeros, int64_t d_out, int64_t d_in, const gptq_config* cfg, float* Y,
                              void* stream);

/* ------------------------------------------------------------------ layer output error
 * E = ||(W - W_hat) X^T||_F^2 (tutorial "阶段一": the squared error of the layer's outputs
 * over the calibration tokens, which GPTQ minimises), and its per-row parts
 * E_o = sum_t ((W - W_hat) X^T)[o, t]^2.
 *   W        device fp32 [d_out, d_in] row-major: the weights before quantization (the
 *            natural-order gptq_quantize_layer overwrites its W, so pass a copy).
 *   W_hat    device fp32 [d_out, d_in] row-major, e.g. from gptq_dequant.
 *   X        device [n, d_in] row-major, bf16 (raw uint16 bit patterns) or fp32.
 *   row_loss device fp64 [d_out] or NULL; receives E_o.
 *   loss     device fp64 [1]; receives E.
 *   ws       device workspace of at least gptq_layer_loss_workspace_bytes(d_out, d_in, n).
 * W - W_hat and X are split into bf16 pairs (16 significant bits; a bf16 X is exact), the
 * product runs on the tensor cores as three bf16 products with fp32 accumulation in
 * segments, and the squares are summed in fp64 in a fixed order (same bits every run).
 * Relative error of E is about 1e-5 (the split and the fp32 accumulation).
 * Requires 1 <= d_out, n <= 2^30, d_in % 8 == 0 with 8 <= d_in <= 65536, all pointers
 * 16-byte aligned (row_loss and loss 8-byte). Nothing is allocated. */
size_t gptq_layer_loss_workspace_bytes(int64_t d_out, int64_t d_in, int64_t n);
gptq_status gptq_layer_loss(const float* W, const float* W_hat, const void* X, gptq_dtype xt, int64_t d_out,
                            int64_t d_in, int64_t n, double* row_loss, double* loss, void* ws, size_t ws_bytes,
                            void* stream);

/* ------------------------------------------------------------------ two-sided rounding
 * GPTQ-2D (GPTQ-2D summary, "方法" steps 1-3 and "核心洞察"): round a real matrix X
 * (m x n) to an integer matrix Z minimising tr((X - Z)^T G_left (X - Z) G_right), given the
 * upper Cholesky factors U_left of G_left^-1 (m x m) and U_right of G_right^-1 (n x n)
 * (for example from gptq_prepare_hinv with damp_rel = 0, or any other source).  The
 * entries are taken anti-diagonal by anti-diagonal (i + j = 0, 1, ...); the entries of one
 * anti-diagonal depend only on earlier ones and are rounded in parallel; each error is
 * pushed forward through both factors.  The integers equal those of one-sided GPTQ run
 * over the column-major vectorisation with the Kronecker Gram G_right (x) G_left.
 *   X        device fp64, batch problems of m x n row-major, problem b at X + b m n.
 *   U_left, U_right  device fp64 row-major, upper triangular, shared by the batch.
 *   Z        device int32, same layout as X; round half to even, no clamp.
 *   ws       device workspace of at least gptq_2d_workspace_bytes(m, n, batch) bytes.
 * All arithmetic in fp64.  A non-finite value or |Z| >= 2^31 is reported by the next
 * gptq_sync_status() (GPTQ_ERR_NONFINITE) and that entry is written as 0.
 * Requires 1 <= m, n <= 16384; 8-byte aligned X, U_left, U_right, ws; 4-byte aligned Z. */
size_t gptq_2d_workspace_bytes(int64_t m, int64_t n, int64_t batch);
gptq_status gptq_2d_round(const double* X, int64_t m, int64_t n, int64_t batch, const double* U_left,
                          const double* U_right, int32_t* Z, void* ws, size_t ws_bytes, void* stream);

/* Synchronise ``stream`` and return (and clear) the device status word. */
gptq_status gptq_sync_status(void* stream);

/* ------------------------------------------------------------------ diagnostics
 * gptq_timing_enable(1): every kernel launch of the library is bracketed by CUDA
 * events on its stream.  gptq_timing_report() synchronises the device, writes a JSON
 * object {"kernel_name": [launches, total_ms], ...} of everything recorded since the
 * last report into buf (NUL-terminated, truncated to len), clears the totals and
 * returns the number of bytes needed; with buf == NULL it only returns that size.  Host-side bookkeeping only; not thread-safe.
 *
 * gptq_selftest_bounded_wait: launches one thread that waits on a barrier nobody
 * arrives at, with a limit of limit_ns nanoseconds, the same bounded wait every
 * pipeline in the library uses; the next gptq_sync_status() returns GPTQ_ERR_TIMEOUT.
 * Used to test the timeout path without faulting or hanging the device.
 *
 * gptq_timing_timeline: the same recorded launches as a JSON list
 * [["kernel_name", stream_index, start_ms, end_ms], ...] in launch order, times from the
 * first recorded launch; start is when the launch's stream reached it (the previous work
 * in that stream done), end when it finished.  Collects, clears and sizes like
 * gptq_timing_report. */
void gptq_timing_enable(int on);
size_t gptq_timing_report(char* buf, size_t len);
size_t gptq_timing_timeline(char* buf, size_t len);
/* gptq_chol_schedule: the order in which the factorization kernel behind
 * gptq_prepare_hinv hands out its 128 x 128 tile products, for a d_in with T = ceil(d_in / 128)
 * tiles per side (host-side; no device work).  Writes up to max_tasks entries of four int32
 * (type, a, b, c) to tasks (may be NULL) and returns the total number of products:
 *   type 0  PANEL(j = b, i = a):     R_ij = A_ij R_jj^-T
 *   type 1  UPDATE(j = c, i = a, k = b): A_ik -= R_ij R_kj^T
 *   type 2  FIN(i = a, m = b):       U_im = -R_ii^-1 S_im
 *   type 3  SUPD(i = a, k = c, m = b):  S_im += R_ik U_km
 *   type 4  DIAG(j = a):             U_jj = R_jj^-1 to U and to the split of U^T (a copy)
 * with Hd = R R^T (R upper), U = R^-1.  The diagonal blocks (R_jj and R_jj^-1 from A_jj) are
 * formed in the order j = T-1 .. 0 by one CTA, which also forms, right after LEAF(j), the two
 * products the next leaf needs: PANEL(j, j-1) and UPDATE(j, j-1, j-1) (not in the list).
 * Every product's inputs come from products earlier in the list or from a leaf step before
 * its own step; returns -1 for T < 1. */
int64_t gptq_chol_schedule(int64_t T, int32_t* tasks, int64_t max_tasks);
gptq_status gptq_selftest_bounded_wait(uint64_t limit_ns, void* stream);

/* ------------------------------------------------------------------ no-allocation variant
 * gptq_hessian_accumulate_fixed_scratch: the same H (+)= 2 X^T X as
 * gptq_hessian_accumulate (the same kernels and the same segmented accumulation, so the
 * same bits for the same X), for callers that cannot hand the library a device
 * workspace: a plain C program that links only this library and has no device
 * allocator of its own, or a plug-in running inside a host application whose memory
 * pool owns the whole device and forbids further cudaMalloc calls.  The pages have no
 * counterpart to this entry point; it exists for those callers only.
 *   - Scratch: a fixed 16 MiB array inside the library (16777216 bytes per GPU),
 *     reserved on every GPU that loads the library until the process exits.  A batch
 *     needs d_in * roundup(n, 64) * 2 bytes for bf16 X, or d_in * roundup(n, 64) * 8
 *     bytes for fp32 X (two tf32 parts); a larger batch returns GPTQ_ERR_INVALID_ARG
 *     with both sizes in gptq_last_error().  Split such a batch and call with
 *     accumulate = 1.
 *   - The first call on each device looks up the array's device address (a set-up the
 *     library does once per device, and again if the device's context was destroyed and
 *     created anew); make that first call before capturing any stream.
 *   - All calls on one device share its array, which keeps the last call's contents.
 *     Calls on one device that may overlap on the GPU (for example on two streams) race
 *     and must be serialised by the caller.  Each call rewrites all of the scratch it
 *     reads, so nothing needs clearing.
 *   - Allocates no device or host memory; arguments as gptq_hessian_accumulate. */
gptq_status gptq_hessian_accumulate_fixed_scratch(const void* X, gptq_dtype xt, int64_t n, int64_t d_in,
                                                  float* H, int accumulate, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* GPTQ_B200_H */
