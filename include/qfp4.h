/*
 * qfp4.h - C ABI of the B200 (sm_100a) FP4 quantized linear layer.
 *
 * What it computes (the pages are web articles on FP4 training; none prints
 * code):
 *  - Micro-scaled FP4 quantization of a bf16 tensor: E2M1 elements with one
 *    E8M0 shared exponent per 32 elements (MXFP4; page "New AMD paper
 *    overturns conventional wisdom: FP4 training...", section "Chto takoe
 *    MXFP4") or one E4M3 scale per 16 elements plus an fp32 tensor scale
 *    (NVFP4; page "Quartet II - obuchenie v NVFP4 s tochnymi nesmeshchyonnymi
 *    gradientami": NVFP4 uses more precise FP8 scales).
 *  - An optional block Hadamard rotation before quantization, deterministic or
 *    with random signs, 16x16 or 32x32 (page "NVIDIA sozdala metod obucheniya
 *    neyrosetey v 4-bit tochnosti", section "Kak eto rabotaet"; AMD page,
 *    section "Poiskovaya eksperimental'naya rabota").
 *  - Three rounding modes: round-to-nearest (AMD page, "Chto takoe MXFP4"),
 *    per-element stochastic rounding (all three pages), and Quartet II, which
 *    keeps round-to-nearest codes and stochastically rounds the per-block
 *    renormalisation <u,u>/<u,q> (about 0.94-1.06) into the scale (Quartet II
 *    page).
 *  - Block-scaled FP4 GEMMs D = A . B^T, and the linear layer's three GEMMs
 *    Fprop Y = X W^T, Dgrad dX = dY W, Wgrad dW = dY^T X (AMD page,
 *    "Poiskovaya eksperimental'naya rabota").
 *
 * Conventions for every call:
 *  - Pointers are DEVICE pointers unless stated otherwise; structs and
 *    recipes are passed by HOST pointer. The library never allocates device
 *    memory: the caller owns every buffer and the workspace.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls are
 *    asynchronous on it; the return value reports argument validation and
 *    launch errors only. Device-side errors (a bounded wait that timed out)
 *    are reported by qfp4_status().
 *  - Errors are negative status codes; nothing aborts, traps or prints.
 *  - Matrices are row-major. "rows x k" is the quantized orientation: k is the
 *    axis the blocks run along, which is the reduction axis of the GEMM.
 *  - Kernels are launched with programmatic dependent launch (each waits for
 *    the previous grid on the stream before touching memory, so stream order
 *    holds as usual). Environment switches, read on every call, select
 *    equivalent paths with the same results: QFP4_PDL=0 (plain launches),
 *    QFP4_FUSED_AMAX=1 (one-launch amax + quantization of an NVFP4 tensor
 *    that fits in L2, a cooperative launch; off by default), QFP4_COL_BANDS=0
 *    (group-walking column quantizer), QFP4_GEMM_PAIR=0/1 (GEMM kernel).
 *  - Each call that touches the device opens an NVTX range named after it.
 */
#ifndef QFP4_H_
#define QFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define QFP4_OK 0
#define QFP4_ERR_INVALID_ARG (-1)      /* bad enum, negative or unsupported size, format mismatch */
#define QFP4_ERR_MISALIGNED (-2)       /* a pointer or row stride breaks the stated alignment */
#define QFP4_ERR_UNSUPPORTED_ARCH (-3) /* the current device is not sm_100 */
#define QFP4_ERR_WORKSPACE (-4)        /* workspace missing or smaller than required */
#define QFP4_ERR_CUDA (-5)             /* a CUDA runtime/driver call failed; see qfp4_last_cuda_error */
#define QFP4_ERR_TIMEOUT (-6)          /* a device-side bounded wait expired (from qfp4_status) */
#define QFP4_ERR_TOO_LARGE (-7)        /* the problem needs more than qfp4_linear_fwd_noalloc's fixed scratch */
#define QFP4_ERR_BOUNDS (-8)           /* bounds-checked build only: a kernel store fell outside its buffer and was
                                          dropped (from qfp4_status) */

/* ---- enums ---------------------------------------------------------------- */
/* QFP4_MXFP4_RU: MXFP4 whose shared exponent is rounded up instead of down,
 * E = the smallest exponent with amax_b <= 6 * 2^E, so that no element of a
 * block clips (a reading the AMD MXFP4 page, "Chto takoe MXFP4", leaves open:
 * it gives the shared exponent only as the block's largest one). Accepted by
 * qfp4_quantize and in recipes; the tensor it writes is an ordinary MXFP4
 * tensor (fmt = QFP4_MXFP4), since only the choice of E differs. */
typedef enum { QFP4_NVFP4 = 0, QFP4_MXFP4 = 1, QFP4_MXFP4_RU = 2 } qfp4_format;
typedef enum { QFP4_RTN = 0, QFP4_SR = 1, QFP4_QUARTET2 = 2 } qfp4_rounding;
typedef enum {
    QFP4_HAD_NONE = 0,
    QFP4_HAD_DET16 = 1,  /* deterministic 16x16 Hadamard (D = I) */
    QFP4_HAD_DET32 = 2,  /* deterministic 32x32 Hadamard */
    QFP4_HAD_RAND16 = 3, /* 16x16 Hadamard with a random sign vector */
    QFP4_HAD_RAND32 = 4  /* 32x32 Hadamard with a random sign vector */
} qfp4_hadamard;
typedef enum { QFP4_AXIS_ROW = 0, QFP4_AXIS_COL = 1 } qfp4_axis;
typedef enum { QFP4_OUT_BF16 = 0, QFP4_OUT_F32 = 1 } qfp4_dtype;
typedef enum { QFP4_PRESET_NVIDIA_NVFP4 = 0, QFP4_PRESET_QUARTET2_NVFP4 = 1, QFP4_PRESET_AMD_MXFP4_H = 2 } qfp4_preset;

/* ---- randomness -------------------------------------------------------------
 * Every random bit is Philox4x32-10 (Salmon et al., SC'11) with key = a 64-bit
 * seed and counter = (i/4 low 32 bits, i/4 high 32 bits, tag | stream << 4, 0);
 * item i uses word i mod 4, and a uniform is (word >> 8) * 2^-24.
 *   tag 0: element stochastic rounding, i = row * k + j in the quantized
 *          orientation, key = sr;
 *   tag 1: Quartet II scale rounding, i = row * (k / block) + block index, key = sr;
 *   tag 2: the random Hadamard sign vector, i = 0, key = rot; bit b of the
 *          word set flips position b of every Hadamard chunk.
 * Reading: the pages name stochastic rounding and random sign flips but no
 * generator; this layout makes every bit reproducible from (seed, position). */
typedef struct {
    uint64_t rot;        /* key of the sign vector */
    uint64_t sr;         /* key of the rounding uniforms */
    uint32_t rot_stream; /* stream id of the sign vector (< 2^28) */
    uint32_t sr_stream;  /* stream id of the rounding uniforms (< 2^28) */
} qfp4_seed;

/* ---- quantized tensor -----------------------------------------------------
 * codes:  rows * k / 2 bytes, row-major [rows][k/2]; element j of a row is the
 *         low nibble of byte j/2 when j is even, the high nibble when odd. A
 *         nibble is sign << 3 | index into {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 *         16-byte aligned.
 * scales: qfp4_scales_bytes(fmt, rows, k) bytes, 16-byte aligned, in the
 *         tcgen05 block-scale layout: 512-byte atoms of 128 rows x 4 scale
 *         columns (byte (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4 of atom
 *         (r / 128) * ceil(k / block / 4) + c / 4); rows and scale columns
 *         are padded to the atom with zero scales. E4M3 codes (NVFP4) or E8M0
 *         codes (MXFP4). qfp4_scale_offset() gives the byte of (r, c).
 * tensor_scale: one fp32, the NVFP4 decode multiplier g (1.0 for MXFP4).
 * An element decodes as e2m1(code) * scale(row, j / block) * g, in the rotated
 * domain when a Hadamard was applied.
 * The caller sets codes, scales and tensor_scale; qfp4_quantize fills the rest. */
typedef struct {
    uint8_t* codes;
    uint8_t* scales;
    float* tensor_scale;
    int64_t rows;
    int64_t k;
    int32_t fmt;         /* qfp4_format */
    int32_t had;         /* qfp4_hadamard applied along k */
    uint64_t rot_seed;   /* sign-vector key (random Hadamard only) */
    uint32_t rot_stream; /* sign-vector stream (random Hadamard only) */
    uint32_t reserved;
} qfp4_tensor;

/* ---- linear-layer recipe ------------------------------------------------- */
typedef struct {
    int32_t fmt;   /* qfp4_format of both operands */
    int32_t rnd_a; /* qfp4_rounding of operand A (the left factor) */
    int32_t rnd_b; /* qfp4_rounding of operand B */
    int32_t had;   /* qfp4_hadamard along the GEMM's reduction axis, both operands */
} qfp4_gemm_cfg;

typedef struct {
    qfp4_gemm_cfg fprop; /* Y  = X W^T:  A = X  (along K),  B = W (along K) */
    qfp4_gemm_cfg dgrad; /* dX = dY W:   A = dY (along N),  B = W (along N) */
    qfp4_gemm_cfg wgrad; /* dW = dY^T X: A = dY (along M),  B = X (along M) */
    int32_t y_dtype, dx_dtype, dw_dtype; /* qfp4_dtype of the three outputs */
    int32_t dw_accumulate; /* 1: dW += dY^T X (fp32 dW only, e.g. a main-grad buffer), 0: dW = dY^T X */
} qfp4_recipe;

/* ---- errors -------------------------------------------------------------- */
/* Static string for a status code. */
const char* qfp4_strerror(int status);
/* The cudaError_t behind the calling thread's last QFP4_ERR_CUDA. */
int qfp4_last_cuda_error(void);

/* ---- sizes and layouts (host-only, no device access) ---------------------- */
/* Bytes of the codes of a rows x k tensor: rows * k / 2. */
size_t qfp4_codes_bytes(int64_t rows, int64_t k);
/* Bytes of the scale buffer: ceil(rows/128) * ceil(k/block/4) * 512. Returns 0 for a bad format. */
size_t qfp4_scales_bytes(int32_t fmt, int64_t rows, int64_t k);
/* Byte offset of the scale of (row r, scale column c) in the scale buffer,
 * or -1 when out of range. */
int64_t qfp4_scale_offset(int32_t fmt, int64_t rows, int64_t k, int64_t r, int64_t c);
/* Workspace bytes qfp4_quantize / qfp4_amax need (fixed: 4096; 0 would do for
 * MXFP4 or when the caller passes the amax). 16-byte aligned. */
size_t qfp4_quantize_workspace_bytes(void);

/* ---- quantization ----------------------------------------------------------
 * qfp4_amax: the NVFP4 tensor amax, max |v| over the rotated tensor v in the
 * given orientation (v = x when had is NONE), written to *amax (device fp32).
 *
 * qfp4_quantize: quantize x (bf16, R x C, row stride ld elements).
 *   axis ROW: blocks run along C; the result is rows = R, k = C.
 *   axis COL: blocks run along R; the result is the quantized transpose,
 *             rows = C, k = R (the Wgrad operand: quantized along tokens).
 * Steps per rows-x-k segment (k the quantized axis):
 *   1. rotate (had != NONE): per n_h chunk v = fp32(1/sqrt(n_h)) * H (D x),
 *      H the Sylvester matrix, D the sign vector (I for deterministic), the
 *      butterflies in ascending half-width order, in fp32;
 *   2. NVFP4: amax over v (or *amax_in when amax_in != NULL), s_enc = 2688 /
 *      amax, g = amax / 2688 (both 1 when amax = 0);
 *   3. block scale: NVFP4 S = E4M3_RN_sat(fp32(amax_b / 6) * s_enc),
 *      r = s_enc / S (0 when S = 0); MXFP4 E = floor(log2 amax_b) - 2 (plus
 *      one for QFP4_MXFP4_RU when amax_b > 6 * 2^E) clamped to [-127, 127],
 *      code E + 127, r = 2^-E (code 0, r = 0 for a zero block);
 *   4. u = v * r; codes by RTN (ties to even, saturating at 6, -0 -> +0), SR
 *      (round up iff uniform < (|u| - lo) / gap), or Quartet II: RTN codes,
 *      then alpha = T(u*u) / T(u*q) (T the halving-stride tree sum over the
 *      block, 1 when the denominator is 0) and the scale becomes SR(S * alpha)
 *      on the E4M3 (saturating at 448) or E8M0 grid.
 * Requirements: R, C >= 0; k a multiple of the block (16 NVFP4, 32 MXFP4) and
 *   of n_h; ld >= C and ld % 8 == 0; x, codes and scales 16-byte aligned;
 *   for NVFP4 without amax_in, workspace >= qfp4_quantize_workspace_bytes(),
 *   16-byte aligned (its contents on entry do not matter). The result depends
 *   only on the inputs and seeds, never on the launch configuration.
 * Kernels: persistent, TMA-fed; along COL with k a multiple of 64 a thread
 *   takes 64 consecutive rows of one column (64-row bands), otherwise one
 *   group of rows; QFP4_COL_BANDS=0 in the environment selects the latter
 *   (same results; read on every call).
 * out: caller sets codes, scales and tensor_scale; the call sets the rest. */
int qfp4_amax(const void* x, int64_t R, int64_t C, int64_t ld, int32_t had, int32_t axis, const qfp4_seed* seed,
              float* amax, void* workspace, size_t workspace_bytes, void* stream);
/* qfp4_amax_rowcol: both orientations' tensor amax of x (bf16, R x C), as
 * qfp4_amax computes them: *amax_row with axis ROW, had_row and seed_row's
 * sign vector, *amax_col with axis COL, had_col and seed_col's (device fp32
 * each; the two GEMMs that use x along both axes rotate with different sign
 * vectors, and may use a deterministic Hadamard on one axis and a random one
 * on the other). Hadamards of one size <= 16 (or none on both axes) take one
 * read of x; size 32 or two different sizes take one read per axis.
 * Requirements: those of qfp4_amax for both axes (R a multiple of had_col's
 * size, C of had_row's); workspace >= qfp4_quantize_workspace_bytes(),
 * 16-byte aligned.
 * This is the fused tensor-scale pass of the backward linear layer (dY is
 * quantized along N for Dgrad and along the tokens for Wgrad; pages: "New AMD
 * paper overturns conventional wisdom: FP4 training...", section
 * "Poiskovaya eksperimental'naya rabota", the three GEMMs of the layer), and
 * lets the forward take the backward's amaxes of X and W in its own read. */
int qfp4_amax_rowcol(const void* x, int64_t R, int64_t C, int64_t ld, int32_t had_row, int32_t had_col,
                     const qfp4_seed* seed_row, const qfp4_seed* seed_col, float* amax_row, float* amax_col,
                     void* workspace, size_t workspace_bytes, void* stream);

int qfp4_quantize(const void* x, int64_t R, int64_t C, int64_t ld, int32_t fmt, int32_t rounding, int32_t had,
                  int32_t axis, const qfp4_seed* seed, const float* amax_in, qfp4_tensor* out, void* workspace,
                  size_t workspace_bytes, void* stream);
/* qfp4_quantize_dual: both orientations of x from one read of it — exactly
 * what qfp4_quantize gives with axis ROW (had_row, seed_row, *amax_row) into
 * out_row and with axis COL (had_col, seed_col, *amax_col) into out_col, same
 * format and rounding. It serves the backward linear layer, where dY is
 * quantized along N for Dgrad and along the tokens for Wgrad (pages: "New AMD
 * paper overturns conventional wisdom: FP4 training...", section
 * "Poiskovaya eksperimental'naya rabota", the three GEMMs of the layer).
 * Requirements: those of qfp4_quantize for both axes; R a multiple of 64,
 * R and C > 0; had_row none or of had_col's size (16 or 32); for NVFP4,
 * amax_row and amax_col are the two tensor amaxes (device fp32, e.g. from
 * qfp4_amax_rowcol or qfp4_amax), required; ignored for MXFP4. No workspace.
 * Unsupported combinations return QFP4_ERR_INVALID_ARG. */
int qfp4_quantize_dual(const void* x, int64_t R, int64_t C, int64_t ld, int32_t fmt, int32_t rounding,
                       int32_t had_row, int32_t had_col, const qfp4_seed* seed_row, const qfp4_seed* seed_col,
                       const float* amax_row, const float* amax_col, qfp4_tensor* out_row, qfp4_tensor* out_col,
                       void* stream);

/* ---- GEMM -------------------------------------------------------------------
 * The three products of a linear layer trained in FP4 (page "New AMD paper
 * overturns conventional wisdom: FP4 training...", section "Poiskovaya
 * eksperimental'naya rabota": Fprop Y = X W^T, Dgrad dX = dY W, Wgrad
 * dW = dY^T X, each with both operands quantized) are all of this form, with
 * the operands quantized along their reduction axis by qfp4_quantize:
 * D[i][j] = gA * gB * sum_k A(i,k) B(j,k) over the decoded FP4 operands, fp32
 * accumulation on the tcgen05 tensor cores, D = A . B^T of shape
 * A.rows x B.rows, written as bf16 or fp32 with row stride ldd elements.
 * Requirements: same format, same k (a multiple of 64), same Hadamard (and for
 * a random one, the same rot_seed and rot_stream, so the rotation cancels);
 * D 16-byte aligned and ldd * element size a multiple of 16; ldd >= B.rows.
 * Kernel: persistent CTA pairs on 256 x 256 tiles (tcgen05 cta_group::2) when
 * A has more than 128 rows, else single CTAs on 128 x 256 tiles; the
 * environment variable QFP4_GEMM_PAIR=1 or =0 forces the pair or the single
 * kernel (same results within the bound). */
int qfp4_gemm(const qfp4_tensor* A, const qfp4_tensor* B, void* D, int64_t ldd, int32_t out_dtype, void* stream);
/* qfp4_gemm_accumulate: D[i][j] += gA * gB * sum_k A(i,k) B(j,k) into an fp32
 * D (beta = 1: the Wgrad accumulation into an fp32 main gradient across
 * micro-batches). The product is formed exactly as by qfp4_gemm with an fp32
 * output, then added to D with one fp32 add (round to nearest) per element;
 * the pair kernel adds through TMA reduce-add stores, the single-CTA kernel
 * by a read-modify-write of the element it owns. D must not be written by
 * anything else until the call completes. Requirements as qfp4_gemm. */
int qfp4_gemm_accumulate(const qfp4_tensor* A, const qfp4_tensor* B, float* D, int64_t ldd, void* stream);
/* qfp4_gemm_quantize: D = A . B^T as qfp4_gemm with a bf16 output, and *out =
 * that bf16 D quantized to MXFP4 along its rows (k = B.rows), round to
 * nearest, with Hadamard `had` and seed->rot / rot_stream for a random one —
 * exactly what qfp4_quantize(D, MXFP4, RTN, had, ROW, seed) gives — so a
 * layer's output is also the next layer's forward operand. With the CTA-pair
 * kernel (A.rows > 128) the quantization happens in the GEMM's epilogue from
 * the values it stores; otherwise D is quantized by a second launch.
 * Requirements: those of qfp4_gemm; B.rows a multiple of 32; out's codes
 * (A.rows x B.rows/2 bytes) and scales (qfp4_scales_bytes(MXFP4, A.rows,
 * B.rows)) 16-byte aligned, and its tensor_scale (set to 1). No workspace. */
int qfp4_gemm_quantize(const qfp4_tensor* A, const qfp4_tensor* B, void* D, int64_t ldd, int32_t had,
                       const qfp4_seed* seed, qfp4_tensor* out, void* stream);
/* qfp4_gemm_amax: D = A . B^T as qfp4_gemm with a bf16 output, and *amax (a
 * device fp32) = the NVFP4 tensor amax of that bf16 D along its rows after
 * the rotation `had` (seed->rot / rot_stream for a random one) — exactly what
 * qfp4_amax(D, A.rows, B.rows, ldd, had, ROW, seed, ...) gives. Passing it as
 * amax_in to qfp4_quantize(D, NVFP4, ..., had, ROW, seed) quantizes a layer's
 * output for the next layer without the separate read of D that the tensor
 * scale otherwise needs (NVFP4's FP32 tensor scale must be known before any
 * block scale; page "Quartet II - obuchenie v NVFP4 s tochnymi
 * nesmeshchyonnymi gradientami" on NVFP4 with FP8 block scales). With the
 * CTA-pair kernel (A.rows > 128) each CTA's epilogue takes the rotated
 * maximum of the rows it stores and a one-CTA reduction combines them;
 * otherwise D is read once more by an amax pass.
 * Requirements: those of qfp4_gemm; B.rows a multiple of 16 and of the
 * Hadamard size; workspace >= qfp4_quantize_workspace_bytes(), 16-byte
 * aligned (its contents on entry do not matter). */
int qfp4_gemm_amax(const qfp4_tensor* A, const qfp4_tensor* B, void* D, int64_t ldd, int32_t had,
                   const qfp4_seed* seed, float* amax, void* workspace, size_t workspace_bytes, void* stream);

/* ---- linear layer -------------------------------------------------------------
 * One linear layer's FP4 forward (Fprop) and backward (Dgrad and Wgrad) pass:
 * six quantizations and three GEMMs (page "New AMD paper overturns
 * conventional wisdom: FP4 training...", section "Poiskovaya
 * eksperimental'naya rabota"; the recipes: QFP4_PRESET_NVIDIA_NVFP4 follows
 * "NVIDIA sozdala metod obucheniya neyrosetey v 4-bit tochnosti", section
 * "Kak eto rabotaet" (16x16 random Hadamard on the Wgrad inputs, stochastic
 * rounding of the gradient); QFP4_PRESET_QUARTET2_NVFP4 follows "Quartet II -
 * obuchenie v NVFP4 s tochnymi nesmeshchyonnymi gradientami" (random rotation
 * and the stochastically rounded scale renormalisation on the backward pass);
 * QFP4_PRESET_AMD_MXFP4_H the AMD page's MXFP4 with a deterministic Hadamard
 * on Wgrad).
 * X [M x K], W [N x K], dY [M x N] bf16 row-major (contiguous); Y [M x N],
 * dX [M x K], dW [N x K] in the recipe's output types (contiguous).
 * Seeds: the sign vector of GEMM g (0 Fprop, 1 Dgrad, 2 Wgrad) uses key
 * seed->rot and stream g, shared by both operands; operand o (0 X and 1 W of
 * Fprop, 2 dY and 3 W of Dgrad, 4 dY and 5 X of Wgrad) rounds with key
 * seed->sr and stream o (the stream fields of *seed are ignored).
 * Requirements: M, N, K multiples of 128; X, W, dY 16-byte aligned; the
 * workspace holds the quantized operands. */
int qfp4_recipe_preset(int32_t preset, qfp4_recipe* out);
size_t qfp4_linear_workspace_bytes(int32_t backward, int64_t M, int64_t N, int64_t K, const qfp4_recipe* recipe);
int qfp4_linear_fwd(const void* X, const void* W, void* Y, int64_t M, int64_t N, int64_t K, const qfp4_recipe* recipe,
                    const qfp4_seed* seed, void* workspace, size_t workspace_bytes, void* stream);
int qfp4_linear_bwd(const void* dY, const void* X, const void* W, void* dX, void* dW, int64_t M, int64_t N, int64_t K,
                    const qfp4_recipe* recipe, const qfp4_seed* seed, void* workspace, size_t workspace_bytes,
                    void* stream);
/* qfp4_linear_fwd_chain: qfp4_linear_fwd for a layer between two FP4 layers,
 * where one layer's output Y is the next layer's input X, so that NVFP4's
 * tensor scale (needed before any block scale) costs no extra read of it:
 *   x_amax (device fp32, or NULL): X's NVFP4 tensor amax for this layer's
 *     Fprop rotation, as the previous layer's call returned it in its y_amax;
 *     X's quantization then skips its amax pass (ignored unless the Fprop
 *     format is NVFP4; NULL: the pass runs as in qfp4_linear_fwd);
 *   y_amax (device fp32, or NULL): receives Y's NVFP4 tensor amax along its
 *     rows for the next layer's Fprop rotation next_had, whose sign vector
 *     is the next layer's (key next_seed->rot, stream 0, by the seed rule
 *     above), taken in the GEMM's epilogue as qfp4_gemm_amax does; needs a
 *     bf16 y_dtype and N a multiple of 16 and of the Hadamard size.
 * The result is bit for bit what qfp4_linear_fwd gives (and y_amax what
 * qfp4_amax(Y, ..., next_had, ROW, ...) gives). Workspace as qfp4_linear_fwd.
 * The pages have no such interface; it applies the tensor scale of NVFP4
 * ("Quartet II - obuchenie v NVFP4 s tochnymi nesmeshchyonnymi gradientami")
 * to a stack of linear layers. */
int qfp4_linear_fwd_chain(const void* X, const void* W, void* Y, int64_t M, int64_t N, int64_t K,
                          const qfp4_recipe* recipe, const qfp4_seed* seed, const float* x_amax, int32_t next_had,
                          const qfp4_seed* next_seed, float* y_amax, void* workspace, size_t workspace_bytes,
                          void* stream);

/* ---- forward pass without any allocation ----------------------------------
 * qfp4_linear_fwd_noalloc: the same computation as qfp4_linear_fwd, for
 * callers that cannot allocate device memory at all: code running under a
 * memory plan fixed at start-up (a serving runtime or an embedded system that
 * forbids device allocation after initialisation), a plugin inside a host
 * framework that owns the allocator and exposes no way to reach it, or a
 * latency-critical path where a cudaMalloc (which may synchronise the device)
 * is not acceptable. The caller passes only X, W and Y. The library's own
 * scratch (the quantized operands and the amax partials) lives in a fixed
 * array of QFP4_NOALLOC_SCRATCH_BYTES (32 MiB) of device memory that every GPU
 * loading the library keeps until the process exits; a layer whose
 * qfp4_linear_workspace_bytes(0, ...) exceeds it is rejected with
 * QFP4_ERR_TOO_LARGE before anything is launched. The call makes no
 * cudaMalloc / cudaFree or other allocation.
 * Set-up: the first call in a CUDA context (a device's primary context, and
 * again after cudaDeviceReset replaces it) looks up the array's device address
 * with the stream's device current, and later calls in that context reuse it;
 * make that first call before any stream capture. All calls share the one
 * array and it keeps the last
 * call's contents; every byte a call reads there it has written first, so
 * nothing needs clearing, but calls that overlap on the GPU (on different
 * streams, or from different threads) race on it: serialise them.
 * The pages have no counterpart to this entry point; it is part of the
 * library's interface only. */
#define QFP4_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
int qfp4_linear_fwd_noalloc(const void* X, const void* W, void* Y, int64_t M, int64_t N, int64_t K,
                            const qfp4_recipe* recipe, const qfp4_seed* seed, void* stream);

/* ---- status ---------------------------------------------------------------
 * Synchronizes `stream`, then reads and clears the library's device error word
 * on the current device. Returns QFP4_OK, QFP4_ERR_TIMEOUT (a bounded wait in
 * a kernel expired; that kernel skipped the rest of its work), QFP4_ERR_BOUNDS
 * (only from the bounds-checked build, libqfp4_bc.so, compiled with
 * QFP4_BOUNDS_CHECK: a kernel computed a store address outside the output
 * buffer the arguments describe; the store went to a scratch sink instead), or
 * QFP4_ERR_CUDA. */
int qfp4_status(void* stream);

/* Number of kernels the library launched on the calling thread since the last
 * reset (reset = 1 zeroes it after reading). */
int64_t qfp4_launch_count(int32_t reset);

/* Self-test of the failure-detection path (no counterpart on the pages):
 * launches one small kernel whose shared-memory mbarrier wait nothing
 * satisfies, waited on with the same bounded wait as the library's kernels
 * but with limit_ns (0 < limit_ns <= 2 s) instead of 2 s. The wait gives up,
 * sets the device error word and the kernel returns: the next qfp4_status on
 * the stream returns QFP4_ERR_TIMEOUT and clears the word, and the context
 * stays usable. Nothing faults, traps or spins without a limit.
 * Returns QFP4_OK (launched), QFP4_ERR_INVALID_ARG or QFP4_ERR_CUDA. */
int qfp4_selftest_wait_timeout(int64_t limit_ns, void* stream);

/* Self-test of the quantizers' element and scale rounding steps: applies one
 * of them, as the quantizer kernels inline it, to each of n fp32 values and
 * writes one code byte per value. Lets a test compare the exact decision of
 * the device code with the definition at chosen points (grid points, the
 * stochastic-rounding thresholds themselves and their neighbouring floats),
 * which the quantizers' own inputs reach only by chance.
 *   op QFP4_ROUND_E2M1_SR: stochastic rounding onto E2M1 with the 16-bit
 *     draw r = w[i] & 0xFFFF (round up iff r * 2^-16 < the fraction between
 *     the two grid neighbours, |x| >= 6 gives 6; [NVIDIA NVFP4] "Kak eto
 *     rabotaet", [Quartet II] on NVIDIA's recipe); |x| < 2^127.
 *   op QFP4_ROUND_E2M1_RN: round-to-nearest-even onto E2M1, saturating at 6
 *     ([AMD MXFP4] "Chto takoe MXFP4").
 *   op QFP4_ROUND_E4M3_SR: stochastic rounding of x >= 0 onto E4M3 with the
 *     uniform (w[i] >> 8) * 2^-24, saturating at 448 (the Quartet II scale
 *     step, [Quartet II]).
 *   op QFP4_ROUND_E4M3_RN: round-to-nearest-even of x >= 0 onto E4M3,
 *     saturating at 448 (the NVFP4 block scale).
 *   op QFP4_ROUND_E8M0_SR: stochastic rounding of x > 0 onto powers of two
 *     with the uniform (w[i] >> 8) * 2^-24, as the E8M0 code (the Quartet II
 *     scale step on an MXFP4 scale).
 * x: n fp32 (device), w: n uint32 (device; may be NULL for the two RN ops),
 * codes: n bytes (device, written; an E2M1 code is sign << 3 | magnitude
 * index, magnitude 0 always code 0). Values outside an op's stated domain
 * give unspecified codes. Stream-ordered. Returns QFP4_OK (launched),
 * QFP4_ERR_INVALID_ARG (unknown op, n < 0, a NULL pointer that the op reads
 * or writes) or QFP4_ERR_CUDA. */
#define QFP4_ROUND_E2M1_SR 0
#define QFP4_ROUND_E2M1_RN 1
#define QFP4_ROUND_E4M3_SR 2
#define QFP4_ROUND_E4M3_RN 3
#define QFP4_ROUND_E8M0_SR 4
int qfp4_selftest_rounding(int32_t op, const float* x, const uint32_t* w, uint8_t* codes, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* QFP4_H_ */
