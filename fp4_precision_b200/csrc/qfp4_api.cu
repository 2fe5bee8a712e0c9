// qfp4_api.cu - the extern "C" entry points of include/qfp4.h: argument
// validation, TMA descriptor encoding, launch of the quantizer and GEMM
// kernels, and the linear layer's composition of six quantizations and three
// GEMMs (page "New AMD paper overturns conventional wisdom: FP4 training...",
// section "Poiskovaya eksperimental'naya rabota": Fprop Y = X W^T, Dgrad
// dX = dY W, Wgrad dW = dY^T X).
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/qfp4.h"
#include "qfp4_internal.h"

namespace qfp4 {
namespace {

thread_local int t_last_cuda_error = 0;

// An NVTX range named after the entry point around every call that touches
// the device, so that a profiler's timeline shows which library call issued
// which launches (header-only NVTX: without an attached tool a push or pop is
// one test of a null function pointer).
struct ApiRange {
    explicit ApiRange(const char* name) { nvtxRangePushA(name); }
    ~ApiRange() { nvtxRangePop(); }
    ApiRange(const ApiRange&) = delete;
    ApiRange& operator=(const ApiRange&) = delete;
};
thread_local int64_t t_launches = 0;

int cuda_fail(cudaError_t e) {
    t_last_cuda_error = (int)e;
    return QFP4_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int block_of(int fmt) { return fmt == kNvfp4 ? 16 : 32; }
bool valid_fmt(int fmt) { return fmt == QFP4_NVFP4 || fmt == QFP4_MXFP4 || fmt == QFP4_MXFP4_RU; }
int had_n(int had) {
    return (had == QFP4_HAD_DET16 || had == QFP4_HAD_RAND16)   ? 16
           : (had == QFP4_HAD_DET32 || had == QFP4_HAD_RAND32) ? 32
                                                               : 0;
}
bool had_random(int had) { return had == QFP4_HAD_RAND16 || had == QFP4_HAD_RAND32; }

// Driver entry points are requested at a fixed ABI version (CUDA 12.0): a
// later default can resolve a name to a newer signature (cuStreamGetCtx, for
// one, gained a third argument in 12.5).
template <typename Fn>
Fn driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<Fn>(p);
    return nullptr;
}

// ---- context binding -----------------------------------------------------------
// The library carries its own (static) CUDA runtime. A caller's thread may have
// no current driver context (e.g. a framework's worker thread), and the right
// GPU is the one the caller's stream lives on, so every entry point that
// touches the device first makes the stream's context current.
using GetCtxFn = CUresult (*)(CUstream, CUcontext*);
using CurCtxFn = CUresult (*)(CUcontext*);
using SetCtxFn = CUresult (*)(CUcontext);



int bind_context(cudaStream_t stream) {
    static GetCtxFn get_stream_ctx = nullptr;
    static CurCtxFn get_cur = nullptr;
    static SetCtxFn set_cur = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        get_stream_ctx = driver_fn<GetCtxFn>("cuStreamGetCtx");
        get_cur = driver_fn<CurCtxFn>("cuCtxGetCurrent");
        set_cur = driver_fn<SetCtxFn>("cuCtxSetCurrent");
    });
    if (!get_stream_ctx || !get_cur || !set_cur) return QFP4_OK;  // nothing to adjust
    CUcontext want = nullptr, cur = nullptr;
    const uintptr_t h = reinterpret_cast<uintptr_t>(stream);
    if (h > 2 && get_stream_ctx(reinterpret_cast<CUstream>(stream), &want) != CUDA_SUCCESS) want = nullptr;
    if (get_cur(&cur) != CUDA_SUCCESS) cur = nullptr;
    if (want != nullptr && want != cur) {
        if (set_cur(want) != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidResourceHandle);
    } else if (want == nullptr && cur == nullptr) {
        // default stream and no current context: the runtime's current device
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaSetDevice(dev);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return QFP4_OK;
}

// ---- device check (sm_100), cached per device --------------------------------
int check_device(int* sm_count) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    static std::mutex mu;
    static int cached_ok[64] = {0};  // 0 unknown, 1 sm_100, -1 other
    static int cached_sms[64] = {0};
    if (dev < 0 || dev >= 64) return QFP4_ERR_UNSUPPORTED_ARCH;
    std::lock_guard<std::mutex> lock(mu);
    if (cached_ok[dev] == 0) {
        int major = 0, minor = 0, sms = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
            return cuda_fail(e);
        if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
            return cuda_fail(e);
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e);
        cached_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
        cached_sms[dev] = sms;
    }
    if (sm_count) *sm_count = cached_sms[dev];
    set_sm_count(cached_sms[dev]);
    return cached_ok[dev] == 1 ? QFP4_OK : QFP4_ERR_UNSUPPORTED_ARCH;
}

// ---- TMA descriptors (driver entry point fetched through the runtime) --------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] { fn = driver_fn<EncodeTiledFn>("cuTensorMapEncodeTiled"); });
    return fn;
}

// 5-D view of a bf16 R x C tensor for the column quantizer: dimensions
// (column, r % 2, r / G, (r / 2) % 4, (r / 8) % (G / 8)), box (64, 2, 4, 4,
// G / 8), 128-byte swizzle. The box lands in shared memory with x-row r at
// 128-byte row s = r%2 + 2 (r/G % 4) + 8 ((r/2) % 4) + 32 ((r/8) % (G/8)).
int make_col_tmap(CUtensorMap* tm, const void* x, int64_t R, int64_t C, int64_t ld, int G) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[5] = {(cuuint64_t)C, 2, (cuuint64_t)(R / G), 4, (cuuint64_t)(G / 8)};
    const cuuint64_t strides[4] = {(cuuint64_t)ld * 2, (cuuint64_t)G * ld * 2, (cuuint64_t)2 * ld * 2,
                                   (cuuint64_t)8 * ld * 2};
    const cuuint32_t box[5] = {64, 2, 4, 4, (cuuint32_t)(G / 8)};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(x), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return QFP4_OK;
}

// 4-D view of a bf16 R x C tensor (R a multiple of 64) for the column
// quantizer over 64-row bands: dimensions (column, r % 2, r / 64, (r / 2) % 32),
// box (64, 2, 4, 32), 128-byte swizzle. The box lands in shared memory with
// x-row r = k + 2 v + 64 q at 128-byte row s = k + 2 q + 8 v. The band count
// bounds the view, so no address past row R - 1 is formed.
int make_col64_tmap(CUtensorMap* tm, const void* x, int64_t R, int64_t C, int64_t ld) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[4] = {(cuuint64_t)C, 2, (cuuint64_t)(R / 64), 32};
    const cuuint64_t strides[3] = {(cuuint64_t)ld * 2, (cuuint64_t)64 * ld * 2, (cuuint64_t)2 * ld * 2};
    const cuuint32_t box[4] = {64, 2, 4, 32};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(x), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return QFP4_OK;
}

// 2-D view of a bf16 R x C tensor for the row quantizer: box 64 columns x 256
// rows (128 bytes per row), 128-byte swizzle.
int make_row_tmap(CUtensorMap* tm, const void* x, int64_t R, int64_t C, int64_t ld) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[2] = {(cuuint64_t)C, (cuuint64_t)R};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {64, 256};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return QFP4_OK;
}

// TMA view of x for a pass in the given orientation (G: column-mode group).
int make_input_tmap(CUtensorMap* tm, const void* x, int64_t R, int64_t C, int64_t ld, int axis, int G) {
    return axis == QFP4_AXIS_ROW ? make_row_tmap(tm, x, R, C, ld) : make_col_tmap(tm, x, R, C, ld, G);
}

// 2-D view of packed FP4 codes [rows][k/2] as bytes, box (128 bytes, box_rows),
// 128-byte swizzle: the K-major operand layout of the MMA.
int make_codes_tmap(CUtensorMap* tm, const void* codes, int64_t rows, int64_t k, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[2] = {(cuuint64_t)(k / 2), (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(k / 2)};
    const cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return QFP4_OK;
}

// 2-D view of the GEMM output D [M][N] (row stride ldd elements, bf16 or fp32)
// for TMA stores: box of 128 bytes x 32 rows, 128-byte swizzle.
int make_out_tmap(CUtensorMap* tm, void* D, int64_t M, int64_t N, int64_t ldd, bool f32) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cuda_fail(cudaErrorNotSupported);
    const cuuint32_t esz = f32 ? 4 : 2;
    const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)ldd * esz};
    const cuuint32_t box[2] = {128 / esz, 32};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(tm, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return QFP4_OK;
}

// 3-D view of a scale buffer as uint32 words: (128 words = one 512-byte atom,
// atoms along k, 128-row blocks), box (128, atoms_per_box, depth). Atoms past
// the buffer read as zero scales.
int make_scale_tmap(CUtensorMap* tm, const void* scales, int64_t rows, int64_t atoms_k, int atoms_per_box,
                    int depth) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[3] = {128, (cuuint64_t)atoms_k, (cuuint64_t)((rows + 127) / 128)};
    const cuuint64_t strides[2] = {512, (cuuint64_t)atoms_k * 512};
    const cuuint32_t box[3] = {128, (cuuint32_t)atoms_per_box, (cuuint32_t)depth};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(scales), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return QFP4_OK;
}

// The band-walking column quantizer is used whenever the quantized axis is a
// multiple of 64; QFP4_COL_BANDS=0 selects the group-walking one instead (same
// results; read on every call).
bool col_bands_enabled() {
    const char* e = std::getenv("QFP4_COL_BANDS");
    return !(e != nullptr && e[0] == '0');
}

// NVFP4 tensors up to this size (bf16 bytes) are quantized by the fused
// one-launch kernel, whose second pass then reads them from L2 (126 MB, split
// between the two dies), when QFP4_FUSED_AMAX=1 (same results; read on every
// call). It is not the default: with programmatic dependent launch the
// separate amax pass and quantizer overlap their boundary and measure 3-9 %
// faster than the one cooperative launch, whose grid barrier waits for the
// slowest CTA of the first pass.
constexpr int64_t kFusedAmaxMaxBytes = (int64_t)96 << 20;
bool fused_amax_enabled() {
    const char* e = std::getenv("QFP4_FUSED_AMAX");
    return e != nullptr && e[0] == '1';
}

// CTA-pair kernel unless A has at most 128 rows (one pair tile would be half
// empty); QFP4_GEMM_PAIR=1 / =0 forces one kernel (read on every call).
bool use_pair_gemm(int64_t M) {
    const char* e = std::getenv("QFP4_GEMM_PAIR");
    if (e != nullptr && (e[0] == '0' || e[0] == '1')) return e[0] == '1';
    return M > kGemmBM;
}

int write_one(float* dst, cudaStream_t s) {
    static const float one = 1.0f;
    cudaError_t e = cudaMemcpyAsync(dst, &one, sizeof(float), cudaMemcpyHostToDevice, s);
    return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
}

int amax_partial_count(int sms, int64_t tiles) {
    int64_t n = 2 * (int64_t)sms;
    if (n > tiles) n = tiles;
    if (n > kMaxAmaxPartials) n = kMaxAmaxPartials;
    return n < 1 ? 1 : (int)n;
}

// Philox4x32-10 word 0 of counter (0, 0, kTagSign | stream << 4, 0): the 32
// random Hadamard sign bits of a call (the kernels receive them as an argument).
uint32_t host_sign_bits(uint64_t seed, uint32_t stream) {
    uint32_t c0 = 0, c1 = 0, c2 = (uint32_t)kTagSign | (stream << 4), c3 = 0;
    uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
    for (int r = 0; r < 10; ++r) {
        if (r) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0, n1 = (uint32_t)p1;
        const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1, n3 = (uint32_t)p0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    return c0;
}

struct Geometry {
    int64_t rows, k;
};

int validate_input(const void* x, int64_t R, int64_t C, int64_t ld, int32_t had, int32_t axis, Geometry* g) {
    if (R < 0 || C < 0 || R > 0x7fffffffLL || C > 0x7fffffffLL) return QFP4_ERR_INVALID_ARG;
    if (axis != QFP4_AXIS_ROW && axis != QFP4_AXIS_COL) return QFP4_ERR_INVALID_ARG;
    if (had < QFP4_HAD_NONE || had > QFP4_HAD_RAND32) return QFP4_ERR_INVALID_ARG;
    if (ld < C) return QFP4_ERR_INVALID_ARG;
    if (R > 0 && C > 0) {
        if (x == nullptr) return QFP4_ERR_INVALID_ARG;
        if (!aligned16(x) || (ld % 8) != 0) return QFP4_ERR_MISALIGNED;
    }
    g->rows = axis == QFP4_AXIS_ROW ? R : C;
    g->k = axis == QFP4_AXIS_ROW ? C : R;
    const int nh = had_n(had);
    if (nh && g->k % nh != 0) return QFP4_ERR_INVALID_ARG;
    return QFP4_OK;
}

// Amax pass into `partials` (their count returned in *n_partials).
int run_amax(const void* x, int64_t R, int64_t C, int64_t ld, int32_t had, int32_t axis, uint32_t signs,
             const Geometry& g, float* partials, int* n_partials, int sms, cudaStream_t s) {
    QuantParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.R = R; p.C = C; p.ld = ld;
    p.rows = g.rows; p.k = g.k;
    p.signs = signs;
    p.amax_out = partials;
    const int nh = had_n(had);
    const int G = col_group(16, nh);
    CUtensorMap tm;
    int rc = make_input_tmap(&tm, x, R, C, ld, axis, G);
    if (rc) return rc;
    *n_partials = amax_partial_count(sms, quant_tiles(axis, g.rows, g.k, G));
    cudaError_t e = launch_amax(p, axis, nh, &tm, *n_partials, s);
    return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
}

int quantize_impl(const void* x, int64_t R, int64_t C, int64_t ld, int32_t fmt, int32_t rounding, int32_t had,
                  int32_t axis, const qfp4_seed* seed, const float* amax_in, qfp4_tensor* out, void* workspace,
                  size_t workspace_bytes, cudaStream_t s) {
    int sms = 0;
    int rc = bind_context(s);
    if (rc) return rc;
    rc = check_device(&sms);
    if (rc) return rc;
    if (!valid_fmt(fmt)) return QFP4_ERR_INVALID_ARG;
    if (rounding < QFP4_RTN || rounding > QFP4_QUARTET2) return QFP4_ERR_INVALID_ARG;
    if (out == nullptr || seed == nullptr) return QFP4_ERR_INVALID_ARG;
    if (seed->rot_stream >= (1u << 28) || seed->sr_stream >= (1u << 28)) return QFP4_ERR_INVALID_ARG;
    Geometry g;
    if ((rc = validate_input(x, R, C, ld, had, axis, &g))) return rc;
    const int NB = block_of(fmt);
    if (g.k % NB != 0) return QFP4_ERR_INVALID_ARG;
    if (out->tensor_scale == nullptr) return QFP4_ERR_INVALID_ARG;
    const bool nonempty = g.rows > 0 && g.k > 0;
    if (nonempty) {
        if (out->codes == nullptr || out->scales == nullptr) return QFP4_ERR_INVALID_ARG;
        if (!aligned16(out->codes) || !aligned16(out->scales)) return QFP4_ERR_MISALIGNED;
    }
    const bool need_ws = nonempty && fmt == QFP4_NVFP4 && amax_in == nullptr;
    if (need_ws) {
        if (workspace == nullptr || workspace_bytes < qfp4_quantize_workspace_bytes()) return QFP4_ERR_WORKSPACE;
        if (!aligned16(workspace)) return QFP4_ERR_MISALIGNED;
    }
    out->rows = g.rows;
    out->k = g.k;
    // the round-up MXFP4 variant only chooses the exponent differently: the
    // result is an ordinary MXFP4 tensor
    const int sfmt = (fmt == QFP4_MXFP4_RU) ? QFP4_MXFP4 : fmt;
    out->fmt = sfmt;
    out->had = had;
    out->rot_seed = had_random(had) ? seed->rot : 0;
    out->rot_stream = had_random(had) ? seed->rot_stream : 0;
    out->reserved = 0;
    if (!nonempty) return write_one(out->tensor_scale, s);

    const uint32_t signs = had_random(had) ? host_sign_bits(seed->rot, seed->rot_stream) : 0u;
    const int nh = had_n(had);
    QuantParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.R = R; p.C = C; p.ld = ld;
    p.rows = g.rows; p.k = g.k;
    p.codes = out->codes;
    p.scales = out->scales;
    p.tensor_scale = out->tensor_scale;
    p.kb4 = (g.k / NB + 3) / 4 * 4;
    p.signs = signs;
    p.sr_seed = seed->sr;
    p.sr_tag_elem = (uint32_t)kTagElement | (seed->sr_stream << 4);
    p.sr_tag_scale = (uint32_t)kTagScale | (seed->sr_stream << 4);
    p.amax_in = amax_in;
    p.mx_round_up = (fmt == QFP4_MXFP4_RU) ? 1u : 0u;
    // the column quantizer walks 64-row bands when the quantized axis allows it
    const bool bands = axis == QFP4_AXIS_COL && g.k % 64 == 0 && col_bands_enabled();
    // An NVFP4 tensor that fits in L2, in the packed unit's cases, is quantized
    // by one cooperative launch that takes its own amax first (the second pass
    // reads from L2) instead of an amax pass, a reduction and the quantizer.
    const bool fused = need_ws && (rounding == QFP4_RTN || rounding == QFP4_QUARTET2) && (nh == 0 || nh == 16) &&
                       (axis == QFP4_AXIS_ROW || bands) && R * C * 2 <= kFusedAmaxMaxBytes && fused_amax_enabled();
    if (fused) {
        float* partials = static_cast<float*>(workspace);
        uint32_t* counter = static_cast<uint32_t*>(workspace) + (kMaxAmaxPartials - 1);
        const cudaError_t e = cudaMemsetAsync(counter, 0, sizeof(uint32_t), s);
        if (e != cudaSuccess) return cuda_fail(e);
        p.amax_out = partials;
        p.amax_partials = partials;
        p.grid_counter = counter;
    } else if (need_ws) {
        int n = 0;
        float* partials = static_cast<float*>(workspace);
        if ((rc = run_amax(x, R, C, ld, had, axis, signs, g, partials, &n, sms, s))) return rc;
        p.amax_partials = partials;
        p.n_partials = n;
    }
    CUtensorMap tm;
    if (bands)
        rc = make_col64_tmap(&tm, x, R, C, ld);
    else
        rc = make_input_tmap(&tm, x, R, C, ld, axis, col_group(NB, nh));
    if (rc) return rc;
    cudaError_t e = fused ? launch_quant_fused(p, rounding, nh, bands ? 2 : axis, &tm, s)
                          : launch_quant(p, sfmt, rounding, nh, bands ? 2 : axis, &tm, s);
    return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
}

// Can one read of x (R x C) give both orientations' quantizations? Same
// format and rounding (caller), R a multiple of 64, the row orientation's
// Hadamard none or of the column one's size.
bool dual_ok(int64_t R, int32_t had_row, int32_t had_col) {
    return R % 64 == 0 && (had_n(had_row) == 0 || had_n(had_row) == had_n(had_col));
}

void fill_out(qfp4_tensor* out, int64_t rows, int64_t k, int32_t fmt, int32_t had, const qfp4_seed* seed) {
    out->rows = rows;
    out->k = k;
    out->fmt = (fmt == QFP4_MXFP4_RU) ? QFP4_MXFP4 : fmt;
    out->had = had;
    out->rot_seed = had_random(had) ? seed->rot : 0;
    out->rot_stream = had_random(had) ? seed->rot_stream : 0;
    out->reserved = 0;
}

int quantize_dual_impl(const void* x, int64_t R, int64_t C, int64_t ld, int32_t fmt, int32_t rounding, int32_t had_row,
                       int32_t had_col, const qfp4_seed* seed_row, const qfp4_seed* seed_col, const float* amax_row,
                       const float* amax_col, qfp4_tensor* out_row, qfp4_tensor* out_col, cudaStream_t s) {
    int sms = 0;
    int rc = bind_context(s);
    if (rc) return rc;
    rc = check_device(&sms);
    if (rc) return rc;
    if (!valid_fmt(fmt)) return QFP4_ERR_INVALID_ARG;
    if (rounding < QFP4_RTN || rounding > QFP4_QUARTET2) return QFP4_ERR_INVALID_ARG;
    if (!out_row || !out_col || !seed_row || !seed_col) return QFP4_ERR_INVALID_ARG;
    for (const qfp4_seed* sd : {seed_row, seed_col})
        if (sd->rot_stream >= (1u << 28) || sd->sr_stream >= (1u << 28)) return QFP4_ERR_INVALID_ARG;
    Geometry gr, gc;
    if ((rc = validate_input(x, R, C, ld, had_row, QFP4_AXIS_ROW, &gr))) return rc;
    if ((rc = validate_input(x, R, C, ld, had_col, QFP4_AXIS_COL, &gc))) return rc;
    const int NB = block_of(fmt);
    if (C % NB != 0 || R % NB != 0) return QFP4_ERR_INVALID_ARG;
    if (R == 0 || C == 0) return QFP4_ERR_INVALID_ARG;
    if (!dual_ok(R, had_row, had_col)) return QFP4_ERR_INVALID_ARG;
    if (fmt == QFP4_NVFP4 && (amax_row == nullptr || amax_col == nullptr)) return QFP4_ERR_INVALID_ARG;
    for (const qfp4_tensor* o : {out_row, out_col}) {
        if (!o->codes || !o->scales || !o->tensor_scale) return QFP4_ERR_INVALID_ARG;
        if (!aligned16(o->codes) || !aligned16(o->scales)) return QFP4_ERR_MISALIGNED;
    }
    fill_out(out_row, R, C, fmt, had_row, seed_row);
    fill_out(out_col, C, R, fmt, had_col, seed_col);
    QuantParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.R = R; p.C = C; p.ld = ld;
    p.rows = C; p.k = R;  // the column orientation
    p.codes = out_col->codes;
    p.scales = out_col->scales;
    p.tensor_scale = out_col->tensor_scale;
    p.kb4 = (R / NB + 3) / 4 * 4;
    p.signs = had_random(had_col) ? host_sign_bits(seed_col->rot, seed_col->rot_stream) : 0u;
    p.sr_seed = seed_col->sr;
    p.sr_tag_elem = (uint32_t)kTagElement | (seed_col->sr_stream << 4);
    p.sr_tag_scale = (uint32_t)kTagScale | (seed_col->sr_stream << 4);
    p.amax_in = amax_col;
    p.mx_round_up = (fmt == QFP4_MXFP4_RU) ? 1u : 0u;
    p.codes_row = out_row->codes;
    p.scales_row = out_row->scales;
    p.tensor_scale_row = out_row->tensor_scale;
    p.amax_in_row = amax_row;
    p.kb4_row = (C / NB + 3) / 4 * 4;
    p.signs_row = had_random(had_row) ? host_sign_bits(seed_row->rot, seed_row->rot_stream) : 0u;
    p.sr_seed_row = seed_row->sr;
    p.sr_tag_elem_row = (uint32_t)kTagElement | (seed_row->sr_stream << 4);
    p.sr_tag_scale_row = (uint32_t)kTagScale | (seed_row->sr_stream << 4);
    CUtensorMap tm;
    if ((rc = make_col64_tmap(&tm, x, R, C, ld))) return rc;
    const int sfmt = (fmt == QFP4_MXFP4_RU) ? QFP4_MXFP4 : fmt;
    cudaError_t e = launch_quant_dual(p, sfmt, rounding, had_n(had_col), had_n(had_row), &tm, s);
    return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
}

// The optional MXFP4 copy of a bf16 GEMM output (qfp4_gemm_quantize).
struct QuantOut {
    int32_t had;
    const qfp4_seed* seed;
    qfp4_tensor* out;
};

// The optional NVFP4 tensor amax of a bf16 GEMM output along its rows
// (qfp4_gemm_amax).
struct AmaxOut {
    int32_t had;
    const qfp4_seed* seed;
    float* amax;
    void* workspace;
    size_t workspace_bytes;
};

int gemm_impl(const qfp4_tensor* A, const qfp4_tensor* B, void* D, int64_t ldd, int32_t out_dtype, bool accumulate,
              cudaStream_t s, const QuantOut* qo = nullptr, const AmaxOut* ao = nullptr) {
    int rc = bind_context(s);
    if (rc) return rc;
    int sms = 0;
    rc = check_device(&sms);
    if (rc) return rc;
    if (A == nullptr || B == nullptr) return QFP4_ERR_INVALID_ARG;
    if (out_dtype != QFP4_OUT_BF16 && out_dtype != QFP4_OUT_F32) return QFP4_ERR_INVALID_ARG;
    if (accumulate && out_dtype != QFP4_OUT_F32) return QFP4_ERR_INVALID_ARG;
    if (qo != nullptr) {
        if (out_dtype != QFP4_OUT_BF16 || qo->out == nullptr || qo->seed == nullptr) return QFP4_ERR_INVALID_ARG;
        if (qo->had < QFP4_HAD_NONE || qo->had > QFP4_HAD_RAND32) return QFP4_ERR_INVALID_ARG;
        if (B->rows % 32 != 0 || A->rows <= 0 || B->rows <= 0 || A->k <= 0) return QFP4_ERR_INVALID_ARG;
        if (!qo->out->codes || !qo->out->scales || !qo->out->tensor_scale) return QFP4_ERR_INVALID_ARG;
        if (!aligned16(qo->out->codes) || !aligned16(qo->out->scales)) return QFP4_ERR_MISALIGNED;
    }
    if (ao != nullptr) {
        if (out_dtype != QFP4_OUT_BF16 || ao->amax == nullptr) return QFP4_ERR_INVALID_ARG;
        if (ao->had < QFP4_HAD_NONE || ao->had > QFP4_HAD_RAND32) return QFP4_ERR_INVALID_ARG;
        if (had_random(ao->had) && ao->seed == nullptr) return QFP4_ERR_INVALID_ARG;
        const int nh = had_n(ao->had);
        if (B->rows % 16 != 0 || (nh && B->rows % nh != 0)) return QFP4_ERR_INVALID_ARG;
        if (ao->workspace == nullptr || ao->workspace_bytes < qfp4_quantize_workspace_bytes())
            return QFP4_ERR_WORKSPACE;
        if (!aligned16(ao->workspace)) return QFP4_ERR_MISALIGNED;
    }
    if (A->fmt != B->fmt || (A->fmt != QFP4_NVFP4 && A->fmt != QFP4_MXFP4)) return QFP4_ERR_INVALID_ARG;
    if (A->k != B->k || A->k < 0 || A->rows < 0 || B->rows < 0) return QFP4_ERR_INVALID_ARG;
    if (A->had != B->had) return QFP4_ERR_INVALID_ARG;
    if (had_random(A->had) && (A->rot_seed != B->rot_seed || A->rot_stream != B->rot_stream))
        return QFP4_ERR_INVALID_ARG;
    if (A->k % 64 != 0) return QFP4_ERR_INVALID_ARG;
    if (A->rows > 0x7fffffffLL || B->rows > 0x7fffffffLL || A->k > 0x7fffffffLL) return QFP4_ERR_INVALID_ARG;
    const int64_t M = A->rows, N = B->rows, K = A->k;
    if (M == 0 || N == 0) {
        if (ao == nullptr) return QFP4_OK;
        const cudaError_t e = cudaMemsetAsync(ao->amax, 0, sizeof(float), s);  // the amax of an empty tensor
        return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
    }
    const size_t esz = out_dtype == QFP4_OUT_F32 ? 4 : 2;
    if (D == nullptr || ldd < N) return QFP4_ERR_INVALID_ARG;
    if (!aligned16(D) || (ldd * (int64_t)esz) % 16 != 0) return QFP4_ERR_MISALIGNED;
    if (K == 0) {
        if (accumulate) return QFP4_OK;  // D += 0
        cudaError_t e = cudaMemset2DAsync(D, (size_t)ldd * esz, 0, (size_t)N * esz, (size_t)M, s);
        if (e == cudaSuccess && ao != nullptr) e = cudaMemsetAsync(ao->amax, 0, sizeof(float), s);
        return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
    }
    if (!A->codes || !B->codes || !A->scales || !B->scales || !A->tensor_scale || !B->tensor_scale)
        return QFP4_ERR_INVALID_ARG;
    if (!aligned16(A->codes) || !aligned16(B->codes) || !aligned16(A->scales) || !aligned16(B->scales))
        return QFP4_ERR_MISALIGNED;
    const bool pair = use_pair_gemm(M);
    CUtensorMap tA, tB;
    if ((rc = make_codes_tmap(&tA, A->codes, M, K, kGemmBM))) return rc;
    if ((rc = make_codes_tmap(&tB, B->codes, N, K, pair ? 128 : kGemmBN))) return rc;
    GemmParams p{};
    p.sfa = A->scales;
    p.sfb = B->scales;
    p.ga = A->tensor_scale;
    p.gb = B->tensor_scale;
    p.D = D;
    p.ldd = ldd;
    p.out_f32 = out_dtype == QFP4_OUT_F32;
    p.accumulate = accumulate ? 1 : 0;
    int nhq = -1;
    if (qo != nullptr && pair) {
        nhq = had_n(qo->had);
        p.q_codes = qo->out->codes;
        p.q_scales = qo->out->scales;
        p.q_kb4 = (N / 32 + 3) / 4 * 4;
        p.q_signs = had_random(qo->had) ? host_sign_bits(qo->seed->rot, qo->seed->rot_stream) : 0u;
    }
    int amx = -1;
    uint32_t amax_signs = 0;
    if (ao != nullptr) {
        amax_signs = had_random(ao->had) ? host_sign_bits(ao->seed->rot, ao->seed->rot_stream) : 0u;
        if (pair) {
            amx = had_n(ao->had);
            p.amax_partials = static_cast<float*>(ao->workspace);
            p.amax_signs = amax_signs;
        }
    }
    p.M = (int)M; p.N = (int)N; p.K = (int)K;
    const int NB = block_of(A->fmt);
    p.atoms_k = (int)((K / NB + 3) / 4);
    cudaError_t e;
    int n_partials = 0;
    if (pair) {
        const int atoms_per_kt = kGemmBK / (4 * NB);
        CUtensorMap tSFA, tSFB, tD;
        if ((rc = make_scale_tmap(&tSFA, A->scales, M, p.atoms_k, atoms_per_kt, 1))) return rc;
        if ((rc = make_scale_tmap(&tSFB, B->scales, N, p.atoms_k, atoms_per_kt, 2))) return rc;
        if ((rc = make_out_tmap(&tD, D, M, N, ldd, p.out_f32))) return rc;
        e = launch_gemm_pair(p, A->fmt, &tA, &tB, &tSFA, &tSFB, &tD, s, sms, nhq, amx, &n_partials);
    } else {
        e = launch_gemm(p, A->fmt, &tA, &tB, s, sms);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    if (ao != nullptr) {
        if (pair) {  // one maximum over the CTAs' partials
            e = launch_reduce_max(p.amax_partials, n_partials, ao->amax, s);
            return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
        }
        // the single-CTA kernel has no amax epilogue: a pass over D afterwards
        Geometry g{M, N};
        int n = 0;
        if ((rc = run_amax(D, M, N, ldd, ao->had, QFP4_AXIS_ROW, amax_signs, g, static_cast<float*>(ao->workspace), &n,
                           sms, s)))
            return rc;
        e = launch_reduce_max(static_cast<const float*>(ao->workspace), n, ao->amax, s);
        return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
    }
    if (qo != nullptr) {
        if (!pair)  // the single-CTA kernel has no quantizing epilogue: quantize D afterwards
            return quantize_impl(D, M, N, ldd, QFP4_MXFP4, QFP4_RTN, qo->had, QFP4_AXIS_ROW, qo->seed, nullptr,
                                 qo->out, nullptr, 0, s);
        fill_out(qo->out, M, N, QFP4_MXFP4, qo->had, qo->seed);
        if ((rc = write_one(qo->out->tensor_scale, s))) return rc;
    }
    return QFP4_OK;
}

// ---- linear layer -------------------------------------------------------------
size_t round_up(size_t v) { return (v + 255) / 256 * 256; }

struct Carver {
    uint8_t* base;
    size_t off;
    void* take(size_t bytes) {
        void* p = base ? base + off : nullptr;
        off += round_up(bytes);
        return p;
    }
};

// Carve one quantized operand (rows x k) out of the workspace.
void carve_operand(Carver& c, qfp4_tensor* t, int fmt, int64_t rows, int64_t k) {
    std::memset(t, 0, sizeof *t);
    t->codes = static_cast<uint8_t*>(c.take(qfp4_codes_bytes(rows, k)));
    t->scales = static_cast<uint8_t*>(c.take(qfp4_scales_bytes(fmt, rows, k)));
    t->tensor_scale = static_cast<float*>(c.take(sizeof(float)));
}

bool valid_cfg(const qfp4_gemm_cfg& g) {
    return valid_fmt(g.fmt) && g.rnd_a >= QFP4_RTN && g.rnd_a <= QFP4_QUARTET2 &&
           g.rnd_b >= QFP4_RTN && g.rnd_b <= QFP4_QUARTET2 && g.had >= QFP4_HAD_NONE && g.had <= QFP4_HAD_RAND32;
}
bool valid_dtype(int32_t d) { return d == QFP4_OUT_BF16 || d == QFP4_OUT_F32; }

int linear_layout(int backward, int64_t M, int64_t N, int64_t K, const qfp4_recipe* r, uint8_t* ws, qfp4_tensor* t,
                  float** partials, size_t* total, float** dy_amax = nullptr) {
    Carver c{ws, 0};
    *partials = static_cast<float*>(c.take(qfp4_quantize_workspace_bytes()));
    if (backward) {
        float* a = static_cast<float*>(c.take(2 * sizeof(float)));  // dY's row and column amax
        if (dy_amax) *dy_amax = a;
    }
    if (!backward) {
        carve_operand(c, &t[0], r->fprop.fmt, M, K);  // X along K
        carve_operand(c, &t[1], r->fprop.fmt, N, K);  // W along K
    } else {
        carve_operand(c, &t[0], r->dgrad.fmt, M, N);  // dY along N
        carve_operand(c, &t[1], r->dgrad.fmt, K, N);  // W^T: W along N
        carve_operand(c, &t[2], r->wgrad.fmt, N, M);  // dY^T: dY along M
        carve_operand(c, &t[3], r->wgrad.fmt, K, M);  // X^T: X along M
    }
    *total = c.off;
    return QFP4_OK;
}

int check_linear_args(int64_t M, int64_t N, int64_t K, const qfp4_recipe* r, const qfp4_seed* seed) {
    if (r == nullptr || seed == nullptr) return QFP4_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0 || (M % 128) || (N % 128) || (K % 128)) return QFP4_ERR_INVALID_ARG;
    if (!valid_cfg(r->fprop) || !valid_cfg(r->dgrad) || !valid_cfg(r->wgrad)) return QFP4_ERR_INVALID_ARG;
    if (!valid_dtype(r->y_dtype) || !valid_dtype(r->dx_dtype) || !valid_dtype(r->dw_dtype)) return QFP4_ERR_INVALID_ARG;
    if (r->dw_accumulate != 0 && (r->dw_accumulate != 1 || r->dw_dtype != QFP4_OUT_F32)) return QFP4_ERR_INVALID_ARG;
    return QFP4_OK;
}

qfp4_seed op_seed(const qfp4_seed* s, uint32_t gemm, uint32_t operand) {
    qfp4_seed o;
    o.rot = s->rot;
    o.sr = s->sr;
    o.rot_stream = gemm;
    o.sr_stream = operand;
    return o;
}

// Both orientations' rotated amax. n_h <= 16: one read of x by the column
// kernel (its tile serves 16-element groups of both axes); n_h = 32: two passes.
int amax_rowcol_impl(const void* x, int64_t R, int64_t C, int64_t ld, int32_t had_row, int32_t had_col,
                     const qfp4_seed* seed_row, const qfp4_seed* seed_col, float* amax_row, float* amax_col,
                     void* workspace, size_t workspace_bytes, cudaStream_t s) {
    int rc = bind_context(s);  // callers may run on threads without a current context
    if (rc) return rc;
    int sms = 0;
    if ((rc = check_device(&sms))) return rc;
    Geometry gr, gc;
    if ((rc = validate_input(x, R, C, ld, had_row, QFP4_AXIS_ROW, &gr))) return rc;
    if ((rc = validate_input(x, R, C, ld, had_col, QFP4_AXIS_COL, &gc))) return rc;
    if (amax_row == nullptr || amax_col == nullptr) return QFP4_ERR_INVALID_ARG;
    if ((had_random(had_row) && seed_row == nullptr) || (had_random(had_col) && seed_col == nullptr))
        return QFP4_ERR_INVALID_ARG;
    if (workspace == nullptr || workspace_bytes < qfp4_quantize_workspace_bytes()) return QFP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QFP4_ERR_MISALIGNED;
    if (R == 0 || C == 0) {
        cudaError_t e = cudaMemsetAsync(amax_row, 0, sizeof(float), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(amax_col, 0, sizeof(float), s);
        return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
    }
    // a deterministic Hadamard is the random one with no sign flips
    const uint32_t signs_row = had_random(had_row) ? host_sign_bits(seed_row->rot, seed_row->rot_stream) : 0u;
    const uint32_t signs_col = had_random(had_col) ? host_sign_bits(seed_col->rot, seed_col->rot_stream) : 0u;
    float* partials = static_cast<float*>(workspace);
    const int nh = had_n(had_col);
    cudaError_t e;
    if (nh <= 16 && had_n(had_row) == nh) {
        QuantParams p{};
        p.x = static_cast<const uint16_t*>(x);
        p.R = R; p.C = C; p.ld = ld;
        p.rows = gc.rows; p.k = gc.k;
        p.signs = signs_col;
        p.signs_row = signs_row;
        // over 64-row bands when R allows it (both orientations packed), else
        // the group-walking column kernel
        const bool bands = R % 64 == 0 && col_bands_enabled();
        const int n = amax_partial_count(
            sms, bands ? amax_rowcol64_tiles(gc.rows, gc.k) : quant_tiles(QFP4_AXIS_COL, gc.rows, gc.k, 16));
        if (2 * n > kMaxAmaxPartials) return QFP4_ERR_WORKSPACE;
        p.amax_out = partials;
        p.amax_out_row = partials + n;
        CUtensorMap tm;
        if (bands) {
            if ((rc = make_col64_tmap(&tm, x, R, C, ld))) return rc;
            e = launch_amax_rowcol64(p, nh, &tm, n, s);
        } else {
            if ((rc = make_input_tmap(&tm, x, R, C, ld, QFP4_AXIS_COL, 16))) return rc;
            e = launch_amax_rowcol(p, nh, &tm, n, s);
        }
        if (e == cudaSuccess) e = launch_reduce_max(partials, n, amax_col, s);
        if (e == cudaSuccess) e = launch_reduce_max(partials + n, n, amax_row, s);
    } else {
        // a 32-point Hadamard, or Hadamards of different sizes: one pass per orientation
        int n = 0;
        if ((rc = run_amax(x, R, C, ld, had_row, QFP4_AXIS_ROW, signs_row, gr, partials, &n, sms, s))) return rc;
        e = launch_reduce_max(partials, n, amax_row, s);
        if (e != cudaSuccess) return cuda_fail(e);
        if ((rc = run_amax(x, R, C, ld, had_col, QFP4_AXIS_COL, signs_col, gc, partials, &n, sms, s))) return rc;
        e = launch_reduce_max(partials, n, amax_col, s);
    }
    return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
}

}  // namespace

void count_launch() { ++t_launches; }

}  // namespace qfp4

using namespace qfp4;

extern "C" {

const char* qfp4_strerror(int status) {
    switch (status) {
        case QFP4_OK: return "ok";
        case QFP4_ERR_INVALID_ARG: return "invalid argument";
        case QFP4_ERR_MISALIGNED: return "misaligned pointer or row stride";
        case QFP4_ERR_UNSUPPORTED_ARCH: return "device is not sm_100 (B200)";
        case QFP4_ERR_WORKSPACE: return "workspace missing or too small";
        case QFP4_ERR_CUDA: return "CUDA error";
        case QFP4_ERR_TIMEOUT: return "device-side bounded wait expired";
        case QFP4_ERR_BOUNDS: return "bounds-checked build: a kernel store fell outside its buffer";
        case QFP4_ERR_TOO_LARGE: return "problem exceeds the fixed scratch of qfp4_linear_fwd_noalloc (32 MiB)";
        default: return "unknown status";
    }
}

int qfp4_last_cuda_error(void) { return t_last_cuda_error; }

int64_t qfp4_launch_count(int32_t reset) {
    const int64_t n = t_launches;
    if (reset) t_launches = 0;
    return n;
}

size_t qfp4_codes_bytes(int64_t rows, int64_t k) { return (rows <= 0 || k <= 0) ? 0 : (size_t)(rows * k / 2); }

size_t qfp4_scales_bytes(int32_t fmt, int64_t rows, int64_t k) {
    if (!valid_fmt(fmt) || rows <= 0 || k <= 0) return 0;
    const int64_t kb = (k + block_of(fmt) - 1) / block_of(fmt);
    return (size_t)(((rows + 127) / 128) * ((kb + 3) / 4) * 512);
}

int64_t qfp4_scale_offset(int32_t fmt, int64_t rows, int64_t k, int64_t r, int64_t c) {
    if (!valid_fmt(fmt) || rows <= 0 || k <= 0) return -1;
    const int64_t kb = (k + block_of(fmt) - 1) / block_of(fmt);
    const int64_t rows_p = (rows + 127) / 128 * 128, kb4 = (kb + 3) / 4 * 4;
    if (r < 0 || c < 0 || r >= rows_p || c >= kb4) return -1;
    return ((r / 128) * (kb4 / 4) + c / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4);
}

size_t qfp4_quantize_workspace_bytes(void) { return (size_t)kMaxAmaxPartials * sizeof(float); }

int qfp4_amax(const void* x, int64_t R, int64_t C, int64_t ld, int32_t had, int32_t axis, const qfp4_seed* seed,
              float* amax, void* workspace, size_t workspace_bytes, void* stream) {
    const ApiRange range("qfp4_amax");
    int sms = 0;
    int rc = bind_context(static_cast<cudaStream_t>(stream));
    if (rc) return rc;
    rc = check_device(&sms);
    if (rc) return rc;
    Geometry g;
    if ((rc = validate_input(x, R, C, ld, had, axis, &g))) return rc;
    if (amax == nullptr || (had_random(had) && seed == nullptr)) return QFP4_ERR_INVALID_ARG;
    if (workspace == nullptr || workspace_bytes < qfp4_quantize_workspace_bytes()) return QFP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QFP4_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (g.rows == 0 || g.k == 0) {
        cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), s);
        return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
    }
    const uint32_t signs = had_random(had) ? host_sign_bits(seed->rot, seed->rot_stream) : 0u;
    int n = 0;
    float* partials = static_cast<float*>(workspace);
    if ((rc = run_amax(x, R, C, ld, had, axis, signs, g, partials, &n, sms, s))) return rc;
    cudaError_t e = launch_reduce_max(partials, n, amax, s);
    return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
}

int qfp4_amax_rowcol(const void* x, int64_t R, int64_t C, int64_t ld, int32_t had_row, int32_t had_col,
                     const qfp4_seed* seed_row, const qfp4_seed* seed_col, float* amax_row, float* amax_col,
                     void* workspace, size_t workspace_bytes, void* stream) {
    const ApiRange range("qfp4_amax_rowcol");
    return amax_rowcol_impl(x, R, C, ld, had_row, had_col, seed_row, seed_col, amax_row, amax_col, workspace,
                            workspace_bytes, static_cast<cudaStream_t>(stream));
}

int qfp4_quantize(const void* x, int64_t R, int64_t C, int64_t ld, int32_t fmt, int32_t rounding, int32_t had,
                  int32_t axis, const qfp4_seed* seed, const float* amax_in, qfp4_tensor* out, void* workspace,
                  size_t workspace_bytes, void* stream) {
    const ApiRange range("qfp4_quantize");
    return quantize_impl(x, R, C, ld, fmt, rounding, had, axis, seed, amax_in, out, workspace, workspace_bytes,
                         static_cast<cudaStream_t>(stream));
}

int qfp4_quantize_dual(const void* x, int64_t R, int64_t C, int64_t ld, int32_t fmt, int32_t rounding,
                       int32_t had_row, int32_t had_col, const qfp4_seed* seed_row, const qfp4_seed* seed_col,
                       const float* amax_row, const float* amax_col, qfp4_tensor* out_row, qfp4_tensor* out_col,
                       void* stream) {
    const ApiRange range("qfp4_quantize_dual");
    return quantize_dual_impl(x, R, C, ld, fmt, rounding, had_row, had_col, seed_row, seed_col, amax_row, amax_col,
                              out_row, out_col, static_cast<cudaStream_t>(stream));
}

int qfp4_gemm(const qfp4_tensor* A, const qfp4_tensor* B, void* D, int64_t ldd, int32_t out_dtype, void* stream) {
    const ApiRange range("qfp4_gemm");
    return gemm_impl(A, B, D, ldd, out_dtype, false, static_cast<cudaStream_t>(stream));
}

int qfp4_gemm_quantize(const qfp4_tensor* A, const qfp4_tensor* B, void* D, int64_t ldd, int32_t had,
                       const qfp4_seed* seed, qfp4_tensor* out, void* stream) {
    const ApiRange range("qfp4_gemm_quantize");
    const QuantOut qo{had, seed, out};
    return gemm_impl(A, B, D, ldd, QFP4_OUT_BF16, false, static_cast<cudaStream_t>(stream), &qo);
}

int qfp4_gemm_amax(const qfp4_tensor* A, const qfp4_tensor* B, void* D, int64_t ldd, int32_t had,
                   const qfp4_seed* seed, float* amax, void* workspace, size_t workspace_bytes, void* stream) {
    const ApiRange range("qfp4_gemm_amax");
    const AmaxOut ao{had, seed, amax, workspace, workspace_bytes};
    return gemm_impl(A, B, D, ldd, QFP4_OUT_BF16, false, static_cast<cudaStream_t>(stream), nullptr, &ao);
}

int qfp4_gemm_accumulate(const qfp4_tensor* A, const qfp4_tensor* B, float* D, int64_t ldd, void* stream) {
    const ApiRange range("qfp4_gemm_accumulate");
    return gemm_impl(A, B, D, ldd, QFP4_OUT_F32, true, static_cast<cudaStream_t>(stream));
}

int qfp4_recipe_preset(int32_t preset, qfp4_recipe* out) {
    if (out == nullptr) return QFP4_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof *out);
    out->y_dtype = QFP4_OUT_BF16;
    out->dx_dtype = QFP4_OUT_BF16;
    out->dw_dtype = QFP4_OUT_F32;
    switch (preset) {
        case QFP4_PRESET_NVIDIA_NVFP4:  // 16x16 random Hadamard on Wgrad inputs, SR of the gradient
            out->fprop = {QFP4_NVFP4, QFP4_RTN, QFP4_RTN, QFP4_HAD_NONE};
            out->dgrad = {QFP4_NVFP4, QFP4_SR, QFP4_RTN, QFP4_HAD_NONE};
            out->wgrad = {QFP4_NVFP4, QFP4_SR, QFP4_RTN, QFP4_HAD_RAND16};
            return QFP4_OK;
        case QFP4_PRESET_QUARTET2_NVFP4:  // RTN forward; random rotation + Quartet II scale SR backward
            out->fprop = {QFP4_NVFP4, QFP4_RTN, QFP4_RTN, QFP4_HAD_DET16};
            out->dgrad = {QFP4_NVFP4, QFP4_QUARTET2, QFP4_QUARTET2, QFP4_HAD_RAND16};
            out->wgrad = {QFP4_NVFP4, QFP4_QUARTET2, QFP4_QUARTET2, QFP4_HAD_RAND16};
            return QFP4_OK;
        case QFP4_PRESET_AMD_MXFP4_H:  // MXFP4 everywhere, deterministic Hadamard on Wgrad
            out->fprop = {QFP4_MXFP4, QFP4_RTN, QFP4_RTN, QFP4_HAD_NONE};
            out->dgrad = {QFP4_MXFP4, QFP4_RTN, QFP4_RTN, QFP4_HAD_NONE};
            out->wgrad = {QFP4_MXFP4, QFP4_RTN, QFP4_RTN, QFP4_HAD_DET32};
            return QFP4_OK;
        default: return QFP4_ERR_INVALID_ARG;
    }
}

size_t qfp4_linear_workspace_bytes(int32_t backward, int64_t M, int64_t N, int64_t K, const qfp4_recipe* recipe) {
    if (recipe == nullptr || M < 0 || N < 0 || K < 0) return 0;
    qfp4_tensor t[4];
    float* partials;
    size_t total = 0;
    linear_layout(backward, M, N, K, recipe, nullptr, t, &partials, &total);
    return total;
}

}  // extern "C"

namespace qfp4 {
namespace {
// The forward pass (qfp4_linear_fwd, qfp4_linear_fwd_chain): X and W quantized
// along K, then Fprop. x_amax (nullable): X's NVFP4 tensor amax for this
// Fprop's rotation, given by the caller; amax_out (nullable): Y's NVFP4 tensor
// amax along its rows for the rotation (next_had, next_seed), from the GEMM.
int linear_fwd_impl(const void* X, const void* W, void* Y, int64_t M, int64_t N, int64_t K, const qfp4_recipe* recipe,
                    const qfp4_seed* seed, const float* x_amax, int32_t next_had, const qfp4_seed* next_seed,
                    float* y_amax, void* workspace, size_t workspace_bytes, cudaStream_t s) {
    int rc = check_linear_args(M, N, K, recipe, seed);
    if (rc) return rc;
    if (!X || !W || !Y) return QFP4_ERR_INVALID_ARG;
    if (y_amax != nullptr) {
        if (recipe->y_dtype != QFP4_OUT_BF16) return QFP4_ERR_INVALID_ARG;
        if (next_had < QFP4_HAD_NONE || next_had > QFP4_HAD_RAND32) return QFP4_ERR_INVALID_ARG;
        if (had_random(next_had) && next_seed == nullptr) return QFP4_ERR_INVALID_ARG;
    }
    if (workspace == nullptr || workspace_bytes < qfp4_linear_workspace_bytes(0, M, N, K, recipe))
        return QFP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QFP4_ERR_MISALIGNED;
    qfp4_tensor t[4];
    float* partials;
    size_t total;
    linear_layout(0, M, N, K, recipe, static_cast<uint8_t*>(workspace), t, &partials, &total);
    const qfp4_gemm_cfg& c = recipe->fprop;
    const size_t pws = qfp4_quantize_workspace_bytes();
    qfp4_seed sx = op_seed(seed, 0, 0), sw = op_seed(seed, 0, 1);
    const float* ax = c.fmt == QFP4_NVFP4 ? x_amax : nullptr;
    if ((rc = quantize_impl(X, M, K, K, c.fmt, c.rnd_a, c.had, QFP4_AXIS_ROW, &sx, ax, &t[0], partials, pws, s)))
        return rc;
    if ((rc = quantize_impl(W, N, K, K, c.fmt, c.rnd_b, c.had, QFP4_AXIS_ROW, &sw, nullptr, &t[1], partials, pws, s)))
        return rc;
    if (y_amax == nullptr) return gemm_impl(&t[0], &t[1], Y, N, recipe->y_dtype, false, s);
    // the next layer rotates its input with the sign vector of its own Fprop:
    // key next_seed->rot, stream 0 (the linear layer's seed rule)
    qfp4_seed ns{};
    if (next_seed != nullptr) ns = op_seed(next_seed, 0, 0);
    const AmaxOut ao{next_had, &ns, y_amax, partials, pws};
    return gemm_impl(&t[0], &t[1], Y, N, QFP4_OUT_BF16, false, s, nullptr, &ao);
}
}  // namespace
}  // namespace qfp4

extern "C" {

int qfp4_linear_fwd(const void* X, const void* W, void* Y, int64_t M, int64_t N, int64_t K, const qfp4_recipe* recipe,
                    const qfp4_seed* seed, void* workspace, size_t workspace_bytes, void* stream) {
    const ApiRange range("qfp4_linear_fwd");
    return linear_fwd_impl(X, W, Y, M, N, K, recipe, seed, nullptr, QFP4_HAD_NONE, nullptr, nullptr, workspace,
                           workspace_bytes, static_cast<cudaStream_t>(stream));
}

int qfp4_linear_fwd_chain(const void* X, const void* W, void* Y, int64_t M, int64_t N, int64_t K,
                          const qfp4_recipe* recipe, const qfp4_seed* seed, const float* x_amax, int32_t next_had,
                          const qfp4_seed* next_seed, float* y_amax, void* workspace, size_t workspace_bytes,
                          void* stream) {
    const ApiRange range("qfp4_linear_fwd_chain");
    return linear_fwd_impl(X, W, Y, M, N, K, recipe, seed, x_amax, next_had, next_seed, y_amax, workspace,
                           workspace_bytes, static_cast<cudaStream_t>(stream));
}

int qfp4_linear_bwd(const void* dY, const void* X, const void* W, void* dX, void* dW, int64_t M, int64_t N, int64_t K,
                    const qfp4_recipe* recipe, const qfp4_seed* seed, void* workspace, size_t workspace_bytes,
                    void* stream) {
    const ApiRange range("qfp4_linear_bwd");
    int rc = check_linear_args(M, N, K, recipe, seed);
    if (rc) return rc;
    if (!dY || !X || !W || !dX || !dW) return QFP4_ERR_INVALID_ARG;
    if (workspace == nullptr || workspace_bytes < qfp4_linear_workspace_bytes(1, M, N, K, recipe))
        return QFP4_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QFP4_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    qfp4_tensor t[4];
    float* partials;
    float* dy_amax;
    size_t total;
    linear_layout(1, M, N, K, recipe, static_cast<uint8_t*>(workspace), t, &partials, &total, &dy_amax);
    const size_t pws = qfp4_quantize_workspace_bytes();
    const qfp4_gemm_cfg& d = recipe->dgrad;
    const qfp4_gemm_cfg& w = recipe->wgrad;
    qfp4_seed s0 = op_seed(seed, 1, 2), s1 = op_seed(seed, 1, 3);
    qfp4_seed s2 = op_seed(seed, 2, 4), s3 = op_seed(seed, 2, 5);
    // dY is quantized along both axes (Dgrad: along N; Wgrad: along M). When
    // both are NVFP4 with the same Hadamard (size <= 16; the sign vectors
    // differ per GEMM), one read of dY gives both tensor amaxes. When both
    // quantizations round to nearest with the same format, one more read gives
    // both quantized operands (memory-bound, so one read instead of two is a
    // quarter faster); stochastic and Quartet II rounding are bound by
    // instruction issue, and there the two separate passes are faster.
    const bool dual = d.fmt == w.fmt && d.rnd_a == QFP4_RTN && w.rnd_a == QFP4_RTN && dual_ok(M, d.had, w.had) &&
                      col_bands_enabled();
    const float* am_row = nullptr;
    const float* am_col = nullptr;
    if (d.fmt == QFP4_NVFP4 && w.fmt == QFP4_NVFP4 && d.had == w.had && had_n(d.had) <= 16) {
        if ((rc = amax_rowcol_impl(dY, M, N, N, d.had, d.had, &s0, &s2, dy_amax, dy_amax + 1, partials, pws, s)))
            return rc;
        am_row = dy_amax;
        am_col = dy_amax + 1;
    } else if (dual && d.fmt == QFP4_NVFP4) {
        if ((rc = qfp4_amax(dY, M, N, N, d.had, QFP4_AXIS_ROW, &s0, dy_amax, partials, pws, s))) return rc;
        if ((rc = qfp4_amax(dY, M, N, N, w.had, QFP4_AXIS_COL, &s2, dy_amax + 1, partials, pws, s))) return rc;
        am_row = dy_amax;
        am_col = dy_amax + 1;
    }
    // Dgrad dX[M,K] = dY[M,N] . W[N,K]: reduce over N.
    if (dual) {
        if ((rc = quantize_dual_impl(dY, M, N, N, d.fmt, d.rnd_a, d.had, w.had, &s0, &s2, am_row, am_col, &t[0],
                                     &t[2], s)))
            return rc;
    } else if ((rc = quantize_impl(dY, M, N, N, d.fmt, d.rnd_a, d.had, QFP4_AXIS_ROW, &s0, am_row, &t[0], partials,
                                   pws, s))) {
        return rc;
    }
    if ((rc = quantize_impl(W, N, K, K, d.fmt, d.rnd_b, d.had, QFP4_AXIS_COL, &s1, nullptr, &t[1], partials, pws, s)))
        return rc;
    if ((rc = gemm_impl(&t[0], &t[1], dX, K, recipe->dx_dtype, false, s))) return rc;
    // Wgrad dW[N,K] = dY^T[N,M] . X[M,K]: reduce over M (tokens).
    if (!dual &&
        (rc = quantize_impl(dY, M, N, N, w.fmt, w.rnd_a, w.had, QFP4_AXIS_COL, &s2, am_col, &t[2], partials, pws, s)))
        return rc;
    if ((rc = quantize_impl(X, M, K, K, w.fmt, w.rnd_b, w.had, QFP4_AXIS_COL, &s3, nullptr, &t[3], partials, pws, s)))
        return rc;
    return gemm_impl(&t[2], &t[3], dW, K, recipe->dw_dtype, recipe->dw_accumulate != 0, s);
}

int qfp4_status(void* stream) {
    const ApiRange range("qfp4_status");
    const int rc = bind_context(static_cast<cudaStream_t>(stream));
    if (rc) return rc;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    uint32_t v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_dev_error, sizeof v)) != cudaSuccess) return cuda_fail(e);
    if (v != 0) {
        const uint32_t zero = 0;
        if ((e = cudaMemcpyToSymbol(g_dev_error, &zero, sizeof zero)) != cudaSuccess) return cuda_fail(e);
        return (v & DEV_ERR_BOUNDS) ? QFP4_ERR_BOUNDS : QFP4_ERR_TIMEOUT;
    }
    return QFP4_OK;
}

// ---- failure-detection self-test ------------------------------------------------
namespace qfp4 {
namespace {
// One CTA: an mbarrier that nothing arrives on, waited on with the library's
// bounded wait; the wait gives up after limit_ns, raises the device error word
// and the kernel returns.
__global__ void wait_timeout_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait_for(&bar, 0, limit_ns);
}
}  // namespace
}  // namespace qfp4

int qfp4_selftest_wait_timeout(int64_t limit_ns, void* stream) {
    const ApiRange range("qfp4_selftest_wait_timeout");
    const int rc = bind_context(static_cast<cudaStream_t>(stream));
    if (rc) return rc;
    if (limit_ns <= 0 || limit_ns > (int64_t)kWaitLimitNs) return QFP4_ERR_INVALID_ARG;
    qfp4::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((uint64_t)limit_ns);
    count_launch();
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
}

// ---- rounding self-test ---------------------------------------------------------
namespace qfp4 {
namespace {
// The quantizers' element and scale rounding steps, one value per thread.
__global__ void rounding_selftest_kernel(int32_t op, const float* x, const uint32_t* w, uint8_t* codes, int64_t n) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const float v = x[i];
        uint32_t code;
        if (op == QFP4_ROUND_E2M1_SR || op == QFP4_ROUND_E2M1_RN) {
            float r[8] = {op == QFP4_ROUND_E2M1_SR ? e2m1_sr_value(v, w[i] << 16) : v, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            code = e2m1x8_rn(r) & 0xFu;
        } else if (op == QFP4_ROUND_E4M3_SR) {
            code = e4m3_sr(v, w[i]);
        } else if (op == QFP4_ROUND_E4M3_RN) {
            code = e4m3_rn(v);
        } else {
            code = e8m0_sr(v, uniform24(w[i]));
        }
        codes[i] = (uint8_t)code;
    }
}
}  // namespace
}  // namespace qfp4

int qfp4_selftest_rounding(int32_t op, const float* x, const uint32_t* w, uint8_t* codes, int64_t n, void* stream) {
    const ApiRange range("qfp4_selftest_rounding");
    const int rc = bind_context(static_cast<cudaStream_t>(stream));
    if (rc) return rc;
    if (op < QFP4_ROUND_E2M1_SR || op > QFP4_ROUND_E8M0_SR || n < 0) return QFP4_ERR_INVALID_ARG;
    const bool needs_w = op != QFP4_ROUND_E2M1_RN && op != QFP4_ROUND_E4M3_RN;
    if (n == 0) return QFP4_OK;
    if (!x || !codes || (needs_w && !w)) return QFP4_ERR_INVALID_ARG;
    const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 8);
    qfp4::rounding_selftest_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(op, x, w, codes, n);
    count_launch();
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QFP4_OK : cuda_fail(e);
}

// ---- forward pass without allocation ------------------------------------------
// The scratch of qfp4_linear_fwd_noalloc: a fixed device array (every GPU that
// loads the library holds it until the process exits). Host code cannot use
// the array's name as a device address; its address is looked up with
// cudaGetSymbolAddress, with the caller's device current. The lookup is done
// once per CUDA context: the cache is keyed by the context's unique ID
// (cuCtxGetId, never reused within a process), so a device that was reset
// (cudaDeviceReset gives it a new primary context) or a stream of another
// context on the same device gets a fresh lookup instead of a stale address.
static __device__ __align__(256) uint8_t g_noalloc_scratch[QFP4_NOALLOC_SCRATCH_BYTES];

static int noalloc_scratch(void** out) {
    using CtxIdFn = CUresult (*)(CUcontext, unsigned long long*);
    using CurCtxFn = CUresult (*)(CUcontext*);
    static CtxIdFn ctx_id = nullptr;
    static CurCtxFn cur_ctx = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        ctx_id = driver_fn<CtxIdFn>("cuCtxGetId");
        cur_ctx = driver_fn<CurCtxFn>("cuCtxGetCurrent");
    });
    static std::mutex mu;
    static unsigned long long key[64] = {0};  // context ID of addr[dev]; 0: none
    static void* addr[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= 64) return QFP4_ERR_UNSUPPORTED_ARCH;
    unsigned long long id = 0;
    CUcontext ctx = nullptr;
    const bool have_id = ctx_id != nullptr && cur_ctx != nullptr && cur_ctx(&ctx) == CUDA_SUCCESS && ctx != nullptr &&
                         ctx_id(ctx, &id) == CUDA_SUCCESS && id != 0;
    std::lock_guard<std::mutex> lock(mu);
    if (!have_id || addr[dev] == nullptr || key[dev] != id) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e);
        addr[dev] = p;
        key[dev] = have_id ? id : 0;
    }
    *out = addr[dev];
    return QFP4_OK;
}

int qfp4_linear_fwd_noalloc(const void* X, const void* W, void* Y, int64_t M, int64_t N, int64_t K,
                            const qfp4_recipe* recipe, const qfp4_seed* seed, void* stream) {
    const ApiRange range("qfp4_linear_fwd_noalloc");
    int rc = check_linear_args(M, N, K, recipe, seed);
    if (rc) return rc;
    if (qfp4_linear_workspace_bytes(0, M, N, K, recipe) > QFP4_NOALLOC_SCRATCH_BYTES) return QFP4_ERR_TOO_LARGE;
    if ((rc = bind_context(static_cast<cudaStream_t>(stream)))) return rc;
    void* scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch))) return rc;
    return qfp4_linear_fwd(X, W, Y, M, N, K, recipe, seed, scratch, QFP4_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
