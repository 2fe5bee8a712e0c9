// quant.cu - sm_100a FP4 quantizers: one HBM read of the bf16 tensor and one
// write of the packed E2M1 codes and block scales.
//
// Method (pages: "New AMD paper overturns conventional wisdom: FP4
// training...", section "Chto takoe MXFP4"; "Quartet II - obuchenie v NVFP4 s
// tochnymi nesmeshchyonnymi gradientami"; "NVIDIA sozdala metod obucheniya
// neyrosetey v 4-bit tochnosti", section "Kak eto rabotaet"): per block of the
// quantized axis, an optional Hadamard rotation (deterministic or random
// signs), a micro-scale (E4M3 per 16 for NVFP4 with an fp32 tensor scale, E8M0
// per 32 for MXFP4), then round-to-nearest, per-element stochastic rounding or
// Quartet II (RTN codes, stochastically rounded renormalised scale).
//
// Structure: persistent CTAs of 8 compute warps and 1 producer warp. The
// producer streams tiles of the bf16 tensor into a multi-stage shared-memory
// ring with TMA; every compute thread owns whole groups (G = max(block, n_h)
// consecutive elements of the quantized axis), so the rotation, the block
// reductions and the rounding run in its registers without shuffles.
//   Row mode (blocks along the contiguous axis): tiles of 256 rows x 64
//     columns (128-byte swizzle); thread t takes row t, i.e. 64 / G groups.
//   Column mode (blocks along the strided axis; the output is the quantized
//     transpose): tiles of 4G rows x 128 columns through a 5-D view of the
//     tensor whose row order makes the transposing ldmatrix reads
//     conflict-free; thread (column c, q) takes rows [Gq, Gq + G) of c.
//
// Every fp32 operation is the one the method states, in its order, with no
// fused multiply-add but the one the Quartet II sums define (their first
// stride, written out as __fmaf_rn / __ffma2_rn; the library is built with
// --fmad=false, and packed f32x2 operations round each lane like the scalar
// instruction), so codes and scales are exactly those of the definition.
#include "qfp4_device.cuh"
#include "qfp4_internal.h"

namespace qfp4 {
namespace {

constexpr int kComputeWarps = 8;
constexpr int kThreads = (kComputeWarps + 1) * 32;  // + one producer warp
constexpr int kRowTileRows = 256, kRowTileCols = 64;
constexpr int kColTileCols = 128;

template <int NH>
__device__ __forceinline__ float had_norm() {
    return NH == 16 ? 0.25f : 0x1.6a09e6p-3f;  // fp32(1/sqrt(16)), fp32(1/sqrt(32))
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// max(a, b, c) in one instruction (IEEE maxNum semantics, like fmaxf).
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Largest |v[e]| of N values, starting from m.
template <int N>
__device__ __forceinline__ float abs_max(float m, const float* v) {
#pragma unroll
    for (int e = 0; e < N; e += 2) m = max3(m, fabsf(v[e]), fabsf(v[e + 1]));
    return m;
}

// x / 6 correctly rounded, for x >= 0 (a block amax), with no division
// subroutine. For finite x >= 2^-125: one product with RN(1/6) and one fused
// correction (the division-by-a-known-divisor method of Brisebarre, Muller and
// Raina, IEEE Trans. Computers 53(8), 2004). Below 2^-125 the quotient is
// subnormal: x = N * 2^-149 with N = the bits of x (exponent field 0 or 1),
// and x / 6 rounds to round-half-even(N / 6) * 2^-149, whose bits are that
// integer. Both are checked against the division for every such fp32 x.
// inf and NaN give x * (1/6) (inf, NaN).
__device__ __forceinline__ float div6(float x) {
    if (x >= 0x1p-125f && x <= 0x1.fffffep127f) {
        constexpr float C = 1.0f / 6.0f;
        const float q = __fmul_rn(x, C);
        const float r = __fmaf_rn(-q, 6.0f, x);
        return __fmaf_rn(r, C, q);
    }
    if (x >= 0.0f && x < 0x1p-125f) {
        const uint32_t n = __float_as_uint(x), q = n / 6u, r = n - 6u * q;
        return __uint_as_float(q + ((2u * r > 6u || (2u * r == 6u && (q & 1u) != 0u)) ? 1u : 0u));
    }
    return __fmul_rn(x, 1.0f / 6.0f);
}
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }

// One butterfly stage of half-width H >= 2 over N elements, packed x2.
template <int N, int H>
__device__ __forceinline__ void fwht_stage(float* v) {
#pragma unroll
    for (int j0 = 0; j0 < N; j0 += 2 * H)
#pragma unroll
        for (int j = j0; j < j0 + H; j += 2) {
            const float2 a = f2(v[j], v[j + 1]), b = f2(v[j + H], v[j + H + 1]);
            const float2 s = __fadd2_rn(a, b), d = __fadd2_rn(a, neg2(b));
            v[j] = s.x; v[j + 1] = s.y;
            v[j + H] = d.x; v[j + H + 1] = d.y;
        }
}

// Hadamard butterflies (ascending half-width, (a, b) -> (a + b, a - b)) over
// n consecutive elements of v, in fp32: half-width 1 scalar, >= 2 packed x2.
template <int N>
__device__ __forceinline__ void fwht(float* v) {
#pragma unroll
    for (int j = 0; j < N; j += 2) {
        const float a = v[j], b = v[j + 1];
        v[j] = __fadd_rn(a, b);
        v[j + 1] = __fsub_rn(a, b);
    }
    fwht_stage<N, 2>(v);
    fwht_stage<N, 4>(v);
    fwht_stage<N, 8>(v);
    if constexpr (N == 32) fwht_stage<N, 16>(v);
}

// max(m, |H D x|) over G elements in groups of NH (no 1/sqrt(n_h)): the
// butterflies but the last, whose two outputs only enter the maximum; of
// RN(a + b) and RN(a - b) the larger magnitude is RN(|a| + |b|) (one exact
// value has magnitude |a| + |b|, the other at most that, and rounding is
// monotone and symmetric).
template <int NH, int G>
__device__ __forceinline__ float rot_abs_max(float m, float* v) {
    if constexpr (NH == 0) {
        return abs_max<G>(m, v);
    } else {
#pragma unroll
        for (int hb = 0; hb < G / NH; ++hb) {
            float* w = v + hb * NH;
#pragma unroll
            for (int j = 0; j < NH; j += 2) {
                const float a = w[j], b = w[j + 1];
                w[j] = __fadd_rn(a, b);
                w[j + 1] = __fsub_rn(a, b);
            }
            fwht_stage<NH, 2>(w);
            if constexpr (NH >= 16) fwht_stage<NH, 4>(w);
            if constexpr (NH == 32) fwht_stage<NH, 8>(w);
            float m1 = 0.0f;
#pragma unroll
            for (int j = 0; j < NH / 2; j += 2) {
                m = fmaxf(m, __fadd_rn(fabsf(w[j]), fabsf(w[j + NH / 2])));
                m1 = fmaxf(m1, __fadd_rn(fabsf(w[j + 1]), fabsf(w[j + 1 + NH / 2])));
            }
            m = fmaxf(m, m1);
        }
        return m;
    }
}

// One stride of the halving tree: s[j] += s[j + ST] for j < ST.
template <int ST>
__device__ __forceinline__ void tree_stage(float* s) {
#pragma unroll
    for (int j = 0; j < ST; ++j) s[j] = __fadd_rn(s[j], s[j + ST]);
}

// Halving-stride tree sum of N = 8 or 16 fp32 terms (s[j] += s[j + stride],
// stride N/2 .. 1).
template <int N>
__device__ __forceinline__ float tree_sum(float* s) {
    if constexpr (N == 16) tree_stage<8>(s);
    tree_stage<4>(s);
    tree_stage<2>(s);
    return __fadd_rn(s[0], s[1]);
}

// First stride of <a, b> over a block of NB terms in the halving-stride
// order: a[j] b[j] fused onto the rounded a[j + NB/2] b[j + NB/2] (one
// multiply-add); tree_sum<NB/2> of these gives the dot product.
__device__ __forceinline__ float dot_first(float a0, float b0, float a1, float b1) {
    return __fmaf_rn(a0, b0, __fmul_rn(a1, b1));
}

// E2M1 pair (one byte) -> two fp32 values (exact through f16).
__device__ __forceinline__ float2 e2m1x2_decode(uint32_t byte) {
    uint32_t h2;
    const uint16_t b = (uint16_t)byte;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u16 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h2) : "h"(b));
    return __half22float2(*reinterpret_cast<__half2*>(&h2));
}

// s_enc = 2688 / amax (clamped to the largest finite fp32), g = amax / 2688
// (both 1 when amax = 0); g written by thread 0 when write_g.
__device__ __forceinline__ float nvfp4_scale_from_amax(float amax, float* tensor_scale, bool write_g) {
    float s_enc = 1.0f, g = 1.0f;
    if (amax > 0.0f) {
        s_enc = __fdiv_rn(2688.0f, amax);
        if (s_enc > 3.402823466e38f) s_enc = 3.402823466e38f;
        g = __fdiv_rn(amax, 2688.0f);
    }
    if (write_g && threadIdx.x == 0) *tensor_scale = g;
    return s_enc;
}

// Barrier of the compute warps only (named barrier 1): the producer warp has
// gone ahead to issue the first loads while they set up the scales.
__device__ __forceinline__ void bar_compute() {
    asm volatile("bar.sync 1, %0;" ::"r"(kComputeWarps * 32) : "memory");
}

// Reduce the CTA's amax partials (NVFP4) to s_enc; CTA 0 writes g. Run by the
// compute warps (threads 0 .. 255).
__device__ float nvfp4_encode_scale(const QuantParams& p, float* red_smem, bool write_g) {
    float amax = 0.0f;
    if (p.amax_in != nullptr) {
        amax = __ldg(p.amax_in);
    } else {
        float m = 0.0f;
        // coherent loads: in the fused pass the partials were written by the
        // other CTAs of this launch
        for (int i = threadIdx.x; i < p.n_partials; i += kComputeWarps * 32) m = fmaxf(m, __ldcg(p.amax_partials + i));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((threadIdx.x & 31) == 0) red_smem[threadIdx.x >> 5] = m;
        bar_compute();
        if (threadIdx.x < 32) {
            m = threadIdx.x < kComputeWarps ? red_smem[threadIdx.x] : 0.0f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (threadIdx.x == 0) red_smem[32] = m;
        }
        bar_compute();
        amax = red_smem[32];
    }
    return nvfp4_scale_from_amax(amax, p.tensor_scale, write_g);
}

// rtab[c] = s_enc / S(c) for every E4M3 code c the saturating conversion can
// produce (1-126; S(0) = 0 gives 0), the same divisions as per block, once per
// CTA, by the compute warps. Ends with their barrier.
__device__ void fill_rtab(float* rtab, float s_enc) {
    for (int c = threadIdx.x; c < 128; c += kComputeWarps * 32)
        rtab[c] = (c == 0 || c == 127) ? 0.0f : __fdiv_rn(s_enc, e4m3_decode((uint32_t)c));
    bar_compute();
}

// The random streams and MXFP4 exponent rule of one orientation (what the
// per-group quantization reads besides the values).
struct Stream {
    uint64_t seed;
    uint32_t tag_elem;   // element SR: kTagElement | stream << 4
    uint32_t tag_scale;  // Quartet II scale SR: kTagScale | stream << 4
    uint32_t mx_round_up;
};
__device__ __forceinline__ Stream col_stream(const QuantParams& p) {
    return Stream{p.sr_seed, p.sr_tag_elem, p.sr_tag_scale, p.mx_round_up};
}
__device__ __forceinline__ Stream row_stream(const QuantParams& p) {
    return Stream{p.sr_seed_row, p.sr_tag_elem_row, p.sr_tag_scale_row, p.mx_round_up};
}

// The four Quartet II scale uniforms of one Philox quad, computed once per quad.
struct ScaleRng {
    uint64_t quad = ~0ull;
    uint4 w;
    // Philox word of the block (its uniform is (word >> 8) * 2^-24).
    __device__ __forceinline__ uint32_t word(const Stream& p, uint64_t block_index) {
        const uint64_t q = block_index >> 2;
        if (q != quad) {
            w = philox_quad(p.seed, p.tag_scale, q);
            quad = q;
        }
        const uint32_t i = (uint32_t)(block_index & 3);
        return i == 0 ? w.x : i == 1 ? w.y : i == 2 ? w.z : w.w;
    }
};

// ---------------------------------------------------------------------------
// One group of G consecutive elements of the quantized axis, in registers.
//   v          : the G values (bf16 widened to fp32), consumed
//   elem0      : index (row * k + j) of v[0] in the quantized orientation
//   block0     : block index of v[0]
//   codes      : G/8 words of packed E2M1 codes (element 0 lowest)
//   scodes     : G/NB scale codes
template <int FMT, int RND, int NH>
struct Group {
    static constexpr int NB = (FMT == kNvfp4) ? 16 : 32;
    static constexpr int G = (NH > NB) ? NH : NB;

    // Sign-flip mask of packed bf16 word i of a group (elements 2i, 2i+1 at
    // bits 15 and 31): the random Hadamard's D applied before widening.
    __device__ __forceinline__ static uint32_t sign_mask(uint32_t signs, int i) {
        const int e = (2 * i) % (NH > 0 ? NH : 32);
        return ((signs >> e) & 1u) << 15 | ((signs >> (e + 1)) & 1u) << 31;
    }

    // v = c * H * (D x) per n_h chunk; D was applied to the packed words.
    // SCALE = false leaves out the factor c (the amax pass applies it once to
    // the maximum: rounding c * y is monotone in y).
    template <bool SCALE = true>
    __device__ __forceinline__ static void rotate(float* v) {
        if constexpr (NH > 0) {
#pragma unroll
            for (int hb = 0; hb < G / NH; ++hb) {
                float* w = v + hb * NH;
                fwht<NH>(w);
                if constexpr (SCALE) {
#pragma unroll
                    for (int e = 0; e < NH; e += 2) {
                        const float2 r = __fmul2_rn(f2(w[e], w[e + 1]), f2(had_norm<NH>(), had_norm<NH>()));
                        w[e] = r.x; w[e + 1] = r.y;
                    }
                }
            }
        }
    }

    // rtab[c] = s_enc / (E4M3 value of c) for codes 1-126, 0 for code 0.
    __device__ __forceinline__ static void quantize(float* v, float s_enc, const float* rtab, const Stream& p,
                                                    uint64_t elem0, uint64_t block0, ScaleRng& srng,
                                                    uint32_t* codes, uint32_t* scodes) {
#pragma unroll
        for (int b = 0; b < G / NB; ++b) {
            float* vb = v + b * NB;
            // block scale from the block amax
            const float am = abs_max<NB>(0.0f, vb);
            float rmul, S;
            uint32_t scode;
            if constexpr (FMT == kNvfp4) {
                const float d = div6(am);
                const float t = __fmul_rn(d, s_enc);
                scode = e4m3_rn(t);  // saturating: codes 0-126
                S = e4m3_decode(scode);
                rmul = rtab[scode];
            } else {
                if (am == 0.0f) {
                    scode = 0u;
                    S = exp2i(-127);
                    rmul = 0.0f;
                } else {
                    const int e = floor_log2(am);
                    int E = e - 2;
                    if (p.mx_round_up) {
                        // the smallest E with am <= 6 * 2^E: one more when
                        // am > 1.5 * 2^e, i.e. 2 (am - 2^e) > 2^e (both exact)
                        const float lo = exp2i(e);
                        if (__fmul_rn(2.0f, __fsub_rn(am, lo)) > lo) ++E;
                    }
                    E = E < -127 ? -127 : (E > 127 ? 127 : E);
                    scode = (uint32_t)(E + 127);
                    S = exp2i(E);
                    rmul = exp2i(-E);
                }
            }
            // scaled values
#pragma unroll
            for (int e = 0; e < NB; e += 2) {
                const float2 r = __fmul2_rn(f2(vb[e], vb[e + 1]), f2(rmul, rmul));
                vb[e] = r.x; vb[e + 1] = r.y;
            }
            // element rounding
            uint32_t* cb = codes + b * (NB / 8);
            if constexpr (RND == kSr) {
                // 16-bit uniforms, two per word: element j = i0 + e takes half
                // j % 2 of word j / 2 of the element stream, i.e. of word
                // (e / 2) % 4 of the Philox quad (i0 + e) / 8 (i0 is a
                // multiple of 16)
                const uint64_t i0 = elem0 + (uint64_t)(b * NB);
#pragma unroll
                for (int e8 = 0; e8 < NB; e8 += 8) {
                    const uint4 w = philox_quad(p.seed, p.tag_elem, (i0 + e8) >> 3);
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        vb[e8 + 2 * h] = e2m1_sr_value(vb[e8 + 2 * h], ws[h] << 16);
                        vb[e8 + 2 * h + 1] = e2m1_sr_value(vb[e8 + 2 * h + 1], ws[h] & 0xFFFF0000u);
                    }
                }
            }
#pragma unroll
            for (int e8 = 0; e8 < NB; e8 += 8) cb[e8 / 8] = e2m1x8_rn(vb + e8);
            if constexpr (RND == kQuartet2) {
                // alpha = <u, u> / <u, q>, each sum's first stride by
                // dot_first on element pairs (j, j + NB/2), then the tree
                constexpr int H = NB / 2;
                float sa[H], sb[H];
#pragma unroll
                for (int j = 0; j < H; j += 2) {
                    const float2 q0 = e2m1x2_decode((cb[j / 8] >> (4 * (j & 7))) & 0xFFu);
                    const float2 q1 = e2m1x2_decode((cb[(j + H) / 8] >> (4 * ((j + H) & 7))) & 0xFFu);
                    sa[j] = dot_first(vb[j], vb[j], vb[j + H], vb[j + H]);
                    sa[j + 1] = dot_first(vb[j + 1], vb[j + 1], vb[j + H + 1], vb[j + H + 1]);
                    sb[j] = dot_first(vb[j], q0.x, vb[j + H], q1.x);
                    sb[j + 1] = dot_first(vb[j + 1], q0.y, vb[j + H + 1], q1.y);
                }
                const float num = tree_sum<H>(sa);
                const float den = tree_sum<H>(sb);
                const float alpha = (den == 0.0f) ? 1.0f : __fdiv_rn(num, den);
                const float t = __fmul_rn(S, alpha);
                const uint32_t rw = srng.word(p, block0 + b);
                if constexpr (FMT == kNvfp4)
                    scode = e4m3_sr(t, rw);
                else
                    scode = e8m0_sr(t, uniform24(rw));
            }
            scodes[b] = scode;
        }
    }
};

// Extents of the output buffers (bytes), for the bounds-checked build.
__device__ __forceinline__ int64_t codes_extent(const QuantParams& p) { return p.rows * (p.k / 2); }
__device__ __forceinline__ int64_t scales_extent(const QuantParams& p) {
    return (p.rows + 127) / 128 * (p.kb4 / 4) * 512;
}
__device__ __forceinline__ int64_t codes_row_extent(const QuantParams& p) { return p.R * (p.C / 2); }
__device__ __forceinline__ int64_t scales_row_extent(const QuantParams& p) {
    return (p.R + 127) / 128 * (p.kb4_row / 4) * 512;
}

// 32 bytes of codes (64 elements of one row): two 16-byte stores, or four
// 8-byte ones when the row length in bytes (k / 2) is not a multiple of 16
// (k a multiple of 16 but not of 32: rows start 8-byte aligned).
__device__ __forceinline__ void store_codes32(uint8_t* dst, const uint32_t* codes, bool aligned16, const void* base,
                                              int64_t extent) {
    if (aligned16) {
        *chk(reinterpret_cast<uint4*>(dst), base, extent) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
        *chk(reinterpret_cast<uint4*>(dst) + 1, base, extent) = make_uint4(codes[4], codes[5], codes[6], codes[7]);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *chk(reinterpret_cast<uint2*>(dst) + i, base, extent) = make_uint2(codes[2 * i], codes[2 * i + 1]);
    }
}

// ===========================================================================
// NVFP4 unit of 64 elements with two blocks per packed lane pair
// ===========================================================================
// The row and band-column kernels give each thread 64 consecutive elements of
// the quantized axis: four NVFP4 blocks. For NVFP4 with no Hadamard or a
// 16-point one, they are processed as two pairs (blocks 0 and 1, then 2 and 3)
// whose blocks sit in the .x and .y lanes of every packed f32x2 value:
// P[j] = (v_{2bp}[j], v_{2bp+1}[j]). All four Hadamard stages, the
// normalisation, the scale product and the Quartet II sums are then one packed
// instruction per pair of lanes, without data movement between lanes, and each
// lane performs exactly its own block's fp32 operations in the stated order.

// bf16 -> fp32 of the low / high element of a packed word, with its sign flip
// m (0 or 0x80000000): low = w * 2^16 + m (adding 2^31 modulo 2^32 flips bit
// 31), high = (w & 0xFFFF0000) ^ m.
__device__ __forceinline__ float bf16lo_flip(uint32_t w, uint32_t m) { return __uint_as_float(w * 65536u + m); }
__device__ __forceinline__ float bf16hi_flip(uint32_t w, uint32_t m) { return __uint_as_float((w & 0xFFFF0000u) ^ m); }

// A zero magnitude keeps code 0 whatever its sign (no -0 codes): per nibble,
// mag + 7 has bit 3 set iff mag >= 1 (no carry leaves a nibble).
__device__ __forceinline__ uint32_t e2m1_clear_neg_zero(uint32_t out) {
    const uint32_t mag = out & 0x77777777u;
    return out & ((mag + 0x77777777u) | 0x77777777u);
}

// Round-to-nearest-even E2M1 codes of eight values (element 0 in the low
// nibble), saturating at +-6.
__device__ __forceinline__ uint32_t e2m1x8_words(float a0, float a1, float a2, float a3, float a4, float a5, float a6,
                                                 float a7) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(a0), "f"(a1), "f"(a2), "f"(a3), "f"(a4), "f"(a5), "f"(a6), "f"(a7));
    return e2m1_clear_neg_zero(out);
}

// The same, also returning the eight code values as f16 pairs (h[i]: elements
// 2i, 2i + 1), decoded from the code bytes before the zero-sign clean-up: a -0
// code decodes to -0, which changes no sum it enters.
__device__ __forceinline__ uint32_t e2m1x8_words_dec(float a0, float a1, float a2, float a3, float a4, float a5,
                                                     float a6, float a7, uint32_t* h) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %8, %7;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %10, %9;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %12, %11;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %4, b3;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out), "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "f"(a0), "f"(a1), "f"(a2), "f"(a3), "f"(a4), "f"(a5), "f"(a6), "f"(a7));
    return e2m1_clear_neg_zero(out);
}

// E4M3 codes (round to nearest even, saturating at 448) of both lanes: the low
// byte is lane .x's, the next byte lane .y's.
__device__ __forceinline__ uint32_t e4m3x2_rn(float2 t) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(t.y), "f"(t.x));
    return r;
}

// x / 6 correctly rounded in both lanes: the packed form of div6 (one product
// with RN(1/6), one fused correction) when both lanes are in [2^-125,
// FLT_MAX], else div6 per lane.
__device__ __forceinline__ float2 div6x2(float2 x) {
    if (fminf(x.x, x.y) >= 0x1p-125f && fmaxf(x.x, x.y) <= 0x1.fffffep127f) {
        constexpr float C = 1.0f / 6.0f;
        const float2 q = __fmul2_rn(x, f2(C, C));
        const float2 r = __ffma2_rn(q, f2(-6.0f, -6.0f), x);
        return __ffma2_rn(r, f2(C, C), q);
    }
    return f2(div6(x.x), div6(x.y));
}

// Largest magnitude of each lane over the 16 packed elements of a pair: a tree
// of three-input maxima (depth 3; the maximum does not depend on the order).
__device__ __forceinline__ float2 abs_max_pair(const float2* P) {
    float x[5], y[5];
#pragma unroll
    for (int i = 0; i < 5; ++i) {
        x[i] = max3(fabsf(P[3 * i].x), fabsf(P[3 * i + 1].x), fabsf(P[3 * i + 2].x));
        y[i] = max3(fabsf(P[3 * i].y), fabsf(P[3 * i + 1].y), fabsf(P[3 * i + 2].y));
    }
    return f2(fmaxf(max3(x[0], x[1], x[2]), max3(x[3], x[4], fabsf(P[15].x))),
              fmaxf(max3(y[0], y[1], y[2]), max3(y[3], y[4], fabsf(P[15].y))));
}

// One butterfly stage of half-width H over the 16 packed elements of a pair.
template <int H>
__device__ __forceinline__ void fwht_pair_stage(float2* P) {
#pragma unroll
    for (int j0 = 0; j0 < 16; j0 += 2 * H)
#pragma unroll
        for (int j = j0; j < j0 + H; ++j) {
            const float2 a = P[j], b = P[j + H];
            P[j] = __fadd2_rn(a, b);
            P[j + H] = __fadd2_rn(a, neg2(b));
        }
}

// dot_tree of the 16 terms of each lane of a pair (two blocks at once): the
// first stride as packed multiply-adds onto packed products, the tree over
// the 8 partial sums as packed sums.
__device__ __forceinline__ float2 dot_tree_pair(const float2* a, const float2* b) {
    float2 s[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j] = __ffma2_rn(a[j], b[j], __fmul2_rn(a[j + 8], b[j + 8]));
#pragma unroll
    for (int st = 4; st >= 1; st >>= 1)
#pragma unroll
        for (int j = 0; j < st; ++j) s[j] = __fadd2_rn(s[j], s[j + st]);
    return s[0];
}

// Per-CTA table of (s_enc / S, S) for every E4M3 code S can take (1-126; code
// 0 gives (0, 0)), the same divisions as per block, by the compute warps. Ends
// with their barrier.
__device__ void fill_tab2(float2* tab, float s_enc) {
    for (int c = threadIdx.x; c < 128; c += kComputeWarps * 32) {
        const float S = e4m3_decode((uint32_t)c);
        tab[c] = (c == 0 || c == 127) ? f2(0.0f, 0.0f) : f2(__fdiv_rn(s_enc, S), S);
    }
    bar_compute();
}

// Hadamard sign flips of the 8 words of a block, at bit 31 of each element:
// lo[i] for element 2i, hi[i] for element 2i + 1.
struct SignFlips {
    uint32_t lo[8], hi[8];
    __device__ __forceinline__ explicit SignFlips(uint32_t signs) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            lo[i] = ((signs >> (2 * i)) & 1u) << 31;
            hi[i] = ((signs >> (2 * i + 1)) & 1u) << 31;
        }
    }
};

// Word i (0-3) of a Philox quad.
__device__ __forceinline__ uint32_t quad_word(uint4 q, uint32_t i) {
    return i == 0 ? q.x : i == 1 ? q.y : i == 2 ? q.z : q.w;
}

// Quantize one 64-element NVFP4 unit. load(c) returns chunk c (elements 8c ..
// 8c + 7 as four packed bf16 words, element 2i of the chunk in the low half
// of word i). elem0: index of element 0 in the quantized orientation (a
// multiple of 16); block0: its block index. Writes the 8 code words and
// returns the scale word (block b's E4M3 code in byte b).
template <int RND, int NH, typename Load>
__device__ __forceinline__ uint32_t nv64_quantize(Load load, const SignFlips& sf, float s_enc, const float2* tab,
                                                  const Stream& st, uint64_t elem0, uint64_t block0, uint32_t* codes) {
    static_assert(NH == 0 || NH == 16, "the packed unit takes no Hadamard or a 16-point one");
    static_assert(RND != kSr, "per-element SR stays on the group path");
    uint32_t scw = 0;
    uint4 rq = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (RND == kQuartet2) {
        // the scale words of the four blocks: one Philox quad when block0 is a
        // multiple of 4, else one per block below
        if ((block0 & 3u) == 0) rq = philox_quad(st.seed, st.tag_scale, block0 >> 2);
    }
#pragma unroll
    for (int bp = 0; bp < 2; ++bp) {
        float2 P[16];
        // blocks 2bp (chunks 4bp, 4bp + 1) and 2bp + 1 (chunks 4bp + 2, 4bp + 3)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint4 a = load(4 * bp + c), b = load(4 * bp + 2 + c);
            const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int wi = 4 * c + i;  // word of the block
                if constexpr (NH > 0) {
                    P[2 * wi] = f2(bf16lo_flip(wa[i], sf.lo[wi]), bf16lo_flip(wb[i], sf.lo[wi]));
                    P[2 * wi + 1] = f2(bf16hi_flip(wa[i], sf.hi[wi]), bf16hi_flip(wb[i], sf.hi[wi]));
                } else {
                    P[2 * wi] = f2(bf16lo(wa[i]), bf16lo(wb[i]));
                    P[2 * wi + 1] = f2(bf16hi(wa[i]), bf16hi(wb[i]));
                }
            }
        }
        if constexpr (NH == 16) {
            fwht_pair_stage<1>(P);
            fwht_pair_stage<2>(P);
            fwht_pair_stage<4>(P);
            fwht_pair_stage<8>(P);
#pragma unroll
            for (int j = 0; j < 16; ++j) P[j] = __fmul2_rn(P[j], f2(0.25f, 0.25f));  // fp32(1/sqrt(16))
        }
        // block scales from the block amaxes
        const float2 t = __fmul2_rn(div6x2(abs_max_pair(P)), f2(s_enc, s_enc));
        const uint32_t sc2 = e4m3x2_rn(t);  // block 2bp in the low byte
        // t >= 0 gives codes 0-126 (0x7F only for a NaN amax): the mask only
        // keeps the table index in range
        const float2 e0 = tab[sc2 & 0x7Fu], e1 = tab[(sc2 >> 8) & 0x7Fu];
        const float2 rr = f2(e0.x, e1.x);
#pragma unroll
        for (int j = 0; j < 16; ++j) P[j] = __fmul2_rn(P[j], rr);
        uint32_t* cw = codes + 4 * bp;  // block 2bp: cw[0..1], block 2bp + 1: cw[2..3]
        if constexpr (RND != kQuartet2) {
            cw[0] = e2m1x8_words(P[0].x, P[1].x, P[2].x, P[3].x, P[4].x, P[5].x, P[6].x, P[7].x);
            cw[1] = e2m1x8_words(P[8].x, P[9].x, P[10].x, P[11].x, P[12].x, P[13].x, P[14].x, P[15].x);
            cw[2] = e2m1x8_words(P[0].y, P[1].y, P[2].y, P[3].y, P[4].y, P[5].y, P[6].y, P[7].y);
            cw[3] = e2m1x8_words(P[8].y, P[9].y, P[10].y, P[11].y, P[12].y, P[13].y, P[14].y, P[15].y);
            scw |= sc2 << (16 * bp);
        } else {
            // RTN codes and their values q; alpha = <u, u> / <u, q> per lane
            uint32_t h[4][4];
            cw[0] = e2m1x8_words_dec(P[0].x, P[1].x, P[2].x, P[3].x, P[4].x, P[5].x, P[6].x, P[7].x, h[0]);
            cw[1] = e2m1x8_words_dec(P[8].x, P[9].x, P[10].x, P[11].x, P[12].x, P[13].x, P[14].x, P[15].x, h[1]);
            cw[2] = e2m1x8_words_dec(P[0].y, P[1].y, P[2].y, P[3].y, P[4].y, P[5].y, P[6].y, P[7].y, h[2]);
            cw[3] = e2m1x8_words_dec(P[8].y, P[9].y, P[10].y, P[11].y, P[12].y, P[13].y, P[14].y, P[15].y, h[3]);
            float2 Q[16];
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
                const float2 qx = __half22float2(*reinterpret_cast<const __half2*>(&h[j / 8][(j % 8) / 2]));
                const float2 qy = __half22float2(*reinterpret_cast<const __half2*>(&h[2 + j / 8][(j % 8) / 2]));
                Q[j] = f2(qx.x, qy.x);
                Q[j + 1] = f2(qx.y, qy.y);
            }
            const float2 num = dot_tree_pair(P, P), den = dot_tree_pair(P, Q);
            const float a0 = (den.x == 0.0f) ? 1.0f : __fdiv_rn(num.x, den.x);
            const float a1 = (den.y == 0.0f) ? 1.0f : __fdiv_rn(num.y, den.y);
            const float2 ts = __fmul2_rn(f2(e0.y, e1.y), f2(a0, a1));
            uint32_t w0, w1;
            if ((block0 & 3u) == 0) {
                w0 = bp ? rq.z : rq.x;
                w1 = bp ? rq.w : rq.y;
            } else {
                const uint64_t b0 = block0 + (uint64_t)(2 * bp), b1 = b0 + 1;
                w0 = quad_word(philox_quad(st.seed, st.tag_scale, b0 >> 2), (uint32_t)b0 & 3u);
                w1 = quad_word(philox_quad(st.seed, st.tag_scale, b1 >> 2), (uint32_t)b1 & 3u);
            }
            scw |= (e4m3_sr(ts.x, w0) | (e4m3_sr(ts.y, w1) << 8)) << (16 * bp);
        }
        // The next pair's loads (volatile) stay after this pair's codes: it
        // bounds the live values to one pair (no spills at 96 registers).
        asm volatile("" ::"r"(cw[0]), "r"(cw[1]), "r"(cw[2]), "r"(cw[3]));
    }
    return scw;
}

// max |H D x| (no 1/sqrt(n_h)) of a 64-element unit loaded by chunks.
template <int NH, typename Load>
__device__ __forceinline__ float rot_amax64(Load load, const SignFlips& sf, float m) {
#pragma unroll
    for (int bp = 0; bp < 2; ++bp) {
        float2 P[16];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint4 a = load(4 * bp + c), b = load(4 * bp + 2 + c);
            const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int wi = 4 * c + i;
                if constexpr (NH > 0) {
                    P[2 * wi] = f2(bf16lo_flip(wa[i], sf.lo[wi]), bf16lo_flip(wb[i], sf.lo[wi]));
                    P[2 * wi + 1] = f2(bf16hi_flip(wa[i], sf.hi[wi]), bf16hi_flip(wb[i], sf.hi[wi]));
                } else {
                    P[2 * wi] = f2(bf16lo(wa[i]), bf16lo(wb[i]));
                    P[2 * wi + 1] = f2(bf16hi(wa[i]), bf16hi(wb[i]));
                }
            }
        }
        if constexpr (NH == 16) {
            fwht_pair_stage<1>(P);
            fwht_pair_stage<2>(P);
            fwht_pair_stage<4>(P);
            // The last stage (half-width 8) only feeds the maximum: of RN(a + b)
            // and RN(a - b) the larger magnitude is RN(|a| + |b|) (one of the two
            // exact values has magnitude |a| + |b|, the other at most that, and
            // rounding is monotone and symmetric), so one scalar sum per pair of
            // outputs replaces the two packed ones, and half as many values
            // enter the maximum.
            float m1 = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
                m = max3(m, __fadd_rn(fabsf(P[j].x), fabsf(P[j + 8].x)), __fadd_rn(fabsf(P[j].y), fabsf(P[j + 8].y)));
                m1 = max3(m1, __fadd_rn(fabsf(P[j + 1].x), fabsf(P[j + 9].x)),
                          __fadd_rn(fabsf(P[j + 1].y), fabsf(P[j + 9].y)));
            }
            m = fmaxf(m, m1);
        } else {
            const float2 am = abs_max_pair(P);
            m = max3(m, am.x, am.y);
        }
    }
    return m;
}

// This CTA's tiles of a tiles_r x tiles_c grid (blockIdx.x, + gridDim.x, ...)
// as (tr, tc), advanced without divisions, with the TMA ring stage and phase
// of each.
template <int STAGES>
struct TileWalk {
    int tr, tc, tiles_c, step_r, step_c, stage = 0;
    uint32_t phase = 0;
    // issued: ring iterations this CTA has already used (a second pass over
    // the same tiles continues the ring where the first one left it)
    __device__ __forceinline__ explicit TileWalk(int tiles_c_, int issued = 0) : tiles_c(tiles_c_) {
        tr = (int)blockIdx.x / tiles_c;
        tc = (int)blockIdx.x % tiles_c;
        step_r = (int)gridDim.x / tiles_c;
        step_c = (int)gridDim.x % tiles_c;
        stage = issued % STAGES;
        phase = (uint32_t)((issued / STAGES) & 1);
    }
    __device__ __forceinline__ void next() {
        tc += step_c;
        tr += step_r;
        if (tc >= tiles_c) {
            tc -= tiles_c;
            ++tr;
        }
        if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
        }
    }
};

// Ring of TMA stages: full[s] completes when the tile landed, empty[s] when all
// compute warps finished with it.
template <int STAGES>
struct Ring {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
};

template <int STAGES>
__device__ __forceinline__ void ring_init(Ring<STAGES>& ring) {
    for (int s = 0; s < STAGES; ++s) {
        mbar_init(&ring.full[s], 1);
        mbar_init(&ring.empty[s], kComputeWarps);
    }
    fence_mbarrier_init();
}

// CTA-wide max over the compute warps' values; thread 0 writes the partial.
__device__ __forceinline__ void write_partial(float m, float* red, float* out) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    asm volatile("bar.sync 1, %0;" ::"r"(kComputeWarps * 32));
    if (threadIdx.x == 0) {
        float r = 0.0f;
        for (int w = 0; w < kComputeWarps; ++w) r = fmaxf(r, red[w]);
        *chk(out + blockIdx.x, out, (int64_t)kMaxAmaxPartials * 4) = r;
    }
}

// Grid-wide barrier of a cooperative launch, by one thread of each CTA: the
// CTA's earlier global writes are published (fence, then one arrival on the
// counter, which the caller zeroed before the launch) and the thread waits,
// bounded, until every CTA has arrived. False (and the device error word set)
// if the wait gave up.
__device__ __forceinline__ bool grid_arrive_and_wait(uint32_t* counter) {
    __threadfence();
    atomicAdd(counter, 1u);
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
        if (v >= gridDim.x) break;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            raise_device_error(DEV_ERR_TIMEOUT);
            return false;
        }
        __nanosleep(64);
    }
    __threadfence();
    return true;
}

// Fused NVFP4 amax (first pass of a two-pass kernel, packed unit): every tile
// of this CTA rotated and its maximum taken; the CTA's partial (times
// 1/sqrt(n_h)) written to p.amax_out[blockIdx.x]; after the grid barrier the
// tensor scale is set up from all partials exactly as the separate amax pass
// and quantizer would (max over the partials, s_enc, g). Returns the ring
// iterations used.
template <int NH, int STAGES, typename LoadAt>
__device__ int fused_amax_pass(const QuantParams& p, Ring<STAGES>& ring, int tiles_c, int tiles_r, float* red,
                               LoadAt load_at) {
    const SignFlips sf(NH > 0 ? p.signs : 0u);
    float m = 0.0f;
    for (TileWalk<STAGES> w(tiles_c); w.tr < tiles_r; w.next()) {
        const int s = w.stage;
        if (!mbar_wait(&ring.full[s], w.phase)) break;
        m = rot_amax64<NH>([&](int c) { return load_at(s, c); }, sf, m);
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(&ring.empty[s]);
    }
    if constexpr (NH > 0) m = __fmul_rn(m, had_norm<NH>());  // c * max |y| = max |c * y|
    write_partial(m, red, p.amax_out);
    if (threadIdx.x == 0) (void)grid_arrive_and_wait(p.grid_counter);
    bar_compute();
    // this CTA's tiles (blockIdx.x, + gridDim.x, ...): the second pass starts
    // the ring there even if a wait above gave up early
    const int64_t total = (int64_t)tiles_c * tiles_r;
    return total > (int64_t)blockIdx.x ? (int)((total - blockIdx.x + gridDim.x - 1) / gridDim.x) : 0;
}

// Occupancy of the persistent quantizers: two CTAs per SM with a 3-stage ring
// (the memory-bound modes need the deeper ring), or three CTAs per SM with a
// 2-stage ring (at most 75 registers) for NVFP4 with per-element SR or Quartet
// II, which are bound by instruction issue and gain from the extra warps
// (measured on the 940 MB dY: Quartet II rows 1-3 %, SR rows 4 % faster; RTN
// rows 6 % slower with the shallower ring).
template <int STAGES>
constexpr int kCtasPerSm = STAGES == 2 ? 3 : 2;
template <int FMT, int RND>
constexpr bool issue_bound_mode() {
    return FMT == kNvfp4 && (RND == kSr || RND == kQuartet2);
}

// ===========================================================================
// Row mode
// ===========================================================================
// FUSED: an NVFP4 tensor that fits in L2 in one cooperative launch — a first
// pass over the tiles takes the rotated amax, a grid barrier, then the
// quantizing pass re-reads the tiles (from L2).
template <int FMT, int RND, int NH, bool AMAX_ONLY, int STAGES, bool FUSED = false>
__global__ void __launch_bounds__(kThreads, kCtasPerSm<STAGES>)
    quant_row_kernel(const __grid_constant__ CUtensorMap tmap, const QuantParams p) {
    using Grp = Group<FMT, RND, NH>;
    constexpr int NB = Grp::NB;
    constexpr int G = AMAX_ONLY ? ((NH > 16) ? NH : 16) : Grp::G;
    constexpr int STAGE_BYTES = kRowTileRows * kRowTileCols * 2;  // 32 KiB
    // NVFP4 with no Hadamard or a 16-point one, round-to-nearest or Quartet
    // II: the packed 64-element unit
    constexpr bool kPacked = FMT == kNvfp4 && (NH == 0 || NH == 16) && RND != kSr && !AMAX_ONLY;
    static_assert(!FUSED || kPacked, "the fused amax pass serves the packed NVFP4 unit");
    extern __shared__ __align__(1024) uint8_t dyn_smem[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    __shared__ Ring<STAGES> ring;
    __shared__ float red[33];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tiles_c = (int)((p.k + kRowTileCols - 1) / kRowTileCols);
    const int tiles_r = (int)((p.rows + kRowTileRows - 1) / kRowTileRows);

    if (tid == 0) {
        prefetch_tmap(&tmap);
        ring_init(ring);
    }
    __syncthreads();
    pdl_wait();  // the previous kernel's writes are visible (and its reads done)
    pdl_launch_dependents();

    if (warp == kComputeWarps) {
        // ---------------- producer ----------------
        if (lane == 0) {
            int i = 0;
            bool ok = true;
            for (int pass = 0; pass < (FUSED ? 2 : 1) && ok; ++pass)
                for (TileWalk<STAGES> w(tiles_c, i); w.tr < tiles_r; w.next(), ++i) {
                    const int s = w.stage;
                    if (i >= STAGES && !mbar_wait(&ring.empty[s], w.phase ^ 1u)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&ring.full[s], STAGE_BYTES);
                    tma_load_2d(tiles + s * STAGE_BYTES, &tmap, &ring.full[s], w.tc * kRowTileCols,
                                w.tr * kRowTileRows);
                }
            drain_loads(ring.full, nullptr, STAGES, i);  // no load lands after this CTA exits
        }
        return;
    }
    __shared__ float rtab[kPacked ? 1 : 128];
    __shared__ float2 tab2[kPacked ? 128 : 1];
    float s_enc = 1.0f;
    int issued = 0;  // ring iterations of the fused amax pass
    if constexpr (FUSED) {
        issued = fused_amax_pass<NH>(p, ring, tiles_c, tiles_r, red, [&](int st, int c) {
            return lds128((smem_u32(tiles) + (uint32_t)(st * STAGE_BYTES) + (uint32_t)tid * 128u +
                           ((uint32_t)(tid & 7) << 4)) ^ ((uint32_t)c << 4));
        });
    }
    if constexpr (!AMAX_ONLY && FMT == kNvfp4) {
        s_enc = nvfp4_encode_scale(p, red, blockIdx.x == 0);
        if constexpr (kPacked)
            fill_tab2(tab2, s_enc);
        else
            fill_rtab(rtab, s_enc);
    }
    if constexpr (!AMAX_ONLY && FMT == kMxfp4) {
        if (blockIdx.x == 0 && tid == 0) *p.tensor_scale = 1.0f;
    }

    // ---------------- compute: thread = one row of the tile ----------------
    const int64_t rows_pad = (p.rows + 127) / 128 * 128;
    float amax_acc = 0.0f;
    ScaleRng srng;
    // Tile-invariant per thread, held in registers: the swizzled 16-byte chunk
    // offsets of its row, the scale byte offset of its row within a 128-row
    // atom block (tiles start at multiples of 256 rows) and the Hadamard sign
    // masks (the per-element SR kernels too: timed 7-9 % faster with them
    // hoisted than recomputing them, with fewer spills).
    constexpr bool kHoist = true;
    uint32_t chunk_off[kPacked ? 1 : kRowTileCols / 8];
    if constexpr (!kPacked) {
#pragma unroll
        for (int c = 0; c < kRowTileCols / 8; ++c) chunk_off[c] = (uint32_t)(tid * 128 + ((c ^ (tid & 7)) << 4));
    }
    const int64_t atom_row_bytes = (p.kb4 / 4) * 512;  // one 128-row block of scale atoms
    const int64_t sc_row_off = (tid / 128) * atom_row_bytes + (tid % 32) * 16 + ((tid / 32) % 4) * 4;
    // the random Hadamard's sign-flip masks of the packed bf16 words of a group
    uint32_t smask[kPacked ? 1 : G / 2];
    if constexpr (!kPacked) {
#pragma unroll
        for (int i = 0; i < G / 2; ++i) smask[i] = Grp::sign_mask(p.signs, i);
    }
    const SignFlips sf(kPacked && NH > 0 ? p.signs : 0u);
    for (TileWalk<STAGES> w(tiles_c, issued); w.tr < tiles_r; w.next()) {
        const int s = w.stage;
        if (!mbar_wait(&ring.full[s], w.phase)) break;
        const int64_t row = (int64_t)w.tr * kRowTileRows + tid;
        const int64_t col0 = (int64_t)w.tc * kRowTileCols;
        const uint32_t sbase = smem_u32(tiles) + (uint32_t)(s * STAGE_BYTES) + (kHoist ? 0u : (uint32_t)tid * 128u);
        uint32_t codes[kRowTileCols / 8];
        uint32_t scodes[kRowTileCols / 16];
        uint32_t scw = 0;
        if constexpr (kPacked) {
            // chunk c of this thread's row: 16-byte chunk c ^ (tid % 8) of its 128-byte line
            const uint32_t rb = smem_u32(tiles) + (uint32_t)(s * STAGE_BYTES) + (uint32_t)tid * 128u +
                                ((uint32_t)(tid & 7) << 4);
            auto load = [&](int c) { return lds128(rb ^ ((uint32_t)c << 4)); };
            scw = nv64_quantize<RND, NH>(load, sf, s_enc, tab2, col_stream(p), (uint64_t)row * (uint64_t)p.k + (uint64_t)col0,
                                         (uint64_t)row * (uint64_t)(p.k / 16) + (uint64_t)(col0 / 16), codes);
        } else {
#pragma unroll
        for (int g = 0; g < kRowTileCols / G; ++g) {
            float v[G];
#pragma unroll
            for (int c8 = 0; c8 < G / 8; ++c8) {
                const int chunk = g * (G / 8) + c8;
                uint32_t w0, w1, w2, w3;
                const uint32_t addr = kHoist ? sbase + chunk_off[chunk] : sbase + ((chunk ^ (tid & 7)) << 4);
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
                             : "r"(addr));
                if (NH > 0 && p.signs != 0u) {
                    w0 ^= kHoist ? smask[4 * c8 + 0] : Grp::sign_mask(p.signs, 4 * c8 + 0);
                    w1 ^= kHoist ? smask[4 * c8 + 1] : Grp::sign_mask(p.signs, 4 * c8 + 1);
                    w2 ^= kHoist ? smask[4 * c8 + 2] : Grp::sign_mask(p.signs, 4 * c8 + 2);
                    w3 ^= kHoist ? smask[4 * c8 + 3] : Grp::sign_mask(p.signs, 4 * c8 + 3);
                }
                v[8 * c8 + 0] = bf16lo(w0); v[8 * c8 + 1] = bf16hi(w0);
                v[8 * c8 + 2] = bf16lo(w1); v[8 * c8 + 3] = bf16hi(w1);
                v[8 * c8 + 4] = bf16lo(w2); v[8 * c8 + 5] = bf16hi(w2);
                v[8 * c8 + 6] = bf16lo(w3); v[8 * c8 + 7] = bf16hi(w3);
            }
            if constexpr (AMAX_ONLY) {
                amax_acc = rot_abs_max<NH, G>(amax_acc, v);
            } else {
                Grp::rotate(v);
                const int64_t j0 = col0 + g * G;
                Grp::quantize(v, s_enc, rtab, col_stream(p), (uint64_t)row * (uint64_t)p.k + (uint64_t)j0,
                              (uint64_t)row * (uint64_t)(p.k / NB) + (uint64_t)(j0 / NB), srng,
                              codes + g * (G / 8), scodes + g * (G / NB));
            }
        }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ring.empty[s]);
        if constexpr (!AMAX_ONLY) {
            if (row < p.rows) {
                uint8_t* dst = p.codes + row * (p.k / 2) + col0 / 2;
                if (col0 + kRowTileCols <= p.k) {
                    store_codes32(dst, codes, ((p.k / 2) & 15) == 0, p.codes, codes_extent(p));
                } else {
#pragma unroll
                    for (int w = 0; w < 8; ++w)
                        if (col0 + 8 * w < p.k) *chk(reinterpret_cast<uint32_t*>(dst) + w, p.codes, codes_extent(p)) = codes[w];
                }
            }
            if (row < rows_pad) {
                // this row's 64 / NB scale bytes: a whole 4-byte atom word (NVFP4) or
                // half of one (MXFP4); past the last column tile the rest of the word
                // is padding and is written as zero.
                const int64_t kb0 = col0 / NB;
                const int64_t off =
                    kHoist ? (2 * (int64_t)w.tr) * atom_row_bytes + (kb0 / 4) * 512 + sc_row_off
                           : ((row / 128) * (p.kb4 / 4) + kb0 / 4) * 512 + (row % 32) * 16 + ((row / 32) % 4) * 4;
                if constexpr (NB == 16) {
                    if constexpr (kPacked)
                        *chk(reinterpret_cast<uint32_t*>(p.scales + off), p.scales, scales_extent(p)) = scw;
                    else
                        *chk(reinterpret_cast<uint32_t*>(p.scales + off), p.scales, scales_extent(p)) =
                            scodes[0] | (scodes[1] << 8) | (scodes[2] << 16) | (scodes[3] << 24);
                } else {
                    const uint32_t half = scodes[0] | (scodes[1] << 8);
                    if ((kb0 & 3) == 0 && col0 + kRowTileCols >= p.k)
                        *chk(reinterpret_cast<uint32_t*>(p.scales + off), p.scales, scales_extent(p)) = half;
                    else
                        *chk(reinterpret_cast<uint16_t*>(p.scales + off + (kb0 & 3)), p.scales, scales_extent(p)) =
                            (uint16_t)half;
                }
            }
        }
    }
    if constexpr (AMAX_ONLY) {
        if constexpr (NH > 0) amax_acc = __fmul_rn(amax_acc, had_norm<NH>());  // c * max |y| = max |c * y|
        write_partial(amax_acc, red, p.amax_out);
    }
}

// ===========================================================================
// Column mode (TMA + transposing ldmatrix)
// ===========================================================================
// Shared-memory row of x-row r within the tile (r = k + 2m + 8u + G q with
// k < 2, m < 4, u < G/8, q < 4): s = k + 2q + 8m + 32u. The 5-D tensor map
// (columns, k, r/G, m, u) delivers rows in this order, so the 8 rows one
// ldmatrix phase reads have s % 8 = k + 2q all distinct: with the 128-byte
// swizzle (16-byte chunk index XOR s % 8) they hit 8 different bank groups.
// Lane l of an ldmatrix.x4 supplies row l % 8 of matrix l / 8, i.e. smem row
// s = l + 32u; after the transposing load, lane (c = l / 4, q = l % 4) holds
// x-rows Gq + 8u + [0, 8) of column c.
template <int FMT, int RND, int NH, bool AMAX_ONLY, int STAGES, bool DUAL = false>
__global__ void __launch_bounds__(kThreads, 2)
    quant_col_kernel(const __grid_constant__ CUtensorMap tmap, const QuantParams p) {
    using Grp = Group<FMT, RND, NH>;
    constexpr int NB = Grp::NB;
    constexpr int G = AMAX_ONLY ? ((NH > 16) ? NH : 16) : Grp::G;
    constexpr int TILE_ROWS = 4 * G;
    constexpr int BOX_BYTES = TILE_ROWS * 64 * 2;
    constexpr int STAGE_BYTES = 2 * BOX_BYTES;
    extern __shared__ __align__(1024) uint8_t dyn_smem[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    __shared__ Ring<STAGES> ring;
    __shared__ float red[33];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tiles_c = (int)((p.rows + kColTileCols - 1) / kColTileCols);  // output rows = x columns
    const int tiles_r = (int)((p.k + TILE_ROWS - 1) / TILE_ROWS);

    if (tid == 0) {
        prefetch_tmap(&tmap);
        ring_init(ring);
    }
    __syncthreads();
    pdl_wait();  // the previous kernel's writes are visible (and its reads done)
    pdl_launch_dependents();

    if (warp == kComputeWarps) {
        if (lane == 0) {
            int i = 0;
            for (TileWalk<STAGES> w(tiles_c); w.tr < tiles_r; w.next(), ++i) {
                const int s = w.stage;
                if (i >= STAGES && !mbar_wait(&ring.empty[s], w.phase ^ 1u)) break;
                const int32_t c0 = w.tc * kColTileCols;
                const int32_t tr4 = 4 * w.tr;
                mbar_arrive_expect_tx(&ring.full[s], STAGE_BYTES);
                tma_load_5d(tiles + s * STAGE_BYTES, &tmap, &ring.full[s], (int32_t)c0, 0, tr4, 0, 0);
                tma_load_5d(tiles + s * STAGE_BYTES + BOX_BYTES, &tmap, &ring.full[s], (int32_t)(c0 + 64), 0, tr4, 0,
                            0);
            }
            drain_loads(ring.full, nullptr, STAGES, i);  // no load lands after this CTA exits
        }
        return;
    }
    __shared__ float rtab[128];
    float s_enc = 1.0f;
    if constexpr (!AMAX_ONLY && FMT == kNvfp4) {
        s_enc = nvfp4_encode_scale(p, red, blockIdx.x == 0);
        fill_rtab(rtab, s_enc);
    }
    if constexpr (!AMAX_ONLY && FMT == kMxfp4) {
        if (blockIdx.x == 0 && tid == 0) *p.tensor_scale = 1.0f;
    }

    const int64_t rows_pad = (p.rows + 127) / 128 * 128;
    const int q = lane & 3;
    float amax_acc = 0.0f, amax_row_acc = 0.0f;
    ScaleRng srng;
    // Quartet II with 16-element groups: the 4 lanes of a column hold the 4
    // blocks of one Philox quad (when k is a multiple of 64), and a warp needs
    // 16 quads per tile (2 chunks x 8 columns). Every other tile, lanes 0-15
    // compute this tile's quads and lanes 16-31 those of the CTA's next tile;
    // the 4 lanes that use a quad take its words by shuffles.
    constexpr bool kSharedQuads = (RND == kQuartet2 && !AMAX_ONLY && G == 16 && NB == 16);
    const bool shared_quads = kSharedQuads && (p.k % 64) == 0;
    uint4 lane_quad = make_uint4(0u, 0u, 0u, 0u);
    uint32_t quad_half = 0;  // 0: compute this and the next tile's quads; 1: use the next tile's
    // Tile-invariant per thread (chunk ci = 0, 1): the column within the tile
    // (tiles start at multiples of 128 columns), the ldmatrix offsets within a
    // stage, the scale byte offset within a 128-row atom block, and the code
    // row offset.
    int cc[2];
    uint32_t lm_off[2][G / 8];
    int64_t sc_off[2], code_off[2], blk_off[2];
#pragma unroll
    for (int ci = 0; ci < 2; ++ci) {
        const int chunk = 2 * warp + ci;  // 16 chunks of 8 columns
        const int box = chunk >> 3, ch = chunk & 7;
        cc[ci] = chunk * 8 + (lane >> 2);
#pragma unroll
        for (int u = 0; u < G / 8; ++u) {
            const int srow = lane + 32 * u;
            lm_off[ci][u] = (uint32_t)(box * BOX_BYTES + srow * 128 + ((ch ^ (srow & 7)) << 4));
        }
        sc_off[ci] = (cc[ci] % 32) * 16 + ((cc[ci] / 32) % 4) * 4;
        code_off[ci] = (int64_t)cc[ci] * (p.k / 2);
        blk_off[ci] = (int64_t)cc[ci] * (p.k / NB);
    }
    const int64_t atom_row_bytes = (p.kb4 / 4) * 512;  // one 128-row block of scale atoms
    uint32_t smask[G / 2];  // the random Hadamard's sign-flip masks of a group's packed words
#pragma unroll
    for (int i = 0; i < G / 2; ++i) smask[i] = Grp::sign_mask(p.signs, i);
    for (TileWalk<STAGES> w(tiles_c); w.tr < tiles_r; w.next()) {
        const int s = w.stage;
        if (!mbar_wait(&ring.full[s], w.phase)) break;
        const int64_t c0 = (int64_t)w.tc * kColTileCols;
        const int64_t r0 = (int64_t)w.tr * TILE_ROWS;
        const uint32_t stage_base = smem_u32(tiles) + (uint32_t)(s * STAGE_BYTES);
        if constexpr (kSharedQuads) {
            if (shared_quads && quad_half == 0) {
                int qtr = w.tr, qtc = w.tc;
                if (lane >= 16) {  // the next tile of this CTA's walk (TileWalk::next)
                    qtc += w.step_c;
                    qtr += w.step_r;
                    if (qtc >= w.tiles_c) {
                        qtc -= w.tiles_c;
                        ++qtr;
                    }
                }
                const int64_t cq = (int64_t)qtc * kColTileCols + (2 * warp + ((lane >> 3) & 1)) * 8 + (lane & 7);
                const int64_t rq = (int64_t)qtr * TILE_ROWS;
                lane_quad = philox_quad(p.sr_seed, p.sr_tag_scale,
                                        ((uint64_t)cq * (uint64_t)(p.k / NB) + (uint64_t)(rq / NB)) >> 2);
            }
        }
#pragma unroll
        for (int ci = 0; ci < 2; ++ci) {
            float v[G];
#pragma unroll
            for (int u = 0; u < G / 8; ++u) {
                const uint32_t addr = stage_base + lm_off[ci][u];
                uint32_t a0, a1, a2, a3;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                             : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                             : "r"(addr));
                if (NH > 0 && p.signs != 0u) {
                    a0 ^= smask[4 * u + 0];
                    a1 ^= smask[4 * u + 1];
                    a2 ^= smask[4 * u + 2];
                    a3 ^= smask[4 * u + 3];
                }
                v[8 * u + 0] = bf16lo(a0); v[8 * u + 1] = bf16hi(a0);
                v[8 * u + 2] = bf16lo(a1); v[8 * u + 3] = bf16hi(a1);
                v[8 * u + 4] = bf16lo(a2); v[8 * u + 5] = bf16hi(a2);
                v[8 * u + 6] = bf16lo(a3); v[8 * u + 7] = bf16hi(a3);
            }
            const int64_t c = c0 + cc[ci];              // x column = output row
            const int64_t r_grp = r0 + (int64_t)G * q;  // first k index of this group
            if constexpr (AMAX_ONLY) {
                amax_acc = rot_abs_max<NH, G>(amax_acc, v);
                if constexpr (DUAL) {
                    // Row orientation from the same tile: thread t takes shared-
                    // memory row t % 64 (some x-row of the tile; the max does not
                    // care which) and its 16-column group 2 (t / 64) + ci, two
                    // 16-byte chunks of a 128-byte swizzled row (8 consecutive
                    // lanes: 8 distinct rows mod 8, conflict-free).
                    static_assert(G == 16, "the row-and-column amax pass uses 16-row groups");
                    const int srow = tid & 63;
                    const int g16 = 2 * (tid >> 6) + ci;  // 0..7 over the tile's 128 columns
                    const uint32_t rb = smem_u32(tiles + s * STAGE_BYTES + (g16 >> 2) * BOX_BYTES) + srow * 128;
                    float vr[16];
#pragma unroll
                    for (int c8 = 0; c8 < 2; ++c8) {
                        const int chunk = 2 * (g16 & 3) + c8;
                        uint32_t w0, w1, w2, w3;
                        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
                                     : "r"(rb + ((chunk ^ (srow & 7)) << 4)));
                        if (NH > 0 && p.signs_row != 0u) {
                            w0 ^= Grp::sign_mask(p.signs_row, 4 * c8 + 0);
                            w1 ^= Grp::sign_mask(p.signs_row, 4 * c8 + 1);
                            w2 ^= Grp::sign_mask(p.signs_row, 4 * c8 + 2);
                            w3 ^= Grp::sign_mask(p.signs_row, 4 * c8 + 3);
                        }
                        vr[8 * c8 + 0] = bf16lo(w0); vr[8 * c8 + 1] = bf16hi(w0);
                        vr[8 * c8 + 2] = bf16lo(w1); vr[8 * c8 + 3] = bf16hi(w1);
                        vr[8 * c8 + 4] = bf16lo(w2); vr[8 * c8 + 5] = bf16hi(w2);
                        vr[8 * c8 + 6] = bf16lo(w3); vr[8 * c8 + 7] = bf16hi(w3);
                    }
                    amax_row_acc = rot_abs_max<NH, 16>(amax_row_acc, vr);
                }
            } else {
                uint32_t codes[G / 8];
                uint32_t scodes[G / NB];
                Grp::rotate(v);
                const uint64_t blk = (uint64_t)(c0 * (p.k / NB) + blk_off[ci] + r_grp / NB);
                if constexpr (kSharedQuads) {
                    if (shared_quads) {  // this group's quad: lane 16 * half + 8 * ci + column
                        const int src = (int)(quad_half << 4) | (ci << 3) | (lane >> 2);
                        srng.w = make_uint4(__shfl_sync(0xffffffffu, lane_quad.x, src),
                                            __shfl_sync(0xffffffffu, lane_quad.y, src),
                                            __shfl_sync(0xffffffffu, lane_quad.z, src),
                                            __shfl_sync(0xffffffffu, lane_quad.w, src));
                        srng.quad = blk >> 2;
                    }
                }
                Grp::quantize(v, s_enc, rtab, col_stream(p), (uint64_t)c * (uint64_t)p.k + (uint64_t)r_grp, blk, srng, codes,
                              scodes);
                if (c < p.rows && r_grp < p.k) {
                    uint8_t* dst = p.codes + c0 * (p.k / 2) + code_off[ci] + r_grp / 2;
                    if constexpr (G == 16)
                        *chk(reinterpret_cast<uint2*>(dst), p.codes, codes_extent(p)) = make_uint2(codes[0], codes[1]);
                    else
                        *chk(reinterpret_cast<uint4*>(dst), p.codes, codes_extent(p)) =
                            make_uint4(codes[0], codes[1], codes[2], codes[3]);
                }
                // Scales: the 4 lanes of column c (q = 0..3, consecutive lanes) hold
                // scale columns kb0 + (G/NB) q + b; gather them into 4-byte atom words.
                const int64_t kb0 = r0 / NB;
                uint32_t mine = scodes[0];
                if constexpr (G / NB == 2) mine |= scodes[1] << 8;
                const uint32_t n1 = __shfl_down_sync(0xffffffffu, mine, 1);
                const uint32_t n2 = __shfl_down_sync(0xffffffffu, mine, 2);
                const uint32_t n3 = __shfl_down_sync(0xffffffffu, mine, 3);
                if (c < rows_pad) {
                    const int64_t rowoff = (c0 / 128) * atom_row_bytes + sc_off[ci];
                    if constexpr (G / NB == 1) {
                        if (q == 0 && kb0 / 4 < p.kb4 / 4)
                            *chk(reinterpret_cast<uint32_t*>(p.scales + rowoff + (kb0 / 4) * 512), p.scales,
                                 scales_extent(p)) = mine | (n1 << 8) | (n2 << 16) | (n3 << 24);
                    } else {
                        if ((q == 0 || q == 2) && kb0 / 4 + q / 2 < p.kb4 / 4)
                            *chk(reinterpret_cast<uint32_t*>(p.scales + rowoff + (kb0 / 4 + q / 2) * 512), p.scales,
                                 scales_extent(p)) = mine | (n1 << 16);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ring.empty[s]);
        if constexpr (kSharedQuads) quad_half ^= 1u;
    }
    if constexpr (AMAX_ONLY) {
        if constexpr (NH > 0) amax_acc = __fmul_rn(amax_acc, had_norm<NH>());  // c * max |y| = max |c * y|
        write_partial(amax_acc, red, p.amax_out);
        if constexpr (DUAL) {
            if constexpr (NH > 0) amax_row_acc = __fmul_rn(amax_row_acc, had_norm<NH>());
            write_partial(amax_row_acc, red + 16, p.amax_out_row);
        }
    }
}

// ===========================================================================
// Column mode, 64-row bands (quantized axis a multiple of 64)
// ===========================================================================
// Tile: 256 x-rows (four bands of 64) x 64 columns. Thread (column c = 8 w +
// l / 4 of warp w, band q = l % 4) takes the 64 consecutive x-rows of band q
// of its column: 64 / G whole groups, four 16-element (or two 32-element)
// scale blocks, i.e. one 4-byte (NVFP4) or 2-byte (MXFP4) scale word, 32
// bytes of codes and, for Quartet II, one Philox quad per tile.
// The 4-D tensor map (column, r % 2, r / 64, (r / 2) % 32) delivers x-row
// r = k + 2 v + 64 q (k < 2, v < 32) to 128-byte shared-memory row
// s = k + 2 q + 8 v. Lane l of ldmatrix.x4 number n (n < 8) supplies smem row
// s = l + 32 n, i.e. matrix l / 8 row l % 8 = (q = (l % 8) / 2, k = l % 2) at
// v = 4 n + l / 8; the 8 rows of a phase have s % 8 = l % 8 all distinct
// (conflict-free with the 128-byte swizzle), and after the transposing load
// lane (c, q) holds x-rows 64 q + 8 n + [0, 8) of column c in order.
// Dual mode's row work on one band tile (see below): thread t quantizes
// shared-memory row t of the stage at `stage`, x-row r = r0 + k + 2 v + 64 q
// (t = k + 2 q + 8 v) over the tile's 64 columns, and stores its codes and
// scale word(s) in the row orientation (rows = R, k = C).
template <int FMT, int RND, int NH_ROW>
__device__ __forceinline__ void dual_row_work(const QuantParams& p, float s_enc_row, const float* rtab_row,
                                              const float2* tab2_row, ScaleRng& srng, uint32_t stage, int tr, int tc) {
    using GrpR = Group<FMT, RND, NH_ROW>;
    constexpr int NB = GrpR::NB;
    constexpr int GR = GrpR::G;
    constexpr bool kPackedRow = FMT == kNvfp4 && (NH_ROW == 0 || NH_ROW == 16) && RND != kSr;
    const int t = threadIdx.x;
    const int64_t r = (int64_t)tr * 256 + (t & 1) + 2 * (t >> 3) + 64 * ((t >> 1) & 3);
    const int64_t c0 = (int64_t)tc * 64;
    if (c0 >= p.C) return;  // the column tiles past C exist for the column orientation's padding only
    const uint32_t rbase = stage + (uint32_t)t * 128u;
    uint32_t codes[8];
    uint32_t scodes[64 / NB];
    uint32_t scw = 0;
    if constexpr (kPackedRow) {
        const SignFlips sf(NH_ROW > 0 ? p.signs_row : 0u);
        const uint32_t rb = rbase + ((uint32_t)(t & 7) << 4);
        auto load = [&](int c) { return lds128(rb ^ ((uint32_t)c << 4)); };
        scw = nv64_quantize<RND, NH_ROW>(load, sf, s_enc_row, tab2_row, row_stream(p),
                                         (uint64_t)r * (uint64_t)p.C + (uint64_t)c0,
                                         (uint64_t)r * (uint64_t)(p.C / 16) + (uint64_t)(c0 / 16), codes);
    } else {
#pragma unroll
    for (int g = 0; g < 64 / GR; ++g) {
        float v[GR];
#pragma unroll
        for (int c8 = 0; c8 < GR / 8; ++c8) {
            const int chunk = g * (GR / 8) + c8;
            uint32_t w0, w1, w2, w3;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3)
                         : "r"(rbase + ((uint32_t)(chunk ^ (t & 7)) << 4)));
            if (NH_ROW > 0 && p.signs_row != 0u) {
                w0 ^= GrpR::sign_mask(p.signs_row, 4 * c8 + 0);
                w1 ^= GrpR::sign_mask(p.signs_row, 4 * c8 + 1);
                w2 ^= GrpR::sign_mask(p.signs_row, 4 * c8 + 2);
                w3 ^= GrpR::sign_mask(p.signs_row, 4 * c8 + 3);
            }
            v[8 * c8 + 0] = bf16lo(w0); v[8 * c8 + 1] = bf16hi(w0);
            v[8 * c8 + 2] = bf16lo(w1); v[8 * c8 + 3] = bf16hi(w1);
            v[8 * c8 + 4] = bf16lo(w2); v[8 * c8 + 5] = bf16hi(w2);
            v[8 * c8 + 6] = bf16lo(w3); v[8 * c8 + 7] = bf16hi(w3);
        }
        GrpR::rotate(v);
        const int64_t j0 = c0 + g * GR;
        GrpR::quantize(v, s_enc_row, rtab_row, row_stream(p), (uint64_t)r * (uint64_t)p.C + (uint64_t)j0,
                       (uint64_t)r * (uint64_t)(p.C / NB) + (uint64_t)(j0 / NB), srng, codes + g * (GR / 8),
                       scodes + g * (GR / NB));
    }
    }
    if (r < p.R) {
        uint8_t* dst = p.codes_row + r * (p.C / 2) + c0 / 2;
        if (c0 + 64 <= p.C) {
            store_codes32(dst, codes, ((p.C / 2) & 15) == 0, p.codes_row, codes_row_extent(p));
        } else {
#pragma unroll
            for (int w = 0; w < 8; ++w)
                if (c0 + 8 * w < p.C)
                    *chk(reinterpret_cast<uint32_t*>(dst) + w, p.codes_row, codes_row_extent(p)) = codes[w];
        }
    }
    if (r < (p.R + 127) / 128 * 128) {
        const int64_t kb0 = c0 / NB;
        uint8_t* sc = p.scales_row + ((r / 128) * (p.kb4_row / 4) + kb0 / 4) * 512 + (r % 32) * 16 +
                      ((r / 32) % 4) * 4;
        if constexpr (NB == 16) {
            if constexpr (kPackedRow)
                *chk(reinterpret_cast<uint32_t*>(sc), p.scales_row, scales_row_extent(p)) = scw;
            else
                *chk(reinterpret_cast<uint32_t*>(sc), p.scales_row, scales_row_extent(p)) =
                    scodes[0] | (scodes[1] << 8) | (scodes[2] << 16) | (scodes[3] << 24);
        } else {
            const uint32_t half = scodes[0] | (scodes[1] << 8);
            if ((kb0 & 3) == 0 && c0 + 64 >= p.C)
                *chk(reinterpret_cast<uint32_t*>(sc), p.scales_row, scales_row_extent(p)) = half;
            else
                *chk(reinterpret_cast<uint16_t*>(sc + (kb0 & 3)), p.scales_row, scales_row_extent(p)) = (uint16_t)half;
        }
    }
}

//
// Dual mode (NH_ROW >= 0): after its column work on a tile, thread t also
// quantizes shared-memory row t, i.e. x-row k + 2 v + 64 q of the tile over its
// 64 columns, in the row orientation (rotation of size NH_ROW with the row
// sign vector, the row tensor amax and random streams), as the row kernel
// would: one read of x gives both orientations.
template <int FMT, int RND, int NH, int STAGES, int NH_ROW = -1, bool FUSED = false>
__global__ void __launch_bounds__(kThreads, kCtasPerSm<STAGES>)
    quant_col64_kernel(const __grid_constant__ CUtensorMap tmap, const QuantParams p) {
    constexpr bool kDual = NH_ROW >= 0;
    using Grp = Group<FMT, RND, NH>;
    constexpr int NB = Grp::NB;
    constexpr int G = Grp::G;
    constexpr int TILE_ROWS = 256, TILE_COLS = 64;
    constexpr int STAGE_BYTES = TILE_ROWS * TILE_COLS * 2;  // 32 KiB
    static_assert(64 % G == 0, "groups tile a 64-row band");
    // NVFP4 with no Hadamard or a 16-point one, round-to-nearest or Quartet
    // II: the packed 64-element unit
    constexpr bool kPacked = FMT == kNvfp4 && (NH == 0 || NH == 16) && RND != kSr;
    constexpr bool kPackedRow = kDual && FMT == kNvfp4 && (NH_ROW == 0 || NH_ROW == 16) && RND != kSr;
    static_assert(!FUSED || (kPacked && !kDual), "the fused amax pass serves the packed NVFP4 unit");
    extern __shared__ __align__(1024) uint8_t dyn_smem[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    __shared__ Ring<STAGES> ring;
    __shared__ float red[33];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // output rows = x columns, walked up to the 128-row padding of the scale
    // atoms: the tiles past the last column read zeros and write zero scales
    const int tiles_c = (int)((p.rows + 127) / 128 * 2);
    const int tiles_r = (int)((p.k + TILE_ROWS - 1) / TILE_ROWS);

    if (tid == 0) {
        prefetch_tmap(&tmap);
        ring_init(ring);
    }
    __syncthreads();
    pdl_wait();  // the previous kernel's writes are visible (and its reads done)
    pdl_launch_dependents();

    if (warp == kComputeWarps) {
        if (lane == 0) {
            int i = 0;
            bool ok = true;
            for (int pass = 0; pass < (FUSED ? 2 : 1) && ok; ++pass)
                for (TileWalk<STAGES> w(tiles_c, i); w.tr < tiles_r; w.next(), ++i) {
                    const int s = w.stage;
                    if (i >= STAGES && !mbar_wait(&ring.empty[s], w.phase ^ 1u)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&ring.full[s], STAGE_BYTES);
                    tma_load_4d(tiles + s * STAGE_BYTES, &tmap, &ring.full[s], w.tc * TILE_COLS, 0, 4 * w.tr, 0);
                }
            drain_loads(ring.full, nullptr, STAGES, i);  // no load lands after this CTA exits
        }
        return;
    }
    __shared__ float rtab[kPacked ? 1 : 128];
    __shared__ float2 tab2[kPacked ? 128 : 1];
    __shared__ float rtab_row[kDual && !kPackedRow ? 128 : 1];
    __shared__ float2 tab2_row[kPackedRow ? 128 : 1];
    float s_enc = 1.0f, s_enc_row = 1.0f;
    int issued = 0;  // ring iterations of the fused amax pass
    if constexpr (FUSED) {
        const uint32_t lm = (uint32_t)lane * 128u + ((uint32_t)(warp ^ (lane & 7)) << 4);
        issued = fused_amax_pass<NH>(p, ring, tiles_c, tiles_r, red, [&](int st, int n) {
            uint4 v;
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(smem_u32(tiles) + (uint32_t)(st * STAGE_BYTES) + lm + (uint32_t)(n * 4096)));
            return v;
        });
    }
    if constexpr (FMT == kNvfp4) {
        s_enc = nvfp4_encode_scale(p, red, blockIdx.x == 0);
        if constexpr (kPacked)
            fill_tab2(tab2, s_enc);
        else
            fill_rtab(rtab, s_enc);
        if constexpr (kDual) {  // the row orientation's amax is always given
            s_enc_row = nvfp4_scale_from_amax(__ldg(p.amax_in_row), p.tensor_scale_row, blockIdx.x == 0);
            if constexpr (kPackedRow)
                fill_tab2(tab2_row, s_enc_row);
            else
                fill_rtab(rtab_row, s_enc_row);
        }
    }
    if constexpr (FMT == kMxfp4) {
        if (blockIdx.x == 0 && tid == 0) {
            *p.tensor_scale = 1.0f;
            if constexpr (kDual) *p.tensor_scale_row = 1.0f;
        }
    }

    const int64_t rows_pad = (p.rows + 127) / 128 * 128;
    const int q = lane & 3;
    const int cc = warp * 8 + (lane >> 2);  // column within the tile
    // ldmatrix address of instruction n: lm_base + 4096 n (smem row lane + 32 n)
    const uint32_t lm_base = (uint32_t)lane * 128u + ((uint32_t)(warp ^ (lane & 7)) << 4);
    const int64_t atom_row_bytes = (p.kb4 / 4) * 512;
    // sign masks held in registers, except in dual mode (registers for the row work)
    uint32_t smask[kDual || kPacked ? 1 : G / 2];
    if constexpr (!kDual && !kPacked) {
#pragma unroll
        for (int i = 0; i < G / 2; ++i) smask[i] = Grp::sign_mask(p.signs, i);
    }
    const SignFlips sf(kPacked && NH > 0 ? p.signs : 0u);
    ScaleRng srng, srng_row;
    for (TileWalk<STAGES> w(tiles_c, issued); w.tr < tiles_r; w.next()) {
        const int s = w.stage;
        if (!mbar_wait(&ring.full[s], w.phase)) break;
        const int64_t c = (int64_t)w.tc * TILE_COLS + cc;          // x column = output row
        const int64_t rb = (int64_t)w.tr * TILE_ROWS + 64 * q;     // first k index of this thread's band
        const uint32_t stage_base = smem_u32(tiles) + (uint32_t)(s * STAGE_BYTES) + lm_base;
        uint32_t codes[8];
        uint32_t scodes[64 / NB];
        uint32_t scw = 0;
        if constexpr (kPacked) {
            // chunk n = rows 8n .. 8n + 7 of the band: ldmatrix number n
            auto load = [&](int n) {
                uint4 v;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                             : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                             : "r"(stage_base + (uint32_t)(n * 4096)));
                return v;
            };
            scw = nv64_quantize<RND, NH>(load, sf, s_enc, tab2, col_stream(p), (uint64_t)c * (uint64_t)p.k + (uint64_t)rb,
                                         (uint64_t)c * (uint64_t)(p.k / 16) + (uint64_t)(rb / 16), codes);
        } else {
#pragma unroll
        for (int g = 0; g < 64 / G; ++g) {
            float v[G];
#pragma unroll
            for (int u = 0; u < G / 8; ++u) {
                const uint32_t addr = stage_base + (uint32_t)((g * (G / 8) + u) * 4096);
                uint32_t a0, a1, a2, a3;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                             : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                             : "r"(addr));
                if (NH > 0 && p.signs != 0u) {
                    if constexpr (kDual) {
                        a0 ^= Grp::sign_mask(p.signs, 4 * u + 0);
                        a1 ^= Grp::sign_mask(p.signs, 4 * u + 1);
                        a2 ^= Grp::sign_mask(p.signs, 4 * u + 2);
                        a3 ^= Grp::sign_mask(p.signs, 4 * u + 3);
                    } else {
                        a0 ^= smask[4 * u + 0];
                        a1 ^= smask[4 * u + 1];
                        a2 ^= smask[4 * u + 2];
                        a3 ^= smask[4 * u + 3];
                    }
                }
                v[8 * u + 0] = bf16lo(a0); v[8 * u + 1] = bf16hi(a0);
                v[8 * u + 2] = bf16lo(a1); v[8 * u + 3] = bf16hi(a1);
                v[8 * u + 4] = bf16lo(a2); v[8 * u + 5] = bf16hi(a2);
                v[8 * u + 6] = bf16lo(a3); v[8 * u + 7] = bf16hi(a3);
            }
            Grp::rotate(v);
            const int64_t r_grp = rb + g * G;
            Grp::quantize(v, s_enc, rtab, col_stream(p), (uint64_t)c * (uint64_t)p.k + (uint64_t)r_grp,
                          (uint64_t)c * (uint64_t)(p.k / NB) + (uint64_t)(r_grp / NB), srng, codes + g * (G / 8),
                          scodes + g * (G / NB));
        }
        }
        if constexpr (kDual) dual_row_work<FMT, RND, NH_ROW>(p, s_enc_row, rtab_row, tab2_row, srng_row,
                                                          smem_u32(tiles) + (uint32_t)(s * STAGE_BYTES), w.tr, w.tc);
        __syncwarp();
        if (lane == 0) mbar_arrive(&ring.empty[s]);
        if (rb < p.k) {  // k is a multiple of 64: a band is wholly inside or wholly outside
            if (c < p.rows) {
                uint4* dst = reinterpret_cast<uint4*>(p.codes + c * (p.k / 2) + rb / 2);
                *chk(dst, p.codes, codes_extent(p)) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
                *chk(dst + 1, p.codes, codes_extent(p)) = make_uint4(codes[4], codes[5], codes[6], codes[7]);
            }
            if (c < rows_pad) {
                const int64_t kb0 = rb / NB;
                uint8_t* sc = p.scales + (c / 128) * atom_row_bytes + (kb0 / 4) * 512 + (c % 32) * 16 + ((c / 32) % 4) * 4;
                if constexpr (NB == 16) {
                    if constexpr (kPacked)
                        *chk(reinterpret_cast<uint32_t*>(sc), p.scales, scales_extent(p)) = scw;
                    else
                        *chk(reinterpret_cast<uint32_t*>(sc), p.scales, scales_extent(p)) =
                            scodes[0] | (scodes[1] << 8) | (scodes[2] << 16) | (scodes[3] << 24);
                } else {
                    // two scale columns: half of an atom word; when this is the
                    // word's first half and the band is the last, the other
                    // half is padding and is written as zero
                    const uint32_t half = scodes[0] | (scodes[1] << 8);
                    if ((kb0 & 3) == 0 && rb + 64 >= p.k)
                        *chk(reinterpret_cast<uint32_t*>(sc), p.scales, scales_extent(p)) = half;
                    else
                        *chk(reinterpret_cast<uint16_t*>(sc + (kb0 & 3)), p.scales, scales_extent(p)) = (uint16_t)half;
                }
            }
        }
    }
}

// ===========================================================================
// Both orientations' rotated amax over 64-row bands
// ===========================================================================
// The band kernel's tile (256 x-rows x 64 columns through the 4-D view) read
// once for both tensor amaxes (the R a multiple of 64 case of
// qfp4_amax_rowcol): thread (column c, band q) takes 64 consecutive rows of
// column c (eight ldmatrix.trans, as the column quantizer) and shared-memory
// row t's 64 columns (as the dual row work), each as two pairs of 16-element
// groups with the butterflies packed across the pair. The rotation's
// 1/sqrt(n_h) is applied once to each CTA's maxima (rounding c * y is
// monotone in y). Zero-filled columns and rows past the tensor add nothing.

template <int NH, int STAGES>
__global__ void __launch_bounds__(kThreads, 2)
    amax_rowcol64_kernel(const __grid_constant__ CUtensorMap tmap, const QuantParams p) {
    static_assert(NH == 0 || NH == 16, "16-element groups");
    constexpr int TILE_ROWS = 256, TILE_COLS = 64;
    constexpr int STAGE_BYTES = TILE_ROWS * TILE_COLS * 2;  // 32 KiB
    extern __shared__ __align__(1024) uint8_t dyn_smem[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    __shared__ Ring<STAGES> ring;
    __shared__ float red[33];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tiles_c = (int)((p.rows + TILE_COLS - 1) / TILE_COLS);  // x columns
    const int tiles_r = (int)((p.k + TILE_ROWS - 1) / TILE_ROWS);     // x rows
    if (tid == 0) {
        prefetch_tmap(&tmap);
        ring_init(ring);
    }
    __syncthreads();
    pdl_wait();  // the previous kernel's writes are visible (and its reads done)
    pdl_launch_dependents();
    if (warp == kComputeWarps) {
        if (lane == 0) {
            int i = 0;
            for (TileWalk<STAGES> w(tiles_c); w.tr < tiles_r; w.next(), ++i) {
                const int s = w.stage;
                if (i >= STAGES && !mbar_wait(&ring.empty[s], w.phase ^ 1u)) break;
                mbar_arrive_expect_tx(&ring.full[s], STAGE_BYTES);
                tma_load_4d(tiles + s * STAGE_BYTES, &tmap, &ring.full[s], w.tc * TILE_COLS, 0, 4 * w.tr, 0);
            }
            drain_loads(ring.full, nullptr, STAGES, i);  // no load lands after this CTA exits
        }
        return;
    }
    const SignFlips sf_col(NH > 0 ? p.signs : 0u), sf_row(NH > 0 ? p.signs_row : 0u);
    // ldmatrix address of instruction n: lm_base + 4096 n (smem row lane + 32 n)
    const uint32_t lm_base = (uint32_t)lane * 128u + ((uint32_t)(warp ^ (lane & 7)) << 4);
    const uint32_t row_off = (uint32_t)tid * 128u + ((uint32_t)(tid & 7) << 4);
    float m_col = 0.0f, m_row = 0.0f;
    for (TileWalk<STAGES> w(tiles_c); w.tr < tiles_r; w.next()) {
        const int s = w.stage;
        if (!mbar_wait(&ring.full[s], w.phase)) break;
        const uint32_t stage = smem_u32(tiles) + (uint32_t)(s * STAGE_BYTES);
        auto load_col = [&](int n) {
            uint4 v;
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(stage + lm_base + (uint32_t)(n * 4096)));
            return v;
        };
        m_col = rot_amax64<NH>(load_col, sf_col, m_col);
        auto load_row = [&](int c) { return lds128((stage + row_off) ^ ((uint32_t)c << 4)); };
        m_row = rot_amax64<NH>(load_row, sf_row, m_row);
        __syncwarp();
        if (lane == 0) mbar_arrive(&ring.empty[s]);
    }
    if constexpr (NH > 0) {
        m_col = __fmul_rn(m_col, had_norm<NH>());  // c * max |y| = max |c * y|
        m_row = __fmul_rn(m_row, had_norm<NH>());
    }
    write_partial(m_col, red, p.amax_out);
    write_partial(m_row, red + 16, p.amax_out_row);
}

int g_sm_count = 0;

int persistent_grid(int64_t tiles, int per_sm) {
    const int sms = g_sm_count > 0 ? g_sm_count : 148;
    int64_t g = (int64_t)sms * per_sm;
    if (g > tiles) g = tiles;
    return g < 1 ? 1 : (int)g;
}

template <typename Kern>
cudaError_t launch_persistent(Kern kern, int grid, int smem, const CUtensorMap& tmap, const QuantParams& p,
                              cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3(grid), dim3(kThreads), (size_t)smem, s, tmap, p);
    count_launch();
    return e;
}

// A cooperative launch (all CTAs co-resident, as the fused kernels' grid
// barrier needs) of a persistent quantizer: at most as many CTAs per SM as
// fit, and no more than two; p.n_partials is set to the grid size (the fused
// amax pass writes one partial per CTA).
template <typename Kern>
cudaError_t launch_cooperative(Kern kern, int64_t tiles, int smem, const CUtensorMap& tmap, const QuantParams& p,
                               cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem)) != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
    const int grid = persistent_grid(tiles, per_sm < 2 ? per_sm : 2);
    QuantParams q = p;
    q.n_partials = grid;
    void* args[] = {const_cast<CUtensorMap*>(&tmap), &q};
    e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid), dim3(kThreads), args,
                                    (size_t)smem, s);
    count_launch();
    return e;
}

constexpr int kRowStages = 3;
template <int G>
constexpr int col_stages() {
    return G == 16 ? 4 : 3;
}

template <int FMT, int RND, int NH, bool AMAX_ONLY>
cudaError_t launch_t(const QuantParams& p, int axis, const CUtensorMap* tmap, int grid, cudaStream_t s) {
    if (axis == 0) {
        const int64_t tiles =
            ((p.rows + kRowTileRows - 1) / kRowTileRows) * ((p.k + kRowTileCols - 1) / kRowTileCols);
        constexpr int S = (!AMAX_ONLY && issue_bound_mode<FMT, RND>()) ? 2 : kRowStages;
        if (grid <= 0) grid = persistent_grid(tiles, kCtasPerSm<S>);
        const int smem = S * kRowTileRows * kRowTileCols * 2 + 1024;
        return launch_persistent(quant_row_kernel<FMT, RND, NH, AMAX_ONLY, S>, grid, smem, *tmap, p, s);
    } else {
        constexpr int NB = (FMT == kNvfp4) ? 16 : 32;
        constexpr int G = AMAX_ONLY ? ((NH > 16) ? NH : 16) : ((NH > NB) ? NH : NB);
        constexpr int S = col_stages<G>();
        const int64_t tiles = ((p.rows + kColTileCols - 1) / kColTileCols) * ((p.k + 4 * G - 1) / (4 * G));
        if (grid <= 0) grid = persistent_grid(tiles, 2);
        const int smem = S * 2 * (4 * G * 64 * 2) + 1024;
        return launch_persistent(quant_col_kernel<FMT, RND, NH, AMAX_ONLY, S>, grid, smem, *tmap, p, s);
    }
}

// Column mode over 64-row bands (axis code 2; the quantized axis a multiple of 64).
template <int FMT, int RND, int NH>
cudaError_t launch_col64(const QuantParams& p, const CUtensorMap* tmap, cudaStream_t s) {
    constexpr int S = issue_bound_mode<FMT, RND>() ? 2 : 3;
    const int64_t tiles = ((p.rows + 127) / 128 * 2) * ((p.k + 255) / 256);
    const int smem = S * 256 * 64 * 2 + 1024;
    return launch_persistent(quant_col64_kernel<FMT, RND, NH, S>, persistent_grid(tiles, kCtasPerSm<S>), smem,
                             *tmap, p, s);
}

// The fused (one-launch) NVFP4 quantization: packed unit, RTN or Quartet II,
// no Hadamard or a 16-point one, along rows (axis 0) or 64-row bands (2).
template <int RND, int NH>
cudaError_t launch_fused_t(const QuantParams& p, int axis, const CUtensorMap* tmap, cudaStream_t s) {
    if (axis == 0) {
        const int64_t tiles =
            ((p.rows + kRowTileRows - 1) / kRowTileRows) * ((p.k + kRowTileCols - 1) / kRowTileCols);
        const int smem = kRowStages * kRowTileRows * kRowTileCols * 2 + 1024;
        return launch_cooperative(quant_row_kernel<kNvfp4, RND, NH, false, kRowStages, true>, tiles, smem, *tmap, p,
                                  s);
    }
    constexpr int S = 3;
    const int64_t tiles = ((p.rows + 127) / 128 * 2) * ((p.k + 255) / 256);
    const int smem = S * 256 * 64 * 2 + 1024;
    return launch_cooperative(quant_col64_kernel<kNvfp4, RND, NH, S, -1, true>, tiles, smem, *tmap, p, s);
}

template <int FMT, int RND>
cudaError_t dispatch_nh(const QuantParams& p, int nh, int axis, const CUtensorMap* tmap, cudaStream_t s) {
    if (axis == 2) {
        switch (nh) {
            case 0: return launch_col64<FMT, RND, 0>(p, tmap, s);
            case 16: return launch_col64<FMT, RND, 16>(p, tmap, s);
            default: return launch_col64<FMT, RND, 32>(p, tmap, s);
        }
    }
    switch (nh) {
        case 0: return launch_t<FMT, RND, 0, false>(p, axis, tmap, 0, s);
        case 16: return launch_t<FMT, RND, 16, false>(p, axis, tmap, 0, s);
        default: return launch_t<FMT, RND, 32, false>(p, axis, tmap, 0, s);
    }
}

// Max of n partial maxima (one CTA).
__global__ void __launch_bounds__(256) reduce_max_kernel(const float* in, int n, float* out) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ float red[8];
    float m = 0.0f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, in[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
        *out = fmaxf(m, red[0]);
    }
}

}  // namespace

void set_sm_count(int sms) { g_sm_count = sms; }

int64_t quant_tiles(int axis, int64_t rows, int64_t k, int G) {
    if (axis == 0) return ((rows + kRowTileRows - 1) / kRowTileRows) * ((k + kRowTileCols - 1) / kRowTileCols);
    return ((rows + kColTileCols - 1) / kColTileCols) * ((k + 4 * G - 1) / (4 * G));
}

cudaError_t launch_reduce_max(const float* in, int n, float* out, cudaStream_t s) {
    const cudaError_t e = launch_pdl(reduce_max_kernel, dim3(1), dim3(256), 0, s, in, n, out);
    count_launch();
    return e;
}

int col_group(int block, int nh) { return nh > block ? nh : block; }

cudaError_t launch_quant_fused(const QuantParams& p, int rnd, int nh, int axis, const CUtensorMap* tmap,
                               cudaStream_t s) {
    if (rnd == kRtn) return nh == 16 ? launch_fused_t<kRtn, 16>(p, axis, tmap, s) : launch_fused_t<kRtn, 0>(p, axis, tmap, s);
    return nh == 16 ? launch_fused_t<kQuartet2, 16>(p, axis, tmap, s) : launch_fused_t<kQuartet2, 0>(p, axis, tmap, s);
}

cudaError_t launch_quant(const QuantParams& p, int fmt, int rnd, int nh, int axis, const CUtensorMap* tmap,
                         cudaStream_t s) {
    if (fmt == kNvfp4) {
        if (rnd == kRtn) return dispatch_nh<kNvfp4, kRtn>(p, nh, axis, tmap, s);
        if (rnd == kSr) return dispatch_nh<kNvfp4, kSr>(p, nh, axis, tmap, s);
        return dispatch_nh<kNvfp4, kQuartet2>(p, nh, axis, tmap, s);
    }
    if (rnd == kRtn) return dispatch_nh<kMxfp4, kRtn>(p, nh, axis, tmap, s);
    if (rnd == kSr) return dispatch_nh<kMxfp4, kSr>(p, nh, axis, tmap, s);
    return dispatch_nh<kMxfp4, kQuartet2>(p, nh, axis, tmap, s);
}

template <int FMT, int RND, int NH, int NH_ROW>
cudaError_t launch_dual_t(const QuantParams& p, const CUtensorMap* tmap, cudaStream_t s) {
    constexpr int S = 3;
    const int64_t tiles = ((p.rows + 127) / 128 * 2) * ((p.k + 255) / 256);
    const int smem = S * 256 * 64 * 2 + 1024;
    return launch_persistent(quant_col64_kernel<FMT, RND, NH, S, NH_ROW>, persistent_grid(tiles, 2), smem, *tmap, p,
                             s);
}

template <int FMT, int RND>
cudaError_t dispatch_dual(const QuantParams& p, int nh, int nh_row, const CUtensorMap* tmap, cudaStream_t s) {
    if (nh == 0) return launch_dual_t<FMT, RND, 0, 0>(p, tmap, s);
    if (nh == 16) return nh_row == 0 ? launch_dual_t<FMT, RND, 16, 0>(p, tmap, s) : launch_dual_t<FMT, RND, 16, 16>(p, tmap, s);
    return nh_row == 0 ? launch_dual_t<FMT, RND, 32, 0>(p, tmap, s) : launch_dual_t<FMT, RND, 32, 32>(p, tmap, s);
}

cudaError_t launch_quant_dual(const QuantParams& p, int fmt, int rnd, int nh, int nh_row, const CUtensorMap* tmap,
                              cudaStream_t s) {
    if (fmt == kNvfp4) {
        if (rnd == kRtn) return dispatch_dual<kNvfp4, kRtn>(p, nh, nh_row, tmap, s);
        if (rnd == kSr) return dispatch_dual<kNvfp4, kSr>(p, nh, nh_row, tmap, s);
        return dispatch_dual<kNvfp4, kQuartet2>(p, nh, nh_row, tmap, s);
    }
    if (rnd == kRtn) return dispatch_dual<kMxfp4, kRtn>(p, nh, nh_row, tmap, s);
    if (rnd == kSr) return dispatch_dual<kMxfp4, kSr>(p, nh, nh_row, tmap, s);
    return dispatch_dual<kMxfp4, kQuartet2>(p, nh, nh_row, tmap, s);
}

cudaError_t launch_amax_rowcol64(const QuantParams& p, int nh, const CUtensorMap* tmap, int n_partials,
                                 cudaStream_t s) {
    constexpr int S = 3;
    const int smem = S * 256 * 64 * 2 + 1024;
    if (nh == 16) return launch_persistent(amax_rowcol64_kernel<16, S>, n_partials, smem, *tmap, p, s);
    return launch_persistent(amax_rowcol64_kernel<0, S>, n_partials, smem, *tmap, p, s);
}

int64_t amax_rowcol64_tiles(int64_t rows, int64_t k) { return ((rows + 63) / 64) * ((k + 255) / 256); }

cudaError_t launch_amax_rowcol(const QuantParams& p, int nh, const CUtensorMap* tmap, int n_partials,
                               cudaStream_t s) {
    constexpr int G = 16, S = col_stages<G>();
    const int smem = S * 2 * (4 * G * 64 * 2) + 1024;
    if (nh == 16)
        return launch_persistent(quant_col_kernel<kNvfp4, kRtn, 16, true, S, true>, n_partials, smem, *tmap, p, s);
    return launch_persistent(quant_col_kernel<kNvfp4, kRtn, 0, true, S, true>, n_partials, smem, *tmap, p, s);
}

cudaError_t launch_amax(const QuantParams& p, int axis, int nh, const CUtensorMap* tmap, int n_partials,
                        cudaStream_t s) {
    switch (nh) {
        case 0: return launch_t<kNvfp4, kRtn, 0, true>(p, axis, tmap, n_partials, s);
        case 16: return launch_t<kNvfp4, kRtn, 16, true>(p, axis, tmap, n_partials, s);
        default: return launch_t<kNvfp4, kRtn, 32, true>(p, axis, tmap, n_partials, s);
    }
}

}  // namespace qfp4
