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
// Row mode (blocks along the contiguous axis): a CTA owns 128 rows x 128
// columns; each thread loads 16-byte chunks of 8 elements, coalesced across the
// warp. The Hadamard butterflies of half-width < 8 run in registers, wider ones
// and the block reductions with warp shuffles between the 2 or 4 lanes of a
// block. Scales are staged in shared memory as whole 512-byte MMA atoms and
// stored with 16-byte writes.
//
// Column mode (blocks along the strided axis; the output is the quantized
// transpose): a CTA owns 4G rows x 128 columns (G = max(block, n_h)), brought
// in by TMA as two 128-byte-swizzled boxes through a 5-D view of the tensor
// whose row order makes the transposing ldmatrix reads conflict-free; each
// thread then holds one whole group of one column in registers.
//
// Every fp32 operation is the one the method states, in its order, with no
// fused multiply-add (the library is built with --fmad=false), so codes and
// scales are exactly those of the definition.
#include <cuda_fp16.h>

#include "qfp4_device.cuh"
#include "qfp4_internal.h"

namespace qfp4 {

namespace {

constexpr int kThreads = 256;
constexpr int kRowTileRows = 128, kRowTileCols = 128;
constexpr int kColTileCols = 128;

template <int NH>
__device__ __forceinline__ float had_norm() {
    return NH == 16 ? 0.25f : 0x1.6a09e6p-3f;  // fp32(1/sqrt(16)), fp32(1/sqrt(32))
}

// In-register butterflies of half-width 1, 2, 4 over 8 consecutive elements.
__device__ __forceinline__ void fwht8(float* v) {
#pragma unroll
    for (int h = 1; h < 8; h <<= 1)
#pragma unroll
        for (int j0 = 0; j0 < 8; j0 += 2 * h)
#pragma unroll
            for (int j = j0; j < j0 + h; ++j) {
                const float a = v[j], b = v[j + h];
                v[j] = __fadd_rn(a, b);
                v[j + h] = __fsub_rn(a, b);
            }
}

// Butterflies of half-width 8 .. n/2 over n elements held by one thread.
template <int N>
__device__ __forceinline__ void fwht_wide(float* v) {
#pragma unroll
    for (int h = 8; h < N; h <<= 1)
#pragma unroll
        for (int j0 = 0; j0 < N; j0 += 2 * h)
#pragma unroll
            for (int j = j0; j < j0 + h; ++j) {
                const float a = v[j], b = v[j + h];
                v[j] = __fadd_rn(a, b);
                v[j + h] = __fsub_rn(a, b);
            }
}

// Reduce the CTA's amax partials (NVFP4) to s_enc and write g from CTA 0.
__device__ float nvfp4_encode_scale(const QuantParams& p, float* red_smem, bool write_g) {
    float amax = 0.0f;
    if (p.amax_in != nullptr) {
        amax = __ldg(p.amax_in);
    } else {
        float m = 0.0f;
        for (int i = threadIdx.x; i < p.n_partials; i += blockDim.x) m = fmaxf(m, __ldg(p.amax_partials + i));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((threadIdx.x & 31) == 0) red_smem[threadIdx.x >> 5] = m;
        __syncthreads();
        if (threadIdx.x < 32) {
            m = threadIdx.x < (blockDim.x >> 5) ? red_smem[threadIdx.x] : 0.0f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (threadIdx.x == 0) red_smem[32] = m;
        }
        __syncthreads();
        amax = red_smem[32];
    }
    float s_enc = 1.0f, g = 1.0f;
    if (amax > 0.0f) {
        s_enc = __fdiv_rn(2688.0f, amax);
        if (s_enc > 3.402823466e38f) s_enc = 3.402823466e38f;
        g = __fdiv_rn(amax, 2688.0f);
    }
    if (write_g && threadIdx.x == 0) *p.tensor_scale = g;
    return s_enc;
}

// Block scale of one block from its amax. Returns the scale code and sets the
// element multiplier r and the decoded scale S.
template <int FMT>
__device__ __forceinline__ uint32_t block_scale(float amax_b, float s_enc, float& rmul, float& S) {
    if constexpr (FMT == kNvfp4) {
        const float d = __fdiv_rn(amax_b, 6.0f);
        const float t = __fmul_rn(d, s_enc);
        const uint32_t code = e4m3_rn(t);
        S = e4m3_decode(code);
        rmul = (S == 0.0f) ? 0.0f : __fdiv_rn(s_enc, S);
        return code;
    } else {
        if (amax_b == 0.0f) {
            S = exp2i(-127);
            rmul = 0.0f;
            return 0u;
        }
        int E = floor_log2(amax_b) - 2;
        E = E < -127 ? -127 : (E > 127 ? 127 : E);
        S = exp2i(E);
        rmul = exp2i(-E);
        return (uint32_t)(E + 127);
    }
}

// Quartet II scale: SR(S * alpha) onto the scale grid with the block's uniform.
template <int FMT>
__device__ __forceinline__ uint32_t quartet2_scale(float num, float den, float S, const QuantParams& p,
                                                   uint64_t block_index) {
    const float alpha = (den == 0.0f) ? 1.0f : __fdiv_rn(num, den);
    const float t = __fmul_rn(S, alpha);
    const uint4 w = philox_quad(p.sr_seed, p.sr_tag_scale, block_index >> 2);
    const uint32_t word = (block_index & 3) == 0 ? w.x : (block_index & 3) == 1 ? w.y : (block_index & 3) == 2 ? w.z : w.w;
    const float rho = uniform24(word);
    if constexpr (FMT == kNvfp4)
        return e4m3_sr(t, rho);
    else
        return e8m0_sr(t, rho);
}

// Write the CTA's staged scale atoms (n_atoms x 512 bytes, contiguous in the
// global layout) unless they fall past the padded scale columns.
__device__ __forceinline__ void store_atoms(const QuantParams& p, const uint8_t* stage, int n_atoms, int64_t row0,
                                            int64_t first_kb) {
    const int64_t atoms_k = p.kb4 / 4;
    const int64_t atom_col = first_kb / 4;
    for (int i = threadIdx.x; i < n_atoms * 32; i += blockDim.x) {
        const int a = i >> 5;
        if (atom_col + a >= atoms_k) continue;
        const int64_t dst = ((row0 / 128) * atoms_k + atom_col + a) * 512 + (i & 31) * 16;
        *reinterpret_cast<uint4*>(p.scales + dst) = *reinterpret_cast<const uint4*>(stage + a * 512 + (i & 31) * 16);
    }
}

__device__ __forceinline__ int atom_offset(int row_in_tile, int kb_local) {
    return (kb_local >> 2) * 512 + (row_in_tile & 31) * 16 + ((row_in_tile >> 5) & 3) * 4 + (kb_local & 3);
}

// ===========================================================================
// Row mode
// ===========================================================================
template <int FMT, int RND, int NH, bool AMAX_ONLY>
__global__ void __launch_bounds__(kThreads) quant_row_kernel(const QuantParams p) {
    constexpr int NB = (FMT == kNvfp4) ? 16 : 32;
    constexpr int CHUNKS = kRowTileRows * kRowTileCols / 8 / kThreads;  // 8 chunks per thread
    __shared__ __align__(16) uint8_t scale_stage[1024];
    __shared__ float red[33];

    const int tid = threadIdx.x;
    const int cc = tid & 15;  // chunk column within the tile
    const int64_t tiles_c = (p.k + kRowTileCols - 1) / kRowTileCols;
    const int64_t tiles_total = tiles_c * ((p.rows + kRowTileRows - 1) / kRowTileRows);

    float s_enc = 1.0f;
    if constexpr (!AMAX_ONLY && FMT == kNvfp4) s_enc = nvfp4_encode_scale(p, red, blockIdx.x == 0);
    if constexpr (!AMAX_ONLY && FMT == kMxfp4) {
        if (blockIdx.x == 0 && tid == 0) *p.tensor_scale = 1.0f;
    }
    float amax_acc = 0.0f;

    for (int64_t tile = blockIdx.x; tile < tiles_total; tile += gridDim.x) {
        const int64_t row0 = (tile / tiles_c) * kRowTileRows;
        const int64_t col0 = (tile % tiles_c) * kRowTileCols;
        const int64_t col = col0 + cc * 8;
        const bool col_ok = col < p.k;

        uint4 raw[CHUNKS];
#pragma unroll
        for (int j = 0; j < CHUNKS; ++j) {
            const int64_t row = row0 + 16 * j + (tid >> 4);
            raw[j] = make_uint4(0u, 0u, 0u, 0u);
            if (col_ok && row < p.rows) raw[j] = __ldg(reinterpret_cast<const uint4*>(p.x + row * p.ld + col));
        }

#pragma unroll
        for (int j = 0; j < CHUNKS; ++j) {
            const int r_in_tile = 16 * j + (tid >> 4);
            const int64_t row = row0 + r_in_tile;
            float v[8];
            v[0] = bf16lo(raw[j].x); v[1] = bf16hi(raw[j].x);
            v[2] = bf16lo(raw[j].y); v[3] = bf16hi(raw[j].y);
            v[4] = bf16lo(raw[j].z); v[5] = bf16hi(raw[j].z);
            v[6] = bf16lo(raw[j].w); v[7] = bf16hi(raw[j].w);

            if constexpr (NH > 0) {
                // 1. rotation: signs, butterflies h = 1, 2, 4 in registers, h = 8 (and
                // 16) across lanes, then one fp32 multiply by 1/sqrt(n_h).
                const uint32_t sbits = p.signs >> (uint32_t)(col % NH);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if ((sbits >> e) & 1u) v[e] = -v[e];
                fwht8(v);
                {
                    const bool lower = ((col >> 3) & 1) == 0;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float o = __shfl_xor_sync(0xffffffffu, v[e], 1);
                        v[e] = lower ? __fadd_rn(v[e], o) : __fsub_rn(o, v[e]);
                    }
                }
                if constexpr (NH == 32) {
                    const bool lower = ((col >> 4) & 1) == 0;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float o = __shfl_xor_sync(0xffffffffu, v[e], 2);
                        v[e] = lower ? __fadd_rn(v[e], o) : __fsub_rn(o, v[e]);
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = __fmul_rn(v[e], had_norm<NH>());
            }

            // 2-3. block amax (shuffles across the 2 or 4 lanes of the block)
            float am = 0.0f;
#pragma unroll
            for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(v[e]));
            if constexpr (AMAX_ONLY) {
                amax_acc = fmaxf(amax_acc, am);
                continue;
            } else {
                am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
                if constexpr (NB == 32) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
                float rmul, S;
                uint32_t scode = block_scale<FMT>(am, s_enc, rmul, S);

                // 4. scaled values and element rounding
                float u[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) u[e] = __fmul_rn(v[e], rmul);
                uint32_t codes;
                if constexpr (RND == kSr) {
                    const uint64_t i0 = (uint64_t)row * (uint64_t)p.k + (uint64_t)col;
                    const uint4 w0 = philox_quad(p.sr_seed, p.sr_tag_elem, i0 >> 2);
                    const uint4 w1 = philox_quad(p.sr_seed, p.sr_tag_elem, (i0 >> 2) + 1);
                    float y[8];
                    y[0] = e2m1_sr_value(u[0], uniform24(w0.x));
                    y[1] = e2m1_sr_value(u[1], uniform24(w0.y));
                    y[2] = e2m1_sr_value(u[2], uniform24(w0.z));
                    y[3] = e2m1_sr_value(u[3], uniform24(w0.w));
                    y[4] = e2m1_sr_value(u[4], uniform24(w1.x));
                    y[5] = e2m1_sr_value(u[5], uniform24(w1.y));
                    y[6] = e2m1_sr_value(u[6], uniform24(w1.z));
                    y[7] = e2m1_sr_value(u[7], uniform24(w1.w));
                    codes = e2m1x8_rn(y);
                } else {
                    codes = e2m1x8_rn(u);
                }
                if constexpr (RND == kQuartet2) {
                    // alpha = T(u*u) / T(u*q): halving-stride tree, the widest strides
                    // across lanes first, then within the thread.
                    float sa[8], sb[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        sa[e] = __fmul_rn(u[e], u[e]);
                        sb[e] = __fmul_rn(u[e], e2m1_decode((codes >> (4 * e)) & 15u));
                    }
                    if constexpr (NB == 32) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            sa[e] = __fadd_rn(sa[e], __shfl_xor_sync(0xffffffffu, sa[e], 2));
                            sb[e] = __fadd_rn(sb[e], __shfl_xor_sync(0xffffffffu, sb[e], 2));
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        sa[e] = __fadd_rn(sa[e], __shfl_xor_sync(0xffffffffu, sa[e], 1));
                        sb[e] = __fadd_rn(sb[e], __shfl_xor_sync(0xffffffffu, sb[e], 1));
                    }
#pragma unroll
                    for (int st = 4; st >= 1; st >>= 1)
#pragma unroll
                        for (int e = 0; e < st; ++e) {
                            sa[e] = __fadd_rn(sa[e], sa[e + st]);
                            sb[e] = __fadd_rn(sb[e], sb[e + st]);
                        }
                    const uint64_t bidx = (uint64_t)row * (uint64_t)(p.k / NB) + (uint64_t)(col / NB);
                    scode = quartet2_scale<FMT>(sa[0], sb[0], S, p, bidx);
                }

                // 5. pack + store (codes of padded rows/columns are not stored)
                if (col_ok && row < p.rows)
                    *reinterpret_cast<uint32_t*>(p.codes + row * (p.k / 2) + col / 2) = codes;
                if ((cc & (NB / 8 - 1)) == 0) scale_stage[atom_offset(r_in_tile, (cc * 8) / NB)] = (uint8_t)scode;
            }
        }
        if constexpr (!AMAX_ONLY) {
            __syncthreads();
            store_atoms(p, scale_stage, kRowTileCols / (4 * NB), row0, col0 / NB);
            __syncthreads();
        }
    }

    if constexpr (AMAX_ONLY) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax_acc = fmaxf(amax_acc, __shfl_xor_sync(0xffffffffu, amax_acc, o));
        if ((tid & 31) == 0) red[tid >> 5] = amax_acc;
        __syncthreads();
        if (tid == 0) {
            float m = 0.0f;
            for (int w = 0; w < kThreads / 32; ++w) m = fmaxf(m, red[w]);
            p.amax_out[blockIdx.x] = m;
        }
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
template <int FMT, int RND, int NH, bool AMAX_ONLY>
__global__ void __launch_bounds__(kThreads) quant_col_kernel(const __grid_constant__ CUtensorMap tmap,
                                                             const QuantParams p) {
    constexpr int NB = AMAX_ONLY ? 16 : ((FMT == kNvfp4) ? 16 : 32);
    constexpr int G = (NH > NB) ? NH : NB;
    constexpr int TILE_ROWS = 4 * G;
    constexpr int BOX_BYTES = TILE_ROWS * 64 * 2;
    extern __shared__ __align__(1024) uint8_t dyn_smem[];
    uint8_t* tile = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(16) uint8_t scale_stage[1024];
    __shared__ __align__(8) uint64_t bar;
    __shared__ float red[33];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t tiles_c = (p.rows + kColTileCols - 1) / kColTileCols;  // output rows = x columns
    const int64_t tiles_total = tiles_c * ((p.k + TILE_ROWS - 1) / TILE_ROWS);

    if (tid == 0) {
        prefetch_tmap(&tmap);
        mbar_init(&bar, 1);
        fence_mbarrier_init();
    }
    __syncthreads();

    float s_enc = 1.0f;
    if constexpr (!AMAX_ONLY && FMT == kNvfp4) s_enc = nvfp4_encode_scale(p, red, blockIdx.x == 0);
    if constexpr (!AMAX_ONLY && FMT == kMxfp4) {
        if (blockIdx.x == 0 && tid == 0) *p.tensor_scale = 1.0f;
    }
    float amax_acc = 0.0f;
    uint32_t phase = 0;
    bool ok = true;

    for (int64_t tile_id = blockIdx.x; tile_id < tiles_total; tile_id += gridDim.x) {
        const int64_t c0 = (tile_id % tiles_c) * kColTileCols;
        const int64_t tr = tile_id / tiles_c;
        const int64_t r0 = tr * TILE_ROWS;
        if (tid == 0) {
            mbar_arrive_expect_tx(&bar, 2 * BOX_BYTES);
            tma_load_5d(tile, &tmap, &bar, (int32_t)c0, 0, (int32_t)(4 * tr), 0, 0);
            tma_load_5d(tile + BOX_BYTES, &tmap, &bar, (int32_t)(c0 + 64), 0, (int32_t)(4 * tr), 0, 0);
        }
        ok = mbar_wait(&bar, phase);
        phase ^= 1u;
        if (!ok) break;

        // ldmatrix lane roles: matrix mm = lane / 8, matrix row pr = lane % 8 -> (q = pr / 2, k = pr % 2)
        const int mm = lane >> 3, pr = lane & 7;
        const int s_lane = (pr & 1) + 2 * (pr >> 1) + 8 * mm;  // + 32 u
#pragma unroll
        for (int ci = 0; ci < 2; ++ci) {
            const int chunk = 2 * warp + ci;  // 16 chunks of 8 columns
            const int box = chunk >> 3, ch = chunk & 7;
            const uint32_t box_base = smem_u32(tile + box * BOX_BYTES);
            float v[G];
#pragma unroll
            for (int u = 0; u < G / 8; ++u) {
                const int s = s_lane + 32 * u;
                const uint32_t addr = box_base + s * 128 + ((ch ^ (s & 7)) << 4);
                uint32_t r0w, r1w, r2w, r3w;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                             : "=r"(r0w), "=r"(r1w), "=r"(r2w), "=r"(r3w)
                             : "r"(addr));
                v[8 * u + 0] = bf16lo(r0w); v[8 * u + 1] = bf16hi(r0w);
                v[8 * u + 2] = bf16lo(r1w); v[8 * u + 3] = bf16hi(r1w);
                v[8 * u + 4] = bf16lo(r2w); v[8 * u + 5] = bf16hi(r2w);
                v[8 * u + 6] = bf16lo(r3w); v[8 * u + 7] = bf16hi(r3w);
            }
            // this thread: x column c, group of G consecutive x rows starting at r_grp
            const int q = lane & 3;
            const int64_t c = c0 + chunk * 8 + (lane >> 2);
            const int64_t r_grp = r0 + (int64_t)G * q;

            if constexpr (NH > 0) {
#pragma unroll
                for (int hb = 0; hb < G / NH; ++hb) {
                    float* w = v + hb * NH;
#pragma unroll
                    for (int e = 0; e < NH; ++e)
                        if ((p.signs >> e) & 1u) w[e] = -w[e];
#pragma unroll
                    for (int e8 = 0; e8 < NH; e8 += 8) fwht8(w + e8);
                    fwht_wide<NH>(w);
#pragma unroll
                    for (int e = 0; e < NH; ++e) w[e] = __fmul_rn(w[e], had_norm<NH>());
                }
            }

            if constexpr (AMAX_ONLY) {
#pragma unroll
                for (int e = 0; e < G; ++e) amax_acc = fmaxf(amax_acc, fabsf(v[e]));
            } else {
                const bool store_codes = (c < p.rows) && (r_grp < p.k);
                const int cl = (int)(c - c0);
#pragma unroll
                for (int b = 0; b < G / NB; ++b) {
                    const float* vb = v + b * NB;
                    float am = 0.0f;
#pragma unroll
                    for (int e = 0; e < NB; ++e) am = fmaxf(am, fabsf(vb[e]));
                    float rmul, S;
                    uint32_t scode = block_scale<FMT>(am, s_enc, rmul, S);
                    float u[NB];
#pragma unroll
                    for (int e = 0; e < NB; ++e) u[e] = __fmul_rn(vb[e], rmul);
                    const int64_t kbase = r_grp + b * NB;  // first k index of the block
                    uint32_t codes[NB / 8];
                    if constexpr (RND == kSr) {
                        const uint64_t i0 = (uint64_t)c * (uint64_t)p.k + (uint64_t)kbase;
#pragma unroll
                        for (int e8 = 0; e8 < NB; e8 += 8) {
                            const uint4 w0 = philox_quad(p.sr_seed, p.sr_tag_elem, (i0 + e8) >> 2);
                            const uint4 w1 = philox_quad(p.sr_seed, p.sr_tag_elem, ((i0 + e8) >> 2) + 1);
                            float y[8];
                            y[0] = e2m1_sr_value(u[e8 + 0], uniform24(w0.x));
                            y[1] = e2m1_sr_value(u[e8 + 1], uniform24(w0.y));
                            y[2] = e2m1_sr_value(u[e8 + 2], uniform24(w0.z));
                            y[3] = e2m1_sr_value(u[e8 + 3], uniform24(w0.w));
                            y[4] = e2m1_sr_value(u[e8 + 4], uniform24(w1.x));
                            y[5] = e2m1_sr_value(u[e8 + 5], uniform24(w1.y));
                            y[6] = e2m1_sr_value(u[e8 + 6], uniform24(w1.z));
                            y[7] = e2m1_sr_value(u[e8 + 7], uniform24(w1.w));
                            codes[e8 / 8] = e2m1x8_rn(y);
                        }
                    } else {
#pragma unroll
                        for (int e8 = 0; e8 < NB; e8 += 8) codes[e8 / 8] = e2m1x8_rn(u + e8);
                    }
                    if constexpr (RND == kQuartet2) {
                        float sa[NB], sb[NB];
#pragma unroll
                        for (int e = 0; e < NB; ++e) {
                            sa[e] = __fmul_rn(u[e], u[e]);
                            sb[e] = __fmul_rn(u[e], e2m1_decode((codes[e / 8] >> (4 * (e & 7))) & 15u));
                        }
#pragma unroll
                        for (int st = NB / 2; st >= 1; st >>= 1)
#pragma unroll
                            for (int e = 0; e < st; ++e) {
                                sa[e] = __fadd_rn(sa[e], sa[e + st]);
                                sb[e] = __fadd_rn(sb[e], sb[e + st]);
                            }
                        const uint64_t bidx = (uint64_t)c * (uint64_t)(p.k / NB) + (uint64_t)(kbase / NB);
                        scode = quartet2_scale<FMT>(sa[0], sb[0], S, p, bidx);
                    }
                    if (store_codes) {
                        uint8_t* dst = p.codes + c * (p.k / 2) + kbase / 2;
                        if constexpr (NB == 16)
                            *reinterpret_cast<uint2*>(dst) = make_uint2(codes[0], codes[1]);
                        else
                            *reinterpret_cast<uint4*>(dst) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
                    }
                    scale_stage[atom_offset(cl, (G * q) / NB + b)] = (uint8_t)scode;
                }
            }
        }
        __syncthreads();  // all ldmatrix reads done before the next TMA overwrites the tile
        if constexpr (!AMAX_ONLY) {
            store_atoms(p, scale_stage, G / NB, c0, r0 / NB);
            __syncthreads();
        }
    }

    if constexpr (AMAX_ONLY) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax_acc = fmaxf(amax_acc, __shfl_xor_sync(0xffffffffu, amax_acc, o));
        if (lane == 0) red[warp] = amax_acc;
        __syncthreads();
        if (tid == 0) {
            float m = 0.0f;
            for (int w = 0; w < kThreads / 32; ++w) m = fmaxf(m, red[w]);
            p.amax_out[blockIdx.x] = m;
        }
    }
}

template <int FMT, int RND, int NH>
cudaError_t launch_quant_t(const QuantParams& p, int axis, const CUtensorMap* tmap, cudaStream_t s) {
    if (axis == 0) {
        const int64_t tiles = ((p.rows + kRowTileRows - 1) / kRowTileRows) * ((p.k + kRowTileCols - 1) / kRowTileCols);
        quant_row_kernel<FMT, RND, NH, false><<<(unsigned)tiles, kThreads, 0, s>>>(p);
    } else {
        constexpr int NB = (FMT == kNvfp4) ? 16 : 32;
        constexpr int G = (NH > NB) ? NH : NB;
        const int64_t tiles = ((p.rows + kColTileCols - 1) / kColTileCols) * ((p.k + 4 * G - 1) / (4 * G));
        const int smem = 2 * (4 * G * 64 * 2) + 1024;
        auto kern = quant_col_kernel<FMT, RND, NH, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)tiles, kThreads, smem, s>>>(*tmap, p);
    }
    count_launch();
    return cudaGetLastError();
}

template <int FMT, int RND>
cudaError_t dispatch_nh(const QuantParams& p, int nh, int axis, const CUtensorMap* tmap, cudaStream_t s) {
    switch (nh) {
        case 0: return launch_quant_t<FMT, RND, 0>(p, axis, tmap, s);
        case 16: return launch_quant_t<FMT, RND, 16>(p, axis, tmap, s);
        default: return launch_quant_t<FMT, RND, 32>(p, axis, tmap, s);
    }
}

template <int NH>
cudaError_t launch_amax_t(const QuantParams& p, int axis, const CUtensorMap* tmap, int n_partials, cudaStream_t s) {
    if (axis == 0) {
        quant_row_kernel<kNvfp4, kRtn, NH, true><<<n_partials, kThreads, 0, s>>>(p);
    } else {
        constexpr int G = (NH > 16) ? NH : 16;
        const int smem = 2 * (4 * G * 64 * 2) + 1024;
        auto kern = quant_col_kernel<kNvfp4, kRtn, NH, true>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kern<<<n_partials, kThreads, smem, s>>>(*tmap, p);
    }
    count_launch();
    return cudaGetLastError();
}

// Max of n partial maxima (one CTA).
__global__ void __launch_bounds__(kThreads) reduce_max_kernel(const float* in, int n, float* out) {
    __shared__ float red[33];
    float m = 0.0f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, in[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w]);
        *out = fmaxf(m, red[0]);
    }
}

}  // namespace

cudaError_t launch_reduce_max(const float* in, int n, float* out, cudaStream_t s) {
    reduce_max_kernel<<<1, kThreads, 0, s>>>(in, n, out);
    count_launch();
    return cudaGetLastError();
}

int col_group(int block, int nh) { return nh > block ? nh : block; }

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

cudaError_t launch_amax(const QuantParams& p, int axis, int nh, const CUtensorMap* tmap, int n_partials,
                        cudaStream_t s) {
    switch (nh) {
        case 0: return launch_amax_t<0>(p, axis, tmap, n_partials, s);
        case 16: return launch_amax_t<16>(p, axis, tmap, n_partials, s);
        default: return launch_amax_t<32>(p, axis, tmap, n_partials, s);
    }
}

}  // namespace qfp4
