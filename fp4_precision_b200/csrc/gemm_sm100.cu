// gemm_sm100.cu - block-scaled FP4 GEMM on the sm_100a tensor cores.
//
// D = gA * gB * (A . B^T), A [M x K] and B [N x K] packed E2M1 (K-major, two
// per byte) with one scale per 16 (NVFP4, E4M3) or 32 (MXFP4, E8M0) elements
// along K. These are the linear layer's Fprop, Dgrad and Wgrad products (page
// "New AMD paper overturns conventional wisdom: FP4 training...", section
// "Poiskovaya eksperimental'naya rabota").
//
// Two kernels share one structure: persistent CTAs (one per SM) walk the
// output tiles in a grouped order (a few row-tiles at a time, so CTAs running
// together share A and B tiles in L2) and issue tcgen05.mma (kind::mxf4nvf4,
// scale_vec::4X for NVFP4; kind::mxf4, scale_vec::2X for MXFP4) with K = 64 per
// instruction and an fp32 accumulator in tensor memory.
//   - CTA pair (default for more than 128 rows of A): 256 x 256 tiles on the
//     two SMs of a cluster with tcgen05.mma.cta_group::2, M = 256, N = 256;
//     each CTA loads half of A and half of B, so an SM moves 32 KiB of
//     operands (+ 6 KiB of scales) per 256-wide k-tile;
//   - single CTA: 128 x 256 tiles, M = 128, N = 256, 48 KiB (+ 6 KiB) per SM
//     per k-tile. Measured on B200, one SM's TMA fill tops out near 106 bytes
//     per cycle, so 54 KiB per 512 cycles of MMA leaves the single-CTA
//     kernel no headroom; the pair kernel's 38 KiB leaves ~30 %.
// Warp roles (14 warps):
//   warp 0, one lane: TMA producer into a shared-memory ring (A and B tiles
//     with 128-byte swizzle, and the scale atoms, which the quantizers store in
//     the MMA's 512-byte atom layout).
//   warp 1, one lane: MMA issuer: one barrier wait, 4 MMAs per 256-wide
//     k-tile and ONE commit, which frees both the ring stage and its
//     tensor-memory scale slot.
//   warps 2-5: scale writers, one per 32-lane quarter of tensor memory. They
//     read the k-tile's scale atoms from shared memory and write them with
//     tcgen05.st into the scale slot of the same index as the ring stage (each
//     quarter holds the same 32 atom rows, as the MMA reads them), then wait
//     for the stage's operand tiles before signalling the MMA warp.
//   warps 6-13: epilogue, two per lane quarter, 128 accumulator columns each:
//     drain tensor memory to registers (tcgen05.ld), hand the accumulator back
//     to the MMA warp before the global stores (bf16) or after the first 32
//     columns (fp32), multiply by gA * gB and store rows while the next tile's
//     MMAs run.
// The tensor pipe queues only a few MMAs, so the issuing thread's work between
// k-tiles shows up directly as idle tensor cycles. Measured on B200: a second
// commit per k-tile cost ~90 cycles per k-tile, a runtime-trip-count MMA loop
// ~160 and descriptors rebuilt from addresses ~50, against 512 cycles of MMA
// work. Hence the single commit, the unrolled 4-MMA k-tile and descriptors
// advanced by adding to a base. (An earlier design copied the scales with
// tcgen05.cp from the MMA thread; at ~110 cycles per copy and 12 per k-tile
// that serialised the tensor pipe.)
// Every wait is bounded (qfp4_device.cuh); on expiry the kernel raises the
// device error word and skips the rest of its work.
#include <cuda_fp16.h>

#include "qfp4_device.cuh"
#include "qfp4_internal.h"

namespace qfp4 {
namespace {

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK;  // BK in elements
constexpr int TMEM_COLS = 512;
// Tensor-memory columns: the 128 x 256 fp32 accumulator, then one scale slot
// of 48 columns (SFA 16, SFB 32) per ring stage (4 stages single, 5 pair: at
// most 256 + 5 * 48 = 496 columns).
constexpr int TMEM_D = 0;
__device__ __forceinline__ uint32_t sfa_col(int slot) { return 256u + 48u * (uint32_t)slot; }
__device__ __forceinline__ uint32_t sfb_col(int slot) { return 256u + 48u * (uint32_t)slot + 16u; }

constexpr int kScaleWarps = 4;
constexpr int kEpiWarps = 8;
constexpr int kFirstScaleWarp = 2, kFirstEpiWarp = 6;
constexpr int kGemmThreads = (2 + kScaleWarps + kEpiWarps) * 32;

// Shared-memory matrix descriptor (tcgen05): K-major, 128-byte swizzle, rows
// 128 bytes apart, 8-row groups 1024 bytes apart, descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);   // start address
    d |= (uint64_t)1 << 16;                     // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;           // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;                     // version
    d |= (uint64_t)2 << 61;                     // SWIZZLE_128B
    return d;
}

// Instruction descriptor of the block-scaled MMA: E2M1 x E2M1, K-major
// operands, M = 128, N = 256, scale type E4M3 (NVFP4) or E8M0 (MXFP4), and the
// byte of the 32-bit scale column each operand's scales start at.
template <int FMT, int MM, int NN>
__device__ __forceinline__ uint32_t idesc_mn(uint32_t a_sf_id, uint32_t b_sf_id) {
    uint32_t d = 0;
    d |= (b_sf_id & 3u) << 4;
    d |= 1u << 7;                 // A: E2M1
    d |= 1u << 10;                // B: E2M1
    d |= (uint32_t)(NN >> 3) << 17;
    d |= (FMT == kMxfp4 ? 1u : 0u) << 23;
    d |= (uint32_t)(MM >> 4) << 24;
    d |= (a_sf_id & 3u) << 29;
    return d;
}
// tcgen05.mma with block scaling, for one CTA or (PAIR) a CTA pair.
#define QFP4_MMA_ASM(GROUP, KIND)                                                                                     \
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"                                                      \
                 "tcgen05.mma.cta_group::" GROUP ".kind::" KIND " [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d_tmem), \
                 "l"(a_desc), "l"(b_desc), "r"(id), "r"(sfa), "r"(sfb), "r"(accumulate)                               \
                 : "memory")
template <int FMT, bool PAIR>
__device__ __forceinline__ void mma_bs(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t id, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate) {
    if constexpr (FMT == kNvfp4 && !PAIR) QFP4_MMA_ASM("1", "mxf4nvf4.block_scale.scale_vec::4X");
    if constexpr (FMT == kNvfp4 && PAIR) QFP4_MMA_ASM("2", "mxf4nvf4.block_scale.scale_vec::4X");
    if constexpr (FMT == kMxfp4 && !PAIR) QFP4_MMA_ASM("1", "mxf4.block_scale.scale_vec::2X");
    if constexpr (FMT == kMxfp4 && PAIR) QFP4_MMA_ASM("2", "mxf4.block_scale.scale_vec::2X");
}
#undef QFP4_MMA_ASM

// One K = 64 block j (0-3) of a k-tile: operand descriptors advance 32 bytes
// (2 in the 16-byte address field) per block; NVFP4 scales take one 4-column
// group per block, MXFP4 scales one per two blocks, the odd block reading the
// upper two bytes of each scale word (scale-factor id 2).
template <int FMT, bool PAIR, int MM>
__device__ __forceinline__ void mma_kblock(uint32_t d, uint64_t ad, uint64_t bd, uint32_t sfa, uint32_t sfb, int j,
                                           bool overwrite) {
    uint32_t sa, sb, id;
    if constexpr (FMT == kNvfp4) {
        sa = sfa + 4u * (uint32_t)j;
        sb = sfb + 8u * (uint32_t)j;
        id = idesc_mn<FMT, MM, BN>(0, 0);
    } else {
        sa = sfa + 4u * (uint32_t)(j >> 1);
        sb = sfb + 8u * (uint32_t)(j >> 1);
        id = idesc_mn<FMT, MM, BN>(2u * (j & 1), 2u * (j & 1));
    }
    mma_bs<FMT, PAIR>(d, ad + 2u * (uint32_t)j, bd + 2u * (uint32_t)j, id, sa, sb, overwrite ? 0u : 1u);
}
// The MMAs of one k-tile of kb K = 64 blocks; a full k-tile (kb = 4) is
// unrolled so the issuing thread does no loop work between MMAs.
template <int FMT, bool PAIR, int MM>
__device__ __forceinline__ void mma_ktile(uint32_t d, uint64_t ad, uint64_t bd, uint32_t sfa, uint32_t sfb, int kb,
                                          bool first) {
    if (kb == 4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_kblock<FMT, PAIR, MM>(d, ad, bd, sfa, sfb, j, first && j == 0);
    } else {
        for (int j = 0; j < kb; ++j) mma_kblock<FMT, PAIR, MM>(d, ad, bd, sfa, sfb, j, first && j == 0);
    }
}

// 32 lanes x 16 consecutive fp32 columns of TMEM into registers (no wait).
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
        "[%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
// 32 lanes x 32 consecutive fp32 columns of TMEM into registers (no wait).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Registers of 32 lanes into 8 / 16 / 32 consecutive 32-bit TMEM columns.
__device__ __forceinline__ void tmem_st_x1(uint32_t taddr, uint32_t r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r) : "memory");
}
__device__ __forceinline__ uint32_t lds32(uint32_t saddr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(saddr));
    return v;
}
__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t* r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Scale writer for TMEM lane quarter q (lanes 32q..32q+31): lane i copies
// line i of the k-tile's scale atoms from shared memory into TMEM lane 32q + i.
// Line i of an atom holds four words, word w the four scales of row i + 32w;
// in tensor memory word w goes to column base + w (the layout
// tcgen05.cp.32x128b.warpx4 produces). The MMA computes output row 32q + i in
// lane quarter q, so for A it reads only word q of each line: only that
// column is written. Every quarter needs all B rows: SFB gets all four words
// of both 128-row blocks. SFA atom a -> column sfa_col + 4a + q; SFB atom a of
// row block rb -> columns sfb_col + 8a + 4rb .. +3.
template <int ATOMS>
__device__ __forceinline__ void write_scales(uint32_t tmem_lane, int slot, uint32_t sfa_smem, uint32_t sfb_smem,
                                             int lane, int q) {
    uint32_t ra[ATOMS], rb[8 * ATOMS];
#pragma unroll
    for (int a = 0; a < ATOMS; ++a) {
        ra[a] = lds32(sfa_smem + a * 512 + lane * 16 + q * 4);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const uint4 w = lds128(sfb_smem + r * (ATOMS * 512) + a * 512 + lane * 16);
            rb[8 * a + 4 * r + 0] = w.x; rb[8 * a + 4 * r + 1] = w.y;
            rb[8 * a + 4 * r + 2] = w.z; rb[8 * a + 4 * r + 3] = w.w;
        }
    }
#pragma unroll
    for (int a = 0; a < ATOMS; ++a) tmem_st_x1(tmem_lane + sfa_col(slot) + 4u * a + (uint32_t)q, ra[a]);
    if constexpr (ATOMS == 4) {
        tmem_st_x32(tmem_lane + sfb_col(slot), rb);
    } else {
        tmem_st_x16(tmem_lane + sfb_col(slot), rb);
    }
    tc_wait_st();
}

// Scaled accumulator pair as two packed bf16 (one packed fp32x2 multiply, one
// conversion).
__device__ __forceinline__ uint32_t pack_bf16(uint32_t a, uint32_t b, float scale) {
    const float2 v = __fmul2_rn(make_float2(__uint_as_float(a), __uint_as_float(b)), make_float2(scale, scale));
    __nv_bfloat162 h = __float22bfloat162_rn(v);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Extents (bytes) of D and of the MXFP4 copy of the output, for the
// bounds-checked build.
__device__ __forceinline__ int64_t d_extent(const GemmParams& p) {
    return p.M <= 0 ? 0 : ((int64_t)(p.M - 1) * p.ldd + p.N) * (p.out_f32 ? 4 : 2);
}
__device__ __forceinline__ int64_t q_codes_extent(const GemmParams& p) { return (int64_t)p.M * (p.N / 2); }
__device__ __forceinline__ int64_t q_scales_extent(const GemmParams& p) {
    return (int64_t)((p.M + 127) / 128) * (p.q_kb4 / 4) * 512;
}

// Epilogue stores of one row's NC columns from column n0, with evict-first
// stores so the output stream does not push the operand tiles out of L2.
// bf16: NC / 2 packed words; fp32: NC accumulator words times gA * gB.
template <int NC>
__device__ __forceinline__ void store_bf16(const GemmParams& p, const uint32_t* w, int row, int n0) {
    if (row >= p.M) return;
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.D) + (int64_t)row * p.ldd + n0;
#pragma unroll
    for (int c = 0; c < NC; c += 8)
        __stcs(chk(reinterpret_cast<uint4*>(dst + c), p.D, d_extent(p)),
               make_uint4(w[c / 2], w[c / 2 + 1], w[c / 2 + 2], w[c / 2 + 3]));
}
// Ragged right edge: the first nv (< NC) of NC bf16 columns, element by element.
template <int NC>
__device__ __forceinline__ void store_bf16_edge(const GemmParams& p, const uint32_t* w, int row, int n0) {
    if (row >= p.M) return;
    uint16_t* d16 = reinterpret_cast<uint16_t*>(p.D) + (int64_t)row * p.ldd + n0;
    const int nv = p.N - n0;
#pragma unroll
    for (int c = 0; c < NC; ++c)
        if (c < nv) *chk(d16 + c, p.D, d_extent(p)) = (uint16_t)(w[c >> 1] >> (16 * (c & 1)));
}
template <int NC>
__device__ __forceinline__ void store_f32(const GemmParams& p, uint32_t* acc, int row, int n0, float scale) {
    if (row >= p.M) return;
    float* dst = reinterpret_cast<float*>(p.D) + (int64_t)row * p.ldd + n0;
#pragma unroll
    for (int c = 0; c < NC; c += 2) {
        const float2 v = __fmul2_rn(make_float2(__uint_as_float(acc[c]), __uint_as_float(acc[c + 1])),
                                    make_float2(scale, scale));
        acc[c] = __float_as_uint(v.x);
        acc[c + 1] = __float_as_uint(v.y);
    }
    if (p.accumulate) {  // D += result: one fp32 add per element (each element has one owner)
        const int nv = p.N - n0;
#pragma unroll
        for (int c = 0; c < NC; ++c)
            if (c < nv) {
                float* d = chk(dst + c, p.D, d_extent(p));
                *d = __fadd_rn(*d, __uint_as_float(acc[c]));
            }
    } else if (n0 + NC <= p.N) {
#pragma unroll
        for (int c = 0; c < NC; c += 4)
            __stcs(chk(reinterpret_cast<uint4*>(dst + c), p.D, d_extent(p)),
                   make_uint4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]));
    } else {  // ragged right edge: nv < NC valid columns, whole 4-column chunks first
        const int nv = p.N - n0, nfull = nv >> 2, rem = nv & 3;
        uint32_t* d32 = reinterpret_cast<uint32_t*>(dst);
#pragma unroll
        for (int c = 0; c < NC; c += 4) {
            if ((c >> 2) < nfull) {
                __stcs(chk(reinterpret_cast<uint4*>(dst + c), p.D, d_extent(p)),
                       make_uint4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]));
            } else if ((c >> 2) == nfull && rem != 0) {
#pragma unroll
                for (int h = 0; h < 3; ++h)
                    if (h < rem) *chk(d32 + c + h, p.D, d_extent(p)) = acc[c + h];
            }
        }
    }
}

// Epilogue of one tile for one warp: 128 accumulator columns of its lane
// quarter. The accumulator goes back to the MMA warp (release()) as soon as
// the values are in registers: all 128 columns for bf16 output (packed, 64
// registers), the last 96 for fp32 after the first 32 are stored.
template <typename Release>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, uint32_t taddr, int row, int n0, float scale,
                                              Release release) {
    if (!p.out_f32 && n0 + 128 > p.N) {
        // ragged right edge (rare): 16 columns at a time, released after the last load
#pragma unroll 1
        for (int h = 0; h < 8; ++h) {
            uint32_t acc[16], w[8];
            tmem_ld_32x32b_x16(taddr + 16 * h, acc);
            tc_wait_ld();
            if (h == 7) {
                tc_fence_before();
                __syncwarp();
                release();
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) w[c] = pack_bf16(acc[2 * c], acc[2 * c + 1], scale);
            if (n0 + 16 * h < p.N) store_bf16_edge<16>(p, w, row, n0 + 16 * h);
        }
    } else if (!p.out_f32) {
        uint32_t w[64];
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // two round trips of 64 columns
            uint32_t acc[64];
            tmem_ld_32x32b_x32(taddr + 64 * h, acc);
            tmem_ld_32x32b_x32(taddr + 64 * h + 32, acc + 32);
            tc_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) w[32 * h + c] = pack_bf16(acc[2 * c], acc[2 * c + 1], scale);
        }
        tc_fence_before();
        __syncwarp();
        release();
        store_bf16<128>(p, w, row, n0);
    } else {
        uint32_t acc[80];
        tmem_ld_32x32b_x16(taddr, acc);
        tmem_ld_32x32b_x32(taddr + 16, acc + 16);
        tc_wait_ld();
        store_f32<48>(p, acc, row, n0, scale);
        tmem_ld_32x32b_x16(taddr + 48, acc);
        tmem_ld_32x32b_x32(taddr + 64, acc + 16);
        tmem_ld_32x32b_x32(taddr + 96, acc + 48);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        release();
        store_f32<80>(p, acc, row, n0 + 48, scale);
    }
}

// The next layer's operand from the epilogue: row r's 128 output columns from
// n0, as packed bf16 words w (the values just stored as D), quantized to MXFP4
// along N exactly as the row quantizer does it (round to nearest, a Hadamard of
// size NHQ with sign bits p.q_signs applied to the bf16 words, the floor
// exponent): four 32-element blocks, 16 bytes of codes each, one scale word.
template <int NHQ>
__device__ __forceinline__ void quantize_out_row128(const GemmParams& p, const uint32_t* w, int r, int n0) {
    using Grp = Group<kMxfp4, kRtn, NHQ>;
    static_assert(Grp::G == 32, "32-element MXFP4 blocks");
    const Stream st{0, 0, 0, 0};
    ScaleRng srng;
    uint32_t scodes[4];
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            uint32_t x = w[16 * blk + i];
            if (NHQ > 0 && p.q_signs != 0u) x ^= Grp::sign_mask(p.q_signs, i);
            v[2 * i] = bf16lo(x);
            v[2 * i + 1] = bf16hi(x);
        }
        Grp::rotate(v);
        uint32_t codes[4];
        Grp::quantize(v, 1.0f, nullptr, st, 0, 0, srng, codes, scodes + blk);
        if (r < p.M && n0 + 32 * blk < p.N)
            *chk(reinterpret_cast<uint4*>(p.q_codes + (int64_t)r * (p.N / 2) + (n0 + 32 * blk) / 2), p.q_codes,
                 q_codes_extent(p)) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
    }
    // rows up to the 128-row padding of the atoms; past M the accumulator is
    // zero (zero-filled A rows), so those scales are the zero padding
    if (r < (p.M + 127) / 128 * 128) {
        const int64_t kb0 = n0 / 32;
        *chk(reinterpret_cast<uint32_t*>(p.q_scales + ((int64_t)(r / 128) * (p.q_kb4 / 4) + kb0 / 4) * 512 +
                                         (r % 32) * 16 + ((r / 32) % 4) * 4),
             p.q_scales, q_scales_extent(p)) = scodes[0] | (scodes[1] << 8) | (scodes[2] << 16) | (scodes[3] << 24);
    }
}

// The NVFP4 tensor amax of the output along its rows, as the next layer's
// quantizer takes it: max |v| over one row's 128 columns (the packed bf16
// words w, exactly the values stored in D) after the rotation of size AMX
// (none, 16 or 32; the sign flips as XORs on the bf16 words, then the
// butterflies) without its 1/sqrt(n_h) factor, which is applied once to the
// CTA's maximum (rounding c * y is monotone in y). Output columns past N are
// zero (zero-filled B rows) and groups never straddle N (a multiple of the
// group), so padding adds nothing.
template <int AMX>
__device__ __forceinline__ float row128_rot_amax(const uint32_t* w, uint32_t signs, float m) {
    using Grp = Group<kNvfp4, kRtn, AMX>;
    constexpr int G = Grp::G;
#pragma unroll
    for (int g = 0; g < 128 / G; ++g) {
        float v[G];
#pragma unroll
        for (int i = 0; i < G / 2; ++i) {
            uint32_t x = w[g * (G / 2) + i];
            if (AMX > 0 && signs != 0u) x ^= Grp::sign_mask(signs, i);
            v[2 * i] = bf16lo(x);
            v[2 * i + 1] = bf16hi(x);
        }
        Grp::template rotate<false>(v);
        m = abs_max<G>(m, v);
    }
    return m;
}

// Epilogue of one tile for one warp with TMA stores (bf16 output): its 32
// rows x 128 columns of the accumulator go to registers (packed bf16), the
// accumulator is released, then each 64-column half is written row by row into
// the warp's 4 KiB shared-memory box in the 128-byte swizzled layout (chunk j
// of row r at chunk j ^ (r % 8): conflict-free) and stored by one TMA bulk
// store, which writes whole lines and clips rows >= M and columns >= N. The
// box is rewritten only after the previous store has read it.
template <int NHQ, int AMX, typename Release>
__device__ __forceinline__ void epilogue_tile_tma(const GemmParams& p, const CUtensorMap* tmD, uint32_t taddr, int row0,
                                                  int n0, float scale, uint32_t obox, int lane, float& amax_acc,
                                                  Release release) {
    uint32_t w[64];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t acc[64];
        tmem_ld_32x32b_x32(taddr + 64 * h, acc);
        tmem_ld_32x32b_x32(taddr + 64 * h + 32, acc + 32);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) w[32 * h + c] = pack_bf16(acc[2 * c], acc[2 * c + 1], scale);
    }
    tc_fence_before();
    __syncwarp();
    release();
    const uint32_t rbase = obox + (uint32_t)lane * 128u;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 8; ++j)
            sts128(rbase + ((uint32_t)(j ^ (lane & 7)) << 4), w[32 * h + 4 * j], w[32 * h + 4 * j + 1],
                   w[32 * h + 4 * j + 2], w[32 * h + 4 * j + 3]);
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0 && row0 < p.M && n0 + 64 * h < p.N) {  // boxes wholly outside D are skipped
            tma_store_2d(tmD, obox, n0 + 64 * h, row0);
            bulk_commit_group();
        }
    }
    if constexpr (NHQ >= 0) {
        if (n0 < p.N) quantize_out_row128<NHQ>(p, w, row0 + lane, n0);
    }
    if constexpr (AMX >= 0) amax_acc = row128_rot_amax<AMX>(w, p.amax_signs, amax_acc);
}

// fp32 output: the same with boxes of 32 rows x 32 columns (128-byte rows),
// four per warp and tile. The first 32 columns are boxed and stored before the
// accumulator is released, the other 96 are held in registers across it.
__device__ __forceinline__ void box_f32(const GemmParams& p, const CUtensorMap* tmD, uint32_t obox, int lane,
                                        const uint32_t* acc, int row0, int x, float scale) {
    if (lane == 0) bulk_wait_group_read0();
    __syncwarp();
    const uint32_t rbase = obox + (uint32_t)lane * 128u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float2 a = __fmul2_rn(make_float2(__uint_as_float(acc[4 * j]), __uint_as_float(acc[4 * j + 1])),
                                    make_float2(scale, scale));
        const float2 b = __fmul2_rn(make_float2(__uint_as_float(acc[4 * j + 2]), __uint_as_float(acc[4 * j + 3])),
                                    make_float2(scale, scale));
        sts128(rbase + ((uint32_t)(j ^ (lane & 7)) << 4), __float_as_uint(a.x), __float_as_uint(a.y),
               __float_as_uint(b.x), __float_as_uint(b.y));
    }
    fence_proxy_async_shared();
    __syncwarp();
    if (lane == 0 && row0 < p.M && x < p.N) {
        if (p.accumulate)
            tma_reduce_add_2d(tmD, obox, x, row0);
        else
            tma_store_2d(tmD, obox, x, row0);
        bulk_commit_group();
    }
}
template <typename Release>
__device__ __forceinline__ void epilogue_tile_tma_f32(const GemmParams& p, const CUtensorMap* tmD, uint32_t taddr,
                                                      int row0, int n0, float scale, uint32_t obox, int lane,
                                                      Release release) {
    uint32_t acc[96];
    tmem_ld_32x32b_x32(taddr, acc);
    tc_wait_ld();
    box_f32(p, tmD, obox, lane, acc, row0, n0, scale);
    tmem_ld_32x32b_x32(taddr + 32, acc);
    tmem_ld_32x32b_x32(taddr + 64, acc + 32);
    tmem_ld_32x32b_x32(taddr + 96, acc + 64);
    tc_wait_ld();
    tc_fence_before();
    __syncwarp();
    release();
#pragma unroll
    for (int b = 0; b < 3; ++b) box_f32(p, tmD, obox, lane, acc + 32 * b, row0, n0 + 32 * (b + 1), scale);
}

// Grouped tile order: GM row-tiles at a time, walking down the group first.
template <int GM>
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int& mb, int& nb) {
    const int per_group = GM * num_n;
    const int first_m = (t / per_group) * GM;
    const int gm = min(num_m - first_m, GM);
    const int r = t % per_group;
    mb = first_m + r % gm;
    nb = r / gm;
}

// ===========================================================================
// Single-CTA kernel: 128 x 256 tiles.
// ===========================================================================
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK / 2;  // 16 KiB
constexpr int B_STAGE = BN * BK / 2;  // 32 KiB
constexpr int SFA_STAGE = 2048;       // up to 4 atoms
constexpr int SFB_STAGE = 4096;       // 2 row blocks x up to 4 atoms
constexpr int SMEM_BYTES = STAGES * (A_STAGE + B_STAGE + SFA_STAGE + SFB_STAGE) + 1024 + 256;
constexpr int GROUP_M = 16;

template <int FMT>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bs_fp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const GemmParams p) {
    constexpr int SF_K = (FMT == kNvfp4) ? 64 : 128;  // K elements covered by one scale atom
    constexpr int ATOMS_PER_KT = BK / SF_K;            // 4 or 2
    extern __shared__ __align__(1024) uint8_t dyn_smem[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = base;
    uint8_t* sB = sA + STAGES * A_STAGE;
    uint8_t* sSFA = sB + STAGES * B_STAGE;
    uint8_t* sSFB = sSFA + STAGES * SFA_STAGE;
    uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + STAGES * SFB_STAGE);  // A and B of stage s landed
    uint64_t* empty = full + STAGES;      // stage s and scale slot s free again
    uint64_t* sf_load = empty + STAGES;   // scale atoms of stage s landed
    uint64_t* sf_full = sf_load + STAGES; // scale slot s written
    uint64_t* acc_full = sf_full + STAGES;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_empty + 1;      // every MMA this CTA issued has completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = (p.K + BK - 1) / BK;
    const int num_m = (p.M + BM - 1) / BM, num_n = (p.N + BN - 1) / BN;
    const int tiles = num_m * num_n;

    if (threadIdx.x == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_load[s], 1);
            mbar_init(&sf_full[s], kScaleWarps);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kEpiWarps);
        mbar_init(drain, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();  // the operands' quantizers have completed (and the previous readers of D)
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                int mb, nb;
                tile_coords<GROUP_M>(t, num_m, num_n, mb, nb);
                const int n0 = nb * BN;
                const int nrb = (n0 + 128 < p.N) ? 2 : 1;  // B row blocks present in the scale buffer
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % STAGES;
                    if (it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) + 1) & 1)) {
                        ok = false;
                        break;
                    }
                    const int kelems = min(BK, p.K - kt * BK);
                    const int atoms = (kelems + SF_K - 1) / SF_K;
                    // scale atoms first, on their own barrier: the scale writers
                    // start while the operand tiles are still in flight
                    mbar_arrive_expect_tx(&sf_load[s], atoms * 512 * (1 + nrb));
                    const int64_t katom = (int64_t)kt * ATOMS_PER_KT;
                    bulk_load(sSFA + s * SFA_STAGE, p.sfa + ((int64_t)mb * p.atoms_k + katom) * 512, atoms * 512,
                              &sf_load[s]);
                    for (int rb = 0; rb < nrb; ++rb)
                        bulk_load(sSFB + s * SFB_STAGE + rb * (ATOMS_PER_KT * 512),
                                  p.sfb + ((int64_t)(n0 / 128 + rb) * p.atoms_k + katom) * 512, atoms * 512,
                                  &sf_load[s]);
                    mbar_arrive_expect_tx(&full[s], A_STAGE + B_STAGE);
                    tma_load_2d(sA + s * A_STAGE, &tmA, &full[s], kt * (BK / 2), mb * BM);
                    tma_load_2d(sB + s * B_STAGE, &tmB, &full[s], kt * (BK / 2), n0);
                }
            }
            drain_loads(full, sf_load, STAGES, it);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint64_t a_desc0 = sw128_desc(smem_u32(sA)), b_desc0 = sw128_desc(smem_u32(sB));
            int s = 0, lt = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++lt) {
                if (lt > 0 && !mbar_wait(acc_empty, (lt - 1) & 1)) break;
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt) {
                    // sf_full[s] completes after the scale writers saw full[s]:
                    // one wait covers the operand tiles and the scales
                    if (!mbar_wait(&sf_full[s], ph)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    mma_ktile<FMT, false, BM>(tmem + TMEM_D, a_desc0 + (uint64_t)(s * (A_STAGE >> 4)),
                                              b_desc0 + (uint64_t)(s * (B_STAGE >> 4)), tmem + sfa_col(s),
                                              tmem + sfb_col(s), min(BK, p.K - kt * BK) / 64, kt == 0);
                    tc_commit(&empty[s]);  // stage s and scale slot s are free once these MMAs finish
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                tc_commit(acc_full);
            }
            // no MMA may still write tensor memory or read shared memory when
            // the CTA frees them (after a timed-out wait too)
            tc_commit(drain);
            (void)mbar_wait(drain, 0);
        }
    } else if (warp < kFirstEpiWarp) {
        // ---------------- scale writers ----------------
        // Stage s's scale atoms arriving (sf_load[s]) implies the MMAs that
        // last read scale slot s have finished: the producer refills a stage
        // only after their commit.
        const uint32_t tmem_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            for (int kt = 0; kt < KT; ++kt) {
                if (!mbar_wait(&sf_load[s], ph)) {
                    ok = false;
                    break;
                }
                write_scales<ATOMS_PER_KT>(tmem_lane, s, smem_u32(sSFA + s * SFA_STAGE), smem_u32(sSFB + s * SFB_STAGE),
                                           lane, warp & 3);
                if (!mbar_wait(&full[s], ph)) {  // the operand tiles too, so the MMA waits once
                    ok = false;
                    break;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_full[s]);
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1;
                }
            }
        }
    } else {
        // ---------------- epilogue ----------------
        const int lq = warp & 3;
        const int chalf = (warp - kFirstEpiWarp) >> 2;
        const float scale = __fmul_rn(__ldg(p.ga), __ldg(p.gb));
        int lt = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
            int mb, nb;
            tile_coords<GROUP_M>(t, num_m, num_n, mb, nb);
            if (!mbar_wait(acc_full, lt & 1)) break;
            tc_fence_after();
            epilogue_tile(p, tmem + ((uint32_t)(lq * 32) << 16) + TMEM_D + chalf * 128, mb * BM + lq * 32 + lane,
                          nb * BN + chalf * 128, scale, [&] {
                              if (lane == 0) mbar_arrive(acc_empty);
                          });
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
        tmem_relinquish();
    }
}

// ===========================================================================
// CTA-pair kernel: 256 x 256 tiles, tcgen05.mma.cta_group::2.
// The leader (rank 0) issues the MMAs. The A and B loads of both CTAs complete
// on the leader's stage barrier; each CTA's scale atoms (its own 128 rows of
// SFA, all 256 rows of SFB; a 3-D view, out-of-range atoms read as zero)
// complete on a barrier of its own, which its scale writers wait on before
// they fill its tensor memory and arrive on the leader's scale-slot barrier.
// The leader's commits arrive on the barriers of both CTAs.
// ===========================================================================
constexpr int P_STAGES = 5;
constexpr int P_A = 128 * BK / 2;   // 16 KiB: this CTA's A rows
constexpr int P_B = 128 * BK / 2;   // 16 KiB: this CTA's B rows
constexpr int P_SFA = 4 * 512;      // up to 4 atoms of this CTA's rows
constexpr int P_SFB = 2 * 4 * 512;  // 2 row blocks x up to 4 atoms
constexpr int P_STAGE = P_A + P_B + P_SFA + P_SFB;
constexpr int P_OUT_BOX = 4096;      // one epilogue warp's TMA-store box (32 rows x 128 B)
constexpr int P_SMEM = P_STAGES * P_STAGE + kEpiWarps * P_OUT_BOX + 1024 + 512;
constexpr int P_GROUP_M = 4;  // 256-row tiles per group of the tile order

template <int FMT, int NHQ = -1, int AMX = -1>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_bs_fp4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                            const __grid_constant__ CUtensorMap tmD, const GemmParams p) {
    constexpr int SF_K = (FMT == kNvfp4) ? 64 : 128;
    constexpr int ATOMS_PER_KT = BK / SF_K;  // 4 or 2
    constexpr uint32_t AB_TX = 2u * (P_A + P_B);            // both CTAs, on the leader
    constexpr uint32_t SF_TX = 3u * ATOMS_PER_KT * 512u;    // this CTA's scale boxes
    extern __shared__ __align__(1024) uint8_t dyn_smem[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = base;
    uint8_t* sB = sA + P_STAGES * P_A;
    uint8_t* sSFA = sB + P_STAGES * P_B;
    uint8_t* sSFB = sSFA + P_STAGES * P_SFA;
    uint8_t* sOut = sSFB + P_STAGES * P_SFB;  // kEpiWarps boxes, 1024-byte aligned
    uint64_t* full = reinterpret_cast<uint64_t*>(sOut + kEpiWarps * P_OUT_BOX);
    uint64_t* empty = full + P_STAGES;
    uint64_t* sf_load = empty + P_STAGES;   // this CTA's scale atoms of stage s landed
    uint64_t* sf_full = sf_load + P_STAGES;  // scale slot s written in both CTAs (leader's)
    uint64_t* acc_full = sf_full + P_STAGES;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_empty + 1;  // every MMA the leader issued has completed (both CTAs)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int KT = (p.K + BK - 1) / BK;
    const int num_m = (p.M + 2 * BM - 1) / (2 * BM), num_n = (p.N + BN - 1) / BN;
    const int tiles = num_m * num_n;
    const int cid = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmSFA);
        prefetch_tmap(&tmSFB);
        prefetch_tmap(&tmD);
        for (int s = 0; s < P_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_load[s], 1);
            mbar_init(&sf_full[s], 2 * kScaleWarps);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * kEpiWarps);
        mbar_init(drain, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, tensor memory allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();  // the operands' quantizers have completed (and the previous readers of D)
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = cid; t < tiles && ok; t += nclusters) {
                int mb, nb;
                tile_coords<P_GROUP_M>(t, num_m, num_n, mb, nb);
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % P_STAGES;
                    if (it >= P_STAGES && !mbar_wait_cluster(&empty[s], ((it / P_STAGES) + 1) & 1)) {
                        ok = false;
                        break;
                    }
                    // scale atoms first: the scale writers start while the
                    // operand tiles are still in flight
                    mbar_arrive_expect_tx(&sf_load[s], SF_TX);
                    tma_load_3d(sSFA + s * P_SFA, &tmSFA, &sf_load[s], 0, kt * ATOMS_PER_KT, 2 * mb + (int)rank);
                    tma_load_3d(sSFB + s * P_SFB, &tmSFB, &sf_load[s], 0, kt * ATOMS_PER_KT, 2 * nb);
                    const uint32_t bar_leader = mapa_shared(smem_u32(&full[s]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], AB_TX);
                    tma_load_2d_pair(sA + s * P_A, &tmA, bar_leader, kt * (BK / 2), mb * 2 * BM + (int)rank * BM);
                    tma_load_2d_pair(sB + s * P_B, &tmB, bar_leader, kt * (BK / 2), nb * BN + (int)rank * 128);
                }
            }
            // both CTAs' operand tiles complete on the leader's full barriers,
            // each CTA's scale atoms on its own sf_load barriers
            drain_loads(rank == 0 ? full : nullptr, sf_load, P_STAGES, it);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader CTA only) ----------------
        if (lane == 0 && rank == 0) {
            const uint64_t a_desc0 = sw128_desc(smem_u32(sA)), b_desc0 = sw128_desc(smem_u32(sB));
            int s = 0, lt = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int t = cid; t < tiles && ok; t += nclusters, ++lt) {
                if (lt > 0 && !mbar_wait_cluster(acc_empty, (lt - 1) & 1)) break;
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt) {
                    // sf_full[s] completes after the leader's scale writers saw
                    // full[s] (both CTAs' operand tiles): one wait covers all
                    if (!mbar_wait_cluster(&sf_full[s], ph)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    mma_ktile<FMT, true, 2 * BM>(tmem + TMEM_D, a_desc0 + (uint64_t)(s * (P_A >> 4)),
                                                 b_desc0 + (uint64_t)(s * (P_B >> 4)), tmem + sfa_col(s),
                                                 tmem + sfb_col(s), min(BK, p.K - kt * BK) / 64, kt == 0);
                    tc_commit_pair(&empty[s]);  // frees stage s and scale slot s in both CTAs
                    if (++s == P_STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                tc_commit_pair(acc_full);  // both CTAs' accumulators are complete
            }
            // no MMA may still write either CTA's tensor memory or read shared
            // memory when the pair frees them (after a timed-out wait too); the
            // peer is held at the final cluster barrier until then
            tc_commit_pair(drain);
            (void)mbar_wait(drain, 0);
        }
    } else if (warp < kFirstEpiWarp) {
        // ---------------- scale writers (both CTAs) ----------------
        // The producer loads stage s's scale atoms only after the commit of
        // the MMAs that last read scale slot s, so sf_load[s] implies the slot
        // is free.
        const uint32_t tmem_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int t = cid; t < tiles && ok; t += nclusters) {
            for (int kt = 0; kt < KT; ++kt) {
                if (!mbar_wait_cluster(&sf_load[s], ph)) {
                    ok = false;
                    break;
                }
                write_scales<ATOMS_PER_KT>(tmem_lane, s, smem_u32(sSFA + s * P_SFA), smem_u32(sSFB + s * P_SFB), lane,
                                           warp & 3);
                // the leader's writers also wait for both CTAs' operand tiles
                // (they complete on the leader's full[s]), so the MMA waits once
                if (rank == 0 && !mbar_wait_cluster(&full[s], ph)) {
                    ok = false;
                    break;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&sf_full[s]), 0));
                if (++s == P_STAGES) {
                    s = 0;
                    ph ^= 1;
                }
            }
        }
    } else {
        // ---------------- epilogue (both CTAs) ----------------
        const int lq = warp & 3;
        const int chalf = (warp - kFirstEpiWarp) >> 2;
        const float scale = __fmul_rn(__ldg(p.ga), __ldg(p.gb));
        const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
        const uint32_t obox = smem_u32(sOut) + (uint32_t)(warp - kFirstEpiWarp) * P_OUT_BOX;
        float amax_acc = 0.0f;
        int lt = 0;
        for (int t = cid; t < tiles; t += nclusters, ++lt) {
            int mb, nb;
            tile_coords<P_GROUP_M>(t, num_m, num_n, mb, nb);
            if (!mbar_wait_cluster(acc_full, lt & 1)) break;
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(lq * 32) << 16) + TMEM_D + chalf * 128;
            const int row0 = mb * 2 * BM + (int)rank * BM + lq * 32;
            auto release = [&] {
                if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
            };
            if (p.out_f32)
                epilogue_tile_tma_f32(p, &tmD, taddr, row0, nb * BN + chalf * 128, scale, obox, lane, release);
            else
                epilogue_tile_tma<NHQ, AMX>(p, &tmD, taddr, row0, nb * BN + chalf * 128, scale, obox, lane, amax_acc,
                                            release);
        }
        if (lane == 0) bulk_wait_group0();  // this warp's stores are complete
        if constexpr (AMX >= 0) {
            // the CTA's partial maximum: warp maxima in shared memory, one
            // barrier of the eight epilogue warps, written by the first
            __shared__ float warp_max[kEpiWarps];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax_acc = fmaxf(amax_acc, __shfl_xor_sync(0xffffffffu, amax_acc, o));
            if (lane == 0) warp_max[warp - kFirstEpiWarp] = amax_acc;
            asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32) : "memory");
            if (warp == kFirstEpiWarp && lane == 0) {
                float m = 0.0f;
#pragma unroll
                for (int i = 0; i < kEpiWarps; ++i) m = fmaxf(m, warp_max[i]);
                if constexpr (AMX > 0) m = __fmul_rn(m, AMX == 16 ? 0.25f : 0x1.6a09e6p-3f);  // fp32(1/sqrt(n_h))
                *chk(p.amax_partials + blockIdx.x, p.amax_partials, (int64_t)gridDim.x * 4) = m;
            }
        }
    }

    tc_fence_before();
    cluster_sync();  // no CTA leaves while its peer may still signal it
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
        tmem_relinquish_pair();
    }
}

}  // namespace

cudaError_t launch_gemm(const GemmParams& p, int fmt, const CUtensorMap* tmapA, const CUtensorMap* tmapB,
                        cudaStream_t s, int sms) {
    const int tiles = ((p.M + BM - 1) / BM) * ((p.N + BN - 1) / BN);
    const int grid = tiles < sms ? tiles : sms;
    cudaError_t e;
    if (fmt == kNvfp4) {
        e = cudaFuncSetAttribute(gemm_bs_fp4_kernel<kNvfp4>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        e = launch_pdl(gemm_bs_fp4_kernel<kNvfp4>, dim3(grid), dim3(kGemmThreads), SMEM_BYTES, s, *tmapA, *tmapB, p);
    } else {
        e = cudaFuncSetAttribute(gemm_bs_fp4_kernel<kMxfp4>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        e = launch_pdl(gemm_bs_fp4_kernel<kMxfp4>, dim3(grid), dim3(kGemmThreads), SMEM_BYTES, s, *tmapA, *tmapB, p);
    }
    count_launch();
    return e;
}

template <int FMT, int NHQ, int AMX = -1>
cudaError_t run_pair(const GemmParams& p, const CUtensorMap* tmapA, const CUtensorMap* tmapB,
                     const CUtensorMap* tmapSFA, const CUtensorMap* tmapSFB, const CUtensorMap* tmapD, cudaStream_t s,
                     int clusters) {
    cudaError_t e = cudaFuncSetAttribute(gemm_bs_fp4_pair_kernel<FMT, NHQ, AMX>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM);
    if (e != cudaSuccess) return e;
    return launch_pdl(gemm_bs_fp4_pair_kernel<FMT, NHQ, AMX>, dim3(2 * clusters), dim3(kGemmThreads), P_SMEM, s,
                      *tmapA, *tmapB, *tmapSFA, *tmapSFB, *tmapD, p);
}

cudaError_t launch_gemm_pair(const GemmParams& p, int fmt, const CUtensorMap* tmapA, const CUtensorMap* tmapB,
                             const CUtensorMap* tmapSFA, const CUtensorMap* tmapSFB, const CUtensorMap* tmapD,
                             cudaStream_t s, int sms, int nhq, int amx, int* n_partials) {
    const int tiles = ((p.M + 2 * BM - 1) / (2 * BM)) * ((p.N + BN - 1) / BN);
    int clusters = sms / 2;
    if (clusters > tiles) clusters = tiles;
    if (clusters < 1) clusters = 1;
    if (n_partials != nullptr) *n_partials = 2 * clusters;
    cudaError_t e;
    if (amx >= 0) {  // bf16 output with the NVFP4 tensor amax of the output
        const bool nv = fmt == kNvfp4;
        switch (amx) {
            case 0: e = nv ? run_pair<kNvfp4, -1, 0>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters)
                           : run_pair<kMxfp4, -1, 0>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters); break;
            case 16: e = nv ? run_pair<kNvfp4, -1, 16>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters)
                            : run_pair<kMxfp4, -1, 16>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters); break;
            default: e = nv ? run_pair<kNvfp4, -1, 32>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters)
                            : run_pair<kMxfp4, -1, 32>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters); break;
        }
        if (e != cudaSuccess) return e;
        count_launch();
        return cudaGetLastError();
    }
    if (fmt == kNvfp4) {
        switch (nhq) {
            case -1: e = run_pair<kNvfp4, -1>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters); break;
            case 0: e = run_pair<kNvfp4, 0>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters); break;
            case 16: e = run_pair<kNvfp4, 16>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters); break;
            default: e = run_pair<kNvfp4, 32>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters); break;
        }
    } else {
        switch (nhq) {
            case -1: e = run_pair<kMxfp4, -1>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters); break;
            case 0: e = run_pair<kMxfp4, 0>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters); break;
            case 16: e = run_pair<kMxfp4, 16>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters); break;
            default: e = run_pair<kMxfp4, 32>(p, tmapA, tmapB, tmapSFA, tmapSFB, tmapD, s, clusters); break;
        }
    }
    if (e != cudaSuccess) return e;
    count_launch();
    return cudaGetLastError();
}

}  // namespace qfp4
