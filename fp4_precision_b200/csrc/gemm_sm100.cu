// gemm_sm100.cu - block-scaled FP4 GEMM on the sm_100a tensor cores.
//
// D = gA * gB * (A . B^T), A [M x K] and B [N x K] packed E2M1 (K-major, two
// per byte) with one scale per 16 (NVFP4, E4M3) or 32 (MXFP4, E8M0) elements
// along K. These are the linear layer's Fprop, Dgrad and Wgrad products (page
// "New AMD paper overturns conventional wisdom: FP4 training...", section
// "Poiskovaya eksperimental'naya rabota").
//
// Persistent CTAs (one per SM) walk 128 x 256 tiles of D in a grouped order
// (8 row-tiles at a time, so concurrent CTAs share A and B tiles in L2) with
// tcgen05.mma (kind::mxf4nvf4 with scale_vec::4X for NVFP4, kind::mxf4 with
// scale_vec::2X for MXFP4), M = 128, N = 256, K = 64 per instruction, fp32
// accumulator in tensor memory:
//   warp 0, one lane: TMA producer. Per 256-wide k-tile it loads the A and B
//     tiles (128-byte swizzled) and, with plain bulk copies, the scale atoms,
//     which the quantizers already store in the MMA's 512-byte atom layout,
//     into a 4-stage shared-memory ring.
//   warp 1, one lane: MMA issuer. Per k-tile it copies the scale atoms to
//     tensor memory (tcgen05.cp 32x128b.warpx4), issues 4 MMAs and commits the
//     stage back to the producer.
//   warps 2-9: epilogue. Two warps per 32-lane quarter of tensor memory each
//     drain 128 accumulator columns into registers (tcgen05.ld), hand the
//     accumulator back to the MMA warp, then multiply by gA * gB and store
//     bf16 or fp32 rows while the next tile's MMAs run.
// Every wait is bounded (qfp4_device.cuh); on expiry the kernel raises the
// device error word and skips the rest of its work.
#include <cuda_fp16.h>

#include "qfp4_device.cuh"
#include "qfp4_internal.h"

namespace qfp4 {
namespace {

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK;  // BK in elements
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK / 2;  // 16 KiB
constexpr int B_STAGE = BN * BK / 2;  // 32 KiB
constexpr int SFA_STAGE = 2048;       // up to 4 atoms
constexpr int SFB_STAGE = 4096;       // 2 row blocks x up to 4 atoms
constexpr int TMEM_COLS = 512;
constexpr int TMEM_D = 0, TMEM_SFA = 256, TMEM_SFB = 272;
constexpr int SMEM_BYTES = STAGES * (A_STAGE + B_STAGE + SFA_STAGE + SFB_STAGE) + 1024 /*align*/ + 256 /*barriers*/;

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

// Descriptor of a 32-row x 16-byte contiguous matrix (a scale atom) for tcgen05.cp:
// no swizzle, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t atom_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(128 >> 4) << 16;   // leading byte offset
    d |= (uint64_t)(128 >> 4) << 32;   // stride byte offset
    d |= (uint64_t)1 << 46;
    return d;
}

// Instruction descriptor of the block-scaled MMA: E2M1 x E2M1, K-major
// operands, M = 128, N = 256, scale type E4M3 (NVFP4) or E8M0 (MXFP4), and the
// byte of the 32-bit scale column each operand's scales start at.
template <int FMT>
__device__ __forceinline__ uint32_t idesc(uint32_t a_sf_id, uint32_t b_sf_id) {
    uint32_t d = 0;
    d |= (b_sf_id & 3u) << 4;
    d |= 1u << 7;                 // A: E2M1
    d |= 1u << 10;                // B: E2M1
    d |= (uint32_t)(BN >> 3) << 17;
    d |= (FMT == kMxfp4 ? 1u : 0u) << 23;
    d |= (uint32_t)(BM >> 4) << 24;
    d |= (a_sf_id & 3u) << 29;
    return d;
}

template <int FMT>
__device__ __forceinline__ void mma_bs(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t id, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate) {
    if constexpr (FMT == kNvfp4) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
                d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(id), "r"(sfa), "r"(sfb), "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
                d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(id), "r"(sfa), "r"(sfb), "r"(accumulate)
            : "memory");
    }
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

// Persistent tile order: groups of GROUP_M row-tiles, walking down the group
// first, so the CTAs running at one time share both A and B tiles in L2.
constexpr int GROUP_M = 8;
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int& mb, int& nb) {
    const int per_group = GROUP_M * num_n;
    const int first_m = (t / per_group) * GROUP_M;
    const int gm = min(num_m - first_m, GROUP_M);
    const int r = t % per_group;
    mb = first_m + r % gm;
    nb = r / gm;
}

constexpr int kEpiWarps = 8;                      // 2 per TMEM lane quarter, 128 columns each
constexpr int kGemmThreads = (2 + kEpiWarps) * 32;  // producer, MMA issuer, epilogue

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
    uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + STAGES * SFB_STAGE);
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;
    uint64_t* acc_empty = acc_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);

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
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kEpiWarps);
        fence_mbarrier_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, num_m, num_n, mb, nb);
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
                    mbar_arrive_expect_tx(&full[s], A_STAGE + B_STAGE + atoms * 512 * (1 + nrb));
                    tma_load_2d(sA + s * A_STAGE, &tmA, &full[s], kt * (BK / 2), mb * BM);
                    tma_load_2d(sB + s * B_STAGE, &tmB, &full[s], kt * (BK / 2), n0);
                    const int64_t katom = (int64_t)kt * ATOMS_PER_KT;
                    bulk_load(sSFA + s * SFA_STAGE, p.sfa + ((int64_t)mb * p.atoms_k + katom) * 512, atoms * 512,
                              &full[s]);
                    for (int rb = 0; rb < nrb; ++rb)
                        bulk_load(sSFB + s * SFB_STAGE + rb * (ATOMS_PER_KT * 512),
                                  p.sfb + ((int64_t)(n0 / 128 + rb) * p.atoms_k + katom) * 512, atoms * 512, &full[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int it = 0, lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++lt) {
                // the epilogue has drained the previous tile's accumulator
                if (lt > 0 && !mbar_wait(acc_empty, (lt - 1) & 1)) break;
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&full[s], (it / STAGES) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int kelems = min(BK, p.K - kt * BK);
                    const int atoms = (kelems + SF_K - 1) / SF_K;
                    const uint32_t sfa_base = smem_u32(sSFA + s * SFA_STAGE);
                    const uint32_t sfb_base = smem_u32(sSFB + s * SFB_STAGE);
                    for (int a = 0; a < atoms; ++a) {
                        tc_cp_32x128b_warpx4(tmem + TMEM_SFA + 4 * a, atom_desc(sfa_base + a * 512));
                        tc_cp_32x128b_warpx4(tmem + TMEM_SFB + 8 * a, atom_desc(sfb_base + a * 512));
                        tc_cp_32x128b_warpx4(tmem + TMEM_SFB + 8 * a + 4,
                                             atom_desc(sfb_base + ATOMS_PER_KT * 512 + a * 512));
                    }
                    const uint32_t a_base = smem_u32(sA + s * A_STAGE);
                    const uint32_t b_base = smem_u32(sB + s * B_STAGE);
                    const int kblocks = kelems / 64;
                    for (int j = 0; j < kblocks; ++j) {
                        const uint64_t ad = sw128_desc(a_base + j * 32);
                        const uint64_t bd = sw128_desc(b_base + j * 32);
                        uint32_t sfa_t, sfb_t, id;
                        if constexpr (FMT == kNvfp4) {
                            sfa_t = tmem + TMEM_SFA + 4 * j;
                            sfb_t = tmem + TMEM_SFB + 8 * j;
                            id = idesc<FMT>(0, 0);
                        } else {
                            sfa_t = tmem + TMEM_SFA + 4 * (j >> 1);
                            sfb_t = tmem + TMEM_SFB + 8 * (j >> 1);
                            id = idesc<FMT>(2 * (j & 1), 2 * (j & 1));
                        }
                        mma_bs<FMT>(tmem + TMEM_D, ad, bd, id, sfa_t, sfb_t, (kt > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);
                }
                tc_commit(acc_full);  // the tile's accumulator is complete
            }
        }
    } else {
        // ---------------- epilogue: warps 2..9 ----------------
        const int lq = warp & 3;          // TMEM lane quarter this warp may access
        const int chalf = (warp - 2) >> 2;  // which 128 accumulator columns
        const float scale = __fmul_rn(__ldg(p.ga), __ldg(p.gb));
        int lt = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
            int mb, nb;
            tile_coords(t, num_m, num_n, mb, nb);
            if (!mbar_wait(acc_full, lt & 1)) break;
            tc_fence_after();
            uint32_t acc[128];
            const uint32_t taddr = tmem + ((uint32_t)(lq * 32) << 16) + TMEM_D + chalf * 128;
            tmem_ld_32x32b_x32(taddr + 0, acc + 0);
            tmem_ld_32x32b_x32(taddr + 32, acc + 32);
            tmem_ld_32x32b_x32(taddr + 64, acc + 64);
            tmem_ld_32x32b_x32(taddr + 96, acc + 96);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);  // the MMA may start the next tile

            const int row = mb * BM + lq * 32 + lane;
            const int nbase = nb * BN + chalf * 128;
            if (row < p.M) {
                if (p.out_f32) {
                    float* dst = reinterpret_cast<float*>(p.D) + (int64_t)row * p.ldd + nbase;
#pragma unroll
                    for (int c = 0; c < 128; c += 4) {
                        const float4 v4 = make_float4(__fmul_rn(__uint_as_float(acc[c]), scale),
                                                      __fmul_rn(__uint_as_float(acc[c + 1]), scale),
                                                      __fmul_rn(__uint_as_float(acc[c + 2]), scale),
                                                      __fmul_rn(__uint_as_float(acc[c + 3]), scale));
                        if (nbase + c + 4 <= p.N) {
                            *reinterpret_cast<float4*>(dst + c) = v4;
                        } else {
                            if (nbase + c < p.N) dst[c] = v4.x;
                            if (nbase + c + 1 < p.N) dst[c + 1] = v4.y;
                            if (nbase + c + 2 < p.N) dst[c + 2] = v4.z;
                        }
                    }
                } else {
                    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.D) + (int64_t)row * p.ldd + nbase;
#pragma unroll
                    for (int c = 0; c < 128; c += 8) {
                        uint32_t w[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            __nv_bfloat162 b2 =
                                __floats2bfloat162_rn(__fmul_rn(__uint_as_float(acc[c + 2 * h]), scale),
                                                      __fmul_rn(__uint_as_float(acc[c + 2 * h + 1]), scale));
                            w[h] = *reinterpret_cast<uint32_t*>(&b2);
                        }
                        if (nbase + c + 8 <= p.N) {
                            *reinterpret_cast<uint4*>(dst + c) = make_uint4(w[0], w[1], w[2], w[3]);
                        } else {
#pragma unroll
                            for (int h = 0; h < 8; ++h)
                                if (nbase + c + h < p.N)
                                    reinterpret_cast<uint16_t*>(dst)[c + h] = (uint16_t)(w[h >> 1] >> (16 * (h & 1)));
                        }
                    }
                }
            }
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

}  // namespace

cudaError_t launch_gemm(const GemmParams& p, int fmt, const CUtensorMap* tmapA, const CUtensorMap* tmapB,
                        cudaStream_t s, int sms) {
    const int tiles = ((p.M + BM - 1) / BM) * ((p.N + BN - 1) / BN);
    const int grid = tiles < sms ? tiles : sms;
    cudaError_t e;
    if (fmt == kNvfp4) {
        e = cudaFuncSetAttribute(gemm_bs_fp4_kernel<kNvfp4>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        gemm_bs_fp4_kernel<kNvfp4><<<grid, kGemmThreads, SMEM_BYTES, s>>>(*tmapA, *tmapB, p);
    } else {
        e = cudaFuncSetAttribute(gemm_bs_fp4_kernel<kMxfp4>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        gemm_bs_fp4_kernel<kMxfp4><<<grid, kGemmThreads, SMEM_BYTES, s>>>(*tmapA, *tmapB, p);
    }
    count_launch();
    return cudaGetLastError();
}

}  // namespace qfp4
