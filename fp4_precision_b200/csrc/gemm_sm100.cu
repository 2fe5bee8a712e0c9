// gemm_sm100.cu - block-scaled FP4 GEMM on the sm_100a tensor cores.
//
// D = gA * gB * (A . B^T), A [M x K] and B [N x K] packed E2M1 (K-major, two
// per byte) with one scale per 16 (NVFP4, E4M3) or 32 (MXFP4, E8M0) elements
// along K. These are the linear layer's Fprop, Dgrad and Wgrad products (page
// "New AMD paper overturns conventional wisdom: FP4 training...", section
// "Poiskovaya eksperimental'naya rabota").
//
// One CTA computes a 128 x 256 tile of D with tcgen05.mma (kind::mxf4nvf4 with
// scale_vec::4X for NVFP4, kind::mxf4 with scale_vec::2X for MXFP4), M = 128,
// N = 256, K = 64 per instruction, fp32 accumulator in tensor memory:
//   warp 0, one lane: TMA producer. Per 256-wide k-tile it loads the A and B
//     tiles (128-byte swizzled) and, with plain bulk copies, the scale atoms,
//     which the quantizers already store in the MMA's 512-byte atom layout,
//     into a 4-stage shared-memory ring.
//   warp 1, one lane: MMA issuer. Per k-tile it copies the scale atoms to
//     tensor memory (tcgen05.cp 32x128b.warpx4), issues 4 MMAs and commits the
//     stage back to the producer.
//   warps 0-3: epilogue. Each reads its 32 accumulator lanes (tcgen05.ld),
//     multiplies by gA * gB and stores bf16 or fp32 rows.
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

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float* out) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    tc_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) out[i] = __uint_as_float(r[i]);
}

template <int FMT>
__global__ void __launch_bounds__(128, 1)
    gemm_bs_fp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const GemmParams p) {
    constexpr int SF_K = (FMT == kNvfp4) ? 64 : 128;   // K elements covered by one scale atom
    constexpr int ATOMS_PER_KT = BK / SF_K;             // 4 or 2
    extern __shared__ __align__(1024) uint8_t dyn_smem[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = base;
    uint8_t* sB = sA + STAGES * A_STAGE;
    uint8_t* sSFA = sB + STAGES * B_STAGE;
    uint8_t* sSFB = sSFA + STAGES * SFA_STAGE;
    uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + STAGES * SFB_STAGE);
    uint64_t* empty = full + STAGES;
    uint64_t* done = empty + STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int KT = (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer ----------------
        const int mblk = m0 / 128;
        for (int kt = 0; kt < KT; ++kt) {
            const int s = kt % STAGES;
            if (kt >= STAGES && !mbar_wait(&empty[s], ((kt / STAGES) + 1) & 1)) break;
            const int kelems = min(BK, p.K - kt * BK);
            const int atoms = (kelems + SF_K - 1) / SF_K;
            const int nrb = (n0 + 128 < p.N) ? 2 : 1;  // B row blocks present in the scale buffer
            mbar_arrive_expect_tx(&full[s], A_STAGE + B_STAGE + atoms * 512 * (1 + nrb));
            tma_load_2d(sA + s * A_STAGE, &tmA, &full[s], kt * (BK / 2), m0);
            tma_load_2d(sB + s * B_STAGE, &tmB, &full[s], kt * (BK / 2), n0);
            const int64_t katom = (int64_t)kt * ATOMS_PER_KT;
            bulk_load(sSFA + s * SFA_STAGE, p.sfa + ((int64_t)mblk * p.atoms_k + katom) * 512, atoms * 512, &full[s]);
            for (int rb = 0; rb < nrb; ++rb)
                bulk_load(sSFB + s * SFB_STAGE + rb * (ATOMS_PER_KT * 512),
                          p.sfb + ((int64_t)(n0 / 128 + rb) * p.atoms_k + katom) * 512, atoms * 512, &full[s]);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer ----------------
        bool ok = true;
        for (int kt = 0; kt < KT && ok; ++kt) {
            const int s = kt % STAGES;
            if (!mbar_wait(&full[s], (kt / STAGES) & 1)) {
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
                tc_cp_32x128b_warpx4(tmem + TMEM_SFB + 8 * a + 4, atom_desc(sfb_base + ATOMS_PER_KT * 512 + a * 512));
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
        tc_commit(done);
    }

    // ---------------- epilogue: all four warps ----------------
    __syncwarp();
    const bool ok = mbar_wait(done, 0);
    tc_fence_after();
    const int row = m0 + warp * 32 + lane;
    const float scale = __fmul_rn(__ldg(p.ga), __ldg(p.gb));
    if (ok && p.K > 0) {
        for (int c = 0; c < BN / 32; ++c) {
            float acc[32];
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + TMEM_D + c * 32, acc);
            const int n = n0 + c * 32;
            if (row >= p.M || n >= p.N) continue;
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[i] = __fmul_rn(acc[i], scale);
            if (p.out_f32) {
                float* dst = reinterpret_cast<float*>(p.D) + (int64_t)row * p.ldd + n;
                if (n + 32 <= p.N) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(dst + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (n + i < p.N) dst[i] = acc[i];
                }
            } else {
                __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.D) + (int64_t)row * p.ldd + n;
                uint32_t packed[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
                    packed[i] = *reinterpret_cast<uint32_t*>(&h);
                }
                if (n + 32 <= p.N) {
#pragma unroll
                    for (int i = 0; i < 16; i += 4)
                        *reinterpret_cast<uint4*>(dst + 2 * i) =
                            make_uint4(packed[i], packed[i + 1], packed[i + 2], packed[i + 3]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (n + i < p.N) dst[i] = __float2bfloat16_rn(acc[i]);
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
                        cudaStream_t s) {
    dim3 grid((p.N + BN - 1) / BN, (p.M + BM - 1) / BM);
    cudaError_t e;
    if (fmt == kNvfp4) {
        e = cudaFuncSetAttribute(gemm_bs_fp4_kernel<kNvfp4>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        gemm_bs_fp4_kernel<kNvfp4><<<grid, 128, SMEM_BYTES, s>>>(*tmapA, *tmapB, p);
    } else {
        e = cudaFuncSetAttribute(gemm_bs_fp4_kernel<kMxfp4>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        gemm_bs_fp4_kernel<kMxfp4><<<grid, 128, SMEM_BYTES, s>>>(*tmapA, *tmapB, p);
    }
    count_launch();
    return cudaGetLastError();
}

}  // namespace qfp4
