// qfp4_device.cuh - device helpers shared by the sm_100a kernels of this library:
// Philox4x32-10, bf16 unpacking, FP4/FP8 conversions, the library's device
// error word, and thin inline-PTX wrappers for mbarrier, TMA and tcgen05.
#pragma once

#include <cstdint>
#include <cstdlib>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <utility>

namespace qfp4 {

// ---------------------------------------------------------------------------
// error word: set by a kernel whose bounded wait expired; read by qfp4_status()
// DEV_ERR_BOUNDS: a bounds-checked build caught a store outside its buffer
enum : uint32_t { DEV_ERR_NONE = 0, DEV_ERR_TIMEOUT = 1, DEV_ERR_BOUNDS = 2 };
// (the library is one translation unit, see qfp4_lib.cu, so this is its only definition)
__device__ uint32_t g_dev_error = 0;

__device__ __forceinline__ void raise_device_error(uint32_t code) { atomicOr(&g_dev_error, code); }

// Store-address check. In a bounds-checked build (-DQFP4_BOUNDS_CHECK, see
// fp4_precision_b200/build.py) every global store of the kernels goes through
// chk(): if the n bytes at p do not lie inside [base, base + size), it raises
// DEV_ERR_BOUNDS and returns a scratch sink instead, so nothing outside the
// buffer is written and nothing traps (qfp4_status then returns
// QFP4_ERR_BOUNDS). In the normal build chk() returns p.
__device__ __align__(16) uint8_t g_bounds_sink[64];
template <typename T>
__device__ __forceinline__ T* chk(T* p, const void* base, int64_t size, int64_t n = (int64_t)sizeof(T)) {
#ifdef QFP4_BOUNDS_CHECK
    const int64_t off = reinterpret_cast<const uint8_t*>(p) - reinterpret_cast<const uint8_t*>(base);
    if (base == nullptr || off < 0 || off + n > size || n > (int64_t)sizeof(g_bounds_sink)) {
        raise_device_error(DEV_ERR_BOUNDS);
        return reinterpret_cast<T*>(g_bounds_sink);
    }
#else
    (void)base;
    (void)size;
    (void)n;
#endif
    return p;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// A bounded wait gives up after this many nanoseconds (kernels here run for
// microseconds to milliseconds; a legitimate wait is far shorter).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): key = 64-bit seed,
// counter = (i/4 lo, i/4 hi, tag | stream << 4, 0).
__device__ __forceinline__ uint4 philox4x32_10(uint4 ctr, uint32_t key_lo, uint32_t key_hi) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        if (round != 0) {
            key_lo += 0x9E3779B9u;
            key_hi += 0xBB67AE85u;
        }
        const uint32_t m0_lo = 0xD2511F53u * ctr.x;
        const uint32_t m0_hi = __umulhi(0xD2511F53u, ctr.x);
        const uint32_t m1_lo = 0xCD9E8D57u * ctr.z;
        const uint32_t m1_hi = __umulhi(0xCD9E8D57u, ctr.z);
        ctr = make_uint4(m1_hi ^ ctr.y ^ key_lo, m1_lo, m0_hi ^ ctr.w ^ key_hi, m0_lo);
    }
    return ctr;
}

// Four consecutive words of stream (tag, stream) starting at item 4*quad.
__device__ __forceinline__ uint4 philox_quad(uint64_t seed, uint32_t tag_stream, uint64_t quad) {
    return philox4x32_10(make_uint4((uint32_t)quad, (uint32_t)(quad >> 32), tag_stream, 0u), (uint32_t)seed,
                         (uint32_t)(seed >> 32));
}

// Uniform in [0, 1) on the 2^-24 grid.
__device__ __forceinline__ float uniform24(uint32_t w) { return __uint2float_rn(w >> 8) * 0x1p-24f; }

// ---------------------------------------------------------------------------
// bf16 pairs -> fp32 (exact)
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------------------
// E2M1: two fp32 -> one byte, `lo` in the low nibble (round-to-nearest-even,
// saturating to +-6). Four pairs -> one 32-bit word, element 0 lowest.
__device__ __forceinline__ uint32_t e2m1x8_rn(const float* v) {
    uint32_t out;
    asm("{\n\t"
        ".reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t"
        "}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    // a zero magnitude keeps code 0 whatever the sign (no -0 codes)
    const uint32_t mag = out & 0x77777777u;
    const uint32_t nonzero = (mag + 0x77777777u) & 0x88888888u;
    return mag | (out & nonzero);
}

// Stochastic rounding of u onto the E2M1 grid with a 16-bit draw h, given as
// hs = h << 16: the lower grid neighbour lo, gap `step`, round up iff
// h * 2^-16 < (|u| - lo) / step; the result is the chosen grid value with the
// sign of u (magnitudes above 6 come out as 6 or 8 and saturate to 6 in the
// E2M1 conversion). Exact, in integer steps: with C the power of two just
// above |u| (at least 2), y = |u| + C rounded upward lies in [C, 2C] and the
// E2M1 gap of |u|'s binade, C/4, is y's top two mantissa bits, so lo + C is y
// with the lower 21 bits cleared and y's lower 21 bits are ceil((|u| - lo) /
// ulp(y)); h * 2^-16 < (|u| - lo) / step <=> 32 h < (|u| - lo) / ulp(y) <=>
// 32 h < ceil(...) for integer h, i.e. h << 16 < y << 11 unsigned. When the
// upward rounding carries into the gap bits (|u| within an ulp below a grid
// point) the fraction left is 0 and the result is that grid point, which is
// also the exact outcome there (the true fraction exceeds 1 - 2^-16).
__device__ __forceinline__ float e2m1_sr_value(float u, uint32_t hs) {
    const uint32_t b = __float_as_uint(u);
    const uint32_t cb = max((b & 0x7F800000u) + 0x00800000u, 0x40000000u);
    const float c = __uint_as_float(cb);
    const uint32_t yb = __float_as_uint(__fadd_ru(fabsf(u), c));
    const uint32_t mb = (yb & 0xFFE00000u) + (hs < (yb << 11) ? 0x00200000u : 0u);
    const float m = __fsub_rn(__uint_as_float(mb), c);  // exact: mb in [c, 2c]
    return __uint_as_float(__float_as_uint(m) | (b & 0x80000000u));
}

// E2M1 code value (signed) of a 4-bit code.
__device__ __forceinline__ float e2m1_decode(uint32_t code) {
    const uint32_t idx = code & 7u;
    float m = (idx < 4u) ? 0.5f * (float)idx : (idx == 4u ? 2.0f : (idx == 5u ? 3.0f : (idx == 6u ? 4.0f : 6.0f)));
    return (code & 8u) ? -m : m;
}

// ---------------------------------------------------------------------------
// E4M3 (OCP FN): fp32 -> code, round-to-nearest-even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_rn(float t) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
    return r & 0xFFu;
}

// E4M3 code -> fp32 (exact, through f16).
__device__ __forceinline__ float e4m3_decode(uint32_t code) {
    uint32_t h2;
    const uint16_t c = (uint16_t)code;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// Stochastic rounding of t >= 0 onto the E4M3 grid (saturating at 448) with
// the Philox word w (uniform rho = (w >> 8) * 2^-24): code of the largest
// E4M3 value lo <= t, plus one iff rho < (t - lo) / gap.
// For t in [2^-6, 448) (normal E4M3 values, 3 mantissa bits) lo is t with its
// fp32 mantissa cut to 3 bits, the code is the fp32 exponent and top 3
// mantissa bits rebased (bias 127 -> 7), and (t - lo) / gap is exactly the
// cut-off 20 mantissa bits over 2^20, so the comparison is an integer one:
// (w >> 8) < (those 20 bits) * 16. Below 2^-6 (subnormal E4M3, gap 2^-9):
// t * 2^9 split into integer code and fraction. Both candidates are formed
// and the right one selected (no branches: both are cheap and a branch costs
// more in the issue-bound quantizers).
__device__ __forceinline__ uint32_t e4m3_sr(float t, uint32_t w) {
    const uint32_t b = __float_as_uint(t);
    const uint32_t normal = ((b >> 20) - (120u << 3)) + ((w >> 8) < ((b & 0xFFFFFu) << 4) ? 1u : 0u);
    const float x = t * 512.0f;  // exact
    const float fl = floorf(x);
    const uint32_t sub = (uint32_t)fl + (uniform24(w) < x - fl ? 1u : 0u);
    const uint32_t c = t >= 0x1p-6f ? normal : sub;
    return t < 448.0f ? c : 0x7Eu;
}

// floor(log2(a)) of a positive finite fp32, exact (subnormals included).
__device__ __forceinline__ int floor_log2(float a) {
    const uint32_t b = __float_as_uint(a);
    const int e = (int)((b >> 23) & 0xFFu);
    if (e != 0) return e - 127;
    return (31 - __clz((int)(b & 0x7FFFFFu))) - 149;
}

// 2^e as fp32 for e in [-149, 127] (exact).
__device__ __forceinline__ float exp2i(int e) {
    if (e >= -126) return __uint_as_float((uint32_t)(e + 127) << 23);
    return __uint_as_float(1u << (e + 149));
}

// Stochastic rounding of t > 0 onto powers of two; returns the E8M0 code.
__device__ __forceinline__ uint32_t e8m0_sr(float t, float rho) {
    int e = floor_log2(t);
    const float lo = exp2i(e);
    // (t - lo) / lo with lo = 2^e: an exact multiplication while 2^-e is finite
    const float p = e >= -126 ? (t - lo) * exp2i(-e) : (t - lo) / lo;
    if (rho < p) e += 1;
    e = e < -127 ? -127 : (e > 127 ? 127 : e);
    return (uint32_t)(e + 127);
}

// ---------------------------------------------------------------------------
// shared-memory / barrier / TMA / tcgen05 wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Wait for the phase with the given parity to complete; false (and the
// device error word set) when the wait exceeded limit_ns.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        for (int i = 0; i < 256; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) {
            raise_device_error(DEV_ERR_TIMEOUT);
            return false;
        }
    }
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    return mbar_wait_for(bar, parity, kWaitLimitNs);
}

// Before a TMA producer thread leaves: wait (bounded) until the loads of its
// last min(issued, stages) ring iterations have landed, so that no TMA write
// into this CTA's shared memory is outstanding when the CTA exits, also after a
// timed-out wait cut the loop short. full and sf_load (either may be null:
// none, or waited elsewhere) are the ring's completion barriers; iteration i
// used stage i % stages with phase parity (i / stages) & 1, which is each
// barrier's latest armed phase.
__device__ __forceinline__ void drain_loads(uint64_t* full, uint64_t* sf_load, int stages, int issued) {
    for (int i = issued > stages ? issued - stages : 0; i < issued; ++i) {
        const uint32_t par = (uint32_t)((i / stages) & 1);
        if (full != nullptr && !mbar_wait(&full[i % stages], par)) return;
        if (sf_load != nullptr && !mbar_wait(&sf_load[i % stages], par)) return;
    }
}

// The same wait with cluster-scope acquire: for barriers the peer CTA of a
// pair arrives on.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        for (int i = 0; i < 256; ++i)
            if (mbar_try_wait_cluster(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            raise_device_error(DEV_ERR_TIMEOUT);
            return false;
        }
    }
}

// 2D/5D tiled TMA load into shared memory, completing on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}
// 2D tiled TMA store of a shared-memory box (bulk-group completion); the
// tensor map clips the parts of the box outside the tensor.
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src_smem, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(tmap),
                 "r"(src_smem), "r"(x), "r"(y)
                 : "memory");
}
// Element-wise fp32 add of a shared-memory box into global memory (TMA
// reduce; the tensor map's element type is fp32).
__device__ __forceinline__ void tma_reduce_add_2d(const void* tmap, uint32_t src_smem, int32_t x, int32_t y) {
    asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     tmap),
                 "r"(src_smem), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// This thread's committed bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// This thread's committed bulk stores are complete.
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void sts128(uint32_t saddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t saddr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(saddr));
    return v;
}
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int32_t x, int32_t y,
                                            int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const void* tmap, uint64_t* bar, int32_t c0, int32_t c1, int32_t c2,
                                            int32_t c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, "
        "%6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void tma_load_5d(void* dst, const void* tmap, uint64_t* bar, int32_t c0, int32_t c1, int32_t c2,
                                            int32_t c3, int32_t c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, "
        "%7}], [%2];" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
        : "memory");
}
// Untiled bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// tcgen05 (5th-generation tensor core) wrappers
__device__ __forceinline__ void tmem_alloc(uint32_t* slot_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// Copy a 32-row x 128-bit shared-memory matrix (512 contiguous bytes) to TMEM
// lanes 0-31 at 4 columns, replicated into the four 32-lane sub-partitions.
__device__ __forceinline__ void tc_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// CTA-pair (cluster of 2) helpers for the 2-SM tensor-core path
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on an mbarrier given by its shared::cluster address (possibly the
// peer's), with the default (CTA-scope release) semantics. The arriving
// threads have already waited for their own tensor-memory operations
// (tcgen05.wait::st / ::ld) and fenced them (tcgen05.fence::before_thread_sync),
// which is all the peer's tensor-core work needs. Measured on B200: the
// .release.cluster form cost ~1500 cycles per arrive, longer than a k-tile's
// MMAs.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA loads into this CTA's shared memory whose completion is counted on the
// pair's leader barrier (`bar_cluster`, a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const void* tmap, uint32_t bar_cluster, int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
        "[%2];" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(bar_cluster), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const void* tmap, uint32_t bar_cluster, int32_t x, int32_t y,
                                                 int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
        "%5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Arrive on the barrier at `bar` in both CTAs of the pair when all prior
// tcgen05 operations of this thread have completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
    const uint16_t mask = 0x3;
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "h"(mask)
                 : "memory");
}
// Each CTA of the pair copies its own 512-byte scale atom at `sdesc` into its
// own tensor memory at `taddr`.
__device__ __forceinline__ void tc_cp_pair_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}


// ---------------------------------------------------------------------------
// Programmatic dependent launch. Every kernel of the library is launched with
// programmatic stream serialization, so the next kernel on the stream can be
// scheduled while this one drains; each kernel does its set-up that touches
// no global memory (barrier init, tensor-memory allocation, descriptor
// prefetch), then waits (griddepcontrol.wait: the previous grid has completed
// and its writes are visible) before its first global read or write, and
// lets its own dependents launch (they start as its CTAs exit and wait the
// same way). QFP4_PDL=0 launches without the attribute (same results).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

inline bool pdl_enabled() {
    const char* e = std::getenv("QFP4_PDL");
    return !(e != nullptr && e[0] == '0');
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace qfp4
