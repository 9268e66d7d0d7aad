// tcgen05 / TMEM / mbarrier wrappers and operand-layout helpers shared by the tensor-core
// kernels (sn_ef_tc.cu: edges, sn_node_tc.cu: atoms).  sm_100a only.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sn_internal.cuh"

namespace sn {
namespace tc {

constexpr int WGT = 128;         // threads per warpgroup (thread t of a group <-> TMEM lane t)
constexpr int FF = 128;          // feature width of the tensor-core kernels
constexpr float LN2F = 0.693147180559945309f;

// ------------------------------------------------------------------ PTX wrappers (sm_100a)
static __device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

static __device__ __forceinline__ void tmem_alloc(uint32_t holder, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(holder), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

static __device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

static __device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
static __device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
static __device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

static __device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

static __device__ __forceinline__ void mma_commit(uint32_t mbar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}

// Non-blocking test of a barrier phase (never suspends the thread).
static __device__ __forceinline__ uint32_t mbar_test_wait(uint32_t mbar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(mbar), "r"(parity)
        : "memory");
    return ok;
}

// 16-byte asynchronous copy global -> shared (both 16-byte aligned), and an arrival on mbar
// once every earlier such copy of this thread has landed (counted in the barrier's expected
// arrivals: .noinc).
static __device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

static __device__ __forceinline__ void cp_async_arrive(uint32_t mbar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(mbar) : "memory");
}

// Named barrier over n threads that also returns whether all of them passed a true predicate.
static __device__ __forceinline__ int named_sync_and(int id, int n, int pred)
{
    int out;
    asm volatile(
        "{\n\t.reg .pred q, p;\n\tsetp.ne.s32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, %3, q;\n\tselp.s32 %0, 1, 0, p;\n\t}\n"
        : "=r"(out)
        : "r"(pred), "r"(id), "r"(n)
        : "memory");
    return out;
}

static __device__ __forceinline__ void named_sync(int id, int n)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

static __device__ __forceinline__ void mbar_arrive(uint32_t mbar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

static __device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

// Wait for a barrier phase, suspending the thread (it issues nothing meanwhile) until the phase
// completes or about 0.2 ms have passed; false in the latter case.  Callers loop on it with
// their own time bound.
static __device__ __forceinline__ uint32_t mbar_try_wait(uint32_t mbar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(mbar), "r"(parity), "r"(200000u)
        : "memory");
    return ok;
}

// Expect `bytes` of asynchronous copies on mbar (counts as this phase's one arrival).
static __device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes)
                 : "memory");
}

// Bulk copy global -> this CTA's shared memory (no multicast), completing on mbar.  Both
// addresses 16-byte aligned, bytes a multiple of 16.
static __device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t mbar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}

// Tensor-memory-accelerator gather (sm_100a): rows r0..r3 of the 2-D tensor described by the
// tensor map at map (generic address of a __grid_constant__ parameter; boxes one row high,
// starting at column x, which must be a multiple of 16 bytes' worth of elements) into four
// consecutive box-sized rows of this CTA's shared memory at dst (128-byte aligned), completing
// on mbar.  No multicast.
static __device__ __forceinline__ void tma_gather4(uint32_t dst, const void *map, int x, int r0, int r1, int r2,
                                                   int r3, uint32_t mbar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
        "l"(map), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(mbar)
        : "memory");
}

// Bounded wait of the whole CTA for phase 0 of mbar (the weight copies); false on time-out.
static __device__ __forceinline__ bool wait_copies(uint32_t mbar, int *d_err)
{
    int ok = 1;
    const long long t0 = clock64();
    while (!mbar_try_wait(mbar, 0))
        if (clock64() - t0 > (1ll << 33)) {
            ok = 0;
            break;
        }
    ok = __syncthreads_and(ok);
    if (!ok && threadIdx.x == 0) atomicOr(d_err, ERRBIT_TIMEOUT);
    return ok != 0;
}

// This lane's 32 consecutive 32-bit TMEM columns starting at taddr (warp w reads lanes 32w..).
static __device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// This lane's 16 consecutive 32-bit TMEM columns starting at taddr.
static __device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Two 16-column loads (this lane's columns at ta and at tb) completed by one wait.
static __device__ __forceinline__ void tmem_ld16_pair(uint32_t ta, uint32_t tb, float (&a)[16], float (&b)[16])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%32];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
        "%29, %30, %31}, [%33];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(ta), "r"(tb)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        a[i] = __uint_as_float(r[i]);
        b[i] = __uint_as_float(r[16 + i]);
    }
}

// This lane's 8 consecutive 32-bit TMEM columns starting at taddr.
static __device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8])
{
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

template <int CH>
static __device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[CH])
{
    static_assert(CH == 8 || CH == 16 || CH == 32, "8, 16 or 32 columns");
    if constexpr (CH == 32) tmem_ld32(taddr, v);
    else if constexpr (CH == 16) tmem_ld16(taddr, v);
    else tmem_ld8(taddr, v);
}

// 16 lanes x 64 bits, 16 repetitions: thread t of the warp receives lane 8 (t % 2) + t / 4 of
// the 16 lanes starting at taddr's lane, columns 2 r + (t / 2) % 2 for r = 0..15 (32 columns in
// all), so the 16 lanes of an M = 64 accumulator quadrant are spread over all 32 threads.
static __device__ __forceinline__ void tmem_ld16x64b_x16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x64b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor, no swizzle (layout type 0), version 1.
static __device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

// Instruction descriptor for kind::f16: fp16 A and B, fp32 D, dense.
static constexpr uint32_t idesc_f16(int M, int N, int a_mn_major, int b_mn_major)
{
    return (1u << 4) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------------ helpers

// 8 values -> one 16-byte fp16 run (hi) and, for SPLIT, the run of residuals (lo)
template <bool SPLIT>
static __device__ __forceinline__ void store8(unsigned char *hi, unsigned char *lo, uint32_t off, const float *v)
{
    __half2 h[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) h[q] = __floats2half2_rn(v[2 * q], v[2 * q + 1]);
    *reinterpret_cast<uint4 *>(hi + off) = make_uint4(*reinterpret_cast<uint32_t *>(&h[0]), *reinterpret_cast<uint32_t *>(&h[1]),
                                                      *reinterpret_cast<uint32_t *>(&h[2]), *reinterpret_cast<uint32_t *>(&h[3]));
    if (SPLIT) {
        __half2 l[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 b = __half22float2(h[q]);
            l[q] = __floats2half2_rn(v[2 * q] - b.x, v[2 * q + 1] - b.y);
        }
        *reinterpret_cast<uint4 *>(lo + off) = make_uint4(*reinterpret_cast<uint32_t *>(&l[0]), *reinterpret_cast<uint32_t *>(&l[1]),
                                                          *reinterpret_cast<uint32_t *>(&l[2]), *reinterpret_cast<uint32_t *>(&l[3]));
    }
}

// Activation tile T[n][f] (edges n contiguous in 16-byte runs): element (n, f) at
// (n % 8) * 2 + (n / 8) * 2048 + (f % 8) * 16 + (f / 8) * 128.  Thread f stores edges
// n0 .. n0+31 of its feature.  TE = 64 edges: 16 KB per fp16 copy.
template <bool SPLIT, int CH>
static __device__ __forceinline__ void store_tile_col(unsigned char *Th, unsigned char *Tl, int f, int n0, const float (&v)[CH])
{
    const uint32_t base = (uint32_t)((f & 7) * 16 + (f >> 3) * 128);
#pragma unroll
    for (int g = 0; g < CH / 8; ++g) store8<SPLIT>(Th, Tl, base + (uint32_t)(((n0 >> 3) + g) * 2048), v + 8 * g);
}

// Named barrier of one warpgroup (ids 1..4; id 0 is __syncthreads).
static __device__ __forceinline__ void wg_sync(int g)
{
    asm volatile("bar.sync %0, %1;" ::"r"(g + 1), "r"(WGT) : "memory");
}

// Warpgroup barrier that also returns whether every thread passed a true predicate.
static __device__ __forceinline__ int wg_sync_and(int g, int pred)
{
    int out;
    asm volatile(
        "{\n\t.reg .pred q, p;\n\tsetp.ne.s32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, %3, q;\n\tselp.s32 %0, 1, 0, p;\n\t}\n"
        : "=r"(out)
        : "r"(pred), "r"(g + 1), "r"(WGT)
        : "memory");
    return out;
}

// Default bound (GPU clock cycles, about 2 s) of every wait of a kernel for its own MMAs and
// copies; the context can shorten the MMA waits to exercise the time-out path.
constexpr long long WAIT_BOUND = 1ll << 32;

// Wait for a barrier phase for at most lim cycles; false on time-out.  The phase is tested
// before the bound, so that a short bound gives up at once on work still in flight.
static __device__ __forceinline__ int bounded_phase_wait(uint32_t mbar, uint32_t parity, long long lim)
{
    const long long t0 = clock64();
    for (;;) {
        if (mbar_test_wait(mbar, parity)) return 1;
        if (clock64() - t0 > lim) return 0;
        if (mbar_try_wait(mbar, parity)) return 1;
    }
}

// Bounded wait for the MMAs committed to a warpgroup's mbarrier; every thread of the group
// calls it at the same point.  On a time-out (never expected with the default bound: nothing
// here waits on another agent) the error bit is set and the whole group returns false.
static __device__ __forceinline__ bool wait_mma(int g, uint32_t mbar, uint32_t &phase, int *d_err,
                                                long long lim = WAIT_BOUND)
{
    int ok = bounded_phase_wait(mbar, phase, lim);
    phase ^= 1u;
    ok = wg_sync_and(g, ok);
    if (!ok && (threadIdx.x % WGT) == 0) atomicOr(d_err, ERRBIT_TIMEOUT);
    tc_fence_after();
    return ok != 0;
}

// The same wait when the whole CTA waits on one mbarrier (every thread calls it).
static __device__ __forceinline__ bool wait_mma_cta(uint32_t mbar, uint32_t &phase, int *d_err,
                                                    long long lim = WAIT_BOUND)
{
    int ok = bounded_phase_wait(mbar, phase, lim);
    phase ^= 1u;
    ok = __syncthreads_and(ok);
    if (!ok && threadIdx.x == 0) atomicOr(d_err, ERRBIT_TIMEOUT);
    tc_fence_after();
    return ok != 0;
}


// Loads issued where they stand: the compiler may move a plain load down to its first use,
// which undoes a read-ahead; volatile asm keeps its place among the barrier operations
// around it.  ".nc" for data that no thread writes during the kernel.
static __device__ __forceinline__ float ld_keep(const float *p)
{
    float v;
    asm volatile("ld.global.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
    return v;
}
static __device__ __forceinline__ float ldnc_keep(const float *p)
{
    float v;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}
static __device__ __forceinline__ int ldnc_keep(const int *p)
{
    int v;
    asm volatile("ld.global.nc.s32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
static __device__ __forceinline__ float4 ldnc_keep(const float4 *p)
{
    float4 v;
    asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
    return v;
}

// Predicated global store (no branch); all stores of a value stream go through it so that
// they keep their program order.
static __device__ __forceinline__ void store_if(float *p, float v, bool c)
{
    asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q st.global.f32 [%0], %1;\n\t}" ::"l"(p), "f"(v),
                 "r"((unsigned)c));
}

constexpr float LOG2EF = 1.4426950408889634f;

// 2^x by the hardware exp2 unit (ex2.approx.ftz.f32, relative error ~2^-22).
static __device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Activations with the hardware exp2/log2 units (__expf, __logf): ssp(x) = max(x, 0) +
// ln(1 + e^-|x|) - ln 2 and sigma(x) = 1 / (1 + e^-x).  Absolute error ~3e-7, below the
// 2^-22 resolution of the split fp16 operands they feed.
static __device__ __forceinline__ float ssp_fast(float x) { return fmaxf(x, 0.0f) + __logf(1.0f + __expf(-fabsf(x))) - LN2F; }
static __device__ __forceinline__ float sigmoid_fast(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

// Activations for the fp16-operand mode, whose outputs are rounded to fp16 (2^-11 relative)
// before the next MMA: one hardware transcendental each instead of two.
//   ssp(x) = max(x, 0) + log1p(e^-|x|) - ln 2, with log1p on [0, 1] replaced by its degree-5
//   Chebyshev interpolant at the first-kind nodes, in monomial form (max |error| 1.1e-5);
//   sigma(x) = (1 + tanh(x / 2)) / 2 with the hardware tanh (tanh.approx.f32).
constexpr float LOG1P_C0 = 1.144709767686436e-05f;
constexpr float LOG1P_C1 = 0.9991664290428162f;
constexpr float LOG1P_C2 = -0.4896990954875946f;
constexpr float LOG1P_C3 = 0.2838231921195984f;
constexpr float LOG1P_C4 = -0.1299571990966797f;
constexpr float LOG1P_C5 = 0.029808765277266502f;

static __device__ __forceinline__ float ssp16(float x)
{
    const float u = ex2_approx(-fabsf(x) * LOG2EF);
    float p = fmaf(LOG1P_C5, u, LOG1P_C4);
    p = fmaf(p, u, LOG1P_C3);
    p = fmaf(p, u, LOG1P_C2);
    p = fmaf(p, u, LOG1P_C1);
    p = fmaf(p, u, LOG1P_C0 - LN2F);
    return fmaxf(x, 0.0f) + p;
}

static __device__ __forceinline__ float tanh_approx(float x)
{
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

static __device__ __forceinline__ float sigmoid16(float x) { return fmaf(0.5f, tanh_approx(0.5f * x), 0.5f); }

// The activation pair of a precision mode: SPLIT (fp32-accurate) or fp16 operands.
template <bool SPLIT>
static __device__ __forceinline__ float ssp_mode(float x)
{
    return SPLIT ? ssp_fast(x) : ssp16(x);
}

template <bool SPLIT>
static __device__ __forceinline__ float sigmoid_mode(float x)
{
    return SPLIT ? sigmoid_fast(x) : sigmoid16(x);
}

// s * sigma(v s + b) for a TMEM accumulator v of an output channel with scale s and bias b
// (hs = s / 2, hb = b / 2): the scale of the channel carried into the operand of a transposed
// product.  With s = 1 the value equals sigma_mode(v + b) exactly.
template <bool SPLIT>
static __device__ __forceinline__ float sigmoid_scaled(float v, float s, float b, float hs, float hb)
{
    if (SPLIT) return s * sigmoid_fast(fmaf(v, s, b));
    return fmaf(hs, tanh_approx(fmaf(v, hs, hb)), hs);
}

}  // namespace tc
}  // namespace sn
