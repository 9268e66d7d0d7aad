// Node (per-atom) networks on the tensor cores: the update network with its residual, the
// readout, and the backward of the update network (FlashSchNet §3.2 "update network with
// residual connection", "Energy readout"; §4.4 applies W16A16 to the update and readout
// networks as well as the filter network).  Per tile of TA = 128 atoms, with feature f =
// TMEM lane f and atoms on the MMA N dimension; the CTA's NG = 4 warpgroups share the tile,
// warpgroup g gathering and finishing atom columns [32g, 32g + 32):
//   update   D_P = U1 h^T, p = D_P + c1;  D_Y = U2 ssp(p)^T, x^{t+1} = x^t + D_Y + c2
//   readout  D_O = R1 x^T (R1 padded to 128 rows), o = D_O + e1; eps = R2 . ssp(o) + e2;
//            obar = R2 (.) sigma(o); D_X = R1^T obar, xbar^T = D_X
//   backward D_Q = U2^T xbar, pbar = D_Q (.) sigma(p);  D_H = U1^T pbar, hbar = D_H
// Operands and precision modes as in sn_ef_tc.cu (fp16, or fp16 hi/lo split).
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "sn_internal.cuh"
#include "sn_tc_common.cuh"

namespace sn {

namespace {

using namespace tc;

constexpr int TA = 128;          // atoms per tile (MMA N)
constexpr int NG = 4;            // warpgroups per CTA, one 32-atom column chunk each
constexpr int NT = WGT * NG;     // threads per CTA

template <bool SPLIT>
struct NodeSmem {
    static constexpr int NS = SPLIT ? 2 : 1;
    static constexpr uint32_t WB = FF * FF * 2;     // one fp16 copy of a 128 x 128 weight
    static constexpr uint32_t TB = TA * FF * 2;     // activation tile
    static constexpr uint32_t W0 = 0;               // first weight (hi, lo)
    static constexpr uint32_t W1 = W0 + NS * WB;    // second weight (hi, lo)
    static constexpr uint32_t T = W1 + NS * WB;
    static constexpr uint32_t MBAR = T + NS * TB;   // uint64
    static constexpr uint32_t WMBAR = MBAR + 8;     // weight copies
    static constexpr uint32_t HOLD = WMBAR + 8;     // TMEM address
    static constexpr uint32_t PR = HOLD + 16;       // float[64][TA] readout products (readout only)
    static constexpr uint32_t BYTES_UPDATE = PR;
    static constexpr uint32_t BYTES_READOUT = PR + 64 * TA * 4;
    // update and backward with fp16 operands: the tile's two input row blocks, fp32 [TA][F]
    // each, staged by bulk copies that complete on LB0 and LB1
    static constexpr uint32_t LB0 = HOLD + 16;
    static constexpr uint32_t LB1 = LB0 + 8;
    static constexpr uint32_t IN0 = (LB1 + 8 + 127) / 128 * 128;
    static constexpr uint32_t IN1 = IN0 + TA * FF * 4;
    static constexpr uint32_t BYTES_STAGED = IN1 + TA * FF * 4;
};

// The input rows of a tile (na <= TA atoms from a0) into the staging blocks: thread 0 announces
// the bytes on both barriers, then thread a copies row a of each input (512 bytes, 16-byte
// aligned) -- row0(a) into IN0 (completing on LB0) and row1(a) into IN1 (on LB1).
template <typename Row0, typename Row1>
__device__ __forceinline__ void stage_rows(unsigned char *sm, int na, Row0 row0, Row1 row1)
{
    using S = NodeSmem<false>;
    const uint32_t lb0 = smem_u32(sm + S::LB0), lb1 = smem_u32(sm + S::LB1);
    if (threadIdx.x == 0) {
        mbar_expect_tx(lb0, (uint32_t)na * FF * 4);
        mbar_expect_tx(lb1, (uint32_t)na * FF * 4);
    }
    __syncthreads();
    if ((int)threadIdx.x < na) {
        bulk_g2s(smem_u32(sm + S::IN0) + threadIdx.x * FF * 4, row0((int)threadIdx.x), FF * 4, lb0);
        bulk_g2s(smem_u32(sm + S::IN1) + threadIdx.x * FF * 4, row1((int)threadIdx.x), FF * 4, lb1);
    }
}

// Every thread waits, bounded, for one staging barrier's phase; false (and the time-out bit) if
// the copies did not land.
__device__ __forceinline__ bool staged(unsigned char *sm, uint32_t off, uint32_t parity, int *d_err)
{
    int ok = bounded_phase_wait(smem_u32(sm + off), parity, 1ll << 33);
    ok = __syncthreads_and(ok);
    if (!ok && threadIdx.x == 0) atomicOr(d_err, ERRBIT_TIMEOUT);
    return ok != 0;
}

// D[o][a] = sum_i W[o][i] T[a][i]  (TRANS = false)  or  D[i][a] = sum_o W[o][i] T[a][o]  (TRANS)
template <bool SPLIT, bool TRANS>
__device__ __forceinline__ void issue_gemm(unsigned char *W, unsigned char *T, uint32_t d)
{
    using S = NodeSmem<SPLIT>;
    constexpr uint32_t ID = idesc_f16(128, TA, TRANS ? 1 : 0, 1);
    const uint32_t wh = smem_u32(W), wl = wh + S::WB;
    const uint32_t th = smem_u32(T), tl = th + S::TB;
    const uint32_t a_lbo = TRANS ? 2048 : 128, a_sbo = TRANS ? 128 : 2048, a_step = TRANS ? 4096 : 256;
#pragma unroll
    for (int j = 0; j < FF / 16; ++j) {
        const uint32_t oa = (uint32_t)j * a_step, ob = (uint32_t)j * 256;
        mma_f16(d, sdesc(wh + oa, a_lbo, a_sbo), sdesc(th + ob, 128, 2048), ID, j > 0);
        if (SPLIT) {
            mma_f16(d, sdesc(wh + oa, a_lbo, a_sbo), sdesc(tl + ob, 128, 2048), ID, 1);
            mma_f16(d, sdesc(wl + oa, a_lbo, a_sbo), sdesc(th + ob, 128, 2048), ID, 1);
        }
    }
}

// The weight copies issued by node_setup land while the first tile is being gathered; the
// first GEMM of a CTA waits for them (weights_ready tracks this).
template <bool SPLIT, bool TRANS>
__device__ __forceinline__ bool gemm_step(unsigned char *W, unsigned char *T, uint32_t d, uint32_t mbar,
                                          uint32_t &phase, int *d_err, bool &weights_ready, uint32_t wmbar,
                                          long long lim)
{
    if (!weights_ready) {
        if (!wait_copies(wmbar, d_err)) return false;
        weights_ready = true;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
        tc_fence_after();
        issue_gemm<SPLIT, TRANS>(W, T, d);
        mma_commit(mbar);
    }
    return wait_mma_cta(mbar, phase, d_err, lim);
}

// After a wait gave up: one more commit, whose completion follows that of every MMA issued,
// waited for with the default bound before TMEM is freed.
__device__ __forceinline__ void drain_cta(uint32_t mbar, uint32_t &phase, int *d_err)
{
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
        tc_fence_after();
        mma_commit(mbar);
    }
    wait_mma_cta(mbar, phase, d_err, WAIT_BOUND);
}

// get(q) for atoms 32 g + q (q < nv) of the tile at column f, into the activation tile (zero
// for q >= nv, past the last atom)
template <bool SPLIT, typename Get>
__device__ __forceinline__ void tile_from(unsigned char *T, int f, int g, int nv, Get get)
{
    using S = NodeSmem<SPLIT>;
    float v[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) v[q] = q < nv ? get(q) : 0.0f;
    store_tile_col<SPLIT, 32>(T, T + S::TB, f, 32 * g, v);
}

// atoms of the tile starting at a0 that column chunk c (32 atoms) holds: min(32, N - a0 - 32 c)
__device__ __forceinline__ int chunk_atoms(int64_t a0, int c, int64_t N)
{
    const int64_t r = N - a0 - 32 * c;
    return r <= 0 ? 0 : (r >= 32 ? 32 : (int)r);
}

__device__ __forceinline__ const float *x_row(const NodeTcArgs &A, int t, int64_t a)
{
    if (t == 0) return A.emb + (int64_t)__ldg(A.types + a) * FF;
    return A.X + ((int64_t)(t - 1) * A.N + a) * FF;
}

template <bool SPLIT, bool STAGED = false>
__device__ __forceinline__ uint32_t node_setup(const NodeTcArgs &A, unsigned char *sm, const void *w0h,
                                               const void *w0l, const void *w1h, const void *w1l, int &skip)
{
    using S = NodeSmem<SPLIT>;
    const uint32_t wmbar = smem_u32(sm + S::WMBAR);
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(sm + S::MBAR), 1);
        mbar_init(wmbar, 1);
        if (STAGED) {
            mbar_init(smem_u32(sm + NodeSmem<false>::LB0), 1);
            mbar_init(smem_u32(sm + NodeSmem<false>::LB1), 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        mbar_expect_tx(wmbar, S::NS * S::WB * (w1h ? 2 : 1));   // constant weights: before the wait
        bulk_g2s(smem_u32(sm + S::W0), w0h, S::WB, wmbar);
        if (SPLIT) bulk_g2s(smem_u32(sm + S::W0 + S::WB), w0l, S::WB, wmbar);
        if (w1h) {
            bulk_g2s(smem_u32(sm + S::W1), w1h, S::WB, wmbar);
            if (SPLIT) bulk_g2s(smem_u32(sm + S::W1 + S::WB), w1l, S::WB, wmbar);
        }
    }
    if ((threadIdx.x >> 5) == 0) tmem_alloc(smem_u32(sm + S::HOLD), 256);
    pdl_trigger();
    pdl_wait();   // from here on: data written by the preceding kernels
    if (threadIdx.x == 0)
        skip = (*((volatile const int *)A.d_err) & (ERRBIT_NONFINITE | ERRBIT_CAPACITY | ERRBIT_TIMEOUT)) != 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *reinterpret_cast<volatile uint32_t *>(sm + S::HOLD);
}

__device__ __forceinline__ void node_teardown(uint32_t tmem, bool weights_ready, uint32_t wmbar, int *d_err)
{
    if (!weights_ready) wait_copies(wmbar, d_err);   // never leave with copies in flight
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if ((threadIdx.x >> 5) == 0) tmem_dealloc(tmem, 256);
}

// p = U1 h + c1 (saved); x^{t+1} = x^t + U2 ssp(p) + c2
template <bool SPLIT>
__global__ void __launch_bounds__(NT, 1) k_node_update_tc(NodeTcArgs A)
{
    using S = NodeSmem<SPLIT>;
    extern __shared__ __align__(128) unsigned char sm[];
    __shared__ int skip;
    const uint32_t tmem = node_setup<SPLIT, !SPLIT>(A, sm, A.U1h, A.U1l, A.U2h, A.U2l, skip);
    const int f = threadIdx.x % WGT, g = threadIdx.x / WGT, c = g;
    const uint32_t lane = (uint32_t)((f >> 5) * 32) << 16;
    const uint32_t mbar = smem_u32(sm + S::MBAR);
    uint32_t phase = 0;
    bool ready = false;
    const uint32_t wmbar = smem_u32(sm + S::WMBAR);
    const int64_t n_tiles = (A.N + TA - 1) / TA;
    if (!skip) {
        const float c1f = A.c1[f], c2f = A.c2[f], su1f = A.su1[f], su2f = A.su2[f];
        unsigned char *T = sm + S::T;
        bool ok = true;
        bool pending = false;   // the second input of a tile copied but not yet waited for
        uint32_t sp = 0;        // parity of this tile's staging barriers
        for (int64_t tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
            sp = (uint32_t)(((tile - blockIdx.x) / gridDim.x) & 1);
            const int64_t a0 = tile * TA, ab = a0 + 32 * c;   // this thread's atoms: ab + q, q < nv
            const int nv = chunk_atoms(a0, c, A.N);
            const float *Hp = A.H + ab * FF + f;
            float *Pp = A.P + ((int64_t)A.t * A.N + ab) * FF + f;
            float *Xp = A.X + ((int64_t)A.t * A.N + ab) * FF + f;
            float xr[32];   // the residual's x^t
            if constexpr (SPLIT) {
                tile_from<SPLIT>(T, f, g, nv, [&](int q) { return Hp[q * FF]; });
#pragma unroll
                for (int q = 0; q < 32; ++q) xr[q] = q < nv ? ldnc_keep(x_row(A, A.t, ab + q) + f) : 0.0f;
            } else {   // h and x^t rows of the tile by bulk copies (x^t waited for at its use)
                const int na = (int)(A.N - a0 < TA ? A.N - a0 : TA);
                stage_rows(sm, na, [&](int a) { return A.H + (a0 + a) * FF; },
                           [&](int a) { return x_row(A, A.t, a0 + a); });
                pending = true;
                if (!(ok = staged(sm, S::LB0, sp, A.d_err))) break;
                const float *sH = reinterpret_cast<const float *>(sm + S::IN0) + 32 * c * FF + f;
                tile_from<SPLIT>(T, f, g, nv, [&](int q) { return sH[q * FF]; });
            }
            if (!(ok = gemm_step<SPLIT, false>(sm + S::W0, T, tmem, mbar, phase, A.d_err, ready, wmbar, A.wait_limit))) break;
            {
                float v[32];
                tmem_ld32(tmem + lane + 32 * c, v);
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    v[q] = fmaf(v[q], su1f, c1f);
                    if (q < nv) Pp[q * FF] = v[q];
                    v[q] = ssp_fast(v[q]);
                }
                store_tile_col<SPLIT, 32>(T, T + S::TB, f, 32 * c, v);
            }
            if (!(ok = gemm_step<SPLIT, false>(sm + S::W1, T, tmem + 128, mbar, phase, A.d_err, ready, wmbar, A.wait_limit))) break;
            if constexpr (!SPLIT) {
                if (!(ok = staged(sm, S::LB1, sp, A.d_err))) break;
                pending = false;
                const float *sX = reinterpret_cast<const float *>(sm + S::IN1) + 32 * c * FF + f;
#pragma unroll
                for (int q = 0; q < 32; ++q) xr[q] = q < nv ? sX[q * FF] : 0.0f;
            }
            {
                float v[32];
                tmem_ld32(tmem + lane + 128 + 32 * c, v);
#pragma unroll
                for (int q = 0; q < 32; ++q)
                    if (q < nv) Xp[q * FF] = fmaf(v[q], su2f, xr[q]) + c2f;
            }
            tc_fence_before();
            __syncthreads();
        }
        if (!ok) {
            drain_cta(mbar, phase, A.d_err);
            if (!SPLIT && pending) staged(sm, NodeSmem<false>::LB1, sp, A.d_err);   // no copy left in flight
        }
    }
    node_teardown(tmem, ready, wmbar, A.d_err);
}

// o = R1 x^T + e1; eps = R2 . ssp(o) + e2; xbar^T = R1^T (R2 (.) sigma(o)); forces = 0
template <bool SPLIT>
__global__ void __launch_bounds__(NT, 1) k_node_readout_tc(NodeTcArgs A)
{
    using S = NodeSmem<SPLIT>;
    extern __shared__ __align__(128) unsigned char sm[];
    __shared__ int skip;
    const uint32_t tmem = node_setup<SPLIT>(A, sm, A.R1h, A.R1l, nullptr, nullptr, skip);
    const int f = threadIdx.x % WGT, g = threadIdx.x / WGT, c = g;
    const uint32_t lane = (uint32_t)((f >> 5) * 32) << 16;
    const uint32_t mbar = smem_u32(sm + S::MBAR);
    float *sPr = reinterpret_cast<float *>(sm + S::PR);
    uint32_t phase = 0;
    bool ready = false;
    const uint32_t wmbar = smem_u32(sm + S::WMBAR);
    const int64_t n_tiles = (A.N + TA - 1) / TA;
    const int H = FF / 2;
    if (!skip) {
        const float e1k = f < H ? A.e1[f] : 0.0f, r2k = f < H ? A.R2[f] : 0.0f, e2 = A.e2[0];
        const float sr1k = A.sr1[f], r2s = r2k * sr1k;   // R1's channel scale (1 past H)
        unsigned char *T = sm + S::T;
        bool ok = true;
        for (int64_t tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
            const int64_t a0 = tile * TA, ab = a0 + 32 * c;
            const int nv = chunk_atoms(a0, c, A.N);
            const float *Xp = A.X + ((int64_t)A.t * A.N + ab) * FF + f;
            tile_from<SPLIT>(T, f, g, nv, [&](int q) { return Xp[q * FF]; });
            if (!(ok = gemm_step<SPLIT, false>(sm + S::W0, T, tmem, mbar, phase, A.d_err, ready, wmbar, A.wait_limit))) break;
            {
                float v[32];
                tmem_ld32(tmem + lane + 32 * c, v);
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const float o = fmaf(v[q], sr1k, e1k);
                    if (f < H) sPr[f * TA + 32 * c + q] = r2k * ssp_fast(o);
                    v[q] = f < H ? r2s * sigmoid_fast(o) : 0.0f;   // R1's transposed operand
                }
                store_tile_col<SPLIT, 32>(T, T + S::TB, f, 32 * c, v);
            }
            if (!(ok = gemm_step<SPLIT, true>(sm + S::W0, T, tmem + 128, mbar, phase, A.d_err, ready, wmbar, A.wait_limit))) break;
            if (threadIdx.x < TA) {   // per-atom energy (fixed summation order) and zero forces
                const int64_t a = a0 + threadIdx.x;
                if (a < A.N) {
                    float e = e2;
                    for (int k = 0; k < H; ++k) e += sPr[k * TA + threadIdx.x];
                    A.eps[a] = e;
                    A.forces[a * 3] = 0.0f;
                    A.forces[a * 3 + 1] = 0.0f;
                    A.forces[a * 3 + 2] = 0.0f;
                }
            }
            {
                float v[32];
                tmem_ld32(tmem + lane + 128 + 32 * c, v);
                float *Bp = A.Xbar + ab * FF + f;
#pragma unroll
                for (int q = 0; q < 32; ++q)
                    if (q < nv) Bp[q * FF] = v[q];
            }
            tc_fence_before();
            __syncthreads();
        }
        if (!ok) drain_cta(mbar, phase, A.d_err);
    }
    node_teardown(tmem, ready, wmbar, A.d_err);
}

// hbar = U1^T (sigma(p) (.) U2^T xbar)   (block t's update network, p = P[t])
template <bool SPLIT>
__global__ void __launch_bounds__(NT, 1) k_node_bwd_tc(NodeTcArgs A)
{
    using S = NodeSmem<SPLIT>;
    extern __shared__ __align__(128) unsigned char sm[];
    __shared__ int skip;
    const uint32_t tmem = node_setup<SPLIT, !SPLIT>(A, sm, A.U2h, A.U2l, A.U1h, A.U1l, skip);
    const int f = threadIdx.x % WGT, g = threadIdx.x / WGT, c = g;
    const uint32_t lane = (uint32_t)((f >> 5) * 32) << 16;
    const uint32_t mbar = smem_u32(sm + S::MBAR);
    uint32_t phase = 0;
    bool ready = false;
    const uint32_t wmbar = smem_u32(sm + S::WMBAR);
    const int64_t n_tiles = (A.N + TA - 1) / TA;
    if (!skip) {
        unsigned char *T = sm + S::T;
        // the operands of U2^T and U1^T carry the channel scales of U2 and U1
        const float su1f = A.su1[f], su2f = A.su2[f];
        bool ok = true;
        bool pending = false;   // the second input of a tile copied but not yet waited for
        uint32_t sp = 0;        // parity of this tile's staging barriers
        for (int64_t tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
            sp = (uint32_t)(((tile - blockIdx.x) / gridDim.x) & 1);
            const int64_t a0 = tile * TA, ab = a0 + 32 * c;
            const int nv = chunk_atoms(a0, c, A.N);
            const float *Bp = A.Xbar + ab * FF + f;
            const float *Pp = A.P + ((int64_t)A.t * A.N + ab) * FF + f;
            float pr[32];   // p of this thread's atoms
            if constexpr (SPLIT) {
                tile_from<SPLIT>(T, f, g, nv, [&](int q) { return Bp[q * FF] * su2f; });
#pragma unroll
                for (int q = 0; q < 32; ++q) pr[q] = q < nv ? ldnc_keep(Pp + q * FF) : 0.0f;
            } else {   // xbar and p rows of the tile by bulk copies (p waited for at its use)
                const int na = (int)(A.N - a0 < TA ? A.N - a0 : TA);
                stage_rows(sm, na, [&](int a) { return A.Xbar + (a0 + a) * FF; },
                           [&](int a) { return A.P + ((int64_t)A.t * A.N + a0 + a) * FF; });
                pending = true;
                if (!(ok = staged(sm, S::LB0, sp, A.d_err))) break;
                const float *sB = reinterpret_cast<const float *>(sm + S::IN0) + 32 * c * FF + f;
                tile_from<SPLIT>(T, f, g, nv, [&](int q) { return sB[q * FF] * su2f; });
            }
            if (!(ok = gemm_step<SPLIT, true>(sm + S::W0, T, tmem, mbar, phase, A.d_err, ready, wmbar, A.wait_limit))) break;
            if constexpr (!SPLIT) {
                if (!(ok = staged(sm, S::LB1, sp, A.d_err))) break;
                pending = false;
                const float *sP = reinterpret_cast<const float *>(sm + S::IN1) + 32 * c * FF + f;
#pragma unroll
                for (int q = 0; q < 32; ++q) pr[q] = q < nv ? sP[q * FF] : 0.0f;
            }
            {
                float v[32];
                tmem_ld32(tmem + lane + 32 * c, v);
#pragma unroll
                for (int q = 0; q < 32; ++q) v[q] *= su1f * sigmoid_fast(pr[q]);
                store_tile_col<SPLIT, 32>(T, T + S::TB, f, 32 * c, v);
            }
            if (!(ok = gemm_step<SPLIT, true>(sm + S::W1, T, tmem + 128, mbar, phase, A.d_err, ready, wmbar, A.wait_limit))) break;
            {
                float v[32];
                tmem_ld32(tmem + lane + 128 + 32 * c, v);
                float *Hp = A.Hbar + ab * FF + f;
#pragma unroll
                for (int q = 0; q < 32; ++q)
                    if (q < nv) Hp[q * FF] = v[q];
            }
            tc_fence_before();
            __syncthreads();
        }
        if (!ok) {
            drain_cta(mbar, phase, A.d_err);
            if (!SPLIT && pending) staged(sm, NodeSmem<false>::LB1, sp, A.d_err);   // no copy left in flight
        }
    }
    node_teardown(tmem, ready, wmbar, A.d_err);
}

template <typename Kern>
cudaError_t launch_k(Kern k, uint32_t bytes, int grid, const NodeTcArgs &a, cudaStream_t s)
{
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    return launch_pdl(k, dim3(grid), dim3(NT), bytes, s, a);
}

}  // namespace

// which: 0 update (block a.t), 1 readout (x^T = X[a.t]), 2 backward of block a.t's update
cudaError_t launch_node_tc(const NodeTcArgs &a, bool split, int which, int n_sm, cudaStream_t s)
{
    const int64_t tiles = (a.N + TA - 1) / TA;
    if (tiles == 0) return cudaSuccess;
    const int grid = (int)(tiles < (int64_t)n_sm ? tiles : (int64_t)n_sm);
    if (split) {
        using S = NodeSmem<true>;
        if (which == 0) return launch_k(k_node_update_tc<true>, S::BYTES_UPDATE, grid, a, s);
        if (which == 1) return launch_k(k_node_readout_tc<true>, S::BYTES_READOUT, grid, a, s);
        return launch_k(k_node_bwd_tc<true>, S::BYTES_UPDATE, grid, a, s);
    }
    using S = NodeSmem<false>;
    static_assert(S::BYTES_STAGED <= 227 * 1024, "shared memory plan exceeds 227 KB");
    if (which == 0) return launch_k(k_node_update_tc<false>, S::BYTES_STAGED, grid, a, s);
    if (which == 1) return launch_k(k_node_readout_tc<false>, S::BYTES_READOUT, grid, a, s);
    return launch_k(k_node_bwd_tc<false>, S::BYTES_STAGED, grid, a, s);
}

}  // namespace sn
