// Edge kernels on the 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// The filter network of every edge tile is a dense contraction (FlashSchNet §3.3 "Mixed
// precision and Tensor Cores", §4.4): per tile of TE = 64 edges
//   forward   D_A[f][n] = W1[f][:] . bt[n][:]          (M = F = 128, N = 64, K = K_P)
//             D_W[f][n] = W2[f][:] . s[n][:]           (M = 128, N = 64, K = F)
//   backward  D_S[i][n] = W2[:][i] . wbar[n][:]        (W2^T, M = 128, N = 64, K = F)
//             D_G[n][k] = abar[n][:] . W1[:][k]        (edges on M: M = 64, N = K_P, K = F)
// with fp16 operands in shared memory and fp32 accumulation in TMEM (the pages' W16A16 for
// MLPs with fp32 accumulation, §4.1).  SPLIT adds an fp32-accurate mode: every operand x is
// split into hi = fp16(x) and lo = fp16(x - hi), and each product is accumulated as
// hi*hi + hi*lo + lo*hi (three MMAs into the same accumulator, ~22 significant bits).
//
// Two kernel shapes.  k_edge_fwd_tc / k_edge_bwd_tc: NW independent warpgroups per CTA (4 for
// fp16, 2 for the split), each owning whole destination rows and walking their edges tile by
// tile through its MMA steps; thread t of a warpgroup is TMEM lane t, i.e. feature f = t for
// the feature-major accumulators.  k_edge_fwd_ws (fp16 forward): one warp-specialised
// pipeline per CTA (producer, MMA, activation and epilogue warps over a ring of tile stages).
// The elementwise work between the MMAs (Gaussians, ssp, gathers, segment sums) runs on the
// CUDA cores.
//
// Shared-memory operand layout: no swizzle, 8 x 16-byte "core matrices".  An element (r, c)
// of a matrix whose contiguous 8-element runs go along c sits at
//   (r % 8) * 16 + (r / 8) * SBO + (c % 8) * 2 + (c / 8) * LBO   bytes.
// The same bytes read as K-major for one GEMM read as MN-major for its transpose with LBO and
// SBO exchanged, so each weight matrix is stored once and serves forward and backward.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <type_traits>

#include "sn_internal.cuh"
#include "sn_tc_common.cuh"

namespace sn {

namespace {

using namespace tc;

constexpr int TE = 64;           // edges per tile
// TMEM: 128 columns per warpgroup (128 * NW per CTA)
// per-warpgroup TMEM columns: a (and later btbar) in [0, 64), w (and later sbar) in [64, 128)
constexpr uint32_t COL_A = 0, COL_W = 64;

// Shared-memory plan (bytes): weights shared by the CTA, then one region per warpgroup.
template <int KP, bool SPLIT, int NW>
struct TcSmem {
    static constexpr int NS = SPLIT ? 2 : 1;
    static constexpr uint32_t W1B = FF * KP * 2;        // one fp16 copy of W1
    static constexpr uint32_t W2B = FF * FF * 2;
    static constexpr uint32_t BB = TE * KP * 2;         // basis tile
    static constexpr uint32_t TB = TE * FF * 2;         // activation tile
    static constexpr uint32_t SW1 = (KP / 8) * 128;     // 8-row group stride of W1 and of the basis tile
    static constexpr uint32_t W1 = 0;
    static constexpr uint32_t W2 = W1 + NS * W1B;
    static constexpr uint32_t GROUPS = W2 + NS * W2B;
    // offsets inside a warpgroup region
    static constexpr uint32_t B = 0;
    static constexpr uint32_t T = B + NS * BB;
    static constexpr uint32_t XO = T + NS * TB;         // int[TE]: offset of the source's x row
    static constexpr uint32_t HO = XO + 4 * TE;         // int[TE]: offset of the source's hbar row
    static constexpr uint32_t DIST = HO + 4 * TE;       // double[TE]
    static constexpr uint32_t DST = DIST + 8 * TE;      // int[TE]
    static constexpr uint32_t UVEC = DST + 4 * TE;      // float[TE][3]
    static constexpr uint32_t FV = UVEC + 12 * TE;      // float[TE][3]
    static constexpr uint32_t MASK = FV + 12 * TE;      // uint32[4]: row starts, empty-row flags
    static constexpr uint32_t CD = MASK + 16;           // float2[TE]: C(d), dC/dd (fp16 backward)
    static constexpr uint32_t PDX = CD + 8 * TE;        // float[4]: force scan, warp 0 -> warp 1
    static constexpr uint32_t MBAR = PDX + 16;          // uint64
    static constexpr uint32_t REGION = (MBAR + 8 + 127) / 128 * 128;
    static constexpr uint32_t HOLD = GROUPS + NW * REGION;
    static constexpr uint32_t WMBAR = HOLD + 8;           // weight copies
    static constexpr uint32_t MUH = WMBAR + 8;            // float[64]: mu_k as a float pair (hi, lo)
    static constexpr uint32_t MUL = MUH + 256;
    static constexpr uint32_t USED = MUL + 256;
    // at least 116 KB so that no two CTAs share an SM
    static constexpr uint32_t BYTES = USED > 116 * 1024 ? USED : 116 * 1024;
};

}  // namespace

namespace {

// What a tile's prologue needs of its edge, loaded one tile ahead in two steps (indices, then
// positions and types) so that the loads overlap the previous tile's work.
struct EdgeIdx {
    int i, j;
};
struct EdgePos {
    float4 ri, rj;
    int tj, rs;   // type of the source (block 0), first edge of the destination's row
    int rsm;      // first edge of the row before the destination's (-1 for row 0)
};

// (loads kept where they stand, so that the read-ahead by a tile really is ahead: see ld_keep)
__device__ __forceinline__ EdgeIdx load_idx(const EdgeTcArgs &A, int e, int e1)
{
    EdgeIdx x{0, 0};
    if (e < e1) {
        x.i = ldnc_keep(A.dst + e);
        x.j = ldnc_keep(A.col + e);
    }
    return x;
}

__device__ __forceinline__ EdgePos load_pos(const EdgeTcArgs &A, EdgeIdx x)
{
    EdgePos p;
    p.ri = ldnc_keep(A.pos4 + x.i);
    p.rj = ldnc_keep(A.pos4 + x.j);
    p.tj = A.t == 0 ? ldnc_keep(A.types + x.j) : 0;
    p.rs = ldnc_keep(A.row_ptr + x.i);
    p.rsm = x.i > 0 ? ldnc_keep(A.row_ptr + x.i - 1) : -1;
    return p;
}

// Feature rows of the current block's input x^t for thread f: x^0 is the embedding of the
// atom's type, x^t (t >= 1) lives in X[t-1].  Source rows are gathered as base + offset with
// the offsets of a tile kept in shared memory.
__device__ __forceinline__ const float *x_base(const EdgeTcArgs &A, int f)
{
    return (A.t == 0 ? A.emb : A.X + (int64_t)(A.t - 1) * A.N * FF) + f;
}

__device__ __forceinline__ const float *x_row(const EdgeTcArgs &A, const float *xbase, int r)
{
    return A.t == 0 ? xbase + (int64_t)__ldg(A.types + r) * FF : xbase + (int64_t)r * FF;
}

// Edge metadata and basis rows of one tile, by 64 PARTS threads: thread t handles edge
// n = t % 64 and part t / 64 of its K_P Gaussians; part 0 also stores the edge's metadata and
// part 1 its gather offsets.  u = r_i - r_j and d in double
// (minimum image on periodic axes); bt_k = exp(-gamma (d - mu_k)^2) C(d) as fp16 (hi/lo);
// also the offsets of the source's feature rows used by the gathers (padding edges: 0).
// SHARED (fp16, warp-specialised producer): part 0 alone forms d and C(d) and leaves them in
// the stage (S::DF, S::CC) for the other parts, after a barrier over the 64 PARTS threads.
// STORE_CD (fp16 backward): part 0 also leaves C(d) and dC/dd of every edge in the stage
// (S::CD, float2[TE]) for the dbar step.
template <class S, int KP, bool SPLIT, bool BWD, int PARTS = 2, bool SHARED = false, bool STORE_CD = false>
__device__ __forceinline__ void tile_prologue(const EdgeTcArgs &A, const unsigned char *sm, unsigned char *R, int t,
                                              int ts, int ne, EdgeIdx x, const EdgePos &p)
{
    const int n = t & (TE - 1), half = t / TE;   // half: the part
    static_assert(KP % (8 * PARTS) == 0, "Gaussians split in whole 8-column groups");
    // gather offsets: int[TE] of x rows (forward), or (x, hbar) int2[TE] over XO..HO (backward)
    int *sXo = reinterpret_cast<int *>(R + S::XO);
    static_assert(S::HO == S::XO + 4 * TE, "the backward's offset pairs span XO and HO");
    int *sDst = reinterpret_cast<int *>(R + S::DST);
    double *sDist = reinterpret_cast<double *>(R + S::DIST);
    float *sU = reinterpret_cast<float *>(R + S::UVEC);
    // (double for the fp32-accurate split mode, float for fp16 operands)
    using real = typename std::conditional<SPLIT, double, float>::type;
    real d = 0;
    // (SHARED: the source rows are copied by offsets the producer holds, so only part 0 works
    // here; the distance and direction arrays serve the backward's forces only)
    if (n < ne && (SHARED ? half == 0 : half <= 1)) {
        const int i = x.i, j = x.j;
        const float4 ri = p.ri, rj = p.rj;
        real dx = (real)ri.x - (real)rj.x, dy = (real)ri.y - (real)rj.y, dz = (real)ri.z - (real)rj.z;
        if (A.geo.periodic[0]) dx -= (real)A.geo.box[0] * rint(dx / (real)A.geo.box[0]);
        if (A.geo.periodic[1]) dy -= (real)A.geo.box[1] * rint(dy / (real)A.geo.box[1]);
        if (A.geo.periodic[2]) dz -= (real)A.geo.box[2] * rint(dz / (real)A.geo.box[2]);
        d = sqrt(dx * dx + dy * dy + dz * dz);
        if (half == 0) {
            sDst[n] = i;
            if constexpr (BWD) {
                sDist[n] = (double)d;
                const real inv = (real)1 / d;
                sU[3 * n] = (float)(dx * inv);
                sU[3 * n + 1] = (float)(dy * inv);
                sU[3 * n + 2] = (float)(dz * inv);
            }
        } else if (half == 1) {
            if (BWD) reinterpret_cast<int2 *>(sXo)[n] = make_int2((A.t == 0 ? p.tj : j) * FF, j * FF);
            else sXo[n] = (A.t == 0 ? p.tj : j) * FF;
        }
    } else if (half == 0) {
        sDst[n] = -1;
        if constexpr (BWD) sDist[n] = 0.0;
    } else if (half == 1 && !SHARED) {
        if (BWD) reinterpret_cast<int2 *>(sXo)[n] = make_int2(0, 0);
        else sXo[n] = 0;
    }
    if (half == 0) {   // warps 0 and 1: the edges that start their row, and whether a row
                       // without edges precedes any of them, one word each
        const bool start = n < ne && ts + n == p.rs;
        const unsigned b = __ballot_sync(0xffffffffu, start);
        const unsigned g = __ballot_sync(0xffffffffu, start && p.rsm == p.rs);
        if ((t & 31) == 0) {
            reinterpret_cast<uint32_t *>(R + S::MASK)[t >> 5] = b;
            reinterpret_cast<uint32_t *>(R + S::MASK)[2 + (t >> 5)] = g;
        }
    }
    // Padding edges (d = 0) and padding Gaussians (k >= K, mu_k = 0) get finite values that
    // never reach a result: W1 is zero in columns k >= K, and padding edges are skipped or
    // zeroed by every consumer.
    float C, d_hi, d_lo;
    if constexpr (SHARED) {
        static_assert(!SPLIT, "shared metadata is for fp16 operands");
        if (half == 0) {
            reinterpret_cast<float *>(R + S::DF)[n] = (float)d;
            reinterpret_cast<float *>(R + S::CC)[n] = 0.5f * (cospif((float)d / A.basis.r_cut) + 1.0f);
        }
        named_sync(5, 64 * PARTS);
        d_hi = reinterpret_cast<const float *>(R + S::DF)[n];
        C = reinterpret_cast<const float *>(R + S::CC)[n];
        d_lo = 0.0f;
    } else if constexpr (STORE_CD) {
        static_assert(!SPLIT, "the stored envelope is for fp16 operands");
        float sn, cs;
        sincospif((float)d / A.basis.r_cut, &sn, &cs);
        C = 0.5f * (cs + 1.0f);
        if (half == 0)
            reinterpret_cast<float2 *>(R + S::CD)[n] = make_float2(C, -0.5f * (float)M_PI / A.basis.r_cut * sn);
        d_hi = (float)d;
        d_lo = 0.0f;
    } else {
        C = 0.5f * (cospif(SPLIT ? (float)((double)d / A.basis.r_cut_d) : (float)d / A.basis.r_cut) + 1.0f);
        d_hi = (float)d;
        d_lo = SPLIT ? (float)((double)d - (double)d_hi) : 0.0f;
    }
    const float g2 = -A.basis.gamma * LOG2EF;
    const float *mh = reinterpret_cast<const float *>(sm + S::MUH) + half * (KP / PARTS);
    const float *ml = reinterpret_cast<const float *>(sm + S::MUL) + half * (KP / PARTS);
    unsigned char *Bh = R + S::B;
    unsigned char *Bl = Bh + S::BB;
    const uint32_t row = (uint32_t)((n & 7) * 16 + (n >> 3) * S::SW1);
#pragma unroll 1
    for (int qq = 0; qq < KP / (8 * PARTS); ++qq) {
        const int q = half * (KP / (8 * PARTS)) + qq;
        float v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int k = 8 * qq + c;
            const float x = SPLIT ? (d_hi - mh[k]) + (d_lo - ml[k]) : d_hi - mh[k];
            v[c] = ex2_approx(x * g2 * x) * C;
        }
        store8<SPLIT>(Bh, Bl, row + (uint32_t)q * 128, v);
    }
}

// D_A[f][n] = sum_k W1[f][k] bt[n][k]                          (M = 128, N = TE)
template <class S, int KP, bool SPLIT>
__device__ __forceinline__ void issue_mma1(unsigned char *sm, unsigned char *R, uint32_t d)
{
    constexpr uint32_t ID = idesc_f16(128, TE, 0, 0);
    const uint32_t wh = smem_u32(sm + S::W1), wl = wh + S::W1B;
    const uint32_t bh = smem_u32(R + S::B), bl = bh + S::BB;
#pragma unroll
    for (int j = 0; j < KP / 16; ++j) {
        const uint32_t o = (uint32_t)j * 256;
        mma_f16(d, sdesc(wh + o, 128, S::SW1), sdesc(bh + o, 128, S::SW1), ID, j > 0);
        if (SPLIT) {
            mma_f16(d, sdesc(wh + o, 128, S::SW1), sdesc(bl + o, 128, S::SW1), ID, 1);
            mma_f16(d, sdesc(wl + o, 128, S::SW1), sdesc(bh + o, 128, S::SW1), ID, 1);
        }
    }
}

// TRANS = false: D[o][n] = sum_i W2[o][i] T[n][i]   (forward filter layer 2)
// TRANS = true : D[i][n] = sum_o W2[o][i] T[n][o]   (backward through layer 2)
template <class S, bool SPLIT, bool TRANS>
__device__ __forceinline__ void issue_mma_w2(unsigned char *sm, unsigned char *R, uint32_t d)
{
    constexpr uint32_t ID = idesc_f16(128, TE, TRANS ? 1 : 0, 1);
    const uint32_t wh = smem_u32(sm + S::W2), wl = wh + S::W2B;
    const uint32_t th = smem_u32(R + S::T), tl = th + S::TB;
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

// D_G[n][k] = sum_f abar[n][f] W1[f][k]   (edges on M: M = TE = 64; row n of D sits in TMEM
// lane (n % 16) + 32 (n / 16))
template <class S, int KP, bool SPLIT>
__device__ __forceinline__ void issue_mma4(unsigned char *sm, unsigned char *R, uint32_t d)
{
    constexpr uint32_t ID = idesc_f16(TE, KP, 1, 1);
    const uint32_t wh = smem_u32(sm + S::W1), wl = wh + S::W1B;
    const uint32_t th = smem_u32(R + S::T), tl = th + S::TB;
#pragma unroll
    for (int j = 0; j < FF / 16; ++j) {
        const uint32_t oa = (uint32_t)j * 256, ob = (uint32_t)j * 2 * S::SW1;
        mma_f16(d, sdesc(th + oa, 128, 2048), sdesc(wh + ob, S::SW1, 128), ID, j > 0);
        if (SPLIT) {
            mma_f16(d, sdesc(tl + oa, 128, 2048), sdesc(wh + ob, S::SW1, 128), ID, 1);
            mma_f16(d, sdesc(th + oa, 128, 2048), sdesc(wl + ob, S::SW1, 128), ID, 1);
        }
    }
}

// Kernel set-up: weights to shared memory by bulk copies, one mbarrier per warpgroup, TMEM
// for the CTA.  Returns the TMEM base; skip is set when a latched condition (or a time-out
// of the copies) means the kernel must do nothing.
template <int KP, bool SPLIT, int NW>
__device__ __forceinline__ uint32_t setup(const EdgeTcArgs &A, unsigned char *sm, int &skip)
{
    using S = TcSmem<KP, SPLIT, NW>;
    const int warp = threadIdx.x >> 5;
    const uint32_t wmbar = smem_u32(sm + S::WMBAR);
    if (threadIdx.x == 0) {
        for (int g = 0; g < NW; ++g) mbar_init(smem_u32(sm + S::GROUPS + g * S::REGION + S::MBAR), 1);
        mbar_init(wmbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        mbar_expect_tx(wmbar, S::NS * (S::W1B + S::W2B));   // constant weights: before the wait
        bulk_g2s(smem_u32(sm + S::W1), A.W1h, S::W1B, wmbar);
        bulk_g2s(smem_u32(sm + S::W2), A.W2h, S::W2B, wmbar);
        if (SPLIT) {
            bulk_g2s(smem_u32(sm + S::W1 + S::W1B), A.W1l, S::W1B, wmbar);
            bulk_g2s(smem_u32(sm + S::W2 + S::W2B), A.W2l, S::W2B, wmbar);
        }
    }
    if (threadIdx.x < 64) {
        reinterpret_cast<float *>(sm + S::MUH)[threadIdx.x] = A.basis.mu_hi[threadIdx.x];
        reinterpret_cast<float *>(sm + S::MUL)[threadIdx.x] = A.basis.mu_lo[threadIdx.x];
    }
    if (warp == 0) tmem_alloc(smem_u32(sm + S::HOLD), 128 * NW);
    pdl_trigger();
    pdl_wait();   // from here on: data written by the preceding kernels
    if (threadIdx.x == 0)
        skip = (*((volatile const int *)A.d_err) & (ERRBIT_NONFINITE | ERRBIT_CAPACITY | ERRBIT_TIMEOUT)) != 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *reinterpret_cast<volatile uint32_t *>(sm + S::HOLD);
}

// The weight copies land while each group gathers its first tile; a group waits for them
// before its first MMA (wait_weights), and the CTA waits once more here so that it never
// leaves with copies in flight (a no-op when they have landed).
template <int KP, bool SPLIT, int NW>
__device__ __forceinline__ void teardown(unsigned char *sm, uint32_t tmem, int *d_err)
{
    using S = TcSmem<KP, SPLIT, NW>;
    wait_copies(smem_u32(sm + S::WMBAR), d_err);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if ((threadIdx.x >> 5) == 0) tmem_dealloc(tmem, 128 * NW);
}

// Per-warpgroup context: group g, thread t in group (= TMEM lane = feature), its shared region,
// mbarrier, TMEM columns and row range.
struct Group {
    int g, t;
    unsigned char *R;
    uint32_t mbar, tm, lane;
    int i0, i1;
    long long lim;   // bound of the waits for this group's MMAs
};

template <int KP, bool SPLIT, int NW>
__device__ __forceinline__ Group make_group(const EdgeTcArgs &A, unsigned char *sm, uint32_t tmem0)
{
    using S = TcSmem<KP, SPLIT, NW>;
    Group G;
    G.g = threadIdx.x / WGT;
    G.t = threadIdx.x % WGT;
    G.R = sm + S::GROUPS + G.g * S::REGION;
    G.mbar = smem_u32(G.R + S::MBAR);
    G.tm = tmem0 + (uint32_t)G.g * 128;
    G.lane = (uint32_t)((G.t >> 5) * 32) << 16;
    const int p = blockIdx.x * NW + G.g;
    G.i0 = A.part[p];
    G.i1 = A.part[p + 1];
    G.lim = A.wait_limit;
    return G;
}

template <int KP, bool SPLIT, int NW>
__device__ __forceinline__ bool wait_weights(const Group &G, unsigned char *sm, int *d_err)
{
    using S = TcSmem<KP, SPLIT, NW>;
    uint32_t parity = 0;
    return wait_mma(G.g, smem_u32(sm + S::WMBAR), parity, d_err, G.lim);
}

// Make this group's shared-memory writes visible to the tensor core, then let thread 0 of the
// group issue the MMAs of `issue` and commit them to the group's mbarrier; all threads wait.
template <typename Issue>
__device__ __forceinline__ bool mma_step(const Group &G, uint32_t &phase, int *d_err, Issue issue)
{
    fence_async_smem();
    tc_fence_before();
    wg_sync(G.g);
    if (G.t == 0) {
        tc_fence_after();
        issue();
        mma_commit(G.mbar);
    }
    return wait_mma(G.g, G.mbar, phase, d_err, G.lim);
}

// After a wait gave up: one more commit, whose completion follows that of every MMA the group
// issued, waited for with the default bound, so that no MMA still writes TMEM when it is freed.
__device__ __forceinline__ void drain_group(const Group &G, uint32_t &phase, int *d_err)
{
    tc_fence_before();
    wg_sync(G.g);
    if (G.t == 0) {
        tc_fence_after();
        mma_commit(G.mbar);
    }
    wait_mma(G.g, G.mbar, phase, d_err, WAIT_BOUND);
}

// s = ssp(a + b1) from TMEM columns [COL_A, COL_A + TE) into the activation tile
template <bool SPLIT, int CH>
__device__ __forceinline__ void ssp_to_tile(const Group &G, float s1f, float b1f, unsigned char *Th, unsigned char *Tl)
{
#pragma unroll 1
    for (int c = 0; c < TE / CH; ++c) {
        float v[CH];
        tmem_ld<CH>(G.tm + G.lane + COL_A + CH * c, v);
#pragma unroll
        for (int q = 0; q < CH; ++q) v[q] = ssp_mode<SPLIT>(fmaf(v[q], s1f, b1f));
        store_tile_col<SPLIT, CH>(Th, Tl, G.t, CH * c, v);
    }
}

template <int KP, bool SPLIT, int NW, int CH>
__global__ void __launch_bounds__(WGT *NW, 1) k_edge_fwd_tc(EdgeTcArgs A)
{
    using S = TcSmem<KP, SPLIT, NW>;
    extern __shared__ __align__(128) unsigned char sm[];
    __shared__ int skip;
    const uint32_t tmem0 = setup<KP, SPLIT, NW>(A, sm, skip);
    const Group G = make_group<KP, SPLIT, NW>(A, sm, tmem0);
    const int f = G.t;
    if (!skip && G.i0 < G.i1) {
        const int e0 = A.row_ptr[G.i0], e1 = A.row_ptr[G.i1];
        const float b1f = A.b1[f], b2f = A.b2[f], s1f = A.s1[f], s2f = A.s2[f];
        const float *xbase = x_base(A, f);
        const int *sXo = reinterpret_cast<const int *>(G.R + S::XO);
        const int *sDst = reinterpret_cast<const int *>(G.R + S::DST);
        unsigned char *Th = G.R + S::T, *Tl = Th + S::TB;
        uint32_t phase = 0;
        int cur = G.i0;
        float hacc = 0.0f;
        // h_i += x_src (.) (w + b2) over one chunk of CH edges, running sums per destination
        // row; a row is written when the next one starts (rows in between have no edges)
        // (one pass per row segment of the chunk, the row change in the code once; padding
        // edges gather row 0 and are not summed)
        const uint32_t *sMask = reinterpret_cast<const uint32_t *>(G.R + S::MASK);
        auto chunk = [&](int c, int ne, uint64_t starts) {
            float v[CH], xs[CH];
            tmem_ld<CH>(G.tm + G.lane + COL_W + CH * c, v);
#pragma unroll
            for (int q = 0; q < CH; ++q) xs[q] = __ldg(xbase + sXo[CH * c + q]);
            const uint32_t m = (uint32_t)(starts >> (CH * c)) & (CH >= 32 ? 0xffffffffu : (1u << (CH & 31)) - 1u);
            const int qend = min(CH, ne - CH * c);
            uint32_t rem = m;
            int q0 = 0;
#pragma unroll 1
            for (;;) {
                const int q1 = rem ? __ffs(rem) - 1 : qend;
#pragma unroll
                for (int q = 0; q < CH; ++q)
                    if (q >= q0 && q < q1) hacc = fmaf(xs[q], fmaf(v[q], s2f, b2f), hacc);
                if (!rem) break;
                const int i = sDst[CH * c + q1];
                A.H[(int64_t)cur * FF + f] = hacc;
                for (int r = cur + 1; r < i; ++r) A.H[(int64_t)r * FF + f] = 0.0f;
                hacc = 0.0f;
                cur = i;
                rem &= rem - 1u;
                q0 = q1;
            }
        };
        bool ok = true;
        const int nf = f & (TE - 1);   // this thread's edge in every tile's prologue
        EdgeIdx nidx = load_idx(A, e0 + nf, e1);
        EdgePos npos = load_pos(A, nidx);
        for (int ts = e0; ts < e1 && ok; ts += TE) {
            const int ne = min(TE, e1 - ts);
            tile_prologue<S, KP, SPLIT, false>(A, sm, G.R, f, ts, ne, nidx, npos);
            const bool more = ts + TE < e1;
            if (more) nidx = load_idx(A, ts + TE + nf, e1);
            if (ts == e0 && !(ok = wait_weights<KP, SPLIT, NW>(G, sm, A.d_err))) break;
            if (!(ok = mma_step(G, phase, A.d_err, [&] { issue_mma1<S, KP, SPLIT>(sm, G.R, G.tm + COL_A); }))) break;
            ssp_to_tile<SPLIT, CH>(G, s1f, b1f, Th, Tl);
            if (more) npos = load_pos(A, nidx);
            if (!(ok = mma_step(G, phase, A.d_err, [&] { issue_mma_w2<S, SPLIT, false>(sm, G.R, G.tm + COL_W); })))
                break;
            const uint64_t starts = (uint64_t)sMask[0] | ((uint64_t)sMask[1] << 32);
#pragma unroll 1
            for (int c = 0; c < TE / CH; ++c)
                if (CH * c < ne) chunk(c, ne, starts);
            tc_fence_before();
            wg_sync(G.g);
        }
        if (ok) {
            A.H[(int64_t)cur * FF + f] = hacc;
            for (int r = cur + 1; r < G.i1; ++r) A.H[(int64_t)r * FF + f] = 0.0f;   // trailing rows without edges
        } else {
            drain_group(G, phase, A.d_err);
        }
    }
    teardown<KP, SPLIT, NW>(sm, tmem0, A.d_err);
}

// Backward of one interaction block over the group's rows (see sn_ef_fp32.cu for the algebra):
// recompute a = W1 bt + b1 and w = W2 ssp(a) + b2; xbar_i += sum_j hbar_j (.) w_ij;
// wbar = x_j (.) hbar_i + x_i (.) hbar_j; sbar = W2^T wbar; abar = sbar (.) sigma(a);
// btbar = W1^T abar (edges on M); dbar = btbar . d(bt)/dd; F_i -= dbar * u_ij / d_ij by the
// row's owner only.  TMEM columns are reused: sbar overwrites w, btbar overwrites a.
template <int KP, bool SPLIT, int NW, int CH>
__global__ void __launch_bounds__(WGT *NW, 1) k_edge_bwd_tc(EdgeTcArgs A)
{
    using S = TcSmem<KP, SPLIT, NW>;
    extern __shared__ __align__(128) unsigned char sm[];
    __shared__ int skip;
    const uint32_t tmem0 = setup<KP, SPLIT, NW>(A, sm, skip);
    const Group G = make_group<KP, SPLIT, NW>(A, sm, tmem0);
    const int f = G.t;
    if (!skip && G.i0 < G.i1) {
        const int e0 = A.row_ptr[G.i0], e1 = A.row_ptr[G.i1];
        const float b1f = A.b1[f], b2f = A.b2[f], s1f = A.s1[f], s2f = A.s2[f];
        const float hs1 = 0.5f * s1f, hb1 = 0.5f * b1f;
        const float *xbase = x_base(A, f), *hbase = A.Hbar + f;
        const int2 *sOff = reinterpret_cast<const int2 *>(G.R + S::XO);
        const uint32_t *sMask = reinterpret_cast<const uint32_t *>(G.R + S::MASK);
        const int *sDst = reinterpret_cast<const int *>(G.R + S::DST);
        const double *sDist = reinterpret_cast<const double *>(G.R + S::DIST);
        const float *sU = reinterpret_cast<const float *>(G.R + S::UVEC);
        float *sFv = reinterpret_cast<float *>(G.R + S::FV);
        unsigned char *Th = G.R + S::T, *Tl = Th + S::TB;
        uint32_t phase = 0;
        bool ok = true;
        // Destination-row state: the running xbar sum of row cur, the row's own xbar, x_i and
        // hbar_i, and the same values of row cur + 1 read ahead (the usual next row).  x_i and
        // hbar_i enter only wbar, which is W2's transposed operand: they carry W2's channel
        // scale s2 (wbar s2 = x_j (hbar_i s2) + (x_i s2) hbar_j).
        int cur = -1, nrow = -1;
        float xbacc = 0.0f, xbold = 0.0f, xi_c = 0.0f, hi_c = 0.0f, nxb = 0.0f, nxi = 0.0f, nhi = 0.0f;
        // the values of row i (read ahead when it is cur + 1): xbar^{t+1}_i, x_i s2, hbar_i s2
        auto row_vals = [&](int i, float &xb, float &xi, float &hi) {
            if (i == nrow) {
                xb = nxb;
                xi = nxi * s2f;
                hi = nhi * s2f;
            } else {
                xb = A.Xbar[(int64_t)i * FF + f];
                xi = __ldg(x_row(A, xbase, i)) * s2f;
                hi = __ldg(hbase + (int64_t)i * FF) * s2f;
            }
        };
        // row i starts with the values (xb, xi, hi); the previous row's xbar is written
        auto open_row = [&](int i, float xb, float xi, float hi, float sum) {
            if (cur >= 0) A.Xbar[(int64_t)cur * FF + f] = xbold + xbacc;
            xbacc = sum;
            cur = i;
            xbold = xb;
            xi_c = xi;
            hi_c = hi;
            nrow = i + 1 < A.N ? i + 1 : -1;
            if (nrow >= 0) {   // discarded unless row i + 1 is this group's next row; the loads
                               // stay here (ld_keep) and are scaled when the row starts
                nxb = ld_keep(A.Xbar + (int64_t)nrow * FF + f);
                nxi = ldnc_keep(x_row(A, xbase, nrow));
                nhi = ldnc_keep(hbase + (int64_t)nrow * FF);
            }
        };
        auto next_row = [&](int i) {
            float xb, xi, hi;
            row_vals(i, xb, xi, hi);
            open_row(i, xb, xi, hi, 0.0f);
        };
        // xbar_i += hbar_j (.) (w + b2) and the tile of wbar = x_j (.) hbar_i + x_i (.) hbar_j over
        // one chunk of CH edges (zero for padding edges)
        // A row changes exactly at the edges that start their row (the tile's row-start mask), so
        // chunks without a start skip the row bookkeeping.
        // (padding edges gather row 0, whose values are then discarded)
        auto chunk = [&](int c, int ne, uint64_t starts) {
            float w[CH], hb[CH], xj[CH];
            tmem_ld<CH>(G.tm + G.lane + COL_W + CH * c, w);
#pragma unroll
            for (int q = 0; q < CH; ++q) {
                const int2 o = sOff[CH * c + q];
                xj[q] = __ldg(xbase + o.x);
                hb[q] = __ldg(hbase + o.y);
            }
            const uint32_t m = (uint32_t)(starts >> (CH * c)) & (CH >= 32 ? 0xffffffffu : (1u << (CH & 31)) - 1u);
            const int qend = min(CH, ne - CH * c);   // valid edges of the chunk (>= 1)
            if (qend == CH && m == 0) {
#pragma unroll
                for (int q = 0; q < CH; ++q) {
                    xbacc = fmaf(hb[q], fmaf(w[q], s2f, b2f), xbacc);
                    xj[q] = xj[q] * hi_c + xi_c * hb[q];
                }
            } else if (qend == CH && (m & (m - 1u)) == 0) {
                // one row starts at edge p: edges before it finish row cur, edges from it use the
                // new row's values (two running sums, one pass)
                const int p = __ffs(m) - 1, r = sDst[CH * c + p];
                float xb, xi, hi;
                row_vals(r, xb, xi, hi);
                float a0 = xbacc, b0 = 0.0f;
#pragma unroll
                for (int q = 0; q < CH; ++q) {
                    const bool before = q < p;
                    const float t0 = fmaf(hb[q], fmaf(w[q], s2f, b2f), before ? a0 : b0);
                    a0 = before ? t0 : a0;
                    b0 = before ? b0 : t0;
                    xj[q] = xj[q] * (before ? hi_c : hi) + (before ? xi_c : xi) * hb[q];
                }
                xbacc = a0;
                open_row(r, xb, xi, hi, b0);
            } else {
                // row starts (or the ragged end of the list) in the chunk: one pass per row
                // segment [q0, q1) over the whole chunk under a predicate, so that the row change
                // is in the code once (the mask holds valid edges only)
                uint32_t rem = m;
                int q0 = 0;
#pragma unroll 1
                for (;;) {
                    const int q1 = rem ? __ffs(rem) - 1 : qend;
#pragma unroll
                    for (int q = 0; q < CH; ++q)
                        if (q >= q0 && q < q1) {
                            xbacc = fmaf(hb[q], fmaf(w[q], s2f, b2f), xbacc);
                            xj[q] = xj[q] * hi_c + xi_c * hb[q];
                        }
                    if (!rem) break;
                    next_row(sDst[CH * c + q1]);
                    rem &= rem - 1u;
                    q0 = q1;
                }
#pragma unroll
                for (int q = 0; q < CH; ++q)
                    if (q >= qend) xj[q] = 0.0f;
            }
            store_tile_col<SPLIT, CH>(Th, Tl, f, CH * c, xj);
        };
        const int nf = f & (TE - 1);   // this thread's edge in every tile's prologue
        EdgeIdx nidx = load_idx(A, e0 + nf, e1);
        EdgePos npos = load_pos(A, nidx);
        for (int ts = e0; ts < e1 && ok; ts += TE) {
            const int ne = min(TE, e1 - ts);
            tile_prologue<S, KP, SPLIT, true, 2, false, !SPLIT>(A, sm, G.R, f, ts, ne, nidx, npos);
            const bool more = ts + TE < e1;
            if (more) nidx = load_idx(A, ts + TE + nf, e1);
            if (ts == e0 && !(ok = wait_weights<KP, SPLIT, NW>(G, sm, A.d_err))) break;
            if (!(ok = mma_step(G, phase, A.d_err, [&] { issue_mma1<S, KP, SPLIT>(sm, G.R, G.tm + COL_A); }))) break;
            ssp_to_tile<SPLIT, CH>(G, s1f, b1f, Th, Tl);
            if (more) npos = load_pos(A, nidx);
            if (!(ok = mma_step(G, phase, A.d_err, [&] { issue_mma_w2<S, SPLIT, false>(sm, G.R, G.tm + COL_W); })))
                break;
            const uint64_t starts = (uint64_t)sMask[0] | ((uint64_t)sMask[1] << 32);
#pragma unroll 1
            for (int c = 0; c < TE / CH; ++c) {
                if (CH * c < ne) {
                    chunk(c, ne, starts);
                } else {   // no edge of the chunk: zero wbar columns
                    float z[CH];
#pragma unroll
                    for (int q = 0; q < CH; ++q) z[q] = 0.0f;
                    store_tile_col<SPLIT, CH>(Th, Tl, f, CH * c, z);
                }
            }
            if (!(ok = mma_step(G, phase, A.d_err, [&] { issue_mma_w2<S, SPLIT, true>(sm, G.R, G.tm + COL_W); })))
                break;
            // abar = sbar (.) sigma(a s1 + b1), times W1's channel scale s1 (W1's transposed operand)
#pragma unroll 1
            for (int c = 0; c < TE / CH; ++c) {
                float sb[CH], a[CH];
                tmem_ld<CH>(G.tm + G.lane + COL_W + CH * c, sb);
                tmem_ld<CH>(G.tm + G.lane + COL_A + CH * c, a);
#pragma unroll
                for (int q = 0; q < CH; ++q) sb[q] *= sigmoid_scaled<SPLIT>(a[q], s1f, b1f, hs1, hb1);
                store_tile_col<SPLIT, CH>(Th, Tl, f, CH * c, sb);
            }
            if (!(ok = mma_step(G, phase, A.d_err, [&] { issue_mma4<S, KP, SPLIT>(sm, G.R, G.tm + COL_A); }))) break;
            // D_G rows (edges) sit in lanes 0-15 of each warp's quadrant; the 16x64b loads give
            // edge n = 16 * quadrant + 8 (l % 2) + l / 4 to lanes l and l ^ 2 of the warp, which
            // take the even and the odd k.  dbar_n = sum_k D_G[n][k] d(bt_k)/dd and its force.
            {
                const int l = f & 31, par = (l >> 1) & 1;
                const int n = 16 * (f >> 5) + 8 * (l & 1) + (l >> 2);
                const bool mine = n < ne;
                const double d = mine ? sDist[n] : 0.0;
                float C, dC;
                if constexpr (SPLIT) {
                    const float ratio = (float)(d / A.basis.r_cut_d);
                    C = 0.5f * (cospif(ratio) + 1.0f);
                    dC = -0.5f * (float)M_PI / A.basis.r_cut * sinpif(ratio);
                } else {   // formed once per edge by the prologue
                    const float2 cd = mine ? reinterpret_cast<const float2 *>(G.R + S::CD)[n] : make_float2(0.0f, 0.0f);
                    C = cd.x;
                    dC = cd.y;
                }
                const float cc = -2.0f * A.basis.gamma * C, g2 = -A.basis.gamma * LOG2EF;
                const float d_hi = (float)d, d_lo = (float)(d - (double)d_hi);
                const float *mh = reinterpret_cast<const float *>(sm + S::MUH) + par;
                const float *ml = reinterpret_cast<const float *>(sm + S::MUL) + par;
                float gsum = 0.0f;
#pragma unroll 1
                for (int c = 0; c < KP / 32; ++c) {
                    float gg[16];
                    tmem_ld16x64b_x16(G.tm + G.lane + COL_A + 32 * c, gg);
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        const int k = 32 * c + 2 * r;   // + par
                        const float x = SPLIT ? (d_hi - mh[k]) + (d_lo - ml[k]) : d_hi - mh[k];
                        const float phi = ex2_approx(x * g2 * x);
                        gsum = fmaf(gg[r], phi * fmaf(x, cc, dC), gsum);
                    }
                }
                gsum += __shfl_xor_sync(0xffffffffu, gsum, 2);
                if (par == 0) {
                    sFv[3 * n] = mine ? -gsum * sU[3 * n] : 0.0f;
                    sFv[3 * n + 1] = mine ? -gsum * sU[3 * n + 1] : 0.0f;
                    sFv[3 * n + 2] = mine ? -gsum * sU[3 * n + 2] : 0.0f;
                }
            }
            tc_fence_before();
            wg_sync(G.g);
            if (f < TE) {
                // the tile's edge forces summed per destination row: segmented scan over edge
                // n = f in the group's first two warps (the second warp's leading segment adds the
                // first warp's last partial sum); the last edge of each segment adds the row's
                // sum to the forces with a reduction that returns nothing.  All additions to a
                // row come from this group, tile after tile, separated by its barriers, so their
                // order is fixed.
                const int lane = f & 31;
                const bool valid = f < ne;
                const int row = valid ? sDst[f] : -1;
                float fx = valid ? sFv[3 * f] : 0.0f, fy = valid ? sFv[3 * f + 1] : 0.0f,
                      fz = valid ? sFv[3 * f + 2] : 0.0f;
                int fl = valid && (f == 0 || sDst[f - 1] != row);
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float px = __shfl_up_sync(0xffffffffu, fx, o);
                    const float py = __shfl_up_sync(0xffffffffu, fy, o);
                    const float pz = __shfl_up_sync(0xffffffffu, fz, o);
                    const int pf = __shfl_up_sync(0xffffffffu, fl, o);
                    if (lane >= o) {
                        if (!fl) {
                            fx += px;
                            fy += py;
                            fz += pz;
                        }
                        fl |= pf;
                    }
                }
                float *sPX = reinterpret_cast<float *>(G.R + S::PDX);
                if (f == 31) {
                    sPX[0] = fx;
                    sPX[1] = fy;
                    sPX[2] = fz;
                }
                named_sync(5 + G.g, TE);
                if (f >= 32 && !fl) {
                    fx += sPX[0];
                    fy += sPX[1];
                    fz += sPX[2];
                }
                if (valid && (f == ne - 1 || sDst[f + 1] != row)) {
                    atomicAdd(A.forces + (int64_t)row * 3, fx);
                    atomicAdd(A.forces + (int64_t)row * 3 + 1, fy);
                    atomicAdd(A.forces + (int64_t)row * 3 + 2, fz);
                }
            }
            wg_sync(G.g);
        }
        if (ok && cur >= 0) A.Xbar[(int64_t)cur * FF + f] = xbold + xbacc;
        if (!ok) drain_group(G, phase, A.d_err);
    }
    teardown<KP, SPLIT, NW>(sm, tmem0, A.d_err);
}

// ---------------------------------------------------------------- warp-specialised forward
// One CTA per SM walks the edges of its rows through a ring of NSTG tile stages, each step on
// its own warps, so that the basis of one tile, the MMAs of another and the activations and
// gathers of two more run at the same time:
//   warps 12-19 P  the source rows x_j gathered into the stage by the    -> full_x[s]
//                  tensor memory accelerator (four rows per instruction,
//                  issued first; they land while the prologue and the
//                  MMAs run)
//                  metadata and basis tile bt of tile k                  -> full_b[s]
//   warp  20    M  MMA1 a = W1 bt (after full_b[s])                      -> full_a[s]
//                  MMA2 w = W2 s  (after full_t[s]), over a's columns    -> full_w[s]
//   warps 4-11  S  s = ssp(a + b1) from TMEM into the stage's T tile     -> full_t[s]
//                  (two warpgroups, 32 of the tile's 64 columns each)
//   warps 0-3   E  h_i += x_j (.) (w + b2), running sums per row         -> free[s]
// Stage s = k % NSTG holds the tile's basis and activation tiles, its metadata, the source
// rows x_j and 64 TMEM columns.  Each barrier of stage s completes once per tile using the stage, so tile k waits
// for parity (k / NSTG) & 1 (and P, before refilling the stage, for the previous use's free).
constexpr int WS_WARPS = 21;
constexpr int WS_P = 2 * WGT, WS_S = 2 * WGT;   // producer and activation threads
// Roles by warp: E 0-3, S 4-11, P 12-19, M 20.  The epilogue, the ring's longest stage, takes
// the lowest warp indices: when several warps of a scheduler can issue, the older (lower)
// warps tend to be picked, and the producer and activation warps have slack to give.
constexpr int WS_E_WARP0 = 0, WS_S_WARP0 = 4, WS_P_WARP0 = 12;
constexpr int WS_M_WARP = 20;
constexpr int WS_CH = 8;   // TMEM columns (edges) per chunk of the activation warps
constexpr int WS_CE = 8;   // and of the epilogue warps
constexpr int WS_THREADS = WS_WARPS * 32;
enum WsBar { WB_FULL_B = 0, WB_FULL_A, WB_FULL_T, WB_FULL_W, WB_FREE, WB_FULL_X, WB_KINDS };

template <int KP, bool SPLIT, int NSTG>
struct WsSmem {
    static constexpr int NS = SPLIT ? 2 : 1;
    static constexpr uint32_t W1B = FF * KP * 2;
    static constexpr uint32_t W2B = FF * FF * 2;
    static constexpr uint32_t BB = TE * KP * 2;
    static constexpr uint32_t TB = TE * FF * 2;
    static constexpr uint32_t SW1 = (KP / 8) * 128;
    static constexpr uint32_t W1 = 0;
    static constexpr uint32_t W2 = W1 + NS * W1B;
    static constexpr uint32_t STAGES = W2 + NS * W2B;
    // offsets inside a stage (names as in TcSmem, which the prologue and MMA helpers use)
    static constexpr uint32_t B = 0;
    static constexpr uint32_t T = B + NS * BB;
    static constexpr uint32_t XO = T + NS * TB;
    static constexpr uint32_t HO = XO + 4 * TE;
    static constexpr uint32_t DST = HO + 4 * TE;
    static constexpr uint32_t DIST = DST + 4 * TE;
    static constexpr uint32_t UVEC = DIST + 8 * TE;
    static constexpr uint32_t FV = UVEC + 12 * TE;
    static constexpr uint32_t MASK = FV + 12 * TE;
    static constexpr uint32_t DF = MASK + 16;                        // float[TE]: d
    static constexpr uint32_t CC = DF + 4 * TE;                      // float[TE]: C(d)
    static constexpr uint32_t XS = (CC + 4 * TE + 127) / 128 * 128;   // float[TE][F]: x_j rows
    static constexpr uint32_t STG = XS + TE * FF * 4;
    static constexpr uint32_t BARS = STAGES + NSTG * STG;          // uint64 [WB_KINDS][NSTG]
    static constexpr uint32_t WMBAR = BARS + 8 * WB_KINDS * NSTG;  // weight copies
    static constexpr uint32_t DRAIN = WMBAR + 8;                   // last MMAs before teardown
    static constexpr uint32_t HOLD = DRAIN + 8;                    // TMEM address
    static constexpr uint32_t ABORT = HOLD + 8;                    // int: a wait timed out
    static constexpr uint32_t SKIP = ABORT + 4;                    // int: an earlier kernel failed
    static constexpr uint32_t MUH = ABORT + 8;
    static constexpr uint32_t MUL = MUH + 256;
    static constexpr uint32_t BYTES = MUL + 256;
    static constexpr uint32_t ALLOC = BYTES + 128;   // with the slack to align the base to 128 bytes
    static constexpr uint32_t TMEM_COLS = NSTG * 64 <= 128 ? 128 : NSTG * 64 <= 256 ? 256 : 512;
};

// Bounded wait on one barrier phase by every thread of a warp.  A time-out raises the CTA's
// abort flag, which ends every other wait of the CTA at once; the result is warp-uniform.
static __device__ __forceinline__ bool ws_wait(uint32_t bar, uint32_t parity, volatile int *abort, int *d_err,
                                               long long lim)
{
    const long long t0 = clock64();
    int ok = 1;
    while (!mbar_test_wait(bar, parity)) {
        if (*abort) {
            ok = 0;
            break;
        }
        if (clock64() - t0 > lim) {
            *abort = 1;
            atomicOr(d_err, ERRBIT_TIMEOUT);
            ok = 0;
            break;
        }
        if (mbar_try_wait(bar, parity)) break;
    }
    return __all_sync(0xffffffffu, ok) != 0;
}

// xmap: the block's source feature rows (x^t, or the embedding table in block 0) as a 2-D
// tensor [rows][F] of fp32 with boxes of one row.  The shared-memory plan starts at the first
// 128-byte boundary of the dynamic window, so that the stages' row tiles, the gathers'
// destinations, are 128-byte aligned.
template <int KP, bool SPLIT, int NSTG, int CH, int CE>
__global__ void __launch_bounds__(WS_THREADS, 1)
    k_edge_fwd_ws(EdgeTcArgs A, int parts_per_cta, const __grid_constant__ CUtensorMap xmap)
{
    using S = WsSmem<KP, SPLIT, NSTG>;
    extern __shared__ __align__(128) unsigned char sm_window[];
    unsigned char *const sm = sm_window + ((128u - (smem_u32(sm_window) & 127u)) & 127u);
    int &skip = *reinterpret_cast<int *>(sm + S::SKIP);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto bar = [&](int kind, int s) { return smem_u32(sm + S::BARS + 8 * (kind * NSTG + s)); };
    auto stage = [&](int s) { return sm + S::STAGES + s * S::STG; };
    volatile int *abort = reinterpret_cast<volatile int *>(sm + S::ABORT);
    const uint32_t wmbar = smem_u32(sm + S::WMBAR), drain = smem_u32(sm + S::DRAIN);
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTG; ++s) {
            mbar_init(bar(WB_FULL_B, s), WS_P);   // each P thread once its stores are done
            mbar_init(bar(WB_FULL_X, s), 2);      // P warps 0 and 1, with the bytes of their gathers
            mbar_init(bar(WB_FULL_A, s), 1);
            mbar_init(bar(WB_FULL_T, s), WS_S);
            mbar_init(bar(WB_FULL_W, s), 1);
            mbar_init(bar(WB_FREE, s), WGT);
        }
        mbar_init(wmbar, 1);
        mbar_init(drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        *abort = 0;
        mbar_expect_tx(wmbar, S::NS * (S::W1B + S::W2B));   // constant weights: before the wait
        bulk_g2s(smem_u32(sm + S::W1), A.W1h, S::W1B, wmbar);
        bulk_g2s(smem_u32(sm + S::W2), A.W2h, S::W2B, wmbar);
        if (SPLIT) {
            bulk_g2s(smem_u32(sm + S::W1 + S::W1B), A.W1l, S::W1B, wmbar);
            bulk_g2s(smem_u32(sm + S::W2 + S::W2B), A.W2l, S::W2B, wmbar);
        }
    }
    if (threadIdx.x < 64) {
        reinterpret_cast<float *>(sm + S::MUH)[threadIdx.x] = A.basis.mu_hi[threadIdx.x];
        reinterpret_cast<float *>(sm + S::MUL)[threadIdx.x] = A.basis.mu_lo[threadIdx.x];
    }
    if (warp == WS_M_WARP) tmem_alloc(smem_u32(sm + S::HOLD), S::TMEM_COLS);
    pdl_trigger();
    pdl_wait();   // from here on: data written by the preceding kernels
    if (threadIdx.x == 0)
        skip = (*((volatile const int *)A.d_err) & (ERRBIT_NONFINITE | ERRBIT_CAPACITY | ERRBIT_TIMEOUT)) != 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + S::HOLD);

    const int r0 = A.part[blockIdx.x * parts_per_cta], r1 = A.part[(blockIdx.x + 1) * parts_per_cta];
    const int e0 = r0 < r1 ? A.row_ptr[r0] : 0, e1 = r0 < r1 ? A.row_ptr[r1] : 0;
    const int nt = (e1 - e0 + TE - 1) / TE;
    if (!skip && r0 < r1) {
        if (warp >= WS_P_WARP0 && warp < WS_M_WARP) {
            // P: the prologue of tile k (edge n = t % 64, a quarter of its Gaussians per
            // thread), with tile k + 1's indices and positions read ahead by part 0 (t < 64),
            // the only part that uses them (metadata, row starts, gathers); the other parts
            // take d and C(d) from the stage
            const int t = threadIdx.x - 32 * WS_P_WARP0, nf = t & (TE - 1);
            const int e_lim = t < TE ? e1 : 0;   // (load_idx gives zeros at or past e_lim)
            EdgeIdx nidx = load_idx(A, e0 + nf, e_lim);
            EdgePos npos{};
            if (t < TE) npos = load_pos(A, nidx);
            for (int k = 0; k < nt; ++k) {
                const int s = k % NSTG, ts = e0 + k * TE, ne = min(TE, e1 - ts);
                int okw = 1;
                if (k >= NSTG) okw = ws_wait(bar(WB_FREE, s), ((k / NSTG) - 1) & 1, abort, A.d_err, A.wait_limit);
                if (!named_sync_and(5, WS_P, okw)) break;   // all P warps go on or stop together
                const EdgeIdx cidx = nidx;
                const EdgePos cpos = npos;
                if (k + 1 < nt) nidx = load_idx(A, ts + TE + nf, e_lim);
                if (t < 64) {
                    // source rows first, so that they land during the prologue: lane 4 g of P
                    // warp w (0 or 1) gathers the rows of edges 32 w + 4 g + [0, 4), which lanes
                    // 4 g .. 4 g + 3 hold (padding edges of the last group read the row of atom 0);
                    // lane 0 first announces the warp's bytes on the stage's barrier
                    const int w = t >> 5, lane = t & 31;
                    const int row = A.t == 0 ? cpos.tj : cidx.j;
                    const int r1 = __shfl_down_sync(0xffffffffu, row, 1);
                    const int r2 = __shfl_down_sync(0xffffffffu, row, 2);
                    const int r3 = __shfl_down_sync(0xffffffffu, row, 3);
                    const int groups = min(8, max(0, (ne - 32 * w + 3) / 4));
                    if (lane == 0) mbar_expect_tx(bar(WB_FULL_X, s), (uint32_t)groups * 4 * FF * 4);
                    __syncwarp();
                    if ((lane & 3) == 0 && (lane >> 2) < groups)
                        tma_gather4(smem_u32(stage(s) + S::XS) + (32 * w + lane) * FF * 4, &xmap, 0, row, r1, r2, r3,
                                    bar(WB_FULL_X, s));
                }
                tile_prologue<S, KP, SPLIT, false, 4, true>(A, sm, stage(s), t, ts, ne, cidx, cpos);
                fence_async_smem();
                mbar_arrive(bar(WB_FULL_B, s));
                if (k + 1 < nt && t < TE) npos = load_pos(A, nidx);
            }
        } else if (warp == WS_M_WARP) {
            // M: lane 0 polls the two queues and issues whichever MMA is ready: MMA1 of the next
            // tile whose basis is in (and whose stage E has released), MMA2 of the oldest tile
            // whose activations S has written.  Decisions are broadcast so the warp stays uniform.
            bool ok = ws_wait(wmbar, 0, abort, A.d_err, A.wait_limit);
            bool issued = false;
            int k1 = 0, k2 = 0;
            long long last = clock64();
            while (ok && k2 < nt) {
                int go1 = 0, go2 = 0;
                if (lane == 0) {
                    if (k1 < nt) {
                        const int s = k1 % NSTG;
                        go1 = mbar_test_wait(bar(WB_FULL_B, s), (k1 / NSTG) & 1) &&
                              (k1 < NSTG || mbar_test_wait(bar(WB_FREE, s), ((k1 / NSTG) - 1) & 1));
                    }
                    if (k2 < k1) go2 = mbar_test_wait(bar(WB_FULL_T, k2 % NSTG), (k2 / NSTG) & 1);
                }
                go1 = __shfl_sync(0xffffffffu, go1, 0);
                go2 = __shfl_sync(0xffffffffu, go2, 0);
                if (go1) {
                    const int s = k1 % NSTG;
                    tc_fence_after();
                    if (lane == 0) {
                        issue_mma1<S, KP, SPLIT>(sm, stage(s), tmem + 64 * s);
                        mma_commit(bar(WB_FULL_A, s));
                    }
                    ++k1;
                    issued = true;
                }
                if (go2) {
                    const int s2 = k2 % NSTG;
                    tc_fence_after();
                    if (lane == 0) {
                        issue_mma_w2<S, SPLIT, false>(sm, stage(s2), tmem + 64 * s2);
                        mma_commit(bar(WB_FULL_W, s2));
                    }
                    ++k2;
                }
                __syncwarp();
                if (go1 || go2) {
                    last = clock64();
                } else if (*abort) {
                    ok = false;
                } else if (clock64() - last > A.wait_limit) {
                    if (lane == 0) {
                        *abort = 1;
                        atomicOr(A.d_err, ERRBIT_TIMEOUT);
                    }
                    ok = false;
                } else {
                    __nanosleep(32);   // nothing ready: leave the issue slots to the other warps
                }
                ok = __all_sync(0xffffffffu, ok);
            }
            if (issued) {   // every MMA of this CTA complete before TMEM is released
                if (lane == 0) mma_commit(drain);
                __syncwarp();
                const long long t0 = clock64();
                while (!mbar_try_wait(drain, 0))
                    if (clock64() - t0 > (1ll << 32)) {
                        if (lane == 0) atomicOr(A.d_err, ERRBIT_TIMEOUT);
                        break;
                    }
                __syncwarp();
            }
        } else if (warp >= WS_S_WARP0) {
            // S: s = ssp(a + b1) into the stage's activation tile, columns [32 sg, 32 sg + 32)
            const int f = (threadIdx.x - 32 * WS_S_WARP0) % WGT, sg = (threadIdx.x - 32 * WS_S_WARP0) / WGT;
            const float b1f = A.b1[f], s1f = A.s1[f];
            const uint32_t lanes = (uint32_t)((warp & 3) * 32) << 16;
            for (int k = 0; k < nt; ++k) {
                const int s = k % NSTG;
                if (!ws_wait(bar(WB_FULL_A, s), (k / NSTG) & 1, abort, A.d_err, A.wait_limit)) break;
                tc_fence_after();
                unsigned char *Th = stage(s) + S::T, *Tl = Th + S::TB;
#pragma unroll 1
                for (int c = sg * (TE / CH / 2); c < (sg + 1) * (TE / CH / 2); ++c) {
                    float v[CH];
                    tmem_ld<CH>(tmem + lanes + 64 * s + CH * c, v);
#pragma unroll
                    for (int q = 0; q < CH; ++q) v[q] = ssp_mode<SPLIT>(fmaf(v[q], s1f, b1f));
                    store_tile_col<SPLIT, CH>(Th, Tl, f, CH * c, v);
                }
                tc_fence_before();
                fence_async_smem();
                mbar_arrive(bar(WB_FULL_T, s));
            }
        } else {
            // E: h_i += x_src (.) (w + b2); a row is written when the next one starts (rows in
            // between, and after the last edge, have no edges and receive zero)
            const int f = threadIdx.x - 32 * WS_E_WARP0;
            const float b2f = A.b2[f], s2f = A.s2[f];
            const uint32_t lanes = (uint32_t)((warp & 3) * 32) << 16;
            int cur = r0;
            float hacc = 0.0f;
            bool ok = true;
            for (int k = 0; k < nt; ++k) {
                const int s = k % NSTG, ne = min(TE, e1 - (e0 + k * TE));
                if (!(ok = ws_wait(bar(WB_FULL_W, s), (k / NSTG) & 1, abort, A.d_err, A.wait_limit))) break;
                // P's metadata (completed already) and the copied source rows
                if (!(ok = ws_wait(bar(WB_FULL_B, s), (k / NSTG) & 1, abort, A.d_err, A.wait_limit))) break;
                if (!(ok = ws_wait(bar(WB_FULL_X, s), (k / NSTG) & 1, abort, A.d_err, A.wait_limit))) break;
                tc_fence_after();
                const float *sXs = reinterpret_cast<const float *>(stage(s) + S::XS) + f;
                const int *sDst = reinterpret_cast<const int *>(stage(s) + S::DST);
                const uint32_t *sMask = reinterpret_cast<const uint32_t *>(stage(s) + S::MASK);
                const uint64_t starts = (uint64_t)sMask[0] | ((uint64_t)sMask[1] << 32);
                // h of the rows started in the chunk: one pass per row segment [q0, q1) over the
                // whole chunk under a predicate, so that the row change is in the code once; a
                // finished row is written when the next starts, rows in between (without edges)
                // receive zero
                auto chunk = [&](int c) {
                    float v[CE], xs[CE];
                    tmem_ld<CE>(tmem + lanes + 64 * s + CE * c, v);
#pragma unroll
                    for (int q = 0; q < CE; ++q) xs[q] = sXs[(CE * c + q) * FF];
                    const uint32_t m = (uint32_t)(starts >> (CE * c)) & (CE >= 32 ? 0xffffffffu : (1u << (CE & 31)) - 1u);
                    const int qend = min(CE, ne - CE * c);   // valid edges of the chunk (>= 1)
                    if (qend == CE && m == 0) {   // the chunk continues the current row
#pragma unroll
                        for (int q = 0; q < CE; ++q) hacc = fmaf(xs[q], fmaf(v[q], s2f, b2f), hacc);
                        return;
                    }
                    if (qend == CE && (m & (m - 1u)) == 0) {
                        // one row starts at edge p of the chunk: edges before it finish row cur,
                        // edges from it open the next row (two running sums, one pass)
                        const int p = __ffs(m) - 1;
                        float a0 = hacc, b0 = 0.0f;
#pragma unroll
                        for (int q = 0; q < CE; ++q) {
                            const bool before = q < p;
                            const float t0 = fmaf(xs[q], fmaf(v[q], s2f, b2f), before ? a0 : b0);
                            a0 = before ? t0 : a0;
                            b0 = before ? b0 : t0;
                        }
                        const int r = sDst[CE * c + p];
                        store_if(A.H + (int64_t)cur * FF + f, a0, true);
                        for (int rr = cur + 1; rr < r; ++rr) store_if(A.H + (int64_t)rr * FF + f, 0.0f, true);
                        cur = r;
                        hacc = b0;
                        return;
                    }
                    uint32_t rem = m;
                    int q0 = 0;
#pragma unroll 1
                    for (;;) {
                        const int q1 = rem ? __ffs(rem) - 1 : qend;
#pragma unroll
                        for (int q = 0; q < CE; ++q)
                            if (q >= q0 && q < q1) hacc = fmaf(xs[q], fmaf(v[q], s2f, b2f), hacc);
                        if (!rem) break;
                        const int r = sDst[CE * c + q1];
                        store_if(A.H + (int64_t)cur * FF + f, hacc, true);
                        for (int rr = cur + 1; rr < r; ++rr) store_if(A.H + (int64_t)rr * FF + f, 0.0f, true);
                        hacc = 0.0f;
                        cur = r;
                        rem &= rem - 1u;
                        q0 = q1;
                    }
                };
#pragma unroll 1
                for (int c = 0; c < TE / CE; ++c)
                    if (CE * c < ne) chunk(c);
                tc_fence_before();
                mbar_arrive(bar(WB_FREE, s));
            }
            if (ok) {
                store_if(A.H + (int64_t)cur * FF + f, hacc, true);
                for (int r = cur + 1; r < r1; ++r) store_if(A.H + (int64_t)r * FF + f, 0.0f, true);
            }
        }
    }
    wait_copies(wmbar, A.d_err);   // never leave with the weight copies in flight
    if (*abort) {
        // after a time-out, give source-row copies that no consumer waited for time to land
        const long long t0 = clock64();
        while (clock64() - t0 < (1ll << 22)) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == WS_M_WARP) tmem_dealloc(tmem, S::TMEM_COLS);
}

template <typename Kern>
cudaError_t prepare(Kern k, uint32_t bytes)
{
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Tensor map of rows x [0, rows) of an fp32 matrix [rows][F] at base (256-byte aligned): boxes
// of one row (F elements), no swizzle, zero fill outside, for the four-row gathers.
cudaError_t make_row_map(CUtensorMap *map, const float *base, int64_t rows)
{
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (rows < 1 || rows > (1ll << 31)) return cudaErrorInvalidValue;
    const cuuint64_t dims[2] = {(cuuint64_t)FF, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)FF * sizeof(float)};
    const cuuint32_t box[2] = {(cuuint32_t)FF, 1};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(base), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int KP, bool SPLIT, int NW, int CH>
cudaError_t launch_t(const EdgeTcArgs &a, bool backward, int G, cudaStream_t s)
{
    using S = TcSmem<KP, SPLIT, NW>;
    static_assert(S::BYTES <= 227 * 1024, "shared memory plan exceeds 227 KB");
    static_assert(NW == 2 || NW == 4, "TMEM allocations are powers of two: 2 or 4 groups");
    cudaError_t e;
    if (backward) {
        if ((e = prepare(k_edge_bwd_tc<KP, SPLIT, NW, CH>, S::BYTES))) return e;
        e = launch_pdl(k_edge_bwd_tc<KP, SPLIT, NW, CH>, dim3(G), dim3(WGT * NW), S::BYTES, s, a);
    } else if constexpr (!SPLIT) {
        constexpr int NSTG = 3;
        using WS = WsSmem<KP, false, NSTG>;
        static_assert(WS::ALLOC <= 227 * 1024, "shared memory plan exceeds 227 KB");
        if ((e = prepare(k_edge_fwd_ws<KP, false, NSTG, WS_CH, WS_CE>, WS::ALLOC))) return e;
        CUtensorMap xmap;
        if ((e = a.t == 0 ? make_row_map(&xmap, a.emb, a.n_types)
                          : make_row_map(&xmap, a.X + (int64_t)(a.t - 1) * a.N * FF, a.N)))
            return e;
        e = launch_pdl(k_edge_fwd_ws<KP, false, NSTG, WS_CH, WS_CE>, dim3(G), dim3(WS_THREADS), WS::ALLOC, s, a, NW,
                       xmap);
    } else {
        if ((e = prepare(k_edge_fwd_tc<KP, SPLIT, NW, CH>, S::BYTES))) return e;
        e = launch_pdl(k_edge_fwd_tc<KP, SPLIT, NW, CH>, dim3(G), dim3(WGT * NW), S::BYTES, s, a);
    }
    return e != cudaSuccess ? e : cudaGetLastError();
}

// The split (fp32-accurate) mode holds two fp16 copies of every operand: two warpgroups fit in
// shared memory.  The fp16 mode runs four (16 warps per SM), with 16-column chunks to stay
// within 128 registers per thread.
constexpr int groups_for(bool split) { return split ? 2 : 4; }

}  // namespace

int tc_groups_per_cta(bool split) { return groups_for(split); }

// G CTAs, each running tc_groups_per_cta(split) independent row ranges: a.part must hold
// G * tc_groups_per_cta(split) + 1 entries.
cudaError_t launch_edge_tc(const EdgeTcArgs &a, int KP, bool split, bool backward, int G, cudaStream_t s)
{
    if (KP == 64) return split ? launch_t<64, true, 2, 16>(a, backward, G, s) : launch_t<64, false, 4, 16>(a, backward, G, s);
    if (KP == 32) return split ? launch_t<32, true, 2, 16>(a, backward, G, s) : launch_t<32, false, 4, 16>(a, backward, G, s);
    return cudaErrorInvalidValue;
}

// Host: one weight matrix W[rows][cols] (fp32, row-major) into the core-matrix layout used by
// the kernels (element (r, c) at half index ((r%8)*16 + (r/8)*SBO + (c%8)*2 + (c/8)*128)/2,
// SBO = (cols_pad/8)*128 bytes, columns cols..cols_pad-1 zero), as fp16 hi and lo = fp16(w - hi)
// of w = W[r][c] / row_scale[r] (the division in fp32).
void tc_pack_matrix(const float *W, int rows, int cols, int cols_pad, const float *row_scale, uint16_t *hi,
                    uint16_t *lo)
{
    const size_t sbo = (size_t)(cols_pad / 8) * 128;
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols_pad; ++c) {
            const float w = c < cols ? W[(size_t)r * cols + c] / row_scale[r] : 0.0f;
            const __half h = __float2half_rn(w);
            const __half l = __float2half_rn(w - __half2float(h));
            const size_t byte = (size_t)(r % 8) * 16 + (size_t)(r / 8) * sbo + (size_t)(c % 8) * 2 + (size_t)(c / 8) * 128;
            hi[byte / 2] = __half_as_ushort(h);
            lo[byte / 2] = __half_as_ushort(l);
        }
}

}  // namespace sn
