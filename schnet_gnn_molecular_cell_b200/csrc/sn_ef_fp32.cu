// Energy and forces, fp32 on CUDA cores.
//
// Forward, per interaction block t (FlashSchNet §4.2 "Flash message passing fused edge
// computation", §4.3 "Destination grouped segmented reduction in forward pass"):
//   k_edge_fwd   each CTA owns a contiguous range of destination rows (balanced on edges +
//                atoms) and streams their edges in tiles of NE = 32.  Per tile: distances,
//                Gaussian basis x cosine envelope (shared memory only), filter network
//                a = W1 bt + b1, s = ssp(a), w = W2 s + b2 (weights resident in shared
//                memory), gather x_src, multiply, and a running per-row sum in registers.
//                Rows never span CTAs, so h_i is written once, without atomics.
//   k_node_fwd   p = U1 h + c1, x^{t+1} = x + U2 ssp(p) + c2; after the last block also the
//                readout eps = R2 ssp(R1 x + e1) + e2 and the start of the backward pass.
// Backward (hand-derived reverse mode of the above; §3.2 "Forces via autodiff"):
//   k_node_bwd   hbar = U1^T (sigma(p) (.) U2^T xbar)           (per atom)
//   k_edge_bwd   per edge j -> i of row i: recompute the filter; xbar_i += hbar_j (.) w_ij;
//                wbar = x_j (.) hbar_i + x_i (.) hbar_j; sbar = W2^T wbar;
//                abar = sbar (.) sigma(a); btbar = W1^T abar; dbar = btbar . d(bt)/dd;
//                F_i -= dbar * u_ij / d_ij.
// The backward uses the symmetry of the list (j -> i present iff i -> j) and w_ij = w_ji:
// the source-grouped sum of §4.3 ("Source grouped segmented reduction in backward pass")
// equals a destination-grouped sum over the same rows, and the two directed edges of a pair
// share one filter Jacobian, so each owner row yields its atom's complete force without a
// second index or any scatter.
#include <cuda_runtime.h>
#include <math.h>

#include "sn_internal.cuh"

namespace sn {

namespace {

constexpr float LN2 = 0.693147180559945309f;

__device__ __forceinline__ float ssp(float x) { return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x))) - LN2; }
__device__ __forceinline__ float sigmoid(float x) { return 1.0f / (1.0f + expf(-x)); }

__device__ __forceinline__ void copy_f4(float *dst, const float *src, int n, int tid, int nthr)
{
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
    float4 *d4 = reinterpret_cast<float4 *>(dst);
    for (int q = tid; q < n / 4; q += nthr) d4[q] = s4[q];
}

// u = r_i - r_j with the minimum image on periodic axes, and d = |u|, in double from the
// float positions (exact differences, one rounding of the length)
__device__ __forceinline__ double pair_vec(float4 ri, float4 rj, const Geometry &g, double3 &u)
{
    double dx = (double)ri.x - (double)rj.x, dy = (double)ri.y - (double)rj.y, dz = (double)ri.z - (double)rj.z;
    if (g.periodic[0]) dx -= (double)g.box[0] * rint(dx / (double)g.box[0]);
    if (g.periodic[1]) dy -= (double)g.box[1] * rint(dy / (double)g.box[1]);
    if (g.periodic[2]) dz -= (double)g.box[2] * rint(dz / (double)g.box[2]);
    u = make_double3(dx, dy, dz);
    return sqrt(dx * dx + dy * dy + dz * dz);
}

// row i of edge e inside the rows [i0, i1): largest i with row_ptr[i] <= e
__device__ __forceinline__ int edge_row(const int32_t *__restrict__ row_ptr, int i0, int i1, int e)
{
    int lo = i0, hi = i1 - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (__ldg(row_ptr + mid) <= e) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ float feat(int t, const float *__restrict__ X, const float *__restrict__ emb,
                                      const int32_t *__restrict__ types, int64_t N, int j, int f, int F)
{
    // x^0 is the embedding of the type; x^t (t >= 1) lives in X[t-1]
    if (t == 0) return __ldg(emb + (int64_t)__ldg(types + j) * F + f);
    return __ldg(X + ((int64_t)(t - 1) * N + j) * F + f);
}

struct EdgeArgs {
    const float4 *pos4;
    const int32_t *types, *row_ptr, *col, *part;
    const int32_t *dst;    // destination row of each edge (tensor-core kernels only)
    const float *emb;
    const float *X;        // [T][N][F]
    float *H;              // [N][F] (fwd out)
    const float *Hbar;     // [N][F] (bwd in)
    float *Xbar;           // [N][F] (bwd in/out)
    float *forces;         // [N][3] (bwd in/out)
    int64_t N;
    Geometry geo;
    Basis basis;
    BlockW w;
    int t;
    const int *d_err;
};

template <int F, int KP>
struct EdgeSmem {
    static constexpr int W1 = F * (KP + 1);
    static constexpr int W2 = F * (F + 1);
    static constexpr int BT = KP * TS;
    static constexpr int FT = F * TS;
    static constexpr int META = 10 * NE;   // d (double), src, dst, u[3], force[3] per edge
    static constexpr int fwd_floats = W1 + W2 + BT + FT + META;
    static constexpr int bwd_floats = W1 + W2 + 2 * BT + 2 * FT + META;
};

// Gaussian basis times envelope (and optionally its derivative) into [k][n] tiles.
template <int F, int KP, bool DERIV>
__device__ __forceinline__ void radial_tile(const Basis &bs, const double *sDistD, int ne, float *sBt, float *sDbt)
{
    const float inv_rc = 1.0f / bs.r_cut;
    for (int q = threadIdx.x; q < KP * NE; q += F) {
        const int k = q / NE, n = q % NE;
        float v = 0.0f, dv = 0.0f;
        if (n < ne && k < bs.K) {
            const double dd = sDistD[n];
            const float x = (float)(dd - bs.mu[k]);
            const float ratio = (float)(dd / bs.r_cut_d);
            const float phi = expf(-bs.gamma * x * x);
            const float C = 0.5f * (cospif(ratio) + 1.0f);
            v = phi * C;
            if (DERIV) {
                const float dC = -0.5f * (float)M_PI * inv_rc * sinpif(ratio);
                dv = -2.0f * bs.gamma * x * phi * C + phi * dC;
            }
        }
        sBt[k * TS + n] = v;
        if (DERIV) sDbt[k * TS + n] = dv;
    }
}

// acc[n] = sum_k M[row][k] * T[k][n] for n < NE, M row stride ld, T tile stride TS
template <int KD>
__device__ __forceinline__ void row_times_tile(const float *__restrict__ Mrow, int step, const float *__restrict__ T,
                                               float acc[NE])
{
#pragma unroll
    for (int n = 0; n < NE; ++n) acc[n] = 0.0f;
#pragma unroll 4
    for (int k = 0; k < KD; ++k) {
        const float wv = Mrow[k * step];
        const float4 *t4 = reinterpret_cast<const float4 *>(T + k * TS);
#pragma unroll
        for (int q = 0; q < NE / 4; ++q) {
            const float4 b = t4[q];
            acc[4 * q + 0] = fmaf(wv, b.x, acc[4 * q + 0]);
            acc[4 * q + 1] = fmaf(wv, b.y, acc[4 * q + 1]);
            acc[4 * q + 2] = fmaf(wv, b.z, acc[4 * q + 2]);
            acc[4 * q + 3] = fmaf(wv, b.w, acc[4 * q + 3]);
        }
    }
}

__device__ __forceinline__ void store_row(float *row, const float v[NE])
{
    float4 *r4 = reinterpret_cast<float4 *>(row);
#pragma unroll
    for (int q = 0; q < NE / 4; ++q) r4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// Per-tile edge metadata: source, owner row, pair vector and length.
template <int F>
__device__ __forceinline__ void edge_meta(const EdgeArgs &A, int i0, int i1, int ts, int ne, int *sSrc, int *sDst,
                                          double *sDistD, float *sU)
{
    const int n = threadIdx.x;
    if (n < NE) {
        if (n < ne) {
            const int e = ts + n;
            const int j = __ldg(A.col + e);
            const int i = edge_row(A.row_ptr, i0, i1, e);
            double3 u;
            const double d = pair_vec(A.pos4[i], A.pos4[j], A.geo, u);
            sSrc[n] = j;
            sDst[n] = i;
            sDistD[n] = d;
            if (sU) {
                // unit vector u/d (force direction)
                sU[3 * n] = (float)(u.x / d);
                sU[3 * n + 1] = (float)(u.y / d);
                sU[3 * n + 2] = (float)(u.z / d);
            }
        } else {
            sSrc[n] = -1;
            sDst[n] = -1;
            sDistD[n] = 0.0;
        }
    }
}

template <int F, int KP>
__global__ void __launch_bounds__(F) k_edge_fwd(EdgeArgs A)
{
    using S = EdgeSmem<F, KP>;
    extern __shared__ float4 smem4[];
    float *sW1 = reinterpret_cast<float *>(smem4);
    float *sW2 = sW1 + S::W1;
    float *sBt = sW2 + S::W2;
    float *sS = sBt + S::BT;
    double *sDist = reinterpret_cast<double *>(sS + S::FT);     // [NE], 8-byte aligned
    int *sSrc = reinterpret_cast<int *>(sDist + NE);
    int *sDst = sSrc + NE;
    __shared__ int skip;

    const int f = threadIdx.x;
    if (f == 0) skip = (*((volatile const int *)A.d_err) & (ERRBIT_NONFINITE | ERRBIT_CAPACITY | ERRBIT_TIMEOUT)) != 0;
    copy_f4(sW1, A.w.W1, S::W1, f, F);
    copy_f4(sW2, A.w.W2, S::W2, f, F);
    const float b1f = A.w.b1[f], b2f = A.w.b2[f];
    __syncthreads();
    if (skip) return;

    const int i0 = A.part[blockIdx.x], i1 = A.part[blockIdx.x + 1];
    if (i0 >= i1) return;
    const int e0 = A.row_ptr[i0], e1 = A.row_ptr[i1];
    int cur = i0;
    float hacc = 0.0f;
    float acc[NE], xv[NE];

    for (int ts = e0; ts < e1; ts += NE) {
        const int ne = min(NE, e1 - ts);
        __syncthreads();
        edge_meta<F>(A, i0, i1, ts, ne, sSrc, sDst, sDist, nullptr);
        __syncthreads();
        radial_tile<F, KP, false>(A.basis, sDist, ne, sBt, nullptr);
        __syncthreads();
        // a = W1 bt + b1 ; s = ssp(a)
        row_times_tile<KP>(sW1 + f * (KP + 1), 1, sBt, acc);
#pragma unroll
        for (int n = 0; n < NE; ++n) acc[n] = ssp(acc[n] + b1f);
        store_row(sS + f * TS, acc);
        __syncthreads();
        // w = W2 s + b2
        row_times_tile<F>(sW2 + f * (F + 1), 1, sS, acc);
        // gather x_src and reduce per destination row
#pragma unroll
        for (int n = 0; n < NE; ++n) xv[n] = (n < ne) ? feat(A.t, A.X, A.emb, A.types, A.N, sSrc[n], f, F) : 0.0f;
#pragma unroll
        for (int n = 0; n < NE; ++n) {
            if (n < ne) {
                const int i = sDst[n];
                if (i != cur) {
                    A.H[(int64_t)cur * F + f] = hacc;
                    for (int r = cur + 1; r < i; ++r) A.H[(int64_t)r * F + f] = 0.0f;
                    hacc = 0.0f;
                    cur = i;
                }
                hacc = fmaf(xv[n], acc[n] + b2f, hacc);
            }
        }
    }
    A.H[(int64_t)cur * F + f] = hacc;
    for (int r = cur + 1; r < i1; ++r) A.H[(int64_t)r * F + f] = 0.0f;
}

template <int F, int KP>
__global__ void __launch_bounds__(F) k_edge_bwd(EdgeArgs A)
{
    using S = EdgeSmem<F, KP>;
    extern __shared__ float4 smem4[];
    float *sW1 = reinterpret_cast<float *>(smem4);
    float *sW2 = sW1 + S::W1;
    float *sBt = sW2 + S::W2;
    float *sDbt = sBt + S::BT;
    float *sS = sDbt + S::BT;       // s, later abar
    float *sWb = sS + S::FT;        // wbar
    double *sDist = reinterpret_cast<double *>(sWb + S::FT);   // [NE], 8-byte aligned
    int *sSrc = reinterpret_cast<int *>(sDist + NE);
    int *sDst = sSrc + NE;
    float *sU = reinterpret_cast<float *>(sDst + NE);          // [NE][3] unit vectors
    float *sFv = sU + 3 * NE;                                  // [NE][3]
    __shared__ int skip;

    const int f = threadIdx.x;
    if (f == 0) skip = (*((volatile const int *)A.d_err) & (ERRBIT_NONFINITE | ERRBIT_CAPACITY | ERRBIT_TIMEOUT)) != 0;
    copy_f4(sW1, A.w.W1, S::W1, f, F);
    copy_f4(sW2, A.w.W2, S::W2, f, F);
    const float b1f = A.w.b1[f], b2f = A.w.b2[f];
    __syncthreads();
    if (skip) return;

    const int i0 = A.part[blockIdx.x], i1 = A.part[blockIdx.x + 1];
    if (i0 >= i1) return;
    const int e0 = A.row_ptr[i0], e1 = A.row_ptr[i1];
    int cur = -1;
    float xbacc = 0.0f, hbi = 0.0f, xi = 0.0f;
    float a[NE], w[NE], hb[NE], xj[NE];

    for (int ts = e0; ts < e1; ts += NE) {
        const int ne = min(NE, e1 - ts);
        __syncthreads();
        edge_meta<F>(A, i0, i1, ts, ne, sSrc, sDst, sDist, sU);
        __syncthreads();
        radial_tile<F, KP, true>(A.basis, sDist, ne, sBt, sDbt);
        __syncthreads();
        row_times_tile<KP>(sW1 + f * (KP + 1), 1, sBt, a);
#pragma unroll
        for (int n = 0; n < NE; ++n) {
            a[n] += b1f;
            w[n] = ssp(a[n]);
        }
        store_row(sS + f * TS, w);
        __syncthreads();
        row_times_tile<F>(sW2 + f * (F + 1), 1, sS, w);
#pragma unroll
        for (int n = 0; n < NE; ++n) {
            w[n] += b2f;
            if (n < ne) {
                const int j = sSrc[n];
                hb[n] = __ldg(A.Hbar + (int64_t)j * F + f);
                xj[n] = feat(A.t, A.X, A.emb, A.types, A.N, j, f, F);
            } else {
                hb[n] = 0.0f;
                xj[n] = 0.0f;
            }
        }
        // xbar_i += sum_j hbar_j (.) w_ij ;  wbar = x_j (.) hbar_i + x_i (.) hbar_j
#pragma unroll
        for (int n = 0; n < NE; ++n) {
            float wb = 0.0f;
            if (n < ne) {
                const int i = sDst[n];
                if (i != cur) {
                    if (cur >= 0) A.Xbar[(int64_t)cur * F + f] += xbacc;
                    xbacc = 0.0f;
                    cur = i;
                    hbi = __ldg(A.Hbar + (int64_t)i * F + f);
                    xi = feat(A.t, A.X, A.emb, A.types, A.N, i, f, F);
                }
                xbacc = fmaf(hb[n], w[n], xbacc);
                wb = xj[n] * hbi + xi * hb[n];
            }
            xj[n] = wb;
        }
        store_row(sWb + f * TS, xj);
        __syncthreads();
        // sbar = W2^T wbar ; abar = sbar (.) sigma(a)
        row_times_tile<F>(sW2 + f, F + 1, sWb, w);
#pragma unroll
        for (int n = 0; n < NE; ++n) w[n] *= sigmoid(a[n]);
        store_row(sS + f * TS, w);
        __syncthreads();
        // btbar = W1^T abar ; per-(k, edge) products with d(bt)/dd
        if (f < KP) {
            row_times_tile<F>(sW1 + f, KP + 1, sS, w);
            const float4 *d4 = reinterpret_cast<const float4 *>(sDbt + f * TS);
            float4 *o4 = reinterpret_cast<float4 *>(sBt + f * TS);
#pragma unroll
            for (int q = 0; q < NE / 4; ++q) {
                const float4 dd = d4[q];
                o4[q] = make_float4(w[4 * q] * dd.x, w[4 * q + 1] * dd.y, w[4 * q + 2] * dd.z, w[4 * q + 3] * dd.w);
            }
        }
        __syncthreads();
        if (f < NE) {
            float fx = 0.0f, fy = 0.0f, fz = 0.0f;
            if (f < ne) {
                float db = 0.0f;
                for (int k = 0; k < KP; ++k) db += sBt[k * TS + f];
                fx = -db * sU[3 * f];
                fy = -db * sU[3 * f + 1];
                fz = -db * sU[3 * f + 2];
            }
            sFv[3 * f] = fx;
            sFv[3 * f + 1] = fy;
            sFv[3 * f + 2] = fz;
        }
        __syncthreads();
        if (f < 3) {
            int row = sDst[0];
            float acc = 0.0f;
            for (int n = 0; n < ne; ++n) {
                if (sDst[n] != row) {
                    A.forces[(int64_t)row * 3 + f] += acc;
                    acc = 0.0f;
                    row = sDst[n];
                }
                acc += sFv[3 * n + f];
            }
            A.forces[(int64_t)row * 3 + f] += acc;
        }
    }
    if (cur >= 0) A.Xbar[(int64_t)cur * F + f] += xbacc;
}

// ------------------------------------------------------------------------------- node kernels
struct NodeArgs {
    const int32_t *types;
    const float *emb;
    float *X;          // [T][N][F]
    float *P;          // [T][N][F]
    const float *H;    // [N][F]
    float *Hbar;       // [N][F]
    float *Xbar;       // [N][F]
    float *eps;        // [N]
    float *forces;     // [N][3]
    int64_t N;
    BlockW w;          // block t (forward) / block t-1 (backward)
    ReadoutW ro;
    int t;
    const int *d_err;
};

template <int F>
struct NodeSmem {
    static constexpr int U = F * (F + 1);
    static constexpr int R = (F / 2) * (F + 1);
    static constexpr int FT = F * TS;
    static constexpr int fwd_floats = 2 * U + 2 * FT;
    static constexpr int last_floats = 2 * U + R + 2 * FT;
    static constexpr int bwd_floats = 2 * U + 2 * FT;
};

// hbar = U1^T (sigma(p) (.) U2^T xbar) for a tile whose xbar sits in sXb[f][n]; p[n] is this
// thread's feature of U1 h + c1.  Uses sTmp as scratch.  Writes Hbar rows a0 .. a0+na-1.
template <int F>
__device__ __forceinline__ void node_backward_tile(const float *sU1, const float *sU2, const float *sXb, float *sTmp,
                                                   const float p[NA], float *Hbar, int64_t a0, int na)
{
    const int g = threadIdx.x;
    float v[NA];
    row_times_tile<F>(sU2 + g, F + 1, sXb, v);        // qbar_g = sum_f U2[f][g] xbar_f
#pragma unroll
    for (int n = 0; n < NA; ++n) v[n] *= sigmoid(p[n]);
    store_row(sTmp + g * TS, v);
    __syncthreads();
    row_times_tile<F>(sU1 + g, F + 1, sTmp, v);       // hbar_g = sum_f U1[f][g] pbar_f
#pragma unroll
    for (int n = 0; n < NA; ++n)
        if (n < na) Hbar[(a0 + n) * F + g] = v[n];
}

template <int F, bool LAST>
__global__ void __launch_bounds__(F) k_node_fwd(NodeArgs A)
{
    using S = NodeSmem<F>;
    constexpr int H = F / 2;
    extern __shared__ float4 smem4[];
    float *sU1 = reinterpret_cast<float *>(smem4);
    float *sU2 = sU1 + S::U;
    float *sA = sU2 + S::U;          // h tile, later x tile, later xbar tile
    float *sB = sA + S::FT;          // q tile, later readout products, later pbar tile
    float *sR1 = sB + S::FT;         // [H][F+1] (LAST only)
    __shared__ int skip;

    const int f = threadIdx.x;
    if (f == 0) skip = (*((volatile const int *)A.d_err) & (ERRBIT_NONFINITE | ERRBIT_CAPACITY | ERRBIT_TIMEOUT)) != 0;
    copy_f4(sU1, A.w.U1, S::U, f, F);
    copy_f4(sU2, A.w.U2, S::U, f, F);
    if (LAST) copy_f4(sR1, A.ro.R1, S::R, f, F);
    const float c1f = A.w.c1[f], c2f = A.w.c2[f];
    __syncthreads();
    if (skip) return;

    const int64_t n_tiles = (A.N + NA - 1) / NA;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int64_t a0 = tile * NA;
        const int na = (int)(A.N - a0 < NA ? A.N - a0 : NA);
        float p[NA], v[NA];
        __syncthreads();
#pragma unroll
        for (int n = 0; n < NA; ++n) sA[f * TS + n] = (n < na) ? A.H[(a0 + n) * F + f] : 0.0f;
        __syncthreads();
        // sA holds h transposed as [f][n]; p_f = sum_g U1[f][g] h_g + c1_f
        row_times_tile<F>(sU1 + f * (F + 1), 1, sA, p);
#pragma unroll
        for (int n = 0; n < NA; ++n) {
            p[n] += c1f;
            if (n < na) A.P[((int64_t)A.t * A.N + a0 + n) * F + f] = p[n];
            v[n] = ssp(p[n]);
        }
        store_row(sB + f * TS, v);
        __syncthreads();
        row_times_tile<F>(sU2 + f * (F + 1), 1, sB, v);
#pragma unroll
        for (int n = 0; n < NA; ++n) {
            if (n < na) {
                const float xo = feat(A.t, A.X, A.emb, A.types, A.N, (int)(a0 + n), f, F);
                v[n] = xo + v[n] + c2f;
                A.X[((int64_t)A.t * A.N + a0 + n) * F + f] = v[n];
            } else {
                v[n] = 0.0f;
            }
        }
        if (!LAST) continue;
        // readout: o = R1 x + e1, eps = R2 . ssp(o) + e2, obar = R2 (.) sigma(o), xbar = R1^T obar
        __syncthreads();
        store_row(sA + f * TS, v);          // x^T as [f][n]
        __syncthreads();
        if (f < H) {
            float o[NA];
            row_times_tile<F>(sR1 + f * (F + 1), 1, sA, o);
            const float e1k = A.ro.e1[f], r2k = A.ro.R2[f];
#pragma unroll
            for (int n = 0; n < NA; ++n) {
                o[n] += e1k;
                sB[f * TS + n] = r2k * ssp(o[n]);
                sB[(H + f) * TS + n] = r2k * sigmoid(o[n]);
            }
        }
        __syncthreads();
        if (f < NA && f < na) {
            float e = A.ro.e2[0];
            for (int k = 0; k < H; ++k) e += sB[k * TS + f];
            A.eps[a0 + f] = e;
            A.forces[(a0 + f) * 3 + 0] = 0.0f;
            A.forces[(a0 + f) * 3 + 1] = 0.0f;
            A.forces[(a0 + f) * 3 + 2] = 0.0f;
        }
        row_times_tile<H>(sR1 + f, F + 1, sB + H * TS, v);   // xbar_f = sum_k R1[k][f] obar_k
#pragma unroll
        for (int n = 0; n < NA; ++n)
            if (n < na) A.Xbar[(a0 + n) * F + f] = v[n];
        __syncthreads();
        store_row(sA + f * TS, v);
        __syncthreads();
        node_backward_tile<F>(sU1, sU2, sA, sB, p, A.Hbar, a0, na);
    }
}

template <int F>
__global__ void __launch_bounds__(F) k_node_bwd(NodeArgs A)
{
    using S = NodeSmem<F>;
    extern __shared__ float4 smem4[];
    float *sU1 = reinterpret_cast<float *>(smem4);
    float *sU2 = sU1 + S::U;
    float *sA = sU2 + S::U;
    float *sB = sA + S::FT;
    __shared__ int skip;

    const int f = threadIdx.x;
    if (f == 0) skip = (*((volatile const int *)A.d_err) & (ERRBIT_NONFINITE | ERRBIT_CAPACITY | ERRBIT_TIMEOUT)) != 0;
    copy_f4(sU1, A.w.U1, S::U, f, F);
    copy_f4(sU2, A.w.U2, S::U, f, F);
    __syncthreads();
    if (skip) return;

    const int64_t n_tiles = (A.N + NA - 1) / NA;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int64_t a0 = tile * NA;
        const int na = (int)(A.N - a0 < NA ? A.N - a0 : NA);
        float p[NA];
        __syncthreads();
#pragma unroll
        for (int n = 0; n < NA; ++n) {
            sA[f * TS + n] = (n < na) ? A.Xbar[(a0 + n) * F + f] : 0.0f;
            p[n] = (n < na) ? A.P[((int64_t)A.t * A.N + a0 + n) * F + f] : 0.0f;
        }
        __syncthreads();
        node_backward_tile<F>(sU1, sU2, sA, sB, p, A.Hbar, a0, na);
    }
}

// Also checks that the list fits the caller's col buffer (cap entries): a row_ptr that points
// past it latches the capacity condition, and every later kernel skips.
__global__ void k_partition(const int32_t *__restrict__ row_ptr, int64_t N, int G, int32_t *__restrict__ part,
                            int64_t cap, int *__restrict__ d_err)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c == 0 && (row_ptr[0] < 0 || (int64_t)row_ptr[N] > cap)) atomicOr(d_err, ERRBIT_CAPACITY);
    if (c > G) return;
    const int64_t total = (int64_t)row_ptr[N] + N;
    const int64_t target = (total * c + G - 1) / G;
    int64_t lo = 0, hi = N;
    while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        if ((int64_t)row_ptr[mid] + mid >= target) hi = mid;
        else lo = mid + 1;
    }
    part[c] = (int32_t)lo;
}

// Row partition (as k_partition) in the first part_blocks blocks; in the others, one warp per
// row writes dst[e] = i for every edge e of row i (the tensor-core kernels read an edge's row
// directly); an edge index outside the buffer latches the capacity condition instead.
__global__ void k_partition_rows(const int32_t *__restrict__ row_ptr, int64_t N, int G, int32_t *__restrict__ part,
                                 unsigned part_blocks, int32_t *__restrict__ dst, int64_t cap, int *__restrict__ d_err)
{
    pdl_trigger();
    pdl_wait();
    if (blockIdx.x < part_blocks) {
        const int c = blockIdx.x * blockDim.x + threadIdx.x;
        if (c > G) return;
        const int64_t total = (int64_t)row_ptr[N] + N;
        const int64_t target = (total * c + G - 1) / G;
        int64_t lo = 0, hi = N;
        while (lo < hi) {
            const int64_t mid = (lo + hi) >> 1;
            if ((int64_t)row_ptr[mid] + mid >= target) hi = mid;
            else lo = mid + 1;
        }
        part[c] = (int32_t)lo;
        return;
    }
    const int64_t i = ((blockIdx.x - part_blocks) * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (i >= N) return;
    const int32_t e0 = row_ptr[i], e1 = row_ptr[i + 1];
    if (e0 < 0 || e1 > cap) {
        if (lane == 0) atomicOr(d_err, ERRBIT_CAPACITY);
        return;
    }
    for (int32_t e = e0 + lane; e < e1; e += 32) dst[e] = (int32_t)i;
}

EdgeTcArgs tc_args(const EdgeArgs &a, const BlockW &bw, int n_types, int *d_err, long long wait_limit)
{
    EdgeTcArgs t{};
    t.n_types = n_types;
    t.wait_limit = wait_limit;
    t.pos4 = a.pos4;
    t.types = a.types;
    t.row_ptr = a.row_ptr;
    t.col = a.col;
    t.part = a.part;
    t.dst = a.dst;
    t.emb = a.emb;
    t.X = a.X;
    t.H = a.H;
    t.Hbar = a.Hbar;
    t.Xbar = a.Xbar;
    t.forces = a.forces;
    t.N = a.N;
    t.geo = a.geo;
    t.basis = a.basis;
    t.W1h = bw.W1h;
    t.W1l = bw.W1l;
    t.W2h = bw.W2h;
    t.W2l = bw.W2l;
    t.b1 = bw.b1;
    t.b2 = bw.b2;
    t.s1 = bw.s1;
    t.s2 = bw.s2;
    t.t = a.t;
    t.d_err = d_err;
    return t;
}

template <typename Kern>
cudaError_t set_smem(Kern k, int bytes)
{
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int F, int KP>
cudaError_t run(const Model &m, const sn_system &sys, const Geometry &geo, const int32_t *types,
                const int32_t *row_ptr, const int32_t *col, EfWork &w, float *forces, int *d_err,
                cudaStream_t s, int n_sm, Tracer *tr)
{
    using ES = EdgeSmem<F, KP>;
    using NS = NodeSmem<F>;
    const int64_t N = (int64_t)sys.n_per_replica * sys.n_replicas;
    const int fwd_bytes = ES::fwd_floats * 4, bwd_bytes = ES::bwd_floats * 4;
    const int nf_bytes = NS::fwd_floats * 4, nl_bytes = NS::last_floats * 4, nb_bytes = NS::bwd_floats * 4;
    cudaError_t e;
    if ((e = set_smem(k_edge_fwd<F, KP>, fwd_bytes))) return e;
    if ((e = set_smem(k_edge_bwd<F, KP>, bwd_bytes))) return e;
    if ((e = set_smem(k_node_fwd<F, false>, nf_bytes))) return e;
    if ((e = set_smem(k_node_fwd<F, true>, nl_bytes))) return e;
    if ((e = set_smem(k_node_bwd<F>, nb_bytes))) return e;

    trace_begin(tr, KK_PARTITION, s);
    const int parts = m.precision == SN_PREC_FP32 ? w.G : w.G * tc_groups_per_cta(m.precision == SN_PREC_TC32);
    if (m.precision != SN_PREC_FP32 && N > 0) {
        // one launch: the first blocks partition the rows, the rest index the edges' rows
        const unsigned pb = (unsigned)((parts + 1 + 255) / 256);
        if ((e = launch_pdl(k_partition_rows, dim3(pb + (unsigned)((32 * N + 255) / 256)), dim3(256), 0, s, row_ptr, N,
                            parts, w.part, pb, w.dst, w.col_cap < w.dst_cap ? w.col_cap : w.dst_cap, d_err)))
            return e;
    } else {
        k_partition<<<(parts + 1 + 127) / 128, 128, 0, s>>>(row_ptr, N, parts, w.part, w.col_cap, d_err);
    }
    trace_end(tr, s);

    EdgeArgs ea{};
    ea.pos4 = w.pos4;
    ea.types = types;
    ea.row_ptr = row_ptr;
    ea.col = col;
    ea.part = w.part;
    ea.dst = w.dst;
    ea.emb = m.emb;
    ea.X = w.x;
    ea.H = w.h;
    ea.Hbar = w.hbar;
    ea.Xbar = w.xbar;
    ea.forces = forces;
    ea.N = N;
    ea.geo = geo;
    ea.basis = m.basis;
    ea.d_err = d_err;

    NodeArgs na{};
    na.types = types;
    na.emb = m.emb;
    na.X = w.x;
    na.P = w.p;
    na.H = w.h;
    na.Hbar = w.hbar;
    na.Xbar = w.xbar;
    na.eps = w.eps;
    na.forces = forces;
    na.N = N;
    na.ro = m.ro;
    na.d_err = d_err;

    const int64_t n_tiles = (N + NA - 1) / NA;
    const unsigned node_grid = (unsigned)(n_tiles < n_sm ? (n_tiles < 1 ? 1 : n_tiles) : n_sm);

    if (m.precision != SN_PREC_FP32) {
        // tensor-core precisions: edge and node networks on tcgen05
        const bool split = m.precision == SN_PREC_TC32;
        NodeTcArgs nt{};
        nt.types = types;
        nt.emb = m.emb;
        nt.X = w.x;
        nt.P = w.p;
        nt.H = w.h;
        nt.Hbar = w.hbar;
        nt.Xbar = w.xbar;
        nt.eps = w.eps;
        nt.forces = forces;
        nt.N = N;
        nt.R1h = m.ro.R1h;
        nt.R1l = m.ro.R1l;
        nt.e1 = m.ro.e1;
        nt.R2 = m.ro.R2;
        nt.e2 = m.ro.e2;
        nt.sr1 = m.ro.sr1;
        nt.d_err = d_err;
        nt.wait_limit = w.wait_limit;
        auto node_args = [&](int t) {
            NodeTcArgs a = nt;
            a.t = t;
            a.U1h = m.blk[t].U1h;
            a.U1l = m.blk[t].U1l;
            a.U2h = m.blk[t].U2h;
            a.U2l = m.blk[t].U2l;
            a.c1 = m.blk[t].c1;
            a.c2 = m.blk[t].c2;
            a.su1 = m.blk[t].su1;
            a.su2 = m.blk[t].su2;
            return a;
        };
        for (int t = 0; t < m.T; ++t) {
            ea.w = m.blk[t];
            ea.t = t;
            trace_begin(tr, KK_EDGE_FWD, s);
            if ((e = launch_edge_tc(tc_args(ea, m.blk[t], m.n_types, d_err, w.wait_limit), KP, split, false, w.G, s))) return e;
            trace_end(tr, s);
            trace_begin(tr, KK_NODE_FWD, s);
            if ((e = launch_node_tc(node_args(t), split, 0, n_sm, s))) return e;
            trace_end(tr, s);
        }
        trace_begin(tr, KK_NODE_FWD, s);
        if ((e = launch_node_tc(node_args(m.T - 1), split, 1, n_sm, s))) return e;   // readout of x^T
        trace_end(tr, s);
        for (int t = m.T - 1; t >= 0; --t) {
            trace_begin(tr, KK_NODE_BWD, s);
            if ((e = launch_node_tc(node_args(t), split, 2, n_sm, s))) return e;     // hbar^t
            trace_end(tr, s);
            ea.w = m.blk[t];
            ea.t = t;
            trace_begin(tr, KK_EDGE_BWD, s);
            if ((e = launch_edge_tc(tc_args(ea, m.blk[t], m.n_types, d_err, w.wait_limit), KP, split, true, w.G, s))) return e;
            trace_end(tr, s);
        }
        return cudaGetLastError();
    }
    for (int t = 0; t < m.T; ++t) {
        ea.w = m.blk[t];
        ea.t = t;
        trace_begin(tr, KK_EDGE_FWD, s);
        k_edge_fwd<F, KP><<<w.G, F, fwd_bytes, s>>>(ea);
        trace_end(tr, s);
        na.w = m.blk[t];
        na.t = t;
        trace_begin(tr, KK_NODE_FWD, s);
        if (t == m.T - 1) k_node_fwd<F, true><<<node_grid, F, nl_bytes, s>>>(na);
        else k_node_fwd<F, false><<<node_grid, F, nf_bytes, s>>>(na);
        trace_end(tr, s);
    }
    for (int t = m.T - 1; t >= 0; --t) {
        ea.w = m.blk[t];
        ea.t = t;
        trace_begin(tr, KK_EDGE_BWD, s);
        k_edge_bwd<F, KP><<<w.G, F, bwd_bytes, s>>>(ea);
        trace_end(tr, s);
        if (t > 0) {
            na.w = m.blk[t - 1];
            na.t = t - 1;
            trace_begin(tr, KK_NODE_BWD, s);
            k_node_bwd<F><<<node_grid, F, nb_bytes, s>>>(na);
            trace_end(tr, s);
        }
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_energy_forces(const Model &m, const sn_system &sys, const Geometry &geo,
                                 const int32_t *types, const int32_t *row_ptr,
                                 const int32_t *col, EfWork &w, float *energy, float *forces,
                                 int *d_err, cudaStream_t s, Tracer *tr)
{
    (void)energy;
    int dev = 0, n_sm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    const int64_t N = (int64_t)sys.n_per_replica * sys.n_replicas;
    if (N == 0) return cudaSuccess;
    if (m.F == 128 && m.KP == 64) return run<128, 64>(m, sys, geo, types, row_ptr, col, w, forces, d_err, s, n_sm, tr);
    if (m.F == 128 && m.KP == 32) return run<128, 32>(m, sys, geo, types, row_ptr, col, w, forces, d_err, s, n_sm, tr);
    if (m.F == 64 && m.KP == 64) return run<64, 64>(m, sys, geo, types, row_ptr, col, w, forces, d_err, s, n_sm, tr);
    if (m.F == 64 && m.KP == 32) return run<64, 32>(m, sys, geo, types, row_ptr, col, w, forces, d_err, s, n_sm, tr);
    return cudaErrorInvalidValue;
}

}  // namespace sn
