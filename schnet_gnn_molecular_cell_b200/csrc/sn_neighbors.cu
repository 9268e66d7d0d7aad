// Neighbour list on the GPU (FlashSchNet §3.2 "Building the neighbor list"; §4.3 "Index
// construction under dynamic neighbor lists"): destination-grouped CSR with sources
// ascending in each row.
//
// Membership test, float32 with every operation rounded on its own (no FMA contraction), so
// that the list is reproducible bit for bit by any IEEE fp32 implementation:
//   dx = x_j - x_i;  periodic axis: dx = dx - L * rint(dx / L)
//   r2 = (dx*dx + dy*dy) + dz*dz;  edge iff r2 < r_cut*r_cut, i != j, same replica.
//
// Two builders:
//   * open boundaries (or a box too small for a 3x3x3 cell stencil): all pairs of a replica,
//     positions staged through shared memory in tiles of 512; sources come out ascending;
//   * periodic boxes with >= 3 cells per axis: cell list (cell side >= r_cut * 1.0001), then
//     each row is sorted by source.  Atoms are binned by their coordinates wrapped into the
//     box in double precision.  The fp32 test on raw coordinates can accept a pair whose
//     exact separation exceeds r_cut by its rounding error, which grows with |x|; while every
//     |coordinate| stays below a bound derived from the cell margin (side - r_cut) that error
//     is smaller than the margin and the 27-cell stencil holds every accepted pair.  An atom
//     beyond the bound raises a flag in the cell workspace and both passes then test all
//     pairs of each replica instead (same list, slower).
// Both run a count pass, an exclusive scan into row_ptr, and a fill pass.
#include <cuda_runtime.h>
#include <math.h>

#include "sn_internal.cuh"

namespace sn {

namespace {

constexpr int BT = 128;   // threads per CTA of the cell-list kernels

__device__ __forceinline__ float min_image_axis(float dx, float L)
{
    float q = rintf(__fdiv_rn(dx, L));
    return __fsub_rn(dx, __fmul_rn(L, q));
}

// returns r2 of the fp32 test (see file header)
__device__ __forceinline__ float pair_r2(float4 pi, float4 pj, const Geometry &g)
{
    float dx = __fsub_rn(pj.x, pi.x);
    float dy = __fsub_rn(pj.y, pi.y);
    float dz = __fsub_rn(pj.z, pi.z);
    if (g.periodic[0]) dx = min_image_axis(dx, g.box[0]);
    if (g.periodic[1]) dy = min_image_axis(dy, g.box[1]);
    if (g.periodic[2]) dz = min_image_axis(dz, g.box[2]);
    float r2 = __fmul_rn(dx, dx);
    r2 = __fadd_rn(r2, __fmul_rn(dy, dy));
    r2 = __fadd_rn(r2, __fmul_rn(dz, dz));
    return r2;
}

__global__ void k_prep_positions(const float *__restrict__ pos, float4 *__restrict__ pos4, int64_t N,
                                 int *__restrict__ d_err)
{
    pdl_trigger();
    pdl_wait();
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= N) return;
    float x = pos[3 * i], y = pos[3 * i + 1], z = pos[3 * i + 2];
    if (!isfinite(x) || !isfinite(y) || !isfinite(z)) {
        atomicOr(d_err, ERRBIT_NONFINITE);
        x = y = z = 0.0f;
    }
    pos4[i] = make_float4(x, y, z, 0.0f);
}

// -------------------------------------------------------------------- all pairs per replica
// CTA (b, r) of 8 warps: destination atoms 32 b + [0, 32) of replica r, 4 per warp.  The
// replica's positions pass through shared memory in tiles of PT; for each of its atoms a warp
// tests 32 sources per step (lane l: source j0 + l), a ballot gives the hits in ascending j,
// and FILL writes them at row_ptr[i] + (hits before it) while the count pass stores their
// number.  Decisions to stop are taken once per CTA (its threads meet at the tile barriers).
constexpr int PT = 512;            // positions per shared-memory tile
constexpr int PW = 4;              // destination atoms per warp
constexpr int PA = 8 * PW;         // destination atoms per CTA

template <bool FILL>
__global__ void __launch_bounds__(256) k_pairs(const float4 *__restrict__ pos4, int n_per, Geometry g, float rc2,
                                               int32_t *__restrict__ cnt, const int32_t *__restrict__ row_ptr,
                                               int32_t *__restrict__ col, int64_t cap, int64_t N,
                                               int *__restrict__ d_err)
{
    pdl_trigger();
    pdl_wait();
    __shared__ float4 sp[PT];
    __shared__ int s_stop;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t base = (int64_t)blockIdx.y * n_per;
    if (threadIdx.x == 0) {
        int stop = (*((volatile int *)d_err) & (ERRBIT_NONFINITE | ERRBIT_CAPACITY)) != 0;
        if (FILL && !stop && (int64_t)row_ptr[N] > cap) {
            atomicOr(d_err, ERRBIT_CAPACITY);
            stop = 1;
        }
        s_stop = stop;
    }
    __syncthreads();
    if (s_stop) return;
    const int il0 = blockIdx.x * PA + wid * PW;   // this warp's first atom (index in the replica)
    float4 pi[PW];
    int32_t w[PW];
#pragma unroll
    for (int a = 0; a < PW; ++a) {
        const bool valid = il0 + a < n_per;
        pi[a] = valid ? __ldg(pos4 + base + il0 + a) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        w[a] = FILL && valid ? row_ptr[base + il0 + a] : 0;
    }
    bool degenerate = false;
    for (int t0 = 0; t0 < n_per; t0 += PT) {
        const int tn = min(PT, n_per - t0);
        __syncthreads();   // the previous tile is read
        for (int q = threadIdx.x; q < tn; q += 256) sp[q] = __ldg(pos4 + base + t0 + q);
        __syncthreads();
#pragma unroll
        for (int a = 0; a < PW; ++a) {
            if (il0 + a >= n_per) continue;   // (warp-uniform)
            for (int j0 = 0; j0 < tn; j0 += 32) {
                const int jl = j0 + lane, j = t0 + jl;
                bool hit = false;
                if (jl < tn && j != il0 + a) {
                    const float r2 = pair_r2(pi[a], sp[jl], g);
                    hit = r2 < rc2;
                    degenerate |= hit && r2 == 0.0f;
                }
                const unsigned m = __ballot_sync(0xffffffffu, hit);
                if (FILL && hit) col[w[a] + __popc(m & ((1u << lane) - 1u))] = (int32_t)(base + j);
                w[a] += __popc(m);
            }
        }
    }
    if (!FILL && lane == 0) {
#pragma unroll
        for (int a = 0; a < PW; ++a)
            if (il0 + a < n_per) cnt[base + il0 + a] = w[a];
    }
    if (FILL && __any_sync(0xffffffffu, degenerate) && lane == 0) atomicOr(d_err, ERRBIT_DEGENERATE);
}

// -------------------------------------------------------------------- cell list (periodic)
struct CellGrid {
    int nc[3];
    double side[3];
    int64_t per_rep;
    int n_per;
    float x_safe;     // |coordinate| bound of the cell stencil (see file header)
    int32_t *flag;    // set when an atom exceeds x_safe (cleared with the cell counters)
};

// cell index along one axis of the coordinate wrapped into [0, L) in double (x is exact in
// double; the wrap and the division add ~1e-16 relative)
__device__ __forceinline__ int cell_coord(float x, float L, double side, int n)
{
    const double xd = (double)x, Ld = (double)L;
    const double w = xd - Ld * floor(xd / Ld);
    const int c = (int)floor(w / side);
    return c < 0 ? 0 : (c >= n ? n - 1 : c);
}

__global__ void k_cell_assign(const float4 *__restrict__ pos4, int64_t N, Geometry g, CellGrid cg,
                              int32_t *__restrict__ cell_of, int32_t *__restrict__ cell_cnt,
                              const int *__restrict__ d_err)
{
    pdl_trigger();
    pdl_wait();
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= N || (*((volatile const int *)d_err) & ERRBIT_NONFINITE)) return;
    float4 p = pos4[i];
    if (fmaxf(fabsf(p.x), fmaxf(fabsf(p.y), fabsf(p.z))) > cg.x_safe) *cg.flag = 1;
    int cx = cell_coord(p.x, g.box[0], cg.side[0], cg.nc[0]);
    int cy = cell_coord(p.y, g.box[1], cg.side[1], cg.nc[1]);
    int cz = cell_coord(p.z, g.box[2], cg.side[2], cg.nc[2]);
    int64_t c = (i / cg.n_per) * cg.per_rep + ((int64_t)cx * cg.nc[1] + cy) * cg.nc[2] + cz;
    cell_of[i] = (int32_t)c;
    atomicAdd(&cell_cnt[c], 1);
}

__global__ void k_cell_scatter(int64_t N, const int32_t *__restrict__ cell_of, int32_t *__restrict__ cursor,
                               int32_t *__restrict__ cell_atoms, const int *__restrict__ d_err)
{
    pdl_trigger();
    pdl_wait();
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= N || (*((volatile const int *)d_err) & ERRBIT_NONFINITE)) return;
    int32_t slot = atomicAdd(&cursor[cell_of[i]], 1);
    cell_atoms[slot] = (int32_t)i;
}

template <bool FILL>
__global__ void __launch_bounds__(BT) k_cell_pairs(const float4 *__restrict__ pos4, int64_t N, Geometry g,
                                                   CellGrid cg, float rc2, const int32_t *__restrict__ cell_of,
                                                   const int32_t *__restrict__ cell_start,
                                                   const int32_t *__restrict__ cell_atoms,
                                                   int32_t *__restrict__ cnt, const int32_t *__restrict__ row_ptr,
                                                   int32_t *__restrict__ col, int64_t cap, int *__restrict__ d_err)
{
    pdl_trigger();
    pdl_wait();
    if (*((volatile int *)d_err) & (ERRBIT_NONFINITE | ERRBIT_CAPACITY)) return;
    if (FILL && (int64_t)row_ptr[N] > cap) {
        if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(d_err, ERRBIT_CAPACITY);
        return;
    }
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= N) return;
    const float4 pi = pos4[i];
    const int64_t c = cell_of[i];
    const int64_t rep0 = (c / cg.per_rep) * cg.per_rep;
    const int64_t lc = c - rep0;
    const int cz = (int)(lc % cg.nc[2]);
    const int cy = (int)((lc / cg.nc[2]) % cg.nc[1]);
    const int cx = (int)(lc / ((int64_t)cg.nc[1] * cg.nc[2]));
    int32_t n = 0;
    const int32_t w0 = FILL ? row_ptr[i] : 0;
    bool degenerate = false;
    if (*((volatile const int32_t *)cg.flag)) {
        // a coordinate beyond the stencil's bound: every source of the replica, ascending
        const int64_t b0 = i / cg.n_per * cg.n_per;
        for (int64_t j = b0; j < b0 + cg.n_per; ++j) {
            if (j == i) continue;
            const float r2 = pair_r2(pi, pos4[j], g);
            if (r2 < rc2) {
                if (FILL) col[w0 + n] = (int32_t)j;
                ++n;
                degenerate |= (r2 == 0.0f);
            }
        }
        if (FILL && degenerate) atomicOr(d_err, ERRBIT_DEGENERATE);
        if (!FILL) cnt[i] = n;
        return;
    }
    for (int ox = -1; ox <= 1; ++ox)
        for (int oy = -1; oy <= 1; ++oy)
            for (int oz = -1; oz <= 1; ++oz) {
                int x = cx + ox, y = cy + oy, z = cz + oz;
                x += (x < 0) ? cg.nc[0] : (x >= cg.nc[0] ? -cg.nc[0] : 0);
                y += (y < 0) ? cg.nc[1] : (y >= cg.nc[1] ? -cg.nc[1] : 0);
                z += (z < 0) ? cg.nc[2] : (z >= cg.nc[2] ? -cg.nc[2] : 0);
                const int64_t cc = rep0 + ((int64_t)x * cg.nc[1] + y) * cg.nc[2] + z;
                for (int32_t q = cell_start[cc]; q < cell_start[cc + 1]; ++q) {
                    const int32_t j = cell_atoms[q];
                    if (j == i) continue;
                    float r2 = pair_r2(pi, pos4[j], g);
                    if (r2 < rc2) {
                        if (FILL) col[w0 + n] = j;
                        ++n;
                        degenerate |= (r2 == 0.0f);
                    }
                }
            }
    if (!FILL) {
        cnt[i] = n;
        return;
    }
    if (degenerate) atomicOr(d_err, ERRBIT_DEGENERATE);
    // insertion sort of the row by source index (rows hold tens of entries)
    int32_t *row = col + w0;
    for (int32_t a = 1; a < n; ++a) {
        int32_t v = row[a];
        int32_t b = a - 1;
        while (b >= 0 && row[b] > v) {
            row[b + 1] = row[b];
            --b;
        }
        row[b + 1] = v;
    }
}

// -------------------------------------------------------------------- exclusive scan
// out[0] = 0, out[q + 1] = in[0] + .. + in[q] (exclusive scan into n + 1 entries) over many
// CTAs, in two launches: k_scan_tiles scans each 4096-entry tile in its own CTA (4 consecutive
// entries per thread; tile-local sums into out, tile totals into tsum); k_scan_add adds the
// totals of the earlier tiles.  Sums beyond int32 latch the capacity condition (a list that
// large cannot be indexed by int32).
__device__ __forceinline__ long long block_scan_1024(long long s, long long &total, long long *warp_sums)
{
    const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
    long long x = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
        long long ws = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, ws, o);
            if (lane >= o) ws += y;
        }
        warp_sums[lane] = ws;
    }
    __syncthreads();
    total = warp_sums[31];
    return x - s + (wid > 0 ? warp_sums[wid - 1] : 0);   // exclusive prefix of s
}

__global__ void __launch_bounds__(1024) k_scan_tiles(const int32_t *__restrict__ in, int32_t *__restrict__ out,
                                                     int64_t n, int32_t *__restrict__ tsum)
{
    pdl_trigger();
    pdl_wait();
    __shared__ long long warp_sums[32];
    const int t = threadIdx.x;
    const int64_t q0 = (int64_t)blockIdx.x * 4096 + 4 * t;
    int v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = q0 + k < n ? in[q0 + k] : 0;
    long long total;
    long long run = block_scan_1024((long long)v[0] + v[1] + v[2] + v[3], total, warp_sums);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (q0 + k < n) {
            run += v[k];
            out[q0 + k + 1] = (int32_t)(run > 0x7fffffffLL ? 0x7fffffff : run);
        }
    if (t == 0) {
        tsum[blockIdx.x] = (int32_t)(total > 0x7fffffffLL ? 0x7fffffff : total);
        if (blockIdx.x == 0) out[0] = 0;
    }
}

__global__ void __launch_bounds__(1024) k_scan_add(int32_t *__restrict__ out, int64_t n,
                                                   const int32_t *__restrict__ tsum, int *__restrict__ d_err)
{
    pdl_trigger();
    pdl_wait();
    __shared__ long long part[32];
    const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
    long long off = 0;
    for (int b = t; b < (int)blockIdx.x; b += 1024) off += tsum[b];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) off += __shfl_xor_sync(0xffffffffu, off, o);
    if (lane == 0) part[wid] = off;
    __syncthreads();
    off = 0;
#pragma unroll 1
    for (int w = 0; w < 32; ++w) off += part[w];
    if (off == 0) return;
    const int64_t q0 = (int64_t)blockIdx.x * 4096 + 4 * t;
    bool over = false;
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (q0 + k < n) {
            const long long v = off + out[q0 + k + 1];
            over |= v > 0x7fffffffLL;
            out[q0 + k + 1] = (int32_t)(v > 0x7fffffffLL ? 0x7fffffff : v);
        }
    if (__any_sync(0xffffffffu, over) && lane == 0) atomicOr(d_err, ERRBIT_CAPACITY);
}

__global__ void k_copy_i32(const int32_t *__restrict__ a, int32_t *__restrict__ b, int64_t n)
{
    pdl_trigger();
    pdl_wait();
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i < n) b[i] = a[i];
}

// out[0] = 0, out[q + 1] = in[0] + .. + in[q] for q < n, over ceil(n / 4096) CTAs in two launches
cudaError_t scan(const int32_t *in, int32_t *out, int64_t n, int32_t *tsum, int *d_err, cudaStream_t s)
{
    const unsigned tiles = (unsigned)((n + 4095) / 4096);
    if (tiles == 0) return cudaMemsetAsync(out, 0, sizeof(int32_t), s);
    cudaError_t e = launch_pdl(k_scan_tiles, dim3(tiles), dim3(1024), 0, s, in, out, n, tsum);
    if (e == cudaSuccess) e = launch_pdl(k_scan_add, dim3(tiles), dim3(1024), 0, s, out, n, (const int32_t *)tsum, d_err);
    return e;
}

bool use_cells(const sn_system &sys, float r_cut, int nc[3])
{
    for (int a = 0; a < 3; ++a) {
        if (!(sys.box[a] > 0.0f)) return false;
        nc[a] = (int)floor((double)sys.box[a] / ((double)r_cut * 1.0001));
        if (nc[a] < 3) return false;
    }
    return true;
}

inline unsigned blocks_for(int64_t n, int bt) { return (unsigned)((n + bt - 1) / bt); }

}  // namespace

int64_t nb_cells_needed(const sn_system &sys, float r_cut, int nc[3])
{
    if (!use_cells(sys, r_cut, nc)) return 0;
    return (int64_t)nc[0] * nc[1] * nc[2] * sys.n_replicas;
}

cudaError_t launch_prep_positions(const float *pos, float4 *pos4, int64_t N, int *d_err, cudaStream_t s,
                                  Tracer *tr)
{
    if (N == 0) return cudaSuccess;
    trace_begin(tr, KK_PREP, s);
    cudaError_t e = launch_pdl(k_prep_positions, dim3(blocks_for(N, 256)), dim3(256), 0, s, pos, pos4, N, d_err);
    trace_end(tr, s);
    return e;
}

cudaError_t launch_neighbors(const sn_system &sys, float r_cut, const float4 *pos4, NbWork &w,
                             int32_t *row_ptr, int32_t *col, int64_t cap, int *d_err,
                             int64_t *n_edges_host, cudaStream_t s, Tracer *tr)
{
    const int64_t N = (int64_t)sys.n_per_replica * sys.n_replicas;
    Geometry g;
    for (int a = 0; a < 3; ++a) {
        g.box[a] = sys.box[a];
        g.periodic[a] = sys.box[a] > 0.0f;
    }
    const float rc2 = r_cut * r_cut;
    cudaError_t e;
    if (N == 0) {
        e = cudaMemsetAsync(row_ptr, 0, sizeof(int32_t), s);
        if (n_edges_host) *n_edges_host = 0;
        return e;
    }
    int nc[3];
    const bool cells = use_cells(sys, r_cut, nc);
    CellGrid cg{};
    if (cells) {
        double margin = 1e300, Lmax = 0.0;
        for (int a = 0; a < 3; ++a) {
            cg.nc[a] = nc[a];
            cg.side[a] = (double)sys.box[a] / (double)nc[a];
            margin = fmin(margin, cg.side[a] - (double)r_cut);
            Lmax = fmax(Lmax, (double)sys.box[a]);
        }
        // Per axis the fp32 test's separation is within 2^-22 |x|max + 2^-24 L of the exact
        // one (rounding of x_j - x_i, of L * rint(.) and of their difference), the distance
        // within sqrt(3) times that plus 2^-22 r_cut.  Half the margin is allowed for it.
        const double slack = 0.5 * margin / sqrt(3.0) - ldexp(Lmax, -24) - ldexp((double)r_cut, -22) / sqrt(3.0);
        cg.x_safe = slack > 0.0 ? (float)ldexp(slack, 22) : 0.0f;
        cg.per_rep = (int64_t)nc[0] * nc[1] * nc[2];
        cg.n_per = sys.n_per_replica;
        const int64_t ncell = cg.per_rep * sys.n_replicas;
        if (ncell > w.ncell_cap) return cudaErrorInvalidValue;
        cg.flag = w.cell_cnt + ncell + 1;
        if ((e = cudaMemsetAsync(w.cell_cnt, 0, sizeof(int32_t) * (ncell + 2), s))) return e;
        trace_begin(tr, KK_CELLS, s);
        if ((e = launch_pdl(k_cell_assign, dim3(blocks_for(N, 256)), dim3(256), 0, s, pos4, N, g, cg, w.cell_of,
                            w.cell_cnt, d_err)))
            return e;
        if ((e = scan(w.cell_cnt, w.cell_start, ncell, w.tsum, d_err, s))) return e;
        // cursor = cell_start (reuse cell_cnt as the cursor array)
        if ((e = launch_pdl(k_copy_i32, dim3(blocks_for(ncell, 256)), dim3(256), 0, s, w.cell_start, w.cell_cnt, ncell)))
            return e;
        if ((e = launch_pdl(k_cell_scatter, dim3(blocks_for(N, 256)), dim3(256), 0, s, N, w.cell_of, w.cell_cnt,
                            w.cell_atoms, d_err)))
            return e;
        trace_end(tr, s);
        trace_begin(tr, KK_NB_COUNT, s);
        if ((e = launch_pdl(k_cell_pairs<false>, dim3(blocks_for(N, BT)), dim3(BT), 0, s, pos4, N, g, cg, rc2,
                            w.cell_of, w.cell_start, w.cell_atoms, w.cnt, row_ptr, col, cap, d_err)))
            return e;
        trace_end(tr, s);
    } else {
        trace_begin(tr, KK_NB_COUNT, s);
        if ((e = launch_pdl(k_pairs<false>, dim3(blocks_for(sys.n_per_replica, PA), sys.n_replicas), dim3(256), 0, s,
                            pos4, sys.n_per_replica, g, rc2, w.cnt, row_ptr, col, cap, N, d_err)))
            return e;
        trace_end(tr, s);
    }
    trace_begin(tr, KK_SCAN, s);
    if ((e = scan(w.cnt, row_ptr, N, w.tsum, d_err, s))) return e;
    trace_end(tr, s);
    if ((e = cudaGetLastError())) return e;
    if (n_edges_host) {
        int32_t E = 0;
        if ((e = cudaMemcpyAsync(&E, row_ptr + N, sizeof(int32_t), cudaMemcpyDeviceToHost, s))) return e;
        if ((e = cudaStreamSynchronize(s))) return e;
        *n_edges_host = E;
        if (E > cap) return cudaSuccess;   // caller reports SN_ERR_CAPACITY
    }
    trace_begin(tr, KK_NB_FILL, s);
    if (cells) {
        if ((e = launch_pdl(k_cell_pairs<true>, dim3(blocks_for(N, BT)), dim3(BT), 0, s, pos4, N, g, cg, rc2, w.cell_of,
                            w.cell_start, w.cell_atoms, w.cnt, row_ptr, col, cap, d_err)))
            return e;
    } else {
        if ((e = launch_pdl(k_pairs<true>, dim3(blocks_for(sys.n_per_replica, PA), sys.n_replicas), dim3(256), 0, s,
                            pos4, sys.n_per_replica, g, rc2, w.cnt, row_ptr, col, cap, N, d_err)))
            return e;
    }
    trace_end(tr, s);
    return cudaGetLastError();
}

}  // namespace sn
