// Internal declarations of the B200 SchNet library: device layouts, error bits, launchers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "sn.h"

namespace sn {

// Kernel classes reported by the tracer (sn_trace_read).
enum KernelKind {
    KK_PREP = 0, KK_NB_COUNT, KK_NB_FILL, KK_SCAN, KK_CELLS, KK_PARTITION, KK_EDGE_FWD, KK_NODE_FWD,
    KK_EDGE_BWD, KK_NODE_BWD, KK_SUMS, KK_KICK_DRIFT, KK_KICK, KK_COUNT
};

// CUDA-event timing of every kernel launch while enabled: a pair of events per launch on the
// launching stream, read back (and reset) by sn_trace_read.
struct Tracer {
    bool on = false;
    std::vector<cudaEvent_t> ev;   // 2 per record: start, end
    std::vector<int> kinds;
    size_t n = 0;
    void begin(int kind, cudaStream_t s);
    void end(cudaStream_t s);
};

inline void trace_begin(Tracer *t, int kind, cudaStream_t s)
{
    if (t && t->on) t->begin(kind, s);
}
inline void trace_end(Tracer *t, cudaStream_t s)
{
    if (t && t->on) t->end(s);
}

// Programmatic dependent launch.  Kernels of one evaluation or MD step are launched with
// launch_pdl: a kernel may then start (and do set-up that reads nothing an earlier kernel
// writes: barrier initialisation, tensor-memory allocation, copies of the constant weights)
// while its predecessor's last CTAs run.  Every such kernel signals pdl_trigger() as it starts,
// and calls pdl_wait() on every thread before its first access to data written by an earlier
// kernel of the stream; pdl_wait returns once the preceding kernels have completed and their
// writes are visible.  Each kernel waits before it ends, so completion stays transitive along
// the chain.  (A dependent grid launches only once every CTA of its predecessor has started.)
#ifdef __CUDACC__
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
#endif

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Conditions latched on the device in ctx->d_err (bitwise OR).  Kernels that run after a
// latched condition return without touching memory.
enum : int {
    ERRBIT_CAPACITY = 1,
    ERRBIT_NONFINITE = 2,
    ERRBIT_DEGENERATE = 4,
    ERRBIT_TIMEOUT = 8,
};

constexpr int NE = 32;        // edges per tile in the fp32 kernels
constexpr int NA = 32;        // atoms per tile in the node kernels
constexpr int TS = NE + 4;    // smem row stride of [feature][edge] tiles (16-byte rows)

// Per-block weights in the fp32 kernel layout (device pointers into one allocation).
// Matrices are stored [out][in] with a row stride of in+1 floats so that both "thread =
// output" and "thread = input" sweeps read shared memory without bank conflicts.
struct BlockW {
    const float *W1;   // [F][KP+1], zero for k >= K
    const float *b1;   // [F]
    const float *W2;   // [F][F+1]
    const float *b2;   // [F]
    const float *U1;   // [F][F+1]
    const float *c1;   // [F]
    const float *U2;   // [F][F+1]
    const float *c2;   // [F]
    // tensor-core precisions: W1, W2, U1, U2 as fp16 hi / lo in the core-matrix layout of
    // sn_ef_tc.cu (lo = fp16(w - hi), used by the split mode)
    const void *W1h, *W1l, *W2h, *W2l, *U1h, *U1l, *U2h, *U2l;
    // per-output-channel scales of W1, W2, U1, U2 ([F] each; all 1 except SN_PREC_FP16_CH):
    // the fp16 matrices hold W[o][:] / s[o]
    const float *s1, *s2, *su1, *su2;
};

struct ReadoutW {
    const float *R1;   // [H][F+1]
    const float *e1;   // [H]
    const float *R2;   // [H]
    const float *e2;   // [1]
    const void *R1h, *R1l;   // tensor-core precisions: R1 padded to 128 rows, fp16 hi / lo
    const float *sr1;        // [128] per-output-channel scales of R1 (1 past H)
};

struct Geometry {
    float box[3];      // > 0 on periodic axes
    int periodic[3];
};

// Radial basis constants.  Centres mu_k = k * r_cut / (K - 1) are kept in double: the
// offsets d - mu_k are formed in double and rounded once, so that the Gaussians carry no
// error from representing d or mu_k in float (a 1e-7 A shift moves exp(-gamma x^2) by
// 2 gamma |x| 1e-7 relative, which the cancellation in dE/dd amplifies).
struct Basis {
    int K, KP;
    float r_cut, gamma;
    double r_cut_d;
    double mu[64];
    // mu_k = mu_hi[k] + mu_lo[k] (float pair, exact to ~2^-48 relative): d - mu_k is formed as
    // (d_hi - mu_hi) + (d_lo - mu_lo) in float by the tensor-core kernels
    float mu_hi[64], mu_lo[64];
};

// ---------------------------------------------------------------- neighbour list
// Builds CSR (row_ptr[N+1], col[<=cap]) for n_per x n_rep atoms into caller-provided work
// buffers.  With n_edges_host != NULL the edge count is copied back (one synchronisation) and
// the fill pass is skipped when it exceeds cap; otherwise capacity is checked on the device
// and an overflow is latched into d_err.
struct NbWork {
    float4 *pos4;      // [N]
    int32_t *cnt;      // [N + 1]
    int32_t *cell_of;  // [N]
    int32_t *cell_cnt; // [ncell + 2]: counts / cursors, then (last entry) the stencil flag
    int32_t *cell_start; // [ncell + 1]
    int32_t *cell_atoms; // [N]
    int32_t *tsum;       // [max(N, ncell) / 4096 + 2]: per-tile sums of the multi-CTA scans
    int64_t ncell_cap;
};

int64_t nb_cells_needed(const sn_system &sys, float r_cut, int nc[3]);
cudaError_t launch_prep_positions(const float *pos, float4 *pos4, int64_t N, int *d_err, cudaStream_t s,
                                  Tracer *tr);
cudaError_t launch_neighbors(const sn_system &sys, float r_cut, const float4 *pos4, NbWork &w,
                             int32_t *row_ptr, int32_t *col, int64_t cap, int *d_err,
                             int64_t *n_edges_host, cudaStream_t s, Tracer *tr);

// ---------------------------------------------------------------- energy and forces
struct EfWork {
    const float4 *pos4;  // [N]
    float *x;            // [T][N][F]   x^1 .. x^T
    float *p;            // [T][N][F]   U1 h + c1 per block
    float *h;            // [N][F]      aggregated messages of the current block
    float *hbar;         // [N][F]      dE/dh of the current block
    float *xbar;         // [N][F]      dE/dx of the current block (in place)
    float *eps;          // [N]         per-atom energies
    int32_t *part;       // [4 G + 1]   rows owned by each CTA (fp32) / warpgroup (tensor cores)
    int32_t *dst;        // [dst_cap]   destination row of every edge (tensor-core kernels)
    int64_t dst_cap;
    int64_t col_cap;     // entries of this call's col buffer (the list must fit in it)
    int G;
    long long wait_limit;   // bound (cycles) of the tensor-core kernels' waits for their MMAs
};

struct Model {
    int F, K, KP, T, H, n_types;
    int precision;       // SN_PREC_*
    Basis basis;
    const float *emb;    // [n_types][F]
    BlockW blk[16];
    ReadoutW ro;
};

cudaError_t launch_energy_forces(const Model &m, const sn_system &sys, const Geometry &geo,
                                 const int32_t *types, const int32_t *row_ptr,
                                 const int32_t *col, EfWork &w, float *energy, float *forces,
                                 int *d_err, cudaStream_t s, Tracer *tr);

// Arguments of the tensor-core edge kernels (F = 128).
struct EdgeTcArgs {
    const float4 *pos4;
    const int32_t *types, *row_ptr, *col, *part;
    const int32_t *dst;    // [E] destination row of each edge
    const float *emb;
    const float *X;        // [T][N][F]
    float *H;              // [N][F]
    const float *Hbar;     // [N][F]
    float *Xbar;           // [N][F]
    float *forces;         // [N][3]
    int64_t N;
    int n_types;           // rows of emb (the source rows of block 0)
    Geometry geo;
    Basis basis;
    const void *W1h, *W1l, *W2h, *W2l;
    const float *b1, *b2;
    const float *s1, *s2;  // [F] output-channel scales of W1 and W2
    int t;
    int *d_err;
    long long wait_limit;  // bound (cycles) of the waits for the kernel's own MMAs
};

cudaError_t launch_edge_tc(const EdgeTcArgs &a, int KP, bool split, bool backward, int G, cudaStream_t s);
int tc_groups_per_cta(bool split);   // independent row ranges per CTA of the tensor-core edge kernels
void tc_pack_matrix(const float *W, int rows, int cols, int cols_pad, const float *row_scale, uint16_t *hi,
                    uint16_t *lo);

// Arguments of the tensor-core node kernels (F = 128).
struct NodeTcArgs {
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
    int t;
    const void *U1h, *U1l, *U2h, *U2l, *R1h, *R1l;
    const float *c1, *c2, *e1, *R2, *e2;
    const float *su1, *su2, *sr1;   // output-channel scales of U1, U2 ([F]) and R1 ([128])
    int *d_err;
    long long wait_limit;           // bound (cycles) of the waits for the kernel's own MMAs
};

// which: 0 update of block a.t, 1 readout of x^T = X[a.t], 2 backward of block a.t's update
cudaError_t launch_node_tc(const NodeTcArgs &a, bool split, int which, int n_sm, cudaStream_t s);

// ---------------------------------------------------------------- integrator
cudaError_t launch_kick_drift(float *pos, float *vel, const float *forces, int64_t N, float c,
                              float dt, float4 *pos4, int *d_err, cudaStream_t s, Tracer *tr);
cudaError_t launch_kick(float *vel, const float *forces, int64_t n3, float c, int *d_err,
                        cudaStream_t s, Tracer *tr);
// BAOAB first half (B, A, O, A) with Philox4x32-10 / Box-Muller noise keyed by (seed, step, atom);
// both drift kernels also refresh the float4 position copy (replacing launch_prep_positions)
cudaError_t launch_langevin_baoa(float *pos, float *vel, const float *forces, int64_t N, float c, float dt, float a,
                                 float b, uint64_t seed, int64_t step, float4 *pos4, int *d_err, cudaStream_t s,
                                 Tracer *tr);
cudaError_t launch_replica_sums(const float *eps, const float *vel, int n_per, int n_rep,
                                float half_m_over_kappa, float *energy, float *kinetic,
                                int *d_err, cudaStream_t s, Tracer *tr);

}  // namespace sn
