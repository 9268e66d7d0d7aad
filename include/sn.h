/*
 * sn.h -- C ABI of the B200 SchNet energy/force library (libsnflash.so).
 *
 * One energy-and-force evaluation of a SchNet continuous-filter-convolution potential over a
 * dynamic neighbour graph, its neighbour builder and a velocity-Verlet step, as described in
 * FlashSchNet (arXiv 2602.13140): §3.2 "SchNet model" defines the pipeline, §4.2 "Flash
 * message passing fused edge computation" the fused per-edge operator, §4.3 "Flash
 * aggregation segmented reductions" the destination-grouped CSR reduction, §4.1 "Precision
 * contract for force-based simulation" the fp32 positions/energies/forces.
 *
 * Model (per interaction block t = 0..T-1, all atoms i, all edges e = (j -> i)):
 *   u_e = r_i - r_j (minimum image on periodic axes), d_e = |u_e|
 *   bt_e[k] = exp(-gamma (d_e - mu_k)^2) * (cos(pi d_e / r_cut) + 1) / 2,  mu_k = k r_cut/(K-1)
 *   w_e = W2 ssp(W1 bt_e + b1) + b2                          (filter network K -> F -> F)
 *   h_i = sum_{e: dst=i} x^t_{src e} (.) w_e                  (message + segment sum)
 *   x^{t+1}_i = x^t_i + U2 ssp(U1 h_i + c1) + c2              (update network, residual)
 * x^0_i = Emb[Z_i];  eps_i = R2 ssp(R1 x^T_i + e1) + e2;  E_r = sum_{i in replica r} eps_i;
 * F_i = -dE/dr_i.  ssp(x) = ln(e^x / 2 + 1/2) (shifted softplus).
 *
 * Conventions
 *  - Every array argument named *_dev is a device pointer owned by the caller; *_host is a
 *    host pointer owned by the caller.  The library never frees caller memory.
 *  - Work is enqueued on the context's CUDA stream and is asynchronous unless stated.
 *    Conditions found on the device (capacity overflow, non-finite input, coincident
 *    atoms) are latched in the context and returned by sn_sync(); kernels enqueued after
 *    such a condition skip their work.
 *  - Errors are status codes; nothing is thrown, no kernel traps.  sn_last_error() gives a
 *    one-line message for the last failing call.
 *  - Units: positions A, energies kcal/mol, forces kcal/mol/A, velocities A/fs, masses amu,
 *    time fs.  All floating-point arrays are float32.
 *  - Atoms are numbered globally: atom i of replica r has index r * n_per_replica + i.
 *    Edges never cross replicas.
 */
#ifndef SN_H
#define SN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SN_OK = 0,
    SN_ERR_INVALID_ARG = 1,   /* bad pointer, size, config or box (r_cut >= box/2)        */
    SN_ERR_CAPACITY = 2,      /* neighbour list does not fit the given capacity           */
    SN_ERR_NONFINITE = 3,     /* a position is NaN or infinite                            */
    SN_ERR_DEGENERATE = 4,    /* two atoms of one replica at distance 0 (direction undefined) */
    SN_ERR_CUDA = 5,          /* a CUDA runtime call failed; message in sn_last_error      */
    SN_ERR_UNSUPPORTED = 6,   /* model size outside what the kernels are built for         */
    SN_ERR_NOMEM = 7,         /* device or host allocation failed                          */
    SN_ERR_TIMEOUT = 8        /* a kernel gave up waiting for its own tensor-core work      */
} sn_status;

/* Arithmetic of the MLPs: filter, update and readout networks alike (every GEMM of a mode
 * uses the same operand precision; positions, distances, the Gaussian basis, energies,
 * forces and all reductions are fp32, or double where stated, in every mode).
 *  SN_PREC_FP32: fp32 on CUDA cores.
 *  SN_PREC_FP16: fp16 operands (weights and activations) on the tensor cores (tcgen05),
 *                fp32 accumulation in TMEM -- the W16A16 precision of FlashSchNet §4.4,
 *                weights cast to fp16 with round-to-nearest (one scale per tensor = 1).
 *  SN_PREC_TC32: fp32-accurate on the tensor cores: every operand split into two fp16
 *                terms, products accumulated as hi*hi + hi*lo + lo*hi (3 MMAs).
 *  SN_PREC_FP16_CH: SN_PREC_FP16 with one scale per output channel (FlashSchNet §4.4
 *                "channel-wise quantization"): every weight matrix W (W1, W2, U1, U2, R1) is
 *                stored as fp16(W[o][:] / s_o), s_o = max_i |W[o][i]| (1 for an all-zero
 *                row), and s_o multiplies the fp32 accumulator of output channel o; the
 *                transposed products of the backward pass take s_o on their operand instead.
 *                The scales are computed from the weights at sn_create (no calibration data).
 * The tensor-core modes need F = 128. */
enum {
    SN_PREC_FP32 = 0,
    SN_PREC_FP16 = 1,
    SN_PREC_TC32 = 2,
    SN_PREC_FP16_CH = 3
};

/* Model hyper-parameters.  Supported: F in {64, 128}, 2 <= K <= 64, T >= 1, n_types >= 1. */
typedef struct {
    int32_t F;          /* hidden features D                                               */
    int32_t K;          /* Gaussian radial basis functions D_r                             */
    int32_t T;          /* interaction blocks                                              */
    int32_t n_types;    /* bead / atom types (rows of the embedding)                       */
    float r_cut;        /* cutoff radius (A); also the last Gaussian centre                */
    float gamma;        /* Gaussian width parameter (A^-2)                                 */
    int32_t precision;  /* SN_PREC_*                                                       */
} sn_config;

/* A batch of n_replicas independent systems of n_per_replica atoms each.  box[a] > 0 makes
 * axis a periodic with that length; all zero = open boundaries.  A periodic axis needs
 * r_cut < box[a] / 2. */
typedef struct {
    int32_t n_per_replica;
    int32_t n_replicas;
    float box[3];
} sn_system;

typedef struct sn_ctx sn_ctx;

/*
 * Create a context on the current CUDA device.
 *   weights_host: the flat float32 weight blob, n_weights floats, in this order (every
 *     Linear is W[out][in] row-major followed by b[out]):
 *       Emb[n_types][F];
 *       per block: W1[F][K] b1[F] W2[F][F] b2[F] U1[F][F] c1[F] U2[F][F] c2[F];
 *       R1[F/2][F] e1[F/2] R2[1][F/2] e2[1].
 *     It is copied (and re-laid out for the kernels); the caller keeps ownership.
 *   cuda_stream: a cudaStream_t (NULL = the legacy default stream) on which all work of
 *     the context is enqueued.
 * Returns SN_ERR_INVALID_ARG for a size mismatch, SN_ERR_UNSUPPORTED for sizes the kernels
 * are not built for.  Synchronous.
 */
sn_status sn_create(const sn_config *cfg, const float *weights_host, int64_t n_weights,
                    void *cuda_stream, sn_ctx **out);

/* Free the context and its device memory (synchronises its stream first). */
sn_status sn_destroy(sn_ctx *ctx);

/* Change the stream used by later calls. */
sn_status sn_set_stream(sn_ctx *ctx, void *cuda_stream);

/*
 * Size the context's device workspace for systems of up to sys->n_per_replica *
 * sys->n_replicas atoms and max_edges directed edges, so that later calls with sizes
 * within these bounds allocate nothing.  Synchronous (may call cudaMalloc).
 */
sn_status sn_reserve(sn_ctx *ctx, const sn_system *sys, int64_t max_edges);

/*
 * Neighbour list (§3.2 "Building the neighbor list"; §4.3 "Index construction under
 * dynamic neighbor lists"): every directed edge j -> i, i != j, i and j in the same
 * replica, with r2 < r_cut^2, where per axis dx = x_j - x_i, on periodic axes
 * dx = dx - L * rint(dx / L), and r2 = (dx*dx + dy*dy) + dz*dz, each float32 operation
 * rounded on its own (no fused multiply-add).  Output is CSR grouped by destination:
 * row_ptr_dev[N+1] (int32, exclusive prefix sums), col_dev[E] (int32 source indices),
 * rows in ascending destination, sources ascending inside each row.
 *   pos_dev: float32 [N][3].
 *   cap: capacity of col_dev in entries.
 *   n_edges_out (host): set to E.  If E > cap, returns SN_ERR_CAPACITY with *n_edges_out =
 *     the required E; col_dev is then unspecified.
 * Synchronises once (to read E back to the host).  Returns SN_ERR_NONFINITE /
 * SN_ERR_DEGENERATE if a position is not finite / two atoms coincide (outputs are
 * still written in the latter case).
 */
sn_status sn_build_neighbors(sn_ctx *ctx, const sn_system *sys, const float *pos_dev,
                             int32_t *row_ptr_dev, int32_t *col_dev, int64_t cap,
                             int64_t *n_edges_out);

/*
 * Energy and forces (§3.2 "Energy readout", "Forces via autodiff"; §4.2; §4.3) over a
 * neighbour list in the layout sn_build_neighbors writes.
 *   pos_dev float32 [N][3]; types_dev int32 [N] in [0, n_types);
 *   row_ptr_dev int32 [N+1], col_dev int32 [n_edges] (n_edges = row_ptr[N]);
 *   energy_dev float32 [n_replicas] (out), forces_dev float32 [N][3] (out).
 * The list must be symmetric (j -> i present iff i -> j present), as sn_build_neighbors
 * produces; the force kernel relies on it.  Asynchronous: a row_ptr whose last entry
 * exceeds n_edges (or whose first is negative) is detected on the device before col is
 * read, and the next sn_sync returns SN_ERR_CAPACITY (outputs unspecified).
 */
sn_status sn_energy_forces(sn_ctx *ctx, const sn_system *sys, const float *pos_dev,
                           const int32_t *types_dev, const int32_t *row_ptr_dev,
                           const int32_t *col_dev, int64_t n_edges, float *energy_dev,
                           float *forces_dev);

/*
 * n_steps of NVE velocity Verlet (cfg3 of the benchmark; the pages' own runs use Langevin,
 * §5.1 "Experimental setting"), each step:
 *   v += dt/2 * kappa * F / m;  r += dt * v;  rebuild the neighbour list (as
 *   sn_build_neighbors, into the context's workspace);  F, E = energy_forces(r);
 *   v += dt/2 * kappa * F / m;  kinetic_r = sum_{i in r} m |v_i|^2 / (2 kappa),
 * kappa = 4.184e-4 A^2 fs^-2 per (kcal/mol)/amu.
 *   pos_dev, vel_dev float32 [N][3] (in/out); forces_dev [N][3]: in F(t0), out F(t_end);
 *   energy_dev, kinetic_dev float32 [n_replicas] (out, after the last step).
 * The context's edge capacity must hold every step's list (sn_reserve); an overflow is
 * latched as SN_ERR_CAPACITY (see sn_sync) and the remaining work of the call is skipped.
 * Asynchronous: no host synchronisation.
 */
sn_status sn_md_step(sn_ctx *ctx, const sn_system *sys, float *pos_dev, float *vel_dev,
                     float *forces_dev, const int32_t *types_dev, float mass_amu, float dt_fs,
                     int32_t n_steps, float *energy_dev, float *kinetic_dev);

/*
 * n_steps of Langevin dynamics (the integrator of FlashSchNet §5.1 "Experimental setting":
 * Langevin dynamics at 300 K, 4 fs), BAOAB splitting, each step:
 *   v += dt/2 kappa F/m;  r += dt/2 v;  v = a v + b xi;  r += dt/2 v;
 *   rebuild the list;  F, E = energy_forces(r);  v += dt/2 kappa F/m,
 * a = exp(-friction_per_fs dt), b = sqrt((1 - a^2) kB T kappa / m), kB = 0.0019872041
 * kcal/mol/K.  xi of step s (= step0 + 0 .. n_steps-1) and atom i: Philox4x32-10 (Salmon et
 * al., 2011) of counter (s mod 2^32, s / 2^32, i, 0) and key (seed mod 2^32, seed / 2^32); its
 * words u_q = (r_q + 1/2) / 2^32 give xi_x, xi_y = sqrt(-2 ln u0) (cos, sin)(2 pi u1) and
 * xi_z = sqrt(-2 ln u2) cos(2 pi u3).  Pass step0 = the number of steps already taken to
 * continue a trajectory.  Arguments, outputs and asynchrony as for sn_md_step.
 */
sn_status sn_md_langevin(sn_ctx *ctx, const sn_system *sys, float *pos_dev, float *vel_dev,
                         float *forces_dev, const int32_t *types_dev, float mass_amu, float dt_fs,
                         int32_t n_steps, float temperature_k, float friction_per_fs, uint64_t seed,
                         int64_t step0, float *energy_dev, float *kinetic_dev);

/*
 * Same as sn_md_step with every array in host memory (pageable or pinned): copies the
 * inputs to the context's device buffers, runs the steps, copies pos, vel, forces, energy
 * and kinetic back, and synchronises.  Returns any latched device condition.
 */
sn_status sn_md_step_host(sn_ctx *ctx, const sn_system *sys, float *pos_host, float *vel_host,
                          float *forces_host, const int32_t *types_host, float mass_amu,
                          float dt_fs, int32_t n_steps, float *energy_host,
                          float *kinetic_host);

/* Wait for the context's stream; return (and clear) the first condition latched on the
 * device since the last sn_sync, or SN_ERR_CUDA if the stream failed. */
sn_status sn_sync(sn_ctx *ctx);

/*
 * Bound, in GPU clock cycles, of the tensor-core kernels' waits for their own MMAs (default
 * 2^32, about 2 s; 0 restores it).  These waits depend on no other agent and end in
 * microseconds; a bound far shorter than an MMA makes them give up: the kernel then latches
 * SN_ERR_TIMEOUT (returned by the next sn_sync), lets every MMA it issued complete under the
 * default bound, releases its tensor memory and returns, and later kernels of the call skip
 * their work.  The context stays usable.  The paper has no counterpart: this exists so that
 * the time-out path can be exercised.  SN_ERR_INVALID_ARG for a negative bound.
 */
sn_status sn_set_wait_limit(sn_ctx *ctx, int64_t cycles);

/*
 * Neighbour list without any device memory allocation.
 *
 * The paper has no counterpart of this entry point; it exists for callers that cannot call
 * cudaMalloc: a host MD engine or framework that has already reserved nearly all device
 * memory for its own pool (a raw cudaMalloc would fail or fragment it), a step loop that
 * must not pay the implicit device synchronisation of cudaMalloc/cudaFree, or a plugin
 * whose host application forbids allocations it does not own.  sn_build_neighbors needs a
 * context, and creating or growing one calls cudaMalloc; this function needs no context.
 *
 * Output, arguments and statuses are those of sn_build_neighbors (same list, same CSR
 * order, bit for bit), with r_cut given directly and the work enqueued on cuda_stream
 * (a cudaStream_t, NULL = legacy default stream); it synchronises that stream once.
 * Its work buffers are one static device array of about 2.3 MB that every GPU which loads
 * the library keeps until the process exits.  Limits: at most SN_NOALLOC_MAX_ATOMS atoms
 * in total and, for periodic boxes built with the cell list, at most SN_NOALLOC_MAX_CELLS
 * cells (n_replicas x cells per box); larger systems get SN_ERR_UNSUPPORTED and nothing
 * is launched.  Every call looks up the array's device address on the current device (a
 * host-side lookup, repeated each call so that an address from before a cudaDeviceReset is
 * never reused); the first call on a device also loads the library's device code there,
 * so make that first call before any stream capture.  All calls share the one array:
 * calls that overlap on the GPU (different streams or host threads at the same time) race
 * and must be serialised by the caller.
 */
#define SN_NOALLOC_MAX_ATOMS 65536
#define SN_NOALLOC_MAX_CELLS 65536
sn_status sn_build_neighbors_noalloc(const sn_system *sys, float r_cut, const float *pos_dev,
                                     int32_t *row_ptr_dev, int32_t *col_dev, int64_t cap,
                                     int64_t *n_edges_out, void *cuda_stream);

/*
 * Kernel tracing.  While enabled, every kernel launch of the context is bracketed by a pair
 * of CUDA events on the context's stream (the events add no device work).  sn_trace_read
 * synchronises the stream, sums the elapsed times per kernel class since the last read (or
 * since enabling), writes up to max_entries entries, resets the record, and returns the
 * number of kernel classes that ran (-1 on error).  Entry names are static strings:
 * prep_positions, neighbor_count, neighbor_fill, scan, cell_bin, partition, edge_fwd,
 * node_fwd, edge_bwd, node_bwd, replica_sums, kick_drift, kick.
 */
typedef struct {
    const char *name;
    int64_t launches;
    double total_ms;
} sn_trace_entry;

sn_status sn_trace_enable(sn_ctx *ctx, int32_t on);
int32_t sn_trace_read(sn_ctx *ctx, sn_trace_entry *out, int32_t max_entries);

/* Number of directed edges of the last list built inside sn_md_step (synchronises). */
int64_t sn_md_edges(sn_ctx *ctx);

/* One-line description of the last error of this context ("" if none).  The string is
 * owned by the context. */
const char *sn_last_error(const sn_ctx *ctx);

/* Library version string, e.g. "snflash 0.1 sm_100a". */
const char *sn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SN_H */
