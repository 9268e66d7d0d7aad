// Neighbour-list build for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: an MD engine or framework that has already reserved
// (almost) all device memory for its own pool, so that a raw cudaMalloc fails or fragments
// it; code that must not trigger the implicit device synchronisation of cudaMalloc/cudaFree
// inside a latency-critical step loop; and plugins whose host application forbids foreign
// allocations.  sn_build_neighbors needs a context, whose creation and workspace growth call
// cudaMalloc.  sn_build_neighbors_noalloc needs neither: its work buffers live in one
// file-scope static device array of fixed size, which every GPU that loads the library holds
// until the process exits.  The caller still provides positions and the output CSR arrays.
#include <cuda_runtime.h>
#include <math.h>

#include "sn_internal.cuh"

namespace {

constexpr int64_t kMaxAtoms = SN_NOALLOC_MAX_ATOMS;
constexpr int64_t kMaxCells = SN_NOALLOC_MAX_CELLS;

constexpr size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// byte offsets inside the static array
constexpr size_t kOffPos4 = 0;                                                  // float4 [kMaxAtoms]
constexpr size_t kOffCnt = align256(kOffPos4 + sizeof(float4) * kMaxAtoms);     // int32 [kMaxAtoms + 1]
constexpr size_t kOffCellOf = align256(kOffCnt + sizeof(int32_t) * (kMaxAtoms + 1));
constexpr size_t kOffCellAtoms = align256(kOffCellOf + sizeof(int32_t) * kMaxAtoms);
constexpr size_t kOffCellCnt = align256(kOffCellAtoms + sizeof(int32_t) * kMaxAtoms);   // [kMaxCells + 2]
constexpr size_t kOffCellStart = align256(kOffCellCnt + sizeof(int32_t) * (kMaxCells + 2));
constexpr size_t kOffTsum = align256(kOffCellStart + sizeof(int32_t) * (kMaxCells + 1));  // scan tile sums
constexpr int64_t kTsum = (kMaxAtoms > kMaxCells ? kMaxAtoms : kMaxCells) / 4096 + 2;
constexpr size_t kOffErr = align256(kOffTsum + sizeof(int32_t) * kTsum);                // int32 error bits
constexpr size_t kScratchBytes = align256(kOffErr + sizeof(int32_t));

static __device__ __align__(256) unsigned char g_nb_scratch[kScratchBytes];

// Device address of g_nb_scratch on the current device.  In host code the symbol is only a
// host-side stand-in; the address a kernel may use comes from cudaGetSymbolAddress with that
// device current.  It is looked up on every call (a host-side table lookup): a cached address
// would go stale when cudaDeviceReset recreates the device's context and module.
sn_status scratch_on_current_device(unsigned char **out)
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_nb_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return SN_ERR_CUDA;
    }
    *out = static_cast<unsigned char *>(p);
    return SN_OK;
}

}  // namespace

extern "C" sn_status sn_build_neighbors_noalloc(const sn_system *sys, float r_cut, const float *pos_dev,
                                                int32_t *row_ptr_dev, int32_t *col_dev, int64_t cap,
                                                int64_t *n_edges_out, void *cuda_stream)
{
    if (!sys || !n_edges_out || !row_ptr_dev || cap < 0 || (cap > 0 && !col_dev)) return SN_ERR_INVALID_ARG;
    if (!(r_cut > 0.0f) || isinf(r_cut) || sys->n_per_replica < 0 || sys->n_replicas < 0) return SN_ERR_INVALID_ARG;
    for (int a = 0; a < 3; ++a) {
        if (!(sys->box[a] >= 0.0f) || isinf(sys->box[a])) return SN_ERR_INVALID_ARG;
        if (sys->box[a] > 0.0f && !(r_cut < 0.5f * sys->box[a])) return SN_ERR_INVALID_ARG;
    }
    const int64_t N = (int64_t)sys->n_per_replica * sys->n_replicas;
    if (N > 0 && !pos_dev) return SN_ERR_INVALID_ARG;
    if (sys->n_replicas > 65535) return SN_ERR_UNSUPPORTED;
    int nc[3];
    const int64_t ncell = sn::nb_cells_needed(*sys, r_cut, nc);
    if (N > kMaxAtoms || ncell > kMaxCells) return SN_ERR_UNSUPPORTED;   // beyond the static scratch

    unsigned char *base = nullptr;
    sn_status st = scratch_on_current_device(&base);
    if (st != SN_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    sn::NbWork w;
    w.pos4 = reinterpret_cast<float4 *>(base + kOffPos4);
    w.cnt = reinterpret_cast<int32_t *>(base + kOffCnt);
    w.cell_of = reinterpret_cast<int32_t *>(base + kOffCellOf);
    w.cell_atoms = reinterpret_cast<int32_t *>(base + kOffCellAtoms);
    w.cell_cnt = reinterpret_cast<int32_t *>(base + kOffCellCnt);
    w.cell_start = reinterpret_cast<int32_t *>(base + kOffCellStart);
    w.tsum = reinterpret_cast<int32_t *>(base + kOffTsum);
    w.ncell_cap = kMaxCells;
    int *d_err = reinterpret_cast<int *>(base + kOffErr);

    // the array keeps the previous call's contents: the error bits must start at zero (the
    // per-cell counters are cleared inside launch_neighbors, every other buffer is fully
    // overwritten before it is read)
    if (cudaMemsetAsync(d_err, 0, sizeof(int), s) != cudaSuccess) return SN_ERR_CUDA;
    if (sn::launch_prep_positions(pos_dev, w.pos4, N, d_err, s, nullptr) != cudaSuccess) return SN_ERR_CUDA;
    int64_t E = 0;
    if (sn::launch_neighbors(*sys, r_cut, w.pos4, w, row_ptr_dev, col_dev, cap, d_err, &E, s, nullptr) != cudaSuccess)
        return SN_ERR_CUDA;
    int bits = 0;
    if (cudaMemcpyAsync(&bits, d_err, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return SN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SN_ERR_CUDA;
    *n_edges_out = E;
    if (bits & sn::ERRBIT_NONFINITE) return SN_ERR_NONFINITE;
    if ((bits & sn::ERRBIT_CAPACITY) || E > cap) return SN_ERR_CAPACITY;
    if (bits & sn::ERRBIT_DEGENERATE) return SN_ERR_DEGENERATE;
    return SN_OK;
}
