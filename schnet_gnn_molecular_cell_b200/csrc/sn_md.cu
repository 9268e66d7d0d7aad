// Velocity Verlet pieces and the per-replica sums (energy E_r = sum of eps_i, kinetic energy).
#include <cuda_runtime.h>

#include "sn_internal.cuh"

namespace sn {

namespace {

constexpr int RB = 256;

__device__ __forceinline__ bool skip_all(const int *d_err)
{
    return (*((volatile const int *)d_err) & (ERRBIT_NONFINITE | ERRBIT_CAPACITY | ERRBIT_TIMEOUT)) != 0;
}

// v += c F ; r += dt v   (c = dt/2 * kappa / m), per component
__global__ void k_kick_drift(float *__restrict__ pos, float *__restrict__ vel, const float *__restrict__ forces,
                             int64_t n3, float c, float dt, const int *__restrict__ d_err)
{
    if (skip_all(d_err)) return;
    int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (q >= n3) return;
    const float v = vel[q] + c * forces[q];
    vel[q] = v;
    pos[q] = pos[q] + dt * v;
}

__global__ void k_kick(float *__restrict__ vel, const float *__restrict__ forces, int64_t n3, float c,
                       const int *__restrict__ d_err)
{
    if (skip_all(d_err)) return;
    int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (q >= n3) return;
    vel[q] = vel[q] + c * forces[q];
}

// one CTA per replica; fixed summation order (strided partial sums, then a tree)
__global__ void __launch_bounds__(RB) k_replica_sums(const float *__restrict__ eps, const float *__restrict__ vel,
                                                     int n_per, float half_m_over_kappa, float *__restrict__ energy,
                                                     float *__restrict__ kinetic, const int *__restrict__ d_err)
{
    __shared__ float se[RB], sk[RB];
    if (skip_all(d_err)) return;
    const int r = blockIdx.x;
    const int64_t base = (int64_t)r * n_per;
    float e = 0.0f, k = 0.0f;
    for (int i = threadIdx.x; i < n_per; i += RB) {
        if (energy) e += eps[base + i];
        if (kinetic) {
            const float vx = vel[3 * (base + i)], vy = vel[3 * (base + i) + 1], vz = vel[3 * (base + i) + 2];
            k += vx * vx + vy * vy + vz * vz;
        }
    }
    se[threadIdx.x] = e;
    sk[threadIdx.x] = k;
    __syncthreads();
    for (int s = RB / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) {
            se[threadIdx.x] += se[threadIdx.x + s];
            sk[threadIdx.x] += sk[threadIdx.x + s];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        if (energy) energy[r] = se[0];
        if (kinetic) kinetic[r] = half_m_over_kappa * sk[0];
    }
}

inline unsigned blocks_for(int64_t n, int bt) { return (unsigned)((n + bt - 1) / bt); }

}  // namespace

cudaError_t launch_kick_drift(float *pos, float *vel, const float *forces, int64_t n3, float c, float dt,
                              int *d_err, cudaStream_t s, Tracer *tr)
{
    if (n3 == 0) return cudaSuccess;
    trace_begin(tr, KK_KICK_DRIFT, s);
    k_kick_drift<<<blocks_for(n3, 256), 256, 0, s>>>(pos, vel, forces, n3, c, dt, d_err);
    trace_end(tr, s);
    return cudaGetLastError();
}

cudaError_t launch_kick(float *vel, const float *forces, int64_t n3, float c, int *d_err, cudaStream_t s,
                        Tracer *tr)
{
    if (n3 == 0) return cudaSuccess;
    trace_begin(tr, KK_KICK, s);
    k_kick<<<blocks_for(n3, 256), 256, 0, s>>>(vel, forces, n3, c, d_err);
    trace_end(tr, s);
    return cudaGetLastError();
}

cudaError_t launch_replica_sums(const float *eps, const float *vel, int n_per, int n_rep, float half_m_over_kappa,
                                float *energy, float *kinetic, int *d_err, cudaStream_t s, Tracer *tr)
{
    if (n_rep == 0) return cudaSuccess;
    trace_begin(tr, KK_SUMS, s);
    k_replica_sums<<<n_rep, RB, 0, s>>>(eps, vel, n_per, half_m_over_kappa, energy, kinetic, d_err);
    trace_end(tr, s);
    return cudaGetLastError();
}

}  // namespace sn
