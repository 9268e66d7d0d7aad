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

// The drifted position also goes to the float4 copy the neighbour and edge kernels read
// (a non-finite coordinate latches the condition and stores zeros there).
__device__ __forceinline__ void store_pos4(float4 *pos4, int64_t i, const float (&x)[3], int *d_err)
{
    if (!isfinite(x[0]) || !isfinite(x[1]) || !isfinite(x[2])) {
        atomicOr(d_err, ERRBIT_NONFINITE);
        pos4[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    } else {
        pos4[i] = make_float4(x[0], x[1], x[2], 0.0f);
    }
}

// v += c F ; r += dt v   (c = dt/2 * kappa / m), per atom
__global__ void k_kick_drift(float *__restrict__ pos, float *__restrict__ vel, const float *__restrict__ forces,
                             int64_t N, float c, float dt, float4 *__restrict__ pos4, int *__restrict__ d_err)
{
    pdl_trigger();
    pdl_wait();
    if (skip_all(d_err)) return;
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= N) return;
    float x[3];
#pragma unroll
    for (int d = 0; d < 3; ++d) {
        const int64_t q = 3 * i + d;
        const float v = vel[q] + c * forces[q];
        vel[q] = v;
        x[d] = pos[q] + dt * v;
        pos[q] = x[d];
    }
    store_pos4(pos4, i, x, d_err);
}

__global__ void k_kick(float *__restrict__ vel, const float *__restrict__ forces, int64_t n3, float c,
                       const int *__restrict__ d_err)
{
    pdl_trigger();
    pdl_wait();
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
    pdl_trigger();
    pdl_wait();
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

// Philox4x32 with 10 rounds (Salmon, Moraes, Dror and Shaw, 2011): each round multiplies
// words 0 and 2 by the two round constants, recombines the 64-bit products with words 1 and 3
// and the key; the key advances by the two Weyl constants between rounds.
__device__ __forceinline__ void philox4x32_10(uint32_t (&c)[4], uint32_t k0, uint32_t k1)
{
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint32_t lo0 = 0xD2511F53u * c[0], hi0 = __umulhi(0xD2511F53u, c[0]);
        const uint32_t lo1 = 0xCD9E8D57u * c[2], hi1 = __umulhi(0xCD9E8D57u, c[2]);
        const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0;
        c[1] = lo1;
        c[2] = n2;
        c[3] = lo0;
    }
}

// Three standard normal deviates of (step, atom): Philox words u_q = (r_q + 1/2) / 2^32,
// Box-Muller (cos, sin) of (u0, u1) and cos of (u2, u3), evaluated in double.
__device__ __forceinline__ void langevin_noise(uint64_t seed, int64_t step, int64_t atom, float (&xi)[3])
{
    uint32_t c[4] = {(uint32_t)step, (uint32_t)((uint64_t)step >> 32), (uint32_t)atom, 0u};
    philox4x32_10(c, (uint32_t)seed, (uint32_t)(seed >> 32));
    double u[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) u[q] = ((double)c[q] + 0.5) * (1.0 / 4294967296.0);
    const double r0 = sqrt(-2.0 * log(u[0])), r2 = sqrt(-2.0 * log(u[2]));
    double s1, c1;
    sincospi(2.0 * u[1], &s1, &c1);
    xi[0] = (float)(r0 * c1);
    xi[1] = (float)(r0 * s1);
    xi[2] = (float)(r2 * cospi(2.0 * u[3]));
}

// BAOAB first half per atom: v += c F; r += dt/2 v; v = a v + b xi; r += dt/2 v
__global__ void k_langevin_baoa(float *__restrict__ pos, float *__restrict__ vel, const float *__restrict__ forces,
                                int64_t N, float c, float dt, float a, float b, uint64_t seed, int64_t step,
                                float4 *__restrict__ pos4, int *__restrict__ d_err)
{
    pdl_trigger();
    pdl_wait();
    if (skip_all(d_err)) return;
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= N) return;
    float xi[3], xn[3];
    langevin_noise(seed, step, i, xi);
#pragma unroll
    for (int d = 0; d < 3; ++d) {
        const int64_t q = 3 * i + d;
        float v = vel[q] + c * forces[q];
        float x = pos[q] + 0.5f * dt * v;
        v = a * v + b * xi[d];
        xn[d] = x + 0.5f * dt * v;
        pos[q] = xn[d];
        vel[q] = v;
    }
    store_pos4(pos4, i, xn, d_err);
}

inline unsigned blocks_for(int64_t n, int bt) { return (unsigned)((n + bt - 1) / bt); }

}  // namespace

cudaError_t launch_langevin_baoa(float *pos, float *vel, const float *forces, int64_t N, float c, float dt, float a,
                                 float b, uint64_t seed, int64_t step, float4 *pos4, int *d_err, cudaStream_t s,
                                 Tracer *tr)
{
    if (N == 0) return cudaSuccess;
    trace_begin(tr, KK_KICK_DRIFT, s);
    cudaError_t e = launch_pdl(k_langevin_baoa, dim3(blocks_for(N, 128)), dim3(128), 0, s, pos, vel, forces, N, c, dt, a,
                               b, seed, step, pos4, d_err);
    trace_end(tr, s);
    return e;
}

cudaError_t launch_kick_drift(float *pos, float *vel, const float *forces, int64_t N, float c, float dt,
                              float4 *pos4, int *d_err, cudaStream_t s, Tracer *tr)
{
    if (N == 0) return cudaSuccess;
    trace_begin(tr, KK_KICK_DRIFT, s);
    cudaError_t e = launch_pdl(k_kick_drift, dim3(blocks_for(N, 256)), dim3(256), 0, s, pos, vel, forces, N, c, dt, pos4,
                               d_err);
    trace_end(tr, s);
    return e;
}

cudaError_t launch_kick(float *vel, const float *forces, int64_t n3, float c, int *d_err, cudaStream_t s,
                        Tracer *tr)
{
    if (n3 == 0) return cudaSuccess;
    trace_begin(tr, KK_KICK, s);
    cudaError_t e = launch_pdl(k_kick, dim3(blocks_for(n3, 256)), dim3(256), 0, s, vel, forces, n3, c, d_err);
    trace_end(tr, s);
    return e;
}

cudaError_t launch_replica_sums(const float *eps, const float *vel, int n_per, int n_rep, float half_m_over_kappa,
                                float *energy, float *kinetic, int *d_err, cudaStream_t s, Tracer *tr)
{
    if (n_rep == 0) return cudaSuccess;
    trace_begin(tr, KK_SUMS, s);
    cudaError_t e = launch_pdl(k_replica_sums, dim3(n_rep), dim3(RB), 0, s, eps, vel, n_per, half_m_over_kappa, energy,
                               kinetic, d_err);
    trace_end(tr, s);
    return e;
}

}  // namespace sn
