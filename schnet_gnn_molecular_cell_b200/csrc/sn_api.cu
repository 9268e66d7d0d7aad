// C ABI of the B200 SchNet library: context, workspace, weight re-layout and the entry points
// declared in sn.h.  All numerical work happens in the kernels of the other .cu files.
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <vector>

#include "sn_internal.cuh"

namespace {

constexpr int MAX_T = 16;
constexpr float KAPPA = 4.184e-4f;   // A^2 fs^-2 per (kcal/mol)/amu

struct DevBuf {
    void *p = nullptr;
    size_t bytes = 0;
};

}  // namespace

struct sn_ctx {
    sn_config cfg{};
    int F = 0, K = 0, KP = 0, T = 0, H = 0;
    cudaStream_t stream = nullptr;
    int device = 0;
    int n_sm = 148;
    float *d_weights = nullptr;
    uint16_t *d_tcw = nullptr;         // fp16 hi/lo filter weights for the tensor-core modes
    sn::Model model{};
    int *d_err = nullptr;
    int32_t *h_err = nullptr;          // pinned
    // workspace
    DevBuf pos4, cnt, cell_of, cell_cnt, cell_start, cell_atoms, tsum;
    DevBuf x, p, h, hbar, xbar, eps, part, dst;
    DevBuf md_row_ptr, md_col;
    int64_t md_cap = 0;                // entries of md_col
    int64_t md_last_N = 0;
    // device mirrors for sn_md_step_host
    DevBuf hc_pos, hc_vel, hc_forces, hc_types, hc_energy, hc_kin;
    sn::Tracer tracer;
    long long wait_limit = 1ll << 32;   // bound of the tensor-core kernels' waits for their MMAs
    char last_error[256] = {0};
};

namespace sn {

void Tracer::begin(int kind, cudaStream_t s)
{
    if (n == kinds.size()) {
        cudaEvent_t a, b;
        if (cudaEventCreate(&a) != cudaSuccess) return;
        if (cudaEventCreate(&b) != cudaSuccess) {
            cudaEventDestroy(a);
            return;
        }
        ev.push_back(a);
        ev.push_back(b);
        kinds.push_back(kind);
    }
    kinds[n] = kind;
    cudaEventRecord(ev[2 * n], s);
}

void Tracer::end(cudaStream_t s)
{
    if (n < kinds.size()) {
        cudaEventRecord(ev[2 * n + 1], s);
        ++n;
    }
}

}  // namespace sn

namespace {

sn_status fail(sn_ctx *c, sn_status st, const char *fmt, ...)
{
    if (c) {
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(c->last_error, sizeof(c->last_error), fmt, ap);
        va_end(ap);
    }
    return st;
}

sn_status cuda_fail(sn_ctx *c, cudaError_t e, const char *where)
{
    return fail(c, SN_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define SN_CUDA(call)                                         \
    do {                                                      \
        cudaError_t e_ = (call);                              \
        if (e_ != cudaSuccess) return cuda_fail(ctx, e_, #call); \
    } while (0)

sn_status grow(sn_ctx *ctx, DevBuf &b, size_t bytes)
{
    if (bytes == 0) bytes = 16;
    if (b.bytes >= bytes) return SN_OK;
    if (b.p) {
        cudaError_t e = cudaStreamSynchronize(ctx->stream);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaStreamSynchronize");
        cudaFree(b.p);
        b.p = nullptr;
        b.bytes = 0;
    }
    cudaError_t e = cudaMalloc(&b.p, bytes);
    if (e != cudaSuccess) {
        b.p = nullptr;
        cudaGetLastError();
        return fail(ctx, SN_ERR_NOMEM, "cudaMalloc(%zu): %s", bytes, cudaGetErrorString(e));
    }
    b.bytes = bytes;
    return SN_OK;
}

void release(DevBuf &b)
{
    if (b.p) cudaFree(b.p);
    b.p = nullptr;
    b.bytes = 0;
}

int64_t n_atoms(const sn_system *s) { return (int64_t)s->n_per_replica * s->n_replicas; }

sn_status check_system(sn_ctx *ctx, const sn_system *s)
{
    if (!s) return fail(ctx, SN_ERR_INVALID_ARG, "system is NULL");
    if (s->n_per_replica < 0 || s->n_replicas < 0) return fail(ctx, SN_ERR_INVALID_ARG, "negative atom count");
    if (s->n_replicas > 65535) return fail(ctx, SN_ERR_UNSUPPORTED, "more than 65535 replicas");
    if (n_atoms(s) >= 0x7fffffffLL) return fail(ctx, SN_ERR_UNSUPPORTED, "more than 2^31-1 atoms");
    for (int a = 0; a < 3; ++a) {
        if (!(s->box[a] >= 0.0f) || isinf(s->box[a])) return fail(ctx, SN_ERR_INVALID_ARG, "box[%d] invalid", a);
        if (s->box[a] > 0.0f && !(ctx->cfg.r_cut < 0.5f * s->box[a]))
            return fail(ctx, SN_ERR_INVALID_ARG, "r_cut %g >= box[%d]/2", ctx->cfg.r_cut, a);
    }
    return SN_OK;
}

// grid of the edge kernels: one CTA per SM (the fp32 kernels hold ~130-160 KB of shared memory)
int edge_grid(const sn_ctx *ctx) { return ctx->n_sm; }

sn_status ensure_nb(sn_ctx *ctx, const sn_system *s)
{
    const int64_t N = n_atoms(s);
    int nc[3];
    const int64_t ncell = sn::nb_cells_needed(*s, ctx->cfg.r_cut, nc);
    sn_status st;
    if ((st = grow(ctx, ctx->pos4, sizeof(float4) * N))) return st;
    if ((st = grow(ctx, ctx->cnt, sizeof(int32_t) * (N + 1)))) return st;
    if ((st = grow(ctx, ctx->cell_of, sizeof(int32_t) * N))) return st;
    if ((st = grow(ctx, ctx->cell_atoms, sizeof(int32_t) * N))) return st;
    if ((st = grow(ctx, ctx->cell_cnt, sizeof(int32_t) * (ncell + 2)))) return st;
    if ((st = grow(ctx, ctx->cell_start, sizeof(int32_t) * (ncell + 1)))) return st;
    if ((st = grow(ctx, ctx->tsum, sizeof(int32_t) * ((N > ncell ? N : ncell) / 4096 + 2)))) return st;
    return SN_OK;
}

sn_status ensure_ef(sn_ctx *ctx, const sn_system *s)
{
    const int64_t N = n_atoms(s);
    const size_t nf = sizeof(float) * (size_t)N * ctx->F;
    sn_status st;
    if ((st = ensure_nb(ctx, s))) return st;
    if ((st = grow(ctx, ctx->x, nf * ctx->T))) return st;
    if ((st = grow(ctx, ctx->p, nf * ctx->T))) return st;
    if ((st = grow(ctx, ctx->h, nf))) return st;
    if ((st = grow(ctx, ctx->hbar, nf))) return st;
    if ((st = grow(ctx, ctx->xbar, nf))) return st;
    if ((st = grow(ctx, ctx->eps, sizeof(float) * N))) return st;
    if ((st = grow(ctx, ctx->part, sizeof(int32_t) * (4 * edge_grid(ctx) + 1)))) return st;
    return SN_OK;
}

sn::NbWork nb_work(sn_ctx *ctx)
{
    sn::NbWork w;
    w.pos4 = (float4 *)ctx->pos4.p;
    w.cnt = (int32_t *)ctx->cnt.p;
    w.cell_of = (int32_t *)ctx->cell_of.p;
    w.cell_cnt = (int32_t *)ctx->cell_cnt.p;
    w.cell_start = (int32_t *)ctx->cell_start.p;
    w.cell_atoms = (int32_t *)ctx->cell_atoms.p;
    w.tsum = (int32_t *)ctx->tsum.p;
    w.ncell_cap = (int64_t)(ctx->cell_cnt.bytes / sizeof(int32_t)) - 2;
    return w;
}

sn::EfWork ef_work(sn_ctx *ctx)
{
    sn::EfWork w;
    w.pos4 = (const float4 *)ctx->pos4.p;
    w.x = (float *)ctx->x.p;
    w.p = (float *)ctx->p.p;
    w.h = (float *)ctx->h.p;
    w.hbar = (float *)ctx->hbar.p;
    w.xbar = (float *)ctx->xbar.p;
    w.eps = (float *)ctx->eps.p;
    w.part = (int32_t *)ctx->part.p;
    w.dst = (int32_t *)ctx->dst.p;
    w.dst_cap = (int64_t)(ctx->dst.bytes / sizeof(int32_t));
    w.col_cap = 0;
    w.G = edge_grid(ctx);
    w.wait_limit = ctx->wait_limit;
    return w;
}

sn::Geometry geometry(const sn_system *s)
{
    sn::Geometry g;
    for (int a = 0; a < 3; ++a) {
        g.box[a] = s->box[a];
        g.periodic[a] = s->box[a] > 0.0f;
    }
    return g;
}

sn_status status_from_bits(sn_ctx *ctx, int bits)
{
    if (bits & sn::ERRBIT_CAPACITY) return fail(ctx, SN_ERR_CAPACITY, "neighbour list exceeded the edge capacity");
    if (bits & sn::ERRBIT_NONFINITE) return fail(ctx, SN_ERR_NONFINITE, "non-finite position");
    if (bits & sn::ERRBIT_DEGENERATE) return fail(ctx, SN_ERR_DEGENERATE, "two atoms at distance 0");
    if (bits & sn::ERRBIT_TIMEOUT) return fail(ctx, SN_ERR_TIMEOUT, "a kernel timed out waiting for its tensor-core work");
    return SN_OK;
}

// synchronise, read and clear the latched device conditions
sn_status drain(sn_ctx *ctx)
{
    SN_CUDA(cudaMemcpyAsync(ctx->h_err, ctx->d_err, sizeof(int), cudaMemcpyDeviceToHost, ctx->stream));
    SN_CUDA(cudaStreamSynchronize(ctx->stream));
    const int bits = *ctx->h_err;
    if (bits) SN_CUDA(cudaMemsetAsync(ctx->d_err, 0, sizeof(int), ctx->stream));
    if (bits) SN_CUDA(cudaStreamSynchronize(ctx->stream));
    return status_from_bits(ctx, bits);
}

// energy + forces on positions already staged in ctx->pos4
sn_status enqueue_ef(sn_ctx *ctx, const sn_system *s, const int32_t *types, const int32_t *row_ptr,
                     const int32_t *col, int64_t n_col, float *energy, float *forces)
{
    sn::EfWork w = ef_work(ctx);
    w.col_cap = n_col;
    const sn::Geometry g = geometry(s);
    cudaError_t e = sn::launch_energy_forces(ctx->model, *s, g, types, row_ptr, col, w, energy, forces,
                                             ctx->d_err, ctx->stream, &ctx->tracer);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "energy/force kernels");
    e = sn::launch_replica_sums(w.eps, nullptr, s->n_per_replica, s->n_replicas, 0.0f, energy, nullptr, ctx->d_err,
                                ctx->stream, &ctx->tracer);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "replica sums");
    return SN_OK;
}

// offsets of the packed device weights (in floats, each array aligned to 64 floats)
struct Packer {
    std::vector<float> buf;
    size_t take(size_t n)
    {
        size_t off = (buf.size() + 63) / 64 * 64;
        buf.resize(off + n, 0.0f);
        return off;
    }
};

}  // namespace

extern "C" {

const char *sn_version(void) { return "snflash 0.1 sm_100a"; }

const char *sn_last_error(const sn_ctx *ctx) { return ctx ? ctx->last_error : "context is NULL"; }

sn_status sn_create(const sn_config *cfg, const float *weights_host, int64_t n_weights, void *cuda_stream,
                    sn_ctx **out)
{
    if (!out) return SN_ERR_INVALID_ARG;
    *out = nullptr;
    if (!cfg || !weights_host) return SN_ERR_INVALID_ARG;
    const int F = cfg->F, K = cfg->K, T = cfg->T, NT = cfg->n_types;
    if (!(cfg->r_cut > 0.0f) || isinf(cfg->r_cut) || !(cfg->gamma > 0.0f) || NT < 1 || K < 2 || T < 1 || F < 2)
        return SN_ERR_INVALID_ARG;
    if (!(F == 64 || F == 128) || K > 64 || T > MAX_T) return SN_ERR_UNSUPPORTED;
    if (cfg->precision != SN_PREC_FP32 && cfg->precision != SN_PREC_FP16 && cfg->precision != SN_PREC_TC32 &&
        cfg->precision != SN_PREC_FP16_CH)
        return SN_ERR_INVALID_ARG;
    if (cfg->precision != SN_PREC_FP32 && F != 128) return SN_ERR_UNSUPPORTED;
    const int H = F / 2;
    const int64_t per_block = (int64_t)F * K + F + 3 * ((int64_t)F * F + F);
    const int64_t expect = (int64_t)NT * F + T * per_block + (int64_t)H * F + H + H + 1;
    if (n_weights != expect) return SN_ERR_INVALID_ARG;

    sn_ctx *ctx = new sn_ctx();
    ctx->cfg = *cfg;
    ctx->F = F;
    ctx->K = K;
    ctx->KP = K <= 32 ? 32 : 64;
    ctx->T = T;
    ctx->H = H;
    ctx->stream = (cudaStream_t)cuda_stream;
    cudaGetDevice(&ctx->device);
    cudaDeviceGetAttribute(&ctx->n_sm, cudaDevAttrMultiProcessorCount, ctx->device);

    // re-lay the blob: matrices [out][in] with row stride in+1 (W1 padded to KP columns)
    const int KP = ctx->KP;
    Packer pk;
    const float *src = weights_host;
    auto copy_plain = [&](int64_t n) {
        size_t off = pk.take(n);
        memcpy(pk.buf.data() + off, src, sizeof(float) * n);
        src += n;
        return off;
    };
    auto copy_padded = [&](int rows, int cols, int ld) {
        size_t off = pk.take((size_t)rows * ld);
        for (int r = 0; r < rows; ++r)
            for (int c = 0; c < cols; ++c) pk.buf[off + (size_t)r * ld + c] = src[(size_t)r * cols + c];
        src += (size_t)rows * cols;
        return off;
    };
    size_t o_emb = copy_plain((int64_t)NT * F);
    size_t o_blk[MAX_T][8];
    for (int t = 0; t < T; ++t) {
        o_blk[t][0] = copy_padded(F, K, KP + 1);
        o_blk[t][1] = copy_plain(F);
        o_blk[t][2] = copy_padded(F, F, F + 1);
        o_blk[t][3] = copy_plain(F);
        o_blk[t][4] = copy_padded(F, F, F + 1);
        o_blk[t][5] = copy_plain(F);
        o_blk[t][6] = copy_padded(F, F, F + 1);
        o_blk[t][7] = copy_plain(F);
    }
    size_t o_R1 = copy_padded(H, F, F + 1);
    size_t o_e1 = copy_plain(H);
    size_t o_R2 = copy_plain(H);
    size_t o_e2 = copy_plain(1);
    for (int64_t q = 0; q < n_weights; ++q) {
        if (!isfinite(weights_host[q])) {
            delete ctx;
            return SN_ERR_INVALID_ARG;
        }
    }

    // Per-output-channel scales (SN_PREC_FP16_CH: the row's largest magnitude, 1 for a zero
    // row; every other mode: 1): per block s1, s2, su1, su2 [F], then sr1 [F] (1 past H).
    const bool per_channel = cfg->precision == SN_PREC_FP16_CH;
    auto row_scales = [&](const float *W, int rows, int cols) {
        size_t off = pk.take(F);
        for (int r = 0; r < F; ++r) {
            float m = 0.0f;
            if (per_channel && r < rows)
                for (int c = 0; c < cols; ++c) m = fmaxf(m, fabsf(W[(size_t)r * cols + c]));
            pk.buf[off + r] = m > 0.0f ? m : 1.0f;
        }
        return off;
    };
    size_t o_scale[MAX_T][4];
    for (int t = 0; t < T; ++t) {
        const float *blk = weights_host + (int64_t)NT * F + t * per_block;
        const float *W2 = blk + (int64_t)F * K + F, *U1 = W2 + (int64_t)F * F + F, *U2 = U1 + (int64_t)F * F + F;
        o_scale[t][0] = row_scales(blk, F, K);
        o_scale[t][1] = row_scales(W2, F, F);
        o_scale[t][2] = row_scales(U1, F, F);
        o_scale[t][3] = row_scales(U2, F, F);
    }
    const size_t o_sr1 = row_scales(weights_host + (int64_t)NT * F + T * per_block, H, F);

    // fp16 hi/lo copies of W1 and W2 in the tensor-core operand layout (per block: W1h W1l W2h W2l)
    std::vector<uint16_t> tcw;
    // per block: W1 hi, lo, W2 hi, lo, U1 hi, lo, U2 hi, lo; then R1 (padded to F rows) hi, lo
    const size_t n_w1 = (size_t)F * KP, n_w2 = (size_t)F * F, per_tc = 2 * n_w1 + 6 * n_w2;
    if (cfg->precision != SN_PREC_FP32) {
        tcw.assign(per_tc * T + 2 * n_w2, 0);
        for (int t = 0; t < T; ++t) {
            const float *blk = weights_host + (int64_t)NT * F + t * per_block;
            uint16_t *o = tcw.data() + per_tc * t;
            const float *W2 = blk + (int64_t)F * K + F, *U1 = W2 + (int64_t)F * F + F, *U2 = U1 + (int64_t)F * F + F;
            const float *sc = pk.buf.data();
            sn::tc_pack_matrix(blk, F, K, KP, sc + o_scale[t][0], o, o + n_w1);
            sn::tc_pack_matrix(W2, F, F, F, sc + o_scale[t][1], o + 2 * n_w1, o + 2 * n_w1 + n_w2);
            sn::tc_pack_matrix(U1, F, F, F, sc + o_scale[t][2], o + 2 * n_w1 + 2 * n_w2, o + 2 * n_w1 + 3 * n_w2);
            sn::tc_pack_matrix(U2, F, F, F, sc + o_scale[t][3], o + 2 * n_w1 + 4 * n_w2, o + 2 * n_w1 + 5 * n_w2);
        }
        const float *R1 = weights_host + (int64_t)NT * F + T * per_block;
        uint16_t *o = tcw.data() + per_tc * T;
        sn::tc_pack_matrix(R1, H, F, F, pk.buf.data() + o_sr1, o, o + n_w2);   // rows H..F-1 stay zero
    }

    cudaError_t e = cudaMalloc(&ctx->d_weights, sizeof(float) * pk.buf.size());
    if (e == cudaSuccess && !tcw.empty()) e = cudaMalloc(&ctx->d_tcw, sizeof(uint16_t) * tcw.size());
    if (e == cudaSuccess && !tcw.empty())
        e = cudaMemcpy(ctx->d_tcw, tcw.data(), sizeof(uint16_t) * tcw.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(ctx->d_weights, pk.buf.data(), sizeof(float) * pk.buf.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMalloc(&ctx->d_err, sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(ctx->d_err, 0, sizeof(int));
    if (e == cudaSuccess) e = cudaMallocHost(&ctx->h_err, sizeof(int32_t));
    if (e != cudaSuccess) {
        cudaGetLastError();
        sn_destroy(ctx);
        return SN_ERR_CUDA;
    }
    const float *W = ctx->d_weights;
    sn::Model &m = ctx->model;
    m.F = F;
    m.K = K;
    m.KP = KP;
    m.T = T;
    m.H = H;
    m.n_types = NT;
    m.precision = cfg->precision;
    m.basis.K = K;
    m.basis.KP = KP;
    m.basis.r_cut = cfg->r_cut;
    m.basis.gamma = cfg->gamma;
    m.basis.r_cut_d = (double)cfg->r_cut;
    for (int k = 0; k < 64; ++k) {
        m.basis.mu[k] = k < K ? (double)k * (double)cfg->r_cut / (double)(K - 1) : 0.0;
        m.basis.mu_hi[k] = (float)m.basis.mu[k];
        m.basis.mu_lo[k] = (float)(m.basis.mu[k] - (double)m.basis.mu_hi[k]);
    }
    m.emb = W + o_emb;
    for (int t = 0; t < T; ++t) {
        m.blk[t].W1 = W + o_blk[t][0];
        m.blk[t].b1 = W + o_blk[t][1];
        m.blk[t].W2 = W + o_blk[t][2];
        m.blk[t].b2 = W + o_blk[t][3];
        m.blk[t].U1 = W + o_blk[t][4];
        m.blk[t].c1 = W + o_blk[t][5];
        m.blk[t].U2 = W + o_blk[t][6];
        m.blk[t].c2 = W + o_blk[t][7];
        m.blk[t].s1 = W + o_scale[t][0];
        m.blk[t].s2 = W + o_scale[t][1];
        m.blk[t].su1 = W + o_scale[t][2];
        m.blk[t].su2 = W + o_scale[t][3];
        if (ctx->d_tcw) {
            const uint16_t *o = ctx->d_tcw + per_tc * t;
            m.blk[t].W1h = o;
            m.blk[t].W1l = o + n_w1;
            m.blk[t].W2h = o + 2 * n_w1;
            m.blk[t].W2l = o + 2 * n_w1 + n_w2;
            m.blk[t].U1h = o + 2 * n_w1 + 2 * n_w2;
            m.blk[t].U1l = o + 2 * n_w1 + 3 * n_w2;
            m.blk[t].U2h = o + 2 * n_w1 + 4 * n_w2;
            m.blk[t].U2l = o + 2 * n_w1 + 5 * n_w2;
        }
    }
    m.ro.R1 = W + o_R1;
    m.ro.e1 = W + o_e1;
    m.ro.R2 = W + o_R2;
    m.ro.e2 = W + o_e2;
    m.ro.sr1 = W + o_sr1;
    if (ctx->d_tcw) {
        m.ro.R1h = ctx->d_tcw + per_tc * T;
        m.ro.R1l = ctx->d_tcw + per_tc * T + n_w2;
    }
    *out = ctx;
    return SN_OK;
}

sn_status sn_destroy(sn_ctx *ctx)
{
    if (!ctx) return SN_ERR_INVALID_ARG;
    cudaStreamSynchronize(ctx->stream);
    DevBuf *bufs[] = {&ctx->pos4, &ctx->cnt, &ctx->cell_of, &ctx->cell_cnt, &ctx->cell_start, &ctx->cell_atoms, &ctx->tsum,
                      &ctx->x, &ctx->p, &ctx->h, &ctx->hbar, &ctx->xbar, &ctx->eps, &ctx->part, &ctx->dst,
                      &ctx->md_row_ptr, &ctx->md_col, &ctx->hc_pos, &ctx->hc_vel, &ctx->hc_forces,
                      &ctx->hc_types, &ctx->hc_energy, &ctx->hc_kin};
    for (DevBuf *b : bufs) release(*b);
    for (cudaEvent_t ev : ctx->tracer.ev) cudaEventDestroy(ev);
    if (ctx->d_weights) cudaFree(ctx->d_weights);
    if (ctx->d_tcw) cudaFree(ctx->d_tcw);
    if (ctx->d_err) cudaFree(ctx->d_err);
    if (ctx->h_err) cudaFreeHost(ctx->h_err);
    delete ctx;
    return SN_OK;
}

sn_status sn_set_stream(sn_ctx *ctx, void *cuda_stream)
{
    if (!ctx) return SN_ERR_INVALID_ARG;
    ctx->stream = (cudaStream_t)cuda_stream;
    return SN_OK;
}

sn_status sn_reserve(sn_ctx *ctx, const sn_system *sys, int64_t max_edges)
{
    if (!ctx) return SN_ERR_INVALID_ARG;
    sn_status st;
    if ((st = check_system(ctx, sys))) return st;
    if (max_edges < 0 || max_edges > 0x7fffffffLL) return fail(ctx, SN_ERR_INVALID_ARG, "max_edges out of range");
    const int64_t N = n_atoms(sys);
    if ((st = ensure_ef(ctx, sys))) return st;
    if ((st = grow(ctx, ctx->md_row_ptr, sizeof(int32_t) * (N + 1)))) return st;
    if ((st = grow(ctx, ctx->md_col, sizeof(int32_t) * (size_t)max_edges))) return st;
    ctx->md_cap = (int64_t)(ctx->md_col.bytes / sizeof(int32_t));
    return SN_OK;
}

sn_status sn_build_neighbors(sn_ctx *ctx, const sn_system *sys, const float *pos_dev, int32_t *row_ptr_dev,
                             int32_t *col_dev, int64_t cap, int64_t *n_edges_out)
{
    if (!ctx) return SN_ERR_INVALID_ARG;
    sn_status st;
    if ((st = check_system(ctx, sys))) return st;
    const int64_t N = n_atoms(sys);
    if (!n_edges_out || !row_ptr_dev || (N > 0 && !pos_dev) || cap < 0 || (cap > 0 && !col_dev))
        return fail(ctx, SN_ERR_INVALID_ARG, "NULL argument or negative capacity");
    if ((st = ensure_nb(ctx, sys))) return st;
    sn::NbWork w = nb_work(ctx);
    cudaError_t e = sn::launch_prep_positions(pos_dev, w.pos4, N, ctx->d_err, ctx->stream, &ctx->tracer);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "prep positions");
    int64_t E = 0;
    e = sn::launch_neighbors(*sys, ctx->cfg.r_cut, w.pos4, w, row_ptr_dev, col_dev, cap, ctx->d_err, &E,
                             ctx->stream, &ctx->tracer);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "neighbour kernels");
    *n_edges_out = E;
    if ((st = drain(ctx))) return st;
    if (E > cap) return fail(ctx, SN_ERR_CAPACITY, "neighbour list needs %lld entries, capacity %lld",
                             (long long)E, (long long)cap);
    return SN_OK;
}

sn_status sn_energy_forces(sn_ctx *ctx, const sn_system *sys, const float *pos_dev, const int32_t *types_dev,
                           const int32_t *row_ptr_dev, const int32_t *col_dev, int64_t n_edges, float *energy_dev,
                           float *forces_dev)
{
    if (!ctx) return SN_ERR_INVALID_ARG;
    sn_status st;
    if ((st = check_system(ctx, sys))) return st;
    const int64_t N = n_atoms(sys);
    if (n_edges < 0 || n_edges > 0x7fffffffLL) return fail(ctx, SN_ERR_INVALID_ARG, "n_edges out of range");
    if ((sys->n_replicas > 0 && !energy_dev) || !row_ptr_dev ||
        (N > 0 && (!pos_dev || !types_dev || !forces_dev)) || (n_edges > 0 && !col_dev))
        return fail(ctx, SN_ERR_INVALID_ARG, "NULL argument");
    if ((st = ensure_ef(ctx, sys))) return st;
    if ((st = grow(ctx, ctx->dst, sizeof(int32_t) * (size_t)n_edges))) return st;
    cudaError_t e = sn::launch_prep_positions(pos_dev, (float4 *)ctx->pos4.p, N, ctx->d_err, ctx->stream, &ctx->tracer);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "prep positions");
    return enqueue_ef(ctx, sys, types_dev, row_ptr_dev, col_dev, n_edges, energy_dev, forces_dev);
}

}  // extern "C"

namespace {

struct LangevinParams {
    float a, b;        // O step: v = a v + b xi
    uint64_t seed;
    int64_t step0;
};

// n_steps of velocity Verlet (lv == nullptr) or BAOAB Langevin, rebuilding the list every step
sn_status md_run(sn_ctx *ctx, const sn_system *sys, float *pos_dev, float *vel_dev, float *forces_dev,
                 const int32_t *types_dev, float mass_amu, float dt_fs, int32_t n_steps, float *energy_dev,
                 float *kinetic_dev, const LangevinParams *lv)
{
    sn_status st;
    if ((st = check_system(ctx, sys))) return st;
    const int64_t N = n_atoms(sys);
    if (n_steps < 0 || !(mass_amu > 0.0f) || !isfinite(dt_fs) || isinf(mass_amu))
        return fail(ctx, SN_ERR_INVALID_ARG, "bad n_steps, mass or dt");
    if ((sys->n_replicas > 0 && (!energy_dev || !kinetic_dev)) ||
        (N > 0 && (!pos_dev || !vel_dev || !forces_dev || !types_dev)))
        return fail(ctx, SN_ERR_INVALID_ARG, "NULL argument");
    if ((st = ensure_ef(ctx, sys))) return st;
    if ((st = grow(ctx, ctx->md_row_ptr, sizeof(int32_t) * (N + 1)))) return st;
    if (ctx->md_cap == 0) {
        // size the edge buffer once from the current positions (one synchronisation)
        sn::NbWork w = nb_work(ctx);
        cudaError_t e = sn::launch_prep_positions(pos_dev, w.pos4, N, ctx->d_err, ctx->stream, &ctx->tracer);
        int64_t E = 0;
        if (e == cudaSuccess)
            e = sn::launch_neighbors(*sys, ctx->cfg.r_cut, w.pos4, w, (int32_t *)ctx->md_row_ptr.p, nullptr, 0,
                                     ctx->d_err, &E, ctx->stream, &ctx->tracer);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "sizing neighbour build");
        if ((st = drain(ctx))) return st;
        if ((st = grow(ctx, ctx->md_col, sizeof(int32_t) * (size_t)(E + E / 2 + 1024)))) return st;
        ctx->md_cap = (int64_t)(ctx->md_col.bytes / sizeof(int32_t));
    }
    if ((st = grow(ctx, ctx->dst, sizeof(int32_t) * (size_t)ctx->md_cap))) return st;
    ctx->md_last_N = N;
    const float c = 0.5f * dt_fs * KAPPA / mass_amu;
    sn::NbWork w = nb_work(ctx);
    int32_t *rp = (int32_t *)ctx->md_row_ptr.p;
    int32_t *cl = (int32_t *)ctx->md_col.p;
    for (int s = 0; s < n_steps; ++s) {
        cudaError_t e;
        if (lv)
            e = sn::launch_langevin_baoa(pos_dev, vel_dev, forces_dev, N, c, dt_fs, lv->a, lv->b, lv->seed,
                                         lv->step0 + s, w.pos4, ctx->d_err, ctx->stream, &ctx->tracer);
        else
            e = sn::launch_kick_drift(pos_dev, vel_dev, forces_dev, N, c, dt_fs, w.pos4, ctx->d_err, ctx->stream,
                                      &ctx->tracer);
        if (e == cudaSuccess)
            e = sn::launch_neighbors(*sys, ctx->cfg.r_cut, w.pos4, w, rp, cl, ctx->md_cap, ctx->d_err, nullptr,
                                     ctx->stream, &ctx->tracer);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "md step: drift / neighbours");
        sn::EfWork ew = ef_work(ctx);
        ew.col_cap = ctx->md_cap;
        e = sn::launch_energy_forces(ctx->model, *sys, geometry(sys), types_dev, rp, cl, ew, nullptr, forces_dev,
                                     ctx->d_err, ctx->stream, &ctx->tracer);
        if (e == cudaSuccess) e = sn::launch_kick(vel_dev, forces_dev, 3 * N, c, ctx->d_err, ctx->stream, &ctx->tracer);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "md step: forces / kick");
    }
    cudaError_t e = sn::launch_replica_sums((const float *)ctx->eps.p, vel_dev, sys->n_per_replica, sys->n_replicas,
                                            0.5f * mass_amu / KAPPA, n_steps > 0 ? energy_dev : nullptr,
                                            kinetic_dev, ctx->d_err, ctx->stream, &ctx->tracer);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "md step: replica sums");
    return SN_OK;
}

}  // namespace

extern "C" {

sn_status sn_md_step(sn_ctx *ctx, const sn_system *sys, float *pos_dev, float *vel_dev, float *forces_dev,
                     const int32_t *types_dev, float mass_amu, float dt_fs, int32_t n_steps, float *energy_dev,
                     float *kinetic_dev)
{
    if (!ctx) return SN_ERR_INVALID_ARG;
    return md_run(ctx, sys, pos_dev, vel_dev, forces_dev, types_dev, mass_amu, dt_fs, n_steps, energy_dev,
                  kinetic_dev, nullptr);
}

sn_status sn_md_langevin(sn_ctx *ctx, const sn_system *sys, float *pos_dev, float *vel_dev, float *forces_dev,
                         const int32_t *types_dev, float mass_amu, float dt_fs, int32_t n_steps, float temperature_k,
                         float friction_per_fs, uint64_t seed, int64_t step0, float *energy_dev, float *kinetic_dev)
{
    if (!ctx) return SN_ERR_INVALID_ARG;
    if (!(temperature_k >= 0.0f) || isinf(temperature_k) || !(friction_per_fs >= 0.0f) || isinf(friction_per_fs) ||
        step0 < 0 || !(mass_amu > 0.0f))
        return fail(ctx, SN_ERR_INVALID_ARG, "bad temperature, friction, step0 or mass");
    const double kB = 0.0019872041;   // kcal/mol/K
    const double a = exp(-(double)friction_per_fs * (double)dt_fs);
    LangevinParams lv;
    lv.a = (float)a;
    lv.b = (float)sqrt((1.0 - a * a) * kB * (double)temperature_k * (double)KAPPA / (double)mass_amu);
    lv.seed = seed;
    lv.step0 = step0;
    return md_run(ctx, sys, pos_dev, vel_dev, forces_dev, types_dev, mass_amu, dt_fs, n_steps, energy_dev,
                  kinetic_dev, &lv);
}

sn_status sn_md_step_host(sn_ctx *ctx, const sn_system *sys, float *pos_host, float *vel_host, float *forces_host,
                          const int32_t *types_host, float mass_amu, float dt_fs, int32_t n_steps, float *energy_host,
                          float *kinetic_host)
{
    if (!ctx) return SN_ERR_INVALID_ARG;
    sn_status st;
    if ((st = check_system(ctx, sys))) return st;
    const int64_t N = n_atoms(sys), R = sys->n_replicas;
    if ((R > 0 && (!energy_host || !kinetic_host)) || (N > 0 && (!pos_host || !vel_host || !forces_host || !types_host)))
        return fail(ctx, SN_ERR_INVALID_ARG, "NULL argument");
    const size_t b3 = sizeof(float) * 3 * N;
    if ((st = grow(ctx, ctx->hc_pos, b3)) || (st = grow(ctx, ctx->hc_vel, b3)) || (st = grow(ctx, ctx->hc_forces, b3)) ||
        (st = grow(ctx, ctx->hc_types, sizeof(int32_t) * N)) || (st = grow(ctx, ctx->hc_energy, sizeof(float) * R)) ||
        (st = grow(ctx, ctx->hc_kin, sizeof(float) * R)))
        return st;
    cudaStream_t s = ctx->stream;
    SN_CUDA(cudaMemcpyAsync(ctx->hc_pos.p, pos_host, b3, cudaMemcpyHostToDevice, s));
    SN_CUDA(cudaMemcpyAsync(ctx->hc_vel.p, vel_host, b3, cudaMemcpyHostToDevice, s));
    SN_CUDA(cudaMemcpyAsync(ctx->hc_forces.p, forces_host, b3, cudaMemcpyHostToDevice, s));
    SN_CUDA(cudaMemcpyAsync(ctx->hc_types.p, types_host, sizeof(int32_t) * N, cudaMemcpyHostToDevice, s));
    st = sn_md_step(ctx, sys, (float *)ctx->hc_pos.p, (float *)ctx->hc_vel.p, (float *)ctx->hc_forces.p,
                    (const int32_t *)ctx->hc_types.p, mass_amu, dt_fs, n_steps, (float *)ctx->hc_energy.p,
                    (float *)ctx->hc_kin.p);
    if (st) return st;
    SN_CUDA(cudaMemcpyAsync(pos_host, ctx->hc_pos.p, b3, cudaMemcpyDeviceToHost, s));
    SN_CUDA(cudaMemcpyAsync(vel_host, ctx->hc_vel.p, b3, cudaMemcpyDeviceToHost, s));
    SN_CUDA(cudaMemcpyAsync(forces_host, ctx->hc_forces.p, b3, cudaMemcpyDeviceToHost, s));
    SN_CUDA(cudaMemcpyAsync(energy_host, ctx->hc_energy.p, sizeof(float) * R, cudaMemcpyDeviceToHost, s));
    SN_CUDA(cudaMemcpyAsync(kinetic_host, ctx->hc_kin.p, sizeof(float) * R, cudaMemcpyDeviceToHost, s));
    return drain(ctx);
}

sn_status sn_sync(sn_ctx *ctx)
{
    if (!ctx) return SN_ERR_INVALID_ARG;
    return drain(ctx);
}

sn_status sn_set_wait_limit(sn_ctx *ctx, int64_t cycles)
{
    if (!ctx) return SN_ERR_INVALID_ARG;
    if (cycles < 0) return fail(ctx, SN_ERR_INVALID_ARG, "negative wait limit");
    ctx->wait_limit = cycles == 0 ? (1ll << 32) : (long long)cycles;
    return SN_OK;
}

sn_status sn_trace_enable(sn_ctx *ctx, int32_t on)
{
    if (!ctx) return SN_ERR_INVALID_ARG;
    ctx->tracer.on = on != 0;
    ctx->tracer.n = 0;
    return SN_OK;
}

int32_t sn_trace_read(sn_ctx *ctx, sn_trace_entry *out, int32_t max_entries)
{
    static const char *names[sn::KK_COUNT] = {"prep_positions", "neighbor_count", "neighbor_fill", "scan",
                                              "cell_bin",       "partition",      "edge_fwd",      "node_fwd",
                                              "edge_bwd",       "node_bwd",       "replica_sums",  "kick_drift",
                                              "kick"};
    if (!ctx || max_entries < 0 || (max_entries > 0 && !out)) return -1;
    if (cudaStreamSynchronize(ctx->stream) != cudaSuccess) return -1;
    double ms[sn::KK_COUNT] = {0};
    int64_t cnt[sn::KK_COUNT] = {0};
    sn::Tracer &tr = ctx->tracer;
    for (size_t q = 0; q < tr.n; ++q) {
        float t = 0.0f;
        if (cudaEventElapsedTime(&t, tr.ev[2 * q], tr.ev[2 * q + 1]) != cudaSuccess) return -1;
        ms[tr.kinds[q]] += t;
        cnt[tr.kinds[q]] += 1;
    }
    tr.n = 0;
    int32_t w = 0;
    for (int k = 0; k < sn::KK_COUNT; ++k) {
        if (!cnt[k]) continue;
        if (w < max_entries) {
            out[w].name = names[k];
            out[w].launches = cnt[k];
            out[w].total_ms = ms[k];
        }
        ++w;
    }
    return w;
}

int64_t sn_md_edges(sn_ctx *ctx)
{
    if (!ctx || !ctx->md_row_ptr.p) return -1;
    int32_t E = -1;
    if (cudaMemcpyAsync(ctx->h_err, (int32_t *)ctx->md_row_ptr.p + ctx->md_last_N, sizeof(int32_t),
                        cudaMemcpyDeviceToHost, ctx->stream) != cudaSuccess)
        return -1;
    if (cudaStreamSynchronize(ctx->stream) != cudaSuccess) return -1;
    E = *ctx->h_err;
    return E;
}

}  // extern "C"
