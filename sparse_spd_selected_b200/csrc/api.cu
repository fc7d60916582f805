// C ABI of libselinv: argument validation, workspace sizing and kernel
// dispatch.  Declarations and the full contract are in include/selinv.h.
#include <stdint.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

using namespace selinv;

namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t elem_size(selinv_dtype d) { return d == SELINV_F64 ? 8 : 4; }

bool valid_dtype(selinv_dtype d) { return d == SELINV_F64 || d == SELINV_F32; }

constexpr int32_t MAX_BLOCK = 128;
constexpr size_t WS_ALIGN = 256;

size_t round_up(size_t x) { return (x + WS_ALIGN - 1) / WS_ALIGN * WS_ALIGN; }

selinv_status chain_check(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b, const void *diag,
                          const void *lower, int32_t *info)
{
    if (!valid_dtype(dtype) || batch < 0 || L < 1 || b < 1) return SELINV_ERR_INVALID_ARG;
    if (b > MAX_BLOCK) return SELINV_ERR_UNSUPPORTED;
    if (batch > 0 && (!diag || !info || (L > 1 && !lower))) return SELINV_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    if (!aligned(diag, es) || !aligned(lower, es) || !aligned(info, 4)) return SELINV_ERR_INVALID_ARG;
    return SELINV_OK;
}

selinv_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SELINV_OK : SELINV_ERR_CUDA; }

template <class T>
selinv_status run_chain(int64_t batch, int64_t L, int32_t b, const void *diag, const void *lower,
                        void *G_diag, void *G_lower, double *logdet, const void *rhs, void *x,
                        int32_t *info, void *ws, cudaStream_t s)
{
    ChainArgs<T> a;
    a.diag = static_cast<const T *>(diag);
    a.lower = static_cast<const T *>(lower);
    a.G_diag = static_cast<T *>(G_diag);
    a.G_lower = static_cast<T *>(G_lower);
    a.logdet = logdet;
    a.rhs = static_cast<const T *>(rhs);
    a.x = static_cast<T *>(x);
    a.info = info;
    a.ws = static_cast<T *>(ws);
    a.batch = batch;
    a.L = L;
    a.b = b;
    if constexpr (std::is_same<T, double>::value) {
        if (chain_tiny_fits(L, b)) return from_cuda(chain_tiny_launch(a, s));
    }
    if (b <= 16) {
        const bool al = aligned(diag, 16) && aligned(lower, 16) && aligned(G_diag, 16) &&
                        aligned(G_lower, 16) && aligned(ws, 16);
        return from_cuda(chain_small_launch<T>(a, al, s));
    }
    if (b <= 32 && rhs == nullptr) {
        const int P = chain_seg_parts(batch, L, b, G_diag != nullptr, false);
        if (P > 0) return from_cuda(chain_seg_launch<T>(a, P, s));
        return from_cuda(chain_mid_launch<T>(a, s));
    }
    return from_cuda(chain_large_launch<T>(a, s));
}

// SELINV_CHECK for a chain call: D_i (lower triangles), B_i and r_i finite.
template <class T>
selinv_status check_chain(int64_t batch, int64_t L, int32_t b, const void *diag, const void *lower,
                          const void *rhs, int32_t *info, cudaStream_t s)
{
    cudaError_t e = check_finite_launch<T>(static_cast<const T *>(diag), batch, L, b, 0, nullptr, info, s);
    if (e == cudaSuccess && L > 1)
        e = check_finite_launch<T>(static_cast<const T *>(lower), batch, L - 1, b, 1, nullptr, info, s);
    if (e == cudaSuccess && rhs)
        e = check_finite_launch<T>(static_cast<const T *>(rhs), batch, L, b, 2, nullptr, info, s);
    if (e == cudaSuccess) e = check_finalize_launch(info, batch, L, s);
    return from_cuda(e);
}

size_t chain_ws(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b, bool want_g, bool want_x)
{
    if (!want_g && !want_x) return 0;
    const size_t es = elem_size(dtype);
    if (b <= 16) return round_up(chain_small_workspace(es, batch, L));
    if (b <= 32 && !want_x) {
        const int P = chain_seg_parts(batch, L, b, want_g, want_x);
        if (P > 0) return round_up(chain_seg_workspace(es, batch, L, b, P, want_g));
        return round_up(chain_mid_workspace(es, batch, L));
    }
    return round_up(chain_large_workspace(es, batch, L, b));
}

}  // namespace

extern "C" {

const char *selinv_status_string(selinv_status s)
{
    switch (s) {
    case SELINV_OK: return "ok";
    case SELINV_ERR_INVALID_ARG: return "invalid argument";
    case SELINV_ERR_NOT_SPD: return "matrix not positive definite";
    case SELINV_ERR_BAD_TREE: return "parent array is not one rooted tree per slot";
    case SELINV_ERR_CUDA: return "CUDA error";
    case SELINV_ERR_WORKSPACE: return "workspace too small";
    case SELINV_ERR_UNSUPPORTED: return "block size not supported";
    case SELINV_ERR_HOST_MEMORY: return "host memory exhausted";
    case SELINV_ERR_TIMEOUT: return "a dependency wait of a tree sweep gave up";
    }
    return "unknown status";
}

int32_t selinv_version(void) { return 100; }

int32_t selinv_max_block(void) { return MAX_BLOCK; }

int32_t selinv_chain_segments(int64_t batch, int64_t L, int32_t b, int32_t want_g, int32_t want_x)
{
    if (batch < 0 || L < 1 || b < 1 || b > MAX_BLOCK) return 0;
    return chain_seg_parts(batch, L, b, want_g != 0, want_x != 0);
}

size_t selinv_chain_workspace_size(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b,
                                   int32_t want_g, int32_t want_x)
{
    if (!valid_dtype(dtype) || batch < 0 || L < 1 || b < 1 || b > MAX_BLOCK) return 0;
    return chain_ws(dtype, batch, L, b, want_g != 0, want_x != 0);
}

selinv_status selinv_chain(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b, const void *diag,
                           const void *lower, void *G_diag, void *G_lower, double *logdet,
                           const void *rhs, void *x, int32_t *info, void *workspace,
                           size_t workspace_bytes, uint32_t flags, void *stream)
{
    selinv_status st = chain_check(dtype, batch, L, b, diag, lower, info);
    if (st != SELINV_OK) return st;
    if (flags & ~(uint32_t)(SELINV_WANT_LOGDET | SELINV_WANT_SOLVE | SELINV_CHECK)) return SELINV_ERR_INVALID_ARG;
    if ((flags & SELINV_WANT_LOGDET) && logdet == nullptr) return SELINV_ERR_INVALID_ARG;
    if ((flags & SELINV_WANT_SOLVE) && (rhs == nullptr || x == nullptr)) return SELINV_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    const bool want_g = G_diag != nullptr;
    const bool want_x = rhs != nullptr;
    if (want_g && L > 1 && G_lower == nullptr) return SELINV_ERR_INVALID_ARG;
    if (!want_g && G_lower != nullptr) return SELINV_ERR_INVALID_ARG;
    if ((rhs == nullptr) != (x == nullptr)) return SELINV_ERR_INVALID_ARG;
    if (!aligned(G_diag, es) || !aligned(G_lower, es) || !aligned(rhs, es) || !aligned(x, es) ||
        !aligned(logdet, 8) || !aligned(workspace, 16))
        return SELINV_ERR_INVALID_ARG;
    const size_t need = chain_ws(dtype, batch, L, b, want_g, want_x);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return SELINV_ERR_WORKSPACE;
    if (batch == 0) return SELINV_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = dtype == SELINV_F64 ? run_chain<double>(batch, L, b, diag, lower, G_diag, G_lower, logdet, rhs, x, info,
                                                 workspace, s)
                             : run_chain<float>(batch, L, b, diag, lower, G_diag, G_lower, logdet, rhs, x, info,
                                                workspace, s);
    if (st != SELINV_OK || !(flags & SELINV_CHECK)) return st;
    return dtype == SELINV_F64
               ? check_chain<double>(batch, L, b, diag, lower, rhs, info, s)
               : check_chain<float>(batch, L, b, diag, lower, rhs, info, s);
}

selinv_status selinv_chain_sample(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b, const void *diag,
                                  const void *lower, const void *rhs, const void *z, void *eta, double *logdet,
                                  int32_t *info, void *workspace, size_t workspace_bytes, void *stream)
{
    selinv_status st = chain_check(dtype, batch, L, b, diag, lower, info);
    if (st != SELINV_OK) return st;
    if (b > 16 && dtype != SELINV_F64) return SELINV_ERR_UNSUPPORTED;
    const size_t es = elem_size(dtype);
    if (batch > 0 && (z == nullptr || eta == nullptr)) return SELINV_ERR_INVALID_ARG;
    if (!aligned(rhs, es) || !aligned(z, es) || !aligned(eta, es) || !aligned(logdet, 8) ||
        !aligned(workspace, 16))
        return SELINV_ERR_INVALID_ARG;
    const size_t need = chain_ws(dtype, batch, L, b, false, true);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return SELINV_ERR_WORKSPACE;
    if (batch == 0) return SELINV_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool al = aligned(diag, 16) && aligned(lower, 16) && aligned(workspace, 16);
    if (dtype == SELINV_F64) {
        ChainArgs<double> a;
        a.diag = static_cast<const double *>(diag);
        a.lower = static_cast<const double *>(lower);
        a.G_diag = a.G_lower = nullptr;
        a.logdet = logdet;
        a.rhs = static_cast<const double *>(rhs);
        a.x = static_cast<double *>(eta);
        a.z = static_cast<const double *>(z);
        a.info = info;
        a.ws = static_cast<double *>(workspace);
        a.batch = batch;
        a.L = L;
        a.b = b;
        if (b > 16) return from_cuda(chain_large_sample_launch(a, s));
        return from_cuda(chain_small_sample_launch<double>(a, al, s));
    }
    ChainArgs<float> a;
    a.diag = static_cast<const float *>(diag);
    a.lower = static_cast<const float *>(lower);
    a.G_diag = a.G_lower = nullptr;
    a.logdet = logdet;
    a.rhs = static_cast<const float *>(rhs);
    a.x = static_cast<float *>(eta);
    a.z = static_cast<const float *>(z);
    a.info = info;
    a.ws = static_cast<float *>(workspace);
    a.batch = batch;
    a.L = L;
    a.b = b;
    return from_cuda(chain_small_sample_launch<float>(a, al, s));
}

selinv_status selinv_bidiag(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b, const void *diag,
                            const void *lower, void *G_diag, void *G_lower, int32_t *info, void *stream)
{
    selinv_status st = chain_check(dtype, batch, L, b, diag, lower, info);
    if (st != SELINV_OK) return st;
    if (b > 16) return SELINV_ERR_UNSUPPORTED;
    const size_t es = elem_size(dtype);
    if (batch > 0 && (!G_diag || (L > 1 && !G_lower))) return SELINV_ERR_INVALID_ARG;
    if (!aligned(G_diag, es) || !aligned(G_lower, es)) return SELINV_ERR_INVALID_ARG;
    if (batch == 0) return SELINV_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool al = aligned(diag, 16) && aligned(lower, 16) && aligned(G_diag, 16) && aligned(G_lower, 16);
    if (dtype == SELINV_F64) {
        BidiagArgs<double> p{static_cast<const double *>(diag), static_cast<const double *>(lower),
                             static_cast<double *>(G_diag), static_cast<double *>(G_lower), info, batch, L, b};
        return from_cuda(bidiag_launch<double>(p, al, s));
    }
    BidiagArgs<float> p{static_cast<const float *>(diag), static_cast<const float *>(lower),
                        static_cast<float *>(G_diag), static_cast<float *>(G_lower), info, batch, L, b};
    return from_cuda(bidiag_launch<float>(p, al, s));
}

selinv_status selinv_bidiag_backward(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b, const void *G_diag,
                                     const void *G_lower, const void *Gb_diag, const void *Gb_lower, void *Mb_diag,
                                     void *Mb_lower, void *stream)
{
    if (!valid_dtype(dtype) || batch < 0 || L < 1 || b < 1) return SELINV_ERR_INVALID_ARG;
    if (b > 16) return SELINV_ERR_UNSUPPORTED;
    if (batch > 0 && (!G_diag || !Mb_diag || (L > 1 && (!G_lower || !Mb_lower)))) return SELINV_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    if (!aligned(G_diag, es) || !aligned(G_lower, es) || !aligned(Gb_diag, es) || !aligned(Gb_lower, es) ||
        !aligned(Mb_diag, es) || !aligned(Mb_lower, es))
        return SELINV_ERR_INVALID_ARG;
    if (batch == 0) return SELINV_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool al = aligned(G_diag, 16) && aligned(G_lower, 16) && aligned(Gb_diag, 16) && aligned(Gb_lower, 16) &&
                    aligned(Mb_diag, 16) && aligned(Mb_lower, 16);
    if (dtype == SELINV_F64) {
        BidiagBwdArgs<double> a{static_cast<const double *>(G_diag), static_cast<const double *>(G_lower),
                                static_cast<const double *>(Gb_diag), static_cast<const double *>(Gb_lower),
                                static_cast<double *>(Mb_diag), static_cast<double *>(Mb_lower), batch, L, b};
        return from_cuda(bidiag_backward_launch<double>(a, al, s));
    }
    BidiagBwdArgs<float> a{static_cast<const float *>(G_diag), static_cast<const float *>(G_lower),
                           static_cast<const float *>(Gb_diag), static_cast<const float *>(Gb_lower),
                           static_cast<float *>(Mb_diag), static_cast<float *>(Mb_lower), batch, L, b};
    return from_cuda(bidiag_backward_launch<float>(a, al, s));
}

size_t selinv_chain_backward_workspace_size(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b)
{
    if (!valid_dtype(dtype) || batch < 0 || L < 1 || b < 1 || b > 16) return 0;
    return round_up(chain_backward_workspace(elem_size(dtype), batch, L));
}

selinv_status selinv_chain_backward(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b, const void *diag,
                                    const void *lower, const void *G_diag, const void *G_lower, const void *Gb_diag,
                                    const void *Gb_lower, void *Db, void *Bb, int32_t *info, void *workspace,
                                    size_t workspace_bytes, void *stream)
{
    selinv_status st = chain_check(dtype, batch, L, b, diag, lower, info);
    if (st != SELINV_OK) return st;
    if (b > 16) return SELINV_ERR_UNSUPPORTED;
    const size_t es = elem_size(dtype);
    if (batch > 0 && (!G_diag || !Db || (L > 1 && (!G_lower || !Bb))))
        return SELINV_ERR_INVALID_ARG;
    if (!aligned(G_diag, es) || !aligned(G_lower, es) || !aligned(Gb_diag, es) || !aligned(Gb_lower, es) ||
        !aligned(Db, es) || !aligned(Bb, es) || !aligned(workspace, 16))
        return SELINV_ERR_INVALID_ARG;
    const size_t need = selinv_chain_backward_workspace_size(dtype, batch, L, b);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return SELINV_ERR_WORKSPACE;
    if (batch == 0) return SELINV_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool al = aligned(diag, 16) && aligned(lower, 16) && aligned(G_diag, 16) && aligned(G_lower, 16) &&
                    aligned(Gb_diag, 16) && aligned(Gb_lower, 16) && aligned(Db, 16) && aligned(Bb, 16);
    auto fill = [&](auto &a, auto *tag) {
        using T = std::remove_pointer_t<decltype(tag)>;
        a.diag = static_cast<const T *>(diag);
        a.lower = static_cast<const T *>(lower);
        a.G_diag = static_cast<const T *>(G_diag);
        a.G_lower = static_cast<const T *>(G_lower);
        a.Gb_diag = static_cast<const T *>(Gb_diag);
        a.Gb_lower = static_cast<const T *>(Gb_lower);
        a.Db = static_cast<T *>(Db);
        a.Bb = static_cast<T *>(Bb);
        a.info = info;
        a.ws = static_cast<T *>(workspace);
        a.batch = batch;
        a.L = L;
        a.b = b;
    };
    if (dtype == SELINV_F64) {
        ChainBwdArgs<double> a;
        fill(a, (double *)nullptr);
        return from_cuda(chain_backward_launch<double>(a, al, s));
    }
    ChainBwdArgs<float> a;
    fill(a, (float *)nullptr);
    return from_cuda(chain_backward_launch<float>(a, al, s));
}

selinv_status chain_solve_multi(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b, int32_t nrhs,
                                const void *diag, const void *lower, const void *rhs, void *x, double *logdet,
                                int32_t *info, void *workspace, size_t workspace_bytes, void *stream)
{
    selinv_status st = chain_check(dtype, batch, L, b, diag, lower, info);
    if (st != SELINV_OK) return st;
    if (nrhs < 1) return SELINV_ERR_INVALID_ARG;
    if (b > 16) return SELINV_ERR_UNSUPPORTED;
    const size_t es = elem_size(dtype);
    if (batch > 0 && (rhs == nullptr || x == nullptr)) return SELINV_ERR_INVALID_ARG;
    if (!aligned(rhs, es) || !aligned(x, es) || !aligned(logdet, 8) || !aligned(workspace, 16))
        return SELINV_ERR_INVALID_ARG;
    const size_t need = chain_ws(dtype, batch, L, b, false, true);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return SELINV_ERR_WORKSPACE;
    if (batch == 0) return SELINV_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool al = aligned(diag, 16) && aligned(lower, 16) && aligned(workspace, 16);
    for (int32_t c0 = 0; c0 < nrhs; c0 += 16) {
        cudaError_t err;
        if (dtype == SELINV_F64) {
            ChainArgs<double> a;
            a.diag = static_cast<const double *>(diag);
            a.lower = static_cast<const double *>(lower);
            a.G_diag = a.G_lower = nullptr;
            a.logdet = logdet;
            a.rhs = static_cast<const double *>(rhs);
            a.x = static_cast<double *>(x);
            a.info = info;
            a.ws = static_cast<double *>(workspace);
            a.batch = batch;
            a.L = L;
            a.b = b;
            a.nrhs = nrhs;
            a.c0 = c0;
            err = chain_small_multi_launch<double>(a, al, s);
        } else {
            ChainArgs<float> a;
            a.diag = static_cast<const float *>(diag);
            a.lower = static_cast<const float *>(lower);
            a.G_diag = a.G_lower = nullptr;
            a.logdet = logdet;
            a.rhs = static_cast<const float *>(rhs);
            a.x = static_cast<float *>(x);
            a.info = info;
            a.ws = static_cast<float *>(workspace);
            a.batch = batch;
            a.L = L;
            a.b = b;
            a.nrhs = nrhs;
            a.c0 = c0;
            err = chain_small_multi_launch<float>(a, al, s);
        }
        if (err != cudaSuccess) return SELINV_ERR_CUDA;
    }
    return SELINV_OK;
}

selinv_status chain_solve(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b, const void *diag,
                          const void *lower, const void *rhs, void *x, double *logdet, int32_t *info,
                          void *workspace, size_t workspace_bytes, void *stream)
{
    if (rhs == nullptr || x == nullptr) return batch == 0 ? SELINV_OK : SELINV_ERR_INVALID_ARG;
    return selinv_chain(dtype, batch, L, b, diag, lower, nullptr, nullptr, logdet, rhs, x, info,
                        workspace, workspace_bytes, 0u, stream);
}

}  // extern "C"
