// selinv_chain_noalloc: the b <= 16 chain path with its scratch in a
// fixed-size device array owned by the library, for callers that cannot
// allocate device memory themselves.
//
// Who needs it: code that runs inside another framework's execution hook --
// an inference-engine plugin's enqueue, a compiler runtime's custom call, a
// real-time loop with a fixed memory budget -- where the host framework owns
// all device memory and a cudaMalloc is either forbidden, fails, or would
// synchronise the device and stall every other stream.  Those callers still
// provide inputs and outputs; this entry point needs nothing else.
//
// The scratch below is a file-scope device array: every GPU that loads this
// library holds NOALLOC_SCRATCH_BYTES of it until the process exits.  Host
// code only ever sees a host-side stand-in for its name, so the device address
// is looked up once per device with cudaGetSymbolAddress (with that device
// current) and passed to the kernel.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = SELINV_CHAIN_NOALLOC_MAX_BYTES;   // 16 MiB per device
constexpr int MAX_DEVICES = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
void *g_scratch_ptr[MAX_DEVICES] = {};

// Device address of the scratch array on the current device (set up on the
// first call per device).  Returns nullptr on failure.
void *scratch_for_current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

bool aligned_to(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

template <class T>
selinv_status run(int64_t batch, int64_t L, int32_t b, const void *diag, const void *lower, void *G_diag,
                  void *G_lower, double *logdet, const void *rhs, void *x, int32_t *info, void *scratch,
                  cudaStream_t s)
{
    selinv::ChainArgs<T> a;
    a.diag = static_cast<const T *>(diag);
    a.lower = static_cast<const T *>(lower);
    a.G_diag = static_cast<T *>(G_diag);
    a.G_lower = static_cast<T *>(G_lower);
    a.logdet = logdet;
    a.rhs = static_cast<const T *>(rhs);
    a.x = static_cast<T *>(x);
    a.info = info;
    a.ws = static_cast<T *>(scratch);
    a.batch = batch;
    a.L = L;
    a.b = b;
    const bool al = aligned_to(diag, 16) && aligned_to(lower, 16) && aligned_to(G_diag, 16) &&
                    aligned_to(G_lower, 16);
    return selinv::chain_small_launch<T>(a, al, s) == cudaSuccess ? SELINV_OK : SELINV_ERR_CUDA;
}

}  // namespace

extern "C" {

selinv_status selinv_chain_noalloc(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b, const void *diag,
                                   const void *lower, void *G_diag, void *G_lower, double *logdet,
                                   const void *rhs, void *x, int32_t *info, void *stream)
{
    if ((dtype != SELINV_F64 && dtype != SELINV_F32) || batch < 0 || L < 1 || b < 1)
        return SELINV_ERR_INVALID_ARG;
    if (b > 16) return SELINV_ERR_UNSUPPORTED;
    if (batch > 0 && (!diag || !info || (L > 1 && !lower))) return SELINV_ERR_INVALID_ARG;
    const size_t es = dtype == SELINV_F64 ? 8 : 4;
    const bool want_g = G_diag != nullptr, want_x = rhs != nullptr;
    if (want_g && L > 1 && G_lower == nullptr) return SELINV_ERR_INVALID_ARG;
    if (!want_g && G_lower != nullptr) return SELINV_ERR_INVALID_ARG;
    if ((rhs == nullptr) != (x == nullptr)) return SELINV_ERR_INVALID_ARG;
    if (!aligned_to(diag, es) || !aligned_to(lower, es) || !aligned_to(G_diag, es) ||
        !aligned_to(G_lower, es) || !aligned_to(rhs, es) || !aligned_to(x, es) || !aligned_to(logdet, 8) ||
        !aligned_to(info, 4))
        return SELINV_ERR_INVALID_ARG;
    // Scratch is batch * (L-1) slots of 192 elements when G or x is asked for.
    // Compared by division so that a huge batch or L cannot wrap the product
    // below the limit.
    if ((want_g || want_x) && L > 1 && batch > 0) {
        const size_t per_chain_limit = NOALLOC_SCRATCH_BYTES / (192 * es);     // slots that fit
        if ((uint64_t)(L - 1) > per_chain_limit || (uint64_t)batch > per_chain_limit / (uint64_t)(L - 1))
            return SELINV_ERR_WORKSPACE;                                    // beyond the built-in scratch
        if (selinv::chain_small_workspace(es, batch, L) > NOALLOC_SCRATCH_BYTES) return SELINV_ERR_WORKSPACE;
    }
    if (batch == 0) return SELINV_OK;
    void *scratch = scratch_for_current_device();
    if (scratch == nullptr) return SELINV_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == SELINV_F64)
        return run<double>(batch, L, b, diag, lower, G_diag, G_lower, logdet, rhs, x, info, scratch, s);
    return run<float>(batch, L, b, diag, lower, G_diag, G_lower, logdet, rhs, x, info, scratch, s);
}

}  // extern "C"
