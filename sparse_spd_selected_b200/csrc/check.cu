// SELINV_CHECK: on-device validation of the inputs of selinv_chain and
// selinv_tree (gabp-sparse-inv 0.3.2, "Quickstart": the check=True option
// validates the input before trusting the result; sparsax "Features": bad input
// is an error, not a silent result).  Every entry the call reads -- the lower
// triangle of each diagonal block, every entry of each off-diagonal block
// (trees: every non-root edge slot), every entry of the right-hand side -- must
// be finite.  The kernels run after the selected-inverse kernels on the same
// stream and overwrite info[e] with -3 - k, k the first block (chain: block
// index i of D_i, B_i = lower[i] or r_i; tree: node v) holding a non-finite
// entry.  Nothing traps; outputs of such an element are unspecified.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace selinv {

namespace {

// Entries not yet finalised are INT_MIN / 2 + k (below every code the
// selected-inverse kernels write: -2, -1, k >= 0), so atomicMin keeps the
// smallest block index and beats a pivot failure that the bad entry caused.
constexpr int32_t CHECK_BASE = INT_MIN / 2;

// blocks [batch, nb, m]: m = b * b (kind 0: lower triangle of diagonal
// blocks, kind 1: whole blocks) or m = b (kind 2: vectors).  parent (trees):
// node e * nb + blk is skipped when it is a root (its edge slot is not read).
template <class T>
__global__ void check_finite_kernel(const T *a, int64_t batch, int64_t nb, int b, int kind, const int32_t *parent,
                                    int32_t *info)
{
    const int64_t m = kind == 2 ? b : (int64_t)b * b;
    const int64_t total = batch * nb * m;
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < total;
         j += (int64_t)gridDim.x * blockDim.x) {
        const int64_t w = j % m;
        if (kind == 0 && (w % b) > (w / b)) continue;          // upper triangle: not read
        const int64_t eb = j / m;                              // e * nb + blk
        if (parent && parent[eb] < 0) continue;                // a root's edge slot: not read
        const T v = a[j];
        if (!isfinite(v)) atomicMin(info + eb / nb, CHECK_BASE + (int32_t)(eb % nb));
    }
}

__global__ void check_finalize_kernel(int32_t *info, int64_t batch, int64_t nb)
{
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= batch) return;
    const int32_t v = info[e];
    if (v >= CHECK_BASE && v < CHECK_BASE + nb) info[e] = -3 - (v - CHECK_BASE);
}

int grid_for(int64_t total)
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (total + 255) / 256;
    const int64_t cap = (int64_t)sms * 8;
    return (int)(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

template <class T>
cudaError_t check_finite_launch(const T *a, int64_t batch, int64_t nb, int b, int kind, const int32_t *parent,
                                int32_t *info, cudaStream_t s)
{
    if (!a || batch <= 0 || nb <= 0) return cudaSuccess;
    const int64_t total = batch * nb * (kind == 2 ? b : (int64_t)b * b);
    check_finite_kernel<T><<<grid_for(total), 256, 0, s>>>(a, batch, nb, b, kind, parent, info);
    return cudaGetLastError();
}

cudaError_t check_finalize_launch(int32_t *info, int64_t batch, int64_t nb, cudaStream_t s)
{
    if (batch <= 0) return cudaSuccess;
    check_finalize_kernel<<<(unsigned)((batch + 255) / 256), 256, 0, s>>>(info, batch, nb);
    return cudaGetLastError();
}

template cudaError_t check_finite_launch<double>(const double *, int64_t, int64_t, int, int, const int32_t *,
                                                 int32_t *, cudaStream_t);
template cudaError_t check_finite_launch<float>(const float *, int64_t, int64_t, int, int, const int32_t *,
                                                int32_t *, cudaStream_t);

}  // namespace selinv
