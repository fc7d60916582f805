// Selected inverse of block lower-bidiagonal matrices with general blocks
// (b <= 16): gabp-sparse-inv 0.3.2 (PyPI page), "Implemented and tested
// kernels" -> Non-symmetric chain:
//   G_ii = M_ii^-1,   G_{i+1,i} = -M_{i+1,i+1}^-1 M_{i+1,i} M_ii^-1
// on M's pattern; no symmetry, no sweep (every block is local).
//
// Every block is local, so the work is spread over all blocks of all chains:
//  * bidiag_inverse_kernel: one half-warp per diagonal block, lane r holding
//    row r.  Gauss-Jordan elimination on [M_ii | I] with partial pivoting: at
//    column k the unused row with the largest |entry| (a half-warp arg-max)
//    is the pivot; it is broadcast by shuffles, scaled and removed from every
//    other row.  No row is moved: the lane that pivots column k ends with row
//    k of G_ii = M_ii^-1 and stores it.  A zero or non-finite pivot marks the
//    block singular (info = the chain's first such block; its outputs are
//    then unspecified).
//  * bidiag_lower_kernel: one warp per sub-diagonal block, after the first
//    kernel: G_{i+1,i} = -G_{i+1,i+1} (M_{i+1,i} G_ii) as two X Y^T products
//    of register tiles on the FP64 tensor cores, G_ii loaded transposed.
#include <type_traits>

#include <algorithm>
#include <climits>

#include "kernels.h"
#include "warp16.cuh"

namespace selinv {

namespace {

constexpr int BD_WARPS = 4;

template <class T> SELINV_DEVINL T hshfl(T v, int src) { return __shfl_sync(FULL_MASK, v, src, 16); }
template <class T> SELINV_DEVINL T hshfl_xor(T v, int m) { return __shfl_xor_sync(FULL_MASK, v, m, 16); }

// Row r (< b) of a row-major b x b block into x[0 .. 15], zero beyond b.
template <class T, bool FULL> SELINV_DEVINL void load_row(T x[16], const T *M, int b, int r, bool live)
{
    if (FULL) {
        using V = typename std::conditional<sizeof(T) == 8, double2, float4>::type;
        constexpr int PER = 16 / sizeof(T);
        const V *src = reinterpret_cast<const V *>(M + r * 16);
#pragma unroll
        for (int j = 0; j < 16 / PER; ++j) {
            const V v = live ? __ldg(src + j) : V{};
            const T *vv = reinterpret_cast<const T *>(&v);
#pragma unroll
            for (int q = 0; q < PER; ++q) x[j * PER + q] = vv[q];
        }
    } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) x[c] = (live && r < b && c < b) ? __ldg(M + r * b + c) : T(0);
    }
}

template <class T, bool FULL> SELINV_DEVINL void store_row(T *M, const T x[16], int b, int r)
{
    if (FULL) {
        using V = typename std::conditional<sizeof(T) == 8, double2, float4>::type;
        constexpr int PER = 16 / sizeof(T);
        V *dst = reinterpret_cast<V *>(M + r * 16);
#pragma unroll
        for (int j = 0; j < 16 / PER; ++j) {
            V v;
            T *vv = reinterpret_cast<T *>(&v);
#pragma unroll
            for (int q = 0; q < PER; ++q) vv[q] = x[j * PER + q];
            __stcs(dst + j, v);
        }
    } else if (r < b) {
#pragma unroll
        for (int c = 0; c < 16; ++c)
            if (c < b) M[r * b + c] = x[c];
    }
}

// Inverse of the b x b block whose row r the lane holds in a (zero beyond b):
// on return the lane holds row krow of the inverse in e (krow = the column it
// pivoted; lanes r >= b hold nothing).  Returns false (for every lane of the
// half) if a pivot is zero or not finite.
template <class T> SELINV_DEVINL bool gj_inverse(T a[16], T e[16], int &krow, int b, int r)
{
#pragma unroll
    for (int c = 0; c < 16; ++c) e[c] = (c == r) ? T(1) : T(0);
    bool used = r >= b;                               // pad rows never pivot
    krow = 0;
    bool ok = true;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        if (k < b) {
            // arg-max of |a[k]| over the unused rows (ties: the lower row)
            T best = used ? T(-1) : fabs(a[k]);
            int who = r;
#pragma unroll
            for (int m = 8; m >= 1; m >>= 1) {
                const T ob = hshfl_xor(best, m);
                const int ow = hshfl_xor(who, m);
                if (ob > best || (ob == best && ow < who)) {
                    best = ob;
                    who = ow;
                }
            }
            const T d = hshfl(a[k], who);
            ok = ok && (fabs(d) > T(0)) && isfinite(d);
            const T inv = T(1) / d;
            const bool piv = r == who;
            const T f = a[k];
            // columns left of k are already eliminated in every unused row
            // (the pivot row included), so a changes only from column k on
#pragma unroll
            for (int c = k; c < 16; ++c) {
                const T pc = hshfl(a[c], who) * inv;
                a[c] = piv ? pc : fma(-f, pc, a[c]);
            }
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const T pc = hshfl(e[c], who) * inv;
                e[c] = piv ? pc : fma(-f, pc, e[c]);
            }
            if (piv) {
                used = true;
                krow = k;
            }
        }
    }
    return ok;
}

// One half-warp per diagonal block (grid-stride): G_ii = M_ii^-1.
template <class T, bool FULL>
__global__ void __launch_bounds__(BD_WARPS * 32) bidiag_inverse_kernel(BidiagArgs<T> p)
{
    const int lane = threadIdx.x & 31, r = lane & 15;
    const int64_t nblk = p.batch * p.L;
    const int64_t halves = (int64_t)gridDim.x * BD_WARPS * 2;
    const int b = p.b;
    const int64_t bb = (int64_t)b * b;
    const int64_t h0 = ((int64_t)blockIdx.x * BD_WARPS + (threadIdx.x >> 5)) * 2 + (lane >> 4);
    // every half of a warp runs the same number of iterations (shuffles span the warp)
    const int64_t w0 = h0 - (lane >> 4);
    for (int64_t base = w0; base < nblk; base += halves) {
        const int64_t blk = base + (lane >> 4);
        const bool live = blk < nblk;
        T a[16], e[16];
        int krow;
        load_row<T, FULL>(a, p.diag + (live ? blk : 0) * bb, b, r, live);
        const bool ok = gj_inverse<T>(a, e, krow, b, r);
        if (live) {
            if (r < b) store_row<T, FULL>(p.G_diag + blk * bb, e, b, krow);
            if (!ok && r == 0) atomicMin(p.info + blk / p.L, (int32_t)(blk % p.L));
        }
    }
}

// Tile of a row-major b x b block, transposed on the way in (zero beyond b).
template <class T> SELINV_DEVINL void load_tile_T(w16::Tile<T> &a, const T *M, int b, int g, int t)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = g + 8 * h, c = w16::tcol(t, q);
            a.v[h][q] = (r < b && c < b) ? __ldcg(M + c * b + r) : T(0);
        }
}

template <class T> SELINV_DEVINL void load_tile_l2(w16::Tile<T> &a, const T *M, int b, int g, int t)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = g + 8 * h, c = w16::tcol(t, q);
            a.v[h][q] = (r < b && c < b) ? __ldcg(M + r * b + c) : T(0);
        }
}

// One warp per sub-diagonal block (grid-stride): G_{i+1,i} = -G_{i+1,i+1} (M_{i+1,i} G_ii).
template <class T>
__global__ void __launch_bounds__(BD_WARPS * 32) bidiag_lower_kernel(BidiagArgs<T> p)
{
    using namespace w16;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *sX = reinterpret_cast<T *>(smem_raw) + (threadIdx.x >> 5) * 2 * SL<T>::ELEMS, *sY = sX + SL<T>::ELEMS;
    const int64_t L1 = p.L - 1, nblk = p.batch * L1;
    const int b = p.b;
    const int64_t bb = (int64_t)b * b;
    for (int64_t k = (int64_t)blockIdx.x * BD_WARPS + (threadIdx.x >> 5); k < nblk;
         k += (int64_t)gridDim.x * BD_WARPS) {
        const int64_t e = k / L1, i = k % L1;
        const T *Gii = p.G_diag + (e * p.L + i) * bb;
        Tile<T> giT, ml, gn, xt, gl;
        load_tile_T<T>(giT, Gii, b, g, t);
        load_tile_l2<T>(ml, p.lower + k * bb, b, g, t);
        load_tile_l2<T>(gn, Gii + bb, b, g, t);
        zero(xt);
        gemm_nt<false>(xt, giT, ml, sX, sY, g, t);     // (M_{i+1,i} G_ii)^T = G_ii^T M_{i+1,i}^T
        zero(gl);
        gemm_nt<true>(gl, gn, xt, sX, sY, g, t);       // -G_{i+1,i+1} (M_{i+1,i} G_ii)
        store_block<T, false>(p.G_lower + k * bb, gl, b, g, t);
    }
}

__global__ void bidiag_info(int32_t *info, int64_t batch, int final_pass)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= batch) return;
    if (!final_pass) info[i] = INT_MAX;
    else if (info[i] == INT_MAX) info[i] = -1;
}

template <class T> cudaError_t launch(const BidiagArgs<T> &p, bool full, cudaStream_t s)
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned ib = (unsigned)ceil_div(p.batch, 256);
    bidiag_info<<<ib, 256, 0, s>>>(p.info, p.batch, 0);
    auto ki = full ? bidiag_inverse_kernel<T, true> : bidiag_inverse_kernel<T, false>;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, ki, BD_WARPS * 32, 0) != cudaSuccess || occ < 1) occ = 2;
    const int64_t halves = p.batch * p.L;
    const int64_t gi = std::min<int64_t>((int64_t)sms * occ, ceil_div(halves, 2 * BD_WARPS));
    ki<<<(unsigned)gi, BD_WARPS * 32, 0, s>>>(p);
    if (p.L > 1) {
        const size_t smem = sizeof(T) * 2 * w16::SL<T>::ELEMS * BD_WARPS;
        auto kl = bidiag_lower_kernel<T>;
        cudaError_t err = cudaFuncSetAttribute(kl, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        int occ_l = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_l, kl, BD_WARPS * 32, smem) != cudaSuccess ||
            occ_l < 1)
            occ_l = 4;
        const int64_t gl = std::min<int64_t>((int64_t)sms * occ_l, ceil_div(p.batch * (p.L - 1), BD_WARPS));
        kl<<<(unsigned)gl, BD_WARPS * 32, smem, s>>>(p);
    }
    bidiag_info<<<ib, 256, 0, s>>>(p.info, p.batch, 1);
    return cudaGetLastError();
}

}  // namespace

template <class T> cudaError_t bidiag_launch(const BidiagArgs<T> &p, bool aligned16, cudaStream_t s)
{
    return launch<T>(p, p.b == 16 && aligned16, s);
}

template cudaError_t bidiag_launch<double>(const BidiagArgs<double> &, bool, cudaStream_t);
template cudaError_t bidiag_launch<float>(const BidiagArgs<float> &, bool, cudaStream_t);

}  // namespace selinv
