// Selected inverse of block lower-bidiagonal matrices with general blocks
// (b <= 16): gabp-sparse-inv 0.3.2 (PyPI page), "Implemented and tested
// kernels" -> Non-symmetric chain:
//   G_ii = M_ii^-1,   G_{i+1,i} = -M_{i+1,i+1}^-1 M_{i+1,i} M_ii^-1
// on M's pattern; no symmetry, no sweep (every block is local).
//
// One half-warp per chain walks i = 0 .. L-1 so that each diagonal block is
// inverted once; lane r of the half holds row r of the block being inverted.
// The inverse is Gauss-Jordan elimination on [M_ii | I] with partial
// pivoting: at column k the unused row with the largest |entry| (a
// half-warp arg-max) is the pivot; it is broadcast by shuffles, scaled, and
// removed from every other row.  No row is moved: the lane that pivots
// column k ends with row k of the inverse, which it writes to shared memory.
// The two products of G_{i+1,i} then read their right-hand factor row by row
// from shared memory (pitch 17: a column of a padded image spans distinct
// banks).  A zero or non-finite pivot marks M_ii singular (info = first such
// block; the chain's outputs are then unspecified).
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace selinv {

namespace {

constexpr int BD_WARPS = 4;
constexpr int BD_PITCH = 17;
constexpr int BD_IMG = 16 * BD_PITCH;                 // one padded 16 x 16 image

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

// Inverse of the b x b block whose row r the lane holds in a (zero beyond b);
// row k(r) of the inverse is written to img[k(r) * BD_PITCH + .].  Returns
// false (for every lane of the half) if a pivot is zero or not finite.
template <class T> SELINV_DEVINL bool gj_inverse(T a[16], T *img, int b, int r)
{
    T e[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) e[c] = (c == r) ? T(1) : T(0);
    bool used = r >= b;                               // pad rows never pivot
    int krow = 0;
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
            T pr[16], pe[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                pr[c] = hshfl(a[c], who) * inv;
                pe[c] = hshfl(e[c], who) * inv;
            }
            if (r == who) {
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    a[c] = pr[c];
                    e[c] = pe[c];
                }
                used = true;
                krow = k;
            } else {
                const T f = a[k];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    a[c] = fma(-f, pr[c], a[c]);
                    e[c] = fma(-f, pe[c], e[c]);
                }
            }
        }
    }
    if (r < b) {
#pragma unroll
        for (int c = 0; c < 16; ++c) img[krow * BD_PITCH + c] = e[c];
    }
    return ok;
}

template <class T, bool FULL>
__global__ void __launch_bounds__(BD_WARPS * 32) bidiag_kernel(BidiagArgs<T> p)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int half = lane >> 4, r = lane & 15;
    const int64_t e = ((int64_t)blockIdx.x * BD_WARPS + wid) * 2 + half;
    if (((int64_t)blockIdx.x * BD_WARPS + wid) * 2 >= p.batch) return;   // whole warp idle
    const bool live = e < p.batch;                    // the second half of the last warp may have no chain
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *base = reinterpret_cast<T *>(smem_raw) + (wid * 2 + half) * 3 * BD_IMG;
    T *timg = base + 2 * BD_IMG;                      // M_{i,i-1} M_{i-1,i-1}^-1 (two images before it
                                                      // hold the inverses of blocks i-1 and i, by parity)
    const int b = p.b;
    const int64_t L = p.L, bb = (int64_t)b * b;
    const int64_t ec = live ? e : 0;
    const T *D = p.diag + ec * L * bb;
    const T *Bl = p.lower + ec * (L - 1) * bb;
    T *Gd = p.G_diag + ec * L * bb;
    T *Gl = p.G_lower + ec * (L - 1) * bb;
    int bad_at = -1;
    for (int64_t i = 0; i < L; ++i) {
        if (live && i + 1 < L) {                      // next step's blocks toward L2
            prefetch_range_l2(D + (i + 1) * bb, bb, r, 16);
            prefetch_range_l2(Bl + i * bb, bb, r, 16);
        }
        T a[16];
        load_row<T, FULL>(a, D + i * bb, b, r, live);
        T *cur = base + (i & 1) * BD_IMG, *prev = base + ((i & 1) ^ 1) * BD_IMG;
        const bool ok = gj_inverse<T>(a, cur, b, r);
        if (!ok && bad_at < 0) bad_at = (int)i;
        __syncwarp();
        T g[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) g[c] = cur[r * BD_PITCH + c];
        if (live) store_row<T, FULL>(Gd + i * bb, g, b, r);     // G_ii = M_ii^-1
        if (i > 0) {
            // T = M_{i,i-1} M_{i-1,i-1}^-1 (row r), then G_{i,i-1} = -M_ii^-1 T
            T m[16], t[16];
            load_row<T, FULL>(m, Bl + (i - 1) * bb, b, r, live);
#pragma unroll
            for (int c = 0; c < 16; ++c) t[c] = T(0);
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if (k < b)
#pragma unroll
                    for (int c = 0; c < 16; ++c) t[c] = fma(m[k], prev[k * BD_PITCH + c], t[c]);
#pragma unroll
            for (int c = 0; c < 16; ++c) timg[r * BD_PITCH + c] = t[c];
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 16; ++c) t[c] = T(0);
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if (k < b)
#pragma unroll
                    for (int c = 0; c < 16; ++c) t[c] = fma(-g[k], timg[k * BD_PITCH + c], t[c]);
            if (live) store_row<T, FULL>(Gl + (i - 1) * bb, t, b, r);
        }
        __syncwarp();                                 // cur becomes prev; timg is free again
    }
    if (live && r == 0) p.info[e] = bad_at;
}

template <class T> cudaError_t launch(const BidiagArgs<T> &p, bool full, cudaStream_t s)
{
    const size_t smem = sizeof(T) * 3 * BD_IMG * 2 * BD_WARPS;
    auto k = full ? bidiag_kernel<T, true> : bidiag_kernel<T, false>;
    cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int64_t warps = ceil_div(p.batch, 2);
    k<<<(unsigned)ceil_div(warps, BD_WARPS), BD_WARPS * 32, smem, s>>>(p);
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
