// Group-level toolkit for blocks with 16 < b <= 32: a group of four warps
// owns one padded 32 x 32 block at a time, warp w holding quadrant
// (I, J) = (w >> 1, w & 1) as a 16 x 16 register tile (the m8n8k4 accumulator
// layout of warp16.cuh).  Blocks smaller than 32 are embedded with an
// identity (diagonal) or zero (off-diagonal) pad.  Operands of products live
// in shared memory as four quadrant images in the swizzled layout of
// warp16.cuh; groups synchronise on their own named barrier.
#pragma once

#include "warp16.cuh"

namespace selinv {
namespace q32 {

using w16::Tile;

constexpr int GW = 4;                  // warps per group
constexpr int GT = GW * 32;            // threads per group

template <class T> struct Lay {        // per-group shared memory of the two-ended kernel (elements)
    static constexpr int E = w16::SL<T>::ELEMS;
    static constexpr int IMG = 4 * E;  // one 32 x 32 block = four quadrant images
    static constexpr int SCR = sizeof(T) == 4 ? 2 * E * GW : 0;   // float products: per-warp scratch
    static constexpr int C = 0, D = IMG, X = 2 * IMG, Y = 3 * IMG, Z = 4 * IMG, Z2 = 5 * IMG, S = 6 * IMG;
    static constexpr int CB = S + SCR;
    static constexpr int CBN = sizeof(T) == 8 ? 4 * 256 : 64;     // inverse scratch (four 16 x 16 images / pivot column)
    static constexpr int GROUP = CB + CBN;
    static constexpr int EXCH = 2 * GROUP;        // exchange image after both groups
    static constexpr int TOTAL = EXCH + IMG;
};

SELINV_DEVINL void group_bar(int id) { asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(GT) : "memory"); }

template <class T> SELINV_DEVINL T *quad(T *img, int r, int c) { return img + (2 * r + c) * w16::SL<T>::ELEMS; }

// Quadrant (i, k) of an operand held as four images: TR = false gives
// M[i][k]; TR = true gives (M^T)[i][k] = M[k][i]^T.
// The image's element type S may be narrower than the tile's A (a float
// input image read into float64 tiles).
template <bool TR, class A, class S> SELINV_DEVINL void qget(w16::Tile<A> &o, S *img, int i, int k, int g, int t)
{
    if (TR) w16::from_smem_T_as<A, S>(o, quad(img, k, i), g, t);
    else w16::from_smem_as<A, S>(o, quad(img, i, k), g, t);
}

// acc += (NEG ? -1 : 1) (X Y^T)_{IJ} = sum_K X_IK Y_JK^T, operands from images.
template <bool NEG, bool TX, bool TY, bool LOWER, class T, class SX, class SY>
SELINV_DEVINL void qgemm(w16::Tile<T> &acc, SX *imgX, SY *imgY, int I, int J, T *s1, T *s2, int g, int t)
{
#pragma unroll
    for (int K = 0; K < 2; ++K) {
        w16::Tile<T> x, y;
        qget<TX>(x, imgX, I, K, g, t);
        qget<TY>(y, imgY, J, K, g, t);
        w16::gemm_nt<NEG, LOWER>(acc, x, y, s1, s2, g, t);
    }
}

// Lower triangle of a diagonal block (row-major b x b, identity pad beyond b)
// into the quadrant images (0,0), (1,0), (1,1); FULL: cp.async chunks.
template <class T, bool FULL> SELINV_DEVINL void load_diag(T *img, const T *D, int b, int tid)
{
    constexpr int CH = 16 / sizeof(T);
    if (FULL) {
        for (int j = tid; j < 32 * (32 / CH); j += GT) {
            const int r = j / (32 / CH), c = (j % (32 / CH)) * CH;
            if (c <= r) cp_async16(quad(img, r >> 4, c >> 4) + w16::SL<T>::idx(r & 15, c & 15), D + r * 32 + c);
        }
    } else {
        for (int j = tid; j < 1024; j += GT) {
            const int r = j >> 5, c = j & 31;
            if (c <= r)
                quad(img, r >> 4, c >> 4)[w16::SL<T>::idx(r & 15, c & 15)] =
                    (r < b && c < b) ? __ldg(D + r * b + c) : (r == c ? T(1) : T(0));
        }
    }
}

// A full off-diagonal block (row-major b x b, zero pad) into four images.
template <class T, bool FULL> SELINV_DEVINL void load_full(T *img, const T *B, int b, int tid)
{
    constexpr int CH = 16 / sizeof(T);
    if (FULL) {
        for (int j = tid; j < 32 * (32 / CH); j += GT) {
            const int r = j / (32 / CH), c = (j % (32 / CH)) * CH;
            cp_async16(quad(img, r >> 4, c >> 4) + w16::SL<T>::idx(r & 15, c & 15), B + r * 32 + c);
        }
    } else {
        for (int j = tid; j < 1024; j += GT) {
            const int r = j >> 5, c = j & 31;
            quad(img, r >> 4, c >> 4)[w16::SL<T>::idx(r & 15, c & 15)] = (r < b && c < b) ? __ldg(B + r * b + c) : T(0);
        }
    }
}

// The same two loads into float64 images from blocks of element type T
// (plain loads, widened; the caller's barrier makes them visible).  For
// T = double they are the cp.async loads above (the caller commits / waits).
template <class T, bool FULL> SELINV_DEVINL void load_diag_f64(double *img, const T *D, int b, int tid)
{
    if constexpr (std::is_same<T, double>::value) {
        load_diag<double, FULL>(img, D, b, tid);
    } else {
        for (int j = tid; j < 1024; j += GT) {
            const int r = j >> 5, c = j & 31;
            if (c <= r)
                quad(img, r >> 4, c >> 4)[w16::SL<double>::idx(r & 15, c & 15)] =
                    (r < b && c < b) ? (double)__ldg(D + r * b + c) : (r == c ? 1.0 : 0.0);
        }
    }
}
template <class T, bool FULL> SELINV_DEVINL void load_full_f64(double *img, const T *B, int b, int tid)
{
    if constexpr (std::is_same<T, double>::value) {
        load_full<double, FULL>(img, B, b, tid);
    } else {
        for (int j = tid; j < 1024; j += GT) {
            const int r = j >> 5, c = j & 31;
            quad(img, r >> 4, c >> 4)[w16::SL<double>::idx(r & 15, c & 15)] =
                (r < b && c < b) ? (double)__ldg(B + r * b + c) : 0.0;
        }
    }
}

// The warp's quadrant of the symmetric block whose lower quadrants are in img.
template <class A, class S> SELINV_DEVINL void sym_quad(w16::Tile<A> &o, S *img, int I, int J, int g, int t)
{
    if (I == J) w16::from_smem_lower_as<A, S>(o, quad(img, I, J), g, t);
    else if (I > J) w16::from_smem_as<A, S>(o, quad(img, I, J), g, t);
    else w16::from_smem_T_as<A, S>(o, quad(img, J, I), g, t);
}

// Store a quadrant tile into a row-major b x b block (TR: transposed position),
// rounded to the block's element type T.
template <class T, bool TR, class A>
SELINV_DEVINL void store_quad(T *G, const w16::Tile<A> &a, int b, int I, int J, int g, int t)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            int r = 16 * I + g + 8 * h, c = 16 * J + w16::tcol(t, q);
            if (TR) {
                const int tmp = r;
                r = c;
                c = tmp;
            }
            if (r < b && c < b) G[r * b + c] = (T)a.v[h][q];
        }
}

// CTA-group inverse of a symmetric positive definite 32 x 32 block held as
// quadrant tiles: the symmetric Gauss-Jordan sweep (A_ij -= A_ik A_kj / d,
// A_ik /= d, A_kj /= d, A_kk = -1/d, then negate); pivots -> det, bad.
template <class T>
SELINV_DEVINL void qinverse_scalar(w16::Tile<T> &a, T *cbuf, int I, int J, int g, int t, int bar, LogAcc &det,
                                   bool &bad)
{
    using V = typename w16::Vec2<T>::type;
    for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            const int k = 16 * kb + kk;
            const int kh = kk >> 3, kt = (kk & 7) >> 1, kq = (kk & 1) | ((kk >> 3) << 1);
            T *cb = cbuf + 32 * (kk & 1);
            const bool col_owner = (J == kb) && (t == kt);
            if (col_owner) {
                cb[16 * I + g] = a.v[0][kq];
                cb[16 * I + g + 8] = a.v[1][kq];
            }
            group_bar(bar);
            const T d = cb[k];
            const T c0 = cb[16 * I + g], c1 = cb[16 * I + g + 8];
            const V r01 = *reinterpret_cast<const V *>(cb + 16 * J + 2 * t);
            const V r23 = *reinterpret_cast<const V *>(cb + 16 * J + 2 * t + 8);
            const T row[4] = {r01.x, r01.y, r23.x, r23.y};
            det.mul((double)d);
            const T p = recip(d);
            bad |= bad_pivot(d, p);
            const T tc[2] = {c0 * p, c1 * p};
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int q = 0; q < 4; ++q) a.v[h][q] = fma(-tc[h], row[q], a.v[h][q]);
            if (col_owner) {
                a.v[0][kq] = tc[0];
                a.v[1][kq] = tc[1];
            }
            if (I == kb && g == (kk & 7)) {
#pragma unroll
                for (int q = 0; q < 4; ++q) a.v[kh][q] = row[q] * p;
                if (col_owner) a.v[kh][kq] = -p;
            }
        }
        det.renorm();
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) a.v[h][q] = -a.v[h][q];
}

// float64 through the 2 x 2 quadrant structure M = [[A, B^T], [B, C]]
// (B = the (1,0) quadrant; M symmetric):
//   T = B A^-1,  S = C - T B^T,
//   M^-1 = [[A^-1 + T^T S^-1 T, -T^T S^-1], [-S^-1 T, S^-1]].
// Warp (0,0) inverts A and warp (1,1) inverts S, each in its own registers
// (two 8-pivot block steps, warp16.cuh; pivots -> det, bad), so the group
// meets at three barriers only; every product is a register-register FP64
// tensor-core product with operands from four 16 x 16 images in buf.
// `idle(phase)` is called by every warp in phases 1 (while warp (0,0) inverts
// A) and 3 (while warp (1,1) inverts S), so that a caller can give the warps
// that wait there independent work; it must not touch `buf`.
constexpr int QSCHUR = 4 * w16::SL<double>::ELEMS;

struct NoIdle {
    SELINV_DEVINL void operator()(int) const {}
};

template <class Idle = NoIdle>
SELINV_DEVINL void qinverse_schur(w16::Tile<double> &a, double *buf, int I, int J, int g, int t, int bar,
                                  LogAcc &det, bool &bad, const Idle &idle = Idle())
{
    using namespace w16;
    constexpr int E = SL<double>::ELEMS;
    double *sAi = buf, *sB = buf + E, *sT = buf + 2 * E, *sSi = buf + 3 * E;
    if (I == 0 && J == 0) {                                          // A^-1
        spd_inverse_blocked(a, g, t, det, bad);
        det.renorm();
        to_smem<double>(sAi, a, g, t);
    } else if (I == 1 && J == 0) {
        to_smem<double>(sB, a, g, t);
    }
    idle(1);
    group_bar(bar);
    if (I == 1 && J == 0) {                                          // T = B A^-1
        Tile<double> ai, tt;
        from_smem<double>(ai, sAi, g, t);
        zero(tt);
        gemm_nt<false>(tt, a, ai, nullptr, nullptr, g, t);
        to_smem<double>(sT, tt, g, t);
        a = tt;
    }
    group_bar(bar);
    if (I == 1 && J == 1) {                                          // S = C - T B^T, S^-1
        Tile<double> tt, bq;
        from_smem<double>(tt, sT, g, t);
        from_smem<double>(bq, sB, g, t);
        gemm_nt<true>(a, tt, bq, nullptr, nullptr, g, t);
        spd_inverse_blocked(a, g, t, det, bad);
        det.renorm();
        to_smem<double>(sSi, a, g, t);
    }
    idle(3);
    group_bar(bar);
    if (!(I == 1 && J == 1)) {
        Tile<double> si, tT;
        from_smem<double>(si, sSi, g, t);
        from_smem_T<double>(tT, sT, g, t);                         // T^T
        if (I == 0 && J == 0) {                                      // A^-1 + T^T (S^-1 T)
            Tile<double> ut;
            zero(ut);
            gemm_nt<false>(ut, tT, si, nullptr, nullptr, g, t);      // T^T S^-1
            gemm_nt<false>(a, tT, ut, nullptr, nullptr, g, t);
        } else if (I == 0) {                                         // -T^T S^-1
            zero(a);
            gemm_nt<true>(a, tT, si, nullptr, nullptr, g, t);
        } else {                                                     // -S^-1 T
            zero(a);
            gemm_nt<true>(a, si, tT, nullptr, nullptr, g, t);
        }
    }
}

template <class T, class Idle = NoIdle>
SELINV_DEVINL void qinverse(w16::Tile<T> &a, T *cbuf, int I, int J, int g, int t, int bar, LogAcc &det, bool &bad,
                            const Idle &idle = Idle())
{
    if constexpr (sizeof(T) == 8) {
        qinverse_schur(a, cbuf, I, J, g, t, bar, det, bad, idle);
    } else {
        idle(1);
        idle(3);
        qinverse_scalar(a, cbuf, I, J, g, t, bar, det, bad);
    }
}

// Copy n elements (a multiple of 16 bytes) from shared to global memory, or
// stage them from global to shared (cp.async; the caller commits / waits).
template <class T> SELINV_DEVINL void copy_out(T *dst, const T *src, int n, int gtid)
{
    using V = typename w16::Vec2<T>::type;
    constexpr int CH = 16 / sizeof(T);
    for (int k = gtid; k < n / CH; k += GT) {
        const V *s4 = reinterpret_cast<const V *>(src + k * CH);
        V *d4 = reinterpret_cast<V *>(dst + k * CH);
        d4[0] = s4[0];
        if (CH == 4) d4[1] = s4[1];
    }
}
template <class T> SELINV_DEVINL void stage_in(T *dst, const T *src, int n, int gtid)
{
    constexpr int CH = 16 / sizeof(T);
    for (int k = gtid; k < n / CH; k += GT) cp_async16(dst + k * CH, src + k * CH);
}

}  // namespace q32
}  // namespace selinv
