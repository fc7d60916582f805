// Block-tridiagonal chains with 16 < b <= 128: one CTA per chain.
//
// gabp-sparse-inv 0.3.2 (PyPI page), "Implemented and tested kernels" ->
// Chain.  Same recursion as the b <= 16 kernel, scaled up: blocks are padded
// to BP in {32, 64, 128} (identity / zero pad), and a CTA of (BP/32)^2 warps
// holds the current BP x BP block as a register tile, each warp a 32 x 32
// quadrant laid out as 4 x 4 accumulator tiles of the m8n8k4 FP64 tensor-core
// instruction.
//
// Per block i:
//   collect     S_i^-1 by a CTA-wide symmetric Gauss-Jordan sweep in registers
//               (one column broadcast through shared memory per pivot; the
//               pivots give log det S_i);
//               W_i = B_i S_i^-1 and S_{i+1} = D_{i+1} - W_i B_i^T on the
//               tensor cores, one operand resident in shared memory and the
//               other (B_i) streamed through 16-wide K panels (cp.async,
//               double-buffered);
//   distribute  G_{i+1,i} = -G_{i+1,i+1} W_i and G_ii = S_i^-1 - W_i^T G_{i+1,i}
//               with G_{i+1,i+1} / G_{i+1,i} resident and W_i streamed from
//               the workspace.
// S_i^-1 and W_i are kept in the caller's workspace between the sweeps (at
// these sizes the products dominate and storing W_i saves recomputing it).
#include "common.cuh"
#include "kernels.h"

namespace selinv {

namespace {

template <int BP> struct Geo {
    static constexpr int RW = BP / 32;       // warps per row (and per column) of the block
    static constexpr int NW = RW * RW;
    static constexpr int NT = NW * 32;
    static constexpr int NP = BP / 16;       // K panels of width 16
};

// Shared-memory image of a row-major matrix of logical pitch P (a multiple
// of 16), stored with four elements of row padding.
//  double: rows P + 4 doubles apart put row r at bank offset 8 r (mod 32), so
//          the tensor-core fragment reads (8 rows x 4 columns, 4 rows x 8
//          columns) and the accumulator-layout stores are conflict-free, and
//          every fragment address is a per-row base plus a constant, which
//          keeps the unrolled product loops' address registers few (an XOR
//          swizzle needed one precomputed offset per row and k step).
//  float:  the same 4-float row padding.
template <class T> struct SW;
template <> struct SW<double> {
    static constexpr int PAD = 4;
    SELINV_DEVINL static int idx(int r, int c, int P) { return r * (P + 4) + c; }
};
template <> struct SW<float> {
    static constexpr int PAD = 4;
    SELINV_DEVINL static int idx(int r, int c, int P) { return r * (P + 4) + c; }
};

template <class T> struct V2;
template <> struct V2<double> { using type = double2; };
template <> struct V2<float> { using type = float2; };

template <class T> struct Big {
    T v[4][4][2];    // [mi][ni][j]: row R(mi) = 32 rw + 8 mi + g, col C(ni, j) = 32 cw + 8 ni + 2 t + j
};

template <class T, int BP> struct Ctx {
    static constexpr int RW = Geo<BP>::RW;
    static constexpr int NT = Geo<BP>::NT;
    static constexpr int BIG = BP * (BP + SW<T>::PAD);           // resident matrix
    static constexpr int PANEL = 16 * (BP + SW<T>::PAD) > BP * (16 + SW<T>::PAD)
                                     ? 16 * (BP + SW<T>::PAD) : BP * (16 + SW<T>::PAD);
    int tid, lane, g, t, rw, cw;
    SELINV_DEVINL void init()
    {
        tid = threadIdx.x;
        lane = tid & 31;
        g = lane >> 2;
        t = lane & 3;
        const int w = tid >> 5;
        rw = w / RW;
        // Quadrants of one row go to four different SM sub-partitions (warp w
        // runs on sub-partition w % 4), shifted by the row: the lower-triangle
        // quadrants that the symmetric steps keep busy are then spread evenly.
#ifndef SELINV_LARGE_ROTATE
#define SELINV_LARGE_ROTATE 1
#endif
        cw = (RW == 4 && SELINV_LARGE_ROTATE) ? (((w & 3) - rw) & 3) : (w % RW);
    }
    // Tile (mi, ni) of this warp's quadrant lies on or below the block diagonal.
    SELINV_DEVINL bool tile_lower(int mi, int ni) const { return 32 * rw + 8 * mi >= 32 * cw + 8 * ni; }
    SELINV_DEVINL bool quad_upper() const { return rw < cw; }
    SELINV_DEVINL int R(int mi) const { return 32 * rw + 8 * mi + g; }
    SELINV_DEVINL int C(int ni, int j) const { return 32 * cw + 8 * ni + 2 * t + j; }
};

template <class T, int BP> constexpr size_t smem_elems()
{
    using X = Ctx<T, BP>;
    return (size_t)X::BIG + 3 * X::PANEL + 2 * BP /*colbuf*/ + 4 * BP /*y, x*/ + 2 * X::RW * BP /*red*/ +
           BP /*z of a draw*/;
}

template <class T> SELINV_DEVINL void zero(Big<T> &a)
{
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) a.v[mi][ni][0] = a.v[mi][ni][1] = T(0);
}


// ---- register tile <-> shared / global -----------------------------------------

template <class T, int BP>
SELINV_DEVINL void to_smem(T *S, const Big<T> &a, const Ctx<T, BP> &x)
{
    using V = typename V2<T>::type;
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) {
            V v;
            v.x = a.v[mi][ni][0];
            v.y = a.v[mi][ni][1];
            *reinterpret_cast<V *>(S + SW<T>::idx(x.R(mi), x.C(ni, 0), BP)) = v;
        }
}

template <class T, int BP>
SELINV_DEVINL void from_smem(Big<T> &a, const T *S, const Ctx<T, BP> &x)
{
    using V = typename V2<T>::type;
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) {
            V v = *reinterpret_cast<const V *>(S + SW<T>::idx(x.R(mi), x.C(ni, 0), BP));
            a.v[mi][ni][0] = v.x;
            a.v[mi][ni][1] = v.y;
        }
}

// lower triangle and its mirror: an exactly symmetric image, every entry written once
template <class T, int BP>
SELINV_DEVINL void to_smem_sym(T *S, const Big<T> &a, const Ctx<T, BP> &x)
{
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int r = x.R(mi), c = x.C(ni, j);
                if (c <= r) S[SW<T>::idx(r, c, BP)] = a.v[mi][ni][j];
                if (c < r) S[SW<T>::idx(c, r, BP)] = a.v[mi][ni][j];
            }
}

// diagonal block (row-major b x b, lower triangle read), identity pad.
// FULL (b == BP): every address is one of two per-thread bases -- D[R(0)][C(0)]
// for entries on or below the diagonal, D[C(0)][R(0)] for their mirrors --
// plus a constant, so the 32 loads in flight need two address registers
// (computing each address separately spilled the kernel).
template <class T, int BP, bool FULL = false>
SELINV_DEVINL void load_sym(Big<T> &a, const T *D, int b, const Ctx<T, BP> &x)
{
    if constexpr (FULL) {
        const T *Dd = D + x.R(0) * BP + x.C(0, 0);
        const T *Dm = D + x.C(0, 0) * BP + x.R(0);
#pragma unroll
        for (int mi = 0; mi < 4; ++mi)
#pragma unroll
            for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                for (int j = 0; j < 2; ++j)
                    a.v[mi][ni][j] = x.C(ni, j) <= x.R(mi) ? __ldg(Dd + (8 * mi) * BP + 8 * ni + j)
                                                           : __ldg(Dm + (8 * ni + j) * BP + 8 * mi);
    } else {
#pragma unroll
        for (int mi = 0; mi < 4; ++mi)
#pragma unroll
            for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int r = x.R(mi), c = x.C(ni, j);
                    const int rr = c <= r ? r : c, cc = c <= r ? c : r;
                    a.v[mi][ni][j] =
                        (r < b && c < b) ? __ldg(D + (int64_t)rr * b + cc) : (r == c ? T(1) : T(0));
                }
    }
}

template <class T, int BP, bool FULL>
SELINV_DEVINL void store_block(T *G, const Big<T> &a, int b, const Ctx<T, BP> &x)
{
    using V = typename V2<T>::type;
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) {
            const int r = x.R(mi), c = x.C(ni, 0);
            if (FULL) {
                V v;
                v.x = a.v[mi][ni][0];
                v.y = a.v[mi][ni][1];
                __stcs(reinterpret_cast<V *>(G + r * BP + c), v);
            } else {
                if (r < b && c < b) G[(int64_t)r * b + c] = a.v[mi][ni][0];
                if (r < b && c + 1 < b) G[(int64_t)r * b + c + 1] = a.v[mi][ni][1];
            }
        }
}

// workspace blocks are always BP x BP row-major
template <class T, int BP>
SELINV_DEVINL void store_ws(T *W, const Big<T> &a, const Ctx<T, BP> &x)
{
    using V = typename V2<T>::type;
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) {
            V v;
            v.x = a.v[mi][ni][0];
            v.y = a.v[mi][ni][1];
            *reinterpret_cast<V *>(W + x.R(mi) * BP + x.C(ni, 0)) = v;
        }
}

template <class T, int BP>
SELINV_DEVINL void load_ws(Big<T> &a, const T *W, const Ctx<T, BP> &x)
{
    using V = typename V2<T>::type;
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) {
            V v = *reinterpret_cast<const V *>(W + x.R(mi) * BP + x.C(ni, 0));
            a.v[mi][ni][0] = v.x;
            a.v[mi][ni][1] = v.y;
        }
}

// ---- K panels -------------------------------------------------------------------

// Column panel: rows 0..BP-1, columns k0..k0+15 of a row-major b x b input block.
template <class T, int BP, bool FULL>
SELINV_DEVINL void load_colpanel(T *P, const T *M, int b, int k0, const Ctx<T, BP> &x)
{
    constexpr int CH = 16 / sizeof(T);
    if (FULL) {
        for (int j = x.tid; j < BP * (16 / CH); j += Ctx<T, BP>::NT) {
            const int r = j / (16 / CH), c = (j % (16 / CH)) * CH;
            cp_async16(P + SW<T>::idx(r, c, 16), M + r * BP + k0 + c);
        }
    } else {
        for (int j = x.tid; j < BP * 16; j += Ctx<T, BP>::NT) {
            const int r = j >> 4, c = j & 15;
            P[SW<T>::idx(r, c, 16)] = (r < b && k0 + c < b) ? __ldg(M + (int64_t)r * b + k0 + c) : T(0);
        }
    }
}

// Row panel: rows k0..k0+15 of a BP x BP workspace block.
template <class T, int BP>
SELINV_DEVINL void load_rowpanel(T *P, const T *M, int k0, const Ctx<T, BP> &x)
{
    constexpr int CH = 16 / sizeof(T);
    for (int j = x.tid; j < 16 * (BP / CH); j += Ctx<T, BP>::NT) {
        const int r = j / (BP / CH), c = (j % (BP / CH)) * CH;
        cp_async16(P + SW<T>::idx(r, c, BP), M + (k0 + r) * BP + c);
    }
}

enum { OP_BIG = 0, OP_COLPANEL = 1, OP_ROWPANEL = 2 };

// acc += (NEG ? -1 : 1) * A B over k = 0..BP-1.  One operand is the resident
// matrix `big` (row-major, A[m][k] or B[k][n]); the other is streamed in
// panels from global memory:
//   A = OP_COLPANEL: A[m][k] = M[m][k] (column panels of M)
//   A = OP_ROWPANEL: A[m][k] = M[k][m] (row panels of M, i.e. M^T)
//   B = OP_COLPANEL: B[k][n] = M[n][k] (column panels of M, i.e. M^T)
//   B = OP_ROWPANEL: B[k][n] = M[k][n] (row panels of M)
// Panels stream through a ring of three buffers: panel p + 2 is issued right
// after the barrier that makes panel p visible, which is also the point every
// warp has finished reading panel p - 1 (the buffer it overwrites), so one
// barrier per panel suffices (plus one at the end, before the caller reuses
// the buffers).
template <class T, int BP, int AOP, int BOP, bool NEG, bool FULL, bool LOWER = false>
SELINV_DEVINL void gemm(Big<T> &acc, const T *big, T *pbuf, const T *M, int b, const Ctx<T, BP> &x)
{
    constexpr int NP = Geo<BP>::NP;
    constexpr int PANEL = Ctx<T, BP>::PANEL;
    constexpr int STREAM = AOP != OP_BIG ? AOP : BOP;
    auto issue = [&](int p) {
        T *dst = pbuf + (p % 3) * PANEL;
        if (STREAM == OP_COLPANEL) load_colpanel<T, BP, FULL>(dst, M, b, 16 * p, x);
        else load_rowpanel<T, BP>(dst, M, 16 * p, x);
        cp_async_commit();
    };
    issue(0);
    if (NP > 1) issue(1);
    for (int p = 0; p < NP; ++p) {
        if (p + 1 < NP) cp_async_wait_one();          // panel p landed (p + 1 may still be in flight)
        else cp_async_wait_all();
        __syncthreads();
        if (p + 2 < NP) issue(p + 2);
        const T *P = pbuf + (p % 3) * PANEL;
        const int k0 = 16 * p;
        if (LOWER && x.quad_upper()) {
            // nothing to compute above the diagonal
        } else if constexpr (sizeof(T) == 8) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                double a[4], bf[4];
                const int kl = 4 * kk + x.t;        // k within the panel for this lane's fragment
#pragma unroll
                for (int mi = 0; mi < 4; ++mi) {
                    const int m = 32 * x.rw + 8 * mi + x.g;
                    double v;
                    if (AOP == OP_BIG) v = big[SW<T>::idx(m, k0 + kl, BP)];
                    else if (AOP == OP_COLPANEL) v = P[SW<T>::idx(m, kl, 16)];
                    else v = P[SW<T>::idx(kl, m, BP)];
                    a[mi] = NEG ? -v : v;
                }
#pragma unroll
                for (int ni = 0; ni < 4; ++ni) {
                    const int n = 32 * x.cw + 8 * ni + x.g;
                    if (BOP == OP_BIG) bf[ni] = big[SW<T>::idx(k0 + kl, n, BP)];
                    else if (BOP == OP_COLPANEL) bf[ni] = P[SW<T>::idx(n, kl, 16)];
                    else bf[ni] = P[SW<T>::idx(kl, n, BP)];
                }
#pragma unroll
                for (int mi = 0; mi < 4; ++mi)
#pragma unroll
                    for (int ni = 0; ni < 4; ++ni)
                        if (!LOWER || x.tile_lower(mi, ni))
                            dmma_8x8x4(acc.v[mi][ni][0], acc.v[mi][ni][1], a[mi], bf[ni]);
            }
        } else {
#pragma unroll 4
            for (int kl = 0; kl < 16; ++kl) {
                float a[4], bf[4][2];
#pragma unroll
                for (int mi = 0; mi < 4; ++mi) {
                    const int m = x.R(mi);
                    float v;
                    if (AOP == OP_BIG) v = big[SW<T>::idx(m, k0 + kl, BP)];
                    else if (AOP == OP_COLPANEL) v = P[SW<T>::idx(m, kl, 16)];
                    else v = P[SW<T>::idx(kl, m, BP)];
                    a[mi] = NEG ? -v : v;
                }
#pragma unroll
                for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int n = x.C(ni, j);
                        if (BOP == OP_BIG) bf[ni][j] = big[SW<T>::idx(k0 + kl, n, BP)];
                        else if (BOP == OP_COLPANEL) bf[ni][j] = P[SW<T>::idx(n, kl, 16)];
                        else bf[ni][j] = P[SW<T>::idx(kl, n, BP)];
                    }
#pragma unroll
                for (int mi = 0; mi < 4; ++mi)
#pragma unroll
                    for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                        for (int j = 0; j < 2; ++j) acc.v[mi][ni][j] = fmaf(a[mi], bf[ni][j], acc.v[mi][ni][j]);
            }
        }
    }
    __syncthreads();
}

// CTA-wide in-register inverse of a symmetric positive definite block by the
// symmetric Gauss-Jordan sweep: for each pivot k (d = A_kk),
// A_ij -= A_ik A_kj / d, A_ik /= d, A_kj /= d, A_kk = -1/d; the result is
// -A^-1 and is negated.  Column k is broadcast through shared memory (row k
// equals it by symmetry).  The product of the pivots is det A.
template <class T, int BP>
SELINV_DEVINL void spd_inverse(Big<T> &a, T *colbuf, const Ctx<T, BP> &x, LogAcc &det, bool &bad)
{
    constexpr int RW = Geo<BP>::RW;
    for (int kb = 0; kb < RW; ++kb) {
#pragma unroll
        for (int kc = 0; kc < 32; ++kc) {
            const int k = 32 * kb + kc;
            const int nik = kc >> 3, tk = (kc & 7) >> 1, jk = kc & 1;
            T *cb = colbuf + (kc & 1) * BP;
            const bool owner = (x.cw == kb) && (x.t == tk);
            if (owner) {
#pragma unroll
                for (int mi = 0; mi < 4; ++mi) cb[x.R(mi)] = a.v[mi][nik][jk];
            }
            __syncthreads();
            const T d = cb[k];
            if (x.tid == 0) det.mul((double)d);
            const T p = T(1) / d;
            bad |= bad_pivot(d, p);
            T cr[4], cc[4][2];
#pragma unroll
            for (int mi = 0; mi < 4; ++mi) cr[mi] = cb[x.R(mi)] * p;
#pragma unroll
            for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                for (int j = 0; j < 2; ++j) cc[ni][j] = cb[x.C(ni, j)];
#pragma unroll
            for (int mi = 0; mi < 4; ++mi)
#pragma unroll
                for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                    for (int j = 0; j < 2; ++j) a.v[mi][ni][j] = fma(-cr[mi], cc[ni][j], a.v[mi][ni][j]);
#pragma unroll
            for (int mi = 0; mi < 4; ++mi) {
                if (x.R(mi) == k) {
#pragma unroll
                    for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                        for (int j = 0; j < 2; ++j) a.v[mi][ni][j] = (x.C(ni, j) == k) ? -p : cc[ni][j] * p;
                } else if (owner) {
                    a.v[mi][nik][jk] = cr[mi];
                }
            }
        }
        if (x.tid == 0) det.renorm();
    }
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) a.v[mi][ni][0] = -a.v[mi][ni][0], a.v[mi][ni][1] = -a.v[mi][ni][1];
}

// Blocked form of the same sweep for float64: pivots are taken eight at a
// time (block K = columns 8K..8K+7).  With P = A_KK and T_i = A_iK P^-1, one
// block step is
//   A_ij -= T_i A_Kj (i, j not in K),  A_iK = T_i,  A_Kj = T_j^T,  A_KK = -P^-1
// (equal to eight scalar sweep steps).  Per step: the owners of column block K
// publish it (BP x 8, shared); every warp inverts the 8 x 8 P in registers (a
// scalar sweep over one 8 x 8 accumulator tile, so P's eight pivots enter
// det), forms T for its rows and applies the rank-8 update on the FP64 tensor
// cores (k permuted to the accumulator layout, as in the 16 x 16 products);
// T is published for the owners of row block K.  Two barriers per eight
// pivots instead of eight.
// DRAW: also v = R z for the Cholesky factor S = R R^T of the input block
// (z in shared memory, zs[r]; vacc[mi] = (R z) at row R(mi), formed by the
// warps of quadrant column 0).  Block step K meets R's block column K:
// R_KK = chol(P), P being the Schur complement the step pivots on, and
// R_iK = T_i R_KK for the rows below, so v_K += R_KK z_K and v_i += T_i (R_KK z_K).
template <int BP, bool DRAW = false>
SELINV_DEVINL void spd_inverse_blocked(Big<double> &a, double *cbuf, double *tbuf, double *big_scratch,
                                       const Ctx<double, BP> &x, LogAcc &det, bool &bad, const double *zs = nullptr,
                                       double *vacc = nullptr)
{
    constexpr int NB = BP / 8;
    // The matrix stays symmetric through the sweep, so the warps holding a
    // quadrant strictly above the diagonal (rw < cw) do no updates at all:
    // their entries are read from the mirrored lower quadrants (the column
    // block K for rows above quadrant row qK is published, transposed, from
    // row block K), and their tiles are rebuilt from the lower ones at the end.
    const bool upper = x.rw < x.cw;
    if (DRAW) vacc[0] = vacc[1] = vacc[2] = vacc[3] = 0.0;
    for (int K = 0; K < NB; ++K) {
        double *cb = cbuf + (K & 1) * BP * 8;                     // cb[r * 8 + c] = A[r][8K + c]
        double *tb = tbuf + (K & 1) * BP * 8;                     // tb[r * 8 + c] = T[r][c]
        const int qK = K >> 2, tK = K & 3;                        // quadrant and tile holding block K
        if (x.cw == qK && !upper) {                               // publish column block K (rows >= 32 qK)
#pragma unroll
            for (int mi = 0; mi < 4; ++mi) {
#pragma unroll
                for (int n = 0; n < 4; ++n)
                    if (n == tK) {
                        double2 u;
                        u.x = a.v[mi][n][0];
                        u.y = a.v[mi][n][1];
                        *reinterpret_cast<double2 *>(cb + x.R(mi) * 8 + 2 * x.t) = u;
                    }
            }
        }
        if (x.rw == qK && x.cw < qK) {                            // rows above: A[c][8K + r] = A[8K + r][c]
#pragma unroll
            for (int m = 0; m < 4; ++m)
                if (m == tK) {
#pragma unroll
                    for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                        for (int j = 0; j < 2; ++j) cb[x.C(ni, j) * 8 + x.g] = a.v[m][ni][j];
                }
        }
        __syncthreads();
        // P^-1 in registers (accumulator layout of one 8 x 8 tile; symmetric)
        // the warps above the diagonal need neither P^-1 nor T: only the barriers
        double pv[2] = {0.0, 0.0};
        double T[4][2] = {};
        double wk = 0.0;                                          // (R_KK z_K) at row 8K + g
        if (!upper) {
            {
                const double2 u = *reinterpret_cast<const double2 *>(cb + (8 * K + x.g) * 8 + 2 * x.t);
                pv[0] = u.x;
                pv[1] = u.y;
            }
            if (DRAW && x.cw == 0)
                inv8_sweep<true>(pv, x.lane, x.g, x.t, det, bad, x.tid == 0, zs[8 * K + 2 * x.t],
                                 zs[8 * K + 2 * x.t + 1], &wk);
            else
                inv8_sweep(pv, x.lane, x.g, x.t, det, bad, x.tid == 0);
            // T = A_{rows,K} P^-1 for this warp's rows: 4 m-tiles x 2 k-steps
#pragma unroll
            for (int mi = 0; mi < 4; ++mi) {
                const double2 arow = *reinterpret_cast<const double2 *>(cb + x.R(mi) * 8 + 2 * x.t);
                dmma_8x8x4(T[mi][0], T[mi][1], arow.x, pv[0]);
                dmma_8x8x4(T[mi][0], T[mi][1], arow.y, pv[1]);
            }
        }
        if (DRAW && x.cw == 0) {                                  // v at this warp's rows
            const double w0 = shfl(wk, (2 * x.t) << 2), w1 = shfl(wk, (2 * x.t + 1) << 2);
#pragma unroll
            for (int mi = 0; mi < 4; ++mi) {
                const int rb = 4 * x.rw + mi;                         // 8-row block of m-tile mi
                if (rb == K) {
                    vacc[mi] += wk;
                } else if (rb > K) {
                    double s2 = fma(T[mi][0], w0, T[mi][1] * w1);
                    s2 += shfl_xor(s2, 1);
                    s2 += shfl_xor(s2, 2);
                    vacc[mi] += s2;
                }
            }
        }
        if (x.cw == 0) {                                          // publish T (one copy per row)
#pragma unroll
            for (int mi = 0; mi < 4; ++mi) {
                double2 u;
                u.x = T[mi][0];
                u.y = T[mi][1];
                *reinterpret_cast<double2 *>(tb + x.R(mi) * 8 + 2 * x.t) = u;
            }
        }
        // rank-8 update A_ij -= T_i A_Kj, A_Kj = A_jK (symmetric): B fragments from cb
        if (!upper) {
#pragma unroll
            for (int ni = 0; ni < 4; ++ni) {
                const double2 u =
                    *reinterpret_cast<const double2 *>(cb + (32 * x.cw + 8 * ni + x.g) * 8 + 2 * x.t);
#pragma unroll
                for (int mi = 0; mi < 4; ++mi) {
                    dmma_8x8x4(a.v[mi][ni][0], a.v[mi][ni][1], -T[mi][0], u.x);
                    dmma_8x8x4(a.v[mi][ni][0], a.v[mi][ni][1], -T[mi][1], u.y);
                }
            }
        }
        if (x.cw == qK && !upper) {                               // column block K: T (rows outside K)
#pragma unroll
            for (int mi = 0; mi < 4; ++mi)
#pragma unroll
                for (int n = 0; n < 4; ++n)
                    if (n == tK) {
                        a.v[mi][n][0] = T[mi][0];
                        a.v[mi][n][1] = T[mi][1];
                    }
        }
        __syncthreads();                                          // T published
        if (x.rw == qK && !upper) {                               // row block K: T_j^T, diagonal block -P^-1
#pragma unroll
            for (int m = 0; m < 4; ++m)
                if (m == tK) {
#pragma unroll
                    for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                        for (int j = 0; j < 2; ++j) a.v[m][ni][j] = tb[x.C(ni, j) * 8 + x.g];
                    if (x.cw == qK) {
#pragma unroll
                        for (int n = 0; n < 4; ++n)
                            if (n == tK) {
                                a.v[m][n][0] = -pv[0];
                                a.v[m][n][1] = -pv[1];
                            }
                    }
                }
        }
        if (x.tid == 0) det.renorm();
    }
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) a.v[mi][ni][0] = -a.v[mi][ni][0], a.v[mi][ni][1] = -a.v[mi][ni][1];
    // the upper quadrants from their mirrors, through the free resident image
    if (!upper) to_smem<double, BP>(big_scratch, a, x);
    __syncthreads();
    if (upper) {
#pragma unroll
        for (int mi = 0; mi < 4; ++mi)
#pragma unroll
            for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                for (int j = 0; j < 2; ++j) a.v[mi][ni][j] = big_scratch[SW<double>::idx(x.C(ni, j), x.R(mi), BP)];
    }
    __syncthreads();
}

// Row sums (over this thread's columns) of a tile times the vector v, reduced
// over the 4 lanes of a row group: the per-warp partial for rows R(mi).
template <class T, int BP>
SELINV_DEVINL void row_partial(T s[4], const Big<T> &a, const T *v, const Ctx<T, BP> &x)
{
#pragma unroll
    for (int mi = 0; mi < 4; ++mi) {
        T acc = T(0);
#pragma unroll
        for (int ni = 0; ni < 4; ++ni)
#pragma unroll
            for (int j = 0; j < 2; ++j) acc = fma(a.v[mi][ni][j], v[x.C(ni, j)], acc);
        acc += shfl_xor(acc, 1);
        acc += shfl_xor(acc, 2);
        s[mi] = acc;
    }
}

// Column sums (over this thread's rows) of a tile weighted by v, reduced over
// the 8 row groups of the warp: the per-warp partial of (A^T v) for cols C.
template <class T, int BP>
SELINV_DEVINL void col_partial(T s[4][2], const Big<T> &a, const T *v, const Ctx<T, BP> &x)
{
#pragma unroll
    for (int ni = 0; ni < 4; ++ni)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            T acc = T(0);
#pragma unroll
            for (int mi = 0; mi < 4; ++mi) acc = fma(a.v[mi][ni][j], v[x.R(mi)], acc);
            acc += shfl_xor(acc, 4);
            acc += shfl_xor(acc, 8);
            acc += shfl_xor(acc, 16);
            s[ni][j] = acc;
        }
}

template <class T, int BP, bool FULL, bool WANT_G, bool WANT_X, bool SAMPLE = false>
__global__ void __launch_bounds__(Geo<BP>::NT) chain_large_kernel(ChainArgs<T> p)
{
    using X = Ctx<T, BP>;
    constexpr int RW = X::RW;
    constexpr int64_t BB = (int64_t)BP * BP;
    X x;
    x.init();
    const int64_t e = blockIdx.x;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *big = reinterpret_cast<T *>(smem_raw);
    T *pbuf = big + X::BIG;
    T *colbuf = pbuf + 3 * X::PANEL;
    T *ybuf = colbuf + 2 * BP;     // two buffers
    T *xbuf = ybuf + 2 * BP;       // two buffers
    T *red1 = xbuf + 2 * BP;       // [RW][BP]
    T *red2 = red1 + RW * BP;      // [RW][BP]
    T *zs = red2 + RW * BP;        // z_i of a draw

    const int b = p.b;
    const int64_t L = p.L;
    const int64_t bb = (int64_t)b * b;
    const T *D = p.diag + e * L * bb;
    const T *Bl = p.lower + e * (L - 1) * bb;
    T *ws = p.ws + e * (L - 1) * 2 * BB;
    const T *Rv = (WANT_X && p.rhs) ? p.rhs + e * L * b : nullptr;   // a draw may come without a mean
    T *Xv = WANT_X ? p.x + e * L * b : nullptr;
    const T *Zv = SAMPLE ? p.z + e * L * b : nullptr;
    constexpr bool KEEP = WANT_G || WANT_X;

    LogAcc det;
    det.init();
    int fail = -1;

    if (WANT_X && x.tid < BP) {
        const T r0 = (Rv && x.tid < b) ? Rv[x.tid] : T(0);
        ybuf[x.tid] = r0;
        if (x.tid < b) Xv[x.tid] = r0;            // y_0 kept in x until the distribute sweep
    }
    Big<T> a;
    load_sym<T, BP, FULL>(a, D, b, x);
    __syncthreads();

    // ---------------- collect sweep ----------------
    for (int64_t i = 0; i < L; ++i) {
        bool bad = false;
        if (i + 1 < L) {                           // next blocks into L2 while this one is inverted
            prefetch_range_l2(D + (i + 1) * bb, bb, x.tid, Geo<BP>::NT);
            if (i + 1 < L - 1) prefetch_range_l2(Bl + (i + 1) * bb, bb, x.tid, Geo<BP>::NT);
        }
        if constexpr (SAMPLE) {
            // Draw: store y_i + R_i z_i for the backward sweep (S_i = R_i R_i^T), so that
            // S_i^-1 (y_i + R_i z_i) = S_i^-1 y_i + R_i^-T z_i turns x = A^-1 r into
            // eta = A^-1 r + L^-T z.  R_i z_i comes out of the blocked inverse.
            if (x.tid < BP) zs[x.tid] = x.tid < b ? Zv[i * b + x.tid] : T(0);   // visible after its first barrier
            double vacc[4];
            spd_inverse_blocked<BP, true>(a, pbuf, pbuf + 2 * BP * 8, big, x, det, bad, zs, vacc);
            if (x.cw == 0 && x.t == 0) {
#pragma unroll
                for (int mi = 0; mi < 4; ++mi) {
                    const int r = x.R(mi);
                    const T yv = ybuf[BP * (i & 1) + r] + vacc[mi];
                    if (r < b) Xv[i * b + r] = yv;
                    if (i == L - 1) ybuf[BP * (i & 1) + r] = yv;   // the backward sweep starts from S^-1 (y + R z)
                }
            }
        } else if constexpr (sizeof(T) == 8) {
            spd_inverse_blocked<BP>(a, pbuf, pbuf + 2 * BP * 8, big, x, det, bad);
        } else {
            spd_inverse<T, BP>(a, colbuf, x, det, bad);
        }
        if (bad && fail < 0) fail = (int)i;
        if (i == L - 1) break;
        if (KEEP) store_ws<T, BP>(ws + (2 * i) * BB, a, x);
        __syncthreads();
        to_smem<T, BP>(big, a, x);
        __syncthreads();
        zero(a);
        gemm<T, BP, OP_COLPANEL, OP_BIG, false, FULL>(a, big, pbuf, Bl + i * bb, b, x);   // W_i = B_i S_i^-1
        if (KEEP) store_ws<T, BP>(ws + (2 * i + 1) * BB, a, x);
        if (WANT_X) {                              // y_{i+1} = r_{i+1} - W_i y_i
            T s[4];
            row_partial<T, BP>(s, a, ybuf + BP * (i & 1), x);
            if (x.t == 0) {
#pragma unroll
                for (int mi = 0; mi < 4; ++mi) red1[x.cw * BP + x.R(mi)] = s[mi];
            }
        }
        to_smem<T, BP>(big, a, x);                 // big: S_i^-1 no longer read after the gemm
        __syncthreads();
        if (WANT_X && x.tid < BP) {
            T s = T(0);
            for (int c = 0; c < RW; ++c) s += red1[c * BP + x.tid];
            const T r = (Rv && x.tid < b) ? Rv[(i + 1) * b + x.tid] : T(0);
            const T yv = r - s;
            ybuf[BP * ((i + 1) & 1) + x.tid] = yv;
            if (x.tid < b) Xv[(i + 1) * b + x.tid] = yv;
        }
        load_sym<T, BP, FULL>(a, D + (i + 1) * bb, b, x);
        gemm<T, BP, OP_BIG, OP_COLPANEL, true, FULL, true>(a, big, pbuf, Bl + i * bb, b, x);   // S_{i+1} = D_{i+1} - W_i B_i^T (lower)
        to_smem_sym<T, BP>(big, a, x);             // complete the upper triangle (big is free after the gemm)
        __syncthreads();
        from_smem<T, BP>(a, big, x);
    }
    if (x.tid == 0) {
        if (p.logdet) p.logdet[e] = det.log_value();
        p.info[e] = fail;
    }
    if (!KEEP) return;

    // ---------------- distribute sweep ----------------
    __syncthreads();
    to_smem_sym<T, BP>(big, a, x);                 // G_{L-1,L-1} = S_{L-1}^-1, exactly symmetric
    __syncthreads();
    from_smem<T, BP>(a, big, x);
    const int64_t last = L - 1;
    if (WANT_G) store_block<T, BP, FULL>(p.G_diag + e * L * bb + last * bb, a, b, x);
    if (WANT_X) {                                  // x_{L-1} = S_{L-1}^-1 y_{L-1}
        T s[4];
        row_partial<T, BP>(s, a, ybuf + BP * (last & 1), x);
        if (x.t == 0) {
#pragma unroll
            for (int mi = 0; mi < 4; ++mi) red1[x.cw * BP + x.R(mi)] = s[mi];
        }
        __syncthreads();
        if (x.tid < BP) {
            T v = T(0);
            for (int c = 0; c < RW; ++c) v += red1[c * BP + x.tid];
            xbuf[BP * (last & 1) + x.tid] = v;
            if (x.tid < b) Xv[last * b + x.tid] = v;
        }
        __syncthreads();
    }

    for (int64_t i = L - 2; i >= 0; --i) {
        const T *Sinv = ws + (2 * i) * BB;
        const T *W = ws + (2 * i + 1) * BB;
        if (i > 0) prefetch_range_l2(ws + (2 * i - 2) * BB, 2 * BB, x.tid, Geo<BP>::NT);   // S_{i-1}^-1, W_{i-1}
        if (WANT_G) {
            zero(a);
            gemm<T, BP, OP_BIG, OP_ROWPANEL, true, FULL>(a, big, pbuf, W, b, x);          // G_{i+1,i} = -G_{i+1,i+1} W_i
            store_block<T, BP, FULL>(p.G_lower + e * (L - 1) * bb + i * bb, a, b, x);
            to_smem<T, BP>(big, a, x);             // all reads of G_{i+1,i+1} ended at the gemm's last barrier
            __syncthreads();
        }
        load_ws<T, BP>(a, Sinv, x);
        if (WANT_X) {                              // x_i = S_i^-1 y_i - W_i^T x_{i+1}; first half
            if (x.tid < BP) ybuf[x.tid] = x.tid < b ? Xv[i * b + x.tid] : T(0);
            __syncthreads();
            T s[4];
            row_partial<T, BP>(s, a, ybuf, x);
            if (x.t == 0) {
#pragma unroll
                for (int mi = 0; mi < 4; ++mi) red1[x.cw * BP + x.R(mi)] = s[mi];
            }
        }
        if (WANT_G) {
            gemm<T, BP, OP_ROWPANEL, OP_BIG, true, FULL, true>(a, big, pbuf, W, b, x);    // G_ii = S_i^-1 - W_i^T G_{i+1,i} (lower)
            to_smem_sym<T, BP>(big, a, x);
            __syncthreads();
            from_smem<T, BP>(a, big, x);
            store_block<T, BP, FULL>(p.G_diag + e * L * bb + i * bb, a, b, x);
        }
        if (WANT_X) {                              // second half: W_i^T x_{i+1}
            load_ws<T, BP>(a, W, x);
            T s[4][2];
            col_partial<T, BP>(s, a, xbuf + BP * ((i + 1) & 1), x);
            if (x.g == 0) {
#pragma unroll
                for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                    for (int j = 0; j < 2; ++j) red2[x.rw * BP + x.C(ni, j)] = s[ni][j];
            }
            __syncthreads();
            if (x.tid < BP) {
                T v = T(0);
                for (int c = 0; c < RW; ++c) v += red1[c * BP + x.tid] - red2[c * BP + x.tid];
                xbuf[BP * (i & 1) + x.tid] = v;
                if (x.tid < b) Xv[i * b + x.tid] = v;
            }
            __syncthreads();
        }
    }
}

template <class T, int BP, bool FULL, bool G, bool Xs, bool SAMPLE = false>
cudaError_t launch_t(const ChainArgs<T> &a, cudaStream_t s)
{
    const size_t smem = sizeof(T) * smem_elems<T, BP>();
    auto k = chain_large_kernel<T, BP, FULL, G, Xs, SAMPLE>;
    cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    k<<<(unsigned)a.batch, Geo<BP>::NT, smem, s>>>(a);
    return cudaGetLastError();
}

template <class T, int BP, bool FULL>
cudaError_t launch_flags(const ChainArgs<T> &a, cudaStream_t s)
{
    const bool G = a.G_diag != nullptr, Xs = a.x != nullptr;
    if (G && Xs) return launch_t<T, BP, FULL, true, true>(a, s);
    if (G) return launch_t<T, BP, FULL, true, false>(a, s);
    if (Xs) return launch_t<T, BP, FULL, false, true>(a, s);
    return launch_t<T, BP, FULL, false, false>(a, s);
}

template <class T, int BP>
cudaError_t launch_bp(const ChainArgs<T> &a, bool full, cudaStream_t s)
{
    return full ? launch_flags<T, BP, true>(a, s) : launch_flags<T, BP, false>(a, s);
}

int padded(int b) { return b <= 32 ? 32 : (b <= 64 ? 64 : 128); }

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

size_t chain_large_workspace(size_t elem, int64_t batch, int64_t L, int b)
{
    const size_t bp = (size_t)padded(b);
    return (size_t)batch * (size_t)(L > 1 ? L - 1 : 0) * 2 * bp * bp * elem;
}

template <class T> cudaError_t chain_large_launch(const ChainArgs<T> &a, cudaStream_t s)
{
    if (a.batch == 0) return cudaSuccess;
    const int bp = padded(a.b);
    const bool full = a.b == bp && al16(a.diag) && al16(a.lower) && al16(a.G_diag) && al16(a.G_lower);
    if (bp == 32) return launch_bp<T, 32>(a, full, s);
    if (bp == 64) return launch_bp<T, 64>(a, full, s);
    return launch_bp<T, 128>(a, full, s);
}

cudaError_t chain_large_sample_launch(const ChainArgs<double> &a, cudaStream_t s)
{
    if (a.batch == 0) return cudaSuccess;
    const int bp = padded(a.b);
    const bool full = a.b == bp && al16(a.diag) && al16(a.lower);
    if (bp == 32) return full ? launch_t<double, 32, true, false, true, true>(a, s)
                              : launch_t<double, 32, false, false, true, true>(a, s);
    if (bp == 64) return full ? launch_t<double, 64, true, false, true, true>(a, s)
                              : launch_t<double, 64, false, false, true, true>(a, s);
    return full ? launch_t<double, 128, true, false, true, true>(a, s)
                : launch_t<double, 128, false, false, true, true>(a, s);
}

template cudaError_t chain_large_launch<double>(const ChainArgs<double> &, cudaStream_t);
template cudaError_t chain_large_launch<float>(const ChainArgs<float> &, cudaStream_t);

}  // namespace selinv
