// Warp-level toolkit for blocks of size b <= 16: one warp owns one padded
// 16 x 16 block at a time.  Blocks smaller than 16 are embedded with an
// identity (diagonal blocks) or zero (off-diagonal blocks) pad, which leaves
// the unpadded part of every Schur complement and inverse unchanged and adds
// log 1 = 0 to the log-determinant.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace selinv {
namespace w16 {

// Register tile.  Lane = 4 g + t holds rows g + 8 h (h = 0, 1) and columns
// tcol(t, q) = 2 t + (q & 1) + 8 (q >> 1) (q = 0..3): the accumulator layout of
// the m8n8k4 FP64 tensor-core instruction, four of whose 8 x 8 tiles cover the
// 16 x 16 block (tile (h, q >> 1)).
template <class T> struct Tile {
    T v[2][4];
};

SELINV_DEVINL int tcol(int t, int q) { return 2 * t + (q & 1) + 8 * (q >> 1); }

// Shared-memory image of a 16 x 16 block.
//  double: 16 doubles per row (8 chunks of 16 B); the chunk index is XORed
//          with f(r) = 4 ((r ^ (r >> 1)) & 1), which puts rows 2j and 2j+1 in
//          opposite halves of the banks (conflict-free 16-byte pair accesses
//          of the register tile) and splits every set of rows {j, j+2, j+4,
//          j+6} two and two (transposed reads of a tile in two wavefronts).
//  float:  row pitch 20 floats (8-byte pairs stay aligned; column reads of 8
//          rows hit distinct banks).
template <class T> struct SL;
template <> struct SL<double> {
    static constexpr int ELEMS = 256;
    SELINV_DEVINL static int idx(int r, int c)
    {
        const int f = ((r ^ (r >> 1)) & 1) << 2;
        return (r << 4) | ((((c >> 1) ^ f) << 1) | (c & 1));
    }
};
template <> struct SL<float> {
    static constexpr int ELEMS = 16 * 20;
    SELINV_DEVINL static int idx(int r, int c) { return r * 20 + c; }
};

template <class T> struct Vec2;
template <> struct Vec2<double> { using type = double2; };
template <> struct Vec2<float> { using type = float2; };

template <class T> SELINV_DEVINL void zero(Tile<T> &a)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) a.v[h][q] = T(0);
}

// ---- shared memory <-> registers -------------------------------------------

template <class T> SELINV_DEVINL void to_smem(T *s, const Tile<T> &a, int g, int t)
{
    using V = typename Vec2<T>::type;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            V v;
            v.x = a.v[h][2 * p];
            v.y = a.v[h][2 * p + 1];
            *reinterpret_cast<V *>(s + SL<T>::idx(g + 8 * h, 2 * t + 8 * p)) = v;
        }
}

template <class T> SELINV_DEVINL void from_smem(Tile<T> &a, const T *s, int g, int t)
{
    using V = typename Vec2<T>::type;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            V v = *reinterpret_cast<const V *>(s + SL<T>::idx(g + 8 * h, 2 * t + 8 * p));
            a.v[h][2 * p] = v.x;
            a.v[h][2 * p + 1] = v.y;
        }
}

// Writes the lower triangle (c <= r) of the tile and its mirror, so the
// shared image is exactly symmetric and every entry is written once.
template <class T> SELINV_DEVINL void to_smem_sym(T *s, const Tile<T> &a, int g, int t)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = g + 8 * h, c = tcol(t, q);
            if (c <= r) s[SL<T>::idx(r, c)] = a.v[h][q];
            if (c < r) s[SL<T>::idx(c, r)] = a.v[h][q];
        }
}

// ---- global memory -----------------------------------------------------------

// Diagonal block D (row-major b x b) into a tile, reading only D's lower
// triangle (upper entries come from their mirror); identity pad beyond b.
template <class T, bool FULL> SELINV_DEVINL void load_sym(Tile<T> &a, const T *D, int b, int g, int t)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = g + 8 * h, c = tcol(t, q);
            const int rr = c <= r ? r : c, cc = c <= r ? c : r;
            if (FULL) {
                a.v[h][q] = __ldg(D + rr * 16 + cc);
            } else {
                a.v[h][q] = (r < b && c < b) ? __ldg(D + rr * b + cc) : (r == c ? T(1) : T(0));
            }
        }
}

// Lower triangle of a diagonal block D (row-major b x b) into shared memory
// (entries with c <= r; identity pad beyond b).  FULL: 16-byte cp.async
// chunks that touch the lower triangle only (caller commits / waits).
// HINT: the copies carry the L2 eviction policy pol.
template <class T, bool FULL, bool HINT = false>
SELINV_DEVINL void load_lower_async(T *s, const T *D, int b, int lane, uint64_t pol = 0)
{
    if (FULL) {
        constexpr int CH = 16 / sizeof(T);
        constexpr int PER_ROW = 16 / CH;
#pragma unroll
        for (int j = lane; j < 16 * PER_ROW; j += 32) {
            const int r = j / PER_ROW, c = (j % PER_ROW) * CH;
            if (c <= r) {
                if (HINT) cp_async16_hint(s + SL<T>::idx(r, c), D + r * 16 + c, pol);
                else cp_async16(s + SL<T>::idx(r, c), D + r * 16 + c);
            }
        }
    } else {
        for (int j = lane; j < 256; j += 32) {
            const int r = j >> 4, c = j & 15;
            if (c <= r) s[SL<T>::idx(r, c)] = (r < b && c < b) ? __ldg(D + r * b + c) : (r == c ? T(1) : T(0));
        }
    }
}

// Tile from a shared image of which only the lower triangle is valid.
template <class T> SELINV_DEVINL void from_smem_lower(Tile<T> &a, const T *s, int g, int t)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = g + 8 * h, c = tcol(t, q);
            a.v[h][q] = c <= r ? s[SL<T>::idx(r, c)] : s[SL<T>::idx(c, r)];
        }
}

// Off-diagonal block (row-major b x b) into shared memory, zero pad beyond b.
// FULL: 16-byte cp.async chunks (caller commits / waits); else plain loads.
// HINT: the copies carry the L2 eviction policy pol.
template <class T, bool FULL, bool HINT = false>
SELINV_DEVINL void load_block_async(T *s, const T *B, int b, int lane, uint64_t pol = 0)
{
    if (FULL) {
        constexpr int CH = 16 / sizeof(T);          // elements per chunk
        constexpr int PER_ROW = 16 / CH;
#pragma unroll
        for (int j = lane; j < 16 * PER_ROW; j += 32) {
            const int r = j / PER_ROW, c = (j % PER_ROW) * CH;
            if (HINT) cp_async16_hint(s + SL<T>::idx(r, c), B + r * 16 + c, pol);
            else cp_async16(s + SL<T>::idx(r, c), B + r * 16 + c);
        }
    } else {
        for (int j = lane; j < 256; j += 32) {
            const int r = j >> 4, c = j & 15;
            s[SL<T>::idx(r, c)] = (r < b && c < b) ? __ldg(B + r * b + c) : T(0);
        }
    }
}

// Full tile to a row-major b x b block in global memory.
template <class T, bool FULL> SELINV_DEVINL void store_block(T *G, const Tile<T> &a, int b, int g, int t)
{
    using V = typename Vec2<T>::type;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int r = g + 8 * h, c = 2 * t + 8 * p;
            if (FULL) {
                V v;
                v.x = a.v[h][2 * p];
                v.y = a.v[h][2 * p + 1];
                __stcs(reinterpret_cast<V *>(G + r * 16 + c), v);
            } else {
                if (r < b && c < b) G[r * b + c] = a.v[h][2 * p];
                if (r < b && c + 1 < b) G[r * b + c + 1] = a.v[h][2 * p + 1];
            }
        }
}

// Transposed tile to a row-major b x b block: G[c][r] = a[r][c].  For each
// register the warp writes four runs of eight consecutive elements.
template <class T, bool FULL> SELINV_DEVINL void store_block_T(T *G, const Tile<T> &a, int b, int g, int t)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = g + 8 * h, c = tcol(t, q);
            if (FULL) __stcs(G + c * 16 + r, a.v[h][q]);
            else if (r < b && c < b) G[c * b + r] = a.v[h][q];
        }
}

// Lower-triangle slot of a symmetric tile in workspace memory (192 elements):
// [0, 64): rows 8..15 x cols 0..7, two entries per lane;
// [64, 192): the two diagonal 8 x 8 tiles' entries of lanes with 2t <= g,
// four per lane.  Exactly the entries with c <= r (plus four on the
// diagonal pairs) are kept; to_smem_sym rebuilds the full block.
constexpr int SLOT_ELEMS = 192;

// HINT: the stores carry the L2 eviction policy pol.
template <class T, bool HINT = false>
SELINV_DEVINL void store_lower_slot(T *slot, const Tile<T> &a, int lane, int g, int t, uint64_t pol = 0)
{
    using V = typename Vec2<T>::type;
    auto put = [&](T *p, V v) {
        if (HINT) st_hint(reinterpret_cast<V *>(p), v, pol);
        else *reinterpret_cast<V *>(p) = v;
    };
    V v;
    v.x = a.v[1][0];
    v.y = a.v[1][1];
    put(slot + 2 * lane, v);
    if (2 * t <= g) {
        V u, w;
        u.x = a.v[0][0];
        u.y = a.v[0][1];
        w.x = a.v[1][2];
        w.y = a.v[1][3];
        put(slot + 64 + 4 * lane, u);
        put(slot + 64 + 4 * lane + 2, w);
    }
}

// Drop a slot's L2 lines without writing them back once the slot has been
// read (lanes 0.. take one 128-byte line each; the slot must start on a
// 128-byte boundary, which the launchers check).
template <class T> SELINV_DEVINL void discard_slot(const T *slot, int lane)
{
    constexpr int LINES = SLOT_ELEMS * (int)sizeof(T) / 128;
    static_assert(SLOT_ELEMS * sizeof(T) % 128 == 0, "slots are whole L2 lines");
    if (lane < LINES) discard_l2_line(reinterpret_cast<const char *>(slot) + 128 * lane);
}

template <class T> SELINV_DEVINL void load_lower_slot(Tile<T> &a, const T *slot, int lane, int g, int t)
{
    using V = typename Vec2<T>::type;
    V v = __ldcs(reinterpret_cast<const V *>(slot + 2 * lane));
    a.v[1][0] = v.x;
    a.v[1][1] = v.y;
    a.v[0][2] = a.v[0][3] = T(0);
    if (2 * t <= g) {
        V u = __ldcs(reinterpret_cast<const V *>(slot + 64 + 4 * lane));
        V w = __ldcs(reinterpret_cast<const V *>(slot + 64 + 4 * lane + 2));
        a.v[0][0] = u.x;
        a.v[0][1] = u.y;
        a.v[1][2] = w.x;
        a.v[1][3] = w.y;
    } else {
        a.v[0][0] = a.v[0][1] = a.v[1][2] = a.v[1][3] = T(0);
    }
}

// The same slot copied to shared memory by each lane for itself (cp.async;
// the caller commits / waits), then read back by the same lane.
template <class T, bool HINT = false>
SELINV_DEVINL void stage_lower_slot(T *stg, const T *slot, int lane, int g, int t, uint64_t pol = 0)
{
    constexpr int CH = 16 / sizeof(T);          // elements per 16-byte chunk
    if (CH == 2) {
        auto cp = [&](T *d, const T *src) {
            if (HINT) cp_async16_hint(d, src, pol);
            else cp_async16(d, src);
        };
        cp(stg + 2 * lane, slot + 2 * lane);
        if (2 * t <= g) {
            cp(stg + 64 + 4 * lane, slot + 64 + 4 * lane);
            cp(stg + 64 + 4 * lane + 2, slot + 64 + 4 * lane + 2);
        }
    } else {                                    // float: 8-byte pairs, plain loads
        *reinterpret_cast<typename Vec2<T>::type *>(stg + 2 * lane) =
            *reinterpret_cast<const typename Vec2<T>::type *>(slot + 2 * lane);
        if (2 * t <= g) {
            *reinterpret_cast<typename Vec2<T>::type *>(stg + 64 + 4 * lane) =
                *reinterpret_cast<const typename Vec2<T>::type *>(slot + 64 + 4 * lane);
            *reinterpret_cast<typename Vec2<T>::type *>(stg + 64 + 4 * lane + 2) =
                *reinterpret_cast<const typename Vec2<T>::type *>(slot + 64 + 4 * lane + 2);
        }
    }
}

template <class T> SELINV_DEVINL void unstage_lower_slot(Tile<T> &a, const T *stg, int lane, int g, int t)
{
    using V = typename Vec2<T>::type;
    V v = *reinterpret_cast<const V *>(stg + 2 * lane);
    a.v[1][0] = v.x;
    a.v[1][1] = v.y;
    a.v[0][2] = a.v[0][3] = T(0);
    if (2 * t <= g) {
        V u = *reinterpret_cast<const V *>(stg + 64 + 4 * lane);
        V w = *reinterpret_cast<const V *>(stg + 64 + 4 * lane + 2);
        a.v[0][0] = u.x;
        a.v[0][1] = u.y;
        a.v[1][2] = w.x;
        a.v[1][3] = w.y;
    } else {
        a.v[0][0] = a.v[0][1] = a.v[1][2] = a.v[1][3] = T(0);
    }
}

// ---- arithmetic --------------------------------------------------------------

// Transposed copy of a tile: out[r][c] = in[c][r], through the shared image s
// (the caller makes s free before and syncs before reusing it).
template <class T> SELINV_DEVINL void from_smem_T(Tile<T> &a, const T *s, int g, int t)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) a.v[h][q] = s[SL<T>::idx(tcol(t, q), g + 8 * h)];
}

// Readers of an S-typed shared image into a tile of element type A (a float
// image widened into a float64 tile; the same reader when A = S).
template <class A, class S> SELINV_DEVINL void from_smem_as(Tile<A> &a, const S *s, int g, int t)
{
    if constexpr (std::is_same<A, S>::value) {
        from_smem<S>(a, s, g, t);
    } else {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) a.v[h][q] = (A)s[SL<S>::idx(g + 8 * h, tcol(t, q))];
    }
}
template <class A, class S> SELINV_DEVINL void from_smem_T_as(Tile<A> &a, const S *s, int g, int t)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) a.v[h][q] = (A)s[SL<S>::idx(tcol(t, q), g + 8 * h)];
}
template <class A, class S> SELINV_DEVINL void from_smem_lower_as(Tile<A> &a, const S *s, int g, int t)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = g + 8 * h, c = tcol(t, q);
            a.v[h][q] = (A)(c <= r ? s[SL<S>::idx(r, c)] : s[SL<S>::idx(c, r)]);
        }
}

// acc += (NEG ? -1 : 1) X Y^T for register tiles X, Y (16 x 16).
//
// double: the FP64 tensor cores.  Each m8n8k4 step s = 0..3 lets lane t carry
// k = 2t, 2t+1, 8+2t, 9+2t respectively (any assignment of the k index that
// both operands share gives the same sum), so the A fragment of row tile m is
// the lane's own X.v[m][s] and the B fragment of column tile n is Y.v[n][s]:
// no data movement at all.  LOWER skips the upper-right 8 x 8 tile of the
// result (products known to be symmetric, rebuilt from the lower half).
// float: plain FMAs from shared copies of X and Y (sX, sY: two free 16 x 16
// images), X and Y written there first.
template <bool NEG, bool LOWER = false>
SELINV_DEVINL void gemm_nt(Tile<double> &acc, const Tile<double> &X, const Tile<double> &Y, double *, double *,
                           int, int)
{
#pragma unroll
    for (int st = 0; st < 4; ++st) {
        const double a0 = NEG ? -X.v[0][st] : X.v[0][st];
        const double a1 = NEG ? -X.v[1][st] : X.v[1][st];
        dmma_8x8x4(acc.v[0][0], acc.v[0][1], a0, Y.v[0][st]);
        if (!LOWER) dmma_8x8x4(acc.v[0][2], acc.v[0][3], a0, Y.v[1][st]);
        dmma_8x8x4(acc.v[1][0], acc.v[1][1], a1, Y.v[0][st]);
        dmma_8x8x4(acc.v[1][2], acc.v[1][3], a1, Y.v[1][st]);
    }
}

template <bool NEG, bool LOWER = false>
SELINV_DEVINL void gemm_nt(Tile<float> &acc, const Tile<float> &X, const Tile<float> &Y, float *sX, float *sY,
                           int g, int t)
{
    using L = SL<float>;
    __syncwarp();
    to_smem<float>(sX, X, g, t);
    to_smem<float>(sY, Y, g, t);
    __syncwarp();
#pragma unroll 4
    for (int k = 0; k < 16; ++k) {
        float a[2], b[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) a[h] = NEG ? -sX[L::idx(g + 8 * h, k)] : sX[L::idx(g + 8 * h, k)];
#pragma unroll
        for (int q = 0; q < 4; ++q) b[q] = sY[L::idx(tcol(t, q), k)];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc.v[h][q] = fmaf(a[h], b[q], acc.v[h][q]);
    }
    __syncwarp();
}

// In-register inverse of a symmetric positive definite tile by the symmetric
// sweep form of Gauss-Jordan elimination (no pivoting): for k = 0..15,
// with d = A_kk,  A_ij -= A_ik A_kj / d (i, j != k),  A_ik /= d,  A_kj /= d,
// A_kk = -1/d; after all k the tile holds -A^-1, which is negated.  The
// pivots d are the successive Schur-complement pivots, so their product is
// det A (multiplied into `det`); a pivot that is not > 0 sets `bad`.
// float32 (one pivot per step): column k is broadcast through `cbuf` (2 x 16
// elements of shared memory, alternating per step so one __syncwarp per step
// suffices); row k is read from the same buffer, the matrix being symmetric.
// float64 (two block steps of eight pivots):  with K = {8K..8K+7}, H the
// other half, P = A_KK (the accumulator tile (K, K) itself) and T = A_HK P^-1,
//   A_HH -= T A_KH,  A_HK = T,  A_KH = T^T,  A_KK = -P^-1,
// which equals eight scalar sweep steps.  P^-1 is an 8 x 8 register sweep
// (shuffles only), T and the rank-8 update are FP64 tensor-core MMAs whose
// k index follows the accumulator layout (P^-1 and A_HK symmetric partners
// supply the B fragments from the lane's own registers), and T^T is formed
// by shuffles.  No shared memory, no barrier.
// DRAW: also v = R z for the Cholesky factor S = R R^T of the input tile
// (zc[q] = z at the lane's column tcol(t, q); v[h] = (R z) at row g + 8h).
// The block steps meet R block by block: R_KK = chol(P) of the pivot block as
// the step finds it (a Schur complement), and below it R_HK = T R_KK, so
//   v_K += R_KK z_K,  v_H += T (R_KK z_K)   (the second only for K = 0);
// R_KK z_K comes out of the pivot block's own sweep.
template <bool DRAW = false>
SELINV_DEVINL void spd_inverse_blocked(Tile<double> &a, int g, int t, LogAcc &det, bool &bad,
                                       const double *zc = nullptr, double *v = nullptr)
{
    const int lane = 4 * g + t;
    if (DRAW) v[0] = v[1] = 0.0;
#pragma unroll
    for (int K = 0; K < 2; ++K) {
        const int H = 1 - K;
        double pv[2] = {a.v[K][2 * K], a.v[K][2 * K + 1]};
        double wk = 0.0;                                  // (R_KK z_K) at row 8K + g
        inv8_sweep<DRAW>(pv, lane, g, t, det, bad, true, DRAW ? zc[2 * K] : 0.0, DRAW ? zc[2 * K + 1] : 0.0, &wk);
        if (DRAW) v[K] += wk;
        double t0 = 0.0, t1 = 0.0;                        // T = A_HK P^-1
        dmma_8x8x4(t0, t1, a.v[H][2 * K], pv[0]);
        dmma_8x8x4(t0, t1, a.v[H][2 * K + 1], pv[1]);
        if (DRAW && K == 0) {                             // v_H += T (R_00 z_0); T at rows 8 + g
            const double w0 = shfl(wk, (2 * t) << 2), w1 = shfl(wk, (2 * t + 1) << 2);
            double s2 = fma(t0, w0, t1 * w1);
            s2 += shfl_xor(s2, 1);
            s2 += shfl_xor(s2, 2);
            v[H] += s2;
        }
        // A_HH -= T A_KH, with A_KH[k][c] = A_HK[c][k]
        dmma_8x8x4(a.v[H][2 * H], a.v[H][2 * H + 1], -t0, a.v[H][2 * K]);
        dmma_8x8x4(a.v[H][2 * H], a.v[H][2 * H + 1], -t1, a.v[H][2 * K + 1]);
        double tt[2];                                     // T^T: lane (g, t) needs T[2t + j][g]
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int src = ((2 * t + j) << 2) | (g >> 1);
            const double u0 = shfl(t0, src), u1 = shfl(t1, src);
            tt[j] = (g & 1) ? u1 : u0;
        }
        a.v[H][2 * K] = t0;
        a.v[H][2 * K + 1] = t1;
        a.v[K][2 * H] = tt[0];
        a.v[K][2 * H + 1] = tt[1];
        a.v[K][2 * K] = -pv[0];
        a.v[K][2 * K + 1] = -pv[1];
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) a.v[h][q] = -a.v[h][q];
}

// DRAW: also v[h] = (R z)[g + 8h] for the Cholesky factor A = R R^T, z at the
// lane's columns tcol(t, q) (zc[q]): the column k published at step k holds,
// in the rows not yet swept (i >= k), the Schur-complement column that
// Cholesky scales, R_ik = A_ik / sqrt(d), so v_i += A_ik z_k / sqrt(d).
template <class T, bool DRAW = false>
SELINV_DEVINL void spd_inverse_scalar(Tile<T> &a, T *cbuf, int g, int t, LogAcc &det, bool &bad,
                                      const T *zc = nullptr, T *v = nullptr)
{
    using V = typename Vec2<T>::type;
    if (DRAW) v[0] = v[1] = T(0);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const int kh = k >> 3, kt = (k & 7) >> 1, kq = (k & 1) | ((k >> 3) << 1);
        T *cb = cbuf + 16 * (k & 1);
        if (t == kt) {                      // the 8 lanes owning column k publish it
            cb[g] = a.v[0][kq];
            cb[g + 8] = a.v[1][kq];
        }
        __syncwarp();
        const T d = cb[k];
        const T c0 = cb[g], c1 = cb[g + 8];
        const V r01 = *reinterpret_cast<const V *>(cb + 2 * t);
        const V r23 = *reinterpret_cast<const V *>(cb + 2 * t + 8);
        const T row[4] = {r01.x, r01.y, r23.x, r23.y};
        det.mul((double)d);
        const T p = recip(d);
        bad |= bad_pivot(d, p);
        if (DRAW) {
            const T s = shfl(zc[kq], kt) * rsqrt_t(d);
            if (g >= k) v[0] = fma(c0, s, v[0]);
            if (g + 8 >= k) v[1] = fma(c1, s, v[1]);
        }
        const T tc[2] = {c0 * p, c1 * p};
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) a.v[h][q] = fma(-tc[h], row[q], a.v[h][q]);
        if (t == kt) {                      // column k: A_ik / d
            a.v[0][kq] = tc[0];
            a.v[1][kq] = tc[1];
        }
        if (g == (k & 7)) {                 // row k: A_kj / d, and A_kk = -1/d
#pragma unroll
            for (int q = 0; q < 4; ++q) a.v[kh][q] = row[q] * p;
            if (t == kt) a.v[kh][kq] = -p;
        }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) a.v[h][q] = -a.v[h][q];
}

// float: one pivot at a time; double: two 8-pivot block steps on the tensor cores.
template <class T> SELINV_DEVINL void spd_inverse(Tile<T> &a, T *cbuf, int g, int t, LogAcc &det, bool &bad)
{
    if constexpr (sizeof(T) == 8) spd_inverse_blocked(a, g, t, det, bad);
    else spd_inverse_scalar(a, cbuf, g, t, det, bad);
}

// Upper-right 8 x 8 tile of a symmetric tile set to the transpose of the
// lower-left one, by shuffles: lane (g, t) takes A[8 + 2t + j][g] from lane
// 4 (2t + j) + g / 2, register g & 1.
template <class T> SELINV_DEVINL void mirror_upper(Tile<T> &a, int g, int t)
{
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int src = ((2 * t + j) << 2) | (g >> 1);
        const T u0 = shfl(a.v[1][0], src), u1 = shfl(a.v[1][1], src);
        a.v[0][2 + j] = (g & 1) ? u1 : u0;
    }
}

// y_r = sum_c A[r][c] x[c] for the lane's rows g, g + 8 (x in shared memory);
// every lane of a row group ends with the full sums.
template <class T> SELINV_DEVINL void row_matvec(T out[2], const Tile<T> &a, const T *x, int t)
{
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        T s = T(0);
#pragma unroll
        for (int q = 0; q < 4; ++q) s = fma(a.v[h][q], x[tcol(t, q)], s);
        s += shfl_xor(s, 1);
        s += shfl_xor(s, 2);
        out[h] = s;
    }
}

}  // namespace w16
}  // namespace selinv
