// Block-tridiagonal chains with b <= 16: one warp per chain.
//
// gabp-sparse-inv 0.3.2 (PyPI page), "Implemented and tested kernels" ->
// Chain: block LDL^T of the chain, then the Takahashi back-recursion.  The
// whole per-chain computation is one fused kernel: the collect sweep
// (Schur complements, the log-determinant and the forward half of the
// solve) runs i = 0..L-1 keeping S_i in registers; the distribute sweep
// (G blocks and the backward half of the solve) runs i = L-2..0.
//
// Per block i the warp holds S_i as a register tile, inverts it in
// registers (symmetric Gauss-Jordan sweep, pivots -> log det), and forms
//   W_i = B_i S_i^-1,  S_{i+1} = D_{i+1} - W_i B_i^T          (collect)
//   G_{i+1,i} = -G_{i+1,i+1} W_i,  G_ii = S_i^-1 - W_i^T G_{i+1,i}  (distribute)
// (G_ii = S_i^-1 - S_i^-1 B_i^T G_{i+1,i} with S_i^-1 B_i^T = W_i^T).  The
// products run on the FP64 tensor cores (m8n8k4) straight from registers;
// the distribute sweep forms W_i^T and G_{i+1,i}^T directly, so nothing is
// transposed (G_{i+1,i} is written out by a transposed store).
// Between the sweeps only the lower triangle of each S_i^-1 is kept, in the
// caller's workspace; W_i is recomputed from B_i in the distribute sweep,
// which moves fewer bytes than storing it.
#include "kernels.h"
#include "warp16.cuh"

namespace selinv {

namespace {

constexpr int WARPS = 4;                 // chains per CTA of the several-right-hand-side kernel

// Chains (warps) per CTA of the selected-inverse kernel, and the resident CTAs
// per SM its register allocation is sized for.
#ifndef SELINV_CHAIN_WARPS
#define SELINV_CHAIN_WARPS 1
#endif
#ifndef SELINV_CHAIN_MINB
#define SELINV_CHAIN_MINB 16
#endif
constexpr int CWARPS = SELINV_CHAIN_WARPS;

// L2 use between the sweeps.  The distribute sweep reads the S_i^-1 slots
// and the B_i back in reverse order, so those of a chain's last blocks are
// read soon after the collect sweep left them.  Mode 3 (default): D is copied
// in with an evict-first policy (read once), B keeps normal priority (the
// distribute sweep reads it again), G leaves through streaming stores, and
// every slot is dropped from L2 once staged (it is dead then, so it is never
// written back).  Mode 1 also copies B evict-first; mode 2 adds evict-last
// stores for the slots of the last L2_KEEP blocks; mode 0 uses no hints.  On
// 4096 chains of 64 blocks of 16 the slot discards cut DRAM traffic by 7 %
// (measured) while the time stays within 0.5 % across modes 0, 1 and 3: this
// kernel is bound by its dependency chains, not by HBM.
#ifndef SELINV_L2MODE
#define SELINV_L2MODE 3
#endif

constexpr int WS_ELEMS = w16::SLOT_ELEMS;   // workspace per block: the S_i^-1 slot
#ifndef SELINV_L2KEEP
#define SELINV_L2KEEP 64
#endif

template <class T> __host__ __device__ constexpr int warp_smem_elems()
{
    return 4 * w16::SL<T>::ELEMS + w16::SLOT_ELEMS + 96;
}

template <class T, bool FULL, bool WANT_G, bool WANT_X, bool SAMPLE = false>
__global__ void __launch_bounds__(CWARPS * 32, SELINV_CHAIN_MINB) chain_small_kernel(ChainArgs<T> p)
{
    using namespace w16;
    constexpr int E = SL<T>::ELEMS;
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t e = (int64_t)blockIdx.x * CWARPS + wid;
    if (e >= p.batch) return;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *sbase = reinterpret_cast<T *>(smem_raw) + wid * warp_smem_elems<T>();
    T *sB = sbase;             // B_i
    T *sD = sB + E;            // D_{i+1} (lower triangle)
    T *sT = sD + E;            // transposes / mirrors
    T *sT2 = sT + E;           // second transpose buffer
    T *stg = sT2 + E;          // staged S_i^-1 slot (distribute sweep)
    T *sy = stg + SLOT_ELEMS;  // y vectors, two buffers of 16
    T *sx = sy + 32;           // x vectors, two buffers of 16
    T *cb = sx + 32;           // pivot-column broadcast, two buffers of 16

    const int b = p.b;
    const int64_t L = p.L;
    const int64_t bb = (int64_t)b * b;
    const T *D = p.diag + e * L * bb;
    const T *Bl = p.lower + e * (L - 1) * bb;
    T *ws = (WANT_G || WANT_X) ? p.ws + e * (L - 1) * WS_ELEMS : nullptr;
    const T *R = (WANT_X && p.rhs) ? p.rhs + e * L * b : nullptr;   // a draw may come without a mean
    T *X = WANT_X ? p.x + e * L * b : nullptr;
    const T *Zv = SAMPLE ? p.z + e * L * b : nullptr;

    LogAcc det;
    det.init();
    int fail = -1;

    constexpr bool HINT = FULL && SELINV_L2MODE > 0;
    constexpr bool HINT_B = HINT && SELINV_L2MODE != 3;   // mode 3: B_i keeps normal priority in the collect
    const uint64_t pol_first = HINT ? l2_evict_first() : 0;
    const uint64_t pol_keep = (HINT && SELINV_L2MODE == 2) ? l2_evict_last() : 0;
    const bool drop = HINT && p.ws_lines;
    Tile<T> a, w, bt;
    load_lower_async<T, FULL, HINT>(sD, D, b, lane, pol_first);
    cp_async_commit();
    cp_async_wait_all();
    __syncwarp();
    from_smem_lower<T>(a, sD, g, t);
    __syncwarp();
    if (L > 1) {
        load_block_async<T, FULL, HINT_B>(sB, Bl, b, lane, pol_first);
        load_lower_async<T, FULL, HINT>(sD, D + bb, b, lane, pol_first);
        cp_async_commit();
    }
    T rn[2] = {T(0), T(0)};    // r_{i+1} at rows g, g+8 (lanes with t == 0)
    T zc[4] = {T(0), T(0), T(0), T(0)};   // z_i at the lane's columns (draws)
    if (WANT_X) {
        if (lane < 16) {
            const T r0 = (R && lane < b) ? R[lane] : T(0);
            sy[lane] = r0;
            if (lane < b) X[lane] = r0;        // y_0 kept in x until the distribute sweep
        }
        if (R && L > 1 && t == 0) {
            rn[0] = g < b ? R[b + g] : T(0);
            rn[1] = g + 8 < b ? R[b + g + 8] : T(0);
        }
    }
    if (SAMPLE) {
#pragma unroll
        for (int q = 0; q < 4; ++q) zc[q] = tcol(t, q) < b ? Zv[tcol(t, q)] : T(0);
    }
    __syncwarp();

    // ---------------- collect sweep ----------------
    for (int64_t i = 0; i < L; ++i) {
        bool bad = false;
        // Draw: with S_i = R_i R_i^T, S_i^-1 (y_i + R_i z_i) = S_i^-1 y_i + R_i^-T z_i, so
        // storing y_i + R_i z_i for the backward sweep turns its x = A^-1 r into
        // eta = A^-1 r + L^-T z (L^-T z_i = R_i^-T z_i - W_i^T (L^-T z)_{i+1}).
        // The inverse's own pivot sweep meets R_i z_i on the way.
        T v[2] = {T(0), T(0)};
        if constexpr (SAMPLE && sizeof(T) == 8) {
            spd_inverse_blocked<true>(a, g, t, det, bad, zc, v);   // a = S_i^-1, v = R_i z_i
        } else if constexpr (SAMPLE) {
            spd_inverse_scalar<T, true>(a, cb, g, t, det, bad, zc, v);
        } else {
            spd_inverse<T>(a, cb, g, t, det, bad);    // a = S_i^-1
        }
        if (SAMPLE) {
            T *ycur = sy + 16 * (i & 1);
            if (t == 0) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int r = g + 8 * h;
                    const T yv = ycur[r] + v[h];
                    if (r < b) X[i * b + r] = yv;
                    if (i == L - 1) ycur[r] = yv;     // the backward sweep starts from S^-1 (y + R z)
                }
            }
            if (i + 1 < L) {
#pragma unroll
                for (int q = 0; q < 4; ++q) zc[q] = tcol(t, q) < b ? Zv[(i + 1) * b + tcol(t, q)] : T(0);
            }
            __syncwarp();
        }
        det.renorm();
        if (bad && fail < 0) fail = (int)i;
        if (i == L - 1) break;

        if (WANT_G || WANT_X) {
            if (HINT && SELINV_L2MODE == 2)
                store_lower_slot<T, true>(ws + i * WS_ELEMS, a, lane, g, t,
                                          L - 1 - i <= SELINV_L2KEEP ? pol_keep : pol_first);
            else
                store_lower_slot<T>(ws + i * WS_ELEMS, a, lane, g, t);
        }
        cp_async_wait_all();
        __syncwarp();
        from_smem<T>(bt, sB, g, t);                   // B_i
        Tile<T> dn;
        from_smem_lower<T>(dn, sD, g, t);             // D_{i+1}
        zero(w);
        gemm_nt<false>(w, bt, a, sT, sT2, g, t);      // W_i = B_i S_i^-1  (S_i^-1 symmetric)
        gemm_nt<true, true>(dn, w, bt, sT, sT2, g, t);   // S_{i+1} = D_{i+1} - W_i B_i^T (lower tiles)
        mirror_upper(dn, g, t);                       // upper-right tile from the lower-left one
        a = dn;

        if (WANT_X) {                                 // y_{i+1} = r_{i+1} - W_i y_i
            T s2[2];
            row_matvec<T>(s2, w, sy + 16 * (i & 1), t);
            if (t == 0) {
                T *ynext = sy + 16 * ((i + 1) & 1);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int r = g + 8 * h;
                    const T yv = rn[h] - s2[h];
                    ynext[r] = yv;
                    if (r < b) X[(i + 1) * b + r] = yv;
                }
            }
        }
        __syncwarp();
        if (i + 1 < L - 1) {
            load_block_async<T, FULL, HINT_B>(sB, Bl + (i + 1) * bb, b, lane, pol_first);
            load_lower_async<T, FULL, HINT>(sD, D + (i + 2) * bb, b, lane, pol_first);
            cp_async_commit();
            if (R && t == 0) {
                rn[0] = g < b ? R[(i + 2) * b + g] : T(0);
                rn[1] = g + 8 < b ? R[(i + 2) * b + g + 8] : T(0);
            }
        }
    }
    if (lane == 0) {
        if (p.logdet) p.logdet[e] = det.log_value();
        p.info[e] = fail;
    }
    if (!(WANT_G || WANT_X)) return;

    // ---------------- distribute sweep ----------------
    // G = S_{L-1}^-1 = G_{L-1,L-1}, made exactly symmetric; kept in registers.
    Tile<T> G;
    __syncwarp();
    to_smem<T>(sT, a, g, t);
    __syncwarp();
    from_smem_lower<T>(G, sT, g, t);
    if (WANT_G) store_block<T, FULL>(p.G_diag + e * L * bb + (L - 1) * bb, G, b, g, t);

    const int64_t last = L - 1;
    // Backward solve in row form: lane (g, t) keeps x_{i+1} at rows g, g + 8
    // (xr) and reads y_i at its four columns tcol(t, q) (yc).
    T xr[2] = {T(0), T(0)};
    T yc[4] = {T(0), T(0), T(0), T(0)};
    if (WANT_X) {               // x_{L-1} = S_{L-1}^-1 y_{L-1}
        const T *y = sy + 16 * (last & 1);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            T s2 = T(0);
#pragma unroll
            for (int q = 0; q < 4; ++q) s2 = fma(G.v[h][q], y[tcol(t, q)], s2);
            s2 += shfl_xor(s2, 1);
            s2 += shfl_xor(s2, 2);
            xr[h] = s2;
        }
        if (t == 0) {
            if (g < b) X[last * b + g] = xr[0];
            if (g + 8 < b) X[last * b + g + 8] = xr[1];
        }
        if (L > 1) {
#pragma unroll
            for (int q = 0; q < 4; ++q) yc[q] = tcol(t, q) < b ? X[(last - 1) * b + tcol(t, q)] : T(0);
        }
    }
    __syncwarp();
    if (L > 1) {
        load_block_async<T, FULL, HINT>(sB, Bl + (L - 2) * bb, b, lane, pol_first);
        stage_lower_slot<T, HINT>(stg, ws + (L - 2) * WS_ELEMS, lane, g, t, pol_first);
        cp_async_commit();
    }

    // W_i^T = S_i^-1 B_i^T and G_{i+1,i}^T = -W_i^T G_{i+1,i+1} are products of
    // the form X Y^T of register tiles (S_i^-1 and G_{i+1,i+1} symmetric), so no
    // operand is ever transposed; G_{i+1,i} leaves through a transposed store.
    for (int64_t i = L - 2; i >= 0; --i) {
        T yi[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) yi[q] = yc[q];
        cp_async_wait_all();
        unstage_lower_slot<T>(a, stg, lane, g, t);
        if (drop) discard_slot<T>(ws + i * WS_ELEMS, lane);   // dead once staged
        to_smem<T>(sT, a, g, t);                      // lower entries valid
        __syncwarp();
        from_smem_lower<T>(a, sT, g, t);              // S_i^-1, full and symmetric
        from_smem<T>(bt, sB, g, t);                   // B_i
        __syncwarp();
        if (i > 0) {
            load_block_async<T, FULL, HINT>(sB, Bl + (i - 1) * bb, b, lane, pol_first);
            stage_lower_slot<T, HINT>(stg, ws + (i - 1) * WS_ELEMS, lane, g, t, pol_first);
            cp_async_commit();
            if (WANT_X) {
#pragma unroll
                for (int q = 0; q < 4; ++q) yc[q] = tcol(t, q) < b ? X[(i - 1) * b + tcol(t, q)] : T(0);
            }
        }
        Tile<T> wt;
        zero(wt);
        gemm_nt<false>(wt, a, bt, sT, sT2, g, t);     // W_i^T = S_i^-1 B_i^T

        if (WANT_X) {                                 // x_i = S_i^-1 y_i - W_i^T x_{i+1}
            T xc[4];                                  // x_{i+1} at the lane's columns
            xc[0] = shfl(xr[0], (2 * t) << 2);
            xc[1] = shfl(xr[0], (2 * t + 1) << 2);
            xc[2] = shfl(xr[1], (2 * t) << 2);
            xc[3] = shfl(xr[1], (2 * t + 1) << 2);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                T s2 = T(0);
#pragma unroll
                for (int q = 0; q < 4; ++q) s2 = fma(a.v[h][q], yi[q], fma(-wt.v[h][q], xc[q], s2));
                s2 += shfl_xor(s2, 1);
                s2 += shfl_xor(s2, 2);
                xr[h] = s2;
            }
            if (t == 0) {
                if (g < b) X[i * b + g] = xr[0];
                if (g + 8 < b) X[i * b + g + 8] = xr[1];
            }
        }
        if (WANT_G) {
            Tile<T> glt;
            zero(glt);
            gemm_nt<true>(glt, wt, G, sT, sT2, g, t);          // G_{i+1,i}^T = -W_i^T G_{i+1,i+1}
            store_block_T<T, FULL>(p.G_lower + e * (L - 1) * bb + i * bb, glt, b, g, t);
            gemm_nt<true, true>(a, wt, glt, sT, sT2, g, t);    // G_ii = S_i^-1 - W_i^T G_{i+1,i} (lower tiles)
            __syncwarp();
            to_smem<T>(sT, a, g, t);
            __syncwarp();
            from_smem_lower<T>(G, sT, g, t);          // exactly symmetric G_ii, next step's G_{i+1,i+1}
            store_block<T, FULL>(p.G_diag + e * L * bb + i * bb, G, b, g, t);
        }
        __syncwarp();
    }
}

// Several right-hand sides: X = A^-1 R for R [L, b, nrhs], 16 columns per
// launch.  The solve recursions act on b x k blocks, so they run transposed,
// as products X Y^T of register tiles on the tensor cores (rows = right-hand
// sides, columns = block rows; no operand transposed):
//   Y_0^T = R_0^T,  Y_{i+1}^T = R_{i+1}^T - Y_i^T W_i^T                 (collect)
//   X_{L-1}^T = Y_{L-1}^T S_{L-1}^-1,  X_i^T = Y_i^T S_i^-1 - X_{i+1}^T W_i  (distribute)
// with W_i^T = S_i^-1 B_i^T formed as in the G sweep.  Y_i is kept in x.
template <class T, bool FULL>
__global__ void __launch_bounds__(WARPS * 32, 3) chain_multi_kernel(ChainArgs<T> p)
{
    using namespace w16;
    constexpr int E = SL<T>::ELEMS;
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t e = (int64_t)blockIdx.x * WARPS + wid;
    if (e >= p.batch) return;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *sbase = reinterpret_cast<T *>(smem_raw) + wid * warp_smem_elems<T>();
    T *sB = sbase, *sD = sB + E, *sT = sD + E, *sT2 = sT + E, *stg = sT2 + E;
    T *cb = stg + SLOT_ELEMS + 64;
    constexpr bool HINT = FULL && SELINV_L2MODE > 0;
    const uint64_t pol_first = HINT ? l2_evict_first() : 0;

    const int b = p.b;
    const int64_t L = p.L;
    const int64_t bb = (int64_t)b * b;
    const int K = p.nrhs, c0 = p.c0;
    const int kc = K - c0 < 16 ? K - c0 : 16;
    const int64_t bk = (int64_t)b * K;
    const T *D = p.diag + e * L * bb;
    const T *Bl = p.lower + e * (L - 1) * bb;
    T *ws = p.ws + e * (L - 1) * SLOT_ELEMS;
    const T *R = p.rhs + e * L * bk;
    T *X = p.x + e * L * bk;
    // block i of R or X as a transposed tile: element (c, r) = M[r][c0 + c]
    auto load_t = [&](Tile<T> &o, const T *M) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int c = g + 8 * h, r = tcol(t, q);
                o.v[h][q] = (c < kc && r < b) ? M[(int64_t)r * K + c0 + c] : T(0);
            }
    };
    auto store_t = [&](T *M, const Tile<T> &o) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int c = g + 8 * h, r = tcol(t, q);
                if (c < kc && r < b) M[(int64_t)r * K + c0 + c] = o.v[h][q];
            }
    };

    LogAcc det;
    det.init();
    int fail = -1;

    Tile<T> a, w, bt, yt;
    load_lower_async<T, FULL>(sD, D, b, lane);
    cp_async_commit();
    cp_async_wait_all();
    __syncwarp();
    from_smem_lower<T>(a, sD, g, t);
    __syncwarp();
    if (L > 1) {
        load_block_async<T, FULL>(sB, Bl, b, lane);
        load_lower_async<T, FULL>(sD, D + bb, b, lane);
        cp_async_commit();
    }
    load_t(yt, R);                                    // Y_0^T = R_0^T
    store_t(X, yt);

    // ---------------- collect sweep ----------------
    for (int64_t i = 0; i < L; ++i) {
        bool bad = false;
        spd_inverse<T>(a, cb, g, t, det, bad);        // a = S_i^-1
        det.renorm();
        if (bad && fail < 0) fail = (int)i;
        if (i == L - 1) break;
        store_lower_slot<T>(ws + i * SLOT_ELEMS, a, lane, g, t);
        cp_async_wait_all();
        __syncwarp();
        from_smem<T>(bt, sB, g, t);                   // B_i
        Tile<T> dn, rt;
        from_smem_lower<T>(dn, sD, g, t);             // D_{i+1}
        load_t(rt, R + (i + 1) * bk);                 // R_{i+1}^T
        zero(w);
        gemm_nt<false>(w, bt, a, sT, sT2, g, t);      // W_i = B_i S_i^-1
        gemm_nt<true, true>(dn, w, bt, sT, sT2, g, t);   // S_{i+1} = D_{i+1} - W_i B_i^T (lower tiles)
        mirror_upper(dn, g, t);
        a = dn;
        gemm_nt<true>(rt, yt, w, sT, sT2, g, t);      // Y_{i+1}^T = R_{i+1}^T - Y_i^T W_i^T
        yt = rt;
        store_t(X + (i + 1) * bk, yt);
        __syncwarp();
        if (i + 1 < L - 1) {
            load_block_async<T, FULL, HINT>(sB, Bl + (i + 1) * bb, b, lane, pol_first);
            load_lower_async<T, FULL, HINT>(sD, D + (i + 2) * bb, b, lane, pol_first);
            cp_async_commit();
        }
    }
    if (lane == 0) {
        if (p.logdet && c0 == 0) p.logdet[e] = det.log_value();
        if (c0 == 0) p.info[e] = fail;
    }

    // ---------------- distribute sweep ----------------
    Tile<T> G, xt;
    __syncwarp();
    to_smem<T>(sT, a, g, t);
    __syncwarp();
    from_smem_lower<T>(G, sT, g, t);                  // S_{L-1}^-1, exactly symmetric
    zero(xt);
    gemm_nt<false>(xt, yt, G, sT, sT2, g, t);         // X_{L-1}^T = Y_{L-1}^T S_{L-1}^-1
    store_t(X + (L - 1) * bk, xt);
    __syncwarp();
    if (L > 1) {
        load_block_async<T, FULL>(sB, Bl + (L - 2) * bb, b, lane);
        stage_lower_slot<T>(stg, ws + (L - 2) * SLOT_ELEMS, lane, g, t);
        cp_async_commit();
        load_t(yt, X + (L - 2) * bk);                 // Y_{L-2}^T
    }
    for (int64_t i = L - 2; i >= 0; --i) {
        cp_async_wait_all();
        unstage_lower_slot<T>(a, stg, lane, g, t);
        to_smem<T>(sT, a, g, t);
        __syncwarp();
        from_smem_lower<T>(a, sT, g, t);              // S_i^-1, full and symmetric
        from_smem<T>(bt, sB, g, t);                   // B_i
        __syncwarp();
        if (i > 0) {
            load_block_async<T, FULL, HINT>(sB, Bl + (i - 1) * bb, b, lane, pol_first);
            stage_lower_slot<T, HINT>(stg, ws + (i - 1) * SLOT_ELEMS, lane, g, t, pol_first);
            cp_async_commit();
        }
        Tile<T> wt, xn;
        zero(wt);
        gemm_nt<false>(wt, a, bt, sT, sT2, g, t);     // W_i^T = S_i^-1 B_i^T
        zero(xn);
        gemm_nt<false>(xn, yt, a, sT, sT2, g, t);     // Y_i^T S_i^-1
        gemm_nt<true>(xn, xt, wt, sT, sT2, g, t);     // - X_{i+1}^T W_i
        xt = xn;
        if (i > 0) load_t(yt, X + (i - 1) * bk);      // Y_{i-1}^T, before X_i overwrites nothing of it
        store_t(X + i * bk, xt);
        __syncwarp();
    }
}

template <class T, bool FULL, bool G, bool X, bool SAMPLE = false>
cudaError_t launch_t(const ChainArgs<T> &a, cudaStream_t s)
{
    const size_t smem = sizeof(T) * warp_smem_elems<T>() * CWARPS;
    auto k = chain_small_kernel<T, FULL, G, X, SAMPLE>;
    cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int64_t blocks = ceil_div(a.batch, CWARPS);
    ChainArgs<T> c = a;
    c.ws_lines = (reinterpret_cast<uintptr_t>(a.ws) & 127) == 0;
    k<<<(unsigned)blocks, CWARPS * 32, smem, s>>>(c);
    return cudaGetLastError();
}

template <class T, bool FULL>
cudaError_t launch_full(const ChainArgs<T> &a, cudaStream_t s)
{
    const bool G = a.G_diag != nullptr, X = a.x != nullptr;
    if (G && X) return launch_t<T, FULL, true, true>(a, s);
    if (G) return launch_t<T, FULL, true, false>(a, s);
    if (X) return launch_t<T, FULL, false, true>(a, s);
    return launch_t<T, FULL, false, false>(a, s);
}

}  // namespace

size_t chain_small_workspace(size_t elem, int64_t batch, int64_t L)
{
    return (size_t)batch * (size_t)(L > 1 ? L - 1 : 0) * WS_ELEMS * elem;
}

template <class T> cudaError_t chain_small_launch(const ChainArgs<T> &a, bool aligned16, cudaStream_t s)
{
    if (a.batch == 0) return cudaSuccess;
    if (a.b == 16 && aligned16) return launch_full<T, true>(a, s);
    return launch_full<T, false>(a, s);
}

template <class T, bool FULL> cudaError_t launch_multi(const ChainArgs<T> &a, cudaStream_t s)
{
    const size_t smem = sizeof(T) * warp_smem_elems<T>() * WARPS;
    auto k = chain_multi_kernel<T, FULL>;
    cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    k<<<(unsigned)ceil_div(a.batch, WARPS), WARPS * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <class T> cudaError_t chain_small_multi_launch(const ChainArgs<T> &a, bool aligned16, cudaStream_t s)
{
    if (a.batch == 0) return cudaSuccess;
    if (a.b == 16 && aligned16) return launch_multi<T, true>(a, s);
    return launch_multi<T, false>(a, s);
}

template cudaError_t chain_small_multi_launch<double>(const ChainArgs<double> &, bool, cudaStream_t);
template cudaError_t chain_small_multi_launch<float>(const ChainArgs<float> &, bool, cudaStream_t);

template <class T> cudaError_t chain_small_sample_launch(const ChainArgs<T> &a, bool aligned16, cudaStream_t s)
{
    if (a.batch == 0) return cudaSuccess;
    if (a.b == 16 && aligned16) return launch_t<T, true, false, true, true>(a, s);
    return launch_t<T, false, false, true, true>(a, s);
}

template cudaError_t chain_small_launch<double>(const ChainArgs<double> &, bool, cudaStream_t);
template cudaError_t chain_small_sample_launch<double>(const ChainArgs<double> &, bool, cudaStream_t);
template cudaError_t chain_small_sample_launch<float>(const ChainArgs<float> &, bool, cudaStream_t);
template cudaError_t chain_small_launch<float>(const ChainArgs<float> &, bool, cudaStream_t);

}  // namespace selinv
