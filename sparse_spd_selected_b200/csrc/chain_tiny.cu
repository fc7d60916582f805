// Short block-tridiagonal chains with small blocks (b <= 8, L <= 16, float64):
// one warp per chain, the whole chain in shared memory, 8 x 8 tiles.
//
// gabp-sparse-inv 0.3.2 (PyPI page), "Implemented and tested kernels" ->
// Chain, at the size of its "Quickstart" (8 blocks of 4): the same collect
// sweep (S_{i+1} = D_{i+1} - B_i S_i^-1 B_i^T, log det, forward solve) and
// distribute sweep (G_{i+1,i} = -G_{i+1,i+1} B_i S_i^-1, G_ii = S_i^-1 -
// S_i^-1 B_i^T G_{i+1,i}, backward solve) as the b <= 16 kernel, but sized
// for latency: one call is a handful of dependent block steps, so
//   - every D_i and B_i of the chain is loaded into shared memory at the
//     start (one memory latency instead of one per step), and each S_i^-1
//     replaces its D_i there, so the two sweeps need no workspace;
//   - blocks are 8 x 8 tiles in the m8n8k4 accumulator layout (lane 4g+t
//     holds row g, columns 2t and 2t+1), padded with identity (diagonal
//     blocks) or zero (off-diagonal blocks): the inverse is one 8-pivot sweep
//     and a product X Y^T two FP64 tensor-core steps, where the b <= 16
//     kernel pads to 16 x 16 (two block steps, sixteen steps per product).
#include "common.cuh"
#include "kernels.h"

namespace selinv {

namespace {

constexpr int TWARPS = 4;                        // chains per CTA
constexpr int TINY_L = 16;                       // longest chain this kernel takes
constexpr int TILE = 64;                         // elements of an 8 x 8 tile
constexpr int WARP_ELEMS = 2 * TINY_L * TILE + TILE + 32;   // D / S^-1, B, scratch, y and x

// acc += (NEG ? -1 : 1) X Y^T for 8 x 8 tiles in the accumulator layout: step
// s lets lane t carry k = 2t + s, the lane's own X.v[s] (A[g][k]) and Y.v[s]
// (B[k][g] = Y[g][k]), so no operand moves.
template <bool NEG> SELINV_DEVINL void mm8(double acc[2], const double X[2], const double Y[2])
{
    dmma_8x8x4(acc[0], acc[1], NEG ? -X[0] : X[0], Y[0]);
    dmma_8x8x4(acc[0], acc[1], NEG ? -X[1] : X[1], Y[1]);
}

SELINV_DEVINL void ld8(double v[2], const double *tile, int g, int t)
{
    const double2 u = *reinterpret_cast<const double2 *>(tile + g * 8 + 2 * t);
    v[0] = u.x;
    v[1] = u.y;
}
SELINV_DEVINL void st8(double *tile, const double v[2], int g, int t)
{
    *reinterpret_cast<double2 *>(tile + g * 8 + 2 * t) = make_double2(v[0], v[1]);
}
// Exactly symmetric tile from a tile whose lower triangle is right: written to
// the scratch tile and read back with each upper entry from its mirror.
SELINV_DEVINL void sym8(double v[2], double *scr, int g, int t)
{
    st8(scr, v, g, t);
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int c = 2 * t + j;
        v[j] = c <= g ? scr[g * 8 + c] : scr[c * 8 + g];
    }
    __syncwarp();
}
// Row sums of a tile times a length-8 vector x (shared): lanes with t == 0 hold row g.
SELINV_DEVINL double rowdot8(const double v[2], const double *x, int t)
{
    double s = fma(v[0], x[2 * t], v[1] * x[2 * t + 1]);
    s += shfl_xor(s, 1);
    s += shfl_xor(s, 2);
    return s;
}

template <bool WANT_G, bool WANT_X>
__global__ void __launch_bounds__(TWARPS * 32) chain_tiny_kernel(ChainArgs<double> p)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t e = (int64_t)blockIdx.x * TWARPS + wid;
    if (e >= p.batch) return;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    double *sD = reinterpret_cast<double *>(smem_raw) + wid * WARP_ELEMS;   // D_i, then S_i^-1
    double *sB = sD + TINY_L * TILE;                                        // B_i
    double *scr = sB + TINY_L * TILE;                                       // scratch tile
    double *sy = scr + TILE;                                                // y (16) and x (16)
    double *sx = sy + 16;

    const int b = p.b;
    const int64_t L = p.L, bb = (int64_t)b * b;
    const double *D = p.diag + e * L * bb;
    const double *Bl = p.lower + e * (L - 1) * bb;
    const double *R = WANT_X ? p.rhs + e * L * b : nullptr;
    double *X = WANT_X ? p.x + e * L * b : nullptr;

    // the whole chain into shared memory: D_i read on its lower triangle and
    // mirrored, identity pad; B_i with zero pad
    for (int64_t k = lane; k < L * TILE; k += 32) {
        const int64_t i = k >> 6;
        const int r = (int)(k >> 3) & 7, c = (int)k & 7;
        const int rr = c <= r ? r : c, cc = c <= r ? c : r;
        sD[k] = (r < b && c < b) ? __ldg(D + i * bb + rr * b + cc) : (r == c ? 1.0 : 0.0);
        if (i < L - 1) sB[k] = (r < b && c < b) ? __ldg(Bl + i * bb + r * b + c) : 0.0;
    }
    if (WANT_X && lane < 16) sy[lane] = 0.0;
    __syncwarp();

    LogAcc det;
    det.init();
    bool bad_any = false;
    int fail = -1;
    double a[2];
    ld8(a, sD, g, t);                                  // S_0 = D_0
    double yv = 0.0;                                   // y_i at row g (lanes with t == 0)
    if (WANT_X && t == 0) yv = g < b ? __ldg(R + g) : 0.0;

    // ---------------- collect sweep ----------------
    for (int64_t i = 0; i < L; ++i) {
        bool bad = false;
        inv8_sweep(a, lane, g, t, det, bad, true);    // a = S_i^-1 (pivots -> det)
        det.renorm();
        if (bad && fail < 0) fail = (int)i;
        bad_any |= bad;
        sym8(a, scr, g, t);
        st8(sD + i * TILE, a, g, t);                   // S_i^-1 replaces D_i
        if (WANT_X) {
            if (t == 0) {
                sy[g] = yv;
                if (g < b) X[i * b + g] = yv;          // y_i kept in x until the distribute sweep
            }
            __syncwarp();
        }
        if (i == L - 1) break;
        double bt[2], w[2] = {0.0, 0.0}, dn[2];
        ld8(bt, sB + i * TILE, g, t);
        mm8<false>(w, bt, a);                          // W_i = B_i S_i^-1
        ld8(dn, sD + (i + 1) * TILE, g, t);
        mm8<true>(dn, w, bt);                          // S_{i+1} = D_{i+1} - W_i B_i^T
        sym8(dn, scr, g, t);
        a[0] = dn[0];
        a[1] = dn[1];
        if (WANT_X) {                                  // y_{i+1} = r_{i+1} - W_i y_i
            const double s = rowdot8(w, sy, t);
            if (t == 0) yv = (g < b ? __ldg(R + (i + 1) * b + g) : 0.0) - s;
            __syncwarp();
        }
    }
    if (lane == 0) {
        if (p.logdet) p.logdet[e] = det.log_value();
        p.info[e] = fail;
    }
    if (!(WANT_G || WANT_X)) return;

    // ---------------- distribute sweep ----------------
    double G[2] = {a[0], a[1]};                        // G_{L-1,L-1} = S_{L-1}^-1 (symmetric)
    auto store_g = [&](double *dst, const double v[2], bool transpose) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int r = g, c = 2 * t + j;
            if (r < b && c < b) {
                if (transpose) dst[c * b + r] = v[j];
                else dst[r * b + c] = v[j];
            }
        }
    };
    if (WANT_G) store_g(p.G_diag + e * L * bb + (L - 1) * bb, G, false);
    double xv = 0.0;                                   // x_{i+1} at row g (lanes with t == 0)
    if (WANT_X) {                                      // x_{L-1} = S_{L-1}^-1 y_{L-1}
        const double s = rowdot8(G, sy, t);
        if (t == 0) {
            xv = s;
            if (g < b) X[(L - 1) * b + g] = s;
        }
    }
    for (int64_t i = L - 2; i >= 0; --i) {
        double sinv[2], bt[2], wt[2] = {0.0, 0.0};
        ld8(sinv, sD + i * TILE, g, t);
        ld8(bt, sB + i * TILE, g, t);
        mm8<false>(wt, sinv, bt);                      // W_i^T = S_i^-1 B_i^T
        if (WANT_X) {                                  // x_i = S_i^-1 y_i - W_i^T x_{i+1}
            if (t == 0) {
                sx[g] = xv;
                sy[g] = g < b ? X[i * b + g] : 0.0;    // y_i
            }
            __syncwarp();
            const double s = rowdot8(sinv, sy, t) - rowdot8(wt, sx, t);
            __syncwarp();
            if (t == 0) {
                xv = s;
                if (g < b) X[i * b + g] = s;
            }
        }
        if (WANT_G) {
            double glt[2] = {0.0, 0.0};
            mm8<true>(glt, wt, G);                     // G_{i+1,i}^T = -W_i^T G_{i+1,i+1}
            store_g(p.G_lower + e * (L - 1) * bb + i * bb, glt, true);
            mm8<true>(sinv, wt, glt);                  // G_ii = S_i^-1 - W_i^T G_{i+1,i}
            sym8(sinv, scr, g, t);
            G[0] = sinv[0];
            G[1] = sinv[1];
            store_g(p.G_diag + e * L * bb + i * bb, G, false);
        }
    }
}

template <bool G, bool Xs> cudaError_t launch(const ChainArgs<double> &a, cudaStream_t s)
{
    const size_t smem = sizeof(double) * WARP_ELEMS * TWARPS;
    auto k = chain_tiny_kernel<G, Xs>;
    cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    k<<<(unsigned)ceil_div(a.batch, TWARPS), TWARPS * 32, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool chain_tiny_fits(int64_t L, int b) { return b <= 8 && L <= TINY_L; }

cudaError_t chain_tiny_launch(const ChainArgs<double> &a, cudaStream_t s)
{
    if (a.batch == 0) return cudaSuccess;
    const bool G = a.G_diag != nullptr, Xs = a.x != nullptr;
    if (G && Xs) return launch<true, true>(a, s);
    if (G) return launch<true, false>(a, s);
    if (Xs) return launch<false, true>(a, s);
    return launch<false, false>(a, s);
}

}  // namespace selinv
