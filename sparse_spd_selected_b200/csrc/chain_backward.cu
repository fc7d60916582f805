// Cotangents of the chain selected inverse (b <= 16, one warp per chain).
//
// gabp-sparse-inv 0.3.2 (PyPI page), "Differentiable selected inverse": the
// gradients of a loss over the selected blocks flow back to the input blocks
// through an analytic two-pass backward, with no tape over the per-block loop.
// Here the two passes are the reverse-mode forms of the forward's two sweeps.
// With P_i = S_i^-1 and W_i = B_i P_i the forward computes
//   collect     S_0 = D_0,  S_{i+1} = D_{i+1} - W_i B_i^T
//   distribute  G_{L-1,L-1} = P_{L-1},  G_{i+1,i} = -G_{i+1,i+1} W_i,
//               G_ii = P_i - W_i^T G_{i+1,i}
// Given the cotangents Gb_ii, Gb_{i+1,i} of the outputs:
// pass 1, i = 0 .. L-1 (the distribute sweep ran L-2 .. 0, so its reverse runs
// forward and can share one sweep with a fresh collect that rebuilds P_i):
//   Ga  = Gb_ii + C_i                       (C_0 = 0: G_ii also fed step i-1)
//   Xb  = Gb_{i+1,i} - W_i Ga               (cotangent of G_{i+1,i})
//   Wb  = -G_{i+1,i} Ga^T - G_{i+1,i+1} Xb  (cotangent of W_i)
//   Pd_i = Ga + B_i^T Wb,   Bd_i = Wb P_i,   C_{i+1} = -Xb W_i^T
//   (Pd_{L-1} = Ga at the last block)
// pass 2, i = L-1 .. 0 (the reverse of the collect sweep), with Sb_L = 0:
//   Pt   = Pd_i - B_i^T Sb_{i+1} B_i
//   Sb_i = -P_i Pt P_i                      (dP = -P dS P)
//   Bb_i = Bd_i - (Sb_{i+1} + Sb_{i+1}^T) W_i
//   Db_i = the lower-triangle read of D_i applied to Sb_i: Sb + Sb^T below the
//          diagonal, Sb on it, zero above.
// P_i (full tile) and Pd_i are kept in the workspace between the passes; Bd_i
// goes straight to the output Bb and is updated in place by pass 2 (the same
// lane writes and reads every element).
#include "kernels.h"
#include "warp16.cuh"

namespace selinv {

namespace {

using namespace w16;

constexpr int BW_WARPS = 4;
constexpr int BW_SLOT = 256;          // one full 16 x 16 tile per block and array

template <class T> __host__ __device__ constexpr int bw_smem_elems() { return 3 * SL<T>::ELEMS + 32; }

// General block (row-major b x b, or a 16-pitch workspace tile) into a tile,
// zero pad beyond b.  Input blocks take the read-only path; workspace and
// output blocks written earlier by this kernel are read through L2.
template <class T, bool FULL, bool RO>
SELINV_DEVINL void load_tile(Tile<T> &a, const T *M, int b, int g, int t)
{
    using V = typename Vec2<T>::type;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int r = g + 8 * h, c = 2 * t + 8 * p;
            if (FULL) {
                const V *src = reinterpret_cast<const V *>(M + r * 16 + c);
                const V v = RO ? __ldg(src) : __ldcg(src);
                a.v[h][2 * p] = v.x;
                a.v[h][2 * p + 1] = v.y;
            } else {
                a.v[h][2 * p] = (r < b && c < b) ? (RO ? __ldg(M + r * b + c) : __ldcg(M + r * b + c)) : T(0);
                a.v[h][2 * p + 1] =
                    (r < b && c + 1 < b) ? (RO ? __ldg(M + r * b + c + 1) : __ldcg(M + r * b + c + 1)) : T(0);
            }
        }
}

// out = in^T through the free shared image s.
template <class T> SELINV_DEVINL void transpose(Tile<T> &out, const Tile<T> &in, T *s, int g, int t)
{
    to_smem<T>(s, in, g, t);
    __syncwarp();
    from_smem_T<T>(out, s, g, t);
    __syncwarp();
}

template <class T> SELINV_DEVINL void add_to(Tile<T> &a, const Tile<T> &x)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) a.v[h][q] += x.v[h][q];
}

template <class T> SELINV_DEVINL void prefetch_block(const T *p, int64_t n, int lane)
{
    prefetch_range_l2(p, n, lane, 32);
}

template <class T, bool FULL>
__global__ void __launch_bounds__(BW_WARPS * 32) chain_backward_kernel(ChainBwdArgs<T> a)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t e = (int64_t)blockIdx.x * BW_WARPS + wid;
    if (e >= a.batch) return;                          // the whole warp leaves together
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *s0 = reinterpret_cast<T *>(smem_raw) + wid * bw_smem_elems<T>();
    T *s1 = s0 + SL<T>::ELEMS, *s2 = s1 + SL<T>::ELEMS, *cb = s2 + SL<T>::ELEMS;
    const int b = a.b;
    const int64_t L = a.L, bb = (int64_t)b * b;
    const T *D = a.diag + e * L * bb;
    const T *Bl = a.lower + e * (L - 1) * bb;
    const T *G = a.G_diag + e * L * bb;
    const T *Gl = a.G_lower + e * (L - 1) * bb;
    const T *Gbd = a.Gb_diag + e * L * bb;
    const T *Gbl = a.Gb_lower + e * (L - 1) * bb;
    T *Db = a.Db + e * L * bb;
    T *Bb = a.Bb + e * (L - 1) * bb;
    T *wsP = a.ws + e * L * 2 * BW_SLOT;               // P_i, then Pd_i
    T *wsPd = wsP + L * BW_SLOT;

    int bad_at = -1;
    Tile<T> S, C;
    load_sym<T, FULL>(S, D, b, g, t);
    zero(C);
    // ---------------- pass 1: collect + reverse distribute, i = 0 .. L-1 ----------------
    for (int64_t i = 0; i < L; ++i) {
        if (i + 1 < L) {                              // next step's blocks toward L2
            if (i + 2 < L) {
                prefetch_block(Bl + (i + 1) * bb, bb, lane);
                prefetch_block(Gl + (i + 1) * bb, bb, lane);
                if (a.Gb_lower) prefetch_block(Gbl + (i + 1) * bb, bb, lane);
                prefetch_block(D + (i + 2) * bb, bb, lane);
                prefetch_block(G + (i + 2) * bb, bb, lane);
            }
            if (a.Gb_diag) prefetch_block(Gbd + (i + 1) * bb, bb, lane);
        }
        LogAcc det;
        det.init();
        bool bad = false;
        Tile<T> P = S;
        spd_inverse<T>(P, cb, g, t, det, bad);        // P = S_i^-1
        if (bad && bad_at < 0) bad_at = (int)i;
        store_block<T, true>(wsP + i * BW_SLOT, P, 16, g, t);
        Tile<T> Ga = C;                                // Ga = Gb_ii + C_i
        if (a.Gb_diag) {
            Tile<T> u;
            load_tile<T, FULL, true>(u, Gbd + i * bb, b, g, t);
            add_to(Ga, u);
        }
        if (i + 1 < L) {
            Tile<T> B, W;
            load_tile<T, FULL, true>(B, Bl + i * bb, b, g, t);
            zero(W);
            gemm_nt<false>(W, B, P, s1, s2, g, t);     // W = B P
            load_sym<T, FULL>(S, D + (i + 1) * bb, b, g, t);
            gemm_nt<true, true>(S, W, B, s1, s2, g, t);   // S_{i+1} = D_{i+1} - W B^T (lower tiles)
            mirror_upper(S, g, t);
            Tile<T> GaT, Xb, Wb;
            transpose(GaT, Ga, s0, g, t);
            if (a.Gb_lower) load_tile<T, FULL, true>(Xb, Gbl + i * bb, b, g, t);
            else zero(Xb);
            gemm_nt<true>(Xb, W, GaT, s1, s2, g, t);   // Xb = Gb_{i+1,i} - W Ga
            {
                Tile<T> X;
                load_tile<T, FULL, true>(X, Gl + i * bb, b, g, t);
                zero(Wb);
                gemm_nt<true>(Wb, X, Ga, s1, s2, g, t);    // Wb = -G_{i+1,i} Ga^T
            }
            {
                Tile<T> XbT, Gd;
                transpose(XbT, Xb, s0, g, t);
                load_tile<T, FULL, true>(Gd, G + (i + 1) * bb, b, g, t);
                gemm_nt<true>(Wb, Gd, XbT, s1, s2, g, t);  // Wb -= G_{i+1,i+1} Xb (symmetric)
            }
            zero(C);
            gemm_nt<true>(C, Xb, W, s1, s2, g, t);         // C_{i+1} = -Xb W^T
            {
                Tile<T> BT, WbT;
                transpose(BT, B, s0, g, t);
                transpose(WbT, Wb, s0, g, t);
                gemm_nt<false>(Ga, BT, WbT, s1, s2, g, t); // Pd_i = Ga + B^T Wb
            }
            store_block<T, true>(wsPd + i * BW_SLOT, Ga, 16, g, t);
            Tile<T> Bd;
            zero(Bd);
            gemm_nt<false>(Bd, Wb, P, s1, s2, g, t);       // Bd_i = Wb P
            store_block<T, FULL>(Bb + i * bb, Bd, b, g, t);
        } else {
            store_block<T, true>(wsPd + i * BW_SLOT, Ga, 16, g, t);   // Pd_{L-1} = Ga
        }
    }
    if (lane == 0) a.info[e] = bad_at;
    __syncwarp();

    // ---------------- pass 2: reverse collect, i = L-1 .. 0 ----------------
    Tile<T> Sg, SgT;                                   // Sb_{i+1} and its transpose
    zero(Sg);
    zero(SgT);
    for (int64_t i = L - 1; i >= 0; --i) {
        if (i > 0) {
            prefetch_block(wsP + (i - 1) * BW_SLOT, BW_SLOT, lane);
            prefetch_block(wsPd + (i - 1) * BW_SLOT, BW_SLOT, lane);
            prefetch_block(Bl + (i - 1) * bb, bb, lane);
            prefetch_block(Bb + (i - 1) * bb, bb, lane);
        }
        Tile<T> P, Pt;
        load_tile<T, true, false>(P, wsP + i * BW_SLOT, 16, g, t);
        load_tile<T, true, false>(Pt, wsPd + i * BW_SLOT, 16, g, t);
        if (i + 1 < L) {
            Tile<T> B, BT;
            load_tile<T, FULL, true>(B, Bl + i * bb, b, g, t);
            transpose(BT, B, s0, g, t);
            {
                Tile<T> Z, ZT;
                zero(Z);
                gemm_nt<false>(Z, Sg, BT, s1, s2, g, t);   // Z = Sb_{i+1} B
                transpose(ZT, Z, s0, g, t);
                gemm_nt<true>(Pt, BT, ZT, s1, s2, g, t);   // Pt = Pd_i - B^T Sb_{i+1} B
            }
            Tile<T> Wt, Bo;
            zero(Wt);
            gemm_nt<false>(Wt, P, B, s1, s2, g, t);        // W_i^T = P B^T
            add_to(Sg, SgT);                               // Sb_{i+1} + Sb_{i+1}^T
            load_tile<T, FULL, false>(Bo, Bb + i * bb, b, g, t);
            gemm_nt<true>(Bo, Sg, Wt, s1, s2, g, t);       // Bb_i = Bd_i - (Sb + Sb^T) W_i
            store_block<T, FULL>(Bb + i * bb, Bo, b, g, t);
        }
        Tile<T> PtT, Q;
        transpose(PtT, Pt, s0, g, t);
        zero(Q);
        gemm_nt<false>(Q, P, PtT, s1, s2, g, t);           // Q = P Pt
        zero(Sg);
        gemm_nt<true>(Sg, Q, P, s1, s2, g, t);             // Sb_i = -P Pt P
        transpose(SgT, Sg, s0, g, t);
        Tile<T> Dt;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = g + 8 * h, c = tcol(t, q);
                Dt.v[h][q] = c < r ? Sg.v[h][q] + SgT.v[h][q] : (c == r ? Sg.v[h][q] : T(0));
            }
        store_block<T, FULL>(Db + i * bb, Dt, b, g, t);
    }
}

// Cotangents of the non-symmetric chain (gabp-sparse-inv: selinv_bidiag's
// analytic backward, one batched block op).  G = M^-1 is block lower
// triangular, so Mb = -G^T Gbar G^T on M's pattern needs only the forward's
// outputs:
//   Mb_ii      = -G_ii^T Gb_ii G_ii^T - G_{i+1,i}^T Gb_{i+1,i} G_ii^T
//                - G_ii^T Gb_{i,i-1} G_{i,i-1}^T
//   Mb_{i+1,i} = -G_{i+1,i+1}^T Gb_{i+1,i} G_ii^T.
// One warp per chain walks i = 0 .. L-1 and forms the transposes
//   Mb_ii^T = -(G_ii Gb_ii^T + G_{i,i-1} Gb_{i,i-1}^T) G_ii - Y_i^T G_{i+1,i},
//   Mb_{i,i-1}^T = -Y_{i-1}^T G_ii,   Y_i^T = G_ii Gb_{i+1,i}^T,
// as X Y^T products of register tiles, written back transposed.
template <class T, bool FULL>
__global__ void __launch_bounds__(BW_WARPS * 32) bidiag_backward_kernel(BidiagBwdArgs<T> a)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t e = (int64_t)blockIdx.x * BW_WARPS + wid;
    if (e >= a.batch) return;                          // the whole warp leaves together
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *s0 = reinterpret_cast<T *>(smem_raw) + wid * bw_smem_elems<T>();
    T *s1 = s0 + SL<T>::ELEMS, *s2 = s1 + SL<T>::ELEMS;
    const int b = a.b;
    const int64_t L = a.L, bb = (int64_t)b * b;
    const T *G = a.G_diag + e * L * bb;
    const T *Gl = a.G_lower + e * (L - 1) * bb;
    const T *Gbd = a.Gb_diag + e * L * bb;
    const T *Gbl = a.Gb_lower + e * (L - 1) * bb;
    T *Mbd = a.Mb_diag + e * L * bb;
    T *Mbl = a.Mb_lower + e * (L - 1) * bb;
    Tile<T> Gp, Lp, Yp;                                // G_{i,i-1}, Gb_{i,i-1}, Y_{i-1}^T
    zero(Gp);
    zero(Lp);
    zero(Yp);
    for (int64_t i = 0; i < L; ++i) {
        if (i + 1 < L) {                              // next step's blocks toward L2
            prefetch_block(G + (i + 1) * bb, bb, lane);
            if (a.Gb_diag) prefetch_block(Gbd + (i + 1) * bb, bb, lane);
            if (i + 2 < L) {
                prefetch_block(Gl + (i + 1) * bb, bb, lane);
                if (a.Gb_lower) prefetch_block(Gbl + (i + 1) * bb, bb, lane);
            }
        }
        Tile<T> Gii, GiiT, U, R;
        load_tile<T, FULL, true>(Gii, G + i * bb, b, g, t);
        transpose(GiiT, Gii, s0, g, t);
        zero(U);
        if (a.Gb_diag) {
            Tile<T> gd;
            load_tile<T, FULL, true>(gd, Gbd + i * bb, b, g, t);
            gemm_nt<false>(U, Gii, gd, s1, s2, g, t);          // G_ii Gb_ii^T
        }
        if (i > 0) {
            gemm_nt<false>(U, Gp, Lp, s1, s2, g, t);            // + G_{i,i-1} Gb_{i,i-1}^T
            Tile<T> ml;
            zero(ml);
            gemm_nt<true>(ml, Yp, GiiT, s1, s2, g, t);          // Mb_{i,i-1}^T = -Y_{i-1}^T G_ii
            store_block_T<T, FULL>(Mbl + (i - 1) * bb, ml, b, g, t);
        }
        zero(R);
        gemm_nt<true>(R, U, GiiT, s1, s2, g, t);                // -U G_ii
        if (i + 1 < L) {
            Tile<T> gl, lb, glT;
            load_tile<T, FULL, true>(gl, Gl + i * bb, b, g, t);
            if (a.Gb_lower) load_tile<T, FULL, true>(lb, Gbl + i * bb, b, g, t);
            else zero(lb);
            zero(Yp);
            gemm_nt<false>(Yp, Gii, lb, s1, s2, g, t);          // Y_i^T = G_ii Gb_{i+1,i}^T
            transpose(glT, gl, s0, g, t);
            gemm_nt<true>(R, Yp, glT, s1, s2, g, t);            // - Y_i^T G_{i+1,i}
            Gp = gl;
            Lp = lb;
        }
        store_block_T<T, FULL>(Mbd + i * bb, R, b, g, t);       // Mb_ii = R^T
    }
}

template <class T> cudaError_t launch_bidiag_bwd(const BidiagBwdArgs<T> &a, bool full, cudaStream_t s)
{
    const size_t smem = sizeof(T) * bw_smem_elems<T>() * BW_WARPS;
    auto k = full ? bidiag_backward_kernel<T, true> : bidiag_backward_kernel<T, false>;
    cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    k<<<(unsigned)ceil_div(a.batch, BW_WARPS), BW_WARPS * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <class T> cudaError_t launch_bwd(const ChainBwdArgs<T> &a, bool full, cudaStream_t s)
{
    const size_t smem = sizeof(T) * bw_smem_elems<T>() * BW_WARPS;
    auto k = full ? chain_backward_kernel<T, true> : chain_backward_kernel<T, false>;
    cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int64_t blocks = ceil_div(a.batch, BW_WARPS);
    k<<<(unsigned)blocks, BW_WARPS * 32, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

size_t chain_backward_workspace(size_t elem, int64_t batch, int64_t L)
{
    return (size_t)batch * (size_t)L * 2 * BW_SLOT * elem;
}

template <class T> cudaError_t chain_backward_launch(const ChainBwdArgs<T> &a, bool aligned16, cudaStream_t s)
{
    return launch_bwd<T>(a, a.b == 16 && aligned16, s);
}

template <class T> cudaError_t bidiag_backward_launch(const BidiagBwdArgs<T> &a, bool aligned16, cudaStream_t s)
{
    return launch_bidiag_bwd<T>(a, a.b == 16 && aligned16, s);
}

template cudaError_t bidiag_backward_launch<double>(const BidiagBwdArgs<double> &, bool, cudaStream_t);
template cudaError_t bidiag_backward_launch<float>(const BidiagBwdArgs<float> &, bool, cudaStream_t);
template cudaError_t chain_backward_launch<double>(const ChainBwdArgs<double> &, bool, cudaStream_t);
template cudaError_t chain_backward_launch<float>(const ChainBwdArgs<float> &, bool, cudaStream_t);

}  // namespace selinv
