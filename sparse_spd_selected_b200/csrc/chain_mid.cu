// Block-tridiagonal chains with 16 < b <= 32 (no right-hand side): one CTA
// of two 4-warp groups per chain, eliminating the chain from both ends.
//
// gabp-sparse-inv 0.3.2 (PyPI page), "Implemented and tested kernels" ->
// Chain and Tree: a chain is a path, and the tree kernel may root it at any
// node (the Quickstart's root-invariance remark: the chain roots the path at
// its last node, the tree at node 0).  Rooting it at the middle block m makes
// the collect sweep two independent half-chains:
//   top    (group 0)  blocks 0, 1, ..., m-1, coupling C = B_i = A_{i+1,i}
//   bottom (group 1)  blocks L-1, L-2, ..., m+1, coupling C = B_{i-1}^T = A_{i-1,i}
// each running S' = D' - C S^-1 C^T toward m; then S_m = D_m - (both
// contributions), G_mm = S_m^-1, and the two distribute sweeps run outward
// again with G_{next,j} = -G_{next} W_j, G_jj = S_j^-1 - W_j^T G_{next,j},
// W_j = C_j S_j^-1.  The two halves run concurrently, halving the
// sequential length of the long chains.
//
// Blocks are padded to 32 (identity / zero pad).  Warp w of a group owns
// quadrant (I, J) = (w >> 1, w & 1) of every 32 x 32 block as a 16 x 16
// register tile; products X Y^T are sums of two tile products whose operand
// quadrants come from shared images, each a register-register FP64
// tensor-core product.  The 32 x 32 inverse: float64 through the quadrant
// Schur complement (the diagonal warps invert A and S = C - B A^-1 B^T in
// their own registers, three group barriers), float32 the symmetric
// Gauss-Jordan sweep over the group, one pivot per barrier.
#include "kernels.h"
#include "quad32.cuh"

namespace selinv {

namespace {

using namespace q32;

template <class T, bool FULL, bool WANT_G>
__global__ void __launch_bounds__(2 * GT) chain_mid_kernel(ChainArgs<T> p)
{
    using namespace w16;
    using Ly = Lay<T>;
    constexpr int E = SL<T>::ELEMS;
    // workspace per eliminated block: the lower quadrant images (0,0), (1,0),
    // (1,1) of S_j^-1, then the four quadrant images of W_j
    constexpr int64_t SLOT = 7 * E;
    const int tid = threadIdx.x;
    const int grp = tid / GT;                         // 0: top half, 1: bottom half
    const int gtid = tid % GT;
    const int wq = gtid >> 5, lane = tid & 31;
    const int I = wq >> 1, J = wq & 1;
    const int g = lane >> 2, t = lane & 3;
    const int bar = 1 + grp;
    const bool bottom = grp == 1;
    const int64_t e = blockIdx.x;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *base = reinterpret_cast<T *>(smem_raw);
    T *gs = base + grp * Ly::GROUP;
    T *sC = gs + Ly::C, *sD = gs + Ly::D, *sX = gs + Ly::X, *sY = gs + Ly::Y, *sZ = gs + Ly::Z, *sZ2 = gs + Ly::Z2;
    T *s1 = sizeof(T) == 4 ? gs + Ly::S + wq * 2 * E : nullptr;
    T *s2 = sizeof(T) == 4 ? s1 + E : nullptr;
    T *cb = gs + Ly::CB;
    T *ex = base + Ly::EXCH;

    const int b = p.b;
    const int64_t L = p.L;
    const int64_t bb = (int64_t)b * b;
    const int64_t m = L / 2;
    const int64_t nh = bottom ? L - 1 - m : m;        // blocks this group eliminates before m
    const T *Dg = p.diag + e * L * bb;
    const T *Bg = p.lower + e * (L - 1) * bb;
    T *ws = WANT_G ? p.ws + e * (L > 1 ? L - 1 : 0) * SLOT : nullptr;
    // j-th block of this half (global index) and the lower block that couples it to the next one
    auto node = [&](int64_t j) { return bottom ? L - 1 - j : j; };
    auto cpl = [&](int64_t j) { return bottom ? L - 2 - j : j; };
    auto slot = [&](int64_t j) { return ws + (bottom ? L - 2 - j : j) * SLOT; };   // top j at j, bottom at L-2-j

    LogAcc det;
    det.init();
    int fail = -1;
    Tile<T> a;

    // ---------------- collect sweep, both halves toward m ----------------
    if (!bottom || nh > 0) {
        load_diag<T, FULL>(sD, Dg + node(0) * bb, b, gtid);
        cp_async_commit();
        cp_async_wait_all();
        group_bar(bar);
        sym_quad<T>(a, sD, I, J, g, t);
        group_bar(bar);
    } else {
        zero(a);                                      // no bottom half: contributes nothing to S_m
    }
    if (nh > 0) {
        load_full<T, FULL>(sC, Bg + cpl(0) * bb, b, gtid);
        if (!bottom || nh > 1) load_diag<T, FULL>(sD, Dg + node(1) * bb, b, gtid);
        cp_async_commit();
    }
    for (int64_t j = 0; j < nh; ++j) {
        bool bad = false;
        qinverse<T>(a, cb, I, J, g, t, bar, det, bad);              // a = S_j^-1
        if (bad && fail < 0) fail = (int)node(j);
        to_smem<T>(quad(sX, I, J), a, g, t);
        cp_async_wait_all();
        group_bar(bar);
        if (WANT_G) {                                                 // keep the lower quadrant images
            copy_out<T>(slot(j), sX, E, gtid);
            copy_out<T>(slot(j) + E, quad(sX, 1, 0), 2 * E, gtid);
        }
        Tile<T> w;
        zero(w);
        if (bottom) qgemm<false, true, false, false>(w, sC, sX, I, J, s1, s2, g, t);   // W_j = C_j S_j^-1
        else qgemm<false, false, false, false>(w, sC, sX, I, J, s1, s2, g, t);
        to_smem<T>(quad(sY, I, J), w, g, t);
        group_bar(bar);
        if (WANT_G) copy_out<T>(slot(j) + 3 * E, sY, 4 * E, gtid);     // and W_j for the distribute sweep
        const bool last = j == nh - 1;
        if (last && bottom) zero(a);                                  // bottom: only the contribution
        else sym_quad<T>(a, sD, I, J, g, t);                          // D of the next block (m for the top)
        if (bottom) qgemm<true, false, true, false>(a, sY, sC, I, J, s1, s2, g, t);    // S' -= W_j C_j^T
        else qgemm<true, false, false, false>(a, sY, sC, I, J, s1, s2, g, t);
        group_bar(bar);
        if (!last) {
            load_full<T, FULL>(sC, Bg + cpl(j + 1) * bb, b, gtid);
            if (bottom ? j + 2 < nh : true) load_diag<T, FULL>(sD, Dg + node(j + 2) * bb, b, gtid);
            cp_async_commit();
        }
    }

    // ---------------- middle block m ----------------
    __syncthreads();
    if (bottom) to_smem<T>(quad(ex, I, J), a, g, t);
    __syncthreads();
    Tile<T> G;
    if (!bottom) {
        Tile<T> u;
        from_smem<T>(u, quad(ex, I, J), g, t);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) a.v[h][q] += u.v[h][q];
        bool bad = false;
        qinverse<T>(a, cb, I, J, g, t, bar, det, bad);               // G_mm = S_m^-1
        if (bad && fail < 0) fail = (int)m;
    }
    __syncthreads();
    if (!bottom) to_smem<T>(quad(ex, I, J), a, g, t);
    __syncthreads();
    sym_quad<T>(G, ex, I, J, g, t);                                   // exactly symmetric G_mm, both groups
    // log det and info.  float64: the pivots live in the diagonal warps (0,0)
    // and (1,1) of each group; float32: every warp saw all of them, so the
    // (1,1) warps add nothing to the log-determinant.
    double *shd = reinterpret_cast<double *>(base + Ly::D);          // group 0's diagonal images are free here
    __syncthreads();
    if ((wq == 0 || wq == GW - 1) && lane == 0) {
        const int d = wq == GW - 1;
        shd[2 * grp + d] = (sizeof(T) == 8 || d == 0) ? det.log_value() : 0.0;
        reinterpret_cast<int *>(shd + 4)[2 * grp + d] = fail;
    }
    __syncthreads();
    if (tid == 0) {
        if (p.logdet) p.logdet[e] = (shd[0] + shd[1]) + (shd[2] + shd[3]);
        const int *fs = reinterpret_cast<const int *>(shd + 4);
        // first failure of each half in its own elimination order (top: lowest
        // index, bottom: highest), then the smaller index of the two halves
        int ft = fs[0], fb = fs[2];
        if (fs[1] >= 0 && (ft < 0 || fs[1] < ft)) ft = fs[1];
        if (fs[3] >= 0 && (fb < 0 || fs[3] > fb)) fb = fs[3];
        int f = ft;
        if (fb >= 0 && (f < 0 || fb < f)) f = fb;
        p.info[e] = f;
    }
    __syncthreads();
    if (!WANT_G) return;
    if (!bottom) store_quad<T, false>(p.G_diag + e * L * bb + m * bb, G, b, I, J, g, t);

    // ---------------- distribute sweeps, outward from m ----------------
    // G_{next} is kept as an image whose lower quadrants are read symmetrically
    // (sZa); S_j^-1 and W_j are staged from the workspace one block ahead into
    // alternating buffers.
    T *sZa = sZ, *sZb = sZ2;
    to_smem<T>(quad(sZa, I, J), G, g, t);
    if (nh > 0) {
        stage_in<T>(sX, slot(nh - 1), E, gtid);
        stage_in<T>(quad(sX, 1, 0), slot(nh - 1) + E, 2 * E, gtid);
        stage_in<T>(sY, slot(nh - 1) + 3 * E, 4 * E, gtid);
        cp_async_commit();
    }
    int cur = 0;
    for (int64_t j = nh - 1; j >= 0; --j) {
        T *bS = cur ? sD : sX, *bW = cur ? sC : sY;
        cp_async_wait_all();
        group_bar(bar);                                               // S_j^-1, W_j staged; G_next image written
        if (j > 0) {                                                  // next block's operands into the other buffers
            T *nS = cur ? sX : sD, *nW = cur ? sY : sC;
            stage_in<T>(nS, slot(j - 1), E, gtid);
            stage_in<T>(quad(nS, 1, 0), slot(j - 1) + E, 2 * E, gtid);
            stage_in<T>(nW, slot(j - 1) + 3 * E, 4 * E, gtid);
            cp_async_commit();
        }
        Tile<T> s, gl;
        sym_quad<T>(s, bS, I, J, g, t);                               // S_j^-1
        zero(gl);
#pragma unroll
        for (int K = 0; K < 2; ++K) {                                 // G_{next,j} = -G_next W_j
            Tile<T> x, y;
            sym_quad<T>(x, sZa, I, K, g, t);
            from_smem_T<T>(y, quad(bW, K, J), g, t);
            gemm_nt<true>(gl, x, y, s1, s2, g, t);
        }
        T *Gl = p.G_lower + e * (L - 1) * bb + cpl(j) * bb;
        if (bottom) store_quad<T, true>(Gl, gl, b, I, J, g, t);       // G_lower = G_{next,j}^T below m
        else store_quad<T, false>(Gl, gl, b, I, J, g, t);
        to_smem<T>(quad(sZb, I, J), gl, g, t);
        group_bar(bar);
        qgemm<true, true, true, false>(s, bW, sZb, I, J, s1, s2, g, t);   // G_jj = S_j^-1 - W_j^T G_{next,j}
        to_smem<T>(quad(sZa, I, J), s, g, t);                         // sZa is free: all read it before the barrier
        group_bar(bar);
        sym_quad<T>(G, sZa, I, J, g, t);                              // exactly symmetric G_jj
        store_quad<T, false>(p.G_diag + e * L * bb + node(j) * bb, G, b, I, J, g, t);
        cur ^= 1;
    }
}

template <class T, bool FULL, bool WANT_G>
cudaError_t launch_t(const ChainArgs<T> &a, cudaStream_t s)
{
    const size_t smem = sizeof(T) * Lay<T>::TOTAL;
    auto k = chain_mid_kernel<T, FULL, WANT_G>;
    cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    k<<<(unsigned)a.batch, 2 * GT, smem, s>>>(a);
    return cudaGetLastError();
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

size_t chain_mid_workspace(size_t elem, int64_t batch, int64_t L)
{
    const size_t E = elem == 8 ? w16::SL<double>::ELEMS : w16::SL<float>::ELEMS;
    return (size_t)batch * (size_t)(L > 1 ? L - 1 : 0) * 7 * E * elem;
}

template <class T> cudaError_t chain_mid_launch(const ChainArgs<T> &a, cudaStream_t s)
{
    if (a.batch == 0) return cudaSuccess;
    const bool full = a.b == 32 && al16(a.diag) && al16(a.lower);
    const bool G = a.G_diag != nullptr;
    if (full) return G ? launch_t<T, true, true>(a, s) : launch_t<T, true, false>(a, s);
    return G ? launch_t<T, false, true>(a, s) : launch_t<T, false, false>(a, s);
}

template cudaError_t chain_mid_launch<double>(const ChainArgs<double> &, cudaStream_t);
template cudaError_t chain_mid_launch<float>(const ChainArgs<float> &, cudaStream_t);

}  // namespace selinv
