// Long block-tridiagonal chains with 16 < b <= 32 when the batch is too small
// to fill the GPU (no right-hand side): each chain is cut into P segments by
// P - 1 separator blocks, and every segment is eliminated by its own group
// of four warps.
//
// gabp-sparse-inv 0.3.2 (PyPI page), "Implemented and tested kernels" ->
// Chain and Tree: the block LDL^T of a chain may take its blocks in any
// order that keeps the elimination a tree elimination (the Quickstart's
// root-invariance remark: the chain roots the path at its last node, the
// tree at node 0); "General sparse selected inverse": the multi-neighbour
// Takahashi recurrence G_{N,j} = -G_{N,N} L_{N,j}, G_jj = S_j^-1 - L_{N,j}^T G_{N,j}
// over the filled pattern.  Here the order is: every segment's blocks first
// (segments in parallel), then the separators.
//
// Segments (lo..hi, separators s_k = sep[k - 1]):
//   end segment 0        blocks 0 .. s_1 - 1, upward toward s_1, no fill;
//   end segment P - 1    blocks L - 1 .. s_{P-1} + 1, downward toward s_{P-1}, no fill;
//   interior segment k   blocks s_k + 1 .. s_{k+1} - 1, upward toward s_{k+1};
//                        block j also couples to the outer separator s = s_k
//                        through the fill block F_j = A_{j,s} (F = B_{s_k} at the
//                        first block).
// Collect, block j with coupling C_j = A_{next,j} (B_j upward, B_{j-1}^T downward):
//   W_j = C_j S_j^-1,  S_next = D_next - W_j C_j^T
//   interior:  V_j = F_j^T S_j^-1,  F_next = -W_j F_j,  U_s += V_j F_j
// The last block of a segment leaves W C^T for its separator (and, interior,
// U_s for the outer one and the fill coupling A'_{s_{k+1}, s_k} = F_next).
// The separators then form a chain of P - 1 blocks, D' = D_s - (both
// contributions), lower' = the fill couplings, solved by the two-ended
// kernel; its G blocks seed the distribute sweep of every segment:
//   G_{next,j} = -(G_{next,next} W_j + G_{s,next}^T V_j)
//   G_{s,j}    = -(G_{s,next} W_j + G_ss V_j)          (interior only)
//   G_jj       = S_j^-1 - W_j^T G_{next,j} - V_j^T G_{s,j}
// with G_{next,j} = G_lower (upward) or its transpose (downward), and
// G_{s,lo}^T = G_lower[s_k] at the end of an interior segment.
//
// Arithmetic is float64 for both element types: float32 blocks are widened as
// they are read and rounded as the G blocks are stored, so the float32 run
// takes the same FP64 tensor-core path as float64 (the scalar float32 path,
// one pivot per barrier on the FP32 pipes, was slower than float64 here), and
// the workspace images between the sweeps are float64.
#include <algorithm>

#include "kernels.h"
#include "quad32.cuh"

namespace selinv {

namespace {

using namespace q32;

constexpr int SEG_MAX = 16;

struct SegGeo {
    int P;                                 // segments
    int64_t sep[SEG_MAX - 1];              // separator blocks, ascending
};

template <class T> struct SegArgs {
    SegGeo geo;
    double *node;             // [batch, L, 11 E]: S_j^-1 lower images, W_j images, V_j images (float64)
    T *cA, *cB;               // [batch, P-1, b*b]: contribution to separator r from the segment below / above
    T *rdiag, *rlower;        // the separators' chain: [batch, P-1, b*b], [batch, P-2, b*b]
    T *rGd, *rGl;             // its G blocks
    double *ld;               // [batch, P] log det of each segment's blocks
    int32_t *fail;            // [batch, P] first failing block of each segment, -1 none
    double *rld;              // [batch] log det of the separators' chain
    int32_t *rinfo;           // [batch]
};

struct SegSpan {
    int64_t lo, hi;           // blocks of the segment
    bool down;                // eliminated from hi toward lo - 1
    bool fill;                // interior: coupled to the outer separator lo - 1
    int target;               // separator index r (0-based) the elimination runs into
};

SELINV_DEVINL SegSpan seg_span(const SegGeo &geo, int64_t L, int k)
{
    SegSpan s;
    const int P = geo.P;
    s.lo = k == 0 ? 0 : geo.sep[k - 1] + 1;
    s.hi = k == P - 1 ? L - 1 : geo.sep[k] - 1;
    s.down = k == P - 1;
    s.fill = k > 0 && k < P - 1;
    s.target = s.down ? P - 2 : k;
    return s;
}

// Per-group shared memory (elements).
template <class T> struct SegLay {
    static constexpr int E = w16::SL<T>::ELEMS;
    static constexpr int IMG = 4 * E;
    static constexpr int SCR = sizeof(T) == 4 ? 2 * E * GW : 0;
    static constexpr int CBN = sizeof(T) == 8 ? QSCHUR : 64;
    // collect: C, D, X (S^-1), Y (W), V, F (two buffers)
    static constexpr int C = 0, D = IMG, X = 2 * IMG, Y = 3 * IMG, V = 4 * IMG, F = 5 * IMG, F2 = 6 * IMG;
    static constexpr int CS = 7 * IMG, CCB = CS + SCR, CTOTAL = CCB + CBN;
    // distribute: A (G_next), B (G_{s,next}), Cg (G_{next,j}), Dg (G_{s,j}), W x 2, V x 2, S
    // (S: quadrant image slots (0,0), (1,0), (1,1) of a four-quadrant image)
    static constexpr int A = 0, B = IMG, CG = 2 * IMG, DG = 3 * IMG, W0 = 4 * IMG, V0 = 6 * IMG, S0 = 8 * IMG;
    static constexpr int DS = S0 + IMG, DTOTAL = DS + SCR;
    static constexpr int64_t NODE = 11 * E;       // workspace per block
};

template <class T> SELINV_DEVINL void combine_det(T *scratch, const LogAcc &det, int fail, int wq, int lane,
                                                  double *ld_out, int32_t *fail_out, bool forward)
{
    // float64: the pivots live in the diagonal warps (0,0) and (1,1); float32:
    // every warp saw all of them.  `forward`: failures are first in index order.
    double *shd = reinterpret_cast<double *>(scratch);
    __syncthreads();
    if ((wq == 0 || wq == GW - 1) && lane == 0) {
        const int d = wq == GW - 1;
        shd[d] = (sizeof(T) == 8 || d == 0) ? det.log_value() : 0.0;
        reinterpret_cast<int *>(shd + 2)[d] = fail;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        *ld_out = shd[0] + shd[1];
        const int *fs = reinterpret_cast<const int *>(shd + 2);
        int f = fs[0];
        if (fs[1] >= 0 && (f < 0 || (forward ? fs[1] < f : fs[1] > f))) f = fs[1];
        *fail_out = f;
    }
    __syncthreads();
}

// Collect sweep of one segment per CTA (one group of four warps).
template <class T, bool FULL, bool WANT_G>
__global__ void __launch_bounds__(GT, 3) seg_collect_kernel(ChainArgs<T> p, SegArgs<T> sa)
{
    using namespace w16;
    using C = double;                           // arithmetic (T: element type of the inputs and outputs)
    using Ly = SegLay<C>;
    constexpr int E = SL<C>::ELEMS;
    const int P = sa.geo.P;
    const int64_t e = blockIdx.x / P;
    const int k = blockIdx.x % P;
    const int gtid = threadIdx.x;
    const int wq = gtid >> 5, lane = gtid & 31;
    const int I = wq >> 1, J = wq & 1;
    const int g = lane >> 2, t = lane & 3;
    constexpr int bar = 1;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    C *base = reinterpret_cast<C *>(smem_raw);
    // C_j and D_next arrive by cp.async in the inputs' own element type and
    // are widened as they are read; every other image is float64
    T *sC = reinterpret_cast<T *>(base + Ly::C), *sD = reinterpret_cast<T *>(base + Ly::D);
    C *sX = base + Ly::X, *sY = base + Ly::Y;
    C *sV = base + Ly::V;
    auto sFb = [&](int64_t j) { return base + ((j & 1) ? Ly::F2 : Ly::F); };   // F_j
    C *s1 = nullptr, *s2 = nullptr;             // float64 products need no scratch
    C *cb = base + Ly::CCB;

    const int b = p.b;
    const int64_t L = p.L;
    const int64_t bb = (int64_t)b * b;
    const SegSpan sp = seg_span(sa.geo, L, k);
    const int64_t n = sp.hi - sp.lo + 1;
    const T *Dg = p.diag + e * L * bb;
    const T *Bg = p.lower + e * (L - 1) * bb;
    C *wsn = WANT_G ? sa.node + e * L * Ly::NODE : nullptr;
    auto node = [&](int64_t j) { return sp.down ? sp.hi - j : sp.lo + j; };
    auto cpl = [&](int64_t j) { return sp.down ? sp.hi - j - 1 : sp.lo + j; };   // lower block of C_j

    LogAcc det;
    det.init();
    int fail = -1;
    Tile<C> a, u;
    zero(u);

    load_diag<T, FULL>(sD, Dg + node(0) * bb, b, gtid);
    if (sp.fill) load_full_f64<T, FULL>(sFb(0), Bg + (sp.lo - 1) * bb, b, gtid);   // F = A_{lo, s} = B_s
    cp_async_commit();
    cp_async_wait_all();
    group_bar(bar);
    sym_quad<C>(a, sD, I, J, g, t);
    group_bar(bar);
    load_full<T, FULL>(sC, Bg + cpl(0) * bb, b, gtid);
    if (n > 1) load_diag<T, FULL>(sD, Dg + node(1) * bb, b, gtid);
    cp_async_commit();

    Tile<C> fn;
    const bool upper = I == 0 && J == 1;
    // Interior segments: F_{j+1} = -W_j F_j and U_s += V_j F_j do not feed
    // S_{j+1}, so they run while block j+1's inverse keeps the group waiting
    // (warp (0,0) while (1,1) inverts S, the others while (0,0) inverts A).
    bool pend = false;
    for (int64_t j = 0; j < n; ++j) {
        bool bad = false;
        auto idle = [&](int phase) {
            if (!pend || phase != ((I == 0 && J == 0) ? 3 : 1)) return;
            Tile<C> f;
            zero(f);
            qgemm<true, false, true, false>(f, sY, sFb(j - 1), I, J, s1, s2, g, t);   // F_j = -W_{j-1} F_{j-1}
            to_smem<C>(quad(sFb(j), I, J), f, g, t);
            if (!upper) qgemm<false, false, true, false>(u, sV, sFb(j - 1), I, J, s1, s2, g, t);   // U_s += V F
        };
        qinverse<C>(a, cb, I, J, g, t, bar, det, bad, idle);        // a = S_j^-1
        if (bad && fail < 0) fail = (int)node(j);
        to_smem<C>(quad(sX, I, J), a, g, t);
        cp_async_wait_all();
        group_bar(bar);
        C *slot = WANT_G ? wsn + node(j) * Ly::NODE : nullptr;
        if (WANT_G) {
            copy_out<C>(slot, sX, E, gtid);
            copy_out<C>(slot + E, quad(sX, 1, 0), 2 * E, gtid);
        }
        Tile<C> w, v;
        zero(w);
        if (sp.down) qgemm<false, true, false, false>(w, sC, sX, I, J, s1, s2, g, t);   // W_j = C_j S_j^-1
        else qgemm<false, false, false, false>(w, sC, sX, I, J, s1, s2, g, t);
        to_smem<C>(quad(sY, I, J), w, g, t);
        if (sp.fill) {
            zero(v);
            qgemm<false, true, false, false>(v, sFb(j), sX, I, J, s1, s2, g, t);    // V_j = F_j^T S_j^-1
            to_smem<C>(quad(sV, I, J), v, g, t);
        }
        group_bar(bar);
        if (WANT_G) {
            copy_out<C>(slot + 3 * E, sY, 4 * E, gtid);
            if (sp.fill) copy_out<C>(slot + 7 * E, sV, 4 * E, gtid);
        }
        const bool last = j == n - 1;
        // S_next and U_s are symmetric and only their lower quadrants are ever
        // read (the next inverse starts from quadrants (0,0), (1,0), (1,1); the
        // separators' D' is read on its lower triangle): warp (0,1) skips them.
        if (last || upper) zero(a);                                   // the separator's contribution only
        else sym_quad<C>(a, sD, I, J, g, t);                          // D_next
        if (!upper) {
            if (sp.down) qgemm<true, false, true, false>(a, sY, sC, I, J, s1, s2, g, t);   // S_next -= W_j C_j^T
            else qgemm<true, false, false, false>(a, sY, sC, I, J, s1, s2, g, t);
        }
        if (sp.fill && last) {                                        // the last block's, at once
            zero(fn);
            qgemm<true, false, true, false>(fn, sY, sFb(j), I, J, s1, s2, g, t);     // F_next = -W_j F_j
            if (!upper) qgemm<false, false, true, false>(u, sV, sFb(j), I, J, s1, s2, g, t);   // U_s += V_j F_j
        }
        pend = sp.fill && !last;
        group_bar(bar);
        if (!last) {
            load_full<T, FULL>(sC, Bg + cpl(j + 1) * bb, b, gtid);
            if (j + 2 < n) load_diag<T, FULL>(sD, Dg + node(j + 2) * bb, b, gtid);
            cp_async_commit();
        }
    }
    // contributions to the separators (a = -W C^T of the last block)
    const int nsep = P - 1;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) a.v[h][q] = -a.v[h][q];
    T *cdst = (sp.down ? sa.cB : sa.cA) + (e * nsep + sp.target) * bb;
    store_quad<T, false>(cdst, a, b, I, J, g, t);
    if (sp.fill) {
        store_quad<T, false>(sa.cB + (e * nsep + (k - 1)) * bb, u, b, I, J, g, t);        // U for s_k
        store_quad<T, false>(sa.rlower + (e * (nsep - 1) + (k - 1)) * bb, fn, b, I, J, g, t);   // A'_{s_{k+1}, s_k}
    }
    combine_det<C>(base + Ly::D, det, fail, wq, lane, sa.ld + e * P + k, sa.fail + e * P + k, !sp.down);
}

// Distribute sweep of one segment per CTA, seeded by the separators' G blocks.
template <class T, bool FULL>
__global__ void __launch_bounds__(GT, 3) seg_distribute_kernel(ChainArgs<T> p, SegArgs<T> sa)
{
    using namespace w16;
    using C = double;                           // arithmetic (T: element type of the inputs and outputs)
    using Ly = SegLay<C>;
    constexpr int E = SL<C>::ELEMS;
    const int P = sa.geo.P;
    const int nsep = P - 1;
    const int64_t e = blockIdx.x / P;
    const int k = blockIdx.x % P;
    const int gtid = threadIdx.x;
    const int wq = gtid >> 5, lane = gtid & 31;
    const int I = wq >> 1, J = wq & 1;
    const int g = lane >> 2, t = lane & 3;
    constexpr int bar = 1;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    C *base = reinterpret_cast<C *>(smem_raw);
    C *sA = base + Ly::A, *sCg = base + Ly::CG;
    auto bW = [&](int c) { return base + Ly::W0 + c * Ly::IMG; };
    auto bV = [&](int c) { return base + Ly::V0 + c * Ly::IMG; };
    C *bS = base + Ly::S0;
    C *s1 = nullptr, *s2 = nullptr;             // float64 products need no scratch

    const int b = p.b;
    const int64_t L = p.L;
    const int64_t bb = (int64_t)b * b;
    const SegSpan sp = seg_span(sa.geo, L, k);
    const int64_t n = sp.hi - sp.lo + 1;
    const C *wsn = sa.node + e * L * Ly::NODE;
    T *Gd = p.G_diag + e * L * bb;
    T *Gl = p.G_lower + e * (L - 1) * bb;
    auto node = [&](int64_t j) { return sp.down ? sp.hi - j : sp.lo + j; };
    auto stage_wv = [&](int64_t j, int c) {
        const C *slot = wsn + node(j) * Ly::NODE;
        stage_in<C>(bW(c), slot + 3 * E, 4 * E, gtid);
        if (sp.fill) stage_in<C>(bV(c), slot + 7 * E, 4 * E, gtid);
    };
    auto stage_s = [&](int64_t j) {
        const C *slot = wsn + node(j) * Ly::NODE;
        stage_in<C>(bS, slot, E, gtid);
        stage_in<C>(quad(bS, 1, 0), slot + E, 2 * E, gtid);
    };

    if (k == 0) {                                                     // the separators' own G blocks
        for (int r = 0; r < nsep; ++r) {
            const T *src = sa.rGd + (e * nsep + r) * bb;
            T *dst = Gd + sa.geo.sep[r] * bb;
            for (int64_t i = gtid; i < bb; i += GT) dst[i] = src[i];
        }
    }
    C *pB = base + Ly::B, *pD = base + Ly::DG;                        // G_{s,next} and the new G_{s,j}
    load_diag_f64<T, FULL>(sA, sa.rGd + (e * nsep + sp.target) * bb, b, gtid);    // G_next = G of the target
    if (sp.fill) {
        load_diag_f64<T, FULL>(pD, sa.rGd + (e * nsep + (k - 1)) * bb, b, gtid);  // G_ss
        load_full_f64<T, FULL>(sCg, sa.rGl + (e * (nsep - 1) + (k - 1)) * bb, b, gtid);   // G_{target, s}
    }
    stage_s(n - 1);
    stage_wv(n - 1, 0);
    cp_async_commit();
    cp_async_wait_all();
    group_bar(bar);
    Tile<C> gss[2];
    if (sp.fill) {
        sym_quad<C>(gss[0], pD, I, 0, g, t);
        sym_quad<C>(gss[1], pD, I, 1, g, t);
        Tile<C> x;
        from_smem_T<C>(x, quad(sCg, J, I), g, t);                     // G_{s,target} = G_{target,s}^T
        to_smem<C>(quad(pB, I, J), x, g, t);
    }
    int cur = 0;
    for (int64_t j = n - 1; j >= 0; --j) {
        cp_async_wait_all();
        group_bar(bar);                                               // block j's operands, G images
        if (j > 0) {
            stage_wv(j - 1, cur ^ 1);
            cp_async_commit();
        }
        Tile<C> s, gl, gs;
        sym_quad<C>(s, bS, I, J, g, t);                               // S_j^-1
        zero(gl);
#pragma unroll
        for (int K = 0; K < 2; ++K) {                                 // G_{next,j} = -G_next W_j ...
            Tile<C> x, y;
            sym_quad<C>(x, sA, I, K, g, t);
            from_smem_T<C>(y, quad(bW(cur), K, J), g, t);
            gemm_nt<true>(gl, x, y, s1, s2, g, t);
        }
        if (sp.fill) {
            zero(gs);
#pragma unroll
            for (int K = 0; K < 2; ++K) {
                Tile<C> x, y, yv;
                from_smem_T<C>(yv, quad(bV(cur), K, J), g, t);
                from_smem_T<C>(x, quad(pB, K, I), g, t);
                gemm_nt<true>(gl, x, yv, s1, s2, g, t);               // ... - G_{s,next}^T V_j
                from_smem<C>(x, quad(pB, I, K), g, t);
                from_smem_T<C>(y, quad(bW(cur), K, J), g, t);
                gemm_nt<true>(gs, x, y, s1, s2, g, t);                // G_{s,j} = -G_{s,next} W_j ...
                gemm_nt<true>(gs, gss[K], yv, s1, s2, g, t);          // ... - G_ss V_j
            }
        }
        const int64_t v = node(j);
        if (sp.down) store_quad<T, true>(Gl + (v - 1) * bb, gl, b, I, J, g, t);   // G_lower[v-1] = G_{v-1,v}^T
        else store_quad<T, false>(Gl + v * bb, gl, b, I, J, g, t);                 // G_lower[v] = G_{v+1,v}
        if (sp.fill && j == 0) store_quad<T, true>(Gl + (sp.lo - 1) * bb, gs, b, I, J, g, t);   // G_{lo,s}
        to_smem<C>(quad(sCg, I, J), gl, g, t);
        if (sp.fill) to_smem<C>(quad(pD, I, J), gs, g, t);
        group_bar(bar);
        if (j > 0) {
            stage_s(j - 1);
            cp_async_commit();
        }
        if (!(I == 0 && J == 1)) {                                    // G_jj is read on its lower quadrants
            qgemm<true, true, true, false>(s, bW(cur), sCg, I, J, s1, s2, g, t);   // G_jj = S_j^-1 - W_j^T G_{next,j}
            if (sp.fill) qgemm<true, true, true, false>(s, bV(cur), pD, I, J, s1, s2, g, t);   // - V_j^T G_{s,j}
            to_smem<C>(quad(sA, I, J), s, g, t);
        }
        group_bar(bar);
        Tile<C> G;
        sym_quad<C>(G, sA, I, J, g, t);                               // exactly symmetric G_jj
        store_quad<T, false>(Gd + v * bb, G, b, I, J, g, t);
        C *tmp = pB;
        pB = pD;
        pD = tmp;
        cur ^= 1;
    }
}

// D' = D_s - (contribution from below) - (contribution from above) for every separator.
template <class T> __global__ void seg_assemble_kernel(ChainArgs<T> p, SegArgs<T> sa)
{
    const int nsep = sa.geo.P - 1;
    const int64_t e = blockIdx.x / nsep;
    const int r = blockIdx.x % nsep;
    const int64_t bb = (int64_t)p.b * p.b;
    const T *D = p.diag + (e * p.L + sa.geo.sep[r]) * bb;
    const T *a = sa.cA + (e * nsep + r) * bb, *c = sa.cB + (e * nsep + r) * bb;
    T *dst = sa.rdiag + (e * nsep + r) * bb;
    for (int64_t i = threadIdx.x; i < bb; i += blockDim.x) dst[i] = D[i] - a[i] - c[i];
}

// log det = segments + separators; info = the smallest block index any part reports.
template <class T> __global__ void seg_finalize_kernel(ChainArgs<T> p, SegArgs<T> sa)
{
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= p.batch) return;
    const int P = sa.geo.P;
    double ld = sa.rld[e];
    int f = sa.rinfo[e] >= 0 ? (int)sa.geo.sep[sa.rinfo[e]] : -1;
    for (int k = 0; k < P; ++k) {
        ld += sa.ld[e * P + k];
        const int fk = sa.fail[e * P + k];
        if (fk >= 0 && (f < 0 || fk < f)) f = fk;
    }
    if (p.logdet) p.logdet[e] = ld;
    p.info[e] = f;
}

// Segment boundaries: end segments RHO times as long as interior ones (the
// interior blocks carry the fill products).
#ifndef SELINV_SEG_RHO
#define SELINV_SEG_RHO 1.7
#endif
constexpr double RHO = SELINV_SEG_RHO;

SegGeo seg_geometry(int64_t L, int P)
{
    SegGeo geo;
    geo.P = P;
    const int64_t free_blocks = L - (P - 1);
    const double unit = (double)free_blocks / (2.0 * RHO + (P - 2));
    int64_t nI = std::max<int64_t>(1, (int64_t)unit);
    int64_t nE0 = std::max<int64_t>(1, (int64_t)(RHO * unit));
    int64_t pos = nE0;                                   // first separator
    for (int k = 0; k < P - 1; ++k) {
        geo.sep[k] = pos;
        pos += 1 + nI;
    }
    return geo;
}

template <class T> size_t seg_bytes(size_t &off, size_t n)
{
    const size_t at = off;
    off += (n * sizeof(T) + 255) / 256 * 256;
    return at;
}

struct SegWs {
    size_t node, cA, cB, rdiag, rlower, rGd, rGl, ld, fail, rld, rinfo, rws, total;
};

template <class T> SegWs seg_ws_layout(int64_t batch, int64_t L, int b, int P, bool want_g)
{
    SegWs w;
    size_t off = 0;
    const size_t bb = (size_t)b * b, nsep = P - 1;
    w.node = seg_bytes<double>(off, want_g ? (size_t)batch * L * SegLay<double>::NODE : 0);
    w.cA = seg_bytes<T>(off, batch * nsep * bb);
    w.cB = seg_bytes<T>(off, batch * nsep * bb);
    w.rdiag = seg_bytes<T>(off, batch * nsep * bb);
    w.rlower = seg_bytes<T>(off, batch * (nsep - 1) * bb);
    w.rGd = seg_bytes<T>(off, want_g ? batch * nsep * bb : 0);
    w.rGl = seg_bytes<T>(off, want_g ? batch * (nsep - 1) * bb : 0);
    w.ld = seg_bytes<double>(off, batch * P);
    w.fail = seg_bytes<int32_t>(off, batch * P);
    w.rld = seg_bytes<double>(off, batch);
    w.rinfo = seg_bytes<int32_t>(off, batch);
    w.rws = off;
    off += (chain_mid_workspace(sizeof(T), batch, nsep) + 255) / 256 * 256;
    w.total = off;
    return w;
}

template <class K> cudaError_t set_smem(K k, size_t bytes)
{
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <class T, bool FULL>
cudaError_t seg_run(const ChainArgs<T> &a, const SegArgs<T> &sa, const SegWs &w, cudaStream_t s)
{
    using Ly = SegLay<double>;
    const int P = sa.geo.P;
    const bool G = a.G_diag != nullptr;
    const unsigned grid = (unsigned)(a.batch * P);
    cudaError_t err;
    if (G) {
        auto kc = seg_collect_kernel<T, FULL, true>;
        if ((err = set_smem(kc, sizeof(double) * Ly::CTOTAL)) != cudaSuccess) return err;
        kc<<<grid, GT, sizeof(double) * Ly::CTOTAL, s>>>(a, sa);
    } else {
        auto kc = seg_collect_kernel<T, FULL, false>;
        if ((err = set_smem(kc, sizeof(double) * Ly::CTOTAL)) != cudaSuccess) return err;
        kc<<<grid, GT, sizeof(double) * Ly::CTOTAL, s>>>(a, sa);
    }
    seg_assemble_kernel<T><<<(unsigned)(a.batch * (P - 1)), 256, 0, s>>>(a, sa);
    ChainArgs<T> r{};
    r.diag = sa.rdiag;
    r.lower = sa.rlower;
    r.G_diag = G ? sa.rGd : nullptr;
    r.G_lower = G ? sa.rGl : nullptr;
    r.logdet = sa.rld;
    r.info = sa.rinfo;
    r.ws = reinterpret_cast<T *>(reinterpret_cast<unsigned char *>(a.ws) + w.rws);
    r.batch = a.batch;
    r.L = P - 1;
    r.b = a.b;
    if ((err = chain_mid_launch<T>(r, s)) != cudaSuccess) return err;
    if (G) {
        auto kd = seg_distribute_kernel<T, FULL>;
        if ((err = set_smem(kd, sizeof(double) * Ly::DTOTAL)) != cudaSuccess) return err;
        kd<<<grid, GT, sizeof(double) * Ly::DTOTAL, s>>>(a, sa);
    }
    seg_finalize_kernel<T><<<(unsigned)ceil_div(a.batch, 128), 128, 0, s>>>(a, sa);
    return cudaGetLastError();
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

int chain_seg_parts(int64_t batch, int64_t L, int b, bool want_g, bool want_x)
{
    if (b <= 16 || b > 32 || !want_g || want_x || batch <= 0) return 0;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // three distribute CTAs fit on an SM; the two-ended kernel already covers
    // two groups per chain
#ifndef SELINV_SEG_SLOTS
#define SELINV_SEG_SLOTS 3
#endif
    const int64_t slots = SELINV_SEG_SLOTS * (int64_t)sms;
    int64_t P = std::min<int64_t>(SEG_MAX, slots / batch);
    P = std::min<int64_t>(P, L / 32);
    return P >= 3 ? (int)P : 0;
}

size_t chain_seg_workspace(size_t elem, int64_t batch, int64_t L, int b, int P, bool want_g)
{
    return elem == 8 ? seg_ws_layout<double>(batch, L, b, P, want_g).total
                     : seg_ws_layout<float>(batch, L, b, P, want_g).total;
}

template <class T> cudaError_t chain_seg_launch(const ChainArgs<T> &a, int P, cudaStream_t s)
{
    if (a.batch == 0) return cudaSuccess;
    const bool G = a.G_diag != nullptr;
    const SegWs w = seg_ws_layout<T>(a.batch, a.L, a.b, P, G);
    unsigned char *ws = reinterpret_cast<unsigned char *>(a.ws);
    SegArgs<T> sa;
    sa.geo = seg_geometry(a.L, P);
    sa.node = reinterpret_cast<double *>(ws + w.node);
    sa.cA = reinterpret_cast<T *>(ws + w.cA);
    sa.cB = reinterpret_cast<T *>(ws + w.cB);
    sa.rdiag = reinterpret_cast<T *>(ws + w.rdiag);
    sa.rlower = reinterpret_cast<T *>(ws + w.rlower);
    sa.rGd = reinterpret_cast<T *>(ws + w.rGd);
    sa.rGl = reinterpret_cast<T *>(ws + w.rGl);
    sa.ld = reinterpret_cast<double *>(ws + w.ld);
    sa.fail = reinterpret_cast<int32_t *>(ws + w.fail);
    sa.rld = reinterpret_cast<double *>(ws + w.rld);
    sa.rinfo = reinterpret_cast<int32_t *>(ws + w.rinfo);
    const bool full = a.b == 32 && al16(a.diag) && al16(a.lower) && (!G || (al16(a.G_diag) && al16(a.G_lower)));
    return full ? seg_run<T, true>(a, sa, w, s) : seg_run<T, false>(a, sa, w, s);
}

template cudaError_t chain_seg_launch<double>(const ChainArgs<double> &, int, cudaStream_t);
template cudaError_t chain_seg_launch<float>(const ChainArgs<float> &, int, cudaStream_t);

}  // namespace selinv
