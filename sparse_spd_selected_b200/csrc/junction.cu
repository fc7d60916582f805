// General block-sparse SPD matrices (b <= 16): gabp-sparse-inv 0.3.2 (PyPI
// page), "General sparse selected inverse (junction tree)": the block pattern
// is completed to its chordal fill S = pattern(L + L^T) by an elimination
// order (greedy minimum degree unless the caller gives one), then the
// multi-neighbour Takahashi recurrence runs over the elimination tree.
//
// With N(v) the neighbours of v still present when v is eliminated (a clique
// after v's elimination), in elimination order:
//  collect (children before parents; left-looking, so every block has one
//  writer): for u in {v} + N(v)
//     A'_{u,v} = A_{u,v} - sum_{k : u, v in N(k)} W_{u,k} A'_{v,k}^T
//     (A_{u,v} = 0 for a fill block), S_v = A'_{v,v}, P_v = S_v^-1,
//     W_{u,v} = A'_{u,v} P_v, log|A| += log det S_v;
//  distribute (parents before children):
//     G_{u,v} = -sum_{l in N(v)} G_{u,l} W_{l,v}   (u in N(v)),
//     G_{v,v} = P_v - sum_{l in N(v)} W_{l,v}^T G_{l,v}.
// All k above are descendants of v in the elimination tree and all u, l are
// ancestors, so each sweep goes level by level (heights for the collect,
// depths for the distribute).  A level of the collect is three launches: one
// 4-warp CTA per target block (the warps split its contributions and add
// their partial sums in a fixed order), one warp per node for P_v, one warp
// per clique entry for W; a level of the distribute is two: one CTA per
// clique entry for G_{u,v}, one CTA per node for G_vv.  Wide cliques near the
// root so spread over many CTAs instead of one warp.
// The host plan holds the symbolic work: order, fill, the tree and its
// levels, the index lists of every contribution and of every G_{u,l} a
// clique reads.  Off-diagonal blocks of S are stored as (i, j), i > j, in the
// caller's numbering; a block met in the other orientation is read or
// written transposed.
#include <algorithm>
#include <climits>
#include <cmath>
#include <map>
#include <memory>
#include <mutex>
#include <new>
#include <set>
#include <unordered_map>
#include <vector>

#include "kernels.h"
#include "warp16.cuh"

struct selinv_junction_plan_s {
    int64_t n = 0, m = 0, nnz = 0, E = 0;       // nodes, input blocks, blocks of S, clique entries
    int device = 0;
    std::vector<int32_t> order, S_i, S_j;       // host copies for the caller
    std::vector<int64_t> c_off, d_off;          // level offsets (collect by height, distribute by depth)
    int32_t *d_c_nodes = nullptr, *d_d_nodes = nullptr;
    int32_t *d_col_ptr = nullptr;               // [n+1] entries of node v: its N(v) in elimination order
    int32_t *d_ent_slot = nullptr;              // [E] block of S holding (u, v)
    int32_t *d_ent_trans = nullptr;             // [E] 1: S holds (v, u), read / write transposed
    int32_t *d_ent_src = nullptr;               // [E] input block index of that slot, or -1 (fill)
    int32_t *d_con_ptr = nullptr;               // [E + n + 1] contributions per target (v, t)
    int32_t *d_con_w = nullptr, *d_con_a = nullptr;   // entries of W_{u,k} and A'_{v,k}
    int32_t *d_pair_ptr = nullptr;              // [n+1] into pair codes (|N(v)|^2 per node)
    int32_t *d_pair = nullptr;                  // -(w+1): diagonal of node w; else 2 * slot + transposed
    // per-level work lists: collect targets (node, t), collect entries (entry, node),
    // distribute entries (entry, node, index in N(node))
    std::vector<int64_t> ct_off, ce_off, de_off;
    int32_t *d_ct_node = nullptr, *d_ct_t = nullptr, *d_ce_ent = nullptr, *d_ce_node = nullptr;
    int32_t *d_de_ent = nullptr, *d_de_node = nullptr, *d_de_a = nullptr;
    int32_t *d_ent_owner = nullptr, *d_ent_u = nullptr;   // [E] node v of entry (u, v) and its u (solve)
    // One call is a few launches per elimination level (thousands on a lattice),
    // each doing little work, so the sequence is recorded once as a CUDA graph
    // per set of arguments and replayed: the graph's kernel nodes carry the
    // pointers, so a call with the same buffers (new values in them) replays it.
    struct Graph {
        int dtype = -1, b = 0;
        int64_t batch = 0;
        const void *ptr[9] = {};           // diag, edge, G_diag, G_lower, logdet, info, workspace, rhs, x
        cudaGraphExec_t exec = nullptr;
        uint64_t used = 0;
    };
    std::vector<Graph> graphs;                  // at most GRAPH_CACHE entries, least recently used replaced
    cudaStream_t capture = nullptr;             // non-blocking stream the graphs are recorded on
    uint64_t calls = 0;
    std::mutex mu;
};

namespace selinv {

namespace {

constexpr int JWARPS = 4;

struct JDev {
    const int32_t *col_ptr, *ent_slot, *ent_trans, *ent_src, *con_ptr, *con_w, *con_a, *pair_ptr, *pair;
    int64_t n, m, nnz, E;
};

template <class T> struct JBufs {
    const T *diag, *edge;
    T *G_diag, *G_lower;
    T *Sinv, *Ap, *W;                            // workspace tiles: [batch][n], [batch][E], [batch][E]
    double *ld;                                  // [batch][n]
    int32_t *info;
    int b;
};

// Tile policies.  Pol16: the 16 x 16 register tile of warp16.cuh (b <= 16).
// Pol8: an 8 x 8 tile in the m8n8 accumulator layout (lane 4g + t holds row
// g, columns 2t, 2t + 1) for b <= 8, where a 16 x 16 tile would be three
// quarters padding: an 8 x 8 x 8 product is two FP64 tensor-core steps whose
// k index follows the lane's own columns (k = 2t + s at step s, the same for
// both operands), transposes and mirrors are shuffles, and the inverse is the
// 8-pivot sweep.  Workspace blocks are SLOT-element tiles of pitch DIM.
template <class T> struct Pol16 {
    using Tile = w16::Tile<T>;
    static constexpr int DIM = 16, SLOT = 256, IMG = w16::SL<T>::ELEMS;
    static SELINV_DEVINL void zero(Tile &a) { w16::zero(a); }
    static SELINV_DEVINL void add(Tile &a, const Tile &x)
    {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) a.v[h][q] += x.v[h][q];
    }
    static SELINV_DEVINL void ld_ws(Tile &a, const T *M, int g, int t, bool trans)
    {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = g + 8 * h, c = w16::tcol(t, q);
                a.v[h][q] = __ldcg(trans ? M + c * 16 + r : M + r * 16 + c);
            }
    }
    static SELINV_DEVINL void st_ws(T *M, const Tile &a, int g, int t)
    {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) M[(g + 8 * h) * 16 + w16::tcol(t, q)] = a.v[h][q];
    }
    static SELINV_DEVINL void ld_blk(Tile &a, const T *M, int b, int g, int t, bool trans, bool l2)
    {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = g + 8 * h, c = w16::tcol(t, q);
                const T *p = trans ? M + c * b + r : M + r * b + c;
                a.v[h][q] = (r < b && c < b) ? (l2 ? __ldcg(p) : __ldg(p)) : T(0);
            }
    }
    static SELINV_DEVINL void st_blk(T *M, const Tile &a, int b, int g, int t, bool trans)
    {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = g + 8 * h, c = w16::tcol(t, q);
                if (r < b && c < b) {
                    if (trans) M[c * b + r] = a.v[h][q];
                    else M[r * b + c] = a.v[h][q];
                }
            }
    }
    static SELINV_DEVINL void load_sym(Tile &a, const T *D, int b, int g, int t) { w16::load_sym<T, false>(a, D, b, g, t); }
    template <bool NEG> static SELINV_DEVINL void gemm(Tile &acc, const Tile &X, const Tile &Y, T *sX, T *sY, int g, int t)
    {
        w16::gemm_nt<NEG>(acc, X, Y, sX, sY, g, t);
    }
    static SELINV_DEVINL void make_sym(Tile &a, int g, int t) { w16::mirror_upper(a, g, t); }
    static SELINV_DEVINL void sym_from_lower(Tile &a, T *img, int g, int t)
    {
        w16::to_smem<T>(img, a, g, t);
        __syncwarp();
        w16::from_smem_lower<T>(a, img, g, t);
        __syncwarp();
    }
    static SELINV_DEVINL void inverse(Tile &a, T *cb, int g, int t, LogAcc &det, bool &bad)
    {
        w16::spd_inverse<T>(a, cb, g, t, det, bad);
    }
    static SELINV_DEVINL void to_img(T *img, const Tile &a, int g, int t) { w16::to_smem<T>(img, a, g, t); }
    static SELINV_DEVINL void from_img(Tile &a, const T *img, int g, int t) { w16::from_smem<T>(a, img, g, t); }
};

template <class T> struct Tile8 {
    T v[2];
};

template <class T> struct Pol8 {
    using Tile = Tile8<T>;
    static constexpr int DIM = 8, SLOT = 64, IMG = 8 * 9;
    static SELINV_DEVINL void zero(Tile &a) { a.v[0] = a.v[1] = T(0); }
    static SELINV_DEVINL void add(Tile &a, const Tile &x)
    {
        a.v[0] += x.v[0];
        a.v[1] += x.v[1];
    }
    static SELINV_DEVINL void ld_ws(Tile &a, const T *M, int g, int t, bool trans)
    {
#pragma unroll
        for (int j = 0; j < 2; ++j) a.v[j] = __ldcg(trans ? M + (2 * t + j) * 8 + g : M + g * 8 + 2 * t + j);
    }
    static SELINV_DEVINL void st_ws(T *M, const Tile &a, int g, int t)
    {
#pragma unroll
        for (int j = 0; j < 2; ++j) M[g * 8 + 2 * t + j] = a.v[j];
    }
    static SELINV_DEVINL void ld_blk(Tile &a, const T *M, int b, int g, int t, bool trans, bool l2)
    {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int r = g, c = 2 * t + j;
            const T *p = trans ? M + c * b + r : M + r * b + c;
            a.v[j] = (r < b && c < b) ? (l2 ? __ldcg(p) : __ldg(p)) : T(0);
        }
    }
    static SELINV_DEVINL void st_blk(T *M, const Tile &a, int b, int g, int t, bool trans)
    {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int r = g, c = 2 * t + j;
            if (r < b && c < b) {
                if (trans) M[c * b + r] = a.v[j];
                else M[r * b + c] = a.v[j];
            }
        }
    }
    static SELINV_DEVINL void load_sym(Tile &a, const T *D, int b, int g, int t)
    {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int r = g, c = 2 * t + j;
            const int rr = c <= r ? r : c, cc = c <= r ? c : r;
            a.v[j] = (r < b && c < b) ? __ldg(D + rr * b + cc) : (r == c ? T(1) : T(0));
        }
    }
    // acc += (NEG ? -1 : 1) X Y^T
    template <bool NEG> static SELINV_DEVINL void gemm(Tile &acc, const Tile &X, const Tile &Y, T *sX, T *sY, int g, int t)
    {
        if constexpr (sizeof(T) == 8) {
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) dmma_8x8x4(acc.v[0], acc.v[1], NEG ? -X.v[s2] : X.v[s2], Y.v[s2]);
        } else {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                sX[g * 9 + 2 * t + j] = X.v[j];
                sY[g * 9 + 2 * t + j] = Y.v[j];
            }
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                T s = T(0);
#pragma unroll
                for (int k = 0; k < 8; ++k) s = fma(sX[g * 9 + k], sY[(2 * t + j) * 9 + k], s);
                acc.v[j] += NEG ? -s : s;
            }
            __syncwarp();
        }
    }
    // entry (c, r) of a, for the lane's (r, c) = (g, 2t + j): held by lane 4c + r / 2, register r & 1
    static SELINV_DEVINL T mirror_of(const Tile &a, int g, int t, int j)
    {
        const int src = ((2 * t + j) << 2) | (g >> 1);
        const T u0 = shfl(a.v[0], src), u1 = shfl(a.v[1], src);
        return (g & 1) ? u1 : u0;
    }
    static SELINV_DEVINL void sym_from_lower(Tile &a, T *, int g, int t)
    {
        const T m0 = mirror_of(a, g, t, 0), m1 = mirror_of(a, g, t, 1);
        if (2 * t > g) a.v[0] = m0;
        if (2 * t + 1 > g) a.v[1] = m1;
    }
    static SELINV_DEVINL void make_sym(Tile &a, int g, int t) { sym_from_lower(a, nullptr, g, t); }
    static SELINV_DEVINL void inverse(Tile &a, T *, int g, int t, LogAcc &det, bool &bad)
    {
        inv8_sweep<false, T>(a.v, 4 * g + t, g, t, det, bad, true);
    }
    static SELINV_DEVINL void to_img(T *img, const Tile &a, int g, int t)
    {
        img[g * 9 + 2 * t] = a.v[0];
        img[g * 9 + 2 * t + 1] = a.v[1];
    }
    static SELINV_DEVINL void from_img(Tile &a, const T *img, int g, int t)
    {
        a.v[0] = img[g * 9 + 2 * t];
        a.v[1] = img[g * 9 + 2 * t + 1];
    }
};

// Four warps split one sum of tile products; warps 1..3 leave their partial
// tiles in shared memory and warp 0 adds them in a fixed order, so the result
// does not depend on timing.  Returns true in warp 0, which holds the total.
template <class T, class Pol> SELINV_DEVINL bool reduce4(typename Pol::Tile &acc, T *img, int wid, int g, int t)
{
    if (wid > 0) Pol::to_img(img + (wid - 1) * Pol::IMG, acc, g, t);
    __syncthreads();
    if (wid != 0) return false;
#pragma unroll
    for (int k = 0; k < JWARPS - 1; ++k) {
        typename Pol::Tile u;
        Pol::from_img(u, img + k * Pol::IMG, g, t);
        Pol::add(acc, u);
    }
    return true;
}

// shared memory of the CTA-per-item kernels: three partial images, then per
// warp two product scratch images (float products) and 32 elements
template <class T, class Pol> __host__ __device__ constexpr int j_smem_elems()
{
    return (JWARPS - 1) * Pol::IMG + JWARPS * (2 * Pol::IMG + 32);
}

// Collect, one CTA per target block (v, t) of a level: t = 0 is S_v, t >= 1
// is A'_{u,v} for u = N(v)[t-1]; the warps split the contributions
// -W_{u,k} A'_{v,k}^T listed by the plan, each loading its next pair of
// tiles before the current product.
template <class T, class Pol>
__global__ void __launch_bounds__(JWARPS * 32)
jn_target_kernel(JBufs<T> p, JDev jd, const int32_t *tnode, const int32_t *tt, int64_t count)
{
    using Tile = typename Pol::Tile;
    constexpr int S = Pol::SLOT;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *img = reinterpret_cast<T *>(smem_raw);
    T *s1 = img + (JWARPS - 1) * Pol::IMG + wid * (2 * Pol::IMG + 32), *s2 = s1 + Pol::IMG;
    const int64_t item = blockIdx.x;
    const int32_t v = tnode[item % count], tg = tt[item % count];
    const int64_t e = item / count;
    const int b = p.b;
    const int64_t bb = (int64_t)b * b;
    const int32_t c0 = jd.col_ptr[v];
    const int64_t tau = (int64_t)c0 + v + tg;
    const T *Ap = p.Ap + e * jd.E * S, *W = p.W + e * jd.E * S;
    Tile acc;
    Pol::zero(acc);
    {
        const int32_t cend = jd.con_ptr[tau + 1];
        int32_t c = jd.con_ptr[tau] + wid;
        Tile w, a;
        if (c < cend) {
            Pol::ld_ws(w, W + (int64_t)jd.con_w[c] * S, g, t, false);
            Pol::ld_ws(a, Ap + (int64_t)jd.con_a[c] * S, g, t, false);
        }
        while (c < cend) {
            const int32_t cn = c + JWARPS;
            Tile wn, an;
            if (cn < cend) {
                Pol::ld_ws(wn, W + (int64_t)jd.con_w[cn] * S, g, t, false);
                Pol::ld_ws(an, Ap + (int64_t)jd.con_a[cn] * S, g, t, false);
            }
            Pol::template gemm<true>(acc, w, a, s1, s2, g, t);        // -= W_{u,k} A'_{v,k}^T
            w = wn;
            a = an;
            c = cn;
        }
    }
    if (!reduce4<T, Pol>(acc, img, wid, g, t)) return;
    Tile a0;
    if (tg == 0) {
        Pol::load_sym(a0, p.diag + (e * jd.n + v) * bb, b, g, t);
    } else {
        const int32_t ent = c0 + tg - 1, src = jd.ent_src[ent];
        if (src >= 0) Pol::ld_blk(a0, p.edge + (e * jd.m + src) * bb, b, g, t, jd.ent_trans[ent] != 0, false);
        else Pol::zero(a0);
    }
    Pol::add(acc, a0);
    if (tg == 0) Pol::st_ws(p.Sinv + (e * jd.n + v) * S, acc, g, t);      // S_v, inverted next
    else Pol::st_ws(p.Ap + (e * jd.E + c0 + tg - 1) * S, acc, g, t);
}

// One warp per node of a level: P_v = S_v^-1 in place, log det, info.
template <class T, class Pol>
__global__ void __launch_bounds__(JWARPS * 32)
jn_inverse_kernel(JBufs<T> p, JDev jd, const int32_t *nodes, int64_t count, int64_t batch)
{
    using Tile = typename Pol::Tile;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *cb = reinterpret_cast<T *>(smem_raw) + wid * 32;
    const int64_t item = (int64_t)blockIdx.x * JWARPS + wid;
    if (item >= count * batch) return;
    const int32_t v = nodes[item % count];
    const int64_t e = item / count;
    T *slot = p.Sinv + (e * jd.n + v) * Pol::SLOT;
    Tile S;
    Pol::ld_ws(S, slot, g, t, false);
    Pol::make_sym(S, g, t);
    LogAcc det;
    det.init();
    bool bad = false;
    Pol::inverse(S, cb, g, t, det, bad);
    if (lane == 0) {
        p.ld[e * jd.n + v] = det.log_value();
        if (bad) atomicMin(p.info + e, v);
    }
    __syncwarp();
    Pol::st_ws(slot, S, g, t);
}

// One warp per clique entry (u, v) of a level: W_{u,v} = A'_{u,v} P_v.
template <class T, class Pol>
__global__ void __launch_bounds__(JWARPS * 32)
jn_w_kernel(JBufs<T> p, JDev jd, const int32_t *ents, const int32_t *enodes, int64_t count, int64_t batch)
{
    using Tile = typename Pol::Tile;
    constexpr int S = Pol::SLOT;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *s1 = reinterpret_cast<T *>(smem_raw) + wid * 2 * Pol::IMG, *s2 = s1 + Pol::IMG;
    const int64_t item = (int64_t)blockIdx.x * JWARPS + wid;
    if (item >= count * batch) return;
    const int32_t ent = ents[item % count], v = enodes[item % count];
    const int64_t e = item / count;
    Tile a, P, w;
    Pol::ld_ws(a, p.Ap + (e * jd.E + ent) * S, g, t, false);
    Pol::ld_ws(P, p.Sinv + (e * jd.n + v) * S, g, t, false);
    Pol::zero(w);
    Pol::template gemm<false>(w, a, P, s1, s2, g, t);            // P symmetric
    Pol::st_ws(p.W + (e * jd.E + ent) * S, w, g, t);
}

// Distribute, one CTA per clique entry (u, v) of a level:
// G_{u,v} = -sum_{l in N(v)} G_{u,l} W_{l,v}, the warps splitting l.
template <class T, class Pol>
__global__ void __launch_bounds__(JWARPS * 32)
jn_gcol_kernel(JBufs<T> p, JDev jd, const int32_t *ents, const int32_t *enodes, const int32_t *eidx, int64_t count)
{
    using Tile = typename Pol::Tile;
    constexpr int S = Pol::SLOT;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *img = reinterpret_cast<T *>(smem_raw);
    T *s1 = img + (JWARPS - 1) * Pol::IMG + wid * (2 * Pol::IMG + 32), *s2 = s1 + Pol::IMG;
    const int64_t item = blockIdx.x;
    const int32_t ent = ents[item % count], v = enodes[item % count], a = eidx[item % count];
    const int64_t e = item / count;
    const int b = p.b;
    const int64_t bb = (int64_t)b * b;
    const int32_t c0 = jd.col_ptr[v], d = jd.col_ptr[v + 1] - c0;
    const T *W = p.W + e * jd.E * S;
    const T *Gd = p.G_diag + e * jd.n * bb, *Gl = p.G_lower + e * jd.nnz * bb;
    const int32_t *pc = jd.pair + jd.pair_ptr[v] + (int64_t)a * d;
    Tile acc;
    Pol::zero(acc);
    auto load_pair = [&](int32_t c, Tile &gul, Tile &wt) {
        const int32_t code = pc[c];
        if (code < 0) Pol::ld_blk(gul, Gd + (int64_t)(-code - 1) * bb, b, g, t, false, true);
        else Pol::ld_blk(gul, Gl + (int64_t)(code >> 1) * bb, b, g, t, (code & 1) != 0, true);
        Pol::ld_ws(wt, W + (int64_t)(c0 + c) * S, g, t, true);            // W_{l,v}^T
    };
    {
        int32_t c = wid;
        Tile gul, wt;
        if (c < d) load_pair(c, gul, wt);
        while (c < d) {
            const int32_t cn = c + JWARPS;
            Tile gn, wn;
            if (cn < d) load_pair(cn, gn, wn);
            Pol::template gemm<true>(acc, gul, wt, s1, s2, g, t);        // -= G_{u,l} W_{l,v}
            gul = gn;
            wt = wn;
            c = cn;
        }
    }
    if (!reduce4<T, Pol>(acc, img, wid, g, t)) return;
    Pol::st_blk(p.G_lower + (e * jd.nnz + jd.ent_slot[ent]) * bb, acc, b, g, t, jd.ent_trans[ent] != 0);
}

// One CTA per node of a level: G_vv = P_v - sum_{l in N(v)} W_{l,v}^T G_{l,v},
// the warps splitting l; written exactly symmetric.
template <class T, class Pol>
__global__ void __launch_bounds__(JWARPS * 32)
jn_gdiag_kernel(JBufs<T> p, JDev jd, const int32_t *nodes, int64_t count)
{
    using Tile = typename Pol::Tile;
    constexpr int S = Pol::SLOT;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *img = reinterpret_cast<T *>(smem_raw);
    T *s1 = img + (JWARPS - 1) * Pol::IMG + wid * (2 * Pol::IMG + 32), *s2 = s1 + Pol::IMG;
    const int64_t item = blockIdx.x;
    const int32_t v = nodes[item % count];
    const int64_t e = item / count;
    const int b = p.b;
    const int64_t bb = (int64_t)b * b;
    const int32_t c0 = jd.col_ptr[v], d = jd.col_ptr[v + 1] - c0;
    const T *W = p.W + e * jd.E * S;
    const T *Gl = p.G_lower + e * jd.nnz * bb;
    Tile acc;
    Pol::zero(acc);
    for (int32_t c = wid; c < d; c += JWARPS) {
        const int32_t ent = c0 + c;
        Tile wt, glT;
        Pol::ld_ws(wt, W + (int64_t)ent * S, g, t, true);                  // W_{l,v}^T
        Pol::ld_blk(glT, Gl + (int64_t)jd.ent_slot[ent] * bb, b, g, t, jd.ent_trans[ent] == 0, true);   // G_{l,v}^T
        Pol::template gemm<true>(acc, wt, glT, s1, s2, g, t);              // -= W^T G
    }
    if (!reduce4<T, Pol>(acc, img, wid, g, t)) return;
    Tile P;
    Pol::ld_ws(P, p.Sinv + (e * jd.n + v) * S, g, t, false);
    Pol::add(acc, P);
    Pol::sym_from_lower(acc, img, g, t);             // exactly symmetric from the lower triangle
    Pol::st_blk(p.G_diag + (e * jd.n + v) * bb, acc, b, g, t, false);
}

// The solve x = A^-1 r from the same factorisation (gabp-sparse-inv, "General
// sparse selected inverse": junction_solve).  With L_{u,v} = W_{u,v} for u in
// N(v) (unit lower in elimination order) and S_v the pivots, A = L diag(S) L^T:
//   forward, children first:  z_v = r_v - sum_{k : v in N(k)} W_{v,k} z_k
//   backward, parents first:  x_v = S_v^-1 z_v - sum_{u in N(v)} W_{u,v}^T x_u
// The k with v in N(k) are exactly the contributions of v's diagonal target
// in the collect, and N(v) its clique entries; z lives in x until the
// backward pass overwrites it.  One warp per node and matrix.
template <class T, class Pol> struct VecOps {
    static constexpr int RH = Pol::DIM == 16 ? 2 : 1;       // rows per lane
    static constexpr int CQ = Pol::DIM == 16 ? 4 : 2;       // columns per lane
    static SELINV_DEVINL int col(int t, int q) { return Pol::DIM == 16 ? w16::tcol(t, q) : 2 * t + q; }
    static SELINV_DEVINL T at(const typename Pol::Tile &a, int h, int q)
    {
        if constexpr (Pol::DIM == 16) return a.v[h][q];
        else return a.v[q];
    }
    static SELINV_DEVINL void gather(T xv[CQ], const T *x, int b, int t)
    {
#pragma unroll
        for (int q = 0; q < CQ; ++q) xv[q] = col(t, q) < b ? __ldcg(x + col(t, q)) : T(0);
    }
    // part[h] += (NEG ? -1 : 1) sum over the lane's columns of a[row][col] x[col]
    template <bool NEG> static SELINV_DEVINL void madd(T part[RH], const typename Pol::Tile &a, const T xv[CQ])
    {
#pragma unroll
        for (int h = 0; h < RH; ++h)
#pragma unroll
            for (int q = 0; q < CQ; ++q) part[h] = fma(NEG ? -at(a, h, q) : at(a, h, q), xv[q], part[h]);
    }
    static SELINV_DEVINL void reduce(T part[RH])
    {
#pragma unroll
        for (int h = 0; h < RH; ++h) {
            part[h] += shfl_xor(part[h], 1);
            part[h] += shfl_xor(part[h], 2);
        }
    }
};

template <class T, class Pol>
__global__ void __launch_bounds__(JWARPS * 32)
jn_solve_fwd_kernel(JBufs<T> p, JDev jd, const int32_t *ent_owner, const int32_t *nodes, int64_t count,
                    int64_t batch, const T *rhs, T *x)
{
    using V = VecOps<T, Pol>;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t item = (int64_t)blockIdx.x * JWARPS + wid;
    if (item >= count * batch) return;
    const int32_t v = nodes[item % count];
    const int64_t e = item / count;
    const int b = p.b;
    const T *W = p.W + e * jd.E * Pol::SLOT;
    T *xe = x + e * jd.n * b;
    const int64_t tau = (int64_t)jd.col_ptr[v] + v;            // v's diagonal target
    T part[V::RH] = {};
    for (int32_t c = jd.con_ptr[tau]; c < jd.con_ptr[tau + 1]; ++c) {
        const int32_t ent = jd.con_w[c];                        // W_{v,k}
        typename Pol::Tile w;
        Pol::ld_ws(w, W + (int64_t)ent * Pol::SLOT, g, t, false);
        T zk[V::CQ];
        V::gather(zk, xe + (int64_t)ent_owner[ent] * b, b, t);
        V::template madd<false>(part, w, zk);
    }
    V::reduce(part);
    if (t == 0) {
#pragma unroll
        for (int h = 0; h < V::RH; ++h) {
            const int r = g + 8 * h;
            if (r < b) xe[(int64_t)v * b + r] = rhs[(e * jd.n + v) * b + r] - part[h];
        }
    }
}

template <class T, class Pol>
__global__ void __launch_bounds__(JWARPS * 32)
jn_solve_bwd_kernel(JBufs<T> p, JDev jd, const int32_t *ent_u, const int32_t *nodes, int64_t count, int64_t batch,
                    T *x)
{
    using V = VecOps<T, Pol>;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t item = (int64_t)blockIdx.x * JWARPS + wid;
    if (item >= count * batch) return;
    const int32_t v = nodes[item % count];
    const int64_t e = item / count;
    const int b = p.b;
    const T *W = p.W + e * jd.E * Pol::SLOT;
    T *xe = x + e * jd.n * b;
    T part[V::RH] = {};
    {
        typename Pol::Tile sinv;
        Pol::ld_ws(sinv, p.Sinv + (e * jd.n + v) * Pol::SLOT, g, t, false);
        T zv[V::CQ];
        V::gather(zv, xe + (int64_t)v * b, b, t);
        V::template madd<false>(part, sinv, zv);                // S_v^-1 z_v
    }
    for (int32_t ent = jd.col_ptr[v]; ent < jd.col_ptr[v + 1]; ++ent) {
        typename Pol::Tile wt;
        Pol::ld_ws(wt, W + (int64_t)ent * Pol::SLOT, g, t, true);   // W_{u,v}^T
        T xu[V::CQ];
        V::gather(xu, xe + (int64_t)ent_u[ent] * b, b, t);
        V::template madd<true>(part, wt, xu);
    }
    V::reduce(part);
    if (t == 0) {
#pragma unroll
        for (int h = 0; h < V::RH; ++h) {
            const int r = g + 8 * h;
            if (r < b) xe[(int64_t)v * b + r] = part[h];
        }
    }
}

__global__ void junction_init(int32_t *info, int64_t batch)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < batch) info[i] = INT_MAX;
}

// log det per matrix = sum of its nodes' log det S_v in node order (deterministic).
__global__ void junction_finalize(const double *ld, int64_t n, int64_t batch, double *logdet, int32_t *info)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= batch) return;
    double s = 0.0;
    for (int64_t v = 0; v < n; ++v) s += ld[i * n + v];
    if (logdet) logdet[i] = s;
    if (info[i] == INT_MAX) info[i] = -1;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

template <class T, int SLOT> size_t ws_bytes(const selinv_junction_plan_s *pl, int64_t batch)
{
    return align256(sizeof(T) * SLOT * (size_t)(batch * pl->n)) +
           2 * align256(sizeof(T) * SLOT * (size_t)(batch * pl->E)) + align256(sizeof(double) * (size_t)(batch * pl->n));
}

// G_diag == nullptr: the solve (rhs -> x) instead of the selected inverse.
template <class T, class Pol>
cudaError_t run_junction(const selinv_junction_plan_s *pl, int b, int64_t batch, const T *diag, const T *edge,
                         T *G_diag, T *G_lower, double *logdet, int32_t *info, void *ws, cudaStream_t s,
                         const T *rhs = nullptr, T *x = nullptr)
{
    constexpr int S = Pol::SLOT;
    char *w = static_cast<char *>(ws);
    JBufs<T> p;
    p.diag = diag;
    p.edge = edge;
    p.G_diag = G_diag;
    p.G_lower = G_lower;
    p.Sinv = reinterpret_cast<T *>(w);
    w += align256(sizeof(T) * S * (size_t)(batch * pl->n));
    p.Ap = reinterpret_cast<T *>(w);
    w += align256(sizeof(T) * S * (size_t)(batch * pl->E));
    p.W = reinterpret_cast<T *>(w);
    w += align256(sizeof(T) * S * (size_t)(batch * pl->E));
    p.ld = reinterpret_cast<double *>(w);
    p.info = info;
    p.b = b;
    JDev jd{pl->d_col_ptr, pl->d_ent_slot, pl->d_ent_trans, pl->d_ent_src, pl->d_con_ptr, pl->d_con_w,
            pl->d_con_a, pl->d_pair_ptr, pl->d_pair, pl->n, pl->m, pl->nnz, pl->E};
    const unsigned ib = (unsigned)ceil_div(batch, 256);
    const size_t smem_r = sizeof(T) * j_smem_elems<T, Pol>();      // CTA-per-item kernels
    const size_t smem_w = sizeof(T) * JWARPS * 2 * Pol::IMG, smem_i = sizeof(T) * JWARPS * 32;
    junction_init<<<ib, 256, 0, s>>>(info, batch);
    for (size_t l = 0; l + 1 < pl->c_off.size(); ++l) {
        const int64_t nt = pl->ct_off[l + 1] - pl->ct_off[l];
        const int64_t nn = pl->c_off[l + 1] - pl->c_off[l];
        const int64_t ne = pl->ce_off[l + 1] - pl->ce_off[l];
        jn_target_kernel<T, Pol><<<(unsigned)(nt * batch), JWARPS * 32, smem_r, s>>>(
            p, jd, pl->d_ct_node + pl->ct_off[l], pl->d_ct_t + pl->ct_off[l], nt);
        jn_inverse_kernel<T, Pol><<<(unsigned)ceil_div(nn * batch, JWARPS), JWARPS * 32, smem_i, s>>>(
            p, jd, pl->d_c_nodes + pl->c_off[l], nn, batch);
        if (ne > 0)
            jn_w_kernel<T, Pol><<<(unsigned)ceil_div(ne * batch, JWARPS), JWARPS * 32, smem_w, s>>>(
                p, jd, pl->d_ce_ent + pl->ce_off[l], pl->d_ce_node + pl->ce_off[l], ne, batch);
    }
    if (G_diag == nullptr) {                                    // solve: forward, then backward
        for (size_t l = 0; l + 1 < pl->c_off.size(); ++l) {
            const int64_t nn = pl->c_off[l + 1] - pl->c_off[l];
            jn_solve_fwd_kernel<T, Pol><<<(unsigned)ceil_div(nn * batch, JWARPS), JWARPS * 32, 0, s>>>(
                p, jd, pl->d_ent_owner, pl->d_c_nodes + pl->c_off[l], nn, batch, rhs, x);
        }
        for (size_t l = 0; l + 1 < pl->d_off.size(); ++l) {
            const int64_t nn = pl->d_off[l + 1] - pl->d_off[l];
            jn_solve_bwd_kernel<T, Pol><<<(unsigned)ceil_div(nn * batch, JWARPS), JWARPS * 32, 0, s>>>(
                p, jd, pl->d_ent_u, pl->d_d_nodes + pl->d_off[l], nn, batch, x);
        }
        junction_finalize<<<ib, 256, 0, s>>>(p.ld, pl->n, batch, logdet, info);
        return cudaGetLastError();
    }
    for (size_t l = 0; l + 1 < pl->d_off.size(); ++l) {
        const int64_t nn = pl->d_off[l + 1] - pl->d_off[l];
        const int64_t ne = pl->de_off[l + 1] - pl->de_off[l];
        if (ne > 0)
            jn_gcol_kernel<T, Pol><<<(unsigned)(ne * batch), JWARPS * 32, smem_r, s>>>(
                p, jd, pl->d_de_ent + pl->de_off[l], pl->d_de_node + pl->de_off[l], pl->d_de_a + pl->de_off[l], ne);
        jn_gdiag_kernel<T, Pol><<<(unsigned)(nn * batch), JWARPS * 32, smem_r, s>>>(p, jd, pl->d_d_nodes + pl->d_off[l],
                                                                                     nn);
    }
    junction_finalize<<<ib, 256, 0, s>>>(p.ld, pl->n, batch, logdet, info);
    return cudaGetLastError();
}

// Shared-memory limits of the kernels run_junction launches (set before a
// capture: attribute calls are not stream work).
template <class T, class Pol> cudaError_t junction_attributes()
{
    const size_t smem_r = sizeof(T) * j_smem_elems<T, Pol>();
    const size_t smem_w = sizeof(T) * JWARPS * 2 * Pol::IMG;
    cudaError_t err = cudaSuccess;
    for (auto k : {(const void *)jn_target_kernel<T, Pol>, (const void *)jn_gcol_kernel<T, Pol>,
                   (const void *)jn_gdiag_kernel<T, Pol>})
        if (err == cudaSuccess) err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_r);
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(jn_w_kernel<T, Pol>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_w);
    return err;
}

constexpr size_t GRAPH_CACHE = 4;

// Launch one call through the plan's graph cache: replay the graph recorded
// for these arguments, or record it (on the plan's own capture stream, so the
// caller's stream may be any stream, the legacy default one included) and
// replay it.  A caller whose stream is itself being captured gets the
// launches directly, inside its own graph.
template <class T, class Pol>
cudaError_t junction_call(selinv_junction_plan_s *pl, int dtype, int b, int64_t batch, const T *diag, const T *edge,
                          T *G_diag, T *G_lower, double *logdet, int32_t *info, void *ws, cudaStream_t s,
                          const T *rhs = nullptr, T *x = nullptr)
{
    cudaError_t err = junction_attributes<T, Pol>();
    if (err != cudaSuccess) return err;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone)
        return run_junction<T, Pol>(pl, b, batch, diag, edge, G_diag, G_lower, logdet, info, ws, s, rhs, x);
    const void *key[9] = {diag, edge, G_diag, G_lower, logdet, info, ws, rhs, x};
    std::lock_guard<std::mutex> lock(pl->mu);
    ++pl->calls;
    for (auto &g : pl->graphs)
        if (g.dtype == dtype && g.b == b && g.batch == batch && std::equal(key, key + 9, g.ptr)) {
            g.used = pl->calls;
            return cudaGraphLaunch(g.exec, s);
        }
    if (!pl->capture && (err = cudaStreamCreateWithFlags(&pl->capture, cudaStreamNonBlocking)) != cudaSuccess)
        return err;
    if ((err = cudaStreamBeginCapture(pl->capture, cudaStreamCaptureModeThreadLocal)) != cudaSuccess) return err;
    cudaError_t run =
        run_junction<T, Pol>(pl, b, batch, diag, edge, G_diag, G_lower, logdet, info, ws, pl->capture, rhs, x);
    cudaGraph_t graph = nullptr;
    err = cudaStreamEndCapture(pl->capture, &graph);
    if (run != cudaSuccess || err != cudaSuccess) {
        if (graph) cudaGraphDestroy(graph);
        cudaGetLastError();
        return run != cudaSuccess ? run : err;
    }
    cudaGraphExec_t exec = nullptr;
    err = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (err != cudaSuccess) return err;
    if (pl->graphs.size() >= GRAPH_CACHE) {                 // replace the least recently used
        auto old = std::min_element(pl->graphs.begin(), pl->graphs.end(),
                                    [](const auto &x, const auto &y) { return x.used < y.used; });
        cudaGraphExecDestroy(old->exec);
        pl->graphs.erase(old);
    }
    selinv_junction_plan_s::Graph g;
    g.dtype = dtype;
    g.b = b;
    g.batch = batch;
    std::copy(key, key + 9, g.ptr);
    g.exec = exec;
    g.used = pl->calls;
    pl->graphs.push_back(g);
    return cudaGraphLaunch(exec, s);
}

bool is_aligned(const void *q, size_t a) { return (reinterpret_cast<uintptr_t>(q) % a) == 0; }

}  // namespace

}  // namespace selinv

using namespace selinv;

extern "C" {

void selinv_junction_plan_free(selinv_junction_plan_t *pl)
{
    if (!pl) return;
    int32_t *arrs[] = {pl->d_c_nodes, pl->d_d_nodes, pl->d_col_ptr, pl->d_ent_slot, pl->d_ent_trans, pl->d_ent_src,
                       pl->d_con_ptr, pl->d_con_w, pl->d_con_a, pl->d_pair_ptr, pl->d_pair, pl->d_ct_node,
                       pl->d_ct_t, pl->d_ce_ent, pl->d_ce_node, pl->d_de_ent, pl->d_de_node, pl->d_de_a,
                       pl->d_ent_owner, pl->d_ent_u};
    for (auto &g : pl->graphs) cudaGraphExecDestroy(g.exec);   // a launch in flight is freed on completion
    if (pl->capture) cudaStreamDestroy(pl->capture);
    for (int32_t *a : arrs) cudaFree(a);
    delete pl;
}

// The symbolic phase: validation, elimination (minimum degree with ties to
// the smaller node, or the given order), the cliques N(v) and the filled
// pattern S with its slots (sorted by j, then i).  Host only.
struct JSym {
    std::vector<int32_t> seq, pos;
    std::vector<std::vector<int32_t>> nbr;
    std::vector<std::pair<int32_t, int32_t>> S;
    std::map<std::pair<int32_t, int32_t>, int32_t> Sset;
    std::unordered_map<int64_t, int32_t> input;       // key i * n + j -> input block index
};

static selinv_status junction_symbolic_impl(int64_t n, int64_t m, const int32_t *ei, const int32_t *ej,
                                            const int32_t *order, JSym &sy)
{
    if (n < 1 || m < 0 || (m > 0 && (!ei || !ej)) || n >= (int64_t)INT32_MAX / 2) return SELINV_ERR_INVALID_ARG;
    auto &seq = sy.seq;
    auto &nbr = sy.nbr;
    auto &S = sy.S;
    auto &Sset = sy.Sset;
    auto &input = sy.input;
    nbr.assign(n, {});
    // pattern: (i, j), 0 <= j < i < n, no repeats
    std::vector<std::set<int32_t>> adj(n);
    for (int64_t k = 0; k < m; ++k) {
        const int32_t i = ei[k], j = ej[k];
        if (j < 0 || i <= j || i >= n) return SELINV_ERR_INVALID_ARG;
        if (!input.emplace((int64_t)i * n + j, (int32_t)k).second) return SELINV_ERR_INVALID_ARG;
        adj[i].insert(j);
        adj[j].insert(i);
    }
    seq.clear();
    seq.reserve(n);
    if (order) {
        std::vector<char> seen(n, 0);
        for (int64_t k = 0; k < n; ++k) {
            const int32_t v = order[k];
            if (v < 0 || v >= n || seen[v]) return SELINV_ERR_INVALID_ARG;
            seen[v] = 1;
        }
    }
    // eliminate: N(v) = the neighbours still present; they become a clique
    std::set<std::pair<int32_t, int32_t>> bydeg;     // (degree, node) of the remaining nodes
    if (!order)
        for (int32_t v = 0; v < n; ++v) bydeg.insert({(int32_t)adj[v].size(), v});
    for (const auto &kv : input) Sset.emplace(std::make_pair((int32_t)(kv.first / n), (int32_t)(kv.first % n)), -1);
    for (int64_t step = 0; step < n; ++step) {
        int32_t v;
        if (order) {
            v = order[step];
        } else {
            v = bydeg.begin()->second;
            bydeg.erase(bydeg.begin());
        }
        std::vector<int32_t> nb(adj[v].begin(), adj[v].end());
        for (size_t a = 0; a < nb.size(); ++a)
            for (size_t c = a + 1; c < nb.size(); ++c) {
                const int32_t x = nb[a], y = nb[c];
                if (adj[x].count(y)) continue;
                if (!order) {
                    bydeg.erase({(int32_t)adj[x].size(), x});
                    bydeg.erase({(int32_t)adj[y].size(), y});
                }
                adj[x].insert(y);
                adj[y].insert(x);
                if (!order) {
                    bydeg.insert({(int32_t)adj[x].size(), x});
                    bydeg.insert({(int32_t)adj[y].size(), y});
                }
                Sset.emplace(std::make_pair(std::max(x, y), std::min(x, y)), -1);
            }
        for (int32_t x : nb) {
            if (!order) bydeg.erase({(int32_t)adj[x].size(), x});
            adj[x].erase(v);
            if (!order) bydeg.insert({(int32_t)adj[x].size(), x});
        }
        adj[v].clear();
        nbr[v] = nb;
        seq.push_back(v);
    }
    sy.pos.assign(n, 0);
    for (int64_t k = 0; k < n; ++k) sy.pos[seq[k]] = (int32_t)k;
    // S sorted by (j, i)
    S.assign(Sset.size(), {});
    {
        size_t k = 0;
        for (const auto &kv : Sset) S[k++] = kv.first;
        std::sort(S.begin(), S.end(), [](const std::pair<int32_t, int32_t> &x, const std::pair<int32_t, int32_t> &y) {
            return x.second != y.second ? x.second < y.second : x.first < y.first;
        });
        for (size_t q = 0; q < S.size(); ++q) Sset[S[q]] = (int32_t)q;
    }
    return SELINV_OK;
}

static selinv_status junction_plan_impl(int64_t n, int64_t m, const int32_t *ei, const int32_t *ej, const int32_t *order,
                                   selinv_junction_plan_t **out)
{
    if (!out) return SELINV_ERR_INVALID_ARG;
    *out = nullptr;
    JSym sy;
    const selinv_status st = junction_symbolic_impl(n, m, ei, ej, order, sy);
    if (st != SELINV_OK) return st;
    auto &seq = sy.seq;
    auto &pos = sy.pos;
    auto &nbr = sy.nbr;
    auto &S = sy.S;
    auto &Sset = sy.Sset;
    auto &input = sy.input;
    auto slot_of = [&](int32_t x, int32_t y) { return Sset.at(std::make_pair(std::max(x, y), std::min(x, y))); };
    // entries: N(v) in elimination order
    std::vector<int32_t> col_ptr(n + 1, 0);
    for (int32_t v = 0; v < n; ++v) {
        std::sort(nbr[v].begin(), nbr[v].end(), [&](int32_t x, int32_t y) { return pos[x] < pos[y]; });
        col_ptr[v + 1] = col_ptr[v] + (int32_t)nbr[v].size();
    }
    const int64_t E = col_ptr[n];
    std::vector<int32_t> ent_slot(std::max<int64_t>(E, 1)), ent_trans(std::max<int64_t>(E, 1)),
        ent_src(std::max<int64_t>(E, 1));
    std::vector<int32_t> slot_src(S.size(), -1);
    for (const auto &kv : input) slot_src[slot_of((int32_t)(kv.first / n), (int32_t)(kv.first % n))] = kv.second;
    for (int32_t v = 0; v < n; ++v)
        for (int32_t a = 0; a < (int32_t)nbr[v].size(); ++a) {
            const int32_t u = nbr[v][a], ent = col_ptr[v] + a;
            ent_slot[ent] = slot_of(u, v);
            ent_trans[ent] = u < v ? 1 : 0;                 // S holds (v, u) = (u, v)^T
            ent_src[ent] = slot_src[ent_slot[ent]];
        }
    // contributions: for k, pairs (v, u) of N(k) with pos[v] <= pos[u] feed target (v, t(u))
    const int64_t T = E + n;
    std::vector<int32_t> tcount(T + 1, 0);
    auto tindex = [&](int32_t v, int32_t u) -> int64_t {
        if (u == v) return (int64_t)col_ptr[v] + v;
        const auto &nv = nbr[v];
        const int32_t a = (int32_t)(std::find(nv.begin(), nv.end(), u) - nv.begin());
        return (int64_t)col_ptr[v] + v + 1 + a;
    };
    std::vector<int32_t> cw, ca;                       // per contribution: W_{u,k} and A'_{v,k} entries
    for (int pass = 0; pass < 2; ++pass) {             // count per target, then fill
        std::vector<int32_t> fillp;
        if (pass == 1) fillp.assign(tcount.begin(), tcount.end() - 1);
        if (pass == 1) {
            cw.assign(tcount[T], 0);
            ca.assign(tcount[T], 0);
        }
        for (int64_t sk = 0; sk < n; ++sk) {
            const int32_t k = seq[sk];
            const auto &nk = nbr[k];
            for (int32_t a = 0; a < (int32_t)nk.size(); ++a)
                for (int32_t c = a; c < (int32_t)nk.size(); ++c) {
                    const int32_t vv = nk[a], uu = nk[c];           // pos[vv] <= pos[uu]
                    const int64_t tgt = tindex(vv, uu);
                    if (pass == 0) {
                        tcount[tgt + 1]++;
                    } else {
                        const int32_t at = fillp[tgt]++;
                        cw[at] = col_ptr[k] + c;                    // W_{uu,k}
                        ca[at] = col_ptr[k] + a;                    // A'_{vv,k}
                    }
                }
        }
        if (pass == 0)
            for (int64_t q = 0; q < T; ++q) tcount[q + 1] += tcount[q];
        if (pass == 1) {
            // tree of the elimination: parent = first-eliminated later neighbour
            std::vector<int32_t> parent(n, -1), height(n, 0), depth(n, 0);
            for (int32_t v = 0; v < n; ++v)
                if (!nbr[v].empty()) parent[v] = nbr[v][0];
            for (int64_t sk = 0; sk < n; ++sk) {
                const int32_t v = seq[sk];
                if (parent[v] >= 0) height[parent[v]] = std::max(height[parent[v]], height[v] + 1);
            }
            for (int64_t sk = n - 1; sk >= 0; --sk) {
                const int32_t v = seq[sk];
                depth[v] = parent[v] < 0 ? 0 : depth[parent[v]] + 1;
            }
            int32_t H = 0, Dm = 0;
            for (int32_t v = 0; v < n; ++v) {
                H = std::max(H, height[v]);
                Dm = std::max(Dm, depth[v]);
            }
            std::vector<int64_t> c_off(H + 2, 0), d_off(Dm + 2, 0);
            for (int32_t v = 0; v < n; ++v) {
                c_off[height[v] + 1]++;
                d_off[depth[v] + 1]++;
            }
            for (int32_t h = 0; h <= H; ++h) c_off[h + 1] += c_off[h];
            for (int32_t h = 0; h <= Dm; ++h) d_off[h + 1] += d_off[h];
            std::vector<int32_t> cn(n), dn(n);
            {
                std::vector<int64_t> pc(c_off.begin(), c_off.end() - 1), pd(d_off.begin(), d_off.end() - 1);
                for (int32_t v = 0; v < n; ++v) {
                    cn[pc[height[v]]++] = v;
                    dn[pd[depth[v]]++] = v;
                }
            }
            // per-level work lists
            std::vector<int64_t> ct_off(1, 0), ce_off(1, 0), de_off(1, 0);
            std::vector<int32_t> ct_node, ct_t, ce_ent, ce_node, de_ent, de_node, de_a;
            for (size_t l = 0; l + 1 < c_off.size(); ++l) {
                for (int64_t q = c_off[l]; q < c_off[l + 1]; ++q) {
                    const int32_t v = cn[q];
                    for (int32_t tt = 0; tt <= (int32_t)nbr[v].size(); ++tt) {
                        ct_node.push_back(v);
                        ct_t.push_back(tt);
                    }
                    for (int32_t a = 0; a < (int32_t)nbr[v].size(); ++a) {
                        ce_ent.push_back(col_ptr[v] + a);
                        ce_node.push_back(v);
                    }
                }
                ct_off.push_back((int64_t)ct_node.size());
                ce_off.push_back((int64_t)ce_ent.size());
            }
            for (size_t l = 0; l + 1 < d_off.size(); ++l) {
                for (int64_t q = d_off[l]; q < d_off[l + 1]; ++q) {
                    const int32_t v = dn[q];
                    for (int32_t a = 0; a < (int32_t)nbr[v].size(); ++a) {
                        de_ent.push_back(col_ptr[v] + a);
                        de_node.push_back(v);
                        de_a.push_back(a);
                    }
                }
                de_off.push_back((int64_t)de_ent.size());
            }
            // distribute pair codes
            std::vector<int32_t> pair_ptr(n + 1, 0), pair;
            for (int32_t v = 0; v < n; ++v) pair_ptr[v + 1] = pair_ptr[v] + (int32_t)(nbr[v].size() * nbr[v].size());
            pair.resize(std::max<int32_t>(pair_ptr[n], 1));
            for (int32_t v = 0; v < n; ++v) {
                const auto &nv = nbr[v];
                const int32_t d = (int32_t)nv.size();
                for (int32_t a = 0; a < d; ++a)
                    for (int32_t c = 0; c < d; ++c) {
                        const int32_t x = nv[a], y = nv[c];
                        pair[pair_ptr[v] + a * d + c] = x == y ? -(x + 1) : 2 * slot_of(x, y) + (x < y ? 1 : 0);
                    }
            }
            // held by a unique_ptr until handed out, so a host allocation
            // failure below (caught at the C ABI) releases it and its tables
            std::unique_ptr<selinv_junction_plan_s, void (*)(selinv_junction_plan_s *)> hold(
                new (std::nothrow) selinv_junction_plan_s(), selinv_junction_plan_free);
            if (!hold) return SELINV_ERR_HOST_MEMORY;
            selinv_junction_plan_s *pl = hold.get();
            pl->n = n;
            pl->m = m;
            pl->nnz = (int64_t)S.size();
            pl->E = E;
            cudaGetDevice(&pl->device);
            pl->order = seq;
            pl->S_i.resize(S.size());
            pl->S_j.resize(S.size());
            for (size_t q = 0; q < S.size(); ++q) {
                pl->S_i[q] = S[q].first;
                pl->S_j[q] = S[q].second;
            }
            pl->c_off = c_off;
            pl->d_off = d_off;
            pl->ct_off = ct_off;
            pl->ce_off = ce_off;
            pl->de_off = de_off;
            bool ok = true;
            auto up = [&](int32_t **dst, const std::vector<int32_t> &src) {
                if (!ok) return;
                const size_t nb = std::max<size_t>(src.size(), 1) * sizeof(int32_t);
                ok = cudaMalloc(dst, nb) == cudaSuccess &&
                     (src.empty() || cudaMemcpy(*dst, src.data(), src.size() * sizeof(int32_t),
                                                cudaMemcpyHostToDevice) == cudaSuccess);
            };
            up(&pl->d_c_nodes, cn);
            up(&pl->d_d_nodes, dn);
            up(&pl->d_col_ptr, col_ptr);
            up(&pl->d_ent_slot, ent_slot);
            up(&pl->d_ent_trans, ent_trans);
            up(&pl->d_ent_src, ent_src);
            up(&pl->d_con_ptr, tcount);
            up(&pl->d_con_w, cw);
            up(&pl->d_con_a, ca);
            up(&pl->d_pair_ptr, pair_ptr);
            up(&pl->d_pair, pair);
            up(&pl->d_ct_node, ct_node);
            up(&pl->d_ct_t, ct_t);
            up(&pl->d_ce_ent, ce_ent);
            up(&pl->d_ce_node, ce_node);
            up(&pl->d_de_ent, de_ent);
            up(&pl->d_de_node, de_node);
            up(&pl->d_de_a, de_a);
            {
                std::vector<int32_t> owner(std::max<int64_t>(E, 1), 0), uu(std::max<int64_t>(E, 1), 0);
                for (int32_t v = 0; v < n; ++v)
                    for (int32_t a = 0; a < (int32_t)nbr[v].size(); ++a) {
                        owner[col_ptr[v] + a] = v;
                        uu[col_ptr[v] + a] = nbr[v][a];
                    }
                up(&pl->d_ent_owner, owner);
                up(&pl->d_ent_u, uu);
            }
            if (!ok) return SELINV_ERR_CUDA;
            *out = hold.release();
        }
    }
    return SELINV_OK;
}

selinv_status selinv_junction_plan(int64_t n, int64_t m, const int32_t *ei, const int32_t *ej, const int32_t *order,
                                   selinv_junction_plan_t **out)
{
    // host tables are C++ containers: no exception may leave the C ABI
    try {
        return junction_plan_impl(n, m, ei, ej, order, out);
    } catch (const std::bad_alloc &) {
        if (out) *out = nullptr;
        return SELINV_ERR_HOST_MEMORY;
    } catch (...) {
        if (out) *out = nullptr;
        return SELINV_ERR_INVALID_ARG;
    }
}

selinv_status selinv_junction_symbolic(int64_t n, int64_t m, const int32_t *ei, const int32_t *ej, const int32_t *order,
                                       int64_t *nnz_S, int32_t *S_i, int32_t *S_j, int64_t capacity,
                                       int32_t *order_out)
{
    try {
        JSym sy;
        const selinv_status st = junction_symbolic_impl(n, m, ei, ej, order, sy);
        if (st != SELINV_OK) return st;
        if (nnz_S) *nnz_S = (int64_t)sy.S.size();
        for (int64_t q = 0; q < (int64_t)sy.S.size() && q < capacity; ++q) {
            if (S_i) S_i[q] = sy.S[q].first;
            if (S_j) S_j[q] = sy.S[q].second;
        }
        if (order_out) std::copy(sy.seq.begin(), sy.seq.end(), order_out);
        return SELINV_OK;
    } catch (const std::bad_alloc &) {
        return SELINV_ERR_HOST_MEMORY;
    } catch (...) {
        return SELINV_ERR_INVALID_ARG;
    }
}

selinv_status selinv_junction_plan_info(const selinv_junction_plan_t *pl, int64_t *nnz_S, int32_t *collect_levels,
                                        int32_t *distribute_levels)
{
    if (!pl) return SELINV_ERR_INVALID_ARG;
    if (nnz_S) *nnz_S = pl->nnz;
    if (collect_levels) *collect_levels = (int32_t)pl->c_off.size() - 1;
    if (distribute_levels) *distribute_levels = (int32_t)pl->d_off.size() - 1;
    return SELINV_OK;
}

int64_t selinv_junction_plan_launches(const selinv_junction_plan_t *pl)
{
    if (!pl) return -1;
    int64_t k = 2;                                     // init, finalize
    for (size_t l = 0; l + 1 < pl->c_off.size(); ++l) k += 2 + (pl->ce_off[l + 1] > pl->ce_off[l] ? 1 : 0);
    for (size_t l = 0; l + 1 < pl->d_off.size(); ++l) k += 1 + (pl->de_off[l + 1] > pl->de_off[l] ? 1 : 0);
    return k;
}

selinv_status selinv_junction_plan_pattern(const selinv_junction_plan_t *pl, int32_t *S_i, int32_t *S_j,
                                           int32_t *order)
{
    if (!pl) return SELINV_ERR_INVALID_ARG;
    if (S_i) std::copy(pl->S_i.begin(), pl->S_i.end(), S_i);
    if (S_j) std::copy(pl->S_j.begin(), pl->S_j.end(), S_j);
    if (order) std::copy(pl->order.begin(), pl->order.end(), order);
    return SELINV_OK;
}

size_t selinv_junction_workspace_size(const selinv_junction_plan_t *pl, selinv_dtype dtype, int32_t b, int64_t batch)
{
    if (!pl || (dtype != SELINV_F64 && dtype != SELINV_F32) || b < 1 || b > 16 || batch < 0) return 0;
    if (b <= 8) return dtype == SELINV_F64 ? ws_bytes<double, 64>(pl, batch) : ws_bytes<float, 64>(pl, batch);
    return dtype == SELINV_F64 ? ws_bytes<double, 256>(pl, batch) : ws_bytes<float, 256>(pl, batch);
}

selinv_status selinv_junction(const selinv_junction_plan_t *pl, selinv_dtype dtype, int32_t b, int64_t batch,
                              const void *diag, const void *edge_val, void *G_diag, void *G_lower, double *logdet,
                              int32_t *info, void *workspace, size_t workspace_bytes, void *stream)
{
    if (!pl || (dtype != SELINV_F64 && dtype != SELINV_F32) || b < 1 || batch < 0) return SELINV_ERR_INVALID_ARG;
    if (b > 16) return SELINV_ERR_UNSUPPORTED;
    if (batch == 0) return SELINV_OK;
    if (!diag || (pl->m > 0 && !edge_val) || !G_diag || (pl->nnz > 0 && !G_lower) || !info)
        return SELINV_ERR_INVALID_ARG;
    const size_t es = dtype == SELINV_F64 ? 8 : 4;
    if (!is_aligned(diag, es) || !is_aligned(edge_val, es) || !is_aligned(G_diag, es) || !is_aligned(G_lower, es) ||
        !is_aligned(logdet, 8) || !is_aligned(info, 4) || !is_aligned(workspace, 256))
        return SELINV_ERR_INVALID_ARG;
    const size_t need = selinv_junction_workspace_size(pl, dtype, b, batch);
    if (!workspace || workspace_bytes < need) return SELINV_ERR_WORKSPACE;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != pl->device) return SELINV_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t err;
    const double *dd = static_cast<const double *>(diag), *de = static_cast<const double *>(edge_val);
    const float *fd = static_cast<const float *>(diag), *fe = static_cast<const float *>(edge_val);
    double *dg = static_cast<double *>(G_diag), *dl = static_cast<double *>(G_lower);
    float *fg = static_cast<float *>(G_diag), *fl = static_cast<float *>(G_lower);
    auto *mp = const_cast<selinv_junction_plan_s *>(pl);      // the graph cache is the plan's own mutable state
    const int dt = (int)dtype;
    if (dtype == SELINV_F64)
        err = b <= 8 ? junction_call<double, Pol8<double>>(mp, dt, b, batch, dd, de, dg, dl, logdet, info, workspace, s)
                     : junction_call<double, Pol16<double>>(mp, dt, b, batch, dd, de, dg, dl, logdet, info, workspace, s);
    else
        err = b <= 8 ? junction_call<float, Pol8<float>>(mp, dt, b, batch, fd, fe, fg, fl, logdet, info, workspace, s)
                     : junction_call<float, Pol16<float>>(mp, dt, b, batch, fd, fe, fg, fl, logdet, info, workspace, s);
    return err == cudaSuccess ? SELINV_OK : SELINV_ERR_CUDA;
}

selinv_status selinv_junction_solve(const selinv_junction_plan_t *pl, selinv_dtype dtype, int32_t b, int64_t batch,
                                    const void *diag, const void *edge_val, const void *rhs, void *x, double *logdet,
                                    int32_t *info, void *workspace, size_t workspace_bytes, void *stream)
{
    if (!pl || (dtype != SELINV_F64 && dtype != SELINV_F32) || b < 1 || batch < 0) return SELINV_ERR_INVALID_ARG;
    if (b > 16) return SELINV_ERR_UNSUPPORTED;
    if (batch == 0) return SELINV_OK;
    if (!diag || (pl->m > 0 && !edge_val) || !rhs || !x || !info) return SELINV_ERR_INVALID_ARG;
    if (rhs == x) return SELINV_ERR_INVALID_ARG;
    const size_t es = dtype == SELINV_F64 ? 8 : 4;
    if (!is_aligned(diag, es) || !is_aligned(edge_val, es) || !is_aligned(rhs, es) || !is_aligned(x, es) ||
        !is_aligned(logdet, 8) || !is_aligned(info, 4) || !is_aligned(workspace, 256))
        return SELINV_ERR_INVALID_ARG;
    const size_t need = selinv_junction_workspace_size(pl, dtype, b, batch);
    if (!workspace || workspace_bytes < need) return SELINV_ERR_WORKSPACE;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != pl->device) return SELINV_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto *mp = const_cast<selinv_junction_plan_s *>(pl);
    const int dt = (int)dtype;
    cudaError_t err;
    if (dtype == SELINV_F64) {
        const double *dd = static_cast<const double *>(diag), *de = static_cast<const double *>(edge_val);
        const double *r = static_cast<const double *>(rhs);
        double *xx = static_cast<double *>(x);
        err = b <= 8 ? junction_call<double, Pol8<double>>(mp, dt, b, batch, dd, de, nullptr, nullptr, logdet, info,
                                                           workspace, s, r, xx)
                     : junction_call<double, Pol16<double>>(mp, dt, b, batch, dd, de, nullptr, nullptr, logdet, info,
                                                            workspace, s, r, xx);
    } else {
        const float *fd = static_cast<const float *>(diag), *fe = static_cast<const float *>(edge_val);
        const float *r = static_cast<const float *>(rhs);
        float *xx = static_cast<float *>(x);
        err = b <= 8 ? junction_call<float, Pol8<float>>(mp, dt, b, batch, fd, fe, nullptr, nullptr, logdet, info,
                                                         workspace, s, r, xx)
                     : junction_call<float, Pol16<float>>(mp, dt, b, batch, fd, fe, nullptr, nullptr, logdet, info,
                                                          workspace, s, r, xx);
    }
    return err == cudaSuccess ? SELINV_OK : SELINV_ERR_CUDA;
}

}  // extern "C"
