// Block trees: plan (host) and the collect / distribute kernels (b <= 16,
// one warp per node at a time).
//
// gabp-sparse-inv 0.3.2 (PyPI page), "Implemented and tested kernels" ->
// Tree: a parent array and one edge block per non-root node,
// edge[v] = A_{parent(v), v}; collect from the leaves to the root, then
// distribute from the root to the leaves.  The package batches its tree
// kernel by elimination level ("General sparse selected inverse": one batched
// step per level instead of per node).  Here the level sets order the work
// but do not separate launches: one launch per sweep over the whole forest.
//  * collect: warps take leaves; a warp that finishes a node and is the last
//    of its parent's children to do so (an atomic count) goes on with the
//    parent, so no warp ever waits;
//  * distribute: warps take non-root nodes in depth order and wait (bounded)
//    for their parent's diagonal block to be published; a parent is always
//    taken before its children by a warp that is already running, so every
//    wait ends.
//
// Collect, node v (all children already done):
//   S_v = D_v - sum_{c in ch(v)} U_c,        U_c = E_c S_c^-1 E_c^T
//   S_v^-1 and log det S_v; if v is not a root, U_v = W_v E_v^T with
//   W_v = E_v S_v^-1 is left in the workspace for the parent.
// Distribute, node v with parent p (G_pp already written):
//   G_edge[v] = -G_pp W_v,   G_vv = S_v^-1 - W_v^T G_edge[v]
// (S_v^-1 E_v^T G_edge[v] = W_v^T G_edge[v]).  Roots get G = S^-1 in collect.
#include <algorithm>
#include <climits>
#include <memory>
#include <new>
#include <vector>

#include "kernels.h"
#include "warp16.cuh"

struct selinv_tree_plan_s {
    int64_t trees = 0, n = 0;
    int device = 0;
    std::vector<int64_t> collect_off;      // [H + 1] into collect_nodes
    std::vector<int64_t> dist_off;         // [Dm + 1] into dist_nodes (depth >= 1)
    int32_t *d_collect_nodes = nullptr;    // global node ids by (height, id)
    int32_t *d_dist_nodes = nullptr;       // non-root global ids by (depth, id)
    int32_t *d_child_ptr = nullptr;        // [trees*n + 1]
    int32_t *d_child_idx = nullptr;        // global ids, ascending per parent
    int32_t *d_cpos = nullptr;             // [trees*n] position of each node in its parent's list, -1 roots
    int32_t *d_cont = nullptr;             // [trees*n] first child of a non-root node, else -1
    int32_t *d_heads = nullptr;            // distribute chain heads by (depth, id)
    int64_t nheads = 0;
    int32_t *d_parent = nullptr;           // global parent id or -1
    int32_t spin_limit = 1 << 22;          // polls before a dependency wait gives up (SPIN_LIMIT)
    int64_t hold = -1;                     // node whose completion is never published (tests)
};

namespace selinv {

namespace {

constexpr int TWARPS = 4;
constexpr int DRAW_SLOT = 256;      // draws: W_v^T per node, 16 x 16 row-major (>= SLOT_ELEMS)

template <class T> __host__ __device__ constexpr int tree_smem_elems() { return 4 * w16::SL<T>::ELEMS + 64; }
// distribute: two (edge, S^-1 slot) buffer sets for the node being processed
// and the next one, plus G_pp and two transpose images
template <class T> __host__ __device__ constexpr int dist_smem_elems()
{
    return 5 * w16::SL<T>::ELEMS + 2 * w16::SLOT_ELEMS;
}

struct TreeDev {
    const int32_t *child_ptr;
    const int32_t *child_idx;
    const int32_t *parent;
    int64_t n;
    int32_t spin_limit;   // polls before a dependency wait gives up
    int64_t hold;         // a node whose completion flag is never published (tests), or -1
    const int32_t *cpos;  // position of each node in its parent's child list (-1 for roots)
    const int32_t *cont;  // first child of a non-root node (its chain goes on there), else -1
};

template <class T> struct TreeBufs {
    const T *diag, *edge;
    T *G_diag, *G_edge;
    const T *z;              // draws: standard normals [N, b]
    T *eta;                  // draws: R_v z_v after the collect sweep, the draw after the distribute sweep
    T *ws_sinv, *ws_u;       // lower slots: S_v^-1 per node, U_v at v's position in its parent's child list
    double *ws_ld;           // per node log det S_v
    int32_t *info;           // per tree, INT_MAX = ok until finalised
    int b;
};

struct TreeSync {
    int32_t *pending;     // [N] children of a node not collected yet
    int32_t *done;        // [N] 1 once G_vv is written (distribute)
    unsigned long long *counters;   // [0] leaves taken, [1] distribute nodes taken
};

constexpr int SPIN_LIMIT = 1 << 22;     // x >= 64 ns per poll: well over a second

// Completion flags of the sweeps: 0 = not yet, 1 = the node's data is
// published, 2 = the node gave up (its own wait ran out, or its parent gave
// up), so its children give up at once instead of each spinning to the limit.
constexpr int FLAG_READY = 1, FLAG_FAILED = 2;

SELINV_DEVINL unsigned long long warp_take(unsigned long long *ctr, int lane)
{
    unsigned long long k = 0;
    if (lane == 0) k = atomicAdd(ctr, 1ull);
    return __shfl_sync(FULL_MASK, k, 0);
}

SELINV_DEVINL int ld_acquire(const int32_t *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Atomic add with acquire-release semantics at GPU scope: releases the
// caller's earlier writes (and, through a preceding warp barrier, its warp's)
// and acquires every write released by earlier adds to the same counter.
SELINV_DEVINL int atom_add_acq_rel(int32_t *p, int v)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;\n" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

SELINV_DEVINL void st_release(int32_t *p, int v)
{
    asm volatile("st.release.gpu.global.s32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait of lane 0 for a parent's completion flag, broadcast to the
// warp: 1 when the parent's data may be read, 0 when the parent gave up or
// the flag stayed unset for td.spin_limit polls.
SELINV_DEVINL int wait_parent(const int32_t *flag, int limit, int lane, unsigned sleep_ns)
{
    int ok = 0;
    if (lane == 0) {
        int n = 0, f;
        while ((f = ld_acquire(flag)) == 0 && ++n <= limit) __nanosleep(sleep_ns);
        ok = f == FLAG_READY;
    }
    return __shfl_sync(FULL_MASK, ok, 0);
}

// Lane 0 publishes node v's completion (after a warp barrier that orders the
// warp's stores before it); a node held back for a test stays unpublished.
SELINV_DEVINL void publish(int32_t *done, const TreeDev &td, int32_t v, int lane)
{
    if (lane == 0 && v != td.hold) st_release(done + v, FLAG_READY);
}

// A wait gave up: the tree reports -2 and v's children (if any) give up too.
SELINV_DEVINL void give_up(int32_t *info, int32_t *done, const TreeDev &td, int32_t v, int lane)
{
    if (lane == 0) {
        atomicMin(info + v / td.n, -2);
        if (td.child_ptr[v + 1] > td.child_ptr[v]) st_release(done + v, FLAG_FAILED);
    }
}

template <class T> SELINV_DEVINL void load_lower_slot_l2(w16::Tile<T> &a, const T *slot, int lane, int g, int t)
{
    using V = typename w16::Vec2<T>::type;
    V v = __ldcg(reinterpret_cast<const V *>(slot + 2 * lane));
    a.v[1][0] = v.x;
    a.v[1][1] = v.y;
    a.v[0][2] = a.v[0][3] = T(0);
    if (2 * t <= g) {
        V u = __ldcg(reinterpret_cast<const V *>(slot + 64 + 4 * lane));
        V w = __ldcg(reinterpret_cast<const V *>(slot + 64 + 4 * lane + 2));
        a.v[0][0] = u.x;
        a.v[0][1] = u.y;
        a.v[1][2] = w.x;
        a.v[1][3] = w.y;
    } else {
        a.v[0][0] = a.v[0][1] = a.v[1][2] = a.v[1][3] = T(0);
    }
}

template <class T, bool FULL, bool DRAW>
SELINV_DEVINL void collect_sweep(const TreeBufs<T> &p, const TreeDev &td, const TreeSync &sy, const int32_t *leaves,
                                 int64_t nleaves)
{
    using namespace w16;
    constexpr int E = SL<T>::ELEMS;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *sB = reinterpret_cast<T *>(smem_raw) + wid * tree_smem_elems<T>();
    T *sD = sB + E, *sT = sD + E, *sT2 = sT + E, *cb = sT2 + E;
    const int b = p.b;
    const int64_t bb = (int64_t)b * b;

    for (;;) {
        const unsigned long long k = warp_take(sy.counters, lane);
        if (k >= (unsigned long long)nleaves) break;
        int32_t v = leaves[k];
        for (;;) {                                   // v, then each parent this warp completes last
            const int32_t par = td.parent[v];
            if (par >= 0) load_block_async<T, FULL>(sB, p.edge + v * bb, b, lane);   // E_v
            load_lower_async<T, FULL>(sD, p.diag + v * bb, b, lane);                 // D_v
            cp_async_commit();
            T zc[4];                                  // draws: z_v at the lane's columns
            if constexpr (DRAW) {
#pragma unroll
                for (int q = 0; q < 4; ++q) zc[q] = tcol(t, q) < b ? p.z[(int64_t)v * b + tcol(t, q)] : T(0);
            }
            Tile<T> acc;                              // sum of the children's U_c (lower slots), two
            zero(acc);                                // children's loads in flight at a time
            const int32_t c0 = td.child_ptr[v], c1 = td.child_ptr[v + 1];
            for (int32_t c = c0; c < c1; c += 2) {    // children's slots sit at their list positions
                Tile<T> u, u2;
                load_lower_slot_l2<T>(u, p.ws_u + (int64_t)c * SLOT_ELEMS, lane, g, t);
                if (c + 1 < c1) load_lower_slot_l2<T>(u2, p.ws_u + (int64_t)(c + 1) * SLOT_ELEMS, lane, g, t);
                else zero(u2);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc.v[h][q] += u.v[h][q] + u2.v[h][q];
            }
            cp_async_wait_all();
            __syncwarp();
            Tile<T> a;
            from_smem_lower<T>(a, sD, g, t);
            if (c1 > c0) {                            // S_v = D_v - sum U_c (mirrored from the lower slots)
                to_smem<T>(sT, acc, g, t);
                __syncwarp();
                from_smem_lower<T>(acc, sT, g, t);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int q = 0; q < 4; ++q) a.v[h][q] -= acc.v[h][q];
            }
            LogAcc det;
            det.init();
            bool bad = false;
            T vv[2] = {T(0), T(0)};                  // draws: R_v z_v at rows g, g + 8 (S_v = R_v R_v^T)
            if constexpr (DRAW) {
                if constexpr (sizeof(T) == 8) spd_inverse_blocked<true>(a, g, t, det, bad, zc, vv);
                else spd_inverse_scalar<T, true>(a, cb, g, t, det, bad, zc, vv);
            } else {
                spd_inverse<T>(a, cb, g, t, det, bad);
            }
            if (lane == 0) {
                p.ws_ld[v] = det.log_value();
                if (bad) atomicMin(p.info + v / td.n, (int32_t)(v % td.n));
            }
            if constexpr (DRAW) {                     // u_v = S_v^-1 R_v z_v = R_v^-T z_v
                if (t == 0) {
                    cb[g] = vv[0];
                    cb[g + 8] = vv[1];
                }
                __syncwarp();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    T s2 = T(0);
#pragma unroll
                    for (int q = 0; q < 4; ++q) s2 = fma(a.v[h][q], cb[tcol(t, q)], s2);
                    s2 += shfl_xor(s2, 1);
                    s2 += shfl_xor(s2, 2);
                    if (t == 0 && g + 8 * h < b) p.eta[(int64_t)v * b + g + 8 * h] = s2;
                }
                if (par < 0) {                        // root: its draw is u_v, published
                    __syncwarp();                     // the warp's stores are ordered before lane 0's release
                    publish(sy.done, td, v, lane);
                    __syncwarp();
                    break;
                }
            }
            if (par < 0) {                            // root: G = S^-1, G_edge = 0, published
                __syncwarp();
                to_smem<T>(sT, a, g, t);
                __syncwarp();
                from_smem_lower<T>(a, sT, g, t);
                store_block<T, FULL>(p.G_diag + v * bb, a, b, g, t);
                Tile<T> z;
                zero(z);
                store_block<T, FULL>(p.G_edge + v * bb, z, b, g, t);
                __syncwarp();                         // the warp's stores are ordered before lane 0's release
                publish(sy.done, td, v, lane);
                __syncwarp();
                break;
            }
            if (!DRAW) store_lower_slot<T>(p.ws_sinv + (int64_t)v * SLOT_ELEMS, a, lane, g, t);
            Tile<T> et, w, u;
            from_smem<T>(et, sB, g, t);               // E_v
            zero(w);
            gemm_nt<false>(w, et, a, sT, sT2, g, t);  // W_v = E_v S_v^-1
            if (DRAW) store_block_T<T, true>(p.ws_sinv + (int64_t)v * DRAW_SLOT, w, 16, g, t);   // W_v^T, 16 x 16
            zero(u);
            gemm_nt<false, true>(u, w, et, sT, sT2, g, t);   // U_v = W_v E_v^T (lower tiles)
            store_lower_slot<T>(p.ws_u + (int64_t)td.cpos[v] * SLOT_ELEMS, u, lane, g, t);
            __syncwarp();                             // the warp's stores are ordered before lane 0's release
            int old = 0;
            if (lane == 0) old = atom_add_acq_rel(sy.pending + par, -1);   // release U_v; the last child acquires all siblings'
            old = __shfl_sync(FULL_MASK, old, 0);
            __syncwarp();                             // every lane's reads of the siblings' U follow lane 0's acquire
            if (old != 1) break;                      // a sibling is still running: it will go on
            v = par;
        }
    }
}

// The collect sweep without and with the draws' extra state; the draw
// variant is held to 96 registers so that five CTAs fit an SM, as for the
// plain sweep.
template <class T, bool FULL>
__global__ void __launch_bounds__(TWARPS * 32)
tree_collect_kernel(TreeBufs<T> p, TreeDev td, TreeSync sy, const int32_t *leaves, int64_t nleaves)
{
    collect_sweep<T, FULL, false>(p, td, sy, leaves, nleaves);
}
template <class T, bool FULL>
__global__ void __launch_bounds__(TWARPS * 32, 5)
tree_collect_draw_kernel(TreeBufs<T> p, TreeDev td, TreeSync sy, const int32_t *leaves, int64_t nleaves)
{
    collect_sweep<T, FULL, true>(p, td, sy, leaves, nleaves);
}

template <class T, bool FULL>
__global__ void __launch_bounds__(TWARPS * 32)
tree_distribute_kernel(TreeBufs<T> p, TreeDev td, TreeSync sy, const int32_t *heads, int64_t count)
{
    using namespace w16;
    constexpr int E = SL<T>::ELEMS;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *base = reinterpret_cast<T *>(smem_raw) + wid * dist_smem_elems<T>();
    // buffers of the current / next node (c = 0, 1), addressed arithmetically so
    // that no pointer array ends up in local memory
    auto sBuf = [&](int c) { return base + c * E; };                      // E_v
    T *sG = base + 2 * E, *sT = sG + E, *sT2 = sT + E;
    auto stg = [&](int c) { return sT2 + E + c * SLOT_ELEMS; };          // S_v^-1 slots
    const int b = p.b;
    const int64_t bb = (int64_t)b * b;
    const unsigned long long cnt = (unsigned long long)count;
    auto prefetch = [&](int32_t u, int c) {
        load_block_async<T, FULL>(sBuf(c), p.edge + u * bb, b, lane);
        stage_lower_slot<T>(stg(c), p.ws_sinv + (int64_t)u * SLOT_ELEMS, lane, g, t);
        cp_async_commit();
    };

    // A warp takes a chain head from the depth-ordered list (every non-root
    // node except the first child of a non-root parent), waits for its parent's
    // flag and reads G_pp, then runs down the chain of first children: each
    // one's G_pp is the G_vv the warp has just formed, in registers, so it
    // neither waits nor loads it.  The next node (the first child, or the next
    // head) is known before the current one is computed, and its edge block
    // and S^-1 slot stream in meanwhile (waiting for "all but the newest group"
    // waits for exactly the current node's data and G_pp).
    int32_t v;
    {
        const unsigned long long k = warp_take(sy.counters + 1, lane);
        v = k < cnt ? heads[k] : -1;
    }
    int cur = 0;
    if (v >= 0) prefetch(v, 0);
    bool head = true;                                 // v came from the list
    bool failed = false;                              // the chain's head gave up
    Tile<T> G;                                        // G_vv of the node before v in its chain
    zero(G);
    while (v >= 0) {
        const int32_t par = td.parent[v];
        const int32_t c = td.cont[v];
        int ok;
        if (head) {
            ok = wait_parent(sy.done + par, td.spin_limit, lane, 64);   // G_pp (bounded wait)
            __syncwarp();                             // every lane's reads below are ordered after lane 0's acquire
            if (ok) load_lower_async<T, FULL>(sG, p.G_diag + (int64_t)par * bb, b, lane);   // G_pp, from L2
            cp_async_commit();
            failed = !ok;
        } else {
            failed = failed || par == td.hold;        // a withheld node's flag would never have come
            ok = !failed;
        }
        int32_t nxt = c;
        if (c < 0) {
            const unsigned long long kn = warp_take(sy.counters + 1, lane);
            nxt = kn < cnt ? heads[kn] : -1;
        }
        if (nxt >= 0) {
            prefetch(nxt, cur ^ 1);
            cp_async_wait_one();
        } else {
            cp_async_wait_all();
        }
        __syncwarp();
        if (!ok) {                                    // the parent never published: report, pass it on
            give_up(p.info, sy.done, td, v, lane);
        } else {
            Tile<T> a;
            unstage_lower_slot<T>(a, stg(cur), lane, g, t);
            to_smem<T>(sT, a, g, t);                  // lower entries of S_v^-1 valid
            __syncwarp();
            from_smem_lower<T>(a, sT, g, t);          // S_v^-1, full
            Tile<T> gp, et, wt, get;
            if (head) from_smem_lower<T>(gp, sG, g, t);   // G_pp, full
            else gp = G;
            from_smem<T>(et, sBuf(cur), g, t);        // E_v
            // W_v^T = S_v^-1 E_v^T and G_edge[v]^T = -W_v^T G_pp are X Y^T products of
            // register tiles (S_v^-1, G_pp symmetric): nothing is transposed.
            zero(wt);
            gemm_nt<false>(wt, a, et, sT, sT2, g, t); // W_v^T = S_v^-1 E_v^T
            zero(get);
            gemm_nt<true>(get, wt, gp, sT, sT2, g, t);   // G_edge[v]^T = -W_v^T G_pp
            store_block_T<T, FULL>(p.G_edge + v * bb, get, b, g, t);
            gemm_nt<true, true>(a, wt, get, sT, sT2, g, t);   // G_vv = S_v^-1 - W_v^T G_edge[v] (lower tiles)
            __syncwarp();
            to_smem<T>(sT, a, g, t);
            __syncwarp();
            from_smem_lower<T>(G, sT, g, t);          // exactly symmetric
            store_block<T, FULL>(p.G_diag + v * bb, G, b, g, t);
            __syncwarp();                             // the warp's stores are ordered before lane 0's release
            if (td.child_ptr[v + 1] - td.child_ptr[v] >= 2) publish(sy.done, td, v, lane);   // heads wait on it
            __syncwarp();
        }
        head = c < 0;
        v = nxt;
        cur ^= 1;
    }
}

// Draws, top-down: w_v = u_v - W_v^T w_p with u_v = R_v^-T z_v and W_v^T
// left by the collect sweep (W_v^T as a 16 x 16 row-major slot, zero outside
// b x b) and w_p published by the parent (or, along a chain, just formed by
// the same warp).  Lane (r, hf) = (lane / 2, lane % 2) holds row r, columns
// 8 hf .. 8 hf + 7.  Every wait ends: a head's parent was handed out earlier,
// to a warp that is running and waits on nothing later.
constexpr int DRAW_THREADS = 256;

template <class T, bool FULL>
__global__ void __launch_bounds__(DRAW_THREADS)
tree_draw_kernel(TreeBufs<T> p, TreeDev td, TreeSync sy, const int32_t *heads, int64_t count)
{
    const int lane = threadIdx.x & 31;
    const int r = lane >> 1, hf = lane & 1;
    const int b = p.b;
    // W_v^T row r (the lane's eight columns) and u_v[r] of node u
    auto load_node = [&](int32_t u, T w[8], T &uu) {
        const T *row = p.ws_sinv + (int64_t)u * DRAW_SLOT + r * 16 + 8 * hf;
        if constexpr (sizeof(T) == 8) {
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                const double2 x = __ldcs(reinterpret_cast<const double2 *>(row + c));
                w[c] = x.x;
                w[c + 1] = x.y;
            }
        } else {
#pragma unroll
            for (int c = 0; c < 8; c += 4) {
                const float4 x = __ldcs(reinterpret_cast<const float4 *>(row + c));
                w[c] = x.x;
                w[c + 1] = x.y;
                w[c + 2] = x.z;
                w[c + 3] = x.w;
            }
        }
        uu = r < b ? p.eta[(int64_t)u * b + r] : T(0);
    };
    // The distribute sweep's chains: a warp takes a chain head, waits for its
    // parent's w_p, and runs down the chain of first children, each one's w_p
    // being the w_v it has just formed (moved to the lanes' columns by
    // shuffles); the next node's W^T row and u are loaded before the current
    // one's wait.  A warp holds no other node while it waits, so a wait that
    // runs out in one tree delays no other tree.
    for (;;) {
        const unsigned long long k = warp_take(sy.counters + 1, lane);
        if (k >= (unsigned long long)count) break;
        int32_t v = heads[k];
        T w[8], u;
        load_node(v, w, u);
        bool head = true, failed = false;
        T wp[8];                                      // w_p at the lane's columns 8 hf .. 8 hf + 7
#pragma unroll
        for (int c = 0; c < 8; ++c) wp[c] = T(0);
        while (v >= 0) {
            const int32_t par = td.parent[v];
            const int32_t cn = td.cont[v];
            T wn[8], un = T(0);
#pragma unroll
            for (int c = 0; c < 8; ++c) wn[c] = T(0);
            if (cn >= 0) load_node(cn, wn, un);
            int ok;
            if (head) {
                ok = wait_parent(sy.done + par, td.spin_limit, lane, 32);   // w_p (bounded wait)
                __syncwarp();                         // every lane's reads below follow lane 0's acquire
                failed = !ok;
                if (ok) {
                    const T *src = p.eta + (int64_t)par * b + 8 * hf;
#pragma unroll
                    for (int c = 0; c < 8; ++c) wp[c] = (FULL || 8 * hf + c < b) ? __ldcg(src + c) : T(0);
                }
            } else {
                failed = failed || par == td.hold;    // a withheld node's flag would never have come
                ok = !failed;
            }
            if (!ok) {                                // the parent never published: report, pass it on
                give_up(p.info, sy.done, td, v, lane);
            } else {
                T s2 = T(0);
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    if (FULL || 8 * hf + c < b) s2 = fma(w[c], wp[c], s2);
                s2 += shfl_xor(s2, 1);
                const T wv = u - s2;                  // w_v[r] (zero for r >= b)
                if (hf == 0 && r < b) p.eta[(int64_t)v * b + r] = wv;
#pragma unroll
                for (int c = 0; c < 8; ++c) wp[c] = __shfl_sync(FULL_MASK, wv, 2 * (8 * hf + c));
                __syncwarp();                         // the warp's stores are ordered before lane 0's release
                if (td.child_ptr[v + 1] - td.child_ptr[v] >= 2) publish(sy.done, td, v, lane);   // heads wait on it
                __syncwarp();
            }
            head = cn < 0;
            v = cn;
#pragma unroll
            for (int c = 0; c < 8; ++c) w[c] = wn[c];
            u = un;
        }
    }
}

// ---------------------------------------------------------------------------
// Cotangents (gabp-sparse-inv, "Differentiable selected inverse": selinv_tree's
// gradients reach diag and edge through an analytic two-pass backward).  The
// passes are the reverse-mode forms of the forward's sweeps, with P_v = S_v^-1,
// W_v = E_v P_v, p = parent(v):
// pass 1, children before parents (a fresh collect that rebuilds P_v, fused
// with the reversed distribute, which ran parents first):
//   Ga   = Gb_vv + sum_{c in ch(v)} C_c
//   Xb   = Gb_edge[v] - W_v Ga,  Wb = -G_edge[v] Ga^T - G_pp Xb
//   C_v  = -Xb W_v^T (to the parent),  Eb_v <- Wb P_v,
//   Pd_v = (Ga + E_v^T Wb) + its transpose   (only symmetric parts matter below)
//   root: Pd = Ga + Ga^T.
// pass 2, parents before children (the reversed collect), Sg = Sb + Sb^T:
//   Sg_v = -P_v (Pd_v - E_v^T Sg_p E_v) P_v   (root: -P Pd P)
//   Db_v = Sg_v below the diagonal, half of it on the diagonal, 0 above
//   Eb_v -= Sg_p W_v
// The root's pass-2 step runs where pass 1 ends, in the warp that reaches it.
template <class T> struct TreeBwdBufs {
    const T *diag, *edge, *G_diag, *G_edge, *Gb_diag, *Gb_edge;
    T *Db, *Eb;
    T *ws_P, *ws_U, *ws_C, *ws_Pd;   // per node: P_v and U_v (later Sg_v) lower slots, C_v full, Pd_v lower
    int32_t *info;
    int b;
};

constexpr int BW_CSLOT = 256;

// Symmetric tile from a lower slot written earlier in this launch (read
// through L2), rebuilt through the shared image s.
template <class T> SELINV_DEVINL void sym_from_slot(w16::Tile<T> &a, const T *slot, T *s, int lane, int g, int t)
{
    load_lower_slot_l2<T>(a, slot, lane, g, t);
    w16::to_smem<T>(s, a, g, t);
    __syncwarp();
    w16::from_smem_lower<T>(a, s, g, t);
    __syncwarp();
}

template <class T> SELINV_DEVINL void transpose_t(w16::Tile<T> &out, const w16::Tile<T> &in, T *s, int g, int t)
{
    w16::to_smem<T>(s, in, g, t);
    __syncwarp();
    w16::from_smem_T<T>(out, s, g, t);
    __syncwarp();
}

template <class T, bool FULL> SELINV_DEVINL void load_gen(w16::Tile<T> &a, const T *M, int b, int g, int t, bool l2)
{
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = g + 8 * h, c = w16::tcol(t, q);
            const int ld = FULL ? 16 : b;
            a.v[h][q] = (FULL || (r < b && c < b)) ? (l2 ? __ldcg(M + r * ld + c) : __ldg(M + r * ld + c)) : T(0);
        }
}

// Db_v from Sg_v, stored; Sg symmetric.
template <class T, bool FULL> SELINV_DEVINL void store_db(T *Db, const w16::Tile<T> &sg, int b, int g, int t)
{
    w16::Tile<T> d;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = g + 8 * h, c = w16::tcol(t, q);
            d.v[h][q] = c < r ? sg.v[h][q] : (c == r ? T(0.5) * sg.v[h][q] : T(0));
        }
    w16::store_block<T, FULL>(Db, d, b, g, t);
}

template <class T, bool FULL>
__global__ void __launch_bounds__(TWARPS * 32)
tree_bw_collect_kernel(TreeBwdBufs<T> p, TreeDev td, TreeSync sy, const int32_t *leaves, int64_t nleaves)
{
    using namespace w16;
    constexpr int E = SL<T>::ELEMS;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *s0 = reinterpret_cast<T *>(smem_raw) + wid * (3 * E + 32);
    T *s1 = s0 + E, *s2 = s1 + E, *cb = s2 + E;
    const int b = p.b;
    const int64_t bb = (int64_t)b * b;

    for (;;) {
        const unsigned long long k = warp_take(sy.counters, lane);
        if (k >= (unsigned long long)nleaves) break;
        int32_t v = leaves[k];
        for (;;) {                                   // v, then each parent this warp completes last
            const int32_t par = td.parent[v];
            Tile<T> S, Ga;
            load_sym<T, FULL>(S, p.diag + v * bb, b, g, t);
            if (p.Gb_diag) load_gen<T, FULL>(Ga, p.Gb_diag + v * bb, b, g, t, false);
            else zero(Ga);
            const int32_t c0 = td.child_ptr[v], c1 = td.child_ptr[v + 1];
            for (int32_t c = c0; c < c1; ++c) {        // S -= U_c, Ga += C_c
                const int32_t ch = td.child_idx[c];
                Tile<T> u, cc;
                sym_from_slot<T>(u, p.ws_U + (int64_t)ch * SLOT_ELEMS, s0, lane, g, t);
                load_gen<T, true>(cc, p.ws_C + (int64_t)ch * BW_CSLOT, 16, g, t, true);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        S.v[h][q] -= u.v[h][q];
                        Ga.v[h][q] += cc.v[h][q];
                    }
            }
            LogAcc det;
            det.init();
            bool bad = false;
            spd_inverse<T>(S, cb, g, t, det, bad);  // S = P_v
            if (lane == 0 && bad) atomicMin(p.info + v / td.n, (int32_t)(v % td.n));
            store_lower_slot<T>(p.ws_P + (int64_t)v * SLOT_ELEMS, S, lane, g, t);
            Tile<T> GaT;
            transpose_t<T>(GaT, Ga, s0, g, t);
            if (par < 0) {                            // root: Pd = Ga + Ga^T, then its pass-2 step
                Tile<T> pd = Ga, q, sg;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int r = 0; r < 4; ++r) pd.v[h][r] += GaT.v[h][r];
                zero(q);
                gemm_nt<false>(q, S, pd, s1, s2, g, t);            // P Pd
                zero(sg);
                gemm_nt<true, true>(sg, q, S, s1, s2, g, t);        // Sg = -P Pd P (lower tiles)
                mirror_upper(sg, g, t);
                store_db<T, FULL>(p.Db + v * bb, sg, b, g, t);
                Tile<T> z;
                zero(z);
                store_block<T, FULL>(p.Eb + v * bb, z, b, g, t);
                store_lower_slot<T>(p.ws_U + (int64_t)v * SLOT_ELEMS, sg, lane, g, t);
                __syncwarp();                         // the warp's stores are ordered before lane 0's release
                publish(sy.done, td, v, lane);
                __syncwarp();
                break;
            }
            Tile<T> Ev, W;
            load_gen<T, FULL>(Ev, p.edge + v * bb, b, g, t, false);
            zero(W);
            gemm_nt<false>(W, Ev, S, s1, s2, g, t);               // W = E P
            {
                Tile<T> u;
                zero(u);
                gemm_nt<false, true>(u, W, Ev, s1, s2, g, t);      // U = W E^T (lower tiles)
                store_lower_slot<T>(p.ws_U + (int64_t)v * SLOT_ELEMS, u, lane, g, t);
            }
            Tile<T> Xb, Wb;
            if (p.Gb_edge) load_gen<T, FULL>(Xb, p.Gb_edge + v * bb, b, g, t, false);
            else zero(Xb);
            gemm_nt<true>(Xb, W, GaT, s1, s2, g, t);              // Xb = Gb_edge - W Ga
            {
                Tile<T> X;
                load_gen<T, FULL>(X, p.G_edge + v * bb, b, g, t, false);
                zero(Wb);
                gemm_nt<true>(Wb, X, Ga, s1, s2, g, t);           // Wb = -G_edge Ga^T
            }
            {
                Tile<T> XbT, Gp;
                transpose_t<T>(XbT, Xb, s0, g, t);
                load_gen<T, FULL>(Gp, p.G_diag + (int64_t)par * bb, b, g, t, false);
                gemm_nt<true>(Wb, Gp, XbT, s1, s2, g, t);         // Wb -= G_pp Xb
            }
            {
                Tile<T> cv;
                zero(cv);
                gemm_nt<true>(cv, Xb, W, s1, s2, g, t);           // C_v = -Xb W^T
                store_block<T, true>(p.ws_C + (int64_t)v * BW_CSLOT, cv, 16, g, t);
            }
            {
                Tile<T> ET, WbT;
                transpose_t<T>(ET, Ev, s0, g, t);
                transpose_t<T>(WbT, Wb, s0, g, t);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int r = 0; r < 4; ++r) Ga.v[h][r] += GaT.v[h][r];
                gemm_nt<false>(Ga, ET, WbT, s1, s2, g, t);        // + E^T Wb
                gemm_nt<false>(Ga, WbT, ET, s1, s2, g, t);        // + Wb^T E
                store_lower_slot<T>(p.ws_Pd + (int64_t)v * SLOT_ELEMS, Ga, lane, g, t);
            }
            {
                Tile<T> ed;
                zero(ed);
                gemm_nt<false>(ed, Wb, S, s1, s2, g, t);          // Eb_v <- Wb P
                store_block<T, FULL>(p.Eb + v * bb, ed, b, g, t);
            }
            __syncwarp();                             // the warp's stores are ordered before lane 0's release
            int old = 0;
            if (lane == 0) old = atom_add_acq_rel(sy.pending + par, -1);
            old = __shfl_sync(FULL_MASK, old, 0);
            __syncwarp();                             // every lane's reads of the siblings' slots follow the acquire
            if (old != 1) break;
            v = par;
        }
    }
}

template <class T, bool FULL>
__global__ void __launch_bounds__(TWARPS * 32)
tree_bw_distribute_kernel(TreeBwdBufs<T> p, TreeDev td, TreeSync sy, const int32_t *nodes, int64_t count)
{
    using namespace w16;
    constexpr int E = SL<T>::ELEMS;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *s0 = reinterpret_cast<T *>(smem_raw) + wid * (3 * E + 32);
    T *s1 = s0 + E, *s2 = s1 + E;
    const int b = p.b;
    const int64_t bb = (int64_t)b * b;
    const unsigned long long cnt = (unsigned long long)count;
    // The distribute sweep's chains, reversed: a warp takes a chain head (every
    // non-root node except the first child of a non-root parent) in depth order,
    // waits for its parent's flag and reads Sg_p, then runs down the chain of
    // first children, each one's Sg_p being the Sg_v the warp has just formed.
    // The next node (first child, or next head) is known before the current one
    // is computed, and its operands are sent toward L2 meanwhile.  Every wait
    // still ends: the smallest unfinished head is some warp's current node, and
    // its parent, earlier in the depth order or earlier in a running chain, is
    // finished or being finished by a warp that waits on nothing later.
    int32_t v;
    {
        const unsigned long long k = warp_take(sy.counters + 1, lane);
        v = k < cnt ? nodes[k] : -1;
    }
    bool head = true, failed = false;
    Tile<T> Sn;                                       // Sg_v of the node before v in its chain
    zero(Sn);
    while (v >= 0) {
        const int32_t par = td.parent[v];
        const int32_t c = td.cont[v];
        int32_t nxt = c;
        if (c < 0) {
            const unsigned long long kn = warp_take(sy.counters + 1, lane);
            nxt = kn < cnt ? nodes[kn] : -1;
        }
        if (nxt >= 0) {
            prefetch_range_l2(p.ws_P + (int64_t)nxt * SLOT_ELEMS, SLOT_ELEMS, lane, 32);
            prefetch_range_l2(p.ws_Pd + (int64_t)nxt * SLOT_ELEMS, SLOT_ELEMS, lane, 32);
            prefetch_range_l2(p.edge + nxt * bb, bb, lane, 32);
            prefetch_range_l2(p.Eb + nxt * bb, bb, lane, 32);
        }
        // operands that do not depend on the parent first
        Tile<T> P, Pt, Ev, ed;
        sym_from_slot<T>(P, p.ws_P + (int64_t)v * SLOT_ELEMS, s0, lane, g, t);
        sym_from_slot<T>(Pt, p.ws_Pd + (int64_t)v * SLOT_ELEMS, s0, lane, g, t);
        load_gen<T, FULL>(Ev, p.edge + v * bb, b, g, t, false);
        load_gen<T, FULL>(ed, p.Eb + v * bb, b, g, t, true);
        int ok;
        if (head) {
            ok = wait_parent(sy.done + par, td.spin_limit, lane, 64);   // Sg_p (bounded wait)
            __syncwarp();                             // every lane's reads below follow lane 0's acquire
            failed = !ok;
        } else {
            failed = failed || par == td.hold;        // a withheld node's flag would never have come
            ok = !failed;
        }
        const bool was_head = head;
        head = c < 0;
        if (!ok) {                                    // the parent never published: report, pass it on
            give_up(p.info, sy.done, td, v, lane);
            v = nxt;
            continue;
        }
        Tile<T> Sp, ET;
        if (was_head) sym_from_slot<T>(Sp, p.ws_U + (int64_t)par * SLOT_ELEMS, s0, lane, g, t);
        else Sp = Sn;
        transpose_t<T>(ET, Ev, s0, g, t);
        {
            Tile<T> zt;
            zero(zt);
            gemm_nt<false>(zt, ET, Sp, s1, s2, g, t);             // E^T Sg_p
            gemm_nt<true>(Pt, zt, ET, s1, s2, g, t);              // Pt = Pd - E^T Sg_p E
        }
        {
            Tile<T> wt;
            zero(wt);
            gemm_nt<false>(wt, P, Ev, s1, s2, g, t);              // W^T = P E^T
            gemm_nt<true>(ed, Sp, wt, s1, s2, g, t);              // Eb_v = Eb_v - Sg_p W
            store_block<T, FULL>(p.Eb + v * bb, ed, b, g, t);
        }
        Tile<T> q, sg;
        zero(q);
        gemm_nt<false>(q, P, Pt, s1, s2, g, t);                   // P Pt (Pt symmetric)
        zero(sg);
        gemm_nt<true, true>(sg, q, P, s1, s2, g, t);              // Sg_v = -P Pt P (lower tiles)
        mirror_upper(sg, g, t);
        store_db<T, FULL>(p.Db + v * bb, sg, b, g, t);
        if (td.child_ptr[v + 1] - td.child_ptr[v] >= 2) {          // chain heads below wait for it
            store_lower_slot<T>(p.ws_U + (int64_t)v * SLOT_ELEMS, sg, lane, g, t);
            __syncwarp();                             // the warp's stores are ordered before lane 0's release
            publish(sy.done, td, v, lane);
            __syncwarp();
        }
        if (c >= 0) {                                 // the first child's Sg_p: exactly symmetric, as read back
            __syncwarp();
            to_smem<T>(s0, sg, g, t);
            __syncwarp();
            from_smem_lower<T>(Sn, s0, g, t);
            __syncwarp();
        }
        v = nxt;
    }
}

__global__ void tree_init(const int32_t *child_ptr, int64_t N, int32_t *pending, int32_t *done,
                          unsigned long long *counters, int32_t *info, int64_t trees)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < N) {
        pending[i] = child_ptr[i + 1] - child_ptr[i];
        done[i] = 0;
    }
    if (i < trees) info[i] = INT_MAX;
    if (i < 2) counters[i] = 0;
}

// log det per tree = sum of its nodes' log det S_v in a fixed order
// (deterministic); info INT_MAX -> -1.  1024 threads, each summing a fixed
// strided subset with four independent partial sums, then a tree in shared
// memory.
constexpr int FIN_THREADS = 1024;

__global__ void __launch_bounds__(FIN_THREADS) tree_finalize(const double *ws_ld, int64_t n, double *logdet,
                                                             int32_t *info)
{
    __shared__ double part[FIN_THREADS];
    const int64_t tr = blockIdx.x;
    const double *x = ws_ld + tr * n;
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
    int64_t v = threadIdx.x;
    for (; v + 3 * FIN_THREADS < n; v += 4 * FIN_THREADS) {
        s0 += x[v];
        s1 += x[v + FIN_THREADS];
        s2 += x[v + 2 * FIN_THREADS];
        s3 += x[v + 3 * FIN_THREADS];
    }
    for (; v < n; v += FIN_THREADS) s0 += x[v];
    part[threadIdx.x] = (s0 + s1) + (s2 + s3);
    __syncthreads();
    for (int w = FIN_THREADS / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        if (logdet) logdet[tr] = part[0];
        if (info[tr] == INT_MAX) info[tr] = -1;
    }
}

__global__ void tree_info_finalize(int32_t *info, int64_t trees)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < trees && info[i] == INT_MAX) info[i] = -1;
}

template <class T> size_t slot_bytes() { return sizeof(T) * w16::SLOT_ELEMS; }

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

template <class T>
cudaError_t run_tree(const selinv_tree_plan_s *pl, int b, const T *diag, const T *edge, T *G_diag, T *G_edge,
                     double *logdet, int32_t *info, void *ws, bool full, cudaStream_t s, const T *z = nullptr,
                     T *eta = nullptr)
{
    const int64_t N = pl->trees * pl->n;
    char *w = static_cast<char *>(ws);
    TreeBufs<T> p;
    p.diag = diag;
    p.edge = edge;
    p.G_diag = G_diag;
    p.G_edge = G_edge;
    p.z = z;
    p.eta = eta;
    const bool draw = z != nullptr;
    p.ws_sinv = reinterpret_cast<T *>(w);
    w += align256(N * sizeof(T) * DRAW_SLOT);
    p.ws_u = reinterpret_cast<T *>(w);
    w += align256(N * slot_bytes<T>());
    p.ws_ld = reinterpret_cast<double *>(w);
    w += align256(N * sizeof(double));
    TreeSync sy;
    sy.pending = reinterpret_cast<int32_t *>(w);
    w += align256(N * sizeof(int32_t));
    sy.done = reinterpret_cast<int32_t *>(w);
    w += align256(N * sizeof(int32_t));
    sy.counters = reinterpret_cast<unsigned long long *>(w);
    p.info = info;
    p.b = b;
    TreeDev td{pl->d_child_ptr, pl->d_child_idx, pl->d_parent, pl->n, pl->spin_limit, pl->hold, pl->d_cpos,
                pl->d_cont};

    const int64_t init_n = std::max<int64_t>(N, pl->trees);
    tree_init<<<(unsigned)ceil_div(init_n, 256), 256, 0, s>>>(pl->d_child_ptr, N, sy.pending, sy.done, sy.counters,
                                                               info, pl->trees);
    const size_t smem = sizeof(T) * tree_smem_elems<T>() * TWARPS;
    const size_t smem_d = sizeof(T) * dist_smem_elems<T>() * TWARPS;
    auto kc = draw ? (full ? tree_collect_draw_kernel<T, true> : tree_collect_draw_kernel<T, false>)
                   : (full ? tree_collect_kernel<T, true> : tree_collect_kernel<T, false>);
    auto kd = full ? tree_distribute_kernel<T, true> : tree_distribute_kernel<T, false>;
    auto kw = full ? tree_draw_kernel<T, true> : tree_draw_kernel<T, false>;
    cudaError_t err = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err == cudaSuccess && !draw)
        err = cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_d);
    if (err != cudaSuccess) return err;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // one resident wave of CTAs per kernel (warps take their work from counters)
    int occ_c = 0, occ_d = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_c, kc, TWARPS * 32, smem) != cudaSuccess || occ_c < 1)
        occ_c = 4;
    if (draw || cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_d, kd, TWARPS * 32, smem_d) != cudaSuccess ||
        occ_d < 1)
        occ_d = 4;
    const int64_t nleaves = pl->collect_off.size() > 1 ? pl->collect_off[1] - pl->collect_off[0] : 0;
    const int64_t ndist = pl->dist_off.empty() ? 0 : pl->dist_off.back();
    const int64_t bc = std::min<int64_t>((int64_t)sms * occ_c, std::max<int64_t>(1, ceil_div(nleaves, TWARPS)));
    kc<<<(unsigned)bc, TWARPS * 32, smem, s>>>(p, td, sy, pl->d_collect_nodes, nleaves);
    if (ndist > 0 && draw) {
        const int64_t wpb = DRAW_THREADS / 32;
        const int64_t bw = std::min<int64_t>((int64_t)sms * 4, ceil_div(pl->nheads, wpb));
        kw<<<(unsigned)bw, DRAW_THREADS, 0, s>>>(p, td, sy, pl->d_heads, pl->nheads);
    } else if (ndist > 0) {
        const int64_t bd = std::min<int64_t>((int64_t)sms * occ_d, ceil_div(pl->nheads, TWARPS));
        kd<<<(unsigned)bd, TWARPS * 32, smem_d, s>>>(p, td, sy, pl->d_heads, pl->nheads);
    }
    tree_finalize<<<(unsigned)pl->trees, FIN_THREADS, 0, s>>>(p.ws_ld, pl->n, logdet, info);
    return cudaGetLastError();
}

size_t tree_bw_workspace(const selinv_tree_plan_s *pl, size_t elem)
{
    const int64_t N = pl->trees * pl->n;
    return 3 * align256((size_t)N * elem * w16::SLOT_ELEMS) + align256((size_t)N * elem * BW_CSLOT) +
           2 * align256((size_t)N * sizeof(int32_t)) + 256;
}

template <class T>
cudaError_t run_tree_backward(const selinv_tree_plan_s *pl, int b, const T *diag, const T *edge, const T *G_diag,
                              const T *G_edge, const T *Gb_diag, const T *Gb_edge, T *Db, T *Eb, int32_t *info,
                              void *ws, bool full, cudaStream_t s)
{
    const int64_t N = pl->trees * pl->n;
    char *w = static_cast<char *>(ws);
    TreeBwdBufs<T> p;
    p.diag = diag;
    p.edge = edge;
    p.G_diag = G_diag;
    p.G_edge = G_edge;
    p.Gb_diag = Gb_diag;
    p.Gb_edge = Gb_edge;
    p.Db = Db;
    p.Eb = Eb;
    p.ws_P = reinterpret_cast<T *>(w);
    w += align256(N * slot_bytes<T>());
    p.ws_U = reinterpret_cast<T *>(w);
    w += align256(N * slot_bytes<T>());
    p.ws_Pd = reinterpret_cast<T *>(w);
    w += align256(N * slot_bytes<T>());
    p.ws_C = reinterpret_cast<T *>(w);
    w += align256(N * sizeof(T) * BW_CSLOT);
    TreeSync sy;
    sy.pending = reinterpret_cast<int32_t *>(w);
    w += align256(N * sizeof(int32_t));
    sy.done = reinterpret_cast<int32_t *>(w);
    w += align256(N * sizeof(int32_t));
    sy.counters = reinterpret_cast<unsigned long long *>(w);
    p.info = info;
    p.b = b;
    TreeDev td{pl->d_child_ptr, pl->d_child_idx, pl->d_parent, pl->n, pl->spin_limit, pl->hold, pl->d_cpos,
                pl->d_cont};

    const int64_t init_n = std::max<int64_t>(N, pl->trees);
    tree_init<<<(unsigned)ceil_div(init_n, 256), 256, 0, s>>>(pl->d_child_ptr, N, sy.pending, sy.done, sy.counters,
                                                               info, pl->trees);
    const size_t smem = sizeof(T) * (3 * w16::SL<T>::ELEMS + 32) * TWARPS;
    auto kc = full ? tree_bw_collect_kernel<T, true> : tree_bw_collect_kernel<T, false>;
    auto kd = full ? tree_bw_distribute_kernel<T, true> : tree_bw_distribute_kernel<T, false>;
    cudaError_t err = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err == cudaSuccess) err = cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int occ_c = 0, occ_d = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_c, kc, TWARPS * 32, smem) != cudaSuccess || occ_c < 1)
        occ_c = 2;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_d, kd, TWARPS * 32, smem) != cudaSuccess || occ_d < 1)
        occ_d = 2;
    const int64_t nleaves = pl->collect_off.size() > 1 ? pl->collect_off[1] - pl->collect_off[0] : 0;
    const int64_t ndist = pl->dist_off.empty() ? 0 : pl->dist_off.back();
    const int64_t bc = std::min<int64_t>((int64_t)sms * occ_c, std::max<int64_t>(1, ceil_div(nleaves, TWARPS)));
    kc<<<(unsigned)bc, TWARPS * 32, smem, s>>>(p, td, sy, pl->d_collect_nodes, nleaves);
    if (ndist > 0) {
        const int64_t bd = std::min<int64_t>((int64_t)sms * occ_d, ceil_div(pl->nheads, TWARPS));
        kd<<<(unsigned)bd, TWARPS * 32, smem, s>>>(p, td, sy, pl->d_heads, pl->nheads);
    }
    tree_info_finalize<<<(unsigned)ceil_div(pl->trees, 256), 256, 0, s>>>(info, pl->trees);
    return cudaGetLastError();
}

bool is_aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

size_t tree_workspace(const selinv_tree_plan_s *pl, size_t elem)
{
    const int64_t N = pl->trees * pl->n;
    return align256((size_t)N * elem * DRAW_SLOT) + align256((size_t)N * elem * w16::SLOT_ELEMS) +
           align256((size_t)N * sizeof(double)) +
           2 * align256((size_t)N * sizeof(int32_t)) + 256;
}

}  // namespace selinv

using namespace selinv;

extern "C" {

static selinv_status tree_plan_impl(const int32_t *parent, int64_t trees, int64_t n, selinv_tree_plan_t **out)
{
    if (!out) return SELINV_ERR_INVALID_ARG;
    *out = nullptr;
    if (!parent || trees < 1 || n < 1 || trees * n >= (int64_t)INT32_MAX) return SELINV_ERR_INVALID_ARG;
    const int64_t N = trees * n;
    std::vector<int32_t> gparent(N), cnt(N + 1, 0), height(N, 0), depth(N, 0), order;
    order.reserve(N);
    for (int64_t tr = 0; tr < trees; ++tr) {
        int64_t root = -1;
        for (int64_t v = 0; v < n; ++v) {
            const int32_t p = parent[tr * n + v];
            if (p == -1) {
                if (root >= 0) return SELINV_ERR_BAD_TREE;
                root = v;
                gparent[tr * n + v] = -1;
            } else {
                if (p < 0 || p >= n || p == v) return SELINV_ERR_BAD_TREE;
                gparent[tr * n + v] = (int32_t)(tr * n + p);
                cnt[tr * n + p + 1]++;
            }
        }
        if (root < 0) return SELINV_ERR_BAD_TREE;
    }
    for (int64_t v = 0; v < N; ++v) cnt[v + 1] += cnt[v];
    std::vector<int32_t> child(std::max<int64_t>(cnt[N], 1)), fill(cnt.begin(), cnt.end() - 1);
    for (int64_t v = 0; v < N; ++v)
        if (gparent[v] >= 0) child[fill[gparent[v]]++] = (int32_t)v;   // ascending per parent
    // breadth-first order per tree from its root; a cycle leaves nodes unreached
    for (int64_t tr = 0; tr < trees; ++tr) {
        const size_t start = order.size();
        for (int64_t v = 0; v < n; ++v)
            if (gparent[tr * n + v] < 0) order.push_back((int32_t)(tr * n + v));
        for (size_t h = start; h < order.size(); ++h) {
            const int32_t v = order[h];
            for (int32_t c = cnt[v]; c < cnt[v + 1]; ++c) {
                depth[child[c]] = depth[v] + 1;
                order.push_back(child[c]);
            }
        }
        if ((int64_t)(order.size() - start) != n) return SELINV_ERR_BAD_TREE;
    }
    for (int64_t i = N - 1; i >= 0; --i) {
        const int32_t v = order[i];
        if (gparent[v] >= 0) height[gparent[v]] = std::max(height[gparent[v]], height[v] + 1);
    }
    int32_t H = 0, Dm = 0;
    for (int64_t v = 0; v < N; ++v) {
        H = std::max(H, height[v]);
        Dm = std::max(Dm, depth[v]);
    }
    // held by a unique_ptr until handed out, so a host allocation failure
    // below (caught at the C ABI) releases it and its device tables
    std::unique_ptr<selinv_tree_plan_s, void (*)(selinv_tree_plan_s *)> hold(new (std::nothrow)
                                                                                 selinv_tree_plan_s(),
                                                                             selinv_tree_plan_free);
    if (!hold) return SELINV_ERR_HOST_MEMORY;
    selinv_tree_plan_s *pl = hold.get();
    pl->trees = trees;
    pl->n = n;
    cudaGetDevice(&pl->device);
    // counting sort by level keeps ascending ids within a level
    std::vector<int32_t> cnodes(N), dnodes;
    pl->collect_off.assign(H + 2, 0);
    for (int64_t v = 0; v < N; ++v) pl->collect_off[height[v] + 1]++;
    for (int32_t h = 0; h <= H; ++h) pl->collect_off[h + 1] += pl->collect_off[h];
    {
        std::vector<int64_t> pos(pl->collect_off.begin(), pl->collect_off.end() - 1);
        for (int64_t v = 0; v < N; ++v) cnodes[pos[height[v]]++] = (int32_t)v;
    }
    pl->dist_off.assign(Dm + 1, 0);     // depths 1..Dm
    for (int64_t v = 0; v < N; ++v)
        if (depth[v] >= 1) pl->dist_off[depth[v]]++;
    for (int32_t d = 1; d <= Dm; ++d) pl->dist_off[d] += pl->dist_off[d - 1];
    dnodes.assign(std::max<int64_t>(pl->dist_off[Dm], 1), 0);
    {
        std::vector<int64_t> pos(Dm + 1, 0);
        for (int32_t d = 1; d <= Dm; ++d) pos[d] = pl->dist_off[d - 1];
        for (int64_t v = 0; v < N; ++v)
            if (depth[v] >= 1) dnodes[pos[depth[v]]++] = (int32_t)v;
    }
    bool ok = true;
    auto up = [&](int32_t **dst, const std::vector<int32_t> &src) {
        if (!ok) return;
        ok = cudaMalloc(dst, src.size() * sizeof(int32_t)) == cudaSuccess &&
             cudaMemcpy(*dst, src.data(), src.size() * sizeof(int32_t), cudaMemcpyHostToDevice) == cudaSuccess;
    };
    up(&pl->d_collect_nodes, cnodes);
    up(&pl->d_dist_nodes, dnodes);
    up(&pl->d_child_ptr, cnt);
    up(&pl->d_child_idx, child);
    {
        std::vector<int32_t> cpos(N, -1), cont(N, -1), heads;
        for (int64_t v = 0; v < N; ++v)
            for (int32_t c = cnt[v]; c < cnt[v + 1]; ++c) cpos[child[c]] = c;
        for (int64_t v = 0; v < N; ++v)
            if (gparent[v] >= 0 && cnt[v + 1] > cnt[v]) cont[v] = child[cnt[v]];
        heads.reserve(dnodes.size());
        for (int64_t i = 0; i < pl->dist_off[Dm]; ++i) {   // depth order, ascending ids within a depth
            const int32_t v = dnodes[i];
            if (cont[gparent[v]] != v) heads.push_back(v);
        }
        pl->nheads = (int64_t)heads.size();
        if (heads.empty()) heads.push_back(0);
        up(&pl->d_cpos, cpos);
        up(&pl->d_cont, cont);
        up(&pl->d_heads, heads);
    }
    up(&pl->d_parent, gparent);
    if (!ok) return SELINV_ERR_CUDA;
    *out = hold.release();
    return SELINV_OK;
}

selinv_status selinv_tree_plan(const int32_t *parent, int64_t trees, int64_t n, selinv_tree_plan_t **out)
{
    // host tables are C++ containers: no exception may leave the C ABI
    try {
        return tree_plan_impl(parent, trees, n, out);
    } catch (const std::bad_alloc &) {
        if (out) *out = nullptr;
        return SELINV_ERR_HOST_MEMORY;
    } catch (...) {
        if (out) *out = nullptr;
        return SELINV_ERR_INVALID_ARG;
    }
}

void selinv_tree_plan_free(selinv_tree_plan_t *pl)
{
    if (!pl) return;
    cudaFree(pl->d_collect_nodes);
    cudaFree(pl->d_dist_nodes);
    cudaFree(pl->d_child_ptr);
    cudaFree(pl->d_child_idx);
    cudaFree(pl->d_cpos);
    cudaFree(pl->d_cont);
    cudaFree(pl->d_heads);
    cudaFree(pl->d_parent);
    delete pl;
}

selinv_status selinv_tree_plan_set_wait(selinv_tree_plan_t *pl, int32_t spin_limit, int64_t withhold)
{
    if (!pl || withhold < -1 || withhold >= pl->trees * pl->n) return SELINV_ERR_INVALID_ARG;
    pl->spin_limit = spin_limit >= 1 ? spin_limit : selinv::SPIN_LIMIT;
    pl->hold = withhold;
    return SELINV_OK;
}

selinv_status selinv_tree_plan_levels(const selinv_tree_plan_t *pl, int32_t *collect, int32_t *distribute)
{
    if (!pl || !collect || !distribute) return SELINV_ERR_INVALID_ARG;
    *collect = (int32_t)pl->collect_off.size() - 1;
    *distribute = (int32_t)pl->dist_off.size();
    return SELINV_OK;
}

size_t selinv_tree_workspace_size(const selinv_tree_plan_t *pl, selinv_dtype dtype, int32_t b)
{
    if (!pl || (dtype != SELINV_F64 && dtype != SELINV_F32) || b < 1 || b > 16) return 0;
    return tree_workspace(pl, dtype == SELINV_F64 ? 8 : 4);
}

selinv_status selinv_tree(const selinv_tree_plan_t *pl, selinv_dtype dtype, int32_t b, const void *diag,
                          const void *edge, void *G_diag, void *G_edge, double *logdet, int32_t *info,
                          void *workspace, size_t workspace_bytes, uint32_t flags, void *stream)
{
    if (!pl || (dtype != SELINV_F64 && dtype != SELINV_F32) || b < 1) return SELINV_ERR_INVALID_ARG;
    if (flags & ~(uint32_t)(SELINV_WANT_LOGDET | SELINV_CHECK)) return SELINV_ERR_INVALID_ARG;
    if ((flags & SELINV_WANT_LOGDET) && logdet == nullptr) return SELINV_ERR_INVALID_ARG;
    if (b > 16) return SELINV_ERR_UNSUPPORTED;
    if (!diag || !edge || !G_diag || !G_edge || !info) return SELINV_ERR_INVALID_ARG;
    const size_t es = dtype == SELINV_F64 ? 8 : 4;
    if (!is_aligned(diag, es) || !is_aligned(edge, es) || !is_aligned(G_diag, es) || !is_aligned(G_edge, es) ||
        !is_aligned(logdet, 8) || !is_aligned(info, 4) || !is_aligned(workspace, 256))
        return SELINV_ERR_INVALID_ARG;
    const size_t need = tree_workspace(pl, es);
    if (!workspace || workspace_bytes < need) return SELINV_ERR_WORKSPACE;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != pl->device) return SELINV_ERR_INVALID_ARG;
    const bool full = b == 16 && is_aligned(diag, 16) && is_aligned(edge, 16) && is_aligned(G_diag, 16) &&
                      is_aligned(G_edge, 16);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t err;
    if (dtype == SELINV_F64)
        err = run_tree<double>(pl, b, static_cast<const double *>(diag), static_cast<const double *>(edge),
                               static_cast<double *>(G_diag), static_cast<double *>(G_edge), logdet, info,
                               workspace, full, s);
    else
        err = run_tree<float>(pl, b, static_cast<const float *>(diag), static_cast<const float *>(edge),
                              static_cast<float *>(G_diag), static_cast<float *>(G_edge), logdet, info,
                              workspace, full, s);
    if (err == cudaSuccess && (flags & SELINV_CHECK)) {       // D_v (lower triangles) and non-root edge[v] finite
        if (dtype == SELINV_F64) {
            err = check_finite_launch<double>(static_cast<const double *>(diag), pl->trees, pl->n, b, 0, nullptr,
                                              info, s);
            if (err == cudaSuccess)
                err = check_finite_launch<double>(static_cast<const double *>(edge), pl->trees, pl->n, b, 1,
                                                  pl->d_parent, info, s);
        } else {
            err = check_finite_launch<float>(static_cast<const float *>(diag), pl->trees, pl->n, b, 0, nullptr,
                                             info, s);
            if (err == cudaSuccess)
                err = check_finite_launch<float>(static_cast<const float *>(edge), pl->trees, pl->n, b, 1,
                                                 pl->d_parent, info, s);
        }
        if (err == cudaSuccess) err = check_finalize_launch(info, pl->trees, pl->n, s);
    }
    return err == cudaSuccess ? SELINV_OK : SELINV_ERR_CUDA;
}

selinv_status selinv_tree_sample(const selinv_tree_plan_t *pl, selinv_dtype dtype, int32_t b, const void *diag,
                                 const void *edge, const void *z, void *eta, double *logdet, int32_t *info,
                                 void *workspace, size_t workspace_bytes, void *stream)
{
    if (!pl || (dtype != SELINV_F64 && dtype != SELINV_F32) || b < 1) return SELINV_ERR_INVALID_ARG;
    if (b > 16) return SELINV_ERR_UNSUPPORTED;
    if (!diag || !edge || !z || !eta || !info) return SELINV_ERR_INVALID_ARG;
    const size_t es = dtype == SELINV_F64 ? 8 : 4;
    if (!is_aligned(diag, es) || !is_aligned(edge, es) || !is_aligned(z, es) || !is_aligned(eta, es) ||
        !is_aligned(logdet, 8) || !is_aligned(info, 4) || !is_aligned(workspace, 256))
        return SELINV_ERR_INVALID_ARG;
    const size_t need = tree_workspace(pl, es);
    if (!workspace || workspace_bytes < need) return SELINV_ERR_WORKSPACE;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != pl->device) return SELINV_ERR_INVALID_ARG;
    const bool full = b == 16 && is_aligned(diag, 16) && is_aligned(edge, 16);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t err;
    if (dtype == SELINV_F64)
        err = run_tree<double>(pl, b, static_cast<const double *>(diag), static_cast<const double *>(edge), nullptr,
                               nullptr, logdet, info, workspace, full, s, static_cast<const double *>(z),
                               static_cast<double *>(eta));
    else
        err = run_tree<float>(pl, b, static_cast<const float *>(diag), static_cast<const float *>(edge), nullptr,
                              nullptr, logdet, info, workspace, full, s, static_cast<const float *>(z),
                              static_cast<float *>(eta));
    return err == cudaSuccess ? SELINV_OK : SELINV_ERR_CUDA;
}

size_t selinv_tree_backward_workspace_size(const selinv_tree_plan_t *pl, selinv_dtype dtype, int32_t b)
{
    if (!pl || (dtype != SELINV_F64 && dtype != SELINV_F32) || b < 1 || b > 16) return 0;
    return tree_bw_workspace(pl, dtype == SELINV_F64 ? 8 : 4);
}

selinv_status selinv_tree_backward(const selinv_tree_plan_t *pl, selinv_dtype dtype, int32_t b, const void *diag,
                                   const void *edge, const void *G_diag, const void *G_edge, const void *Gb_diag,
                                   const void *Gb_edge, void *Db, void *Eb, int32_t *info, void *workspace,
                                   size_t workspace_bytes, void *stream)
{
    if (!pl || (dtype != SELINV_F64 && dtype != SELINV_F32) || b < 1) return SELINV_ERR_INVALID_ARG;
    if (b > 16) return SELINV_ERR_UNSUPPORTED;
    if (!diag || !edge || !G_diag || !G_edge || !Db || !Eb || !info) return SELINV_ERR_INVALID_ARG;
    const size_t es = dtype == SELINV_F64 ? 8 : 4;
    const void *ptrs[8] = {diag, edge, G_diag, G_edge, Gb_diag, Gb_edge, Db, Eb};
    bool al16 = b == 16;
    for (const void *q : ptrs) {
        if (!is_aligned(q, es)) return SELINV_ERR_INVALID_ARG;
        al16 = al16 && is_aligned(q, 16);
    }
    if (!is_aligned(info, 4) || !is_aligned(workspace, 256)) return SELINV_ERR_INVALID_ARG;
    const size_t need = tree_bw_workspace(pl, es);
    if (!workspace || workspace_bytes < need) return SELINV_ERR_WORKSPACE;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != pl->device) return SELINV_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t err;
    if (dtype == SELINV_F64)
        err = run_tree_backward<double>(pl, b, static_cast<const double *>(diag), static_cast<const double *>(edge),
                                        static_cast<const double *>(G_diag), static_cast<const double *>(G_edge),
                                        static_cast<const double *>(Gb_diag), static_cast<const double *>(Gb_edge),
                                        static_cast<double *>(Db), static_cast<double *>(Eb), info, workspace,
                                        al16, s);
    else
        err = run_tree_backward<float>(pl, b, static_cast<const float *>(diag), static_cast<const float *>(edge),
                                       static_cast<const float *>(G_diag), static_cast<const float *>(G_edge),
                                       static_cast<const float *>(Gb_diag), static_cast<const float *>(Gb_edge),
                                       static_cast<float *>(Db), static_cast<float *>(Eb), info, workspace,
                                       al16, s);
    return err == cudaSuccess ? SELINV_OK : SELINV_ERR_CUDA;
}

}  // extern "C"
