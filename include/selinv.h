/*
 * libselinv -- batched block selected inverse of sparse SPD matrices whose
 * block graph is a chain (block tridiagonal) or a tree, on NVIDIA B200
 * (sm_100a).
 *
 * The problem (gabp-sparse-inv 0.3.2, PyPI page, "Implemented and tested
 * kernels" -> Chain and Tree; "Quickstart"): for an SPD matrix A made of
 * b x b blocks, return only the blocks of A^-1 on A's own pattern -- the
 * diagonal blocks G_vv = (A^-1)_vv and one off-diagonal block per edge --
 * never the dense inverse.  The same block LDL^T factorisation also gives
 * log det A and the solve x = A^-1 r ("junction_solve", "junction_logdet";
 * sparsax, PyPI page, "Factor once, do everything").
 *
 * Method: a collect sweep of Schur complements
 *     S_0 = D_0,  S_{i+1} = D_{i+1} - B_i S_i^-1 B_i^T
 * (tree: S_v = D_v - sum_{c child of v} E_c S_c^-1 E_c^T, leaves to root),
 * log det A = sum_v log det S_v, then the distribute sweep (the Takahashi
 * back-recursion)
 *     G_{L-1,L-1} = S_{L-1}^-1,
 *     G_{i+1,i} = -G_{i+1,i+1} B_i S_i^-1,  G_ii = S_i^-1 - S_i^-1 B_i^T G_{i+1,i}
 * (tree: G_edge[v] = -G_{p(v)} E_v S_v^-1, G_vv = S_v^-1 - S_v^-1 E_v^T G_edge[v],
 * root to leaves).
 *
 * Conventions shared by every entry point
 *   - All block arrays are dense, contiguous, row-major b x b blocks in
 *     DEVICE memory, in the precision named by `dtype` (float64 or float32).
 *     Leading batch dimensions are flattened into `batch` by the caller.
 *   - Only the lower triangle of each diagonal block D is read; the upper
 *     triangle is taken as its mirror.  Every G_vv is written in full and
 *     exactly symmetric.
 *   - log-determinants are always written as float64 (natural log).
 *   - info[e] (int32, device) is written for every batch element: -1 when
 *     all Schur complements were positive definite, else the index of a
 *     block (chain) or node (tree) whose pivot was not > 0 (or NaN): the
 *     first one in elimination order -- 0 -> L-1 for chains, except that
 *     chains with 16 < b <= 32 and no right-hand side are eliminated from
 *     both ends toward the middle block and report the smaller of the two
 *     halves' first failures.  The outputs of such an element are
 *     unspecified.  Kernels never trap.  A tree distribute step whose wait
 *     for its parent timed out (not expected for a valid plan) reports -2.
 *     With SELINV_CHECK, an element holding a non-finite input entry
 *     reports -3 - k instead, k the first block (chain) or node (tree)
 *     holding one.
 *   - The caller owns every buffer, including the workspace, whose size the
 *     *_workspace_size functions give (0 means none is needed; the pointer
 *     may then be NULL).  Workspace and outputs must not overlap inputs.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and returns without synchronising.  Argument errors are
 *     reported synchronously, before anything is launched.
 *   - Supported block sizes: 1 <= b <= selinv_max_block().
 *   - Device pointers must be aligned to their element size; 16-byte
 *     alignment of every array enables the vectorised paths.
 */
#ifndef SELINV_H
#define SELINV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SELINV_OK = 0,
    SELINV_ERR_INVALID_ARG = 1,   /* bad size, NULL or misaligned pointer, bad dtype */
    SELINV_ERR_NOT_SPD = 2,       /* returned by bindings that read info[] back */
    SELINV_ERR_BAD_TREE = 3,      /* parent array is not one rooted tree per slot */
    SELINV_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    SELINV_ERR_WORKSPACE = 5,     /* workspace smaller than *_workspace_size */
    SELINV_ERR_UNSUPPORTED = 6,   /* block size beyond selinv_max_block() */
    SELINV_ERR_HOST_MEMORY = 7,   /* a plan's host-side tables could not be allocated */
    SELINV_ERR_TIMEOUT = 8        /* returned by bindings that read info[] back: a bounded
                                     dependency wait of a tree sweep gave up (info = -2) */
} selinv_status;

typedef enum { SELINV_F64 = 0, SELINV_F32 = 1 } selinv_dtype;

/* Human-readable name of a status code (static string). */
const char *selinv_status_string(selinv_status s);

/* Library version as major*10000 + minor*100 + patch. */
int32_t selinv_version(void);

/* Largest supported block size b. */
int32_t selinv_max_block(void);

/*
 * Workspace bytes selinv_chain / chain_solve need for these sizes and
 * outputs (want_g: G_diag/G_lower requested; want_x: a solve requested).
 */
size_t selinv_chain_workspace_size(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b,
                                   int32_t want_g, int32_t want_x);

/*
 * How many segments selinv_chain cuts each chain into for these sizes on the
 * current device (0: it does not).  Only 16 < b <= 32 with G requested and no
 * right-hand side is cut, and only when the batch is too small to fill the
 * GPU (fewer than three chains per SM's worth of segments) and L >= 96.  The
 * P - 1 separator blocks are eliminated last, so the blocks reach the same
 * factorisation in another order (gabp-sparse-inv, "Implemented and tested
 * kernels" -> Chain and Tree: a chain may be rooted at any node).  The
 * workspace size depends on the answer, hence on the current device's SM
 * count.  With segments, info reports the smallest block index at which any
 * segment (in its own elimination order) or the separators' chain met a
 * pivot that is not > 0.
 */
int32_t selinv_chain_segments(int64_t batch, int64_t L, int32_t b, int32_t want_g, int32_t want_x);

/*
 * Flags of selinv_chain and selinv_tree.  The outputs a call computes follow
 * from which pointers are non-NULL; SELINV_WANT_LOGDET (logdet) and
 * SELINV_WANT_SOLVE (rhs and x; chains only) make the call reject the
 * request with SELINV_ERR_INVALID_ARG when those pointers are missing.
 * SELINV_CHECK (gabp-sparse-inv, "Quickstart": check=True) adds an on-device
 * pass, after the selected inverse on the same stream, that checks every
 * entry the call reads -- the lower triangle of each diagonal block, every
 * entry of each off-diagonal block (trees: non-root edge slots), the
 * right-hand side -- and writes info = -3 - k for an element whose block k
 * holds a non-finite value; nothing traps.  Unknown bits are rejected.
 */
enum { SELINV_WANT_LOGDET = 1, SELINV_WANT_SOLVE = 2, SELINV_CHECK = 4 };

/*
 * Selected inverse, log-determinant and (optionally) solve of `batch`
 * independent block-tridiagonal SPD chains of L blocks of size b.
 * (gabp-sparse-inv, "Implemented and tested kernels" -> Chain, and the
 * "Quickstart" call selected_inverse_chain(diag, lower).)
 *
 *   diag    [batch, L, b, b]    D_i = A_{i,i} (lower triangle read)
 *   lower   [batch, L-1, b, b]  B_i = A_{i+1,i}; may be NULL when L == 1
 *   G_diag  [batch, L, b, b]    out: (A^-1)_{i,i}          } both NULL, or
 *   G_lower [batch, L-1, b, b]  out: (A^-1)_{i+1,i}        } both given
 *   logdet  [batch] float64     out: log det A; may be NULL
 *   rhs     [batch, L, b]       right-hand side r; NULL for no solve
 *   x       [batch, L, b]       out: A^-1 r; given iff rhs is given
 *   info    [batch] int32       out: see the conventions above (required)
 *   flags   SELINV_* bits below, or 0
 * Returns SELINV_OK once the work is enqueued.
 */
selinv_status selinv_chain(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b,
                           const void *diag, const void *lower,
                           void *G_diag, void *G_lower, double *logdet,
                           const void *rhs, void *x, int32_t *info,
                           void *workspace, size_t workspace_bytes, uint32_t flags, void *stream);

/*
 * Solve only: x = A^-1 r for each chain, from the same block LDL^T factor,
 * without forming any block of A^-1 (sparsax, "Features": solve, and
 * gabp-sparse-inv "junction_solve").  Arguments as in selinv_chain; logdet
 * may be NULL; rhs, x and info are required.
 */
selinv_status chain_solve(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b,
                          const void *diag, const void *lower, const void *rhs, void *x,
                          double *logdet, int32_t *info,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * Solve with several right-hand sides from the same factorisation: X = A^-1 R
 * for each chain, R and X [batch, L, b, nrhs] (row-major: block i of a chain
 * is b x nrhs).  (sparsax, "Features": multiple right-hand sides, b may be
 * (n,) or (n, n_rhs); "Factor once, do everything".)  b <= 16 (larger b:
 * SELINV_ERR_UNSUPPORTED); nrhs >= 1.  Up to 16 right-hand sides share one
 * pass over the factorisation; larger nrhs is taken 16 columns per pass.
 * logdet may be NULL; info as in selinv_chain.  Workspace:
 * selinv_chain_workspace_size(dtype, batch, L, b, 0, 1) bytes.
 */
selinv_status chain_solve_multi(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b, int32_t nrhs,
                                const void *diag, const void *lower, const void *rhs, void *x,
                                double *logdet, int32_t *info,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * Gaussian draw from the same factorisation (sparsax, "Factor once, do
 * everything": sample_gaussian returns eta = A^-1 b + P^T L^-T z with
 * A = P^T L L^T P its Cholesky factorisation; gabp-sparse-inv, "Gaussian
 * sampling": x ~ N(0, A^-1) reusing the factor).  A chain is factorised in
 * its own block order, so P = I and L is its block lower-bidiagonal Cholesky
 * factor (diagonal blocks R_i with S_i = R_i R_i^T, R_i lower; sub-diagonal
 * blocks B_i R_i^-T).  For each chain:
 *
 *   eta = A^-1 rhs + L^-T z        (eta = L^-T z when rhs is NULL)
 *
 * so that eta ~ N(A^-1 rhs, A^-1) when z ~ N(0, I).  The standard normals z
 * are the caller's (the library draws no random numbers).
 *
 *   diag, lower   as in selinv_chain; b <= 16, or 16 < b <= 128 in float64
 *                 (float32 with b > 16: SELINV_ERR_UNSUPPORTED)
 *   rhs     [batch, L, b]   mean's right-hand side, or NULL
 *   z       [batch, L, b]   required
 *   eta     [batch, L, b]   out, required
 *   logdet  [batch] float64 out: log det A; may be NULL
 *   info    [batch] int32   out: -1, or the first block whose Schur complement
 *                           is not positive definite (eta then unspecified)
 * Workspace: selinv_chain_workspace_size(dtype, batch, L, b, 0, 1) bytes.
 */
selinv_status selinv_chain_sample(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b,
                                  const void *diag, const void *lower, const void *rhs,
                                  const void *z, void *eta, double *logdet, int32_t *info,
                                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * Selected inverse of block lower-bidiagonal matrices with general
 * (non-symmetric) blocks, b <= 16: gabp-sparse-inv 0.3.2, "Implemented and
 * tested kernels" -> Non-symmetric chain:
 *   G_ii = M_ii^-1,   G_{i+1,i} = -M_{i+1,i+1}^-1 M_{i+1,i} M_ii^-1,
 * the blocks of M^-1 on M's pattern.
 *   diag  [batch, L, b, b]    M_ii, read in full (no symmetry assumed)
 *   lower [batch, L-1, b, b]  M_{i+1,i} (NULL when L = 1)
 *   G_diag, G_lower           outputs, same shapes
 *   info [batch]              -1, or the first block i whose M_ii is singular
 *                             (a zero or non-finite pivot under partial
 *                             pivoting; that chain's outputs are then
 *                             unspecified)
 * No workspace.  b > 16 returns SELINV_ERR_UNSUPPORTED.
 */
selinv_status selinv_bidiag(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b, const void *diag,
                            const void *lower, void *G_diag, void *G_lower, int32_t *info, void *stream);

/*
 * Cotangents of selinv_bidiag (b <= 16): the pages' hand-written analytic
 * backward of selinv_bidiag, one batched block op.  From its outputs G_diag,
 * G_lower and their cotangents Gb_diag, Gb_lower (NULL = zero) writes the
 * cotangents of M:
 *   Mb_diag [batch, L, b, b]    Mb_ii = -G_ii^T Gb_ii G_ii^T
 *                                     - G_{i+1,i}^T Gb_{i+1,i} G_ii^T
 *                                     - G_ii^T Gb_{i,i-1} G_{i,i-1}^T
 *   Mb_lower [batch, L-1, b, b] Mb_{i+1,i} = -G_{i+1,i+1}^T Gb_{i+1,i} G_ii^T
 * (Mb = -G^T Gbar G^T on M's pattern, dG = -G dM G; M^-1 block lower
 * triangular leaves only these terms).  M itself is not needed; G_lower,
 * Gb_lower and Mb_lower may be NULL when L = 1.  No workspace.
 */
selinv_status selinv_bidiag_backward(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b,
                                     const void *G_diag, const void *G_lower, const void *Gb_diag,
                                     const void *Gb_lower, void *Mb_diag, void *Mb_lower, void *stream);

/*
 * Cotangents of the chain selected inverse (b <= 16): given the cotangents
 * Gb_diag [batch, L, b, b] and Gb_lower [batch, L-1, b, b] of a loss with
 * respect to selinv_chain's outputs G_diag and G_lower, writes the
 * cotangents with respect to its inputs:
 *   Db [batch, L, b, b]    of diag; lower-triangular, because selinv_chain
 *                          reads only the lower triangle of each D_i (an entry
 *                          below the diagonal stands for both mirror places,
 *                          so it receives Ab[r][c] + Ab[c][r]; upper entries
 *                          receive 0);
 *   Bb [batch, L-1, b, b]  of lower (B_i sits at (i+1, i) and, transposed, at
 *                          (i, i+1)),
 * where Ab = -A^-1 Gbar A^-1 is the cotangent of A as a whole matrix (dG =
 * -G dA G).  (gabp-sparse-inv 0.3.2, "Differentiable selected inverse":
 * gradients over the selected blocks flow back to the input blocks through
 * an analytic two-pass backward.)  The two passes are the reverse-mode forms
 * of the forward's collect and distribute sweeps; nothing dense is formed.
 *   diag, lower, G_diag, G_lower  the forward's inputs and outputs (device);
 *                                 lower, G_lower, Gb_lower and Bb may be NULL
 *                                 when L = 1
 *   Gb_diag, Gb_lower   NULL stands for a zero cotangent
 *   info [batch]    -1, or the first block whose Schur complement is not
 *                   positive definite (the outputs are then unspecified)
 * Workspace: selinv_chain_backward_workspace_size(dtype, batch, L, b) bytes
 * (two 16 x 16 tiles per block).  b > 16 returns SELINV_ERR_UNSUPPORTED.
 */
size_t selinv_chain_backward_workspace_size(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b);

selinv_status selinv_chain_backward(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b,
                                    const void *diag, const void *lower, const void *G_diag,
                                    const void *G_lower, const void *Gb_diag, const void *Gb_lower,
                                    void *Db, void *Bb, int32_t *info, void *workspace,
                                    size_t workspace_bytes, void *stream);

/*
 * Same computation as selinv_chain for b <= 16, with no workspace argument
 * and no allocation of any kind.  The pages have no counterpart: this entry
 * point exists for callers that cannot allocate device memory -- code running
 * inside another framework's execution hook (an inference-engine plugin's
 * enqueue, a compiler runtime's custom call, a fixed-budget real-time loop),
 * where the framework owns all device memory and a cudaMalloc is forbidden,
 * fails, or would synchronise the device.  Such callers pass inputs and
 * outputs only (arguments and layouts as in selinv_chain).
 *
 * The scratch is a library-owned device array of SELINV_CHAIN_NOALLOC_MAX_BYTES
 * (16 MiB) that every GPU loading the library keeps until the process
 * exits.  Requests needing more -- batch * (L-1) * 192 * sizeof(element) bytes
 * when G or x is asked for -- return SELINV_ERR_WORKSPACE before anything is
 * launched.  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  All calls share the one array and it keeps the
 * last call's contents; nothing needs clearing, because every slot a call
 * reads is written earlier in the same call.  Calls whose executions overlap
 * on the GPU (different streams, or different host threads) race on it.
 */
#define SELINV_CHAIN_NOALLOC_MAX_BYTES ((size_t)16 << 20)

selinv_status selinv_chain_noalloc(selinv_dtype dtype, int64_t batch, int64_t L, int32_t b,
                                   const void *diag, const void *lower,
                                   void *G_diag, void *G_lower, double *logdet,
                                   const void *rhs, void *x, int32_t *info, void *stream);

/*
 * General block-sparse SPD matrices (b <= 16): gabp-sparse-inv 0.3.2,
 * "General sparse selected inverse (junction tree)".  The block pattern is
 * completed to its chordal fill S by an elimination order, then the
 * multi-neighbour Takahashi recurrence returns A^-1 on S.
 *
 * selinv_junction_plan (host work, cached per pattern): n nodes, m lower
 * blocks (ei[k], ej[k]) with 0 <= ej[k] < ei[k] < n, no repeats (HOST int32
 * arrays); order = a permutation of 0..n-1 (HOST) or NULL for greedy minimum
 * degree on the elimination graph, ties to the smaller node index.  Builds
 * the fill, the elimination tree, its levels and the index lists, and copies
 * them to the current device.  Bad input returns SELINV_ERR_INVALID_ARG.
 * selinv_junction_plan_info: nnz_S (blocks of S below the diagonal) and the
 * number of levels of each sweep.  selinv_junction_plan_pattern: S as
 * (S_i[k], S_j[k]), S_i > S_j, sorted by S_j then S_i, and the elimination
 * order (HOST outputs of nnz_S and n entries; any may be NULL).
 *
 * selinv_junction: for `batch` matrices on the plan's pattern:
 *   diag     [batch, n, b, b]     D_v (lower triangle read)
 *   edge_val [batch, m, b, b]     A_{ei[k], ej[k]}
 *   G_diag   [batch, n, b, b]     (A^-1)_vv, exactly symmetric
 *   G_lower  [batch, nnz_S, b, b] (A^-1)_{S_i[k], S_j[k]}
 *   logdet [batch] (may be NULL), info [batch]: -1, or a node whose Schur
 *   complement is not positive definite (outputs then unspecified)
 * Workspace: selinv_junction_workspace_size(plan, dtype, b, batch) bytes.
 * Each level of the collect is three launches (target blocks, inverses,
 * W products), each level of the distribute two (clique columns, diagonals).
 * The first call with a given set of arguments (pointers, batch, b, dtype)
 * records that launch sequence as a CUDA graph held by the plan (up to four,
 * least recently used replaced, on a stream the plan creates for recording)
 * and every call replays it on `stream`, so a call whose buffers hold new
 * values replays the same graph; a call made while `stream` is itself being
 * captured launches the kernels directly into that capture.  The plan's
 * lock serialises the host side of concurrent calls on one plan.
 */
typedef struct selinv_junction_plan_s selinv_junction_plan_t;

selinv_status selinv_junction_plan(int64_t n, int64_t m, const int32_t *ei, const int32_t *ej,
                                   const int32_t *order, selinv_junction_plan_t **out);
void selinv_junction_plan_free(selinv_junction_plan_t *plan);
selinv_status selinv_junction_plan_info(const selinv_junction_plan_t *plan, int64_t *nnz_S,
                                        int32_t *collect_levels, int32_t *distribute_levels);
selinv_status selinv_junction_plan_pattern(const selinv_junction_plan_t *plan, int32_t *S_i, int32_t *S_j,
                                           int32_t *order);
/* The plan's symbolic phase alone, on the host (no device touched): the same
 * validation, order and filled pattern as selinv_junction_plan.  Writes
 * *nnz_S, the first min(nnz_S, capacity) pairs of S to S_i / S_j and the
 * order to order_out [n] (any of them may be NULL). */
selinv_status selinv_junction_symbolic(int64_t n, int64_t m, const int32_t *ei, const int32_t *ej,
                                       const int32_t *order, int64_t *nnz_S, int32_t *S_i, int32_t *S_j,
                                       int64_t capacity, int32_t *order_out);

/* Kernel launches one selinv_junction call makes with this plan (-1 for NULL). */
int64_t selinv_junction_plan_launches(const selinv_junction_plan_t *plan);
size_t selinv_junction_workspace_size(const selinv_junction_plan_t *plan, selinv_dtype dtype, int32_t b,
                                      int64_t batch);
selinv_status selinv_junction(const selinv_junction_plan_t *plan, selinv_dtype dtype, int32_t b, int64_t batch,
                              const void *diag, const void *edge_val, void *G_diag, void *G_lower,
                              double *logdet, int32_t *info, void *workspace, size_t workspace_bytes,
                              void *stream);

/*
 * Solve x = A^-1 r for `batch` general block-sparse SPD matrices on the
 * plan's pattern, from the same factorisation (gabp-sparse-inv, "General
 * sparse selected inverse": junction_solve).  With W_{u,v} = A'_{u,v} S_v^-1
 * for u in N(v), the factor is unit lower in elimination order and
 *   z_v = r_v - sum_{k: v in N(k)} W_{v,k} z_k      (children first)
 *   x_v = S_v^-1 z_v - sum_{u in N(v)} W_{u,v}^T x_u  (parents first).
 *   diag, edge_val  as in selinv_junction
 *   rhs [batch, n, b]  r;  x [batch, n, b] out (must not alias rhs)
 *   logdet [batch] (may be NULL), info [batch] as in selinv_junction
 * Workspace: selinv_junction_workspace_size(plan, dtype, b, batch) bytes.
 * Same launch sequence caching as selinv_junction (keyed on rhs and x too).
 */
selinv_status selinv_junction_solve(const selinv_junction_plan_t *plan, selinv_dtype dtype, int32_t b,
                                    int64_t batch, const void *diag, const void *edge_val, const void *rhs,
                                    void *x, double *logdet, int32_t *info, void *workspace,
                                    size_t workspace_bytes, void *stream);

/*
 * Tree plan: validates `trees` parent arrays of n nodes each (HOST memory,
 * parent [trees, n] int32, exactly one root per tree with parent = -1, no
 * cycles, indices in [0, n)), builds the level-set schedule -- nodes grouped
 * by height for the collect sweep and by depth for the distribute sweep,
 * children in ascending index, each node's position in its parent's child
 * list, and the chains of first children whose heads the distribute sweep,
 * a draw's and the backward's parents-first pass take in depth order -- and
 * copies it to the current device.
 * (gabp-sparse-inv, "Implemented and tested kernels" -> Tree, and the
 * level-set batched path of "General sparse selected inverse": one batched
 * step per elimination level.)  The plan is owned by the library until
 * selinv_tree_plan_free.  Synchronous.  Returns SELINV_ERR_BAD_TREE for a
 * malformed parent array.
 */
typedef struct selinv_tree_plan_s selinv_tree_plan_t;

selinv_status selinv_tree_plan(const int32_t *parent, int64_t trees, int64_t n,
                               selinv_tree_plan_t **out);

void selinv_tree_plan_free(selinv_tree_plan_t *plan);

/*
 * Dependency waits of the tree sweeps.  A chain head of the distribute sweep
 * (and of a draw's and the backward's parents-first pass) waits for its
 * parent's completion flag with a bounded spin: after spin_limit polls (each at least
 * 32-64 ns apart) it gives up, writes info = -2 for its tree (outputs of that
 * tree unspecified) and marks itself failed, so its own descendants give up
 * at once; the other trees are unaffected and the call returns normally.  A
 * valid plan never reaches the limit: every parent is handed to a running
 * warp before its children.  Default spin_limit 4194304 (values < 1 restore
 * it).  withhold: a node (global index tree * n + v) whose completion the
 * sweeps never publish, or -1 for none -- a test hook that makes that
 * node's children give up (those that wait run out their bound; its first
 * child, which follows it in a chain without waiting, gives up at once).
 * Host only; applies to later calls with this plan.
 */
selinv_status selinv_tree_plan_set_wait(selinv_tree_plan_t *plan, int32_t spin_limit, int64_t withhold);

/* Levels of a plan: *collect = max height + 1, *distribute = max depth + 1. */
selinv_status selinv_tree_plan_levels(const selinv_tree_plan_t *plan, int32_t *collect,
                                      int32_t *distribute);

size_t selinv_tree_workspace_size(const selinv_tree_plan_t *plan, selinv_dtype dtype, int32_t b);

/*
 * Selected inverse and log-determinant of block-tree SPD matrices.
 *   diag   [trees, n, b, b]  D_v (lower triangle read)
 *   edge   [trees, n, b, b]  edge[v] = A_{parent(v), v}; root slot ignored
 *   G_diag [trees, n, b, b]  out: (A^-1)_{v,v}
 *   G_edge [trees, n, b, b]  out: (A^-1)_{parent(v), v}; root slot written 0
 *   logdet [trees] float64   out; may be NULL
 *   info   [trees] int32     out: -1, or a node whose pivot failed, or -2 when
 *                            a dependency wait gave up (selinv_tree_plan_set_wait),
 *                            or -3 - v (SELINV_CHECK: node v holds a non-finite entry)
 *   flags  SELINV_WANT_LOGDET, SELINV_CHECK, or 0
 */
selinv_status selinv_tree(const selinv_tree_plan_t *plan, selinv_dtype dtype, int32_t b,
                          const void *diag, const void *edge,
                          void *G_diag, void *G_edge, double *logdet, int32_t *info,
                          void *workspace, size_t workspace_bytes, uint32_t flags, void *stream);

/*
 * Gaussian draw on block trees (gabp-sparse-inv, "Gaussian sampling":
 * sample_gaussian_tree draws x ~ N(0, A^-1) reusing the factorisation):
 *   eta = P^T L^-T z,  A = P^T L L^T P
 * with P the tree's own elimination order (children before parents; the
 * factor's blocks do not depend on the order among siblings): L_vv = R_v,
 * S_v = R_v R_v^T, and L_{parent(v), v} = edge[v] R_v^-T.  z [trees, n, b]
 * are the caller's standard normals, eta [trees, n, b] the draw; diag, edge,
 * logdet, info, workspace and errors as in selinv_tree (b <= 16).
 */
selinv_status selinv_tree_sample(const selinv_tree_plan_t *plan, selinv_dtype dtype, int32_t b,
                                 const void *diag, const void *edge, const void *z, void *eta,
                                 double *logdet, int32_t *info,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * Cotangents of the tree selected inverse (b <= 16): the tree form of
 * selinv_chain_backward.  From the cotangents Gb_diag, Gb_edge [trees, n, b, b]
 * of selinv_tree's outputs (NULL = zero; the root's Gb_edge slot is ignored)
 * writes Db [trees, n, b, b] (lower-triangular: only D_v's lower triangle is
 * read) and Eb [trees, n, b, b] (edge[v] sits at (p(v), v) and, transposed,
 * at (v, p(v)); the root slot is written 0), Ab = -A^-1 Gbar A^-1 read back
 * onto the inputs.  (gabp-sparse-inv 0.3.2, "Differentiable selected
 * inverse": selinv_tree's gradients reach diag and edge through an analytic
 * two-pass backward.)  Pass 1 runs children before parents, pass 2 parents
 * before children, like the forward's sweeps.
 *   diag, edge, G_diag, G_edge  the forward's inputs and outputs (device)
 *   info [trees]   -1, or a node whose Schur complement is not positive
 *                  definite (outputs then unspecified)
 * Workspace: selinv_tree_backward_workspace_size(plan, dtype, b) bytes.
 */
size_t selinv_tree_backward_workspace_size(const selinv_tree_plan_t *plan, selinv_dtype dtype, int32_t b);

selinv_status selinv_tree_backward(const selinv_tree_plan_t *plan, selinv_dtype dtype, int32_t b,
                                   const void *diag, const void *edge, const void *G_diag,
                                   const void *G_edge, const void *Gb_diag, const void *Gb_edge,
                                   void *Db, void *Eb, int32_t *info, void *workspace,
                                   size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SELINV_H */
