// Internal interface between the C ABI (api.cu) and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace selinv {

// One batched chain call: all arrays device, row-major, contiguous.
template <class T> struct ChainArgs {
    const T *diag;      // [batch, L, b, b]
    const T *lower;     // [batch, L-1, b, b]
    T *G_diag;          // [batch, L, b, b] or null
    T *G_lower;         // [batch, L-1, b, b] or null (with G_diag)
    double *logdet;     // [batch] or null
    const T *rhs;       // [batch, L, b] or null
    T *x;               // [batch, L, b] or null (with rhs)
    const T *z = nullptr;   // [batch, L, b] standard normals of a Gaussian draw, or null
    int nrhs = 0;           // > 0: rhs / x are [batch, L, b, nrhs]; this launch takes columns
    int c0 = 0;             //      c0 .. c0 + 15 (fewer at the end)
    int32_t *info;      // [batch]
    T *ws;              // workspace
    int64_t batch;
    int64_t L;
    int b;
    bool ws_lines = false;  // workspace starts on a 128-byte boundary (its slots may be dropped from L2)
};

// b <= 16: one warp per chain.
size_t chain_small_workspace(size_t elem, int64_t batch, int64_t L);
template <class T> cudaError_t chain_small_launch(const ChainArgs<T> &a, bool aligned16, cudaStream_t s);
// x = A^-1 rhs for nrhs right-hand sides (columns c0 .. c0 + 15 of them per launch; no G).
template <class T> cudaError_t chain_small_multi_launch(const ChainArgs<T> &a, bool aligned16, cudaStream_t s);
// The same kernel drawing eta = A^-1 rhs + L^-T z into a.x (rhs may be null; no G).
template <class T> cudaError_t chain_small_sample_launch(const ChainArgs<T> &a, bool aligned16, cudaStream_t s);

// Short chains with small blocks (float64, b <= 8, L <= 16): one warp per
// chain, the chain held in shared memory, 8 x 8 tiles; no workspace.
bool chain_tiny_fits(int64_t L, int b);
cudaError_t chain_tiny_launch(const ChainArgs<double> &a, cudaStream_t s);

// 16 < b <= 32, no right-hand side: one CTA of two 4-warp groups per chain,
// eliminating from both ends toward the middle block.
size_t chain_mid_workspace(size_t elem, int64_t batch, int64_t L);
template <class T> cudaError_t chain_mid_launch(const ChainArgs<T> &a, cudaStream_t s);

// 16 < b <= 32 with G and no right-hand side, long chains and a batch too
// small to fill the GPU: P segments per chain, one 4-warp CTA each (0 = not
// used; depends on the current device's SM count).
int chain_seg_parts(int64_t batch, int64_t L, int b, bool want_g, bool want_x);
size_t chain_seg_workspace(size_t elem, int64_t batch, int64_t L, int b, int P, bool want_g);
template <class T> cudaError_t chain_seg_launch(const ChainArgs<T> &a, int P, cudaStream_t s);

// 16 < b <= 128: one CTA per chain.
size_t chain_large_workspace(size_t elem, int64_t batch, int64_t L, int b);
template <class T> cudaError_t chain_large_launch(const ChainArgs<T> &a, cudaStream_t s);
// The same kernel drawing eta = A^-1 rhs + L^-T z into a.x (float64; rhs may be null; no G).
cudaError_t chain_large_sample_launch(const ChainArgs<double> &a, cudaStream_t s);

// Cotangents of the chain selected inverse (b <= 16: one warp per chain).
template <class T> struct ChainBwdArgs {
    const T *diag, *lower;          // forward inputs
    const T *G_diag, *G_lower;      // forward outputs
    const T *Gb_diag, *Gb_lower;    // their cotangents
    T *Db, *Bb;                     // cotangents of diag (lower-triangular) and lower
    int32_t *info;                  // [batch]
    T *ws;
    int64_t batch;
    int64_t L;
    int b;
};
size_t chain_backward_workspace(size_t elem, int64_t batch, int64_t L);
template <class T> cudaError_t chain_backward_launch(const ChainBwdArgs<T> &a, bool aligned16, cudaStream_t s);

// Block lower-bidiagonal matrices with general blocks (b <= 16).
template <class T> struct BidiagArgs {
    const T *diag, *lower;          // M_ii [batch, L, b, b], M_{i+1,i} [batch, L-1, b, b]
    T *G_diag, *G_lower;            // (M^-1)_ii, (M^-1)_{i+1,i}
    int32_t *info;                  // [batch]
    int64_t batch;
    int64_t L;
    int b;
};
template <class T> cudaError_t bidiag_launch(const BidiagArgs<T> &p, bool aligned16, cudaStream_t s);
// Its cotangents from the forward's outputs (b <= 16).
template <class T> struct BidiagBwdArgs {
    const T *G_diag, *G_lower;      // forward outputs
    const T *Gb_diag, *Gb_lower;    // their cotangents (null = zero)
    T *Mb_diag, *Mb_lower;          // cotangents of M_ii and M_{i+1,i}
    int64_t batch;
    int64_t L;
    int b;
};
template <class T> cudaError_t bidiag_backward_launch(const BidiagBwdArgs<T> &a, bool aligned16, cudaStream_t s);

// SELINV_CHECK: finiteness of every entry a call reads, reported in info as
// -3 - k (k = first block with a non-finite entry); runs after the call's
// kernels.  kind 0: lower triangles of b x b blocks, 1: whole blocks, 2:
// length-b vectors; a: [batch, nb, ...]; parent (trees): skip root slots.
template <class T>
cudaError_t check_finite_launch(const T *a, int64_t batch, int64_t nb, int b, int kind, const int32_t *parent,
                                int32_t *info, cudaStream_t s);
cudaError_t check_finalize_launch(int32_t *info, int64_t batch, int64_t nb, cudaStream_t s);

}  // namespace selinv
