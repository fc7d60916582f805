// Shared device helpers for libselinv's kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/selinv.h"

#define SELINV_DEVINL __device__ __forceinline__

namespace selinv {

constexpr unsigned FULL_MASK = 0xffffffffu;

// 16-byte asynchronous global->shared copy (bypasses L1).
SELINV_DEVINL void cp_async16(void *smem, const void *gmem)
{
    unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
// L2 eviction policies (createpolicy) for cache-hinted copies and stores:
// data streamed once leaves L2 first, so lines that are read back soon (the
// workspace slots between the two sweeps) stay resident.
SELINV_DEVINL uint64_t l2_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
    return p;
}
SELINV_DEVINL uint64_t l2_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;\n" : "=l"(p));
    return p;
}
// cp_async16 with an L2 eviction policy.
SELINV_DEVINL void cp_async16_hint(void *smem, const void *gmem, uint64_t pol)
{
    unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "l"(pol)
                 : "memory");
}
// 16-byte store of two doubles (or floats) with an L2 eviction policy.
SELINV_DEVINL void st_hint(double2 *p, double2 v, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v2.f64 [%0], {%1, %2}, %3;\n" ::"l"(p), "d"(v.x), "d"(v.y), "l"(pol)
                 : "memory");
}
SELINV_DEVINL void st_hint(float2 *p, float2 v, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;\n" ::"l"(p), "f"(v.x), "f"(v.y), "l"(pol)
                 : "memory");
}
// Drop the 128-byte L2 line at p (128-byte aligned) without writing it back:
// for scratch lines that are dead once read.
SELINV_DEVINL void discard_l2_line(const void *p)
{
    asm volatile("discard.global.L2 [%0], 128;\n" ::"l"(p) : "memory");
}
SELINV_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
SELINV_DEVINL void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
// Wait until at most one committed group (the most recent) is still in flight.
SELINV_DEVINL void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// Prefetch into L2 every 128-byte line of n elements at p (lines split over
// nthreads threads; every address issued lies inside the range).
SELINV_DEVINL void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p)); }
template <class T> SELINV_DEVINL void prefetch_range_l2(const T *p, int64_t n, int tid, int nthreads)
{
    const char *c = reinterpret_cast<const char *>(p);
    const int64_t bytes = n * (int64_t)sizeof(T);
    for (int64_t off = (int64_t)tid * 128; off < bytes; off += (int64_t)nthreads * 128) prefetch_l2(c + off);
}

// Read-only global loads that should not linger in L1.
template <class T> SELINV_DEVINL T ldg_stream(const T *p) { return __ldcs(p); }

// One FP64 tensor-core step: {d0,d1} += a (8x4 row fragment) * b (4x8 col fragment).
// Fragment ownership (lane = 4 g + t): a = A[g][t], b = B[t][g], d = C[g][2t..2t+1].
SELINV_DEVINL void dmma_8x8x4(double &d0, double &d1, double a, double b)
{
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
                 : "+d"(d0), "+d"(d1)
                 : "d"(a), "d"(b));
}

// Reciprocal of a pivot d in [2^-1022, 2^1022): the hardware approximation
// refined by one cubic Newton-Raphson step, r <- r (1 + e + e^2) with
// e = 1 - d r, which triples the number of correct bits of the estimate
// (about 20 -> full precision).  Outside that range the flush-to-zero
// estimate is wrong (a subnormal d flushes to zero, a reciprocal below
// 2^-1022 flushes to zero); bad_pivot reports such pivots as failures (a test
// off the sweep's dependency chain, unlike a branch to IEEE division here,
// which lengthened every pivot step).
SELINV_DEVINL double recip(double d)
{
    double r;
    asm("rcp.approx.ftz.f64 %0, %1;\n" : "=d"(r) : "d"(d));
    const double e = fma(-d, r, 1.0);
    return fma(r, fma(e, e, e), r);
}
SELINV_DEVINL float recip(float d) { return __frcp_rn(d); }

// A pivot the sweeps cannot use.  float64: not in [2^-1022, 2^1022) (this
// covers d <= 0 and NaN, and every pivot whose fast reciprocal would be
// wrong); float32 (IEEE reciprocal): not > 0, or a reciprocal that overflows.
SELINV_DEVINL bool bad_pivot(double d, double) { return !(d >= 0x1p-1022 && d < 0x1p1022); }
SELINV_DEVINL bool bad_pivot(float d, float p) { return !(d > 0.0f) || !(p <= 3.4028234663852886e38f); }
SELINV_DEVINL double rsqrt_t(double d) { return rsqrt(d); }
SELINV_DEVINL float rsqrt_t(float d) { return rsqrtf(d); }

template <class T> SELINV_DEVINL T shfl(T v, int src) { return __shfl_sync(FULL_MASK, v, src); }
template <class T> SELINV_DEVINL T shfl_xor(T v, int m) { return __shfl_xor_sync(FULL_MASK, v, m); }

// Running product of pivots kept as mantissa * 2^exponent (no overflow
// across a long sweep); log taken once at the end.
struct LogAcc {
    double m;
    int e;
    SELINV_DEVINL void init() { m = 1.0; e = 0; }
    SELINV_DEVINL void mul(double x) { m *= x; }
    SELINV_DEVINL void renorm()
    {
        int k;
        m = frexp(m, &k);
        e += k;
    }
    SELINV_DEVINL double log_value() const { return log(m) + (double)e * 0.69314718055994530942; }
};

// Inverse of a symmetric positive definite 8 x 8 matrix held by one warp in
// the m8n8 accumulator layout (lane 4g+t: v = P[g][2t], P[g][2t+1]) by the
// symmetric Gauss-Jordan sweep: for each pivot k (d = P_kk),
// P_ij -= P_ik P_kj / d, P_ik /= d, P_kj /= d, P_kk = -1/d, then negated.
// Row and column k travel by shuffles.  The pivots are multiplied into det
// (when `count`), a pivot that is not > 0 sets bad.
// DRAW: also rz = (R z)[g] for the Cholesky factor P = R R^T and z at the
// lane's columns 2t, 2t+1 (z0, z1).  At step k the entries P[i][k], i >= k,
// not yet swept are the Schur-complement column that Cholesky scales:
// R[i][k] = P[i][k] / sqrt(d), so rz += P[g][k] z_k / sqrt(d) for g >= k.
// The sweep's own chain does not wait for this sum.
template <bool DRAW = false, class T = double>
SELINV_DEVINL void inv8_sweep(T v[2], int lane, int g, int t, LogAcc &det, bool &bad, bool count,
                              T z0 = T(0), T z1 = T(0), T *rz = nullptr)
{
    // v = P[g][2t], P[g][2t+1] of a symmetric positive definite 8 x 8 P
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int kt = k >> 1, kj = k & 1;
        const T c = shfl(v[kj], (lane & ~3) | kt);               // P[g][k]
        T row[2];
        row[0] = shfl(v[0], (k << 2) | t);                         // P[k][2t]
        row[1] = shfl(v[1], (k << 2) | t);                         // P[k][2t+1]
        const T d = shfl(v[kj], (k << 2) | kt);                    // P[k][k]
        if (count) det.mul((double)d);
        const T p = recip(d);
        bad |= bad_pivot(d, p);
        if (DRAW) {
            const T zk = shfl(kj ? z1 : z0, (lane & ~3) | kt);
            if (g >= k) *rz = fma(c, zk * rsqrt_t(d), *rz);
        }
        const T tc = c * p;
        v[0] = fma(-tc, row[0], v[0]);
        v[1] = fma(-tc, row[1], v[1]);
        if (t == kt) v[kj] = tc;
        if (g == k) {
            v[0] = row[0] * p;
            v[1] = row[1] * p;
            if (t == kt) v[kj] = -p;
        }
    }
    v[0] = -v[0];
    v[1] = -v[1];
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace selinv
