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
SELINV_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
SELINV_DEVINL void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
// Wait until at most one committed group (the most recent) is still in flight.
SELINV_DEVINL void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

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

// Reciprocal of a positive normal d: the hardware approximation refined by one
// cubic Newton-Raphson step, r <- r (1 + e + e^2) with e = 1 - d r, which
// triples the number of correct bits of the estimate (about 20 -> full
// precision).  Not for zero, negative, subnormal or non-finite d (the callers
// flag such pivots as failures and do not use the result).
SELINV_DEVINL double recip(double d)
{
    double r;
    asm("rcp.approx.ftz.f64 %0, %1;\n" : "=d"(r) : "d"(d));
    const double e = fma(-d, r, 1.0);
    return fma(r, fma(e, e, e), r);
}
SELINV_DEVINL float recip(float d) { return __frcp_rn(d); }

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

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace selinv
