// exact_budget.cuh -- the token budget Bhat = ceil(min(N, max(Bmin, e^y))),
// y = a*H + b, decided exactly.
//
// "Token Radius Attention for Efficient Video Generation" (gist.science
// summary), section 2, Intuition I: the budget of a query grows as
// tau * exp(H_i); here B = exp(a*H + b), clamped to [Bmin, N] and rounded up.
//
// For a double y != 0, e^y is irrational, so ceil(e^y) has one exact answer.
// An fp64 exponential with an error of a few ulps decides it unless e^y lies
// within those ulps of an integer -- which happens for whole classes of
// inputs, e.g. a = 0 and b = ln(k) (a fixed budget of k tokens): fp64(ln k)
// misses ln k by up to half an ulp, so e^b misses k by a few ulps of k, and
// two exponentials that differ in the last bit put the ceiling on k or k + 1.
// So when the fp64 value falls within 16 ulps of an integer, e^y is
// recomputed in double-double arithmetic (about 100 significant bits) and the
// side of the integer it falls on is read from that.
//
// The double-double steps are the classic error-free transformations: Knuth's
// two-sum, the product error from one fused multiply-add, and division by a
// small integer with its exact remainder from a fused multiply-add.  e^y is
// reduced as y = n*ln2 + r with ln 2 split into three parts of at most 32,
// 32 and 53 bits (n*part exact for |n| < 2^20), and e^r (|r| <= ln2/2) is
// the Taylor series to r^27/27!, evaluated as 1 + r(1 + r/2(1 + r/3(...))).
// Every operation is an explicitly rounded IEEE operation (no contraction).
#pragma once
#include <cmath>
#include <cuda_runtime.h>

namespace tra {

namespace xb {

#ifdef __CUDA_ARCH__
__device__ __forceinline__ double add(double a, double b) { return __dadd_rn(a, b); }
__device__ __forceinline__ double sub(double a, double b) { return __dsub_rn(a, b); }
__device__ __forceinline__ double mul(double a, double b) { return __dmul_rn(a, b); }
__device__ __forceinline__ double div(double a, double b) { return __ddiv_rn(a, b); }
__device__ __forceinline__ double fma(double a, double b, double c) { return __fma_rn(a, b, c); }
#else
// host copies (the file is built with -ffp-contract=off; volatile keeps each
// operation a separately rounded one)
inline double add(double a, double b) { volatile double r = a + b; return r; }
inline double sub(double a, double b) { volatile double r = a - b; return r; }
inline double mul(double a, double b) { volatile double r = a * b; return r; }
inline double div(double a, double b) { volatile double r = a / b; return r; }
inline double fma(double a, double b, double c) { return std::fma(a, b, c); }
#endif

struct dd {
    double hi, lo;
};

// s + e == a + b exactly (Knuth)
__host__ __device__ __forceinline__ dd two_sum(double a, double b)
{
    const double s = add(a, b);
    const double bb = sub(s, a);
    const double e = add(sub(a, sub(s, bb)), sub(b, bb));
    return {s, e};
}

// the same for |a| >= |b| (or a == 0)
__host__ __device__ __forceinline__ dd quick_two_sum(double a, double b)
{
    const double s = add(a, b);
    return {s, sub(b, sub(s, a))};
}

__host__ __device__ __forceinline__ dd dd_add(dd x, dd y)
{
    const dd s = two_sum(x.hi, y.hi);
    return quick_two_sum(s.hi, add(s.lo, add(x.lo, y.lo)));
}

__host__ __device__ __forceinline__ dd dd_mul(dd x, dd y)
{
    const double p = mul(x.hi, y.hi);
    double e = fma(x.hi, y.hi, -p);          // the exact error of the product
    e = fma(x.hi, y.lo, e);
    e = fma(x.lo, y.hi, e);
    return quick_two_sum(p, e);
}

// x / k for a small positive integer k
__host__ __device__ __forceinline__ dd dd_div_int(dd x, int k)
{
    const double kd = (double)k;
    const double q = div(x.hi, kd);
    const double rem = fma(-q, kd, x.hi);    // x.hi - q*k, exact
    return quick_two_sum(q, div(add(rem, x.lo), kd));
}

// e^y as a double-double, for |y| < 700
__host__ __device__ inline dd exp_dd(double y)
{
    const double LN2_1 = 0x1.62e42ff000000p-1;     // ln 2 = LN2_1 + LN2_2 + LN2_3 + O(2^-122)
    const double LN2_2 = -0x1.718432a200000p-35;
    const double LN2_3 = 0x1.3c7673007e5edp-69;
    const double INV_LN2 = 0x1.71547652b82fep+0;
    const double n = rint(mul(y, INV_LN2));
    // r = y - n*ln2: n*LN2_1 and n*LN2_2 are exact products
    dd r = two_sum(y, -mul(n, LN2_1));
    r = dd_add(r, dd{-mul(n, LN2_2), 0.0});
    const double p3 = mul(n, LN2_3);
    r = dd_add(r, dd{-p3, -fma(n, LN2_3, -p3)});
    dd t = {1.0, 0.0};
    for (int k = 27; k >= 1; --k) t = dd_add(dd{1.0, 0.0}, dd_div_int(dd_mul(r, t), k));
    const int ni = (int)n;
    return {ldexp(t.hi, ni), ldexp(t.lo, ni)};
}

}  // namespace xb

// Bhat = ceil(min(N, max(Bmin, e^y))), exactly; a NaN y gives Bmin.
__host__ __device__ inline long long budget_from_exponent(double y, long long N, long long Bmin)
{
    if (y != y) return Bmin;
    const double e = exp(y);
    if (e >= (double)N + 2.0) return N;
    if (e <= 0.5) return Bmin;                      // e^y < 1: ceil is 1 <= Bmin
    double c = ceil(e);
    // within 16 ulps of an integer (c itself or c - 1): settle the side exactly
    const double tol = e * 0x1p-48;
    if (c - e <= tol || e - (c - 1.0) <= tol) {
        const xb::dd x = xb::exp_dd(y);
        const double k = ceil(x.hi);
        c = (x.hi == k && x.lo > 0.0) ? k + 1.0 : k;    // x.hi a whole number: x.lo decides
    }
    long long B = (long long)c;
    if (B < Bmin) B = Bmin;
    if (B > N) B = N;
    return B;
}

}  // namespace tra
