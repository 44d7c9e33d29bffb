// Host build of the library's exact budget rule (csrc/exact_budget.cuh) for
// the CPU tests: reads "y N Bmin" lines (y as a C99 hex float) from stdin
// and prints Bhat = ceil(min(N, max(Bmin, e^y))) per line.
#include <cstdio>
#include <cstdlib>

#include "exact_budget.cuh"

int main()
{
    char buf[128];
    long long N, Bmin;
    while (std::scanf("%127s %lld %lld", buf, &N, &Bmin) == 3) {
        const double y = std::strtod(buf, nullptr);
        std::printf("%lld\n", tra::budget_from_exponent(y, N, Bmin));
    }
    return 0;
}
