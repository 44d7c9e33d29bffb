// pipeline.cuh -- helpers shared by the tensor-core kernels: the per-device
// error word, bounded role waits, and the per-row key masks inside a tile.
#pragma once
#include "sm100.cuh"
#include "tra_common.cuh"

namespace tra {

// Per-device error word: bit 0 = a bounded wait gave up, bit 1 = an index
// check failed.  Read and cleared by the host after a stream sync.
__device__ unsigned int g_tra_error;

// Bounded wait that also gives up as soon as another role has aborted.  On
// give-up it raises the CTA's abort flag and the device error word.  A zero
// limit gives up at once (the timeout-path test hook).
__device__ __forceinline__ bool role_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                          volatile int* abort_flag)
{
    if (limit_ns == 0) {           // test hook: give up without waiting
        *abort_flag = 1;
        atomicOr(&g_tra_error, TRA_ERRBIT_TIMEOUT);
        return false;
    }
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 15u) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                atomicOr(&g_tra_error, TRA_ERRBIT_TIMEOUT);
                return false;
            }
        }
    }
}

// For event-driven issuers that poll several barriers: returns false (and
// raises the abort flag and the error word) once no progress has been made
// for limit_ns, or as soon as another role has aborted.
__device__ __forceinline__ bool poll_alive(uint64_t& t_last, bool progress, uint64_t limit_ns, volatile int* abort_flag)
{
    if (progress) {
        t_last = globaltimer_ns();
        return true;
    }
    if (*abort_flag) return false;
    if (globaltimer_ns() - t_last > limit_ns) {
        *abort_flag = 1;
        atomicOr(&g_tra_error, TRA_ERRBIT_TIMEOUT);
        return false;
    }
    __nanosleep(32);
    return true;
}

// A shared-memory lock that keeps the MMA groups of two issuers from
// interleaving in the tensor pipe (an issue occupies the issuing thread about
// as long as the MMA runs, so a group issued under the lock runs as a block).
__device__ __forceinline__ bool issue_lock(int* lock, uint64_t limit_ns, volatile int* abort_flag)
{
    if (atomicCAS(lock, 0, 1) == 0) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        __nanosleep(20);
        if (atomicCAS(lock, 0, 1) == 0) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            atomicOr(&g_tra_error, TRA_ERRBIT_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void issue_unlock(int* lock) { atomicExch(lock, 0); }

// One 64-column panel of a 128-row tile (frame t, tile row tr, tile column
// tc, head g) into shared memory.  Tile-major inputs: rows tile*128 ..
// tile*128+127 of a [rows][d] map.  Natural inputs: a {64, tw, th, 1} box of a
// [heads*T][H][W][d] map, which lands in the same row order (row = (h - h0)*tw
// + (w - w0)); positions past the grid's edge read as zeros.
__device__ __forceinline__ void load_tile_panel(void* dst, const CUtensorMap* m, const Geom& G, int p, int g, int t,
                                                int tr, int tc, uint64_t* bar)
{
    if (G.natural)
        tma_load_4d(dst, m, p * 64, tc * G.tw, tr * G.th, g * G.T + t, bar);
    else
        tma_load_2d(dst, m, p * 64, g * G.N_pad + ((t * G.nTh + tr) * G.nTw + tc) * 128, bar);
}

// Keep-bits of one query row inside a key tile, as four 32-column words.
// Key (a, b) of the tile (a = key row, b = key column) is kept iff
// a_lo <= a <= a_hi and b_lo <= b <= b_hi.
template <int TWL>
__device__ __forceinline__ void row_keep_bits(int a_lo, int a_hi, int b_lo, int b_hi, uint32_t (&m)[4])
{
    constexpr int TW = 1 << TWL;
    uint32_t cb = 0;
    if (b_lo <= b_hi) cb = (2u << b_hi) - (1u << b_lo);     // b_hi = 31 wraps to the right mask
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
        uint32_t v = 0;
#pragma unroll
        for (int k = 0; k < 32 / TW; ++k) {
            const int a = (wd * 32) / TW + k;
            const int sh = (a * TW) & 31;
            if (a >= a_lo && a <= a_hi) v |= cb << sh;
        }
        m[wd] = v;
    }
}

}  // namespace tra
