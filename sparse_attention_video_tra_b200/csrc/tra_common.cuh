// tra_common.cuh -- device helpers shared by all kernels: the spatial
// half-width and the tile-major geometry.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "tra_geom.h"

namespace tra {

// floor(r * g + 1e-9) with the product and the sum rounded separately
// (the spatial half-width at decay g)
__device__ __forceinline__ int halfwidth(int r, double g)
{
    double p = __dmul_rn((double)r, g);
    double s = __dadd_rn(p, 1e-9);
    return (int)floor(s);
}

// a half-width at which the disk already covers any frame of at most
// TRA_MAX_HW x TRA_MAX_HW keys (keeps s*s below 2^20)
constexpr int TRA_DISK_S_CLAMP = 1023;

// the largest x >= 0 with x*x <= n, for 0 <= n <= 1023^2.  n is exact in
// fp32 and sqrtf rounds correctly; with k = that x, sqrt(n) lies in
// [k, k + 1 - 1/(2(k+1))] and 1/(2(k+1)) >= 2^-11 exceeds half an fp32 ulp
// at k + 1 <= 1024 (2^-14), so the rounded root never reaches k + 1 and its
// floor is k.
__device__ __forceinline__ int isqrt_floor(int n)
{
    return (int)sqrtf((float)n);
}

// tile index -> (frame, tile row, tile col)
__device__ __forceinline__ void tile_coords(const Geom& G, int tile, int& t, int& tr, int& tc)
{
    t = tile / G.tiles_per_frame;
    int rem = tile - t * G.tiles_per_frame;
    tr = rem / G.nTw;
    tc = rem - tr * G.nTw;
}

// Row of token (t, h, w) of head g in the caller's layout: natural order, or
// row `tile_row` (tile*128 + in-tile row) of the tile-major layout.
__device__ __forceinline__ size_t io_row(const Geom& G, int g, int t, int h, int w, int tile_row)
{
    return G.natural ? (size_t)g * G.N + ((size_t)t * G.H + h) * G.W + w : (size_t)g * G.N_pad + tile_row;
}

}  // namespace tra
