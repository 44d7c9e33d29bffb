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

// tile index -> (frame, tile row, tile col)
__device__ __forceinline__ void tile_coords(const Geom& G, int tile, int& t, int& tr, int& tc)
{
    t = tile / G.tiles_per_frame;
    int rem = tile - t * G.tiles_per_frame;
    tr = rem / G.nTw;
    tc = rem - tr * G.nTw;
}

}  // namespace tra
