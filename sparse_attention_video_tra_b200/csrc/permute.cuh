// permute.cuh -- natural frame-major rows <-> padded tile-major rows.
//
// "Token Radius Attention for Efficient Video Generation" (gist.science
// summary), "Le Pipeline TRA", Disposition Tile-Major: tokens are reordered so
// that spatial neighbours (the ones a radius keeps) sit next to each other in
// the sequence.  Natural order n = (t*H + h)*W + w ("Token Radius Attention"
// blog post, sections 5.1 and 9.1).
//
// One thread moves 16 bytes; a row of d elements (bf16 or fp32) is d*size/16
// threads.  HBM-bound.
#pragma once
#include "tra_common.cuh"

namespace tra {

__global__ void __launch_bounds__(256) permute_kernel(const Geom G, const uint4* __restrict__ src,
                                                      uint4* __restrict__ dst, int to_tile_major, int elem_bytes)
{
    const int chunks = (G.D * elem_bytes) >> 4;      // 16-byte chunks per row
    const size_t total = (size_t)G.G * G.N_pad * chunks;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (size_t)gridDim.x * blockDim.x) {
        const int ch = (int)(i % chunks);
        const size_t prow = i / chunks;              // g * N_pad + p
        const int g = (int)(prow / G.N_pad);
        const int p = (int)(prow - (size_t)g * G.N_pad);
        const int tile = p >> 7, in = p & 127;
        int t, tr, tc;
        tile_coords(G, tile, t, tr, tc);
        const int h = tr * G.th + (in >> G.tw_log2);
        const int w = tc * G.tw + (in & (G.tw - 1));
        const bool valid = h < G.H && w < G.W;
        const size_t nrow = (size_t)g * G.N + ((size_t)t * G.H + h) * G.W + w;
        if (to_tile_major) {
            dst[i] = valid ? src[nrow * chunks + ch] : make_uint4(0, 0, 0, 0);
        } else if (valid) {
            dst[nrow * chunks + ch] = src[i];
        }
    }
}

}  // namespace tra
