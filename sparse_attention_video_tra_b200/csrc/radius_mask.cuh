// radius_mask.cuh -- budget, radius and block-sparse mask in one launch.
//
// "Token Radius Attention for Efficient Video Generation" (gist.science
// summary), section 2: Intuition I (entropy -> token budget), "Budget-vers-
// Rayon" (budget -> query radius, shrunk per frame by the temporal decay), and
// "Noyaux CUDA Fusionnes" (distance computation, radius comparison, block
// pruning and token voting fused into one kernel that emits a block-sparse
// mask).  Token voting is read as an OR vote: a key tile is listed for a query
// tile iff some retained token pair falls in it, so skipping unlisted tiles
// never changes the attention output.
//
// One CTA per (query tile, head), one thread per tile row (token).
//   1. Bhat = ceil(min(N, max(Bmin, exp(a*H + b)))), y = a*H + b in fp64 and
//      the ceiling of e^y decided exactly.
//   2. r = the smallest r in [0, r_cap] whose clipped neighbourhood count
//      reaches Bhat (binary search; the count is monotone in r).
//   3. Per frame distance |dt|: every query's neighbourhood is a rectangle of
//      key tiles that contains the query tile's own tile position, so for a
//      key tile row the union over the tile's queries is one interval of tile
//      columns (warp min/max reductions), and the "full" tiles (every valid
//      pair retained) are the intersection of per-query rectangles.
//   4. The active tiles of the frames within Rt' are written in ascending
//      tile order after a block-wide prefix sum over (frame, tile row).
// With radius-sorted query groups (a scheduling choice of this library) each
// CTA first finds the radii of both tiles of its pair (2p, 2p+1: side by side
// in one tile row), orders the pair's 256 rows by (radius, row), and then
// speaks for the 128 queries of its own group instead of its own tile's rows;
// step 3 still holds because every member's rectangle contains its own tile
// column, one of two adjacent columns of the same tile row.
#pragma once
#include "exact_budget.cuh"
#include "tra_common.cuh"

namespace tra {

// clipped neighbourhood count c(r) of the query at (t, h, w): per frame the
// Chebyshev square is a clipped rectangle; the disk sums, key row by key row,
// the clipped width 2*isqrt(s^2 - dh^2) + 1
template <bool DISK>
__device__ __forceinline__ long long nbr_count(const Geom& G, int t, int h, int w, int r)
{
    long long c = 0;
    for (int dl = 0; dl <= G.rte; ++dl) {
        const int m = (t + dl < G.T ? 1 : 0) + (dl > 0 && t - dl >= 0 ? 1 : 0);
        if (m == 0) break;                         // farther frames are out of the grid too
        const int s = halfwidth(r, G.g[dl]);
        if constexpr (DISK) {
            // key rows h - k (k <= up) and h + k (k <= dn) share the half-width
            // isqrt(s^2 - k^2)
            const int sc = min(s, TRA_DISK_S_CLAMP);
            const int up = min(sc, h), dn = min(sc, G.H - 1 - h);
            const int kmax = max(up, dn), s2 = sc * sc;
            long long X = 0;
            for (int k = 0; k <= kmax; ++k) {
                const int half = isqrt_floor(s2 - k * k);
                const int wid = min(G.W - 1, w + half) - max(0, w - half) + 1;
                X += k == 0 ? wid : (k <= up ? wid : 0) + (k <= dn ? wid : 0);
            }
            c += m * X;
        } else {
            const int X = min(h, s) + min(G.H - 1 - h, s) + 1;
            const int Y = min(w, s) + min(G.W - 1 - w, s) + 1;
            c += (long long)(m * X) * Y;
        }
    }
    return c;
}

// Bhat = ceil(min(N, max(Bmin, exp(a*H + b)))): a*H and + b rounded
// separately in fp64, the ceiling decided exactly (exact_budget.cuh)
__device__ __forceinline__ long long budget_hat(const Geom& G, float Hent)
{
    const double y = __dadd_rn(__dmul_rn(G.a, (double)Hent), G.b);
    return budget_from_exponent(y, G.N, G.Bmin);
}

// r = the smallest r in [0, r_cap] whose neighbourhood count reaches bh (the
// count is monotone in r; r_cap when none does); c = that count.
template <bool DISK>
__device__ __forceinline__ int find_radius(const Geom& G, int t, int h, int w, long long bh, long long& c)
{
    int lo = 0, hi = G.r_cap;
    if constexpr (DISK) {
        // the disk lies inside the square of the same half-width, so its
        // radius is at least the square's; search [r_sq, 2 r_sq + 2] when
        // that bracket reaches the budget, else the rest up to r_cap
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (nbr_count<false>(G, t, h, w, mid) >= bh) hi = mid; else lo = mid + 1;
        }
        const int r2 = min(G.r_cap, 2 * lo + 2);
        if (nbr_count<true>(G, t, h, w, r2) >= bh) hi = r2;
        else { lo = min(r2 + 1, G.r_cap); hi = G.r_cap; }
    }
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (nbr_count<DISK>(G, t, h, w, mid) >= bh) hi = mid; else lo = mid + 1;
    }
    c = nbr_count<DISK>(G, t, h, w, lo);
    return lo;
}

// Dynamic shared memory of the mask kernel, sized from the plan so that small
// reaches keep many CTAs resident: per (frame distance, tile row) the active
// column interval [lo, hi] and the disk's full-column bits, and per list row
// (frame, tile row) its length.
// With radius-sorted groups it also holds the pair's 256 counts, radii and
// the group order.
__host__ __device__ inline int mask_smem_bytes(int rte, int nTh, bool qsort)
{
    return (qsort ? 256 * (8 + 4 + 4) : 0) + (3 * (rte + 1) * nTh + (2 * rte + 1) * nTh) * 4;
}

template <bool DISK, bool QS>
__global__ void __launch_bounds__(128) radius_mask_kernel(const Geom G, const float* __restrict__ Hent,
                                                          uint8_t* __restrict__ mask)
{
    extern __shared__ __align__(16) long long mask_smem[];
    const int RS = G.nTh;                                         // stride of one frame distance
    long long* s_qc = mask_smem;                                  // QS: [256] counts of the pair's rows
    int* s_qr = reinterpret_cast<int*>(s_qc + (QS ? 256 : 0));    // QS: [256] radii of the pair's rows
    int* s_qp = s_qr + (QS ? 256 : 0);                            // QS: [256] pair rows in group order
    int* s_lo = s_qp + (QS ? 256 : 0);                            // [rte + 1][nTh]
    int* s_hi = s_lo + (G.rte + 1) * RS;                          // [rte + 1][nTh]
    uint32_t* s_fullbits = reinterpret_cast<uint32_t*>(s_hi + (G.rte + 1) * RS);   // disk: full tile columns
    int* s_len = reinterpret_cast<int*>(s_fullbits + (G.rte + 1) * RS);            // [(2 rte + 1) nTh]
    __shared__ int s_full[TRA_MAX_RT_EFF + 1][4];
    __shared__ long long s_pairs[4];
    __shared__ int s_warp[4];

    const int tile = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int t, trq, tcq;
    tile_coords(G, tile, t, trq, tcq);

    for (int i = tid; i < (G.rte + 1) * RS; i += 128) {
        s_lo[i] = 0x7fffffff;
        s_hi[i] = -1;
        s_fullbits[i] = 0xffffffffu;
    }
    if (tid < G.rte + 1) {
        s_full[tid][0] = -0x7fffffff; s_full[tid][1] = 0x7fffffff;
        s_full[tid][2] = -0x7fffffff; s_full[tid][3] = 0x7fffffff;
    }

    // ---- budget and radius of the query this thread speaks for: its own row
    // of the tile, or (QS) a slot of the tile's radius-sorted group
    int h, w, r = -1;
    bool valid;
    long long c = 0;
    if constexpr (!QS) {
        h = trq * G.th + (tid >> G.tw_log2);
        w = tcq * G.tw + (tid & (G.tw - 1));
        valid = h < G.H && w < G.W;
        if (valid) r = find_radius<DISK>(G, t, h, w, budget_hat(G, Hent[io_row(G, g, t, h, w, tile * 128 + tid)]), c);
        reinterpret_cast<int32_t*>(mask + G.off_radius)[(size_t)g * G.N_pad + (size_t)tile * 128 + tid] = r;
    } else {
        // both tiles of the pair (tiles 2p, 2p+1 side by side in one tile row)
        const int pb = tile & ~1;
        for (int k = 0; k < 2; ++k) {
            const int hk = trq * G.th + (tid >> G.tw_log2);
            const int wk = (tcq - (tile & 1) + k) * G.tw + (tid & (G.tw - 1));
            int rk = -1;
            long long ck = 0;
            if (hk < G.H && wk < G.W)
                rk = find_radius<DISK>(G, t, hk, wk, budget_hat(G, Hent[io_row(G, g, t, hk, wk, (pb + k) * 128 + tid)]), ck);
            s_qr[k * 128 + tid] = rk;
            s_qc[k * 128 + tid] = ck;
            if (pb + k == tile)
                reinterpret_cast<int32_t*>(mask + G.off_radius)[(size_t)g * G.N_pad + (size_t)tile * 128 + tid] = rk;
        }
        __syncthreads();
        // order the pair's rows by (radius, row); pad rows (radius -1) first
        for (int k = 0; k < 2; ++k) {
            const int l = k * 128 + tid, rl = s_qr[l];
            int rank = 0;
            for (int j = 0; j < 256; ++j) {
                const int rj = s_qr[j];
                rank += (rj < rl || (rj == rl && j < l)) ? 1 : 0;
            }
            s_qp[rank] = l;
        }
        __syncthreads();
        const int l = s_qp[(tile & 1) * 128 + tid];
        h = trq * G.th + ((l & 127) >> G.tw_log2);
        w = (tcq - (tile & 1) + (l >> 7)) * G.tw + (l & (G.tw - 1));
        valid = h < G.H && w < G.W;
        r = s_qr[l];
        c = s_qc[l];
        mask[G.off_group + ((size_t)g * G.nQ + tile) * 128 + tid] = (uint8_t)l;
    }

    // ---- retained pairs of the tile
    long long cs = c;
    for (int o = 16; o > 0; o >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, o);
    if (lane == 0) s_pairs[warp] = cs;
    __syncthreads();
    if (tid == 0)
        reinterpret_cast<long long*>(mask + G.off_pairs)[(size_t)g * G.nQ + tile] =
            s_pairs[0] + s_pairs[1] + s_pairs[2] + s_pairs[3];

    // ---- per frame distance: active tile-column interval per tile row, full rectangle
    for (int dl = 0; dl <= G.rte; ++dl) {
        if (!(t + dl < G.T || t - dl >= 0)) break;    // uniform over the CTA
        int rl = 0x7fffffff, rh = -1, cl = 0, ch = -1;
        int frl = -0x7fffffff, frh = 0x7fffffff, fcl = -0x7fffffff, fch = 0x7fffffff;
        if (valid) {
            const int s = halfwidth(r, G.g[dl]);
            rl = max(0, h - s) >> G.th_log2;
            rh = min(G.H - 1, h + s) >> G.th_log2;
            cl = max(0, w - s) >> G.tw_log2;
            ch = min(G.W - 1, w + s) >> G.tw_log2;
            frl = (h - s <= 0) ? 0 : ((h - s + G.th - 1) >> G.th_log2);
            frh = (h + s >= G.H - 1) ? G.nTh - 1 : (((h + s + 1) >> G.th_log2) - 1);
            fcl = (w - s <= 0) ? 0 : ((w - s + G.tw - 1) >> G.tw_log2);
            fch = (w + s >= G.W - 1) ? G.nTw - 1 : (((w + s + 1) >> G.tw_log2) - 1);
        }
        frl = __reduce_max_sync(0xffffffffu, frl);
        frh = __reduce_min_sync(0xffffffffu, frh);
        fcl = __reduce_max_sync(0xffffffffu, fcl);
        fch = __reduce_min_sync(0xffffffffu, fch);
        if (lane == 0) {
            atomicMax(&s_full[dl][0], frl); atomicMin(&s_full[dl][1], frh);
            atomicMax(&s_full[dl][2], fcl); atomicMin(&s_full[dl][3], fch);
        }
        const int r_lo = __reduce_min_sync(0xffffffffu, rl);
        const int r_hi = __reduce_max_sync(0xffffffffu, rh);
        for (int tr = r_lo; tr <= r_hi; ++tr) {
            const bool in = rl <= tr && tr <= rh;
            int c_lo = cl, c_hi = ch;
            if (DISK && in) {
                // the disk is widest on the tile row's key row nearest to h
                const int s = min(halfwidth(r, G.g[dl]), TRA_DISK_S_CLAMP);
                const int k0 = tr * G.th, k1 = min(G.H - 1, k0 + G.th - 1);
                const int dh = h < k0 ? k0 - h : (h > k1 ? h - k1 : 0);
                const int half = isqrt_floor(s * s - dh * dh);
                c_lo = max(0, w - half) >> G.tw_log2;
                c_hi = min(G.W - 1, w + half) >> G.tw_log2;
            }
            const int lo = __reduce_min_sync(0xffffffffu, in ? c_lo : 0x7fffffff);
            const int hi = __reduce_max_sync(0xffffffffu, in ? c_hi : -1);
            if (lane == 0 && hi >= 0) {
                atomicMin(&s_lo[dl * RS + tr], lo);
                atomicMax(&s_hi[dl * RS + tr], hi);
            }
        }
    }
    __syncthreads();

    // ---- disk: a listed tile is full iff, for every valid query, its valid
    // key rectangle's farthest corner lies in the disk (the disk is convex)
    if constexpr (DISK) {
        for (int dl = 0; dl <= G.rte; ++dl) {
            if (!(t + dl < G.T || t - dl >= 0)) break;
            const int s = valid ? min(halfwidth(r, G.g[dl]), TRA_DISK_S_CLAMP) : 0;
            for (int tr = 0; tr < G.nTh; ++tr) {
                const int lo = s_lo[dl * RS + tr], hi = s_hi[dl * RS + tr];
                if (hi < 0) continue;
                const int k0 = tr * G.th, k1 = min(G.H - 1, k0 + G.th - 1);
                const int dh = max(abs(h - k0), abs(h - k1));
                uint32_t bits = 0;
                for (int tc = lo; tc <= hi; ++tc) {
                    const int j0 = tc * G.tw, j1 = min(G.W - 1, j0 + G.tw - 1);
                    const int dw = max(abs(w - j0), abs(w - j1));
                    const bool in = !valid || (long long)dh * dh + (long long)dw * dw <= (long long)s * s;
                    if (__all_sync(0xffffffffu, in)) bits |= 1u << tc;
                }
                if (lane == 0) atomicAnd(&s_fullbits[dl * RS + tr], bits | ~(((2u << hi) - 1u) ^ ((1u << lo) - 1u)));
            }
        }
        __syncthreads();
    }

    // ---- list rows (frame, tile row) in ascending tile order; block prefix sum
    const int t0 = max(0, t - G.rte), t1 = min(G.T - 1, t + G.rte);
    const int R = (t1 - t0 + 1) * G.nTh;
    for (int i = tid; i < R; i += 128) {
        const int f = i / G.nTh, tr = i - f * G.nTh;
        const int dl = abs(t0 + f - t);
        s_len[i] = s_hi[dl * RS + tr] >= 0 ? s_hi[dl * RS + tr] - s_lo[dl * RS + tr] + 1 : 0;
    }
    __syncthreads();
    const int per = (R + 127) >> 7;
    const int beg = min(R, tid * per), end = min(R, beg + per);
    int local = 0;
    for (int i = beg; i < end; ++i) local += s_len[i];
    int incl = local;
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int off = incl - local;
    for (int k = 0; k < warp; ++k) off += s_warp[k];
    uint16_t* list = reinterpret_cast<uint16_t*>(mask + G.off_list) + ((size_t)g * G.nQ + tile) * G.list_cap;
    for (int i = beg; i < end; ++i) {
        const int f = i / G.nTh, tr = i - f * G.nTh;
        const int dl = abs(t0 + f - t);
        const int lo = s_lo[dl * RS + tr], hi = s_hi[dl * RS + tr];
        const bool row_full = s_full[dl][0] <= tr && tr <= s_full[dl][1];
        const uint32_t fbits = s_fullbits[dl * RS + tr];
        const int base = ((t0 + f) * G.nTh + tr) * G.nTw;
        for (int tc = lo; tc <= hi; ++tc) {
            const bool full = DISK ? ((fbits >> tc) & 1u) != 0
                                     : (row_full && s_full[dl][2] <= tc && tc <= s_full[dl][3]);
            list[off++] = (uint16_t)((base + tc) | (full ? 0x8000 : 0));
        }
    }
    if (tid == 0)
        reinterpret_cast<int32_t*>(mask + G.off_count)[(size_t)g * G.nQ + tile] =
            s_warp[0] + s_warp[1] + s_warp[2] + s_warp[3];
}

}  // namespace tra
