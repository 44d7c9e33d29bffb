// radius_mask.cuh -- budget, radius and block-sparse mask in one launch.
//
// "Token Radius Attention for Efficient Video Generation" (gist.science
// summary), section 2: Intuition I (entropy -> token budget), "Budget-vers-
// Rayon" (budget -> query radius, shrunk per frame by the temporal decay), and
// "Noyaux CUDA Fusionnes" (distance computation, radius comparison, block
// pruning and token voting fused into one kernel that emits a block-sparse
// mask).  Token voting is read as an OR vote: a key tile is listed for a query
// set iff some retained token pair falls in it, so skipping unlisted tiles
// never changes the attention output.
//
// One CTA per (strip, head), one thread per row.  A strip is U tiles: with
// radius-sorted query groups (a scheduling choice of this library) the U =
// nTh tiles of one tile column of one frame, otherwise a single tile.
//   0. The half-widths s(r, |dt|) = floor(r * gamma^|dt| + 1e-9) of every r in
//      [0, r_cap] go into a shared table when it is small (the same fp64 rule,
//      evaluated once per entry instead of once per search probe).
//   1. Bhat = ceil(min(N, max(Bmin, exp(a*H + b)))), y = a*H + b in fp64 and
//      the ceiling of e^y decided exactly.
//   2. r = the smallest r in [0, r_cap] whose clipped neighbourhood count
//      reaches Bhat (binary search; the count is monotone in r).
//   3. Groups: with query groups the strip's 128*U rows are ordered by
//      (radius, strip row), pad rows first (each warp sorts its 32 keys with
//      shuffles; a key's rank adds its position in its own warp to a binary
//      search in every other warp's sorted keys); warpgroup u then speaks for
//      the u-th block of 128, the group of the strip's tile in tile row u.
//      Without groups warpgroup 0 speaks for its tile's own rows.
//   4. Per group and frame distance |dt|: every member's neighbourhood is a
//      rectangle of key tiles that contains the member's own tile column --
//      the strip's column -- so for a key tile row the union over the members
//      is one interval of tile columns (warp min/max reductions), and the
//      "full" tiles (every valid pair retained) are the intersection of the
//      members' rectangles.
//   5. Each group's active tiles of the frames within Rt' are written in
//      ascending tile order after a prefix sum over (frame, tile row).
#pragma once
#include "exact_budget.cuh"
#include "tra_common.cuh"

namespace tra {

// the spatial half-width at radius r and frame distance dl: from the shared
// table when the plan has one, else evaluated
__device__ __forceinline__ int hw_at(const Geom& G, const uint16_t* tab, int r, int dl)
{
    return tab ? (int)tab[dl * (G.r_cap + 1) + r] : halfwidth(r, G.g[dl]);
}

// Per query: what the neighbourhood count needs besides r.  Frames t + dt
// and t - dt hold the same clipped rectangle, so the count is
//   c(r) = P(0) + 2 * sum_{1 <= dt <= lo} P(dt) + sum_{lo < dt <= hi} P(dt)
// with lo / hi the smaller / larger of the reaches min(Rt', T-1-t) and
// min(Rt', t) on the two sides, and P(dt) the in-frame count at half-width
// s(r, dt).
struct CountCtx {
    int h, w, hb, wb;      // distances to the top / left and bottom / right edges
    int lo, hi;            // both sides within lo frames; one side up to hi
};

__device__ __forceinline__ CountCtx count_ctx(const Geom& G, int t, int h, int w)
{
    CountCtx x;
    x.h = h; x.w = w;
    x.hb = G.H - 1 - h; x.wb = G.W - 1 - w;
    const int fwd = min(G.rte, G.T - 1 - t), bwd = min(G.rte, t);
    x.lo = min(fwd, bwd);
    x.hi = max(fwd, bwd);
    return x;
}

// The disk-row table of half-width s (s <= disk_smax): entry k <= s holds the
// row half-width f_s(k) = isqrt(s^2 - k^2) (low 16 bits) and the running sum
// F_s(k) = f_s(0) + ... + f_s(k) (high 16 bits; F_s(s) <= s (s + 1) < 2^16).
// Row s starts at entry s (s + 1) / 2.
__device__ __forceinline__ const uint32_t* disk_row(const uint32_t* dtab, int s)
{
    return dtab + (s * (s + 1) >> 1);
}

// sum over key rows k = 0 .. n (n <= s) of min(cap, f_s(k)): f_s decreases,
// and f_s(k) >= cap  <=>  k^2 <= s^2 - cap^2  <=>  k <= f_s(cap) for cap < s,
// so the rows up to J = f_s(cap) contribute cap each and the rest f_s(k)
__device__ __forceinline__ int disk_capped_sum(const uint32_t* row, int s, int n, int cap)
{
    if (cap >= s) return (int)(row[n] >> 16);
    const int J = (int)(row[cap] & 0xffffu);
    return n <= J ? cap * (n + 1) : cap * (J + 1) + (int)(row[n] >> 16) - (int)(row[J] >> 16);
}

// in-frame clipped count at half-width s: the Chebyshev square is a clipped
// rectangle; the disk sums, key row by key row, the clipped width
// min(w, f) + min(W-1-w, f) + 1 with f = isqrt(s^2 - dh^2) -- from the
// disk-row table in O(1) when there is one (s >= disk_smax covers the frame,
// so s is capped there), else row by row
template <bool DISK>
__device__ __forceinline__ int frame_count(const Geom& G, const CountCtx& x, int s, const uint32_t* dtab)
{
    if constexpr (DISK) {
        if (dtab) {
            const int sc = min(s, G.disk_smax);
            const uint32_t* row = disk_row(dtab, sc);
            const int up = min(sc, x.h), dn = min(sc, x.hb);
            // rows h .. h - up and h .. h + dn; row h is in both
            const int cu = up + 1 + disk_capped_sum(row, sc, up, x.w) + disk_capped_sum(row, sc, up, x.wb);
            const int cd = dn + 1 + disk_capped_sum(row, sc, dn, x.w) + disk_capped_sum(row, sc, dn, x.wb);
            return cu + cd - (min(x.w, sc) + min(x.wb, sc) + 1);
        }
        // key rows h - k (k <= up) and h + k (k <= dn) share the half-width
        // isqrt(s^2 - k^2)
        const int sc = min(s, TRA_DISK_S_CLAMP);
        const int up = min(sc, x.h), dn = min(sc, x.hb);
        const int kmax = max(up, dn), s2 = sc * sc;
        int X = 0;
        for (int k = 0; k <= kmax; ++k) {
            const int half = isqrt_floor(s2 - k * k);
            const int wid = min(x.wb, half) + min(x.w, half) + 1;
            X += k == 0 ? wid : (k <= up ? wid : 0) + (k <= dn ? wid : 0);
        }
        return X;
    } else {
        return (min(x.h, s) + min(x.hb, s) + 1) * (min(x.w, s) + min(x.wb, s) + 1);
    }
}

// clipped neighbourhood count c(r) (at most N < 2^31)
template <bool DISK>
__device__ __forceinline__ long long nbr_count(const Geom& G, const uint16_t* tab, const uint32_t* dtab,
                                               const CountCtx& x, int r)
{
    int one = 0, two = 0;
    for (int dl = 1; dl <= x.lo; ++dl) two += frame_count<DISK>(G, x, hw_at(G, tab, r, dl), dtab);
    for (int dl = x.lo + 1; dl <= x.hi; ++dl) one += frame_count<DISK>(G, x, hw_at(G, tab, r, dl), dtab);
    return (long long)frame_count<DISK>(G, x, hw_at(G, tab, r, 0), dtab) + 2ll * two + one;
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
__device__ __forceinline__ int find_radius(const Geom& G, const uint16_t* tab, const uint32_t* dtab, int t, int h,
                                           int w, long long bh, long long& c)
{
    const CountCtx x = count_ctx(G, t, h, w);
    int lo = 0, hi = G.r_cap;
    if (DISK && !dtab) {
        // row-by-row disk counts: the disk lies inside the square of the same
        // half-width, so its radius is at least the square's; search
        // [r_sq, 2 r_sq + 2] when that bracket reaches the budget, else the
        // rest up to r_cap
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (nbr_count<false>(G, tab, dtab, x, mid) >= bh) hi = mid; else lo = mid + 1;
        }
        const int r2 = min(G.r_cap, 2 * lo + 2);
        if (nbr_count<true>(G, tab, dtab, x, r2) >= bh) hi = r2;
        else { lo = min(r2 + 1, G.r_cap); hi = G.r_cap; }
    }
    long long c_hi = -1;                  // the count at hi, once evaluated
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const long long cm = nbr_count<DISK>(G, tab, dtab, x, mid);
        if (cm >= bh) { hi = mid; c_hi = cm; } else lo = mid + 1;
    }
    c = c_hi >= 0 ? c_hi : nbr_count<DISK>(G, tab, dtab, x, lo);
    return lo;
}

// Rows of a strip: 128 per tile, at most TRA_MAX_STRIP_TILES tiles.
constexpr int MASK_MAX_ROWS = 128 * TRA_MAX_STRIP_TILES;

// Dynamic shared memory of the mask kernel, sized from the plan so that small
// reaches keep many CTAs resident.  In order: the half-width table (uint16,
// when the plan has one), the disk-row table (uint32, when the plan has one),
// and per group u < U the column interval [lo, hi] and the disk's full-column
// bits of every (frame distance, tile row), the length of every list row
// (frame, tile row).
__host__ __device__ inline int mask_tab_bytes(int rte, int r_cap, bool tab)
{
    return tab ? ((rte + 1) * (r_cap + 1) * 2 + 15) & ~15 : 0;
}
__host__ __device__ inline int mask_disk_bytes(int disk_smax)
{
    return disk_smax >= 0 ? ((disk_smax + 1) * (disk_smax + 2) / 2 * 4 + 15) & ~15 : 0;
}
__host__ __device__ inline int mask_smem_bytes(int rte, int nTh, int r_cap, bool tab, int disk_smax, int U)
{
    return mask_tab_bytes(rte, r_cap, tab) + mask_disk_bytes(disk_smax) +
           U * (3 * (rte + 1) * nTh + (2 * rte + 1) * nTh) * 4;
}

// MAXT: the block size the instance is built for (128 * U); the register
// budget follows from it (three strips of three tiles per SM, or eight tiles)
template <bool DISK, bool QS, int MAXT>
__global__ void __launch_bounds__(MAXT, MAXT == 128 ? 8 : (MAXT == 384 ? 3 : 2)) radius_mask_kernel(const Geom G, const float* __restrict__ Hent,
                                                                    uint8_t* __restrict__ mask)
{
    extern __shared__ __align__(16) uint8_t mask_dyn[];
    const int U = QS ? G.nTh : 1;                                 // tiles (and groups) of this CTA
    const int RS = G.nTh;                                         // stride of one frame distance
    const uint16_t* tab = G.hw_tab ? reinterpret_cast<const uint16_t*>(mask_dyn) : nullptr;
    const int tab_bytes = mask_tab_bytes(G.rte, G.r_cap, G.hw_tab != 0);
    const uint32_t* dtab = DISK && G.disk_smax >= 0 ? reinterpret_cast<const uint32_t*>(mask_dyn + tab_bytes) : nullptr;
    int* grp_base = reinterpret_cast<int*>(mask_dyn + tab_bytes + (DISK ? mask_disk_bytes(G.disk_smax) : 0));
    const int GS = 3 * (G.rte + 1) * RS + (2 * G.rte + 1) * RS;   // ints per group
    constexpr int QR = QS ? MASK_MAX_ROWS : 1;
    __shared__ int s_key[QR];                  // QS: warp-sorted keys (radius + 1) << 10 | strip row
    __shared__ int s_order[QR];                // QS: strip rows in group order
    __shared__ int s_rad[QR];                  // QS: radius of every strip row
    __shared__ long long s_cnt[QR];            // QS: its count c(r)
    __shared__ int s_full[TRA_MAX_STRIP_TILES][TRA_MAX_RT_EFF + 1][4];
    __shared__ long long s_pairs[MASK_MAX_ROWS / 32];
    __shared__ int s_warp[MASK_MAX_ROWS / 32];

    const int g = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int u = tid >> 7, i = tid & 127;                        // group (warpgroup) and slot
    // the strip: frame t, tile column tc (QS); or tile blockIdx.x
    int t, tr0, tc;
    if (QS) {
        t = blockIdx.x / G.nTw;
        tc = blockIdx.x - t * G.nTw;
        tr0 = 0;
    } else {
        tile_coords(G, blockIdx.x, t, tr0, tc);
    }
    auto strip_tile = [&](int uu) { return (t * G.nTh + tr0 + uu) * G.nTw + tc; };

    if (tab) {
        uint16_t* wtab = reinterpret_cast<uint16_t*>(mask_dyn);
        for (int dl = 0; dl <= G.rte; ++dl)
            for (int rr = tid; rr <= G.r_cap; rr += blockDim.x)
                wtab[dl * (G.r_cap + 1) + rr] = (uint16_t)halfwidth(rr, G.g[dl]);
    }
    if (dtab) {
        // one disk row per thread: half-widths and their running sum
        uint32_t* wd = reinterpret_cast<uint32_t*>(mask_dyn + tab_bytes);
        for (int sd = tid; sd <= G.disk_smax; sd += blockDim.x) {
            uint32_t* row = wd + (sd * (sd + 1) >> 1);
            int acc = 0;
            for (int k = 0; k <= sd; ++k) {
                const int f = isqrt_floor(sd * sd - k * k);
                acc += f;
                row[k] = (uint32_t)f | ((uint32_t)acc << 16);
            }
        }
    }
    int* s_lo = grp_base + u * GS;                                // [rte + 1][nTh]
    int* s_hi = s_lo + (G.rte + 1) * RS;                          // [rte + 1][nTh]
    uint32_t* s_fullbits = reinterpret_cast<uint32_t*>(s_hi + (G.rte + 1) * RS);   // disk: full tile columns
    int* s_len = reinterpret_cast<int*>(s_fullbits + (G.rte + 1) * RS);            // [(2 rte + 1) nTh]
    for (int e = i; e < (G.rte + 1) * RS; e += 128) {
        s_lo[e] = 0x7fffffff;
        s_hi[e] = -1;
        s_fullbits[e] = 0xffffffffu;
    }
    if (i < G.rte + 1) {
        s_full[u][i][0] = -0x7fffffff; s_full[u][i][1] = 0x7fffffff;
        s_full[u][i][2] = -0x7fffffff; s_full[u][i][3] = 0x7fffffff;
    }
    __syncthreads();

    // ---- budget and radius of strip row `tid` (tile u of the strip, row i)
    int h = (tr0 + u) * G.th + (i >> G.tw_log2);
    int w = tc * G.tw + (i & (G.tw - 1));
    bool valid = h < G.H && w < G.W;
    int r = -1;
    long long c = 0;
    if (valid) r = find_radius<DISK>(G, tab, dtab, t, h, w, budget_hat(G, Hent[io_row(G, g, t, h, w, strip_tile(u) * 128 + i)]), c);
    reinterpret_cast<int32_t*>(mask + G.off_radius)[(size_t)g * G.N_pad + (size_t)strip_tile(u) * 128 + i] = r;

    if constexpr (QS) {
        // ---- order the strip's rows by (radius, row), pads (radius -1) first
        s_rad[tid] = r;
        s_cnt[tid] = c;
        int key = ((r + 1) << 10) | tid;
        for (int k = 2; k <= 32; k <<= 1)
            for (int j = k >> 1; j > 0; j >>= 1) {
                const int other = __shfl_xor_sync(0xffffffffu, key, j);
                const bool up = (lane & k) == 0, low = (lane & j) == 0;
                key = (low == up) ? min(key, other) : max(key, other);
            }
        s_key[tid] = key;
        __syncthreads();
        // keys of every other warp below `key` (independent searches, unrolled)
        int rank = lane;
#pragma unroll
        for (int ow = 0; ow < MASK_MAX_ROWS / 32; ++ow) {
            if (ow >= 4 * U || ow == warp) continue;
            const int* sk = s_key + ow * 32;
            int lo = 0;
#pragma unroll
            for (int step = 16; step > 0; step >>= 1)
                if (sk[lo + step - 1] < key) lo += step;
            lo += sk[lo] < key ? 1 : 0;
            rank += lo;
        }
        s_order[rank] = key & 1023;
        __syncthreads();
        const int l = s_order[tid];                               // the strip row group u's slot i speaks for
        h = (l >> 7) * G.th + ((l & 127) >> G.tw_log2);
        w = tc * G.tw + (l & (G.tw - 1));
        valid = h < G.H && w < G.W;
        r = s_rad[l];
        c = s_cnt[l];
        reinterpret_cast<uint16_t*>(mask + G.off_group)[((size_t)g * G.nQ + strip_tile(u)) * 128 + i] = (uint16_t)l;
    }
    const int tile = strip_tile(u);                               // this group's mask slot

    // ---- retained pairs of the group
    long long cs = c;
    for (int o = 16; o > 0; o >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, o);
    if (lane == 0) s_pairs[warp] = cs;
    __syncthreads();
    if (i == 0)
        reinterpret_cast<long long*>(mask + G.off_pairs)[(size_t)g * G.nQ + tile] =
            s_pairs[4 * u] + s_pairs[4 * u + 1] + s_pairs[4 * u + 2] + s_pairs[4 * u + 3];

    // ---- per frame distance: active tile-column interval per tile row, full rectangle
    for (int dl = 0; dl <= G.rte; ++dl) {
        if (!(t + dl < G.T || t - dl >= 0)) break;    // uniform over the CTA
        int rl = 0x7fffffff, rh = -1, cl = 0, ch = -1;
        int frl = -0x7fffffff, frh = 0x7fffffff, fcl = -0x7fffffff, fch = 0x7fffffff;
        const int s = valid ? hw_at(G, tab, r, dl) : 0;
        if (valid) {
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
            atomicMax(&s_full[u][dl][0], frl); atomicMin(&s_full[u][dl][1], frh);
            atomicMax(&s_full[u][dl][2], fcl); atomicMin(&s_full[u][dl][3], fch);
        }
        // the union of the members' column intervals over key tile row tr
        auto row_union = [&](int tr) {
            const bool in = rl <= tr && tr <= rh;
            int c_lo = cl, c_hi = ch;
            if (DISK && in) {
                // the disk is widest on the tile row's key row nearest to h
                const int sc = min(s, TRA_DISK_S_CLAMP);
                const int k0 = tr * G.th, k1 = min(G.H - 1, k0 + G.th - 1);
                const int dh = h < k0 ? k0 - h : (h > k1 ? h - k1 : 0);
                const int half = isqrt_floor(sc * sc - dh * dh);
                c_lo = max(0, w - half) >> G.tw_log2;
                c_hi = min(G.W - 1, w + half) >> G.tw_log2;
            }
            const int lo = __reduce_min_sync(0xffffffffu, in ? c_lo : 0x7fffffff);
            const int hi = __reduce_max_sync(0xffffffffu, in ? c_hi : -1);
            if (lane == 0 && hi >= 0) {
                atomicMin(&s_lo[dl * RS + tr], lo);
                atomicMax(&s_hi[dl * RS + tr], hi);
            }
        };
        if constexpr (QS) {
            // a strip has at most TRA_MAX_STRIP_TILES tile rows: all of them,
            // as independent reductions
#pragma unroll
            for (int tr = 0; tr < TRA_MAX_STRIP_TILES; ++tr)
                if (tr < G.nTh) row_union(tr);
        } else {
            // a lone tile walks the warp's row range
            const int r_lo = __reduce_min_sync(0xffffffffu, rl);
            const int r_hi = __reduce_max_sync(0xffffffffu, rh);
            for (int tr = r_lo; tr <= r_hi; ++tr) row_union(tr);
        }
    }
    __syncthreads();

    // ---- disk: a listed tile is full iff, for every valid query, its valid
    // key rectangle's farthest corner lies in the disk (the disk is convex)
    if constexpr (DISK) {
        for (int dl = 0; dl <= G.rte; ++dl) {
            if (!(t + dl < G.T || t - dl >= 0)) break;
            const int s = valid ? min(hw_at(G, tab, r, dl), TRA_DISK_S_CLAMP) : 0;
            for (int tr = 0; tr < G.nTh; ++tr) {
                const int lo = s_lo[dl * RS + tr], hi = s_hi[dl * RS + tr];
                if (hi < 0) continue;
                const int k0 = tr * G.th, k1 = min(G.H - 1, k0 + G.th - 1);
                const int dh = max(abs(h - k0), abs(h - k1));
                uint32_t bits = 0;
                for (int tcol = lo; tcol <= hi; ++tcol) {
                    const int j0 = tcol * G.tw, j1 = min(G.W - 1, j0 + G.tw - 1);
                    const int dw = max(abs(w - j0), abs(w - j1));
                    const bool in = !valid || (long long)dh * dh + (long long)dw * dw <= (long long)s * s;
                    if (__all_sync(0xffffffffu, in)) bits |= 1u << tcol;
                }
                if (lane == 0) atomicAnd(&s_fullbits[dl * RS + tr], bits | ~(((2u << hi) - 1u) ^ ((1u << lo) - 1u)));
            }
        }
        __syncthreads();
    }

    // ---- list rows (frame, tile row) in ascending tile order; prefix sum over the group
    const int t0 = max(0, t - G.rte), t1 = min(G.T - 1, t + G.rte);
    const int R = (t1 - t0 + 1) * G.nTh;
    for (int e = i; e < R; e += 128) {
        const int f = e / G.nTh, tr = e - f * G.nTh;
        const int dl = abs(t0 + f - t);
        s_len[e] = s_hi[dl * RS + tr] >= 0 ? s_hi[dl * RS + tr] - s_lo[dl * RS + tr] + 1 : 0;
    }
    __syncthreads();
    const int per = (R + 127) >> 7;
    const int beg = min(R, i * per), end = min(R, beg + per);
    int local = 0;
    for (int e = beg; e < end; ++e) local += s_len[e];
    int incl = local;
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int off = incl - local;
    for (int k = 4 * u; k < warp; ++k) off += s_warp[k];
    uint16_t* list = reinterpret_cast<uint16_t*>(mask + G.off_list) + ((size_t)g * G.nQ + tile) * G.list_cap;
    for (int e = beg; e < end; ++e) {
        const int f = e / G.nTh, tr = e - f * G.nTh;
        const int dl = abs(t0 + f - t);
        const int lo = s_lo[dl * RS + tr], hi = s_hi[dl * RS + tr];
        const bool row_full = s_full[u][dl][0] <= tr && tr <= s_full[u][dl][1];
        const uint32_t fbits = s_fullbits[dl * RS + tr];
        const int base = ((t0 + f) * G.nTh + tr) * G.nTw;
        for (int tcol = lo; tcol <= hi; ++tcol) {
            const bool full = DISK ? ((fbits >> tcol) & 1u) != 0
                                   : (row_full && s_full[u][dl][2] <= tcol && tcol <= s_full[u][dl][3]);
            list[off++] = (uint16_t)((base + tcol) | (full ? 0x8000 : 0));
        }
    }
    if (i == 0)
        reinterpret_cast<int32_t*>(mask + G.off_count)[(size_t)g * G.nQ + tile] =
            s_warp[4 * u] + s_warp[4 * u + 1] + s_warp[4 * u + 2] + s_warp[4 * u + 3];
}

}  // namespace tra
