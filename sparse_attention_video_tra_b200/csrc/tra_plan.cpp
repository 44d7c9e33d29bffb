// tra_plan.cpp -- host side of a plan: argument validation, the tile shape,
// the decay table, r_cap, the mask-buffer layout and the kernel parameter
// block.  No CUDA call is made here, so plans can be built without a GPU.
//
// Compiled with -ffp-contract=off: r * g and + 1e-9 stay two rounded
// operations, as on the device.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>

#include "../../include/tra.h"
#include "tra_geom.h"
#include "tra_plan_impl.h"

namespace {

int ilog2(int v)
{
    int l = 0;
    while ((1 << l) < v) ++l;
    return l;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// floor(r * g + 1e-9), product and sum rounded separately (host copy of the
// device half-width; both follow the same definition)
long long host_halfwidth(long long r, double g)
{
    volatile double p = (double)r * g;
    volatile double s = p + 1e-9;
    return (long long)std::floor(s);
}

}  // namespace

extern "C" tra_status tra_plan_create(tra_plan* out, int T, int H, int W, int heads, int d,
                                      double a, double b, double gamma, int Rt, int Bmin, unsigned flags)
{
    if (!out) return TRA_ERR_INVALID_ARG;
    *out = nullptr;
    if (T < 1 || H < 1 || W < 1 || heads < 1) return TRA_ERR_INVALID_ARG;
    if (!std::isfinite(a) || !std::isfinite(b)) return TRA_ERR_INVALID_ARG;
    if (!(gamma > 0.0 && gamma <= 1.0)) return TRA_ERR_INVALID_ARG;
    if (Rt < 0) return TRA_ERR_INVALID_ARG;
    const long long N = (long long)T * H * W;
    if (Bmin < 1 || (long long)Bmin > N) return TRA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return TRA_ERR_UNSUPPORTED;
    if (flags & ~(TRA_FLAG_TILE_W_MASK | TRA_FLAG_DEBUG_NO_WAIT | TRA_FLAG_OUT_BF16 | TRA_FLAG_NATURAL |
                  TRA_FLAG_DISK | TRA_FLAG_QSORT))
        return TRA_ERR_INVALID_ARG;

    if (H > TRA_MAX_HW || W > TRA_MAX_HW) return TRA_ERR_UNSUPPORTED;
    const int rte = Rt < T - 1 ? Rt : T - 1;
    if (rte > TRA_MAX_RT_EFF) return TRA_ERR_UNSUPPORTED;

    // tile shape: (1, 128/tw, tw), tw in {4, 8, 16, 32}; the least padding wins.
    // On a tie the tile's long side runs along the frame's short side (the
    // taller tile when H <= W): neighbourhoods span the short side first, so
    // the union of a tile's 128 neighbourhoods grows less along it (measured at
    // 45 x 80: 16 x 8 tiles compute 4 % fewer tile pairs than 8 x 16 ones and
    // run 9 % faster).  At most 32 tile columns per frame.
    const int forced = (int)((flags & TRA_FLAG_TILE_W_MASK) >> 8);
    if (forced && forced != 4 && forced != 8 && forced != 16 && forced != 32) return TRA_ERR_INVALID_ARG;
    int best_tw = 0;
    long long best_pad = 0;
    for (int tw = 4; tw <= 32; tw *= 2) {
        if (forced && tw != forced) continue;
        const int th = 128 / tw;
        const long long nTh = (H + th - 1) / th, nTw = (W + tw - 1) / tw;
        if (nTw > 32 || nTh > TRA_MAX_TILES_H) continue;
        const long long pad = nTh * nTw * 128;
        if (best_tw == 0 || pad < best_pad || (pad == best_pad && (H <= W ? tw < best_tw : tw > best_tw))) {
            best_tw = tw;
            best_pad = pad;
        }
    }
    if (best_tw == 0) return TRA_ERR_UNSUPPORTED;

    tra::Geom G;
    std::memset(&G, 0, sizeof G);
    G.T = T; G.H = H; G.W = W; G.G = heads; G.D = d;
    G.tw = best_tw; G.th = 128 / best_tw;
    G.tw_log2 = ilog2(G.tw); G.th_log2 = ilog2(G.th);
    G.nTh = (H + G.th - 1) / G.th;
    G.nTw = (W + G.tw - 1) / G.tw;
    G.tiles_per_frame = G.nTh * G.nTw;
    const long long nQ = (long long)T * G.tiles_per_frame;
    if (nQ > 32767) return TRA_ERR_UNSUPPORTED;               // uint16 tile ids, bit 15 = full
    G.nQ = (int)nQ;
    const long long N_pad = nQ * 128;
    if (N_pad * heads > (1ll << 31) - 1) return TRA_ERR_UNSUPPORTED;  // 32-bit TMA row coordinates
    G.N = (int)N;
    G.N_pad = (int)N_pad;
    G.rte = rte;
    if ((2 * rte + 1) * G.nTh > TRA_MAX_LIST_ROWS) return TRA_ERR_UNSUPPORTED;
    G.list_cap = (2 * rte + 1) * G.tiles_per_frame;
    if (G.list_cap > TRA_MAX_LIST_CAP) return TRA_ERR_UNSUPPORTED;
    for (int k = 0; k <= rte; ++k) G.g[k] = std::pow(gamma, (double)k);

    // r_cap: the smallest r whose farthest-frame half-width s(r, Rt') reaches
    // every key of a frame from every query: s >= max(H, W) - 1 for the
    // Chebyshev square, s >= ceil(sqrt((H-1)^2 + (W-1)^2)) for the disk
    const bool disk = (flags & TRA_FLAG_DISK) != 0;
    long long need = (H > W ? H : W) - 1;
    if (disk) {
        const long long d2 = (long long)(H - 1) * (H - 1) + (long long)(W - 1) * (W - 1);
        need = 0;
        while (need * need < d2) ++need;
    }
    const double gl = G.g[rte];
    if ((double)need / gl > (double)TRA_MAX_R_CAP) return TRA_ERR_UNSUPPORTED;
    long long r = (long long)((double)need / gl) - 2;
    if (r < 0) r = 0;
    while (r > 0 && host_halfwidth(r - 1, gl) >= need) --r;
    while (host_halfwidth(r, gl) < need) {
        ++r;
        if (r >= TRA_MAX_R_CAP) return TRA_ERR_UNSUPPORTED;
    }
    G.r_cap = (int)r;
    G.disk = disk ? 1 : 0;
    // a disk of half-width >= need covers the frame, so the mask kernel's
    // disk-row table needs the half-widths 0 .. need only
    G.disk_smax = disk && (need + 1) * (need + 2) / 2 <= TRA_MAX_DISK_TAB ? (int)need : -1;

    G.a = a; G.b = b; G.Bmin = Bmin;
    G.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d));
    G.wait_ns = (flags & TRA_FLAG_DEBUG_NO_WAIT) ? 0ull : 2000000000ull;
    G.natural = (flags & TRA_FLAG_NATURAL) ? 1 : 0;
    // radius-sorted groups sort the rows of a tile-column strip (one tile
    // column of one frame, nTh tiles) in one CTA of 128 * nTh threads
    G.qsort = (flags & TRA_FLAG_QSORT) ? 1 : 0;
    if (G.qsort && G.nTh > TRA_MAX_STRIP_TILES) return TRA_ERR_UNSUPPORTED;
    G.hw_tab = (long long)(rte + 1) * (G.r_cap + 1) <= TRA_MAX_HW_TAB ? 1 : 0;
    G.drain_ns = 2000000000ull;

    // mask buffer layout
    size_t off = 0;
    G.off_radius = (long long)off;  off = align256(off + sizeof(int) * (size_t)heads * N_pad);
    G.off_count = (long long)off;   off = align256(off + sizeof(int) * (size_t)heads * nQ);
    G.off_pairs = (long long)off;   off = align256(off + sizeof(long long) * (size_t)heads * nQ);
    G.off_list = (long long)off;    off = align256(off + sizeof(uint16_t) * (size_t)heads * nQ * G.list_cap);
    G.off_group = 0;
    if (G.qsort) { G.off_group = (long long)off; off = align256(off + sizeof(uint16_t) * (size_t)heads * nQ * 128); }

    tra_plan_s* p = new (std::nothrow) tra_plan_s;
    if (!p) return TRA_ERR_INVALID_ARG;
    p->geom = G;
    p->gamma = gamma;
    p->Rt = Rt;
    p->flags = flags;
    p->mask_bytes = off;
    *out = p;
    return TRA_OK;
}

extern "C" void tra_plan_destroy(tra_plan plan) { delete plan; }

extern "C" tra_status tra_plan_query(tra_plan plan, tra_plan_info* info)
{
    if (!plan || !info) return TRA_ERR_INVALID_ARG;
    const tra::Geom& G = plan->geom;
    std::memset(info, 0, sizeof *info);
    info->T = G.T; info->H = G.H; info->W = G.W; info->heads = G.G; info->d = G.D;
    info->N = G.N; info->N_pad = G.N_pad;
    info->tile_h = G.th; info->tile_w = G.tw;
    info->n_tiles_h = G.nTh; info->n_tiles_w = G.nTw; info->n_tiles = G.nQ;
    info->rt_eff = G.rte; info->r_cap = G.r_cap; info->list_cap = G.list_cap;
    info->mask_bytes = plan->mask_bytes;
    info->off_radius = (size_t)G.off_radius;
    info->off_tile_count = (size_t)G.off_count;
    info->off_tile_pairs = (size_t)G.off_pairs;
    info->off_list = (size_t)G.off_list;
    info->off_group = (size_t)G.off_group;
    return TRA_OK;
}

// Least squares of ln k on H in one pass over the rows (running means and
// co-moments, updated row by row so no second pass or large sums are needed):
// with dx = x - mean_x before the row and mean_y after it,
// C_xx += dx * (x - mean_x'), C_xy += dx * (y - mean_y').
extern "C" tra_status tra_calibrate_fit(const float* H, const int32_t* k, long long n, double* a, double* b,
                                        long long* rows_used)
{
    if (!H || !k || !a || !b || n < 0) return TRA_ERR_INVALID_ARG;
    long long m = 0;
    double mean_x = 0.0, mean_y = 0.0, cxx = 0.0, cxy = 0.0;
    for (long long i = 0; i < n; ++i) {
        const double x = (double)H[i];
        if (k[i] < 1 || !std::isfinite(x)) continue;
        const double y = std::log((double)k[i]);
        ++m;
        const double dx = x - mean_x;
        mean_x += dx / (double)m;
        mean_y += (y - mean_y) / (double)m;
        cxx += dx * (x - mean_x);
        cxy += dx * (y - mean_y);
    }
    if (rows_used) *rows_used = m;
    if (m < 2 || !(cxx > 0.0)) return TRA_ERR_INVALID_ARG;
    *a = cxy / cxx;
    *b = mean_y - *a * mean_x;
    return TRA_OK;
}

extern "C" const char* tra_status_string(tra_status s)
{
    switch (s) {
        case TRA_OK: return "ok";
        case TRA_ERR_INVALID_ARG: return "invalid argument";
        case TRA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
        case TRA_ERR_WORKSPACE: return "mask buffer too small";
        case TRA_ERR_CUDA: return "CUDA call failed";
        case TRA_ERR_TIMEOUT: return "a kernel wait gave up (timeout)";
        case TRA_ERR_DEVICE_CHECK: return "a kernel index check failed";
    }
    return "unknown status";
}
