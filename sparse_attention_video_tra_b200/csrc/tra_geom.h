// tra_geom.h -- the plan as seen by the kernels: plain data, passed by value
// to every launch.  Built on the host by the plan code (tra_plan.cpp).
#pragma once
#include <cstdint>

#define TRA_MAX_RT_EFF 31            // decay table holds gamma^0 .. gamma^31
#define TRA_MAX_TILES_H 64           // tile rows per frame the mask kernel handles
#define TRA_MAX_LIST_ROWS 4096       // (2Rt'+1) * tile rows per frame
#define TRA_MAX_R_CAP (1 << 20)
#define TRA_MAX_LIST_CAP 2048         // key tiles listed per query tile
#define TRA_MAX_HW 256                // largest H and W (half-widths kept as bytes)
#define TRA_MAX_STRIP_TILES 4         // tile rows per frame with radius-sorted query groups
#define TRA_MAX_HW_TAB 8192           // half-width table entries (Rt'+1)(r_cap+1) kept in shared memory
#define TRA_MAX_DISK_TAB 12288        // disk row half-width / running-sum entries (S+1)(S+2)/2 kept in shared memory
#define TRA_ERRBIT_TIMEOUT 1u
#define TRA_ERRBIT_CHECK 2u

namespace tra {

struct Geom {
    int T, H, W, G, D;               // grid, heads, head dim
    int N, N_pad;                    // tokens per head, tile-major rows per head
    int th, tw, th_log2, tw_log2;    // (1, th, tw) tiles, th*tw = 128
    int nTh, nTw, tiles_per_frame, nQ;
    int rte, r_cap, list_cap;
    int Bmin;
    double a, b;
    double g[TRA_MAX_RT_EFF + 1];    // gamma^delta
    long long off_radius, off_count, off_pairs, off_list, off_group;
    float scale_log2;                // log2(e) / sqrt(d)
    unsigned long long wait_ns;      // limit of a pipeline wait
    unsigned long long drain_ns;     // limit of the waits that drain in-flight copies
    int natural;                     // q/k/v/out/entropies in natural token order (4-D TMA boxes)
    int disk;                        // spatial test dh^2 + dw^2 <= s^2 instead of the Chebyshev square
    int qsort;                       // radius-sorted query groups of tile-column strips
    int hw_tab;                      // the mask kernel tabulates s(r, |dt|) for r <= r_cap
    int disk_smax;                   // disk: the mask kernel tabulates the disk rows of half-widths
                                     // 0 .. disk_smax (the frame's cover radius); -1: no table
};

}  // namespace tra
