// topk.cuh -- calibration workload: per sampled query, the fewest top keys
// that hold a given share of its attention mass, with the query's entropy.
//
// "Token Radius Attention for Efficient Video Generation" (gist.science
// summary), section 2, Intuition I: the density of keys a query needs follows
// its attention entropy, B ~ tau * exp(H_i); fitting ln k_i = a * H_i + b over
// queries gives the budget's constants from data.
//
// k_i(m) = the smallest k whose k largest probabilities p_ij (dense softmax over
// all N keys) sum to at least m.  With x_j = s_ij * log2(e)/sqrt(d) - max (the
// log2-domain score, <= 0) and Z = sum_j 2^x_j, k_i is the number of keys with
// x_j >= tau*, where tau* is the largest threshold whose kept mass
// sum_{x_j >= tau} 2^x_j still reaches m * Z.  The kernel finds tau* by
// bisection: pass 0 is the entropy pass (max, Z, and H exactly as in
// tra_entropy), then every pass p >= 1 recomputes the row's scores on the
// tensor cores and measures (count, mass) at the midpoint of the row's current
// bracket [lo, hi] (lo keeps >= m*Z, hi keeps less), halving it.  After
// TOPK_PASSES - 1 halvings of [-160, 1] the bracket is below fp32 resolution,
// and k_i is the count kept at lo.
//
// One CTA per sampled query tile, 192 threads: warps 0-3 statistics (thread r
// = query row r = TMEM lane r), warp 4 TMA producer (Q once, then every key
// tile once per pass through a 5-stage ring), warp 5 MMA issuer into two S
// buffers (S_{u%2} for global key step u = pass * n + j).
#pragma once
#include "pipeline.cuh"
#include "entropy.cuh"

namespace tra {

constexpr int TOPK_PASSES = 33;          // 1 entropy pass + 32 bisection passes

template <int D>
struct TopkCfg {
    static constexpr int PANEL = 128 * 128;
    static constexpr int NP = D / 64;
    static constexpr int TILE = NP * PANEL;
    static constexpr int KST = (D == 128) ? 5 : 10;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE;
    static constexpr int OFF_BAR = OFF_K + KST * TILE;
    static constexpr int NBAR = 1 + 2 * KST + 4 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static constexpr int THREADS = 192;
    static constexpr int WARP_LOAD = 4, WARP_MMA = 5;
};

template <int D, int TWL>
__global__ void __launch_bounds__(192, 1)
topk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, const Geom G,
            int qstride, int n_sample, float mass, float* __restrict__ Hout, int* __restrict__ Kout)
{
    using C = TopkCfg<D>;
    constexpr int TW = 1 << TWL;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* sK = smem + C::OFF_K;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + C::KST;
    uint64_t* s_full = k_empty + C::KST;     // [2]
    uint64_t* s_empty = s_full + 2;          // [2]
    uint64_t* drain = s_empty + 2;           // [1]
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    const int sample = blockIdx.x, g = blockIdx.y;
    const int qt = sample * qstride;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = G.nQ;                                      // key tiles per pass (all keys)
    const long long total = (long long)TOPK_PASSES * n;      // key steps over all passes

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < C::KST; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 128); }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == C::WARP_MMA) { tmem_alloc(s_tmem, 256); tmem_relinquish(); }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == C::WARP_LOAD) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_q); prefetch_tmap(&tm_k);
            mbar_arrive_expect_tx(q_full, C::TILE);
            int tq, trq, tcq;
            tile_coords(G, qt, tq, trq, tcq);
#pragma unroll
            for (int p = 0; p < C::NP; ++p) load_tile_panel(sQ + p * C::PANEL, &tm_q, G, p, g, tq, trq, tcq, q_full);
            long long issued = 0;
            for (long long u = 0; u < total; ++u) {
                const int st = (int)(u % C::KST);
                if (u >= C::KST && !role_wait(&k_empty[st], (uint32_t)((u / C::KST) - 1) & 1, G.wait_ns, s_abort))
                    break;
                mbar_arrive_expect_tx(&k_full[st], C::TILE);
                int tk, trk, tck;
                tile_coords(G, (int)(u % n), tk, trk, tck);
#pragma unroll
                for (int p = 0; p < C::NP; ++p)
                    load_tile_panel(sK + st * C::TILE + p * C::PANEL, &tm_k, G, p, g, tk, trk, tck, &k_full[st]);
                ++issued;
            }
            mbar_wait(q_full, 0, G.drain_ns);
            for (long long u = issued > C::KST ? issued - C::KST : 0; u < issued; ++u)
                mbar_wait(&k_full[u % C::KST], (uint32_t)(u / C::KST) & 1, G.drain_ns);
        }
    } else if (warp == C::WARP_MMA) {
        // ------------------------------------------------ MMA issuer: S_{u%2} = Q K_u^T
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, false);
            const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK);
            bool ok = role_wait(q_full, 0, G.wait_ns, s_abort);
            for (long long u = 0; ok && u < total; ++u) {
                const int ks = (int)(u % C::KST), b = (int)(u & 1);
                if (!role_wait(&k_full[ks], (uint32_t)(u / C::KST) & 1, G.wait_ns, s_abort)) break;
                if (u >= 2 && !role_wait(&s_empty[b], (uint32_t)((u - 2) >> 1) & 1, G.wait_ns, s_abort)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::PANEL + (kk & 3) * 32;
                    mma_ss(tmem + b * 128, smem_desc_sw128(sQa + off, 16, 1024),
                           smem_desc_sw128(sKa + ks * C::TILE + off, 16, 1024), IDESC, kk > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[b]);
                mma_commit(&k_empty[ks]);
            }
            mma_commit(drain);
            mbar_wait(drain, 0, G.drain_ns);
        }
    } else {
        // ------------------------------------------------ statistics (warps 0-3)
        const int row = tid;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const float c = G.scale_log2;
        float m = -1e30f, Z = 0.f, A = 0.f;
        // bisection state in the x = s*c - m domain
        float lo = -160.f, hi = 1.f, mid = 0.f;
        int cnt_lo = G.N, cnt = 0;
        float kept = 0.f;
        bool ok = true;
        for (long long u = 0; ok && u < total; ++u) {
            const int pass = (int)(u / n), j = (int)(u % n);
            if (pass > 0 && j == 0) {
                // a new bisection pass: midpoint of the bracket
                mid = 0.5f * (lo + hi);
                cnt = 0;
                kept = 0.f;
            }
            int tk, trk, tck;
            tile_coords(G, j, tk, trk, tck);
            const int khv = min(G.th, G.H - trk * G.th), kwv = min(TW, G.W - tck * TW);
            const bool edge = khv < G.th || kwv < TW;
            const int b = (int)(u & 1);
            const bool got = role_wait(&s_full[b], (uint32_t)(u >> 1) & 1, G.wait_ns, s_abort);
            if (__any_sync(0xffffffffu, !got)) { ok = false; break; }
            tc_fence_after();
            __syncwarp();
            uint32_t v[4][32];
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_ld32(tmem + lane_base + b * 128 + q * 32, v[q]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&s_empty[b]);
            if (pass == 0) {
                ent_tile_update<TWL>(v, edge, khv, kwv, c, m, Z, A);
            } else {
                if (edge) {
                    uint32_t keep[4];
                    row_keep_bits<TWL>(0, khv - 1, 0, kwv - 1, keep);
#pragma unroll
                    for (int i = 0; i < 128; ++i)
                        if (!(keep[i >> 5] & (1u << (i & 31)))) v[i >> 5][i & 31] = __float_as_uint(-1e30f);
                }
                // keys with x >= mid: count them and add their 2^x
                float k4[4] = {0.f, 0.f, 0.f, 0.f};
                int c2[2] = {0, 0};
#pragma unroll
                for (int i = 0; i < 128; ++i) {
                    const float x = fmaf(__uint_as_float(v[i >> 5][i & 31]), c, -m);
                    const bool in = x >= mid;
                    k4[i & 3] += in ? ex2(x) : 0.f;
                    c2[i & 1] += in ? 1 : 0;
                }
                kept += (k4[0] + k4[1]) + (k4[2] + k4[3]);
                cnt += c2[0] + c2[1];
                if (j == n - 1) {
                    // end of a pass: keep the half of the bracket that holds tau*
                    if (kept >= mass * Z) { lo = mid; cnt_lo = cnt; }
                    else hi = mid;
                }
            }
        }
        int tq, trq, tcq;
        tile_coords(G, qt, tq, trq, tcq);
        const int hq = trq * G.th + (row >> TWL), wq = tcq * TW + (row & (TW - 1));
        const bool valid = hq < G.H && wq < G.W;
        const size_t o = ((size_t)g * n_sample + sample) * 128 + row;
        if (ok) {
            Hout[o] = valid ? logf(Z) - 0.69314718055994531f * (A / Z) : __int_as_float(0x7fc00000);
            Kout[o] = valid ? cnt_lo : -1;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace tra
