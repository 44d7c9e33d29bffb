// entropy.cuh -- per-query softmax entropy of the warm-up attention, on the
// sm_100a tensor cores (tcgen05 + TMEM), K tiles staged by TMA.
//
// "Token Radius Attention for Efficient Video Generation" (gist.science
// summary), section 2, "Entropie-vers-Budget": a dense warm-up step measures
// every query's attention entropy, which later steps reuse; the daily-ai-
// frontier TL;DR of the same paper calls it fused entropy extraction.
//
// With u_j = (q.k_j / sqrt d) * log2(e) and a running maximum m, the kernel
// keeps Z = sum_j 2^(u_j - m) and A = sum_j 2^(u_j - m) (u_j - m); then
//   H = -sum_j p_j ln p_j = ln Z - ln(2) * A / Z.
// When m grows to m': A <- 2^(m-m') (A + (m - m') Z), Z <- 2^(m-m') Z.
// Key subsampling (key_tile_stride s > 1) visits the key tiles whose index is
// a multiple of s and adds ln(N / |S|) (host-computed) so that a uniform
// distribution still reads ln N.
//
// One CTA per pair of query tiles (A = 2p, B = 2p+1) of one head; every K tile
// is loaded once and multiplied with both.  352 threads:
//   warps 0-3 statistics of tile A, warps 4-7 of tile B (thread r = query row
//   r = TMEM lane r); warp 8 TMA producer (Q_A, Q_B, then the K ring); warps 9
//   and 10 MMA issuers for tiles A and B (warp 9 also allocates TMEM):
//   S_w[j%2] = Q_w K_j^T, two 128-column fp32 buffers per query tile.
// TMEM columns: S_A[0] [0,128), S_A[1] [128,256), S_B[0] [256,384), S_B[1] [384,512).
#pragma once
#include "pipeline.cuh"

namespace tra {

template <int D>
struct EntCfg {
    static constexpr int PANEL = 128 * 128;
    static constexpr int NP = D / 64;
    static constexpr int TILE = NP * PANEL;
    static constexpr int KST = (D == 128) ? 4 : 8;
    static constexpr int OFF_Q = 0;                     // Q_A, Q_B
    static constexpr int OFF_K = 2 * TILE;
    static constexpr int OFF_BAR = OFF_K + KST * TILE;
    static constexpr int NBAR = 1 + 2 * KST + 8 + 2;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static constexpr int THREADS = 352;
    static constexpr int WARP_LOAD = 8, WARP_MMA = 9;     // MMA issuers: warps 9 (tile A), 10 (tile B)
};

// One key tile's contribution to a query row's online entropy statistics in
// the log2 domain: m = running maximum of s*c, Z = sum 2^(s*c - m), A = sum
// 2^(s*c - m) * (s*c - m); the entropy is then ln Z - ln2 * A / Z.  v holds the
// row's 128 raw scores s of the tile; pad keys of edge tiles are dropped.
template <int TWL>
__device__ __forceinline__ void ent_tile_update(uint32_t (&v)[4][32], bool edge, int khv, int kwv, float c,
                                                float& m, float& Z, float& A)
{
    if (edge) {                     // pad keys of edge tiles take no probability
        uint32_t keep[4];
        row_keep_bits<TWL>(0, khv - 1, 0, kwv - 1, keep);
#pragma unroll
        for (int i = 0; i < 128; ++i)
            if (!(keep[i >> 5] & (1u << (i & 31)))) v[i >> 5][i & 31] = __float_as_uint(-1e30f);
    }
    // four independent max chains, then combine
    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < 64; ++i)
        m4[i & 3] = max3(m4[i & 3], __uint_as_float(v[i >> 4][(2 * i) & 31]), __uint_as_float(v[i >> 4][(2 * i + 1) & 31]));
    const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * c;
    if (mt > m) {
        const float alpha = ex2(m - mt);
        A = alpha * fmaf(m - mt, Z, A);
        Z *= alpha;
        m = mt;
    }
    // u = s*c - m (<= 0), e = 2^u; Z += e, A += e*u, all in packed pairs;
    // four independent accumulator chains
    const f2_t c2 = f2_pack(c, c), nm2 = f2_pack(-m, -m);
    f2_t z2[4] = {0ull, 0ull, 0ull, 0ull}, a2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const f2_t u2 = f2_fma(f2_pack(__uint_as_float(v[i >> 4][(2 * i) & 31]),
                                       __uint_as_float(v[i >> 4][(2 * i + 1) & 31])), c2, nm2);
        float u0, u1;
        f2_unpack(u2, u0, u1);
        const f2_t e2 = f2_pack(ex2(u0), ex2(u1));
        z2[i & 3] = f2_add(z2[i & 3], e2);
        a2[i & 3] = f2_fma(e2, u2, a2[i & 3]);
    }
    const f2_t zs = f2_add(f2_add(z2[0], z2[1]), f2_add(z2[2], z2[3]));
    const f2_t as = f2_add(f2_add(a2[0], a2[1]), f2_add(a2[2], a2[3]));
    float zl, zh, al, ah;
    f2_unpack(zs, zl, zh);
    f2_unpack(as, al, ah);
    Z += zl + zh;
    A += al + ah;
}

template <int D, int TWL>
__global__ void __launch_bounds__(352, 1)
entropy_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const Geom G, int stride, float corr, float* __restrict__ Hout)
{
    using C = EntCfg<D>;
    constexpr int TW = 1 << TWL;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* sK = smem + C::OFF_K;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + C::KST;
    uint64_t* s_full = k_empty + C::KST;     // [w * 2 + buffer]
    uint64_t* s_empty = s_full + 4;          // [w * 2 + buffer]
    uint64_t* drain = s_empty + 4;           // [2]
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    int* s_lock = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);

    const int pair = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qa = 2 * pair, qb = 2 * pair + 1;
    const bool hasB = qb < G.nQ;
    const int n = (G.nQ + stride - 1) / stride;              // key tiles visited

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < C::KST; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 2); }
        for (int i = 0; i < 4; ++i) { mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 128); }
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        *s_abort = 0;
        *s_lock = 0;
        fence_barrier_init();
    }
    if (warp == C::WARP_MMA) { tmem_alloc(s_tmem, 512); tmem_relinquish(); }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == C::WARP_LOAD) {
        if (lane == 0) {
            prefetch_tmap(&tm_q); prefetch_tmap(&tm_k);
            mbar_arrive_expect_tx(q_full, C::TILE * (hasB ? 2 : 1));
            int ta, tra_, tca, tb, trb, tcb;
            tile_coords(G, qa, ta, tra_, tca);
            tile_coords(G, hasB ? qb : qa, tb, trb, tcb);
#pragma unroll
            for (int p = 0; p < C::NP; ++p) {
                load_tile_panel(sQ + p * C::PANEL, &tm_q, G, p, g, ta, tra_, tca, q_full);
                if (hasB) load_tile_panel(sQ + C::TILE + p * C::PANEL, &tm_q, G, p, g, tb, trb, tcb, q_full);
            }
            int issued = 0;
            for (int j = 0; j < n; ++j) {
                const int st = j % C::KST;
                if (j >= C::KST && !role_wait(&k_empty[st], ((j / C::KST) - 1) & 1, G.wait_ns, s_abort)) break;
                mbar_arrive_expect_tx(&k_full[st], C::TILE);
                int tk, trk, tck;
                tile_coords(G, j * stride, tk, trk, tck);
#pragma unroll
                for (int p = 0; p < C::NP; ++p)
                    load_tile_panel(sK + st * C::TILE + p * C::PANEL, &tm_k, G, p, g, tk, trk, tck, &k_full[st]);
                ++issued;
            }
            mbar_wait(q_full, 0, G.drain_ns);
            for (int j = max(0, issued - C::KST); j < issued; ++j)
                mbar_wait(&k_full[j % C::KST], (j / C::KST) & 1, G.drain_ns);
        }
    } else if (warp >= C::WARP_MMA) {
        // One MMA issuer per query tile (issuing tcgen05.mma occupies the thread
        // about as long as the tensor core runs it): S_w[j%2] = Q_w K_j^T once
        // K_j has landed and the softmax of tile j-2 has released that buffer.
        // Each issuer's commit is one of the two arrivals that free a K stage.
        const int w = warp - C::WARP_MMA;
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, false);
            const uint32_t sQa = smem_u32(sQ) + w * C::TILE, sKa = smem_u32(sK);
            const bool active = w == 0 || hasB;
            bool ok = role_wait(q_full, 0, G.wait_ns, s_abort);
            for (int j = 0; ok && j < n; ++j) {
                const int ks = j % C::KST, b = j & 1;
                if (!role_wait(&k_full[ks], (j / C::KST) & 1, G.wait_ns, s_abort)) break;
                if (!active) { mbar_arrive(&k_empty[ks]); continue; }
                if (j >= 2 && !role_wait(&s_empty[w * 2 + b], ((j - 2) >> 1) & 1, G.wait_ns, s_abort)) break;
                if (!issue_lock(s_lock, G.wait_ns, s_abort)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::PANEL + (kk & 3) * 32;
                    mma_ss(tmem + (w * 2 + b) * 128, smem_desc_sw128(sQa + off, 16, 1024),
                           smem_desc_sw128(sKa + ks * C::TILE + off, 16, 1024), IDESC, kk > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[w * 2 + b]);
                mma_commit(&k_empty[ks]);
                issue_unlock(s_lock);
            }
            mma_commit(&drain[w]);
            mbar_wait(&drain[w], 0, G.drain_ns);
        }
    } else {
        const int w = warp >> 2;
        const int row = tid & 127;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const float c = G.scale_log2;
        float m = -1e30f, Z = 0.f, A = 0.f;
        bool ok = w == 0 || hasB;
        // (tile row, tile column) of key tile j*stride, advanced by the stride
        // (sr, sc) = stride mod tiles-per-frame, so the loop divides nothing
        const int smod = stride % G.tiles_per_frame, sr = smod / G.nTw, sc = smod - sr * G.nTw;
        int trk = 0, tck = 0;
        for (int j = 0; ok && j < n; ++j) {
            const int khv = min(G.th, G.H - trk * G.th), kwv = min(TW, G.W - tck * TW);
            const bool edge = khv < G.th || kwv < TW;
            tck += sc;
            trk += sr;
            if (tck >= G.nTw) { tck -= G.nTw; ++trk; }
            if (trk >= G.nTh) trk -= G.nTh;
            const int bs = w * 2 + (j & 1);
            const bool got = role_wait(&s_full[bs], (j >> 1) & 1, G.wait_ns, s_abort);
            if (__any_sync(0xffffffffu, !got)) { ok = false; break; }
            tc_fence_after();
            __syncwarp();
            uint32_t v[4][32];
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_ld32(tmem + lane_base + bs * 128 + q * 32, v[q]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&s_empty[bs]);
            ent_tile_update<TWL>(v, edge, khv, kwv, c, m, Z, A);
        }
        if (ok) {
            const float H = logf(Z) - 0.69314718055994531f * (A / Z) + corr;
            const int qt = w ? qb : qa;
            int tq, trq, tcq;
            tile_coords(G, qt, tq, trq, tcq);
            const int hq = trq * G.th + (row >> TWL), wq = tcq * TW + (row & (TW - 1));
            if (!G.natural || (hq < G.H && wq < G.W)) Hout[io_row(G, g, tq, hq, wq, qt * 128 + row)] = H;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tra
