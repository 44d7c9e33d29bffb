// attention.cuh -- block-sparse attention with exact token masking on the
// sm_100a tensor cores (tcgen05 + TMEM), K/V tiles staged by TMA.
//
// "Token Radius Attention for Efficient Video Generation" (gist.science
// summary), section 2, "Execution Efficace": the radius masks become
// block-sparse masks and attention runs on the kept query-key blocks only.
// Here every listed key tile is also masked token by token (Chebyshev test
// against the query's per-frame half-width), so the result is exactly
// softmax attention under the radius mask.
//
// One CTA per (query tile of 128 tokens, head).  352 threads:
//   warps 0-7  softmax: query row r = TMEM lane r is shared by warps r/32 and
//              r/32 + 4, each taking 64 of the 128 key columns.  Reads S from
//              TMEM, masks, combines the two halves' row maxima through shared
//              memory, keeps the running max m (lazy rescale: O is rescaled
//              only when the max grows by more than 2^8), writes
//              P = 2^(S*scale - m) as bf16 into TMEM, and in the end divides O
//              by the row sum and stores the rows.
//   warp 8     TMA producer for Q and the K ring.
//   warp 9     TMA producer for the V ring.
//   warp 10    TMEM allocator and single-thread MMA issuer:
//                S[j%2] = Q K_j^T        (A, B from smem, K-major)
//                O     += P_j V_j        (A = P from TMEM, B = V from smem, MN-major)
//                L     += P_j 1          (B = a bf16 ones tile in smem)
//              so the row sum L is the fp32 sum of exactly the bf16 P values
//              the tensor core multiplied, and O / L is their weighted mean.
// TMEM columns: S0 [0,128), S1 [128,256), O [256,256+D), P [384,448), L [448,464).
#pragma once
#include "pipeline.cuh"

namespace tra {

template <int D>
struct AttnCfg {
    static constexpr int PANEL = 128 * 128;                 // one 64-column panel of 128 rows, bytes
    static constexpr int NP = D / 64;                       // panels per 128-row tile
    static constexpr int TILE = NP * PANEL;                 // bytes of a 128 x D bf16 tile
    static constexpr int KST = (D == 128) ? 3 : 4;          // K ring depth
    static constexpr int VST = (D == 128) ? 2 : 3;          // V ring depth
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE;
    static constexpr int OFF_V = OFF_K + KST * TILE;
    static constexpr int OFF_ONES = OFF_V + VST * TILE;     // 16 x 64 bf16 ones (2 KB)
    static constexpr int OFF_LIST = OFF_ONES + 2048;        // decoded key tiles, uint32 [LIST_CAP]
    static constexpr int OFF_RED = OFF_LIST + TRA_MAX_LIST_CAP * 4;   // row-max exchange [2][2][128] f32
    static constexpr int OFF_BAR = OFF_RED + 2 * 2 * 128 * 4;
    static constexpr int NBAR = 1 + 2 * KST + 2 * VST + 2 + 2 + 1 + 1 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;       // + alignment slack
    static constexpr int SOFTMAX_WARPS = 8;                 // two per TMEM lane quarter
    static constexpr int WARP_K = 8, WARP_V = 9, WARP_MMA = 10;
    static constexpr int THREADS = 352;
    static constexpr uint32_t COL_S = 0, COL_O = 256, COL_P = 384, COL_L = 448;
    // exp2 of the P pairs with (pair % POLY_MOD) == POLY_MOD - 1 runs on the FMA
    // pipe, the rest on the MUFU unit
    static constexpr int POLY_MOD = 3;
};

// A listed key tile decoded once per CTA: frame (15 bits), tile row (6),
// tile column (5), full flag (bit 31).
__device__ __forceinline__ uint32_t pack_tile(int t, int tr, int tc, bool full)
{
    return (uint32_t)t | ((uint32_t)tr << 15) | ((uint32_t)tc << 21) | (full ? 0x80000000u : 0u);
}

__device__ __forceinline__ void named_bar(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <int D, int TWL, bool OUT_BF16>
__global__ void __launch_bounds__(352, 1)
attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const Geom G, const uint8_t* __restrict__ mask,
                 void* __restrict__ out)
{
    using C = AttnCfg<D>;
    constexpr int TW = 1 << TWL;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* sK = smem + C::OFF_K;
    uint8_t* sV = smem + C::OFF_V;
    uint32_t* sOnes = reinterpret_cast<uint32_t*>(smem + C::OFF_ONES);
    uint32_t* list = reinterpret_cast<uint32_t*>(smem + C::OFF_LIST);
    float* s_red = reinterpret_cast<float*>(smem + C::OFF_RED);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + C::KST;
    uint64_t* v_full = k_empty + C::KST;
    uint64_t* v_empty = v_full + C::VST;
    uint64_t* s_full = v_empty + C::VST;
    uint64_t* s_empty = s_full + 2;
    uint64_t* p_full = s_empty + 2;
    uint64_t* pv_done = p_full + 1;
    uint64_t* drain = pv_done + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    const int tile = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = reinterpret_cast<const int32_t*>(mask + G.off_count)[(size_t)g * G.nQ + tile];
    const uint16_t* glist = reinterpret_cast<const uint16_t*>(mask + G.off_list) + ((size_t)g * G.nQ + tile) * G.list_cap;
    for (int i = tid; i < n; i += C::THREADS) {
        const int e = glist[i];
        int tk, trk, tck;
        tile_coords(G, e & 0x7fff, tk, trk, tck);
        list[i] = pack_tile(tk, trk, tck, (e & 0x8000) != 0);
    }
    for (int i = tid; i < 512; i += C::THREADS) sOnes[i] = 0x3F803F80u;    // bf16 1.0 pairs
    fence_proxy_async_smem();                                              // visible to the tensor core
    const int row0 = g * G.N_pad + tile * 128;               // first tile-major row of this tile

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < C::KST; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
        for (int i = 0; i < C::VST; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 32 * C::SOFTMAX_WARPS); }
        mbar_init(p_full, 32 * C::SOFTMAX_WARPS);
        mbar_init(pv_done, 1);
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == C::WARP_MMA) { tmem_alloc(s_tmem, 512); tmem_relinquish(); }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const int kbase = g * G.N_pad;
    auto key_row = [&](int j) {
        const uint32_t e = list[j];
        return kbase + (((int)(e & 0x7fff) * G.nTh + (int)((e >> 15) & 63)) * G.nTw + (int)((e >> 21) & 31)) * 128;
    };

    if (warp == C::WARP_K) {
        // ------------------------------------------------ Q + K producer
        if (lane == 0 && n > 0) {
            prefetch_tmap(&tm_q); prefetch_tmap(&tm_k);
            mbar_arrive_expect_tx(q_full, C::TILE);
#pragma unroll
            for (int p = 0; p < C::NP; ++p) tma_load_2d(sQ + p * C::PANEL, &tm_q, p * 64, row0, q_full);
            int issued = 0;
            for (int j = 0; j < n; ++j) {
                const int st = j % C::KST;
                if (j >= C::KST && !role_wait(&k_empty[st], ((j / C::KST) - 1) & 1, G.wait_ns, s_abort)) break;
                const int y = key_row(j);
                mbar_arrive_expect_tx(&k_full[st], C::TILE);
#pragma unroll
                for (int p = 0; p < C::NP; ++p)
                    tma_load_2d(sK + st * C::TILE + p * C::PANEL, &tm_k, p * 64, y, &k_full[st]);
                ++issued;
            }
            // copies still in flight must land before the CTA exits
            mbar_wait(q_full, 0, G.drain_ns);
            for (int j = max(0, issued - C::KST); j < issued; ++j)
                mbar_wait(&k_full[j % C::KST], (j / C::KST) & 1, G.drain_ns);
        }
    } else if (warp == C::WARP_V) {
        // ------------------------------------------------ V producer
        if (lane == 0 && n > 0) {
            prefetch_tmap(&tm_v);
            int issued = 0;
            for (int j = 0; j < n; ++j) {
                const int st = j % C::VST;
                if (j >= C::VST && !role_wait(&v_empty[st], ((j / C::VST) - 1) & 1, G.wait_ns, s_abort)) break;
                const int y = key_row(j);
                mbar_arrive_expect_tx(&v_full[st], C::TILE);
#pragma unroll
                for (int p = 0; p < C::NP; ++p)
                    tma_load_2d(sV + st * C::TILE + p * C::PANEL, &tm_v, p * 64, y, &v_full[st]);
                ++issued;
            }
            for (int j = max(0, issued - C::VST); j < issued; ++j)
                mbar_wait(&v_full[j % C::VST], (j / C::VST) & 1, G.drain_ns);
        }
    } else if (warp == C::WARP_MMA) {
        // ------------------------------------------------ MMA issuer
        // order: QK_0, then for each j: QK_{j+1} (as soon as its S buffer is
        // free), PV_j (once P_j is written), so S is ready ahead of the softmax
        if (lane == 0 && n > 0) {
            constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false);
            constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
            constexpr uint32_t IDESC_L = idesc_bf16_f32(128, 16, false);
            const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV), sOa = smem_u32(sOnes);
            auto issue_qk = [&](int j) -> bool {
                const int ks = j % C::KST;
                if (!role_wait(&k_full[ks], (j / C::KST) & 1, G.wait_ns, s_abort)) return false;
                if (j >= 2 && !role_wait(&s_empty[j & 1], ((j - 2) >> 1) & 1, G.wait_ns, s_abort)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::PANEL + (kk & 3) * 32;
                    mma_ss(tmem + C::COL_S + (j & 1) * 128, smem_desc_sw128(sQa + off, 16, 1024),
                           smem_desc_sw128(sKa + ks * C::TILE + off, 16, 1024), IDESC_QK, kk > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[j & 1]);
                mma_commit(&k_empty[ks]);
                return true;
            };
            auto issue_pv = [&](int i) -> bool {
                const int vs = i % C::VST;
                if (!role_wait(p_full, i & 1, G.wait_ns, s_abort)) return false;
                if (!role_wait(&v_full[vs], (i / C::VST) & 1, G.wait_ns, s_abort)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a_t = tmem + C::COL_P + kk * 8;
                    const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
                    mma_ts(tmem + C::COL_O, a_t, smem_desc_sw128(sVa + vs * C::TILE + kk * 2048, C::PANEL, 1024),
                           IDESC_PV, acc);
                    mma_ts(tmem + C::COL_L, a_t, smem_desc_sw128(sOa + (kk & 3) * 32, 16, 1024), IDESC_L, acc);
                }
                mma_commit(pv_done);
                mma_commit(&v_empty[vs]);
                return true;
            };
            bool ok = role_wait(q_full, 0, G.wait_ns, s_abort) && issue_qk(0);
            for (int j = 0; ok && j < n; ++j) {
                if (j + 1 < n && !issue_qk(j + 1)) { ok = false; break; }
                if (!issue_pv(j)) { ok = false; break; }
            }
            // every issued MMA must finish before TMEM is freed
            mma_commit(drain);
            mbar_wait(drain, 0, G.drain_ns);
        }
    } else {
        // ------------------------------------------------ softmax / epilogue (warps 0-7)
        // warp w and warp w+4 share TMEM lanes 32*(w%4) .. +31 (query rows);
        // half h = w/4 takes key columns [64h, 64h+64) and O columns [h*D/2, (h+1)*D/2)
        const int quarter = warp & 3, half = warp >> 2;
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        int tq, trq, tcq;
        tile_coords(G, tile, tq, trq, tcq);
        const int hq = trq * G.th + (row >> TWL);
        const int wq = tcq * TW + (row & (TW - 1));
        const bool qvalid = hq < G.H && wq < G.W;
        const int rq = qvalid ? reinterpret_cast<const int32_t*>(mask + G.off_radius)[row0 + row] : -1;
        const float sc = G.scale_log2;

        float m_run = -1e30f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const uint32_t e = list[j];
            const int tk = (int)(e & 0x7fff), trk = (int)((e >> 15) & 63), tck = (int)((e >> 21) & 31);
            const int h0 = trk * G.th, w0 = tck * TW;
            const int khv = min(G.th, G.H - h0), kwv = min(TW, G.W - w0);
            const bool full = (e >> 31) != 0;
            const bool need_mask = !full || khv < G.th || kwv < TW;
            uint32_t keep[2] = {~0u, ~0u};
            if (need_mask) {
                const int s = full ? 1 << 20 : (qvalid ? halfwidth(rq, G.g[abs(tk - tq)]) : -1);
                int a_lo = max(0, hq - s - h0), a_hi = min(khv - 1, hq + s - h0);
                const int b_lo = max(0, wq - s - w0), b_hi = min(kwv - 1, wq + s - w0);
                if (!qvalid) { a_lo = 1; a_hi = 0; }
                uint32_t k4[4];
                row_keep_bits<TWL>(a_lo, a_hi, b_lo, b_hi, k4);
                keep[0] = half ? k4[2] : k4[0];
                keep[1] = half ? k4[3] : k4[1];
            }

            const bool got = role_wait(&s_full[j & 1], (j >> 1) & 1, G.wait_ns, s_abort);
            if (__any_sync(0xffffffffu, !got)) { ok = false; break; }
            tc_fence_after();
            __syncwarp();
            float s[64];
            {
                uint32_t v[2][32];
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    tmem_ld32(tmem + lane_base + C::COL_S + (j & 1) * 128 + half * 64 + c * 32, v[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(v[c][i]);
            }
            tc_fence_before();
            mbar_arrive(&s_empty[j & 1]);

            if (need_mask) {
#pragma unroll
                for (int c = 0; c < 64; ++c) s[c] = (keep[c >> 5] & (1u << (c & 31))) ? s[c] : -INFINITY;
            }
            float m4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float a = max3(s[q * 16], s[q * 16 + 1], s[q * 16 + 2]);
#pragma unroll
                for (int i = 3; i < 15; i += 2) a = max3(a, s[q * 16 + i], s[q * 16 + i + 1]);
                m4[q] = fmaxf(a, s[q * 16 + 15]);
            }
            float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            // combine the two halves of the row
            s_red[((j & 1) * 2 + half) * 128 + row] = mx;
            named_bar(1 + quarter, 64);
            mx = fmaxf(mx, s_red[((j & 1) * 2 + (half ^ 1)) * 128 + row]);
            const float m_tile = mx * sc;
            const bool need = m_tile > m_run + 8.0f;
            float alpha = 1.f;
            if (need) { alpha = ex2(m_run - m_tile); m_run = m_tile; }
            const bool rescale = j > 0 && __any_sync(0xffffffffu, need);

            const float neg_m = -m_run;
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const float x0 = fmaf(s[2 * c], sc, neg_m);
                const float x1 = fmaf(s[2 * c + 1], sc, neg_m);
                float p0, p1;
                if ((c % C::POLY_MOD) == C::POLY_MOD - 1) { p0 = ex2_poly<3>(x0); p1 = ex2_poly<3>(x1); }
                else { p0 = ex2(x0); p1 = ex2(x1); }
                pk[c] = pack_bf16x2(p0, p1);
            }
            // PV_{j-1} must be done: it reads P (single buffer) and writes O and L
            if (j > 0) {
                const bool done = role_wait(pv_done, (j - 1) & 1, G.wait_ns, s_abort);
                if (__any_sync(0xffffffffu, !done)) { ok = false; break; }
            }
            tc_fence_after();
            __syncwarp();
            if (rescale) {
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t v[32];
                    const uint32_t col = C::COL_O + half * (D / 2) + c * 32;
                    tmem_ld32(tmem + lane_base + col, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
                    tmem_st32(tmem + lane_base + col, v);
                }
                if (half == 0) {
                    uint32_t v[16];
                    tmem_ld16(tmem + lane_base + C::COL_L, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
                    tmem_st16(tmem + lane_base + C::COL_L, v);
                }
            }
            tmem_st32(tmem + lane_base + C::COL_P + half * 32, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        if (ok && n > 0) {
            ok = role_wait(pv_done, (n - 1) & 1, G.wait_ns, s_abort);
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                __syncwarp();
                uint32_t lv[16];
                tmem_ld16(tmem + lane_base + C::COL_L, lv);
                tmem_wait_ld();
                const float l = __uint_as_float(lv[0]);
                const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t v[32];
                    const int col = half * (D / 2) + c * 32;
                    tmem_ld32(tmem + lane_base + C::COL_O + col, v);
                    tmem_wait_ld();
                    if constexpr (OUT_BF16) {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + (size_t)(row0 + row) * D + col);
                        uint32_t o[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            o[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv, __uint_as_float(v[2 * i + 1]) * inv);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                    } else {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + (size_t)(row0 + row) * D + col);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[i] = make_float4(__uint_as_float(v[4 * i]) * inv, __uint_as_float(v[4 * i + 1]) * inv,
                                                 __uint_as_float(v[4 * i + 2]) * inv, __uint_as_float(v[4 * i + 3]) * inv);
                    }
                }
            }
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
