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
// One CTA per (query tile of 128 tokens, head).  224 threads:
//   warps 0-3  softmax: thread i owns query row i = TMEM lane i.  Reads S from
//              TMEM, masks, keeps the running max m and sum l (lazy rescale:
//              O is rescaled only when the max grows by more than 2^8), writes
//              P = 2^(S*scale - m) as bf16 into TMEM, and in the end reads O,
//              divides by l and stores fp32 rows (bf16 rows on request).
//   warp 4     TMA producer for Q and the K ring.
//   warp 5     TMA producer for the V ring.
//   warp 6     TMEM allocator and single-thread MMA issuer:
//              S[j%2] = Q K_j^T (A, B from smem, K-major), then
//              O += P[j-1] V[j-1] (A = P from TMEM, B = V from smem, MN-major).
// TMEM columns: S0 [0,128), S1 [128,256), O [256,256+D), P0 [384,448), P1 [448,512).
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
    static constexpr int OFF_STAB = OFF_V + VST * TILE;     // int16 half-widths [32][128]
    static constexpr int OFF_LIST = OFF_STAB + (TRA_MAX_RT_EFF + 1) * 128 * 2;   // uint16 [LIST_MAX]
    static constexpr int OFF_BAR = OFF_LIST + TRA_MAX_LIST_CAP * 2;
    static constexpr int NBAR = 1 + 2 * KST + 2 * VST + 2 * 4 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;       // + alignment slack
    static constexpr int THREADS = 224;
    static constexpr uint32_t COL_S = 0, COL_O = 256, COL_P = 384;
};

template <int D, int TWL, bool OUT_BF16>
__global__ void __launch_bounds__(224, 1)
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
    int16_t* s_tab = reinterpret_cast<int16_t*>(smem + C::OFF_STAB);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + C::KST;
    uint64_t* v_full = k_empty + C::KST;
    uint64_t* v_empty = v_full + C::VST;
    uint64_t* s_full = v_empty + C::VST;
    uint64_t* s_empty = s_full + 2;
    uint64_t* p_full = s_empty + 2;
    uint64_t* pv_done = p_full + 2;
    uint64_t* drain = pv_done + 2;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    const int tile = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = reinterpret_cast<const int32_t*>(mask + G.off_count)[(size_t)g * G.nQ + tile];
    const uint16_t* glist = reinterpret_cast<const uint16_t*>(mask + G.off_list) + ((size_t)g * G.nQ + tile) * G.list_cap;
    uint16_t* list = reinterpret_cast<uint16_t*>(smem + C::OFF_LIST);
    for (int i = tid; i < n; i += C::THREADS) list[i] = glist[i];
    const int row0 = g * G.N_pad + tile * 128;               // first tile-major row of this tile

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < C::KST; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
        for (int i = 0; i < C::VST; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 128);
            mbar_init(&p_full[i], 128); mbar_init(&pv_done[i], 1);
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 6) { tmem_alloc(s_tmem, 512); tmem_relinquish(); }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 4) {
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
                const int kb = list[j] & 0x7fff;
                mbar_arrive_expect_tx(&k_full[st], C::TILE);
#pragma unroll
                for (int p = 0; p < C::NP; ++p)
                    tma_load_2d(sK + st * C::TILE + p * C::PANEL, &tm_k, p * 64, g * G.N_pad + kb * 128, &k_full[st]);
                ++issued;
            }
            // copies still in flight must land before the CTA exits
            mbar_wait(q_full, 0, G.drain_ns);
            for (int j = max(0, issued - C::KST); j < issued; ++j)
                mbar_wait(&k_full[j % C::KST], (j / C::KST) & 1, G.drain_ns);
        }
    } else if (warp == 5) {
        // ------------------------------------------------ V producer
        if (lane == 0 && n > 0) {
            prefetch_tmap(&tm_v);
            int issued = 0;
            for (int j = 0; j < n; ++j) {
                const int st = j % C::VST;
                if (j >= C::VST && !role_wait(&v_empty[st], ((j / C::VST) - 1) & 1, G.wait_ns, s_abort)) break;
                const int kb = list[j] & 0x7fff;
                mbar_arrive_expect_tx(&v_full[st], C::TILE);
#pragma unroll
                for (int p = 0; p < C::NP; ++p)
                    tma_load_2d(sV + st * C::TILE + p * C::PANEL, &tm_v, p * 64, g * G.N_pad + kb * 128, &v_full[st]);
                ++issued;
            }
            for (int j = max(0, issued - C::VST); j < issued; ++j)
                mbar_wait(&v_full[j % C::VST], (j / C::VST) & 1, G.drain_ns);
        }
    } else if (warp == 6) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && n > 0) {
            constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false);
            constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
            const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
            bool ok = role_wait(q_full, 0, G.wait_ns, s_abort);
            auto issue_pv = [&](int i) -> bool {
                const int vs = i % C::VST;
                if (!role_wait(&p_full[i & 1], (i >> 1) & 1, G.wait_ns, s_abort)) return false;
                if (!role_wait(&v_full[vs], (i / C::VST) & 1, G.wait_ns, s_abort)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a_t = tmem + C::COL_P + (i & 1) * 64 + kk * 8;
                    const uint64_t bd = smem_desc_sw128(sVa + vs * C::TILE + kk * 2048, C::PANEL, 1024);
                    mma_ts(tmem + C::COL_O, a_t, bd, IDESC_PV, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&pv_done[i & 1]);
                mma_commit(&v_empty[vs]);
                return true;
            };
            for (int j = 0; ok && j < n; ++j) {
                const int ks = j % C::KST;
                if (!role_wait(&k_full[ks], (j / C::KST) & 1, G.wait_ns, s_abort)) { ok = false; break; }
                if (j >= 2 && !role_wait(&s_empty[j & 1], ((j - 2) >> 1) & 1, G.wait_ns, s_abort)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::PANEL + (kk & 3) * 32;
                    const uint64_t ad = smem_desc_sw128(sQa + off, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(sKa + ks * C::TILE + off, 16, 1024);
                    mma_ss(tmem + C::COL_S + (j & 1) * 128, ad, bd, IDESC_QK, kk > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[j & 1]);
                mma_commit(&k_empty[ks]);
                if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
            }
            if (ok) ok = issue_pv(n - 1);
            // every issued MMA must finish before TMEM is freed
            mma_commit(drain);
            mbar_wait(drain, 0, G.drain_ns);
        }
    } else {
        // ------------------------------------------------ softmax / epilogue (warps 0-3)
        const int row = tid;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        int tq, trq, tcq;
        tile_coords(G, tile, tq, trq, tcq);
        const int hq = trq * G.th + (row >> TWL);
        const int wq = tcq * TW + (row & (TW - 1));
        const bool qvalid = hq < G.H && wq < G.W;
        const int rq = qvalid ? reinterpret_cast<const int32_t*>(mask + G.off_radius)[row0 + row] : -1;
        for (int dl = 0; dl <= G.rte; ++dl)
            s_tab[dl * 128 + row] = (int16_t)(qvalid ? min(halfwidth(rq, G.g[dl]), 32767) : -1);

        float m_run = -1e30f, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const int e = list[j];
            const int kb = e & 0x7fff;
            int tk, trk, tck;
            tile_coords(G, kb, tk, trk, tck);
            const int h0 = trk * G.th, w0 = tck * TW;
            const int khv = min(G.th, G.H - h0), kwv = min(TW, G.W - w0);
            const bool need_mask = !(e & 0x8000) || khv < G.th || kwv < TW;
            uint32_t keep[4] = {~0u, ~0u, ~0u, ~0u};
            if (need_mask) {
                const int s = (e & 0x8000) ? 1 << 20 : (int)s_tab[abs(tk - tq) * 128 + row];
                int a_lo = max(0, hq - s - h0), a_hi = min(khv - 1, hq + s - h0);
                const int b_lo = max(0, wq - s - w0), b_hi = min(kwv - 1, wq + s - w0);
                if (!qvalid) { a_lo = 1; a_hi = 0; }
                row_keep_bits<TWL>(a_lo, a_hi, b_lo, b_hi, keep);
            }

            const int bs = j & 1;
            const bool got = role_wait(&s_full[bs], (j >> 1) & 1, G.wait_ns, s_abort);
            if (__any_sync(0xffffffffu, !got)) { ok = false; break; }
            tc_fence_after();
            __syncwarp();
            float s[128];
            {
                uint32_t v[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    tmem_ld32(tmem + lane_base + C::COL_S + bs * 128 + c * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(v[i]);
                }
            }
            tc_fence_before();
            mbar_arrive(&s_empty[bs]);

            if (need_mask) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (!((keep[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
            }
            float mx = s[0];
#pragma unroll
            for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
            const float m_tile = mx * G.scale_log2;
            const bool need = m_tile > m_run + 8.0f;
            if (__any_sync(0xffffffffu, need)) {
                float alpha = 1.f;
                if (need) { alpha = ex2(m_run - m_tile); m_run = m_tile; }
                l *= alpha;
                if (j > 0) {
                    if (!role_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, G.wait_ns, s_abort)) { ok = false; }
                    if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                    tc_fence_after();
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_base + C::COL_O + c * 32, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
                        tmem_st32(tmem + lane_base + C::COL_O + c * 32, v);
                    }
                    tmem_wait_st();
                }
            }
            // P goes to the tensor core as bf16; l sums those same rounded values,
            // so O = sum(P v) / sum(P) is an exact weighted mean of the kept v rows
            const float neg_m = -m_run;
            float lsum = 0.f;
            uint32_t pk[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float p0 = ex2(fmaf(s[2 * c], G.scale_log2, neg_m));
                const float p1 = ex2(fmaf(s[2 * c + 1], G.scale_log2, neg_m));
                pk[c] = pack_bf16x2(p0, p1);
                lsum += __uint_as_float(pk[c] << 16) + __uint_as_float(pk[c] & 0xffff0000u);
            }
            l += lsum;
            if (j >= 2) {
                if (!role_wait(&pv_done[bs], ((j - 2) >> 1) & 1, G.wait_ns, s_abort)) ok = false;
                if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
            }
            tc_fence_after();
            __syncwarp();
            tmem_st32(tmem + lane_base + C::COL_P + bs * 64, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(tmem + lane_base + C::COL_P + bs * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[bs]);
        }
        if (ok && n > 0) {
            const int jl = n - 1;
            ok = role_wait(&pv_done[jl & 1], (jl >> 1) & 1, G.wait_ns, s_abort);
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                __syncwarp();
                const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_base + C::COL_O + c * 32, v);
                    tmem_wait_ld();
                    if constexpr (OUT_BF16) {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + (size_t)(row0 + row) * D);
                        uint32_t o[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            o[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv, __uint_as_float(v[2 * i + 1]) * inv);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[c * 4 + i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                    } else {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + (size_t)(row0 + row) * D);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[c * 8 + i] = make_float4(__uint_as_float(v[4 * i]) * inv, __uint_as_float(v[4 * i + 1]) * inv,
                                                         __uint_as_float(v[4 * i + 2]) * inv, __uint_as_float(v[4 * i + 3]) * inv);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 6) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tra
