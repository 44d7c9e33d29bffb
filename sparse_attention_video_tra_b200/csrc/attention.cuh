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
// One CTA per pair of query tiles (A = tile 2p, B = tile 2p+1) of one head.
// The two tiles' key-tile lists are merged (a union with per-tile "listed" and
// "full" flags); each merged key tile is loaded once and used by whichever of
// A and B lists it.  The merged order puts the tiles only one of A and B
// lists first, alternating A-only and B-only, then the tiles both list: the
// two query tiles then work on different key tiles at the same time instead
// of one idling while the other's own tiles stream past (the two rings are
// only two tiles deep), so a CTA takes about max(|A|, |B|) chain steps rather
// than |A u B|.  384 threads:
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread r of a
//              warpgroup owns query row r (TMEM lane r).  Reads S from TMEM,
//              applies the token mask as an additive 0 / -inf bias (per key
//              column and key row of the tile), keeps the running max m (lazy
//              rescale: O is rescaled only when the max grows by more than
//              2^8) and the row sum l of the bf16-rounded P it writes back into
//              the first 64 columns of S.  Scale, bias and row sum use packed
//              fp32x2 arithmetic.
//              The two warpgroups work on independent tiles, so one computes
//              while the other waits for the tensor core.
//   warp 8     TMA producer: Q_A, Q_B, then the K ring.
//   warp 11    TMA producer of the V ring (its own thread, so K tiles run
//              ahead as far as the K ring allows, whatever the V ring waits on).
//   warps 9,10 MMA issuers for tiles A and B (warp 9 also allocates TMEM): for
//              each listed key tile j, O_w += P_w(j) V(j), and in the same issue
//              group S_w = Q_w K(j')^T for the next listed tile j' once its K
//              has landed (the tensor pipe runs one thread's MMAs in order, so
//              the QK overwrites S, where P_w lives, only after the PV has read
//              it); the two tiles progress independently.
//   Register rebalancing: the softmax warpgroups run with 216 registers,
//   warps 8-11 with 72.
// With radius-sorted query groups the CTA takes two mask slots instead (slot s
// of frames 2f and 2f+1: groups of like radius), gathers each slot's 128 query
// rows (rows of its tile-column strip) from global memory straight into the Q
// tiles before the roles start; each softmax thread then speaks for its slot's
// query and writes that query's output row.
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512)
// (P_A, P_B as bf16 pairs in the first 64 columns of S_A, S_B).
#pragma once
#include "pipeline.cuh"

namespace tra {

template <int D>
struct AttnCfg {
    static constexpr int PANEL = 128 * 128;                 // one 64-column panel of 128 rows, bytes
    static constexpr int NP = D / 64;                       // panels per 128-row tile
    static constexpr int TILE = NP * PANEL;                 // bytes of a 128 x D bf16 tile
    static constexpr int KST = (D == 128) ? 2 : 3;          // K ring depth
    static constexpr int VST = (D == 128) ? 2 : 3;          // V ring depth
    static constexpr int OFF_Q = 0;                         // Q_A, Q_B
    static constexpr int OFF_K = 2 * TILE;
    static constexpr int OFF_V = OFF_K + KST * TILE;
    static constexpr int OFF_DYN = OFF_V + VST * TILE;      // lists, half-widths, bitmaps, barriers
    static constexpr int WARP_LOAD = 8, WARP_MMA = 9;       // MMA issuers: warps 9 (tile A), 10 (tile B)
    static constexpr int WARP_VLOAD = 11;                   // V-ring producer
    static constexpr int THREADS = 384;
    // registers after rebalancing: softmax warpgroups 0, 1 and warpgroup 2
    // (384 x 168 at launch = 2 x 128 x 216 + 128 x 72)
    static constexpr int REGS_SOFTMAX = 216, REGS_OTHER = 72;
};

// TMEM columns of the S (and P) and O accumulators of query tile w = 0 (A), 1 (B)
__device__ __forceinline__ uint32_t col_s(int w) { return w ? 128u : 0u; }
__device__ __forceinline__ uint32_t col_o(int w) { return w ? 384u : 256u; }

// Shared-memory layout after the fixed Q/K/V region; sizes depend on the plan.
struct AttnDyn {
    int merged, stab, bits, bars, misc, total, bw;
    __host__ __device__ static AttnDyn make(int list_cap, int rte, int tiles_per_frame)
    {
        AttnDyn L;
        // key tiles a pair of query tiles can reach: frames t-Rt' .. t+1+Rt'
        L.bw = ((2 * rte + 2) * tiles_per_frame + 31) / 32;
        L.merged = 0;                                               // uint32 [2 * list_cap]
        L.stab = L.merged + 8 * list_cap;                           // uint16 [2][rte + 1][128]
        L.bits = L.stab + ((2 * (rte + 1) * 128 * 2 + 15) & ~15);   // uint32 [7][bw]
        L.bars = L.bits + ((7 * L.bw * 4 + 15) & ~15);              // uint64 [32]
        L.misc = L.bars + 8 * 32;
        L.total = L.misc + 32;
        return L;
    }
};

template <int D>
inline int attn_smem_bytes(int list_cap, int rte, int tiles_per_frame)
{
    return AttnCfg<D>::OFF_DYN + AttnDyn::make(list_cap, rte, tiles_per_frame).total + 1024;
}

// A merged key tile: frame (15 bits), tile row (6), tile column (5), then
// listed-by-A (26), listed-by-B (27), full-for-A (28), full-for-B (29).
__device__ __forceinline__ uint32_t pack_tile(int t, int tr, int tc)
{
    return (uint32_t)t | ((uint32_t)tr << 15) | ((uint32_t)tc << 21);
}
constexpr uint32_t MT_IN0 = 1u << 26, MT_FULL0 = 1u << 28;

template <int D, int TWL, bool OUT_BF16, bool DISK>
__global__ void __launch_bounds__(384, 1)
attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const Geom G, const uint8_t* __restrict__ mask,
                 void* __restrict__ out, const void* __restrict__ qraw)
{
    using C = AttnCfg<D>;
    constexpr int TW = 1 << TWL;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const AttnDyn L = AttnDyn::make(G.list_cap, G.rte, G.tiles_per_frame);
    uint8_t* dyn = smem + C::OFF_DYN;
    uint32_t* merged = reinterpret_cast<uint32_t*>(dyn + L.merged);
    uint16_t* s_tab = reinterpret_cast<uint16_t*>(dyn + L.stab);
    // [7][bw]: listed by A, by B, full for A, full for B, then the word
    // offsets of the A-only, B-only and both-listed classes
    uint32_t* bits = reinterpret_cast<uint32_t*>(dyn + L.bits);
    uint64_t* bars = reinterpret_cast<uint64_t*>(dyn + L.bars);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + C::KST;
    uint64_t* v_full = k_empty + C::KST;
    uint64_t* v_empty = v_full + C::VST;
    uint64_t* s_full = v_empty + C::VST;     // [2]: A, B
    uint64_t* p_full = s_full + 2;           // [2]
    uint64_t* pv_done = p_full + 2;          // [2]
    uint64_t* drain = pv_done + 2;           // [2]
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(dyn + L.misc);
    volatile int* s_abort = reinterpret_cast<volatile int*>(dyn + L.misc + 4);
    int* s_n = reinterpret_cast<int*>(dyn + L.misc + 8);
    int* s_lock = reinterpret_cast<int*>(dyn + L.misc + 12);
    int* s_cls = reinterpret_cast<int*>(dyn + L.misc + 16);         // [2]: A-only and B-only counts

    const int pair = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the CTA's two query tiles, or with radius-sorted groups two mask slots of
    // like size and heavily overlapping lists: slot s of frames 2f and 2f + 1
    // (both small-radius groups or both large-radius ones, one frame apart),
    // so that the two per-slot chains stay about equally long and interleave.
    // An odd last frame has no partner frame: its slots pair with each other
    // (slots 2k and 2k + 1 of that frame, neighbouring strips), so that no
    // CTA runs a lone chain while a slot of the frame is left to pair with.
    const int tpf = G.tiles_per_frame;
    const int paired = (G.T / 2) * tpf;                 // CTAs of the frame pairs
    int qa = 2 * pair, qb = qa + 1;
    if (G.qsort && pair < paired) {
        qa = 2 * (pair / tpf) * tpf + pair % tpf;
        qb = qa + tpf;
    } else if (G.qsort) {
        qa = (G.T - 1) * tpf + 2 * (pair - paired);
        qb = qa + 1;
    }
    const bool hasB = qb < G.nQ;
    const int32_t* counts = reinterpret_cast<const int32_t*>(mask + G.off_count) + (size_t)g * G.nQ;
    const uint16_t* lists = reinterpret_cast<const uint16_t*>(mask + G.off_list) + (size_t)g * G.nQ * G.list_cap;
    int nA = counts[qa], nB = hasB ? counts[qb] : 0;
    // the mask buffer is caller memory: a count outside [0, list_cap] is an
    // error (recorded; this CTA then does nothing)
    if (nA < 0 || nA > G.list_cap || nB < 0 || nB > G.list_cap) {
        if (threadIdx.x == 0) atomicOr(&g_tra_error, TRA_ERRBIT_CHECK);
        nA = 0;
        nB = 0;
    }
    const int ta = qa / G.tiles_per_frame, tb = qb / G.tiles_per_frame;
    const int base = max(0, ta - G.rte) * G.tiles_per_frame;   // first key tile either list can hold

    // ---- merge the two sorted lists: set bits, scan per-class word counts,
    // expand (A-only and B-only alternating, then the tiles both list)
    for (int i = tid; i < 7 * L.bw; i += C::THREADS) bits[i] = 0;
    __syncthreads();
    for (int i = tid; i < nA + nB; i += C::THREADS) {
        const bool isB = i >= nA;
        const int e = isB ? lists[(size_t)qb * G.list_cap + (i - nA)] : lists[(size_t)qa * G.list_cap + i];
        const int bit = (e & 0x7fff) - base;
        // a key tile its own query tile cannot reach (outside the grid, or more
        // than Rt' frames from that tile's frame) is an error: recorded, skipped
        const int fe = (e & 0x7fff) / G.tiles_per_frame;
        if (bit < 0 || bit >= 32 * L.bw || (e & 0x7fff) >= G.nQ || abs(fe - (isB ? tb : ta)) > G.rte) {
            atomicOr(&g_tra_error, TRA_ERRBIT_CHECK);
            continue;
        }
        atomicOr(&bits[(isB ? 1 : 0) * L.bw + (bit >> 5)], 1u << (bit & 31));
        if (e & 0x8000) atomicOr(&bits[(isB ? 3 : 2) * L.bw + (bit >> 5)], 1u << (bit & 31));
    }
    __syncthreads();
    if (L.bw <= 32) {
        // every warp scans the (at most 32) words itself, in registers: lane j
        // holds word j's class counts and their exclusive prefix, so no
        // barrier is needed before the expansion
        const uint32_t ja = lane < L.bw ? bits[lane] : 0u, jb = lane < L.bw ? bits[L.bw + lane] : 0u;
        int ex[3], tot[3];
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            const int cnt = __popc(c == 0 ? (ja & ~jb) : (c == 1 ? (jb & ~ja) : (ja & jb)));
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            ex[c] = incl - cnt;
            tot[c] = __shfl_sync(0xffffffffu, incl, 31);
        }
        if (tid == 0) *s_n = tot[0] + tot[1] + tot[2];
        const int nAo = tot[0], nBo = tot[1], m2 = min(nAo, nBo);
        // one thread per bit position; a warp's 32 positions are one word, so
        // the word's class offsets come from its lane by shuffle
        for (int idx = tid; idx < 32 * L.bw; idx += C::THREADS) {
            const int w = idx >> 5, b = idx & 31;
            const int o0 = __shfl_sync(0xffffffffu, ex[0], w), o1 = __shfl_sync(0xffffffffu, ex[1], w),
                      o2 = __shfl_sync(0xffffffffu, ex[2], w);
            const uint32_t ia = bits[w], ib = bits[L.bw + w], bit = 1u << b;
            if (!((ia | ib) & bit)) continue;
            const int c = (ia & bit) ? ((ib & bit) ? 2 : 0) : 1;
            const uint32_t m = c == 0 ? (ia & ~ib) : (c == 1 ? (ib & ~ia) : (ia & ib));
            const int k = (c == 0 ? o0 : (c == 1 ? o1 : o2)) + __popc(m & (bit - 1u));
            const int pos = c == 2 ? nAo + nBo + k : (k < m2 ? 2 * k + c : m2 + k);
            const uint32_t fa = bits[2 * L.bw + w], fb = bits[3 * L.bw + w];
            int tk, trk, tck;
            tile_coords(G, base + idx, tk, trk, tck);
            merged[pos] = pack_tile(tk, trk, tck) | ((ia & bit) ? MT_IN0 : 0u) | ((ib & bit) ? (MT_IN0 << 1) : 0u) |
                          ((fa & bit) ? MT_FULL0 : 0u) | ((fb & bit) ? (MT_FULL0 << 1) : 0u);
        }
    } else {
        if (warp == 0) {
            int carry[3] = {0, 0, 0};
            for (int w0 = 0; w0 < L.bw; w0 += 32) {
                const int w = w0 + lane;
                const uint32_t ia = w < L.bw ? bits[w] : 0u, ib = w < L.bw ? bits[L.bw + w] : 0u;
                const uint32_t cls[3] = {ia & ~ib, ib & ~ia, ia & ib};
#pragma unroll
                for (int c = 0; c < 3; ++c) {
                    const int cnt = __popc(cls[c]);
                    int incl = cnt;
                    for (int o = 1; o < 32; o <<= 1) {
                        const int v = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += v;
                    }
                    if (w < L.bw) bits[(4 + c) * L.bw + w] = carry[c] + incl - cnt;
                    carry[c] += __shfl_sync(0xffffffffu, incl, 31);
                }
            }
            if (lane == 0) {
                s_cls[0] = carry[0];
                s_cls[1] = carry[1];
                *s_n = carry[0] + carry[1] + carry[2];
            }
        }
        __syncthreads();
        {
            // one thread per bit position: an entry's rank in its class is its
            // word's class offset plus the class bits below it in the word
            const int nAo = s_cls[0], nBo = s_cls[1], m2 = min(nAo, nBo);
            for (int idx = tid; idx < 32 * L.bw; idx += C::THREADS) {
                const int w = idx >> 5, b = idx & 31;
                const uint32_t ia = bits[w], ib = bits[L.bw + w], bit = 1u << b;
                if (!((ia | ib) & bit)) continue;
                const int c = (ia & bit) ? ((ib & bit) ? 2 : 0) : 1;
                const uint32_t m = c == 0 ? (ia & ~ib) : (c == 1 ? (ib & ~ia) : (ia & ib));
                const int k = (int)bits[(4 + c) * L.bw + w] + __popc(m & (bit - 1u));
                // A-only rank k goes to 2k, B-only to 2k + 1 while both classes
                // last; the longer one's rest follows; then the tiles both list
                const int pos = c == 2 ? nAo + nBo + k : (k < m2 ? 2 * k + c : m2 + k);
                const uint32_t fa = bits[2 * L.bw + w], fb = bits[3 * L.bw + w];
                int tk, trk, tck;
                tile_coords(G, base + idx, tk, trk, tck);
                merged[pos] = pack_tile(tk, trk, tck) | ((ia & bit) ? MT_IN0 : 0u) | ((ib & bit) ? (MT_IN0 << 1) : 0u) |
                              ((fa & bit) ? MT_FULL0 : 0u) | ((fb & bit) ? (MT_FULL0 << 1) : 0u);
            }
        }
    }
    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < C::KST; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 2); }
        for (int i = 0; i < C::VST; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 2); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1); mbar_init(&p_full[i], 128); mbar_init(&pv_done[i], 1); mbar_init(&drain[i], 1);
        }
        *s_abort = 0;
        *s_lock = 0;
        fence_barrier_init();
    }
    if (warp == C::WARP_MMA) { tmem_alloc(s_tmem, 512); tmem_relinquish(); }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const int n = *s_n;
    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* sK = smem + C::OFF_K;
    uint8_t* sV = smem + C::OFF_V;
    const int kbase = g * G.N_pad;
    // the first ring-depth of K and V tiles goes out now, so that their
    // latency overlaps the query gather
    static_assert(C::KST == C::VST, "one ring depth for K and V");
    const int pre = min(n, C::KST);
    if ((warp == C::WARP_LOAD || warp == C::WARP_VLOAD) && lane == 0) {
        const bool isK = warp == C::WARP_LOAD;
        for (int j = 0; j < pre; ++j) {
            const uint32_t e = merged[j];
            const int tk = (int)(e & 0x7fff), trk = (int)((e >> 15) & 63), tck = (int)((e >> 21) & 31);
            mbar_arrive_expect_tx(&(isK ? k_full : v_full)[j], C::TILE);
#pragma unroll
            for (int p = 0; p < C::NP; ++p)
                load_tile_panel((isK ? sK : sV) + j * C::TILE + p * C::PANEL, isK ? &tm_k : &tm_v, G, p, g, tk, trk, tck,
                                &(isK ? k_full : v_full)[j]);
        }
    }
    // radius-sorted query groups: row r of slot s holds strip row grp_s[r] of
    // the slot's strip (tile row grp >> 7, row grp & 127 of that tile)
    const uint16_t* grp_a = reinterpret_cast<const uint16_t*>(mask + G.off_group) + ((size_t)g * G.nQ + qa) * 128;
    const uint16_t* grp_b = grp_a + (size_t)(qb - qa) * 128;
    if (G.qsort && n > 0) {
        // gather both slots' query rows into Q_A / Q_B (128-byte swizzle),
        // 16 bytes per load; rows outside the grid are zeros
        constexpr int CH = D / 8;                           // 16-byte chunks of a row
        const int np = hasB ? 2 : 1;
        int tqa_, tra_, tca_, tqb_, trb_, tcb_;
        tile_coords(G, qa, tqa_, tra_, tca_);
        tile_coords(G, hasB ? qb : qa, tqb_, trb_, tcb_);
        // batches of QB independent loads (all in flight at once), then their stores
        constexpr int QB = 4;
        for (int e0 = tid; e0 < 128 * np * CH; e0 += QB * C::THREADS) {
            uint4 qv[QB];
#pragma unroll
            for (int k = 0; k < QB; ++k) {
                const int e = e0 + k * C::THREADS;
                qv[k] = make_uint4(0u, 0u, 0u, 0u);
                if (e < 128 * np * CH) {
                    const int d = e / CH, ch = e - d * CH;
                    const int sl = d >> 7, dr = d & 127;
                    const int l = (sl ? grp_b : grp_a)[dr];
                    const int tq = sl ? tqb_ : tqa_, tcq = sl ? tcb_ : tca_;
                    const int hq = (l >> 7) * G.th + ((l & 127) >> TWL), wq = tcq * TW + (l & (TW - 1));
                    if (hq < G.H && wq < G.W) {
                        const int tl = (tq * G.nTh + (l >> 7)) * G.nTw + tcq;
                        const size_t qrow = io_row(G, g, tq, hq, wq, tl * 128 + (l & 127));
                        qv[k] = __ldg(reinterpret_cast<const uint4*>(qraw) + qrow * CH + ch);
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < QB; ++k) {
                const int e = e0 + k * C::THREADS;
                if (e < 128 * np * CH) {
                    const int d = e / CH, ch = e - d * CH;
                    const int sl = d >> 7, dr = d & 127, pn = ch >> 3, cc = ch & 7;
                    *reinterpret_cast<uint4*>(sQ + sl * C::TILE + pn * C::PANEL + dr * 128 + ((cc ^ (dr & 7)) << 4)) = qv[k];
                }
            }
        }
        fence_proxy_async_smem();                               // generic smem writes -> tensor-core reads
        __syncthreads();
    }

    if (warp >= C::WARP_LOAD) {
      regs_dec<C::REGS_OTHER>();
      if (warp == C::WARP_LOAD || warp == C::WARP_VLOAD) {
        // ------------------------------------------------ TMA producers: Q_A, Q_B and the K ring
        // (warp 8), the V ring (warp 11); each walks the merged list on its own
        const bool isK = warp == C::WARP_LOAD;
        if (lane == 0 && n > 0) {
            if (isK) {
                prefetch_tmap(&tm_q); prefetch_tmap(&tm_k);
            } else {
                prefetch_tmap(&tm_v);
            }
            if (isK && !G.qsort) {                                  // else gathered above
                mbar_arrive_expect_tx(q_full, C::TILE * (hasB ? 2 : 1));
                int tqa, trqa, tcqa, tqb, trqb, tcqb;
                tile_coords(G, qa, tqa, trqa, tcqa);
                tile_coords(G, hasB ? qb : qa, tqb, trqb, tcqb);
#pragma unroll
                for (int p = 0; p < C::NP; ++p) {
                    load_tile_panel(sQ + p * C::PANEL, &tm_q, G, p, g, tqa, trqa, tcqa, q_full);
                    if (hasB) load_tile_panel(sQ + C::TILE + p * C::PANEL, &tm_q, G, p, g, tqb, trqb, tcqb, q_full);
                }
            }
            static_assert(C::KST == C::VST, "one ring depth for K and V");
            constexpr int ST = C::KST;
            uint64_t* fullb = isK ? k_full : v_full;
            uint64_t* emptyb = isK ? k_empty : v_empty;
            uint8_t* ring = isK ? sK : sV;
            const CUtensorMap* tm = isK ? &tm_k : &tm_v;
            int iss = pre;                              // the first ring-depth went out before the gather
            for (int j = pre; j < n; ++j) {
                const uint32_t e = merged[j];
                const int tk = (int)(e & 0x7fff), trk = (int)((e >> 15) & 63), tck = (int)((e >> 21) & 31);
                const int st = j % ST;
                if (j >= ST && !role_wait(&emptyb[st], ((j / ST) - 1) & 1, G.wait_ns, s_abort)) break;
                mbar_arrive_expect_tx(&fullb[st], C::TILE);
#pragma unroll
                for (int p = 0; p < C::NP; ++p)
                    load_tile_panel(ring + st * C::TILE + p * C::PANEL, tm, G, p, g, tk, trk, tck, &fullb[st]);
                ++iss;
            }
            // copies still in flight must land before the CTA exits
            if (isK && !G.qsort) mbar_wait(q_full, 0, G.drain_ns);
            for (int j = max(0, iss - ST); j < iss; ++j) mbar_wait(&fullb[j % ST], (j / ST) & 1, G.drain_ns);
        }
      } else if (warp == C::WARP_MMA || warp == C::WARP_MMA + 1) {
        // ------------------------------------------------ MMA issuers, one per query tile
        // Issuing tcgen05.mma occupies the issuing thread about as long as the
        // tensor core runs it, so each query tile w gets its own issuer; both walk
        // the merged list in order.  For a tile w lists: S_w = Q_w K^T, then,
        // once the softmax has written P_w, O_w += P_w V followed in the same
        // group by the next listed tile's QK.  Either way it releases the K and V
        // ring stages (two arrivals per occupant): a commit after its MMAs, or a
        // plain arrive once the tile has landed.  The softmax rescales O_w at
        // tile k only after s_full of tile k, whose commit covers every earlier
        // MMA of this thread, the PV of tile k-1 included.
        const int w = warp - C::WARP_MMA;
        if (lane == 0 && n > 0) {
            constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false);
            constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
            const uint32_t sQa = smem_u32(sQ) + w * C::TILE, sKa = smem_u32(sK), sVa = smem_u32(sV);
            const uint32_t in_bit = MT_IN0 << w;
            bool ok = G.qsort || role_wait(q_full, 0, G.wait_ns, s_abort);     // grouped Q is already in place
            int cnt = 0;
            int qk_ahead = -1;                  // entry whose QK went out with the previous PV group
            auto issue_qk = [&](int jj) {
                const int kss = jj % C::KST;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::PANEL + (kk & 3) * 32;
                    mma_ss(tmem + col_s(w), smem_desc_sw128(sQa + off, 16, 1024),
                           smem_desc_sw128(sKa + kss * C::TILE + off, 16, 1024), IDESC_QK, kk > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[w]);
                mma_commit(&k_empty[kss]);
            };
            // An entry this tile does not list is released as soon as its K has
            // landed; its V stage is released one step later (at the next entry,
            // after that entry's QK has gone out), so a V tile that lands late
            // never holds up this tile's next QK.  At most one V release is
            // pending, so the V ring always moves on.
            int pend_v = -1;
            auto release_v = [&]() -> bool {
                if (pend_v < 0) return true;
                const int pj = pend_v;
                pend_v = -1;
                if (!role_wait(&v_full[pj % C::VST], (pj / C::VST) & 1, G.wait_ns, s_abort)) return false;
                mbar_arrive(&v_empty[pj % C::VST]);
                return true;
            };
            for (int j = 0; ok && j < n; ++j) {
                const bool uses = (merged[j] & in_bit) != 0;
                const int ks = j % C::KST, vs = j % C::VST;
                if (!uses) {
                    if (!release_v()) { ok = false; break; }
                    if (!role_wait(&k_full[ks], (j / C::KST) & 1, G.wait_ns, s_abort)) { ok = false; break; }
                    mbar_arrive(&k_empty[ks]);
                    pend_v = j;
                    continue;
                }
                if (qk_ahead != j) {
                    if (!role_wait(&k_full[ks], (j / C::KST) & 1, G.wait_ns, s_abort)) { ok = false; break; }
                    if (!issue_lock(s_lock, G.wait_ns, s_abort)) { ok = false; break; }
                    tc_fence_after();
                    issue_qk(j);
                    issue_unlock(s_lock);
                }
                if (!release_v()) { ok = false; break; }
                // This tile's next listed entry j' joins this group when its K has
                // landed: the tensor pipe runs the MMAs of one thread in order, so
                // the QK overwrites S (holding P) only after this PV has read it.
                // Only j' <= j + KST is looked at: every earlier entry of j''s
                // ring stage has then been waited for by this thread, so the
                // parity test names j''s own landing.
                int jn = j + 1;
                while (jn < n && jn <= j + C::KST && !(merged[jn] & in_bit)) ++jn;
                const bool has_next = jn < n && jn <= j + C::KST;
                // V has usually landed long before the softmax ends: wait for it
                // first, so that only the lock follows the softmax's hand-off
                if (!role_wait(&v_full[vs], (j / C::VST) & 1, G.wait_ns, s_abort)) { ok = false; break; }
                if (!role_wait(&p_full[w], cnt & 1, G.wait_ns, s_abort)) { ok = false; break; }
                if (!issue_lock(s_lock, G.wait_ns, s_abort)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + col_o(w), tmem + col_s(w) + kk * 8,
                           smem_desc_sw128(sVa + vs * C::TILE + kk * 2048, C::PANEL, 1024), IDESC_PV,
                           (cnt > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&v_empty[vs]);
                if (has_next && mbar_test(&k_full[jn % C::KST], (jn / C::KST) & 1)) {
                    tc_fence_after();
                    issue_qk(jn);
                    qk_ahead = jn;
                }
                // only the epilogue waits for the last PV; a commit covers every
                // earlier MMA of this thread, so this one may follow the QK
                mma_commit(&pv_done[w]);
                issue_unlock(s_lock);
                ++cnt;
            }
            if (ok && !release_v()) ok = false;
            // every issued MMA must finish before TMEM is freed
            mma_commit(&drain[w]);
            mbar_wait(&drain[w], 0, G.drain_ns);
        }
      }
    } else {
        regs_inc<C::REGS_SOFTMAX>();
        // ------------------------------------------------ softmax / epilogue (warps 0-7)
        const int w = warp >> 2;                             // 0: tile A, 1: tile B
        const int row = tid & 127;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t colS = col_s(w), colO = col_o(w);
        const bool active = w == 0 || hasB;
        // this thread's query: row `row` of tile qa / qb, or the strip row of
        // its group slot (radius-sorted groups)
        int qt = w ? qb : qa, qrow = row;
        bool grp_ok = true;
        if (G.qsort && active) {
            // strip row l: row l & 127 of the tile in tile row l >> 7 of the
            // slot's tile column and frame.  The group section is caller
            // memory: a row past the strip is recorded and the slot left empty.
            int l = (w ? grp_b : grp_a)[row];
            if (l >= 128 * G.nTh) {
                atomicOr(&g_tra_error, TRA_ERRBIT_CHECK);
                l = 0;
                grp_ok = false;
            }
            int t0, tr0, tc0;
            tile_coords(G, qt, t0, tr0, tc0);
            qt = (t0 * G.nTh + (l >> 7)) * G.nTw + tc0;
            qrow = l & 127;
        }
        int tq, trq, tcq;
        tile_coords(G, active ? qt : qa, tq, trq, tcq);
        const int hq = trq * G.th + (qrow >> TWL);
        const int wq = tcq * TW + (qrow & (TW - 1));
        const bool qvalid = active && grp_ok && hq < G.H && wq < G.W;
        const int rq = qvalid ? reinterpret_cast<const int32_t*>(mask + G.off_radius)[kbase + qt * 128 + qrow] : -1;
        uint16_t* my_tab = s_tab + w * (G.rte + 1) * 128;
        for (int dl = 0; dl <= G.rte; ++dl)
            my_tab[dl * 128 + row] = (uint16_t)(qvalid ? min(halfwidth(rq, G.g[dl]), TRA_DISK_S_CLAMP) : 0);
        const float sc = G.scale_log2;
        const uint32_t in_bit = MT_IN0 << w, full_bit = MT_FULL0 << w;

        // m_run: the log2-domain maximum P is taken relative to (anchored at the
        // first kept maximum, raised lazily when a tile exceeds it by 2^8);
        // l: the sum of the bf16-rounded P values, in the same frame.
        float m_run = 0.f, l = 0.f;
        const f2_t sc2 = f2_pack(sc, sc);
        constexpr int KR = 128 >> TWL;                       // key rows of a tile
        constexpr int CP = TW / 2;                           // column pairs of a key row
        int k = 0;                                           // tiles processed by this query tile
        bool ok = true;
        for (int j = 0; active && j < n; ++j) {
            const uint32_t e = merged[j];
            if (!(e & in_bit)) continue;
            const int tk = (int)(e & 0x7fff), trk = (int)((e >> 15) & 63), tck = (int)((e >> 21) & 31);
            const int h0 = trk * G.th, w0 = tck * TW;
            const int khv = min(G.th, G.H - h0), kwv = min(TW, G.W - w0);
            const bool full = (e & full_bit) != 0;
            // kept keys of this row inside the tile: key rows [a_lo, a_hi] x columns [b_lo, b_hi]
            int a_lo = 0, a_hi = khv - 1, b_lo = 0, b_hi = kwv - 1;
            const int s = full ? 0 : (int)my_tab[abs(tk - tq) * 128 + row];
            if (!full) {
                a_lo = max(0, hq - s - h0); a_hi = min(khv - 1, hq + s - h0);
                b_lo = max(0, wq - s - w0); b_hi = min(kwv - 1, wq + s - w0);
            }
            if (!qvalid) { a_lo = 1; a_hi = 0; }
            // column bias (0 kept, -inf masked) as pairs; the row bias is added per key row
            f2_t colb[CP];
            // disk: squared column distance dw^2 per key column (INT_MAX past the
            // grid edge); key row a keeps the columns with dw^2 <= s^2 - dh^2
            int cdw2[DISK ? TW : 1];
            if constexpr (DISK) {
#pragma unroll
                for (int b = 0; b < TW; ++b) {
                    const int dw = w0 + b - wq;
                    cdw2[b] = b < kwv ? dw * dw : INT_MAX;
                }
            } else {
#pragma unroll
                for (int bp = 0; bp < CP; ++bp)
                    colb[bp] = f2_pack((2 * bp >= b_lo && 2 * bp <= b_hi) ? 0.f : -INFINITY,
                                       (2 * bp + 1 >= b_lo && 2 * bp + 1 <= b_hi) ? 0.f : -INFINITY);
            }

            const bool got = role_wait(&s_full[w], k & 1, G.wait_ns, s_abort);
            if (__any_sync(0xffffffffu, !got)) { ok = false; break; }
            tc_fence_after();
            __syncwarp();
            uint32_t v[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_base + colS + c * 32, v[c]);
            tmem_wait_ld();
            // x = S * scale - m_run + bias  (log2 domain), packed in pairs
            f2_t x[64];
#pragma unroll
            for (int a = 0; a < KR; ++a) {
                const float rb = (a >= a_lo && a <= a_hi) ? -m_run : -INFINITY;
                const f2_t rb2 = f2_pack(rb, rb);
                if constexpr (DISK) {
                    // the disk keeps (a, b) iff dh^2 + dw^2 <= s^2 (a full tile
                    // keeps every valid column); the row bias is the FMA's addend
                    const int dh = h0 + a - hq;
                    const int thr = full ? INT_MAX - 1 : s * s - dh * dh;
#pragma unroll
                    for (int bp = 0; bp < CP; ++bp) {
                        const int i = a * CP + bp, c = (2 * i) >> 5, o = (2 * i) & 31;
                        float x0, x1;
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(v[c][o]), __uint_as_float(v[c][o + 1])), sc2, rb2), x0, x1);
                        x[i] = f2_pack(cdw2[2 * bp] <= thr ? x0 : -INFINITY, cdw2[2 * bp + 1] <= thr ? x1 : -INFINITY);
                    }
                } else {
#pragma unroll
                    for (int bp = 0; bp < CP; ++bp) {
                        const int i = a * CP + bp, c = (2 * i) >> 5, o = (2 * i) & 31;
                        x[i] = f2_add(f2_fma(f2_pack(__uint_as_float(v[c][o]), __uint_as_float(v[c][o + 1])), sc2, colb[bp]), rb2);
                    }
                }
            }
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                float x0, x1;
                f2_unpack(x[i], x0, x1);
                m4[i & 3] = max3(m4[i & 3], x0, x1);
            }
            const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));   // relative to m_run
            // shift the frame: to the first kept maximum, or up when a tile exceeds 2^8
            float delta = 0.f, alpha = 1.f;
            bool resc = false;
            if (mx > -INFINITY) {
                if (l == 0.f) delta = mx;
                else if (mx > 8.f) { delta = mx; alpha = ex2(-mx); resc = true; }
            }
            if (delta != 0.f) {
                m_run += delta;
                const f2_t nd = f2_pack(-delta, -delta);
#pragma unroll
                for (int i = 0; i < 64; ++i) x[i] = f2_add(x[i], nd);
            }
            l *= alpha;
            const bool rescale = k > 0 && __any_sync(0xffffffffu, resc);
            f2_t ls[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    float x0, x1;
                    f2_unpack(x[c * 16 + q], x0, x1);
                    pk[q] = pack_bf16x2(ex2(x0), ex2(x1));
                    // the row sum adds exactly the bf16 values the tensor core will use
                    ls[q & 3] = f2_add(ls[q & 3], f2_pack(__uint_as_float(pk[q] << 16), __uint_as_float(pk[q] & 0xffff0000u)));
                }
                tmem_st16(tmem + lane_base + colS + c * 16, pk);
            }
            {
                float s0, s1, s2, s3, s4, s5, s6, s7;
                f2_unpack(ls[0], s0, s1); f2_unpack(ls[1], s2, s3); f2_unpack(ls[2], s4, s5); f2_unpack(ls[3], s6, s7);
                l += ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
            }
            // O_w is complete up to tile k-1 (s_full of this tile covers that PV);
            // rescale it before the PV of this tile is issued (after p_full)
            if (rescale) {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t vo[32];
                    tmem_ld32(tmem + lane_base + colO + c * 32, vo);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) vo[i] = __float_as_uint(__uint_as_float(vo[i]) * alpha);
                    tmem_st32(tmem + lane_base + colO + c * 32, vo);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[w]);
            ++k;
        }
        if (ok && k > 0) {
            ok = role_wait(&pv_done[w], (k - 1) & 1, G.wait_ns, s_abort);
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                __syncwarp();
                const float inv = l > 0.f ? 1.f / l : 0.f;
                const bool store = !G.natural || qvalid;          // natural layout has no pad rows
                const size_t orow = io_row(G, g, tq, hq, wq, qt * 128 + qrow) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_base + colO + c * 32, v);
                    tmem_wait_ld();
                    if (!store) continue;
                    if constexpr (OUT_BF16) {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + orow + c * 32);
                        uint32_t o[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            o[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv, __uint_as_float(v[2 * i + 1]) * inv);
#pragma unroll
                        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                    } else {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + orow + c * 32);
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
