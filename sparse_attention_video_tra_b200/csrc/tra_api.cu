// tra_api.cu -- the extern "C" entry points that launch the kernels: argument
// checks, TMA tensor maps, kernel selection by (head dim, tile width), and the
// device error word.  All kernels are compiled into this one translation unit.
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/tra.h"
#include "tra_plan_impl.h"
#include "pipeline.cuh"
#include "permute.cuh"
#include "radius_mask.cuh"
#include "entropy.cuh"
#include "attention.cuh"
#include "topk.cuh"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [rows][D] bf16 rows, 128-row x 64-column boxes, 128-byte swizzle
bool make_row_map(CUtensorMap* m, const void* base, uint64_t rows, int D)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [heads*T][H][W][D] bf16 in natural token order, {64, tw, th, 1} boxes (one
// panel of one (1, th, tw) tile; coordinates past the grid read as zeros)
bool make_natural_map(CUtensorMap* m, const void* base, const tra::Geom& G)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)G.D, (cuuint64_t)G.W, (cuuint64_t)G.H, (cuuint64_t)G.T * G.G};
    const cuuint64_t strides[3] = {(cuuint64_t)G.D * 2, (cuuint64_t)G.W * G.D * 2, (cuuint64_t)G.H * G.W * G.D * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)G.tw, (cuuint32_t)G.th, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// the input map for the plan's layout
bool make_input_map(CUtensorMap* m, const void* base, const tra::Geom& G)
{
    return G.natural ? make_natural_map(m, base, G) : make_row_map(m, base, (uint64_t)G.G * G.N_pad, G.D);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

tra_status launch_status()
{
    return cudaGetLastError() == cudaSuccess ? TRA_OK : TRA_ERR_CUDA;
}

template <class K>
bool set_smem(K kernel, int bytes)
{
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

// largest dynamic shared memory a CTA may use on sm_100
constexpr int kMaxSmem = 232448;

template <int D, int TWL, bool OB, bool DISK>
tra_status run_attention(const tra::Geom& G, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                         const uint8_t* mask, void* out, const void* qraw, cudaStream_t st)
{
    using C = tra::AttnCfg<D>;
    auto kern = tra::attention_kernel<D, TWL, OB, DISK>;
    const int smem = tra::attn_smem_bytes<D>(G.list_cap, G.rte, G.tiles_per_frame);
    if (smem > kMaxSmem) return TRA_ERR_UNSUPPORTED;
    if (!set_smem(kern, smem)) return TRA_ERR_CUDA;
    // two query tiles per CTA; with radius-sorted groups, the same slot of
    // frames 2f and 2f + 1, then an odd last frame's slots two by two
    const int ctas = G.qsort ? G.T / 2 * G.tiles_per_frame + (G.T % 2) * ((G.tiles_per_frame + 1) / 2)
                             : (G.nQ + 1) / 2;
    kern<<<dim3(ctas, G.G), C::THREADS, smem, st>>>(q, k, v, G, mask, out, qraw);
    return launch_status();
}

template <int D, int TWL>
tra_status run_entropy(const tra::Geom& G, const CUtensorMap& q, const CUtensorMap& k, int stride, float corr,
                       float* H, cudaStream_t st)
{
    using C = tra::EntCfg<D>;
    auto kern = tra::entropy_kernel<D, TWL>;
    if (!set_smem(kern, C::SMEM)) return TRA_ERR_CUDA;
    kern<<<dim3((G.nQ + 1) / 2, G.G), C::THREADS, C::SMEM, st>>>(q, k, G, stride, corr, H);
    return launch_status();
}

template <int D, int TWL>
tra_status run_topk(const tra::Geom& G, const CUtensorMap& q, const CUtensorMap& k, int stride, int n_sample,
                    float mass, float* H, int* K, cudaStream_t st)
{
    using C = tra::TopkCfg<D>;
    auto kern = tra::topk_kernel<D, TWL>;
    if (!set_smem(kern, C::SMEM)) return TRA_ERR_CUDA;
    kern<<<dim3(n_sample, G.G), C::THREADS, C::SMEM, st>>>(q, k, G, stride, n_sample, mass, H, K);
    return launch_status();
}

}  // namespace

extern "C" tra_status tra_permute(tra_plan plan, const void* src, void* dst, int to_tile_major, int elem_bytes,
                                  tra_stream stream)
{
    if (!plan || !src || !dst || !aligned(src, 16) || !aligned(dst, 16)) return TRA_ERR_INVALID_ARG;
    if (elem_bytes != 2 && elem_bytes != 4) return TRA_ERR_INVALID_ARG;
    const tra::Geom& G = plan->geom;
    const size_t total = (size_t)G.G * G.N_pad * (G.D * elem_bytes / 16);
    const int blocks = (int)std::min<size_t>((total + 255) / 256, 148 * 32);
    tra::permute_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(G, (const uint4*)src, (uint4*)dst,
                                                                   to_tile_major ? 1 : 0, elem_bytes);
    return launch_status();
}

extern "C" tra_status tra_entropy(tra_plan plan, const void* q, const void* k, float* Hout, int key_tile_stride,
                                  tra_stream stream)
{
    if (!plan || !q || !k || !Hout || !aligned(q, 16) || !aligned(k, 16) || !aligned(Hout, 4))
        return TRA_ERR_INVALID_ARG;
    const tra::Geom& G = plan->geom;
    if (key_tile_stride < 1 || key_tile_stride > G.nQ) return TRA_ERR_INVALID_ARG;
    // |S| = valid keys in the sampled tiles; corr = ln(N / |S|)
    float corr = 0.f;
    if (key_tile_stride > 1) {
        long long nS = 0;
        for (int kb = 0; kb < G.nQ; kb += key_tile_stride) {
            const int rem = kb % G.tiles_per_frame;
            const int tr = rem / G.nTw, tc = rem % G.nTw;
            nS += (long long)std::min(G.th, G.H - tr * G.th) * std::min(G.tw, G.W - tc * G.tw);
        }
        corr = (float)std::log((double)G.N / (double)nS);
    }
    CUtensorMap mq, mk;
    if (!make_input_map(&mq, q, G) || !make_input_map(&mk, k, G)) return TRA_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    const int key = G.D * 100 + G.tw_log2;
    switch (key) {
        case 6402: return run_entropy<64, 2>(G, mq, mk, key_tile_stride, corr, Hout, st);
        case 6403: return run_entropy<64, 3>(G, mq, mk, key_tile_stride, corr, Hout, st);
        case 6404: return run_entropy<64, 4>(G, mq, mk, key_tile_stride, corr, Hout, st);
        case 6405: return run_entropy<64, 5>(G, mq, mk, key_tile_stride, corr, Hout, st);
        case 12802: return run_entropy<128, 2>(G, mq, mk, key_tile_stride, corr, Hout, st);
        case 12803: return run_entropy<128, 3>(G, mq, mk, key_tile_stride, corr, Hout, st);
        case 12804: return run_entropy<128, 4>(G, mq, mk, key_tile_stride, corr, Hout, st);
        case 12805: return run_entropy<128, 5>(G, mq, mk, key_tile_stride, corr, Hout, st);
    }
    return TRA_ERR_UNSUPPORTED;
}

extern "C" tra_status tra_radius_and_mask(tra_plan plan, const float* Hent, void* mask, size_t mask_bytes,
                                          tra_stream stream)
{
    if (!plan || !Hent || !mask || !aligned(Hent, 4) || !aligned(mask, 256)) return TRA_ERR_INVALID_ARG;
    if (mask_bytes < plan->mask_bytes) return TRA_ERR_WORKSPACE;
    tra::Geom G = plan->geom;
    // one CTA per tile-column strip (query groups) or per tile
    const int U = G.qsort ? G.nTh : 1;
    const dim3 grid(G.qsort ? G.T * G.nTw : G.nQ, G.G);
    int smem = tra::mask_smem_bytes(G.rte, G.nTh, G.r_cap, G.hw_tab != 0, G.disk_smax, U);
    if (G.disk_smax >= 0 && smem > kMaxSmem - 16 * 1024) {
        // no room for the disk-row table: count the disk row by row
        G.disk_smax = -1;
        smem = tra::mask_smem_bytes(G.rte, G.nTh, G.r_cap, G.hw_tab != 0, G.disk_smax, U);
    }
    if (smem > kMaxSmem - 16 * 1024) return TRA_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t* m = (uint8_t*)mask;
    auto go = [&](auto kern) -> bool {
        if (smem > 48 * 1024 && !set_smem(kern, smem)) return false;
        kern<<<grid, 128 * U, smem, st>>>(G, Hent, m);
        return true;
    };
    bool ok;
    if (!G.qsort) ok = G.disk ? go(tra::radius_mask_kernel<true, false, 128>) : go(tra::radius_mask_kernel<false, false, 128>);
    else if (U <= 3) ok = G.disk ? go(tra::radius_mask_kernel<true, true, 384>) : go(tra::radius_mask_kernel<false, true, 384>);
    else ok = G.disk ? go(tra::radius_mask_kernel<true, true, 512>) : go(tra::radius_mask_kernel<false, true, 512>);
    if (!ok) return TRA_ERR_CUDA;
    return launch_status();
}

namespace {

template <int D, int TWL>
tra_status attention_variant(const tra::Geom& G, bool ob, bool disk, const CUtensorMap& q, const CUtensorMap& k,
                             const CUtensorMap& v, const uint8_t* m, void* out, const void* qr, cudaStream_t st)
{
    if (ob) return disk ? run_attention<D, TWL, true, true>(G, q, k, v, m, out, qr, st)
                        : run_attention<D, TWL, true, false>(G, q, k, v, m, out, qr, st);
    return disk ? run_attention<D, TWL, false, true>(G, q, k, v, m, out, qr, st)
                : run_attention<D, TWL, false, false>(G, q, k, v, m, out, qr, st);
}

// kernel instance by (head dim, tile width, output type, spatial metric)
tra_status dispatch_attention(const tra::Geom& G, bool ob, bool disk, const CUtensorMap& q, const CUtensorMap& k,
                              const CUtensorMap& v, const uint8_t* m, void* out, const void* qr, cudaStream_t st)
{
    switch (G.D * 100 + G.tw_log2) {
        case 6402: return attention_variant<64, 2>(G, ob, disk, q, k, v, m, out, qr, st);
        case 6403: return attention_variant<64, 3>(G, ob, disk, q, k, v, m, out, qr, st);
        case 6404: return attention_variant<64, 4>(G, ob, disk, q, k, v, m, out, qr, st);
        case 6405: return attention_variant<64, 5>(G, ob, disk, q, k, v, m, out, qr, st);
        case 12802: return attention_variant<128, 2>(G, ob, disk, q, k, v, m, out, qr, st);
        case 12803: return attention_variant<128, 3>(G, ob, disk, q, k, v, m, out, qr, st);
        case 12804: return attention_variant<128, 4>(G, ob, disk, q, k, v, m, out, qr, st);
        case 12805: return attention_variant<128, 5>(G, ob, disk, q, k, v, m, out, qr, st);
    }
    return TRA_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" tra_status tra_attention(tra_plan plan, const void* q, const void* k, const void* v, const void* mask,
                                    void* out, tra_stream stream)
{
    if (!plan || !q || !k || !v || !mask || !out) return TRA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(mask, 256))
        return TRA_ERR_INVALID_ARG;
    const tra::Geom& G = plan->geom;
    CUtensorMap mq, mk, mv;
    if (!make_input_map(&mq, q, G) || !make_input_map(&mk, k, G) || !make_input_map(&mv, v, G))
        return TRA_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    const uint8_t* m = (const uint8_t*)mask;
    const bool ob = (plan->flags & TRA_FLAG_OUT_BF16) != 0;
    const bool disk = G.disk != 0;
    return dispatch_attention(G, ob, disk, mq, mk, mv, m, out, q, st);
}

extern "C" tra_status tra_calibrate_topk(tra_plan plan, const void* q, const void* k, double mass,
                                         int query_tile_stride, float* H_out, int* k_out, tra_stream stream)
{
    if (!plan || !q || !k || !H_out || !k_out) return TRA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(H_out, 4) || !aligned(k_out, 4)) return TRA_ERR_INVALID_ARG;
    if (!(mass > 0.0 && mass < 1.0) || query_tile_stride < 1) return TRA_ERR_INVALID_ARG;
    const tra::Geom& G = plan->geom;
    const int n_sample = (G.nQ + query_tile_stride - 1) / query_tile_stride;
    CUtensorMap mq, mk;
    if (!make_input_map(&mq, q, G) || !make_input_map(&mk, k, G)) return TRA_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    const float m = (float)mass;
    switch (G.D * 100 + G.tw_log2) {
        case 6402: return run_topk<64, 2>(G, mq, mk, query_tile_stride, n_sample, m, H_out, k_out, st);
        case 6403: return run_topk<64, 3>(G, mq, mk, query_tile_stride, n_sample, m, H_out, k_out, st);
        case 6404: return run_topk<64, 4>(G, mq, mk, query_tile_stride, n_sample, m, H_out, k_out, st);
        case 6405: return run_topk<64, 5>(G, mq, mk, query_tile_stride, n_sample, m, H_out, k_out, st);
        case 12802: return run_topk<128, 2>(G, mq, mk, query_tile_stride, n_sample, m, H_out, k_out, st);
        case 12803: return run_topk<128, 3>(G, mq, mk, query_tile_stride, n_sample, m, H_out, k_out, st);
        case 12804: return run_topk<128, 4>(G, mq, mk, query_tile_stride, n_sample, m, H_out, k_out, st);
        case 12805: return run_topk<128, 5>(G, mq, mk, query_tile_stride, n_sample, m, H_out, k_out, st);
    }
    return TRA_ERR_UNSUPPORTED;
}

extern "C" tra_status tra_plan_status(tra_plan plan)
{
    (void)plan;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, tra::g_tra_error, sizeof word) != cudaSuccess) return TRA_ERR_CUDA;
    if (word) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(tra::g_tra_error, &zero, sizeof zero) != cudaSuccess) return TRA_ERR_CUDA;
    }
    if (word & TRA_ERRBIT_TIMEOUT) return TRA_ERR_TIMEOUT;
    if (word & TRA_ERRBIT_CHECK) return TRA_ERR_DEVICE_CHECK;
    return TRA_OK;
}
