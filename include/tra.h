/*
 * tra.h -- C ABI of the Token Radius Attention (TRA) hot path for NVIDIA B200
 * (sm_100a): per-query attention entropy, entropy -> token budget -> radius,
 * radius -> block-sparse tile mask, and exact-masked block-sparse attention
 * over a T x H x W video-latent token grid.
 *
 * Method: "Token Radius Attention for Efficient Video Generation" (gist.science
 * technical summary), section 2 "Methodologie": Intuition I (the retained
 * density of a query follows its attention entropy log-linearly, so the
 * entropy maps straight to a token budget), Intuition II (a query's dominant
 * keys form a neighbourhood centred on it whose spatial radius shrinks with
 * temporal distance), and "Le Pipeline TRA" (warm-up entropy reused across
 * denoising steps; budget -> radius; tile-major token order; one fused kernel
 * that turns the radius mask into a block-sparse mask).
 *
 * What each call computes (all fp64 decisions, fp32 statistics):
 *   entropy   H_i = -sum_j p_ij ln p_ij,  p_i. = softmax_j(q_i.k_j / sqrt d)
 *   budget    B_i = min(N, max(Bmin, exp(a*H_i + b))),  Bhat_i = ceil(B_i)
 *   radius    r_i = smallest integer r in [0, r_cap] whose neighbourhood
 *             count c_i(r) reaches Bhat_i (else r_cap), where the
 *             neighbourhood of (t,h,w) holds the in-grid keys with
 *             |dt| <= Rt' = min(Rt, T-1) and Chebyshev distance
 *             max(|dh|,|dw|) <= floor(r * gamma^|dt| + 1e-9)
 *   mask      per (head, query tile, key tile): active iff some retained
 *             token pair lies in it; "full" iff every valid pair does
 *   attention O_i = sum_{j in M_i} softmax_j(q_i.k_j/sqrt d) v_j, exactly
 *             masked at token level, inactive tiles skipped.
 *
 * Token order.  The natural order is frame-major, n = (t*H + h)*W + w (the
 * "Token Radius Attention" blog post, sections 5.1 and 9.1).  The kernels
 * work on the tile-major order of "Le Pipeline TRA" ("Disposition
 * Tile-Major"): the grid is cut into (1, tile_h, tile_w) boxes of 128 tokens
 * (tile_h * tile_w = 128, tile_w in {4,8,16,32}), tile index
 * (t*n_tiles_h + h/tile_h)*n_tiles_w + w/tile_w, row (h%tile_h)*tile_w +
 * w%tile_w inside the tile.  Boxes at the bottom/right edge are padded; pad
 * rows are never attended and their outputs are unspecified.
 *
 * Ownership.  The caller allocates every device buffer and the stream; the
 * library allocates no device memory.  A plan holds host scalars only.
 *
 * Errors.  Host-side validation is synchronous and returns a status.  Kernel
 * launches are asynchronous: a failed launch returns TRA_ERR_CUDA.  Faults a
 * kernel detects itself (a bounded wait that gave up; a mask buffer whose
 * tile counts or listed key tiles are out of range) are recorded in a
 * per-device error word and reported by
 * tra_plan_status() after the caller synchronises the stream.  On any error
 * the outputs are unspecified.
 *
 * Thread safety.  A plan is read-only after creation; calls on different
 * streams with distinct buffers may run concurrently.  The device error word
 * is shared by every plan on a device.
 */
#ifndef TRA_H
#define TRA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TRA_API __attribute__((visibility("default")))
#else
#define TRA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* an opaque host-side plan */
typedef struct tra_plan_s* tra_plan;

/* a CUDA stream (the same type as cudaStream_t); NULL = legacy default stream */
typedef struct CUstream_st* tra_stream;

typedef enum {
    TRA_OK = 0,
    TRA_ERR_INVALID_ARG = 1,   /* bad argument: null/misaligned pointer, bad size */
    TRA_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels support */
    TRA_ERR_WORKSPACE = 3,     /* mask buffer smaller than tra_plan_info.mask_bytes */
    TRA_ERR_CUDA = 4,          /* a CUDA runtime/driver call or launch failed */
    TRA_ERR_TIMEOUT = 5,       /* a kernel's bounded wait gave up (device side) */
    TRA_ERR_DEVICE_CHECK = 6   /* a kernel's own index check failed (device side) */
} tra_status;

/* plan flags */
#define TRA_FLAG_TILE_W(tw)    ((unsigned)(tw) << 8)   /* force tile_w (4, 8, 16 or 32) */
#define TRA_FLAG_TILE_W_MASK   (0xFFu << 8)
#define TRA_FLAG_DEBUG_NO_WAIT (1u << 16)  /* test hook: pipeline waits give up at
                                              once, exercising the timeout path */
#define TRA_FLAG_OUT_BF16      (1u << 17)  /* tra_attention writes bf16 instead of fp32 */
#define TRA_FLAG_NATURAL       (1u << 18)  /* q, k, v, out and the entropies are in the
                                              natural frame-major token order
                                              n = (t*H + h)*W + w: [heads][N][d] and
                                              [heads][N], no pad rows.  The kernels
                                              load each (1, th, tw) tile straight from
                                              it with a 4-D TMA box and store results
                                              back to their natural rows, so no
                                              tra_permute pass is needed. */
#define TRA_FLAG_DISK          (1u << 19)  /* Euclidean-disk spatial test
                                              dh^2 + dw^2 <= s^2 (the summary's
                                              circular neighbourhoods) instead of
                                              the Chebyshev square max(|dh|,|dw|)
                                              <= s; same half-width s.  r_cap is
                                              then the smallest r with
                                              s(r, Rt')^2 >= (H-1)^2 + (W-1)^2. */
#define TRA_FLAG_QSORT         (1u << 20)  /* radius-sorted query groups (a scheduling
                                              choice of this library; the results are
                                              the same attention): the rows of each
                                              tile-column strip (one tile column of
                                              one frame: its n_tiles_h tiles, top to
                                              bottom, strip row l = 128*u + i for row
                                              i of the tile in tile row u) are ordered
                                              by (radius, l), pad rows first, and the
                                              u-th block of 128 takes the block-mask
                                              slot of the strip's tile in tile row u.
                                              Each group's key-tile list is the union
                                              over its own queries, so a group of like
                                              radii computes fewer tile pairs than a
                                              spatial tile.  Needs n_tiles_h <= 4;
                                              otherwise TRA_ERR_UNSUPPORTED. */

/* everything a caller needs to size and read buffers */
typedef struct {
    int T, H, W, heads, d;
    int N;                 /* T*H*W tokens per head */
    int N_pad;             /* tile-major rows per head = n_tiles * 128 */
    int tile_h, tile_w;    /* (1, tile_h, tile_w) boxes of 128 tokens */
    int n_tiles_h, n_tiles_w;
    int n_tiles;           /* tiles per head = T * n_tiles_h * n_tiles_w */
    int rt_eff;            /* Rt' = min(Rt, T-1) */
    int r_cap;             /* smallest r with s = floor(r*gamma^Rt' + 1e-9) >= max(H,W)-1;
                              with TRA_FLAG_DISK, s^2 >= (H-1)^2 + (W-1)^2 */
    int list_cap;          /* max key tiles listed per query tile = (2Rt'+1) * tiles/frame */
    size_t mask_bytes;     /* size of the mask buffer tra_radius_and_mask fills */
    /* byte offsets inside the mask buffer (each 256-byte aligned):
       radius     int32  [heads][N_pad]        r_i per tile-major row, -1 on pad rows
       tile_count int32  [heads][n_tiles]      number of active key tiles
       tile_pairs int64  [heads][n_tiles]      sum of c_i(r_i) over the tile's queries
       list       uint16 [heads][n_tiles][list_cap]  active key-tile indices in
                  ascending order; bit 15 set = full tile (no token inside is masked)
       group      uint16 [heads][n_tiles][128]  TRA_FLAG_QSORT only: the query of
                  each slot of the tile's group as a strip row l (row l % 128
                  of the tile in tile row l / 128 of the same tile column and
                  frame); tile_count, tile_pairs and list then describe the
                  group, not the tile.  off_group = 0 without the flag. */
    size_t off_radius, off_tile_count, off_tile_pairs, off_list;
    size_t off_group;
} tra_plan_info;

/*
 * tra_plan_create -- validate the problem and choose the tiling.
 *   T, H, W   token grid (frames, height, width); N = T*H*W >= 1
 *   heads     independent attention problems (batch folded in)
 *   d         head dimension, 64 or 128
 *   a, b      budget map B = exp(a*H + b) ("Token Radius Attention for
 *             Efficient Video Generation", Intuition I: B ~ tau*exp(H_i) is
 *             a = 1, b = ln tau); any finite values
 *   gamma     temporal decay of the radius, 0 < gamma <= 1 (Intuition II,
 *             phi(delta) = exp(-gamma' delta) with gamma = exp(-gamma'))
 *   Rt        temporal reach in frames, 0 <= min(Rt, T-1) <= 31
 *   Bmin      smallest budget, 1 <= Bmin <= N
 *   flags     TRA_FLAG_*; 0 = defaults (tile shape with the least padding; on
 *             a tie the tile's long side runs along the frame's short side,
 *             the taller tile when H <= W)
 * Returns TRA_ERR_INVALID_ARG for impossible values, TRA_ERR_UNSUPPORTED for
 * shapes the kernels do not handle (d not 64/128, H or W above 256, > 32 tile
 * columns per frame, > 32767 tiles per head, > 2048 key tiles listed per
 * query tile, r_cap >= 2^20).  No CUDA call is made.
 */
TRA_API tra_status tra_plan_create(tra_plan* out, int T, int H, int W, int heads, int d,
                           double a, double b, double gamma, int Rt, int Bmin,
                           unsigned flags);

/* release a plan (NULL is ignored) */
TRA_API void tra_plan_destroy(tra_plan plan);

/* copy the plan's sizes and layout into *info; no CUDA call */
TRA_API tra_status tra_plan_query(tra_plan plan, tra_plan_info* info);

/*
 * tra_permute -- reorder rows of d elements between the natural frame-major
 * order and the padded tile-major order ("Le Pipeline TRA", Disposition
 * Tile-Major).
 *   src, dst    device buffers, 16-byte aligned.  to_tile_major = 1: src is
 *               [heads][N][d] natural, dst is [heads][N_pad][d] tile-major with
 *               pad rows written as zeros.  to_tile_major = 0: the reverse (pad
 *               rows of src are ignored).
 *   elem_bytes  2 (bf16 q/k/v rows) or 4 (fp32 attention output rows)
 * src and dst must not overlap.  Asynchronous on `stream`.
 */
TRA_API tra_status tra_permute(tra_plan plan, const void* src, void* dst, int to_tile_major,
                       int elem_bytes, tra_stream stream);

/*
 * tra_entropy -- per-query softmax entropy of the dense warm-up step
 * ("Entropie-vers-Budget": dense warm-up attention with fused entropy
 * extraction) or its estimate from a strided key subsample.
 *   q, k   device bf16 [heads][N_pad][d] tile-major, 16-byte aligned; pad rows
 *          must hold finite values (tra_permute writes zeros)
 *   Hout   device fp32 [heads][N_pad]; pad rows are unspecified
 *          (with TRA_FLAG_NATURAL: q, k bf16 [heads][N][d] and Hout fp32
 *          [heads][N], natural token order)
 *   key_tile_stride  1 = all N keys (exact).  s > 1 = only the valid keys of
 *          key tiles whose index is a multiple of s, plus ln(N / |S|) where S
 *          is that key set (the plug-in entropy of the subsample, shifted so a
 *          uniform distribution still reads ln N).
 * Asynchronous on `stream`.
 */
TRA_API tra_status tra_entropy(tra_plan plan, const void* q, const void* k, float* Hout,
                       int key_tile_stride, tra_stream stream);

/*
 * tra_radius_and_mask -- budget, radius and block-sparse mask in one launch
 * ("Budget-vers-Rayon" and "Noyaux CUDA Fusionnes": distance computation,
 * radius comparison, block pruning and token voting).
 *   Hent       device fp32 [heads][N_pad] tile-major entropies (pad rows ignored);
 *              [heads][N] in natural order with TRA_FLAG_NATURAL
 *   mask       device buffer of at least mask_bytes (tra_plan_info), 256-byte
 *              aligned; layout as described in tra_plan_info.  Every field is
 *              rewritten by each call; entries past tile_count are unspecified.
 * The mask may be reused by later tra_attention calls ("Reutilisation
 * Inter-Etapes").  Asynchronous on `stream`.
 */
TRA_API tra_status tra_radius_and_mask(tra_plan plan, const float* Hent, void* mask, size_t mask_bytes,
                               tra_stream stream);

/*
 * tra_attention -- block-sparse attention with exact token masking
 * (O_i = sum over the retained keys j of softmax(q_i.k_j/sqrt d) v_j):
 * "Token Radius Attention for Efficient Video Generation", section 2,
 * "Execution Efficace" (attention runs on the query-key blocks the radius
 * mask keeps) and "Budget-vers-Rayon" (the token mask itself).
 * Inactive key tiles are skipped; inside listed tiles every token pair is
 * tested, so the result equals dense attention under the token mask.  QK^T
 * and PV run on the tensor cores in bf16 with fp32 accumulation; P is
 * rounded to bf16 and O is normalised by the sum of those rounded values.
 *   q, k, v    device bf16 [heads][N_pad][d] tile-major, 16-byte aligned,
 *              finite pad rows
 *   mask       the buffer written by tra_radius_and_mask for this plan; a
 *              tile count outside [0, list_cap] or a listed tile no query of
 *              the tile can reach is recorded as TRA_ERR_DEVICE_CHECK (read by
 *              tra_plan_status) and never dereferenced
 *   out        device [heads][N_pad][d] tile-major, fp32 (bf16 when the plan
 *              has TRA_FLAG_OUT_BF16); pad rows unspecified
 * With TRA_FLAG_NATURAL q, k, v and out are [heads][N][d] in natural token
 * order (the mask buffer is the same either way).
 * Asynchronous on `stream`.
 */
TRA_API tra_status tra_attention(tra_plan plan, const void* q, const void* k, const void* v,
                         const void* mask, void* out, tra_stream stream);

/*
 * tra_calibrate_topk -- calibration workload (the summary's Intuition I: the
 * key density a query needs follows its entropy, B ~ tau * exp(H_i)).  For the
 * queries of every s-th query tile it returns the dense entropy H_i (computed
 * as tra_entropy with stride 1, bit for bit) and k_i, the fewest of the
 * query's highest-probability keys whose probabilities sum to at least
 * `mass`.  A log-linear fit ln k = a*H + b over the returned pairs gives the
 * plan's (a, b).  k_i is found by bisection on a log2-domain score threshold
 * (33 passes over all keys, scores recomputed on the tensor cores); with
 * near-equal probabilities at the cut it may differ from an exact sort by the
 * keys whose fp32 and exact scores order differently.
 *   q, k    bf16 queries and keys in the plan's layout (as tra_entropy)
 *   mass    0 < mass < 1
 *   query_tile_stride  s >= 1; n_sample = ceil(n_tiles / s) tiles per head
 *   H_out   device fp32 [heads][n_sample][128]: tile-major rows of each
 *           sampled tile (sampled tile i is tile i*s); NaN on pad rows
 *   k_out   device int32 [heads][n_sample][128]; -1 on pad rows
 * Returns TRA_ERR_INVALID_ARG for a mass outside (0, 1) or s < 1.
 * Asynchronous on `stream`.
 */
TRA_API tra_status tra_calibrate_topk(tra_plan plan, const void* q, const void* k, double mass,
                                      int query_tile_stride, float* H_out, int* k_out, tra_stream stream);

/*
 * tra_calibrate_fit -- the plan's budget constants from calibration pairs
 * (the summary's Intuition I: the number of keys a query needs grows
 * log-linearly with its entropy, B ~ tau * exp(H_i); the fit lets the slope
 * differ from 1).  Ordinary least squares of ln k_i on H_i,
 *     ln k = a * H + b,
 * over the rows with k_i >= 1 and a finite H_i (so the pad rows of
 * tra_calibrate_topk, NaN / -1, drop out).  The result goes straight into
 * tra_plan_create(..., a, b, ...).
 *   H, k       HOST arrays of n rows: fp32 entropies and int32 counts (the
 *              outputs of tra_calibrate_topk copied to the host, any order)
 *   a, b       out: slope and intercept
 *   rows_used  out, may be NULL: the number of rows the fit used
 * Returns TRA_ERR_INVALID_ARG for a null pointer, n < 0, fewer than two
 * usable rows, or usable rows that all share one H (a and b are then left
 * unchanged).  Host arithmetic only (fp64); no CUDA call.
 */
TRA_API tra_status tra_calibrate_fit(const float* H, const int32_t* k, long long n, double* a, double* b,
                                     long long* rows_used);

/*
 * tra_plan_status -- read and clear the current device's error word.  Call
 * after synchronising the streams that ran this library's kernels.  Returns
 * TRA_OK, TRA_ERR_TIMEOUT or TRA_ERR_DEVICE_CHECK (or TRA_ERR_CUDA if the
 * read itself failed).
 */
TRA_API tra_status tra_plan_status(tra_plan plan);

/* a static English name for a status */
TRA_API const char* tra_status_string(tra_status s);

#ifdef __cplusplus
}
#endif

#endif /* TRA_H */
