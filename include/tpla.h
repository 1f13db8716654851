/*
 * tpla.h -- C ABI of libtpla.so: TPLA (Tensor-Parallel Latent Attention)
 * decode on NVIDIA B200 (sm_100a).
 *
 * The method (paper "TPLA: Tensor Parallel Latent Attention for Efficient
 * Disaggregated Prefill & Decode Inference", arXiv 2508.15881):
 *   - MLA caches one low-rank latent cKV per token (Abstract).
 *   - TPLA cuts that latent, and each head's (absorbed) query input
 *     dimension, into g shards; every shard runs attention on its own slice
 *     with its own softmax, and the shard results are added by an
 *     all-reduce (Abstract; edgentiq blog "Introducing TPLA").
 *   - Before slicing, an orthogonal transform (Hadamard or PCA) is applied
 *     to the latent, and RMSNorm is computed per shard (edgentiq blog
 *     "How TPLA Works: Smart Slicing and Reparameterization"; paperbot
 *     summary, extended abstract).
 * On one GPU the all-reduce is an on-chip sum in the combine kernel.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library allocates no device memory per call.  Scratch space is the
 *     caller's `workspace`, sized by tpla_decode_workspace_size().
 *   - Every tensor is dense, row-major (C order), 16-byte aligned.
 *   - bf16 values are passed as raw 16-bit patterns (tpla_bf16).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work
 *     is enqueued asynchronously on it; nothing is synchronised unless the
 *     function says so.
 *   - Kernels are launched with programmatic stream serialisation: one may
 *     start while the previous kernel on the stream is finishing, if that
 *     kernel allows it early.  This library's kernels allow it only after
 *     their own wait, and wait for the previous kernel before they read any
 *     argument, with one exception: the combine stage (tpla_combine, and the
 *     second stage of tpla_decode / tpla_decode_shard / mla_decode) reads
 *     w_uv and seq_lens before that wait.  So when tpla_combine follows a
 *     kernel of the caller's own that signals programmatic completion early
 *     (griddepcontrol.launch_dependents), that kernel must not write w_uv or
 *     seq_lens after its signal.
 *   - Return value: TPLA_OK, or a tpla_status_t.  A non-zero status means
 *     nothing was enqueued, except TPLA_ERR_CUDA (a launch failed).
 *     Errors that only the device can see (a sequence longer than its
 *     pages, a page index outside the cache, an append position outside the
 *     sequence's pages, a pipeline wait that ran out) are recorded in a
 *     per-device status word and reported by tpla_check_device_status().
 *
 * Cache layout (fixed when the cache is allocated, by g):
 *   ckv_cache [num_pages][g][64][L/g]   bf16   shard-contiguous pages:
 *             token slot t of page p, shard s, starts at
 *             ((p*g + s)*64 + t) * (L/g) elements; rows are L/g*2 bytes.
 *   kpe_cache [num_pages][64][R]        bf16   the decoupled RoPE key, one
 *             copy shared by all shards (every shard adds the full
 *             q_pe . k_pe term to its scores).
 *   Token i of sequence b lives in page block_table[b][i/64], slot i%64.
 *   block_table may be NULL: then page = b*max_pages_per_seq + i/64.
 *
 * Query basis: q_nope_absorbed is the absorbed query W_UK q_nope expressed
 * in the transformed latent basis (R . (gamma * W_UK q)), and w_uv holds the
 * W_UV rows in the same basis, so the cache holds the transformed,
 * per-shard-normalised latent that tpla_append_kv writes.
 */
#ifndef TPLA_H
#define TPLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t tpla_bf16;             /* raw bfloat16 bit pattern */

typedef enum {
    TPLA_OK = 0,
    TPLA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, misaligned pointer */
    TPLA_ERR_UNSUPPORTED = 2,   /* a size outside the supported set (see tpla_dims_t) */
    TPLA_ERR_LAYOUT = 3,        /* cache layout does not match the call (mla_decode with g != 1) */
    TPLA_ERR_WORKSPACE = 4,     /* workspace NULL or smaller than tpla_decode_workspace_size() */
    TPLA_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
    TPLA_ERR_TIMEOUT = 6,       /* a bounded device wait ran out (device status) */
    TPLA_ERR_INDEX = 7          /* a device-side index was out of range (device status) */
} tpla_status_t;

/*
 * Problem sizes.  Supported set:
 *   1 <= H <= 128;  L in {64, 128, 256, 512, 1024} with L % g == 0;
 *   g in {1, 2, 4, 8} with L/g in {32, 64, 128, 256, 512};
 *   R in {16, 32, 64};  1 <= dv <= 256, dv % 8 == 0;  page_size == 64;
 *   B >= 0 (B == 0 is a no-op);  max_pages_per_seq >= 1;  num_pages >= 1.
 *   softmax_scale: multiplies every score (the usual 1/sqrt(qk_nope + R)).
 */
typedef struct {
    int B;                  /* sequences in the batch (decode) / new tokens (append) */
    int H;                  /* attention heads */
    int L;                  /* latent width, kv_lora_rank */
    int R;                  /* decoupled RoPE key width */
    int dv;                 /* value head width (columns of W_UV) */
    int g;                  /* latent shards (TP degree the cache is laid out for) */
    int page_size;          /* tokens per page, must be 64 */
    int max_pages_per_seq;  /* columns of block_table */
    int num_pages;          /* pages in ckv_cache / kpe_cache */
    float softmax_scale;
} tpla_dims_t;

/* Human-readable name of a status code (static storage, never NULL). */
const char* tpla_status_string(int status);

/*
 * Bytes of workspace every decode entry point below needs for `dims`
 * (the same bound covers all shards, one shard, and mla_decode).
 * Host-only; returns 0 if `dims` is NULL or unsupported.
 */
size_t tpla_decode_workspace_size(const tpla_dims_t* dims);

/*
 * tpla_decode -- one decode step over all g shards, shard results summed on
 * the GPU (the all-reduce of the TPLA Abstract as an on-chip sum).
 *
 *   q_nope_absorbed [B][H][L] bf16   absorbed queries, transformed basis
 *   q_pe            [B][H][R] bf16   RoPE part of the queries (post-RoPE)
 *   ckv_cache, kpe_cache             cache, layout above, read only
 *   block_table     [B][max_pages_per_seq] int32, or NULL (identity)
 *   seq_lens        [B] int32        tokens to attend to per sequence
 *                                    (0 gives an all-zero output row)
 *   w_uv            [H][L][dv] bf16  per-head up-projection, or NULL
 *   out             w_uv != NULL: [B][H][dv] fp32
 *                                   out[b,h] = sum_s W_UV_h[s*L/g:(s+1)*L/g]^T o_{b,h,s}
 *                   w_uv == NULL: [B][H][L] fp32, the shard outputs o_{b,h,s}
 *                                 side by side (latent-space attention output)
 *   workspace       device scratch of ws_bytes >= tpla_decode_workspace_size(dims)
 * Per shard s and head h:  z_t = scale * (q~_h[s-slice] . c_{t,s} + q_pe_h . k_pe_t),
 * p = softmax_t(z),  o_{b,h,s} = sum_t p_t c_{t,s}   (t < seq_lens[b]).
 */
int tpla_decode(const tpla_dims_t* dims,
                const tpla_bf16* q_nope_absorbed, const tpla_bf16* q_pe,
                const tpla_bf16* ckv_cache, const tpla_bf16* kpe_cache,
                const int32_t* block_table, const int32_t* seq_lens,
                const tpla_bf16* w_uv, float* out,
                void* workspace, size_t ws_bytes, void* stream);

/*
 * tpla_decode_shard -- exactly the work of tensor-parallel rank `shard`
 * (0 <= shard < g) at TP degree g (TPLA Abstract: each device holds one
 * slice of the latent): reads only shard `shard` of ckv_cache, the RoPE
 * cache, the query columns [shard*L/g, (shard+1)*L/g) and the matching
 * W_UV rows.  Arguments as tpla_decode (full-width q and w_uv), except
 *   out   w_uv != NULL: [B][H][dv] fp32, this rank's term
 *                       W_UV_h[s-rows]^T o_{b,h,s} (the all-reduce input);
 *         w_uv == NULL: [B][H][L/g] fp32, o_{b,h,s}.
 */
int tpla_decode_shard(const tpla_dims_t* dims, int shard,
                      const tpla_bf16* q_nope_absorbed, const tpla_bf16* q_pe,
                      const tpla_bf16* ckv_cache, const tpla_bf16* kpe_cache,
                      const int32_t* block_table, const int32_t* seq_lens,
                      const tpla_bf16* w_uv, float* out,
                      void* workspace, size_t ws_bytes, void* stream);

/*
 * mla_decode -- plain MLA decode in absorbed form: tpla_decode on a cache
 * laid out with g == 1 (TPLA with one shard is MLA; the Abstract calls TPLA
 * drop-in for MLA checkpoints).  dims->g != 1 returns TPLA_ERR_LAYOUT.
 */
int mla_decode(const tpla_dims_t* dims,
               const tpla_bf16* q_nope_absorbed, const tpla_bf16* q_pe,
               const tpla_bf16* ckv_cache, const tpla_bf16* kpe_cache,
               const int32_t* block_table, const int32_t* seq_lens,
               const tpla_bf16* w_uv, float* out,
               void* workspace, size_t ws_bytes, void* stream);

/*
 * tpla_decode_static -- tpla_decode for callers that cannot allocate device
 * memory and so cannot pass a workspace: code running inside a memory-pool or
 * allocator callback, under a framework that owns all device memory, or in a
 * loop where an allocation may block.  The TPLA paper has no counterpart;
 * this is a property of this library only.
 *
 * Same arguments and result as tpla_decode, without workspace/ws_bytes.
 * Its scratch is one file-scope device array of 32 MiB, which every GPU that
 * loads the library holds until the process exits; the call allocates and
 * frees nothing (no cudaMalloc, no allocating library routine).
 *   - Size limit: the split-KV partials of B*g (sequence, shard) pairs plus at
 *     least one worker must fit in 32 MiB, i.e. roughly
 *     (B*g + 1) * H * (L/g) * 4 bytes plus a small header; larger problems
 *     return TPLA_ERR_WORKSPACE with nothing enqueued.  Near the limit the
 *     call uses fewer split-KV workers than tpla_decode (same result up to
 *     fp32 rounding, possibly slower).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, once per device, with that device current);
 *     make that first call before any stream capture.
 *   - Every call on a device shares the one array, and it keeps the last
 *     call's contents (nothing in it needs to start at zero).  Calls that
 *     overlap on the GPU (different streams, or two host threads) race on
 *     it: order them, e.g. on one stream.
 */
int tpla_decode_static(const tpla_dims_t* dims,
                       const tpla_bf16* q_nope_absorbed, const tpla_bf16* q_pe,
                       const tpla_bf16* ckv_cache, const tpla_bf16* kpe_cache,
                       const int32_t* block_table, const int32_t* seq_lens,
                       const tpla_bf16* w_uv, float* out, void* stream);

/*
 * The two stages of a decode call, for callers that time or overlap them.
 * tpla_attention runs the split-KV attention of all shards (shard == -1) or
 * of one shard and leaves per-split partial outputs and log-sum-exps in
 * `workspace`; tpla_combine then merges the splits, applies W_UV (or not)
 * and sums over shards into `out`, exactly as tpla_decode /
 * tpla_decode_shard document.  The combine must use the same dims, shard,
 * seq_lens contents and workspace as the attention call before it, on the
 * same stream (or after it in stream order), with the same options set (the options decide the
 * attention kernel, and with it the split-KV worker count the combine expects).
 */
int tpla_attention(const tpla_dims_t* dims, int shard,
                   const tpla_bf16* q_nope_absorbed, const tpla_bf16* q_pe,
                   const tpla_bf16* ckv_cache, const tpla_bf16* kpe_cache,
                   const int32_t* block_table, const int32_t* seq_lens,
                   void* workspace, size_t ws_bytes, void* stream);

int tpla_combine(const tpla_dims_t* dims, int shard, const int32_t* seq_lens,
                 const tpla_bf16* w_uv, float* out,
                 void* workspace, size_t ws_bytes, void* stream);

/* transform argument of tpla_append_kv */
#define TPLA_TRANSFORM_NONE      0   /* identity */
#define TPLA_TRANSFORM_HADAMARD  1   /* Sylvester Hadamard / sqrt(L), natural order; L a power of two */
#define TPLA_TRANSFORM_DENSE     2   /* caller's orthogonal R_dense (e.g. a PCA basis) */
#define TPLA_TRANSFORM_BLOCK_HADAMARD 3  /* block-diagonal: Sylvester Hadamard / sqrt(L/g) on each
                                            shard's L/g columns of x, so a shard's values depend on
                                            its own slice only (edgentiq blog, "Real-World Impact
                                            and Future Directions": cheaper Hadamard-like transforms
                                            as the next step); equals HADAMARD when g == 1 */

/*
 * tpla_append_kv -- write one new token per sequence into the cache
 * (edgentiq blog "How TPLA Works": orthogonal transform before slicing,
 * then RMSNorm computed per shard).  For new token b (0 <= b < dims->B):
 *   y   = R x_b                  (x_b = latent_raw[b], the pre-norm latent)
 *   c_s = y_s / sqrt(mean(y_s^2) + eps) [* norm_weight[s-slice]]  per shard s
 *   ckv_cache[page][s][slot][:] = bf16_rn(c_s),   kpe_cache[page][slot][:] = kpe_new[b]
 * with page = block_table[b][positions[b] / 64] (or the identity layout) and
 * slot = positions[b] % 64.
 *   latent_raw  [B][L] bf16;  kpe_new [B][R] bf16 (post-RoPE);
 *   transform   TPLA_TRANSFORM_* (an unknown value returns TPLA_ERR_INVALID_ARG);
 *               R_dense [L][L] fp32 row-major (y_i = sum_j R[i][j] x_j),
 *               required for TPLA_TRANSFORM_DENSE, ignored otherwise;
 *   norm_weight [L] fp32 or NULL (weight applied in the transformed basis);
 *   eps         added to the mean square (>= 0);
 *   positions   [B] int32 device array: slot index of the new token
 *               (usually the sequence length before the append; the caller
 *               increments seq_lens).  A position outside
 *               [0, 64*max_pages_per_seq) or a page outside [0, num_pages) is
 *               skipped and recorded as TPLA_ERR_INDEX in the device status.
 */
int tpla_append_kv(const tpla_dims_t* dims,
                   const tpla_bf16* latent_raw, const tpla_bf16* kpe_new,
                   int transform, const float* R_dense, const float* norm_weight, float eps,
                   const int32_t* positions, const int32_t* block_table,
                   tpla_bf16* ckv_cache, tpla_bf16* kpe_cache, void* stream);

/*
 * tpla_append_kv_shard -- the append of one tensor-parallel rank: the same transform of the whole
 * new latent x_b and the RMSNorm of shard `shard` (0 <= shard < dims->g) only, written into a cache
 * that holds that shard alone (TPLA Abstract: each device keeps its slice of the latent):
 *   ckv_shard_cache [num_pages][64][L/g] bf16: token slot t of page p starts at (p*64 + t) * (L/g)
 *   kpe_cache       [num_pages][64][R]   bf16 (every rank keeps the whole RoPE key)
 * Other arguments, results and errors as tpla_append_kv; shard outside [0, g) returns
 * TPLA_ERR_INVALID_ARG.  A rank then decodes its shard with tpla_decode on dims with L = L/g and
 * g = 1, its slice q~[:, :, shard*L/g : (shard+1)*L/g] of the absorbed query and its rows of W_UV;
 * the sum of the ranks' outputs (an all-reduce) is tpla_decode's result on the g-shard cache.
 */
int tpla_append_kv_shard(const tpla_dims_t* dims, int shard,
                         const tpla_bf16* latent_raw, const tpla_bf16* kpe_new,
                         int transform, const float* R_dense, const float* norm_weight, float eps,
                         const int32_t* positions, const int32_t* block_table,
                         tpla_bf16* ckv_shard_cache, tpla_bf16* kpe_cache, void* stream);

/*
 * Synchronises `stream`, then returns and clears the current device's status
 * word: TPLA_OK, TPLA_ERR_INDEX or TPLA_ERR_TIMEOUT (or TPLA_ERR_CUDA if the
 * stream reports an error).
 */
int tpla_check_device_status(void* stream);

/* Options (process-wide, for testing and tuning). */
#define TPLA_OPT_ATTENTION_KERNEL  1  /* 0 auto (tcgen05 where supported), 1 CUDA-core kernel, 2 tcgen05 kernel
                                         (R == 64 and L/g in {64, 128, 256, 512}; other shapes return
                                         TPLA_ERR_UNSUPPORTED) */
#define TPLA_OPT_MAX_WORKERS       2  /* cap on split-KV workers per call (0 = one per SM) */
#define TPLA_OPT_WAIT_LIMIT        3  /* spin iterations before a pipeline wait gives up (0 = default) */
#define TPLA_OPT_DEBUG_STALL       4  /* 1: the tcgen05 kernel waits on a barrier nothing signals, to
                                         exercise the bounded-wait path (returns TPLA_ERR_TIMEOUT) */
#define TPLA_OPT_LAST_ATTENTION_KERNEL 5  /* read-only: kernel of the last attention launch in this
                                             process (0 none yet, 1 CUDA-core, 2 tcgen05 with 128-token
                                             tiles (L/g <= 256), 3 tcgen05 CTA pair (L/g == 512)) */
#define TPLA_OPT_TILE_TOKENS       6  /* tokens per tile of the tcgen05 kernel for L/g <= 256: 64 (one page per
                                         tile, more stages in flight) or 128 (two pages, fewer QK^T steps per
                                         token); 0 = the library's default.  Results are the same up to fp32
                                         rounding order. */
int tpla_set_option(int option, int value);
int tpla_get_option(int option);

/* Version string of the library build. */
const char* tpla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TPLA_H */
