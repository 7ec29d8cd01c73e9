/*
 * vggt_attn.h -- C ABI of libvggt_attn.so: the attention core of the VGGT
 * aggregator (frame, global and compressed-descriptor attention, each with a
 * fused per-head QK LayerNorm + 2D RoPE prologue) for NVIDIA B200 (sm_100a).
 *
 * Operation (all variants, per head h):
 *   q_hat = RoPE2D(LayerNorm(q), pos),  k_hat = RoPE2D(LayerNorm(k), pos_k)
 *   out_i = sum_j softmax_j(q_hat_i . k_hat_j / sqrt(D)) v_j
 * - LayerNorm over the D = 64 dims of one head, centered, biased variance,
 *   eps = 1e-5, no scale/shift ("Norm: Layer Normalization" slide of the VGGT
 *   paper-report deck; layer_norm_eps 1e-05 in the VGGT-Omega config.json
 *   field table).
 * - 2D RoPE, base 100 (rope_base 100.0, VGGT-Omega config.json field table):
 *   dims 0-31 turn by the row position, dims 32-63 by the column position;
 *   inside each half, dim j pairs with dim j+16 and turns by
 *   pos * 100^(-2j/32) (frequency schedule of the sinusoidal formula on the
 *   deck's "Positional Encoding (4/6)" slide).
 * - softmax(Q K^T / sqrt(d_k)) V: deck, Section V "Attention" slides.
 *
 * Data layout (every pointer is DEVICE memory owned by the caller):
 *   q, k, v, out : [S, T, H, D] bf16 (raw uint16 bits), contiguous, token-major
 *                  with heads interleaved -- the [B, N, H, D] layout of the
 *                  vggt-jax README attention table.
 *   pos          : [S, T, 2] fp32 (row, col). VGGT places the five special
 *                  tokens (camera + 4 registers) at (0, 0) and patch (r, c) at
 *                  (r + 1, c + 1); the library uses whatever pos holds.
 *   Each frame holds T = 5 + g*g tokens: the 5 special tokens first, then the
 *   g x g patch grid row-major. Only the descriptor pooling depends on this
 *   order; frame and global attention use pos alone. The _ex calls lift this:
 *   frame and global attention take any T >= 1, and the descriptor calls
 *   take a vggt_frame_layout (rectangular grid, trailing tokens).
 *
 * Common rules:
 *   - D must be 64 (VGGT: 16 heads x 64 dims). H >= 1 is free.
 *   - Every bf16 pointer must be 16-byte aligned (TMA and 16-byte vector
 *     access); positions (pos, pos_out) 8-byte aligned (read as pairs).
 *   - S == 0 or H == 0 is an empty problem: VGGT_OK, nothing is launched.
 *   - Everything is asynchronous on `stream`; no call synchronises it.
 *   - Scratch (normalised q/k, pooled k/v) comes from a stream-ordered memory
 *     pool the library owns (one per device) and is released to it with
 *     cudaFreeAsync on `stream`. The pool keeps that memory for later calls
 *     instead of returning it to the system at every synchronisation (which
 *     would cost milliseconds of host time per call to take it back), so
 *     after a call the library holds up to the largest scratch any call
 *     needed -- about 4 * S*T * H * D bytes; vggt_release_scratch returns it.
 *     The environment variable VGGT_SCRATCH_POOL_MAX_BYTES (a positive decimal
 *     byte count), read when a device's pool is created, caps that pool: a
 *     call whose scratch does not fit returns VGGT_ERR_ALLOC and launches
 *     nothing. Calls that need no scratch (vggt_attn_core,
 *     vggt_attn_global_noalloc, the status and wait-limit calls) never create
 *     the pool.
 *   - Outputs must not overlap inputs.
 *   - Every argument is checked on the host before any launch; an invalid call
 *     returns a negative vggt_status and launches nothing.
 *   - No call traps on the device. Device-side waits are bounded; a wait that
 *     runs out sets a device status word that vggt_get_device_status() reads.
 *   - The attention calls can be captured into a CUDA graph (stream capture on
 *     `stream`); a replay repeats the call on the same buffers. The first call
 *     on each device creates the library's scratch pool and sets kernel
 *     attributes, which cannot happen during a capture: make one ordinary
 *     call per device (and per variant: frame/global/descriptor, fp32 mode)
 *     before capturing.
 *   - Every kernel is launched with programmatic dependent launch and waits
 *     (griddepcontrol.wait) for the previous work in its stream to complete
 *     before it touches memory, so calls are ordered in their stream exactly
 *     as ordinary launches are. A caller's own kernel that it launches right
 *     after a call with the programmatic-stream-serialization attribute may
 *     start early, like the library's, and must wait the same way before it
 *     reads the call's outputs.
 *   - Host threads may call the library concurrently (each on its own
 *     stream); a device's one-time set-up is serialised inside. A descriptor
 *     cache handle is not: one thread (or one stream order) at a time.
 *     vggt_set_wait_limit is meant for set-up, not for concurrent use.
 */
#ifndef VGGT_ATTN_H
#define VGGT_ATTN_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define VGGT_API __attribute__((visibility("default")))
#else
#define VGGT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t vggt_bf16; /* raw bf16 bits */

typedef enum vggt_status {
    VGGT_OK = 0,
    VGGT_ERR_NULL = -1,        /* a required pointer is NULL                      */
    VGGT_ERR_UNSUPPORTED = -2, /* D != 64, a misaligned pointer, a cache used on
                                  another device than its own, or a QK LayerNorm
                                  affine that is not finite (see vggt_qk_norm)    */
    VGGT_ERR_SHAPE = -3,       /* negative sizes, T != 5 + g*g (plain calls) or a
                                  layout that does not add up to T, bad kv_down, or
                                  a size beyond the library's limits              */
    VGGT_ERR_ALLOC = -4,       /* scratch allocation failed (device memory, or the
                                  VGGT_SCRATCH_POOL_MAX_BYTES cap); nothing was
                                  launched and no output written                  */
    VGGT_ERR_CUDA = -5,        /* a CUDA runtime call or launch failed             */
    VGGT_ERR_TIMEOUT = -6,     /* a bounded device-side wait ran out (reported by
                                  vggt_get_device_status)                          */
    VGGT_ERR_RANGE = -7        /* an attention row's softmax sum was not a positive
                                  finite number: vggt_attn_core was given vectors
                                  outside its norm bound (use vggt_attn_core_online
                                  for those; reported by vggt_get_device_status)  */
} vggt_status;

/* Number of special (camera + register) tokens at the head of every frame. */
#define VGGT_N_SPECIAL 5
/* Head dimension the kernels are built for. */
#define VGGT_HEAD_DIM 64
/* Largest S*T (or S*T_k) accepted: keeps every row index inside int32 and
   every tensor below 2^31 elements of one head-major scratch plane. */
#define VGGT_MAX_TOKENS (1 << 21)

/*
 * Frame attention: every token attends only to the T tokens of its own frame
 * ("Frame Attention" panel, "Global + Frame Attention" architecture slide).
 * kv_down must be 0 or 1. Writes out[S, T, H, D].
 */
VGGT_API int vggt_attn_frame(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                    const float* pos, vggt_bf16* out,
                    int S, int T, int H, int D, int kv_down, cudaStream_t stream);

/*
 * Global attention: all S*T tokens attend to all S*T tokens ("Global
 * Attention" panel of the same slide; vggt-jax README global shape
 * [1, 1860, 16, 64]). kv_down must be 0 or 1. Writes out[S, T, H, D].
 */
VGGT_API int vggt_attn_global(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                     const float* pos, vggt_bf16* out,
                     int S, int T, int H, int D, int kv_down, cudaStream_t stream);

/*
 * Compressed-descriptor attention (FlashVGGT README, Overview; --kv_downfactor,
 * default 4): K/V are first pooled per frame as vggt_kv_pool does, then every
 * query of every frame attends to all S frames' descriptors (S * T_k keys).
 * The pooled keys get the prologue at their pooled positions; pooled values
 * are used as stored. kv_down >= 1 (kv_down == 1 is dense global attention).
 * Writes out[S, T, H, D].
 */
VGGT_API int vggt_attn_descriptor(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                         const float* pos, vggt_bf16* out,
                         int S, int T, int H, int D, int kv_down, cudaStream_t stream);

/*
 * The QK prologue on its own: for every token t < N and head h < H,
 *   x_hat[h, t, :] = RoPE2D(LayerNorm(x[t, h, :]), pos[t])
 * with the LayerNorm and rotary embedding defined at the top of this header.
 * x [N, H, D] bf16 token-major in; x_hat [H, N, D] bf16 head-major out (the
 * layout the attention kernel reads); pos [N, 2] fp32. The attention entry
 * points run this step internally; it is exported for users who need the
 * normalised, rotated vectors themselves. N == 0 or H == 0 is a no-op.
 */
VGGT_API int vggt_qk_prologue(const vggt_bf16* x, const float* pos, vggt_bf16* x_hat,
                              int N, int H, int D, cudaStream_t stream);

/*
 * Attention on vectors that already went through the prologue (for callers
 * that reuse normalised keys across calls, or attend between arbitrary token
 * sets). Segment s (0 <= s < n_seg): queries [s*q_len, (s+1)*q_len) attend to
 * keys [s*k_len, (s+1)*k_len); softmax(q_hat k_hat^T / sqrt(D)) v.
 *   q_hat [H, n_seg*q_len, D], k_hat [H, n_seg*k_len, D] bf16 head-major (the
 *   layout vggt_qk_prologue writes); v [n_seg*k_len, H, D] and
 *   out [n_seg*q_len, H, D] bf16 token-major.
 * Frame attention is n_seg = S, q_len = k_len = T; global attention is
 * n_seg = 1, q_len = k_len = S*T. Takes no scratch. n_seg, q_len or k_len
 * == 0, or H == 0, is a no-op.
 * Norm bound: the softmax is evaluated as exp(score) with no row maximum
 * subtracted, which is exact up to rounding because softmax ignores a common
 * factor, and safe because the prologue's vectors have norm below 8 (so
 * |score| < 8). Every head vector of q_hat and k_hat must have Euclidean norm
 * at most 16 (|score| <= 32, exponentials within 2^+-46); beyond that the
 * fp32/bf16 exponentials and sums may overflow. A row whose sum of exponentials is not a positive finite number
 * sets VGGT_ERR_RANGE for vggt_get_device_status (best effort: results of
 * out-of-bound inputs are undefined either way).
 */
VGGT_API int vggt_attn_core(const vggt_bf16* q_hat, const vggt_bf16* k_hat, const vggt_bf16* v,
                            vggt_bf16* out, int n_seg, int q_len, int k_len, int H, int D,
                            cudaStream_t stream);

/*
 * vggt_attn_core for any finite q_hat and k_hat: the softmax keeps a running
 * row maximum (FlashAttention's online softmax, "Attention" slides of the
 * VGGT paper-report deck, Section V) and rescales the row's sums only when
 * that maximum grows by more than 2^8 in exp2 terms. Same arguments, layouts
 * and rules as vggt_attn_core; no norm bound. Unlike vggt_attn_core it keeps
 * q_hat exactly as given (the core scales q_hat by log2(e)/8 and rounds it to
 * bf16 once more), so scores are exact fp32 dot products of the bf16 inputs.
 * Slower than vggt_attn_core (a shared-memory exchange of block maxima per
 * key block). Takes no scratch.
 */
VGGT_API int vggt_attn_core_online(const vggt_bf16* q_hat, const vggt_bf16* k_hat, const vggt_bf16* v,
                                   vggt_bf16* out, int n_seg, int q_len, int k_len, int H, int D,
                                   cudaStream_t stream);

/*
 * Per-frame K/V descriptors (FlashVGGT README: "spatially resampling keys and
 * values"; the grid is g x g with g = sqrt(T - 5)):
 *   - the 5 special tokens of each frame are copied unchanged;
 *   - the grid is cut into ceil(g/kv_down)^2 cells of up to kv_down x kv_down
 *     patches (edge cells keep only the patches inside the grid); each cell
 *     becomes one token whose K and V are, per channel, the float32 sum of its
 *     members in row-major order divided in float32 by the member count and
 *     rounded to bf16 (nearest, ties to even); its position is the same
 *     float32 mean of the members' positions.
 * Outputs: k_out, v_out [S, T_k, H, D] bf16, pos_out [S, T_k, 2] fp32 with
 * T_k = vggt_kv_pool_tokens(T, kv_down). kv_down >= 1.
 */
VGGT_API int vggt_kv_pool(const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                 vggt_bf16* k_out, vggt_bf16* v_out, float* pos_out,
                 int S, int T, int H, int D, int kv_down, cudaStream_t stream);

/*
 * Streaming (chunk-recursive) descriptor attention -- the FlashVGGTStream
 * mode: "the compactness of the descriptors enables online inference over
 * long sequences via a chunk-recursive mechanism that reuses cached
 * descriptors from previous chunks" (FlashVGGT README, Overview; streaming
 * inference with --chunksize, default 10, Key Arguments). Frames arrive in
 * chunks; every query of a chunk attends to the descriptors of all frames
 * seen so far -- the cached descriptors of earlier chunks and its own
 * chunk's (pooled exactly as vggt_kv_pool, keys normalised by the prologue
 * at their cell-mean positions).
 *
 * A vggt_desc_cache holds those descriptors on one device: normalised keys,
 * values and positions of up to max_frames frames. It is owned by the caller
 * (create / destroy) and used by one sequence at a time (reset starts a new
 * one). Calls that use a cache must be ordered by the caller (one stream, or
 * streams synchronised with each other).
 */
typedef struct vggt_desc_cache vggt_desc_cache;

/* Creates a cache on the current device for up to max_frames frames of T =
   5 + g*g tokens, H heads of D = 64 dims, pooled kv_down x kv_down. Takes
   max_frames * T_k * H * D * 2 * 2 + max_frames * T_k * 8 bytes with
   cudaMalloc (T_k = vggt_kv_pool_tokens(T, kv_down)). On failure *cache is
   NULL and a negative vggt_status is returned (VGGT_ERR_NULL, _SHAPE,
   _UNSUPPORTED for D != 64, _ALLOC, _CUDA). Host only; synchronous. */
VGGT_API int vggt_desc_cache_create(vggt_desc_cache** cache, int max_frames, int T, int H, int D,
                                    int kv_down);

/* Frees the cache's memory (cudaFree, on the cache's device) and the cache.
   NULL is a no-op. Make sure no call that uses it is still running. */
VGGT_API int vggt_desc_cache_destroy(vggt_desc_cache* cache);

/* Frames the cache holds (>= 0), or VGGT_ERR_NULL. Host only. */
VGGT_API int vggt_desc_cache_frames(const vggt_desc_cache* cache);

/* Forgets every cached frame (a new sequence). Host only; no device work. */
VGGT_API int vggt_desc_cache_reset(vggt_desc_cache* cache);

/*
 * One chunk of C frames of the sequence:
 *   1. pools the chunk's K/V per frame (as vggt_kv_pool) and appends the
 *      descriptors to the cache, their keys normalised once, in the cache;
 *   2. every token of the chunk attends to all descriptors now in the cache.
 * q, k, v, out: [C, T, H, D] bf16; pos [C, T, 2] fp32 (the cache's T, H, D).
 * out is the same as vggt_attn_descriptor over all frames cached so far,
 * restricted to the chunk's queries. Runs on the cache's device (else
 * VGGT_ERR_UNSUPPORTED); fails with VGGT_ERR_SHAPE, launching nothing and
 * leaving the cache unchanged, if the chunk does not fit. C == 0 is a no-op.
 * The cache's frame count grows by C when the call returns VGGT_OK.
 * Scratch: the chunk's q_hat, from the scratch pool. Three launches: the
 * query prologue, the pooling fused with the prologue of the new keys, then
 * the attention.
 */
VGGT_API int vggt_attn_descriptor_chunk(vggt_desc_cache* cache, const vggt_bf16* q,
                                        const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                                        vggt_bf16* out, int C, cudaStream_t stream);

/* ------------------------------------------------------------------ _ex calls
 *
 * Frame layout: every frame holds n_front special tokens, then a
 * grid_h x grid_w patch grid in row-major order, then n_back trailing tokens:
 * T = n_front + grid_h * grid_w + n_back. VGGT-1B frames are {5, g, g, 0}
 * (the default wherever a layout pointer may be NULL); the vggt-jax README's
 * two-image benchmark feeds 350 x 518 images, a 25 x 37 grid; the VGGT-Omega
 * page appends its 16 register tokens after each frame's patches
 * ({0, 32, 32, 16} at 512 px, patch 16). Pooling copies front and trailing
 * tokens and averages the grid's cells: a pooled frame is the n_front
 * tokens, the ceil(grid_h/kv_down) x ceil(grid_w/kv_down) cells row-major,
 * then the n_back tokens.
 */
typedef struct vggt_frame_layout {
    int n_front;
    int grid_h;
    int grid_w;
    int n_back;
} vggt_frame_layout;

/*
 * QK LayerNorm affine: after the per-head LayerNorm, y = y * weight + bias per
 * dim, the same D = 64 values for every head (the scale and shift a trained
 * LayerNorm carries; the pages give none, so without it there is no affine).
 * Separate arrays for queries and keys; each is a HOST array of D fp32
 * values or NULL (weight 1, bias 0), read during the call (no reference is
 * kept). Values must be finite; any finite values are accepted.
 * Which softmax runs: with Bq = 8 * max|q_weight| + ||q_bias||_2 (a bound on
 * the norm of a normalised query, the plain LayerNorm's being below 8) and Bk
 * likewise, every score is at most Bq * Bk / 8 in magnitude. While
 * Bq * Bk / 8 * log2(e) * 1.01 <= 64 (e.g. weights up to 2.3 with zero bias)
 * the attention kernel evaluates exp(score) without a row maximum (exact up
 * to rounding: softmax ignores a common factor); beyond it the kernel keeps a
 * running row maximum and rescales its sums when it grows (online softmax).
 * Both give the same result up to rounding. Large affines make the scores
 * large, and the normalised q and k are stored in bf16 (relative rounding
 * 2^-9 per element), so a score's error grows with Bq * Bk: results stay
 * close to exact only while that error (about 2^-9 * |q_hat| * |k_hat| / 8)
 * is small beside the gaps between a row's largest scores.
 */
typedef struct vggt_qk_norm {
    const float* q_weight;
    const float* q_bias;
    const float* k_weight;
    const float* k_bias;
} vggt_qk_norm;

/* vggt_attn_frame / vggt_attn_global with any T >= 1 (these do not look at
   the token order) and an optional QK LayerNorm affine (norm may be NULL). */
VGGT_API int vggt_attn_frame_ex(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                                const float* pos, vggt_bf16* out, int S, int T, int H, int D,
                                const vggt_qk_norm* norm, cudaStream_t stream);
VGGT_API int vggt_attn_global_ex(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                                 const float* pos, vggt_bf16* out, int S, int T, int H, int D,
                                 const vggt_qk_norm* norm, cudaStream_t stream);

/* vggt_attn_descriptor with a frame layout (NULL: {5, g, g, 0}) and an
   optional QK LayerNorm affine (NULL: none). */
VGGT_API int vggt_attn_descriptor_ex(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                                     const float* pos, vggt_bf16* out, int S, int T, int H, int D,
                                     int kv_down, const vggt_frame_layout* layout,
                                     const vggt_qk_norm* norm, cudaStream_t stream);

/*
 * Attention over a subset of the tokens -- the VGGT-Omega layout (VGGT-Omega
 * page: 16 register tokens after each frame's patches that take part in
 * attention only at blocks [2, 6, 9, 14, 20]; 4 storage tokens shared by the
 * whole sequence; one camera token for all frames).
 *   Tokens: S frames of T tokens, then n_extra sequence tokens (rows S*T ..
 *   S*T + n_extra - 1) -- q, k, v, out [S*T + n_extra, H, D] bf16, pos
 *   [S*T + n_extra, 2] fp32.
 *   The last n_skip_back tokens of every frame take no part: they are neither
 *   queries nor keys, and their output rows are not written (0 <= n_skip_back
 *   <= T; at the register blocks n_skip_back = 0).
 *   global == 0: frame attention over each frame's T - n_skip_back kept tokens;
 *   the sequence tokens take no part (their output rows are not written).
 *   global == 1: every kept token and every sequence token attends to all of
 *   them. How the storage and camera tokens attend is not on the page; this
 *   call treats them as ordinary tokens of the global sequence, outside every
 *   frame.
 * norm: optional QK LayerNorm affine (vggt_qk_norm, may be NULL). With
 * n_skip_back == 0 and n_extra == 0 this is vggt_attn_frame_ex /
 * vggt_attn_global_ex. Scratch: q_hat and k_hat of the kept rows, plus their
 * gathered values when n_skip_back > 0.
 */
VGGT_API int vggt_attn_subset(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                              const float* pos, vggt_bf16* out, int S, int T, int n_skip_back,
                              int n_extra, int H, int D, int global, const vggt_qk_norm* norm,
                              cudaStream_t stream);

/*
 * The fp32 mode: frame / global attention (as vggt_attn_frame_ex /
 * vggt_attn_global_ex, any T >= 1, optional QK LayerNorm affine) on fp32
 * q, k, v [S*T, H, D] with fp32 out -- the precision the vggt-jax README's
 * FP32 parity runs use (its attention: TF32x3 Triton kernels). The prologue
 * runs in fp32; both attention products run on the bf16 tensor cores with
 * every fp32 operand x carried as `terms` bf16 terms x_0 = bf16(x),
 * x_1 = bf16(x - x_0), x_2 = bf16(x - x_0 - x_1); a b is the sum of the term
 * products a_i b_j with i + j < terms, accumulated in fp32, exponentials to
 * ~2^-22:
 *   terms == 2: 3 products, the dropped ones ~2^-18 a b (at most 2^-16);
 *               outputs to ~1e-5 of max|v|; about 3x the tensor-core work
 *               of the bf16 path;
 *   terms == 3: 6 products, the dropped ones ~2^-27 a b (at most 2^-23);
 *               outputs to about fp32 rounding, ~1e-6 of max|v|; about 6x.
 * Other values of terms: VGGT_ERR_UNSUPPORTED.
 * Pointers: q, k, v, out 16-byte aligned (fp32 arrays), pos 8-byte aligned.
 * Scratch: 4 + 4*terms bytes per (token, head, dim) -- fp32 q_hat and the
 * bf16 terms of k_hat and v.
 */
VGGT_API int vggt_attn_frame_f32(const float* q, const float* k, const float* v, const float* pos, float* out,
                                 int S, int T, int H, int D, const vggt_qk_norm* norm, int terms,
                                 cudaStream_t stream);
VGGT_API int vggt_attn_global_f32(const float* q, const float* k, const float* v, const float* pos, float* out,
                                  int S, int T, int H, int D, const vggt_qk_norm* norm, int terms,
                                  cudaStream_t stream);

/*
 * Several scenes per call (the vggt-jax README feeds [B, S, 3, H, W] image
 * batches): q, k, v, out [B, S, T, H, D] and pos [B, S, T, 2], scene b being
 * token rows [b*S*T, (b+1)*S*T). Every scene is attended on its own: global
 * attention over its S*T tokens, or descriptor attention over its S*T_k
 * pooled descriptors (layout and affine as in the _ex calls; either may be
 * NULL). B == 1 is vggt_attn_global_ex / vggt_attn_descriptor_ex; B == 0 is a
 * no-op. Frame attention needs no batched form: B scenes of S frames are
 * B*S frames. One launch per step for all scenes, so small scenes fill the
 * GPU together. B*S*T <= VGGT_MAX_TOKENS.
 */
VGGT_API int vggt_attn_global_batch(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                                    const float* pos, vggt_bf16* out, int B, int S, int T, int H, int D,
                                    const vggt_qk_norm* norm, cudaStream_t stream);
VGGT_API int vggt_attn_descriptor_batch(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                                        const float* pos, vggt_bf16* out, int B, int S, int T, int H, int D,
                                        int kv_down, const vggt_frame_layout* layout, const vggt_qk_norm* norm,
                                        cudaStream_t stream);

/* vggt_kv_pool and vggt_kv_pool_tokens with a frame layout (NULL: default). */
VGGT_API int vggt_kv_pool_ex(const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                             vggt_bf16* k_out, vggt_bf16* v_out, float* pos_out, int S, int T, int H,
                             int D, int kv_down, const vggt_frame_layout* layout, cudaStream_t stream);
VGGT_API int vggt_kv_pool_tokens_ex(int T, int kv_down, const vggt_frame_layout* layout);

/* vggt_qk_prologue with an optional affine (HOST arrays of D fp32 values or
   NULL, as in vggt_qk_norm; no score bound applies here). */
VGGT_API int vggt_qk_prologue_ex(const vggt_bf16* x, const float* pos, vggt_bf16* x_hat, int N, int H,
                                 int D, const float* ln_weight, const float* ln_bias,
                                 cudaStream_t stream);

/*
 * The descriptor keys in one memory pass: pools k/v/pos exactly as
 * vggt_kv_pool_ex, and instead of storing the pooled keys normalises and
 * rotates them at their pooled positions (the prologue, with the optional
 * key affine) -- the inputs the attention kernel reads. Bit-identical to
 * vggt_kv_pool_ex followed by vggt_qk_prologue_ex on the pooled keys, with
 * one less write and read of the pooled keys. The descriptor calls and the
 * streaming cache use this pass internally.
 *   k_hat [H, S*T_k, D] bf16 head-major; v_out [S, T_k, H, D] bf16;
 *   pos_out [S, T_k, 2] fp32; T_k = vggt_kv_pool_tokens_ex(T, kv_down, layout).
 */
VGGT_API int vggt_descriptor_keys(const vggt_bf16* k, const vggt_bf16* v, const float* pos,
                                  vggt_bf16* k_hat, vggt_bf16* v_out, float* pos_out, int S, int T,
                                  int H, int D, int kv_down, const vggt_frame_layout* layout,
                                  const float* ln_weight, const float* ln_bias, cudaStream_t stream);

/* vggt_desc_cache_create with a frame layout and a QK LayerNorm affine
   (either may be NULL); the cache keeps copies of both and applies them to
   every chunk. */
VGGT_API int vggt_desc_cache_create_ex(vggt_desc_cache** cache, int max_frames, int T, int H, int D,
                                       int kv_down, const vggt_frame_layout* layout,
                                       const vggt_qk_norm* norm);

/* Size of the fixed scratch array vggt_attn_global_noalloc draws on. */
#define VGGT_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * Global attention that allocates nothing, for callers that must not allocate
 * device memory while they run -- e.g. inference loops that reserve their
 * whole memory budget at start-up, or processes without the stream-ordered
 * allocator. (No counterpart on the pages: it exists only for such callers.)
 * Same arguments, layouts and result as vggt_attn_global; the caller still
 * provides q, k, v, pos and out. The normalised q and k live in a fixed
 * VGGT_NOALLOC_SCRATCH_BYTES array inside the library, so the call needs
 * 2 * S*T * H * D * 2 bytes <= VGGT_NOALLOC_SCRATCH_BYTES (S*T <= 4096 at
 * H = 16) and returns VGGT_ERR_SHAPE beyond that, launching nothing.
 * - The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 * - Every GPU that loads the library keeps the array until the process exits.
 * - All calls share the array: calls that overlap on the GPU (e.g. on two
 *   unordered streams) race and corrupt each other's results. Order them.
 * - It never calls cudaMalloc, cudaMallocAsync, cudaFree or any allocator.
 */
VGGT_API int vggt_attn_global_noalloc(const vggt_bf16* q, const vggt_bf16* k, const vggt_bf16* v,
                                      const float* pos, vggt_bf16* out,
                                      int S, int T, int H, int D, int kv_down,
                                      cudaStream_t stream);

/* Tokens per frame after pooling (5 + ceil(g/kv_down)^2), or a negative
   vggt_status when T is not 5 + g*g or kv_down < 1. Host only. */
VGGT_API int vggt_kv_pool_tokens(int T, int kv_down);

/* Synchronises `stream`, then returns and clears the device status word of
   the current device: VGGT_OK; VGGT_ERR_TIMEOUT when a bounded device wait
   ran out since the last call; else VGGT_ERR_RANGE when an attention row sum
   was out of range (see vggt_attn_core); VGGT_ERR_CUDA if the
   synchronisation failed. */
VGGT_API int vggt_get_device_status(cudaStream_t stream);

/* Returns the library's unused scratch memory on the current device to the
   system (memory whose cudaFreeAsync has not yet executed in its stream stays
   reserved: synchronise those streams first). Later calls take it back as
   they need it. VGGT_OK, or VGGT_ERR_CUDA. Host only. (No counterpart on the
   pages: memory management of this library.) */
VGGT_API int vggt_release_scratch(void);

/* Whether the library's scratch pool exists on the current device (*exists
   = 0 or 1: the first call that needs scratch creates it) and how many bytes
   it currently holds from the system (*reserved, 0 when it does not exist).
   VGGT_OK, VGGT_ERR_NULL or VGGT_ERR_CUDA. Host only. (No counterpart on the
   pages: memory management of this library.) */
VGGT_API int vggt_scratch_pool_info(int* exists, unsigned long long* reserved);

/* Human-readable name of a vggt_status value (static storage). */
VGGT_API const char* vggt_status_string(int status);

/* Upper bound, in SM clock cycles, of every device-side wait in the library's
   kernels (default about 2^32 cycles, roughly two seconds). Values < 1 restore
   the default. Returns the previous limit. Applies to launches made after the
   call on the current device. */
VGGT_API long long vggt_set_wait_limit(long long cycles);

/* Launches one block that waits, with the current limit, on a barrier that
   nothing ever completes, then records VGGT_ERR_TIMEOUT in the status word.
   It exercises the timeout path without any risk to the device. */
VGGT_API int vggt_debug_wait_timeout(cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* VGGT_ATTN_H */
