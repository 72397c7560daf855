/*
 * lcsa.h - C ABI of the B200 (sm_100a) locality-constrained block-sparse
 * causal attention library (liblcsa.so).
 *
 * The method is FlashVSR's sparse attention ("FlashVSR: Towards Real-time
 * Diffusion-Based Streaming Video Super-Resolution"; fmread summary of the
 * paper, section 2.2 "stage 2: block-sparse causal attention adaptation",
 * section 2.2 "stage 3" for the KV cache, section 2.3 "locality-constrained
 * sparse attention"). One streaming step is four calls, all asynchronous on
 * the caller's CUDA stream:
 *
 *   lcsa_pool_qk        mean-pool Q (and K) over 2x8x8 (t,y,x) token blocks
 *   lcsa_kv_append      write the chunk's K, V and pooled K into the ring cache
 *                       (pooling K on the way when no pooled K is given)
 *   lcsa_select_blocks  coarse block scores + causal/window masks + top-K
 *   lcsa_sparse_attn_fwd  online-softmax attention over the kept blocks
 *
 * and, for training with the same mask, lcsa_sparse_attn_bwd (dQ, dK, dV).
 *
 * Conventions
 * - Memory: the caller owns every buffer. The library allocates no device or
 *   host memory (the attention kernel allocates tensor memory on the SM for
 *   its own lifetime only), except the streaming pipeline: lcsa_pipeline_create
 *   allocates its input sets, scratch, O and streams, and
 *   lcsa_pipeline_destroy frees them. Its only other device state is a
 *   per-device error word and the fixed scratch array of
 *   lcsa_select_blocks_noalloc. A call writes only its output arguments (and
 *   that array).
 * - Pointers named "device" must be CUDA device pointers on the current
 *   device; all others are host pointers.
 * - Errors: argument and shape errors are returned synchronously, before any
 *   launch, and leave every output untouched. Errors detected inside a kernel
 *   (a wait that timed out, an index out of range) are recorded in a
 *   per-device error word that lcsa_last_device_error() reads and clears;
 *   kernels never trap.
 * - Element types: Q, K, V, O are bf16 (raw 16-bit storage); pooled features
 *   and block scores are float64; LSE is float32; block ids are int32.
 * - Token tensors use lcsa_tensor: extents [B][H][T][Y][X][D], D unit stride,
 *   element strides for B, H, T, Y, X. Requirements: D is 64 or 128; Y and X
 *   multiples of 8; data 16-byte aligned; every stride a multiple of 8
 *   elements; stride_b == H * stride_h (batch and heads must merge).
 * - Blocks: 2 (t) x 8 (y) x 8 (x) = 128 tokens. In time, blocks are counted
 *   backwards from the newest frame, so a tensor with an odd frame count has
 *   a one-frame (64-token) OLDEST block. Block id within a frame sequence:
 *   t_blk * Hb * Wb + y_blk * Wb + x_blk, t_blk oldest first, Hb = Y/8,
 *   Wb = X/8.
 */
#ifndef LCSA_H
#define LCSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LCSA_API __attribute__((visibility("default")))
#else
#define LCSA_API
#endif

#define LCSA_ABI_VERSION 1
#define LCSA_MAX_STREAMS 64

/* A cudaStream_t passed through as an opaque handle (NULL = default stream). */
typedef void* lcsa_stream_t;

typedef enum lcsa_status {
  LCSA_OK = 0,
  LCSA_ERR_INVALID_ARG = -1,  /* null pointer, bad enum, bad parameter value  */
  LCSA_ERR_SHAPE = -2,        /* extents inconsistent or unsupported           */
  LCSA_ERR_ALIGN = -3,        /* pointer or stride misaligned                  */
  LCSA_ERR_CAPACITY = -4,     /* KV cache or blk_idx row capacity exceeded     */
  LCSA_ERR_WORKSPACE = -5,    /* workspace missing or too small                */
  LCSA_ERR_CUDA = -6,         /* a CUDA runtime/driver call failed             */
  LCSA_ERR_TIMEOUT = -7,      /* a kernel wait gave up (device error word)     */
  LCSA_ERR_DEVICE_BOUNDS = -8, /* a kernel saw an out-of-range block id        */
  LCSA_ERR_SCRATCH_LIMIT = -9  /* request exceeds the library's fixed scratch   */
} lcsa_status;

enum {
  LCSA_WINDOW_TRUNCATE = 0,         /* block window, clipped at the frame edge      */
  LCSA_WINDOW_PRESERVE = 1,         /* block window, shifted inward at the edge      */
  LCSA_WINDOW_TRUNCATE_TOKENS = 2,  /* token window, clipped at the frame edge      */
  LCSA_WINDOW_PRESERVE_TOKENS = 3   /* token window, shifted inward at the edge      */
};

/* A token tensor [B][H][T][Y][X][D] of bf16 in device memory. */
typedef struct lcsa_tensor {
  void* data;  /* device */
  int32_t B, H, T, Y, X, D;
  int64_t stride_b, stride_h, stride_t, stride_y, stride_x; /* in elements */
} lcsa_tensor;

/*
 * Streaming KV cache of B streams (section 2.2, stage 3: later layers refine
 * temporal consistency through a KV cache; section 3: 8-frame chunks).
 *
 * k, v    device, bf16, contiguous [B][H][cap_frames][Y][X][D]
 * k_pool  device, float64, contiguous [B][H][cap_frames/2][Y/8][X/8][D]
 * begin, end  host-side state of stream b: absolute indices of its oldest
 *         valid frame and one past its newest; 0 <= end-begin <= cap_frames.
 *         Absolute frame a lives in ring slot a % cap_frames; block m covers
 *         absolute frames 2m and 2m+1 and its pooled K lives in slot
 *         m % (cap_frames/2). end is kept even, so blocks never straddle a
 *         chunk boundary; a stream whose first chunk has an odd number of
 *         frames starts at an odd begin (its oldest block has one frame).
 * cap_frames must be even. A fresh cache has begin[b] == end[b] == 0.
 * The caller may also wrap plain K/V tensors of F frames (F even) as a cache
 * with cap_frames = F, begin = 0, end = F and k_pool = their pooled K.
 */
typedef struct lcsa_kv_cache {
  void* k;         /* device */
  void* v;         /* device */
  double* k_pool;  /* device */
  int32_t B, H, cap_frames, Y, X, D;
  int64_t begin[LCSA_MAX_STREAMS];
  int64_t end[LCSA_MAX_STREAMS];
} lcsa_kv_cache;

/*
 * Parameters of the block selection (section 2.2 stage 2: coarse block map
 * and top-K; section 2.3: locality window with boundary-preserve or
 * boundary-truncate rules).
 *
 * top_k     > 0: keep min(C_i, top_k) blocks per query block;
 *           0: keep K_i = min(C_i, max(1, ceil(density * C_i))) where C_i is
 *           the number of allowed (causal, in-window) key blocks of the row
 *           and density * C_i is a float64 product.
 * window    0: no window. Block modes: the odd side length of the square
 *           spatial window in blocks (radius window/2), centred on the query
 *           block. Token modes: the window's side in tokens (e.g. 72 for
 *           1152 px): each query token t sees [t - window/2, t - window/2 +
 *           window) per axis; a key block is a candidate when some token of
 *           the query block sees some token of it, and the attention masks
 *           each key token outside the query token's window
 *           (lcsa_sparse_attn_fwd_window).
 * window_mode  LCSA_WINDOW_TRUNCATE(_TOKENS): clip the window at the frame
 *           edge; LCSA_WINDOW_PRESERVE(_TOKENS): shift it inward so it keeps
 *           its width (start = max(0, min(c - window/2, n - window))).
 * tie_eps   near-tie band (1e-5): with tau the K_i-th largest score, blocks
 *           with score > tau+eps are kept and the remaining places go to the
 *           lowest-index blocks with tau-eps <= score <= tau+eps.
 * kmax      row capacity of blk_idx (>= every K_i; see lcsa_select_kmax).
 */
typedef struct lcsa_select_params {
  int32_t top_k;
  int32_t window;
  int32_t window_mode;
  int32_t kmax;
  double density;
  double tie_eps;
} lcsa_select_params;

/* ABI version of the loaded library (LCSA_ABI_VERSION). */
LCSA_API int32_t lcsa_abi_version(void);

/* Static description of a status code. */
LCSA_API const char* lcsa_status_string(lcsa_status s);

/*
 * lcsa_pool_qk - block mean-pooling of Q and K (section 2.2, stage 2:
 * "average pooling yields compact block-level features").
 *
 * q, k     token tensors (k may be NULL to pool Q only); their B, H, Y, X, D
 *          must agree, T may differ.
 * q_pool   device, float64, contiguous [B][H][ceil(Tq/2)][Y/8][X/8][D]
 * k_pool   device, float64, contiguous [B][H][ceil(Tk/2)][Y/8][X/8][D]
 *          (ignored when k is NULL).
 * Each output is the arithmetic mean of the block's tokens (128, or 64 for a
 * one-frame oldest block), accumulated in float64 (exact for bf16 inputs
 * whose non-zero values in one block span at most 38 binades).
 */
LCSA_API lcsa_status lcsa_pool_qk(const lcsa_tensor* q, const lcsa_tensor* k,
                         double* q_pool, double* k_pool, lcsa_stream_t stream);

/*
 * lcsa_kv_append - append a chunk to the streaming KV cache (section 2.2,
 * stage 3 KV cache) and drop frames past the capacity.
 *
 * kv          cache (device buffers + host begin/end, updated on success).
 * k_new, v_new  token tensors [Bn][H][Tn][Y][X][D] with the cache's H, Y, X,
 *             D; they fill cache streams [stream_offset, stream_offset+Bn).
 * k_pool_new  device, float64 [Bn][H][ceil(Tn/2)][Y/8][X/8][D], the pooled
 *             K of the chunk (lcsa_pool_qk on k_new), or NULL: the call then
 *             pools k_new itself while copying it (one HBM read of K for both;
 *             the same float64 means lcsa_pool_qk gives).
 * Tn must be even, except for the first chunk of an empty stream, whose
 * frames are then placed so that the oldest block holds one frame. Only the
 * newest cap_frames frames of a chunk longer than the cache are written.
 */
LCSA_API lcsa_status lcsa_kv_append(lcsa_kv_cache* kv, const lcsa_tensor* k_new,
                           const lcsa_tensor* v_new, const double* k_pool_new,
                           int32_t stream_offset, lcsa_stream_t stream);

/*
 * lcsa_ingest_chunk - lcsa_pool_qk of the queries and lcsa_kv_append of the
 * chunk's keys and values (K pooled on the way) in one launch: q is pooled
 * into q_pool (layout as lcsa_pool_qk's q_pool), k_new / v_new are written
 * into the cache as by lcsa_kv_append with k_pool_new = NULL. Same errors as
 * those two calls; q's H, Y, X, D must match the cache.
 */
LCSA_API lcsa_status lcsa_ingest_chunk(const lcsa_tensor* q, double* q_pool, lcsa_kv_cache* kv,
                              const lcsa_tensor* k_new, const lcsa_tensor* v_new,
                              int32_t stream_offset, lcsa_stream_t stream);

/*
 * lcsa_kv_advance - the host-side part of lcsa_kv_append alone: advance the
 * begin / end of streams [stream_offset, stream_offset + n_streams) as
 * appending `frames` frames would, launching nothing. For replaying a
 * captured CUDA graph of a streaming step: the graph performs the device
 * writes, this call keeps the cache state in step. The library passes frame
 * numbers to its kernels shifted down by whole multiples of cap_frames, so
 * the launches of a stream in steady state repeat every cap_frames / frames
 * steps. Same errors as lcsa_kv_append's state checks.
 */
LCSA_API lcsa_status lcsa_kv_advance(lcsa_kv_cache* kv, int32_t frames, int32_t n_streams,
                            int32_t stream_offset);

/*
 * Row capacity blk_idx needs for a selection with these parameters over the
 * cache's current state and q_frames query frames (the largest K_i).
 * Returns 0 on invalid arguments.
 */
LCSA_API int32_t lcsa_select_kmax(const lcsa_kv_cache* kv, int32_t q_frames,
                         const lcsa_select_params* p);

/*
 * Bytes of device workspace lcsa_select_blocks needs for this cache state and
 * q_frames query frames: one 64-bit key per (query block, causal candidate),
 * B*H*ceil(q_frames/2)*Hb*Wb rows of (longest stream's temporal blocks)*Hb*Wb.
 * Returns 0 on invalid arguments.
 */
LCSA_API size_t lcsa_select_workspace_bytes(const lcsa_kv_cache* kv, int32_t q_frames);

/*
 * lcsa_select_blocks - coarse block map, masks and top-K (section 2.2,
 * stage 2: "coarse block-to-block attention map ... keep only the most
 * relevant top-K block pairs", causal masking; section 2.3 locality window).
 *
 * q_pool    device, float64 [B][H][ceil(q_frames/2)][Y/8][X/8][D]; the query
 *           frames are the newest q_frames frames of every stream's cache.
 * kv        cache whose k_pool holds the pooled keys; B, H, Y, X, D as q_pool.
 * blk_idx   device, int32 [B][H][nQB][kmax]; row i receives the ids of its
 *           kept key blocks in ascending order (id = t*Hb*Wb + y*Wb + x, t
 *           counted from the stream's oldest cached block), unused tail
 *           entries are -1.
 * blk_cnt   device, int32 [B][H][nQB]; K_i per row.
 * workspace device scratch of at least lcsa_select_workspace_bytes() bytes,
 *           16-byte aligned, owned by the caller; its contents are undefined
 *           afterwards and two calls in flight must not share it.
 * Scores are s_ij = (qbar_i . kbar_j) / sqrt(D) in float64, the dot product
 * summed in channel order with every product rounded before it is added, so
 * selections are reproducible bit for bit. Key block j is a candidate of
 * query block i iff t_j <= t_i (block-level causality) and j lies in i's
 * window. At most 2048 causal candidates per query block (longest stream's
 * temporal blocks x Hb x Wb), else LCSA_ERR_SHAPE. LCSA_ERR_WORKSPACE if
 * workspace_bytes is too small.
 */
LCSA_API lcsa_status lcsa_select_blocks(const double* q_pool, int32_t q_frames,
                               const lcsa_kv_cache* kv,
                               const lcsa_select_params* p, int32_t* blk_idx,
                               int32_t* blk_cnt, void* workspace,
                               size_t workspace_bytes, lcsa_stream_t stream);

/*
 * lcsa_select_blocks_noalloc - lcsa_select_blocks with library-owned scratch.
 *
 * The paper has no counterpart to this call. It is for callers that cannot
 * allocate device memory for a workspace: a plugin or engine whose device
 * memory is all owned by a host framework's pool and that has nothing to
 * hand out per call, or a real-time frame loop that must never call
 * cudaMalloc, because an allocation can synchronise the device and stall
 * the stream. The caller still provides q_pool, kv, blk_idx and blk_cnt,
 * with the same meaning, layout and results as lcsa_select_blocks.
 *
 * Scratch: a fixed device array of LCSA_SELECT_STATIC_SCRATCH_BYTES (8 MiB)
 * inside the library, used in place of the workspace. It exists on every
 * GPU where the library's kernels are loaded and stays there until the
 * process exits. The call allocates nothing: no cudaMalloc, cudaFree or
 * allocating library routine.
 * - The first call on a device, with that device current, looks up the
 *   array's device address (cudaGetSymbolAddress). Make that first call
 *   before any stream capture begins.
 * - All calls share the one array and it keeps the previous call's contents.
 *   Nothing in it has to start at zero: every entry the selection reads was
 *   written earlier in the same call.
 * - Calls whose work overlaps on the GPU (different streams, several host
 *   threads) race on the array. Keep them ordered on one stream or otherwise
 *   serialised.
 * Limit: lcsa_select_workspace_bytes(kv, q_frames) must not exceed
 * LCSA_SELECT_STATIC_SCRATCH_BYTES, else LCSA_ERR_SCRATCH_LIMIT, returned
 * before any device work. Four streams of 768x1408 frames (12 heads, an
 * 8-frame cache) need 6.7 MB and fit; one 1536x2688 stream with a 6-frame
 * cache (12 heads x 252 query blocks x 756 candidates) needs 18.3 MB and
 * does not.
 * Other errors are those of lcsa_select_blocks (LCSA_ERR_CUDA also if the
 * address look-up fails).
 */
#define LCSA_SELECT_STATIC_SCRATCH_BYTES ((size_t)8 << 20)
LCSA_API lcsa_status lcsa_select_blocks_noalloc(const double* q_pool, int32_t q_frames,
                                       const lcsa_kv_cache* kv,
                                       const lcsa_select_params* p, int32_t* blk_idx,
                                       int32_t* blk_cnt, lcsa_stream_t stream);

/*
 * lcsa_sparse_attn_fwd - attention inside the kept blocks (section 2.2,
 * stage 2: "apply full attention within the selected regions").
 *
 * q        token tensor [B][H][Tq][Y][X][D]: the newest Tq frames of each
 *          stream of kv (a stream holding fewer frames has padding query
 *          frames, see lcsa_segment_blocks).
 * kv       cache holding K and V (B, H, Y, X, D as q).
 * blk_idx, blk_cnt, kmax  as written by lcsa_select_blocks (device).
 * o        token tensor like q (bf16), device; receives
 *          O_r = sum_t softmax_t(q_r . k_t / sqrt(D)) v_t over the tokens t of
 *          the kept blocks of r's query block (a one-frame block contributes
 *          its 64 tokens).
 * lse      device, float32 contiguous [B][H][Tq][Y][X] natural-log
 *          log-sum-exp of each row's scaled logits, or NULL.
 * bf16 tensor-core products with float32 accumulation and softmax.
 * LCSA_ERR_SHAPE, before any device work, also when a cache holds 2^22 or
 * more key blocks ((cap_frames / 2) * (Y / 8) * (X / 8)): the kernel splits
 * block ids with a float reciprocal that is exact below that.
 */
LCSA_API lcsa_status lcsa_sparse_attn_fwd(const lcsa_tensor* q, const lcsa_kv_cache* kv,
                                 const int32_t* blk_idx, const int32_t* blk_cnt,
                                 int32_t kmax, lcsa_tensor* o, float* lse,
                                 lcsa_stream_t stream);

/*
 * lcsa_sparse_attn_fwd_window - lcsa_sparse_attn_fwd with the token-level
 * locality window (section 2.3: at inference each query's attention is limited
 * to a local neighbourhood, e.g. 1152 x 1152 px = 72 x 72 tokens, with a
 * boundary-truncate or boundary-preserve rule), applied inside the kept
 * blocks: query token (y, x) sees key token (y', x') iff y' and x' lie in its
 * window along each axis, [c - window/2, c - window/2 + window) clipped to the
 * frame (LCSA_WINDOW_TRUNCATE_TOKENS) or shifted inward to keep its width
 * (LCSA_WINDOW_PRESERVE_TOKENS). Use it with selections made with the same
 * window and mode. A query token that sees no key of its kept blocks gets
 * O = 0 and LSE = -inf. window = 0 is lcsa_sparse_attn_fwd. Other arguments
 * and errors as lcsa_sparse_attn_fwd; LCSA_ERR_INVALID_ARG for a block-level
 * window_mode with window > 0.
 */
LCSA_API lcsa_status lcsa_sparse_attn_fwd_window(const lcsa_tensor* q, const lcsa_kv_cache* kv,
                                        const int32_t* blk_idx, const int32_t* blk_cnt,
                                        int32_t kmax, int32_t window, int32_t window_mode,
                                        lcsa_tensor* o, float* lse, lcsa_stream_t stream);

/*
 * lcsa_sparse_attn_fwd_ex - lcsa_sparse_attn_fwd_window with an optional
 * workspace (device, 16-byte aligned, owned by the caller) of
 * lcsa_sparse_attn_fwd_workspace_bytes(D) bytes. With it, when the query
 * blocks do not fill the GPU's last wave of CTAs (one CTA per SM) and at most
 * half the SMs would be busy in it, each of those last query blocks runs as
 * two CTAs over the two halves of its kept blocks and a second kernel merges
 * the halves (fp32, by their log-sum-exps); without it (NULL) the result is
 * computed as by lcsa_sparse_attn_fwd. Both give the same output up to fp32
 * rounding of the merge. At most LCSA_ATTN_SPLIT_MAX query blocks are split.
 */
#define LCSA_ATTN_SPLIT_MAX 128
LCSA_API size_t lcsa_sparse_attn_fwd_workspace_bytes(int32_t head_dim);
LCSA_API lcsa_status lcsa_sparse_attn_fwd_ex(const lcsa_tensor* q, const lcsa_kv_cache* kv,
                                    const int32_t* blk_idx, const int32_t* blk_cnt,
                                    int32_t kmax, int32_t window, int32_t window_mode,
                                    lcsa_tensor* o, float* lse, void* workspace,
                                    size_t workspace_bytes, lcsa_stream_t stream);

/*
 * lcsa_segment_blocks - block lists for dense attention confined to one
 * segment (section 2.2, stage 1: joint video-image training with a
 * block-diagonal segment mask, so that attention stays inside one video clip
 * or one image; an image is a one-frame video).
 *
 * Each stream of kv is one segment: its cached frames [begin, end), 1 to
 * q_frames of them. The query tensor of the attention calls has q_frames
 * frames per stream; segment b's queries are its newest end-begin frames and
 * older query frames are padding. Every query block holding at least one of
 * the segment's frames keeps every key block of the segment, ascending (no
 * causal limit, no top-K); a query block of padding only keeps none, so the
 * forward writes zeros and LSE = -inf there (pass dO = 0 for padding rows to
 * the backward). blk_idx [B][H][nQB][kmax], blk_cnt [B][H][nQB] as for
 * lcsa_select_blocks; kmax >= lcsa_segment_kmax(kv), else LCSA_ERR_CAPACITY.
 * The lists feed lcsa_sparse_attn_fwd / lcsa_sparse_attn_bwd unchanged.
 * lcsa_segment_kmax returns the number of key blocks of the longest segment
 * (its temporal blocks x Y/8 x X/8), or 0 for a NULL or invalid kv.
 */
LCSA_API int32_t lcsa_segment_kmax(const lcsa_kv_cache* kv);
LCSA_API lcsa_status lcsa_segment_blocks(int32_t q_frames, const lcsa_kv_cache* kv, int32_t kmax,
                                int32_t* blk_idx, int32_t* blk_cnt, lcsa_stream_t stream);

/*
 * lcsa_sparse_attn_bwd - gradients of lcsa_sparse_attn_fwd for training with
 * the block-sparse causal mask (section 2.2, stage 2: the model is adapted to
 * block-sparse causal attention and trained with the flow-matching loss; stage
 * 3 trains the one-step student with the same mask). The selection (blk_idx,
 * blk_cnt, kmax, as passed to the forward) is held fixed.
 *
 * q, kv, blk_idx, blk_cnt, kmax  exactly as given to lcsa_sparse_attn_fwd.
 * o, lse      the forward's output and log-sum-exp (lse required).
 * d_o         token tensor like q: dLoss/dO.
 * dq          token tensor like q (bf16), device: receives dLoss/dQ.
 * dk, dv      device, bf16, contiguous in the cache layout
 *             [B][H][cap_frames][Y][X][D]: every ring slot of a frame in
 *             [begin, end) of each stream receives dLoss/dK, dLoss/dV (zero
 *             for keys no query kept); other slots are not written.
 * workspace   device scratch of at least lcsa_sparse_attn_bwd_workspace_bytes()
 *             bytes, 16-byte aligned, owned by the caller.
 * With P = exp(Q K^T / sqrt(D) - LSE), dP = dO V^T, delta = rowsum(dO * O) and
 * dS = P (dP - delta): dQ = dS K / sqrt(D), dK = dS^T Q / sqrt(D), dV = P^T dO,
 * summed over every query block that kept a key block. bf16 tensor-core
 * products with float32 accumulation; P and dS rounded to bf16 before their
 * products. Deterministic: no floating-point atomics. Errors as for the
 * forward; LCSA_ERR_WORKSPACE if workspace_bytes is too small.
 */
LCSA_API size_t lcsa_sparse_attn_bwd_workspace_bytes(const lcsa_kv_cache* kv, int32_t q_frames);
LCSA_API lcsa_status lcsa_sparse_attn_bwd(const lcsa_tensor* q, const lcsa_kv_cache* kv,
                                 const int32_t* blk_idx, const int32_t* blk_cnt,
                                 int32_t kmax, const lcsa_tensor* o, const float* lse,
                                 const lcsa_tensor* d_o, lcsa_tensor* dq, void* dk, void* dv,
                                 void* workspace, size_t workspace_bytes,
                                 lcsa_stream_t stream);

/*
 * Synchronise `stream`, then read and clear the current device's error word.
 * Returns LCSA_OK, LCSA_ERR_TIMEOUT or LCSA_ERR_DEVICE_BOUNDS (first set
 * bit wins), or LCSA_ERR_CUDA if the synchronisation itself failed. The word
 * is shared by every stream on the device.
 */
LCSA_API lcsa_status lcsa_last_device_error(lcsa_stream_t stream);

/*
 * Test hook: make the library's next kernel launches, on every device and
 * from every host thread of the process (the limit is one process-wide
 * setting, not a per-device one), see a wait limit of `ns` nanoseconds (0
 * restores the default of about one second). Used to exercise the timeout
 * path without any fault.
 */
LCSA_API lcsa_status lcsa_debug_set_wait_limit_ns(uint64_t ns);

/*
 * Test hook: launch one thread that waits on a barrier nothing will ever
 * arrive at, with a wait limit of `limit_ns` (1 ns .. 10 s). The wait gives up,
 * the kernel records LCSA_ERR_TIMEOUT in the device error word and returns;
 * the context stays usable. No fault, trap or hang is involved.
 */
LCSA_API lcsa_status lcsa_debug_stalled_wait(uint64_t limit_ns, lcsa_stream_t stream);

/*
 * Test hook: y[i] = 2^x[i] (x[i] <= 8) evaluated with the FMA-pipe
 * polynomial that was measured as a stand-in for part of the attention
 * softmax's special-function-unit exponentials (slower there; the kernel
 * does not use it): range reduction x = n + f, |f| <= 1/2, degree-3
 * minimax polynomial for 2^f, exponent add for 2^n. x, y: device float32
 * arrays of n elements.
 */
LCSA_API lcsa_status lcsa_debug_exp2_poly(const float* x, float* y, int64_t n,
                                          lcsa_stream_t stream);

/*
 * Streaming pipeline (section 3: the model runs as a stream, 8 video frames =
 * 2 latent frames per chunk, with a KV cache): chunks come from host memory
 * and their outputs go back there, with the copies of one chunk overlapping
 * the step of its neighbours.
 *
 * lcsa_pipeline_create - a pipeline over the caller's cache `kv`, chunks of
 *   q_frames frames per stream, selection parameters `params` (kmax is
 *   computed here, params->kmax is ignored; a token-level window mode also
 *   sets the attention's token window). The pipeline allocates, on the
 *   current device, two device input sets (Q, K, V), the step's scratch and O;
 *   lcsa_pipeline_destroy frees them. kv must stay valid, and must not be
 *   used by other calls, while the pipeline exists: each submit advances its
 *   host-side state as lcsa_ingest_chunk does. Errors: as check of kv,
 *   LCSA_ERR_SHAPE for q_frames outside [1, cap_frames], LCSA_ERR_INVALID_ARG
 *   for a bad window mode, LCSA_ERR_CUDA if an allocation fails (nothing is
 *   then kept). *out receives the pipeline, or NULL on error.
 * lcsa_pipeline_submit - queue one chunk: q_host, k_host, v_host each hold
 *   [B][H][q_frames][Y][X][D] bf16, contiguous, in host memory; o_host receives
 *   O in the same layout. Per chunk: three host-to-device copies on an upload
 *   stream, then lcsa_ingest_chunk, lcsa_select_blocks and
 *   lcsa_sparse_attn_fwd_ex on a compute stream, then the device-to-host copy
 *   of O on a read-back stream, all ordered by events; it returns once the
 *   work is queued. For the copies to overlap the steps the host buffers must
 *   be page-locked (cudaHostAlloc or cudaHostRegister). Host inputs must stay
 *   unchanged, and o_host unread, until lcsa_pipeline_sync returns. Call from
 *   the device the pipeline was created on (else LCSA_ERR_INVALID_ARG).
 *   Errors: LCSA_ERR_INVALID_ARG for a NULL argument or another device (nothing
 *   queued); LCSA_ERR_CUDA if a copy, event or stream call fails; otherwise
 *   the first error of the step's three calls (e.g. LCSA_ERR_SHAPE for an odd
 *   q_frames once a stream holds frames, as lcsa_ingest_chunk). After any
 *   error other than the first kind, part of the chunk may be queued and kv
 *   may have advanced: call lcsa_pipeline_sync, then restore kv's state or
 *   destroy the pipeline.
 * lcsa_pipeline_sync - wait for every queued chunk; returns the device error
 *   status as lcsa_last_device_error does.
 * lcsa_pipeline_start_timer / lcsa_pipeline_elapsed_ms - time, with events
 *   on the pipeline's own streams, from the first upload of the next submit
 *   to the read-back of the last chunk submitted (elapsed_ms waits for it).
 *   elapsed_ms returns LCSA_ERR_INVALID_ARG while start_timer has not yet
 *   been followed by a submit, and LCSA_ERR_CUDA if no timer was started.
 */
typedef struct lcsa_pipeline lcsa_pipeline;
LCSA_API lcsa_status lcsa_pipeline_create(lcsa_kv_cache* kv, int32_t q_frames,
                                          const lcsa_select_params* params, lcsa_pipeline** out);
LCSA_API lcsa_status lcsa_pipeline_submit(lcsa_pipeline* pl, const void* q_host, const void* k_host,
                                          const void* v_host, void* o_host);
LCSA_API lcsa_status lcsa_pipeline_sync(lcsa_pipeline* pl);
LCSA_API lcsa_status lcsa_pipeline_start_timer(lcsa_pipeline* pl);
LCSA_API lcsa_status lcsa_pipeline_elapsed_ms(lcsa_pipeline* pl, float* ms);
LCSA_API void lcsa_pipeline_destroy(lcsa_pipeline* pl);

#ifdef __cplusplus
}
#endif

#endif /* LCSA_H */
