/*
 * ca2.h -- C ABI of libca2.so: the Ca2-VDM cached attention path on one NVIDIA B200.
 *
 * Ca2-VDM (arXiv 2411.16375, "Ca2-VDM: Efficient Autoregressive Video Diffusion Model with
 * Causal Generation and Cache Sharing"; ICML 2025 papernotes page, sections 整体框架 and
 * 关键设计 1-5) generates video chunk by chunk.  Each autoregressive (AR) step runs T
 * denoising steps that READ a KV cache of clean prefix frames, then one cache-writing
 * pass over the denoised chunk that APPENDS its K/V.  The cache does not depend on the
 * denoising step (prefix frames use tEmb(0)), so one copy serves all T steps.
 *
 * Conventions shared by every call:
 *   - Elements are bfloat16.  Spatial chunk tensors (q, k, v, out of the spatial call and
 *     the k_s, v_s given to the cache write) are frame-major [B][n][HW][H][D]: video, frame
 *     of the chunk, spatial token, head, head dim -- the (B*T) x S x C view a spatial block
 *     works in.  Temporal chunk tensors (q, k, v, out of the temporal call and the k_t, v_t
 *     given to the cache write) are token-major [B][HW][n][H][D] -- the (B*S) x T x C view a
 *     temporal block works in.  A row (one token of one frame) holds the H*D elements of
 *     this cache's heads; consecutive rows are cfg.row_pitch elements apart (default H*D),
 *     so a caller whose activations carry more heads (a rank owning heads [h0, h0+H) of a
 *     wider model) passes pointers to element h0*D of the first row and the full width as
 *     row_pitch.  All device pointers must be 16-byte aligned.
 *   - The caller owns all device memory (allocate it however you like, e.g. torch).
 *     The library stores the two cache pointers given to ca2_cache_init and never
 *     frees or reallocates them.
 *   - Device calls are asynchronous on the caller's stream (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream) and never synchronise.  Ring indices live
 *     on the host and reach the kernels as launch arguments, so host state advances at
 *     call time: issue calls in the order they must execute.
 *   - The attention calls, ca2_kv_proj_write and ca2_tpe_add are launched with
 *     programmatic dependent launch: their CTAs may start their set-up while the previous
 *     kernel on the stream drains, but read no input and write no output before it has
 *     completed.  Before that point the temporal call only asks L2 to prefetch ring data of
 *     this cache, a hint with no visible effect (L2 is the point of coherence), so the
 *     previous kernel may write any buffer, the caches included.
 *   - Errors are returned as ca2_status codes.  Nothing aborts, throws or traps.  A
 *     launch failure is CA2_ERR_CUDA.  A kernel whose bounded wait gave up records it in a
 *     device status word, read (with a device synchronisation) by ca2_device_status.
 *   - A handle is not thread-safe.
 *
 * Cache memory layout (both buffers caller-allocated, sizes from ca2_cache_bytes):
 *   temporal: [N_L][2][B][HW][H][Pmax][D]   (index 0 = K ring, 1 = V ring; token-major and
 *                                            head-major within a token: one head's Pmax
 *                                            slots are contiguous)
 *   spatial : [N_L][2][P'][B][HW][H][D]
 * K is stored in bf16 and V in fp16, the operand type of the attention's P V products (each
 * bf16 value converted exactly; |v| <= 65504).
 * The i-th oldest queued frame (i = 0 .. count-1) is in ring slot (head + i) mod Pmax;
 * spatial slot j (j < sp_count) holds the j-th of the last sp_count frames written,
 * oldest first.  Slots that hold no queued frame may contain anything: they are masked,
 * and their values never reach an output.
 *
 * Required order within one AR step:
 *   T x { for each layer: ca2_spatial_prefix_attn(use_prefix=1), ca2_temporal_attn }
 *   cache-writing pass: for each layer: ca2_spatial_prefix_attn(use_prefix=0), ca2_temporal_attn
 *   ca2_cache_evict_for(n) (evicts max(0, count + n - Pmax) frames)   then   ca2_cache_write(n)
 * The pass's attention reads the queue before eviction overwrites its oldest slots;
 * stream order keeps that true on the device.
 */
#ifndef CA2_H
#define CA2_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ca2_cache ca2_cache;   /* opaque host-side handle */

typedef struct {
    int n_layers;   /* N_L >= 1: attention blocks, each with its own cache                */
    int batch;      /* B >= 1 videos                                                       */
    int hw;         /* HW >= 1 spatial tokens per frame                                    */
    int heads;      /* H >= 1                                                              */
    int head_dim;   /* D: multiple of 8, 8 <= D <= 128                                     */
    int chunk_len;  /* l: frames per AR chunk, 1 <= l <= 8                                 */
    int p_max;      /* l <= Pmax <= 512: capacity of the temporal queue, in frames         */
    int p_spatial;  /* P': 0 <= P' <= l prefix frames kept for spatial attention           */
    int tpe_len;    /* N_tpe >= 1: temporal positional table length; 0 selects Pmax + l     */
    int row_pitch;  /* elements from one row of a chunk tensor to the next: 0 selects H*D,
                       else a multiple of 8, >= H*D (the activations' full width)          */
} ca2_config;

typedef enum {
    CA2_OK = 0,
    CA2_ERR_ARG = -1,       /* null pointer, bad flag, layer out of range                 */
    CA2_ERR_SHAPE = -2,     /* a size outside the documented range                        */
    CA2_ERR_CAPACITY = -3,  /* write would overflow the queue, or a buffer is too small   */
    CA2_ERR_ALIGN = -4,     /* a pointer is not 16-byte aligned                           */
    CA2_ERR_CUDA = -5,      /* a CUDA runtime call or kernel launch failed                */
    CA2_ERR_TIMEOUT = -6,   /* a kernel's bounded wait gave up (see ca2_device_status)     */
    CA2_ERR_RANGE = -7,     /* a device input outside the supported range (see
                               ca2_device_status): V values beyond |v| <= 65504, the fp16
                               range the caches and the P V products hold V in           */
    CA2_ERR_BOUNDS = -8     /* debug build only: a kernel's bounds check failed and the
                               access was skipped (see ca2_device_status, ca2_debug_build) */
} ca2_status;

/* Sizes in bytes of the temporal and spatial cache buffers for a configuration:
 * temporal = 2 * N_L * Pmax * B*HW*H*D * 2, spatial = 2 * N_L * P' * B*HW*H*D * 2.
 * One cache serves every denoising step (papernotes page, 关键设计 2), so the size has
 * no factor T.  Either out pointer may be NULL.  CA2_ERR_SHAPE on an invalid config. */
int ca2_cache_bytes(const ca2_config *cfg, size_t *temporal_bytes, size_t *spatial_bytes);

/* Create a handle over caller-allocated cache buffers.  temporal_buf / spatial_buf are
 * device pointers of at least the sizes above (spatial_buf may be NULL when P' = 0).
 * Contents need no initialisation: the queue starts empty (head = count = 0).
 * *out receives a host-allocated handle, released with ca2_cache_destroy. */
int ca2_cache_init(const ca2_config *cfg, void *temporal_buf, size_t temporal_bytes,
                   void *spatial_buf, size_t spatial_bytes, ca2_cache **out);

/* Release the handle (not the caller's buffers).  NULL is accepted. */
int ca2_cache_destroy(ca2_cache *cache);

/* The handle's configuration with the defaults resolved (tpe_len = Pmax + l and row_pitch =
 * H*D when given as 0).  Host-only. */
int ca2_cache_config(const ca2_cache *cache, ca2_config *out);

/* Byte offsets, within the temporal and the spatial cache buffer, of layer `layer`'s K
 * (kv = 0) or V (kv = 1) ring [B][HW][H][Pmax][D] and spatial cache [P'][B][HW][H][D], for
 * callers that inspect or fill them.  Either out pointer may be NULL.  Host-only. */
int ca2_cache_layer_offsets(const ca2_cache *cache, int layer, int kv, size_t *temporal_offset,
                            size_t *spatial_offset);

/* Dequeue the n oldest queued frames (papernotes page, 关键设计 4: once the queue reaches
 * Pmax the earliest cache entries leave it).  Host-only: head = (head + n) mod Pmax,
 * count -= n.  0 <= n <= count, else CA2_ERR_CAPACITY. */
int ca2_cache_evict(ca2_cache *cache, int n_frames);

/* Make room for n_new frames (papernotes page, 关键设计 4: once the queue reaches Pmax its
 * earliest entries leave it): evict exactly e = max(0, count + n_new - Pmax) oldest frames, as
 * ca2_cache_evict(e), and store e in *evicted (may be NULL).  Host-only.
 * 0 <= n_new <= Pmax, else CA2_ERR_SHAPE (nothing evicted). */
int ca2_cache_evict_for(ca2_cache *cache, int n_new, int *evicted);

/* Cache-writing stage (papernotes page, 整体框架 and 关键设计 4-5).  For every layer L:
 * frames j = 0..n-1 of k_t[L], v_t[L] are copied into ring slots
 * (head + count + j) mod Pmax; then the spatial cache of layer L is overwritten with the
 * last min(P', n) frames of k_s[L], v_s[L].  count += n.  One kernel launch for all
 * layers; a bit-exact copy, except that V is stored as fp16 (the same values; |v| >= 65536,
 * inf or NaN there is recorded as CA2_ERR_RANGE, read by ca2_device_status).
 * k_t[L], v_t[L] are token-major [B][HW][n][H][D]; k_s[L],
 * v_s[L] are frame-major [B][n][HW][H][D].  k_t, v_t, k_s, v_s are HOST arrays of N_L
 * device pointers (k_s, v_s may be NULL when P' = 0); their rows are row_pitch elements
 * apart.  1 <= n <= l; count + n > Pmax is CA2_ERR_CAPACITY (evict first).  Every argument
 * of every layer is validated before the first launch; the write is one launch per 64
 * layers, and if a later launch fails (CA2_ERR_CUDA) the queue state does not advance and
 * the cache contents of the layers already written are undefined until the next write. */
int ca2_cache_write(ca2_cache *cache, const void *const *k_t, const void *const *v_t,
                    const void *const *k_s, const void *const *v_s, int n_frames, void *stream);

/* Cache-writing stage fused into the K/V projection of one layer (papernotes page, 整体框架:
 * the cache-writing stage is one forward pass over the denoised chunk that computes and
 * stores the new KV cache; 关键设计 4 and 5: the temporal queue and the spatial cache).
 *   temporal: [K | V] = x_t w_t^T + b_t for every row (b, s, f) of x_t; K and V of chunk
 *             frame f go to ring slot (head + count + f) mod Pmax of layer `layer`;
 *   spatial : [K | V] = x_s w_s^T + b_s for the chunk's last n_sp = min(P', n) frames of
 *             x_s; frame f goes to spatial-cache frame f - (n - n_sp).
 * x_t: token-major [B][HW][n][Cin]; x_s: frame-major [B][n][HW][Cin], where Cin = row_pitch
 * (every element of a row is an input channel; Cin = C = H*D by default); w_t, w_s:
 * [2C][Cin] row-major, row o = output channel o (K channels 0..C-1 as (head, dim), then V);
 * b_t, b_s: [2C] or NULL for no bias.  All bf16, device memory, 16-byte aligned.  fp32
 * accumulation on the tensor cores, then the bias, then one rounding to bf16 (nearest,
 * ties to even); V is stored as the fp16 of that bf16 value (see the cache layout above).  x_s, w_s, b_s are not read when n_sp = 0 (may be NULL).
 * The queue does not advance: after this call for every layer, call ca2_cache_commit(n)
 * (evict first, as for ca2_cache_write).  1 <= n <= chunk_len and count + n <= Pmax, else
 * CA2_ERR_SHAPE / CA2_ERR_CAPACITY.  Asynchronous on `stream`. */
int ca2_kv_proj_write(ca2_cache *cache, int layer, const void *x_t, const void *w_t, const void *b_t,
                      const void *x_s, const void *w_s, const void *b_s, int n_frames, void *stream);

/* Advance the queue after ca2_kv_proj_write of every layer: count += n, the spatial cache
 * now holds min(P', n) frames, frames_written += n.  Host-only.  Same limits as
 * ca2_kv_proj_write. */
int ca2_cache_commit(ca2_cache *cache, int n_frames);

/* Causal temporal attention of one layer (papernotes page, 关键设计 1, equation
 * CausalAttn; bohrium arXiv 2411.16375 page, formula with M_ij = -inf for i < j).
 * For every (b, s, h) and chunk frame c:
 *   out[b][s][c][h] = sum_j softmax_j(q[b][s][c][h] . k_j / sqrt(D)) v_j
 * over the keys j = the count queued frames followed by chunk frames 0..c of k, v (the
 * queued frames are all visible, so their order does not matter).  The cache is only
 * read.  q, k, v, out: token-major [B][HW][n][H][D] device pointers; out must not
 * overlap the inputs.  1 <= n <= l.  fp32 softmax and accumulation, bf16 output (round
 * to nearest even).  The probability-weighted sum of V runs in fp16 (P with 11 significant
 * bits), so V must lie within |v| <= 65504: a larger chunk V (or inf / NaN) is recorded as
 * CA2_ERR_RANGE, read by ca2_device_status. */
int ca2_temporal_attn(ca2_cache *cache, int layer, const void *q, const void *k, const void *v,
                      void *out, int n_frames, void *stream);

/* Prefix-enhanced spatial attention of one layer (papernotes page, 关键设计 3).  For every
 * (b, frame f, h) and token i:
 *   out[b][f][i][h] = sum_j softmax_j(q_i . k_j / sqrt(D)) v_j
 * use_prefix = 1 (denoising targets): keys/values are frame f's own HW tokens followed
 *   by the HW tokens of each of the sp_count spatial-cache frames, an attention map of
 *   HW x ((1 + sp_count) HW).
 * use_prefix = 0 (clean prefix frames, the cache-writing pass): keys/values are frame f's
 *   own tokens repeated P'+1 times; repetition leaves softmax attention unchanged, so
 *   the kernel reads them once.
 * q, k, v, out: frame-major [B][n][HW][H][D]; 1 <= n <= l.  Scores and softmax in fp32;
 * the probability-weighted sum of V runs on the tensor cores in fp16 (P with 11 significant
 * bits, fp32 accumulation), so V values must lie within the fp16 range |v| <= 65504: larger
 * ones (and inf / NaN in V) are recorded as CA2_ERR_RANGE, read by ca2_device_status. */
int ca2_spatial_prefix_attn(ca2_cache *cache, int layer, const void *q, const void *k,
                            const void *v, void *out, int n_frames, int use_prefix, void *stream);

/* Cyclic temporal positional embedding added to a chunk (papernotes page, 关键设计 4,
 * Cyclic-TPEs): frame c of the chunk (global frame first_global_frame + c) gets row
 *   (offset + first_global_frame + c) mod N_tpe
 * of `table` added to every token's C = H*D vector:
 *   out[b][s][c][:] = round_bf16(x[b][s][c][:] + table[row(c)][:])
 * The sum is taken in float32 and rounded once (nearest, ties to even).
 * table: device, [N_tpe][H][D] bf16 (N_tpe = the cache's tpe_len), read only.
 * x, out: device, token-major [B][HW][n][H][D] (the temporal branch's layout); the rows of
 * x, out and table are row_pitch elements apart and the add covers their first H*D; out may be
 * x itself (in place), otherwise they must not overlap.  1 <= n <= l.  All three 16-byte
 * aligned.  Asynchronous on `stream`; the cache state is not touched.
 * Errors: ARG (null pointer, negative frame or offset), SHAPE (n, or a chunk of 2^35 bytes or
 * more), ALIGN, CUDA. */
int ca2_tpe_add(const ca2_cache *cache, long long first_global_frame, int offset, const void *table,
                const void *x, void *out, int n_frames, void *stream);

/* Cyclic temporal positional-embedding indices (papernotes page, 关键设计 4, Cyclic-TPEs):
 * out_host[c] = (offset + first_global_frame + c) mod N_tpe for c < n.  Host-only.
 * first_global_frame >= 0, offset >= 0, n >= 0; out_host may be NULL only when n = 0. */
int ca2_tpe_indices(const ca2_cache *cache, long long first_global_frame, int offset, int n,
                    int *out_host);

/* Queue state: ring slot of the oldest frame, queued frames, spatial frames, and the
 * total number of frames ever written.  Any out pointer may be NULL. */
int ca2_cache_state(const ca2_cache *cache, int *head, int *count, int *sp_count,
                    long long *frames_written);

/* Synchronise the current device and return what the kernels of this library recorded since
 * the last call (clearing the record): CA2_ERR_TIMEOUT if a bounded wait gave up,
 * CA2_ERR_RANGE if an input was outside the supported range, CA2_ERR_BOUNDS if a bounds check
 * of the debug build failed (the first record wins), else CA2_OK (or CA2_ERR_CUDA if the
 * synchronisation itself fails). */
int ca2_device_status(void);

/* Self-test of the bounded-wait path: launches one block that waits on a barrier nothing
 * will ever complete, with a wait limit of about wait_us microseconds; the kernel gives up,
 * records the timeout and returns.  Follow with ca2_device_status, which must report
 * CA2_ERR_TIMEOUT.  1 <= wait_us <= 1000000. */
int ca2_selftest_timeout(int wait_us, void *stream);

/* Head partition for running one layer on `world` ranks without a collective on the path:
 * every temporal (token, head) history and every spatial (frame, head) map is independent, so
 * a rank owns the contiguous heads [*h0, *h0 + *h_count) of every layer (caches sized for
 * h_count heads) and runs them on the full-width activations through ca2_config.row_pitch.
 * The first (heads mod world) ranks take one head more.  Host-only.  1 <= world <= heads and
 * 0 <= rank < world, else CA2_ERR_SHAPE; either out pointer may be NULL. */
int ca2_head_shard(int heads, int world, int rank, int *h0, int *h_count);

/* 1 for the debug build (libca2_debug.so, compiled with -DCA2_DEBUG), else 0.  In the debug
 * build every global access a kernel addresses itself -- plain loads and stores and bulk
 * copies -- is checked against the extent of its buffer as the call describes it (the
 * chunk tensors from their pointers and row pitch, the caches from the handle's sizes); a
 * failed check skips the access and records CA2_ERR_BOUNDS for ca2_device_status.  Accesses
 * through tensor maps are bounded by the maps in both builds.  The checks cost time; the
 * release build has none.  Host-only. */
int ca2_debug_build(void);

/* Static description of an error code. */
const char *ca2_status_string(int status);

/* Text of the last CUDA error met by a call of this library on the calling host thread
 * (the cause behind a CA2_ERR_CUDA), or "no error".  The string is static. */
const char *ca2_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* CA2_H */
