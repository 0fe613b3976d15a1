/*
 * e2d2_attn.h -- C ABI of the E2D2 fused block-diffusion attention for NVIDIA B200 (sm_100a).
 *
 * The operations are the attention calls of the E2D2 encoder-decoder block diffusion
 * language model, as the pages describe them:
 *   [E2D2 notes]  "Encoder-Decoder Diffusion Language Models for Efficient Training and
 *                 Inference" (paper notes): sec. 2 "two connection variants" (last hidden
 *                 state / shared KV cache; self- and cross-attention fused in one call),
 *                 sec. 3 "sampling algorithm", sec. 4 "training algorithm" (block-causal
 *                 encoder mask; decoder mask over 2L keys; FLOPs table).
 *   [BD3LM blog]  "Block Diffusion: Interpolating Between Autoregressive and Diffusion
 *                 Language Models", sec. 3 "block decomposition": position i is in block
 *                 floor(i / S).
 *
 * Common conventions
 *   - Every tensor is a plain device pointer to contiguous row-major memory, head_dim
 *     innermost.  Q/K/V/O and KV caches are bfloat16; LSE is float32.  The caller owns all
 *     memory; the library never allocates device memory.
 *   - q, out: [batch][q_heads][len][head_dim]; k, v: [batch][kv_heads][len][head_dim];
 *     KV cache: [batch][kv_heads][capacity][head_dim]; lse: [batch][q_heads][len].
 *   - GQA: query head h reads kv head h / (q_heads / kv_heads).
 *   - scale <= 0 selects 1/sqrt(head_dim).  lse is the natural-log log-sum-exp of the scaled
 *     scores of each query row; pass NULL to skip it.
 *   - Every call is enqueued on `stream` and never synchronises.  Argument errors are
 *     reported before anything is launched; nothing is launched then.  E2D2_ERR_CUDA means a
 *     launch or driver call failed.  A device-side wait that times out (bounded spin) sets a
 *     device error word that e2d2_last_device_error() reads.
 *   - Supported: head_dim in {32, 64, 128}; q_heads % kv_heads == 0; pointers 16-byte
 *     aligned; lengths below 2^31 elements per dimension.
 *   - The last-hidden-state and shared-KV-cache variants ([E2D2 notes, sec. 2]) are the same
 *     calls: they differ only in which K/V the caller passes as the encoder side.
 */
#ifndef E2D2_ATTN_H_
#define E2D2_ATTN_H_

#include <stddef.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define E2D2_API __attribute__((visibility("default")))
#else
#define E2D2_API
#endif

/* Size of the scratch array behind e2d2_attn_decoder_sample_noalloc (bytes). */
#define E2D2_SAMPLE_NOALLOC_MAX_BYTES (((size_t)32) << 20)

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    E2D2_OK = 0,
    E2D2_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad GQA ratio            */
    E2D2_ERR_UNSUPPORTED = 2, /* head_dim not in {32, 64, 128}, or not an sm_100 device     */
    E2D2_ERR_SHAPE = 3,       /* a dimension too large for the 32-bit row indexing           */
    E2D2_ERR_ALIGNMENT = 4,   /* a pointer not 16-byte aligned                              */
    E2D2_ERR_CAPACITY = 5,    /* P + S_new > capacity, or P > capacity                      */
    E2D2_ERR_WORKSPACE = 6,   /* workspace missing or smaller than the _workspace query     */
    E2D2_ERR_CUDA = 7,        /* a CUDA runtime / driver call failed                        */
    E2D2_ERR_TIMEOUT = 8,     /* a bounded device-side wait gave up (see e2d2_last_device_error) */
    E2D2_ERR_DEVICE_CHECK = 9 /* debug library: a device-side bounds check failed              */
} e2d2_status;

typedef struct {
    int batch;
    int q_heads;
    int kv_heads;
    int head_dim;
    float scale; /* <= 0: 1/sqrt(head_dim) */
} e2d2_dims;

/*
 * Encoder block-causal self-attention over clean tokens ([E2D2 notes, sec. 4]): query i
 * attends to every key j with floor(j/S) <= floor(i/S) (its own block, bidirectionally, and
 * every earlier block).
 *   q   [batch][q_heads][L][d]   k, v [batch][kv_heads][L][d]   out [batch][q_heads][L][d]
 *   lse [batch][q_heads][L] or NULL.   Requires L >= 1 and S >= 1.  If S does not divide L the
 *   last block is shorter (L mod S rows, as block diffusion allows: "Block Diffusion:
 *   Interpolating Between Autoregressive and Diffusion Language Models", sec. 3); S >= L makes
 *   the whole sequence one block.
 */
E2D2_API e2d2_status e2d2_attn_encoder_blockcausal(const void* q, const void* k, const void* v, void* out,
                                          float* lse, e2d2_dims dims, int L, int S,
                                          cudaStream_t stream);

/*
 * Decoder fused self+cross attention, training mode ([E2D2 notes, sec. 2 and 4]): the L noised
 * queries attend over 2L keys in one call -- the encoder-side keys k_enc/v_enc of the clean
 * blocks strictly before the query's block, and the decoder-side keys k_dec/v_dec of the
 * query's own block (bidirectional inside the block).
 *   q_dec [batch][q_heads][L][d]; k_enc, v_enc, k_dec, v_dec [batch][kv_heads][L][d];
 *   out [batch][q_heads][L][d]; lse [batch][q_heads][L] or NULL.  Blocks as for the encoder
 *   call (a shorter last block when S does not divide L).
 */
E2D2_API e2d2_status e2d2_attn_decoder_train(const void* q_dec, const void* k_enc, const void* v_enc,
                                    const void* k_dec, const void* v_dec, void* out, float* lse,
                                    e2d2_dims dims, int L, int S, cudaStream_t stream);

/*
 * Backward of the two train calls ([E2D2 notes, sec. 4]: one encoder and one decoder pass with
 * custom masks train all blocks; the page gives no backward, so these are the plain derivatives
 * of the two calls that a gradient step through them needs).  Gradients of
 * sum(dout * out) with respect to every input, the probabilities recomputed from the forward's
 * lse:  p_ij = exp(scale q_i.k_j - lse_i) over the keys the forward's mask lets row i see,
 * dp_ij = dout_i.v_j,  D_i = sum_j p_ij dp_ij (formed from the probabilities, not from out),
 * dq_i = scale sum_j p_ij (dp_ij - D_i) k_j,  dv_j = sum_i p_ij dout_i,
 * dk_j = scale sum_i p_ij (dp_ij - D_i) q_i, the sums over i running over every query head
 * that shares k_j's kv head (GQA).
 *   q, k, v (or q_dec, k_enc, v_enc, k_dec, v_dec), dims, L, S: exactly as passed to the
 *   forward call; out and lse (both NOT NULL) are that call's outputs; dout
 *   [batch][q_heads][L][d] bf16.  out serves only as a reference value: dq is accumulated as
 *   sum_j p_ij (dp_ij - c_i) k_j - (D_i - c_i) sum_j p_ij k_j with c_i = dout_i.out_i, which is
 *   the same gradient for any c_i and keeps its bf16 operands small where one key carries a
 *   row's weight; any finite out gives the derivative of the forward, the forward's own out the
 *   smallest rounding error.
 *   dq [batch][q_heads][L][d]; dk, dv (dk_enc, dv_enc, dk_dec, dv_dec) [batch][kv_heads][L][d],
 *   bf16, every element written (no accumulation into them, no atomics: two calls with the same
 *   inputs give the same bits).
 *   workspace: device memory of at least e2d2_attn_train_backward_workspace(dims, L) bytes
 *   (2 * batch * q_heads * ceil(L/128)*128 floats; the query returns 0 for invalid dims or
 *   L <= 0 and needs no GPU), 16-byte aligned, contents ignored (holds D_i and the scaled lse
 *   between the two launches of the call); calls that may run at the same time (different
 *   streams) need different workspaces.
 *   Launches two kernels on `stream`: dq with D_i (query rows on the tensor-memory lanes),
 *   then dk/dv (keys on the lanes).  Errors as for the forward calls; a NULL out or lse is
 *   E2D2_ERR_INVALID_ARG; a small workspace is E2D2_ERR_WORKSPACE.
 */
E2D2_API size_t e2d2_attn_train_backward_workspace(e2d2_dims dims, int L);

E2D2_API e2d2_status e2d2_attn_encoder_backward(const void* q, const void* k, const void* v, const void* out,
                                                const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                                e2d2_dims dims, int L, int S, void* workspace, size_t ws_bytes,
                                                cudaStream_t stream);

E2D2_API e2d2_status e2d2_attn_decoder_train_backward(const void* q_dec, const void* k_enc, const void* v_enc,
                                                      const void* k_dec, const void* v_dec, const void* out,
                                                      const float* lse, const void* dout, void* dq, void* dk_enc,
                                                      void* dv_enc, void* dk_dec, void* dv_dec, e2d2_dims dims,
                                                      int L, int S, void* workspace, size_t ws_bytes,
                                                      cudaStream_t stream);

/*
 * Bytes of scratch workspace that e2d2_attn_decoder_sample needs for these dims and block
 * size (split-KV partial results and per-split tickets).  Needs no GPU.  The caller
 * allocates it once, zero-filled; every completed call leaves its ticket words at zero again,
 * so the same workspace can be reused by later calls on the same stream.  Calls that may run
 * at the same time (different streams) need different workspaces.  After E2D2_ERR_TIMEOUT
 * the workspace must be zero-filled again.
 */
E2D2_API size_t e2d2_attn_decoder_sample_workspace(e2d2_dims dims, int S, int capacity);

/*
 * Decoder sampling step ([E2D2 notes, sec. 3]): the S noised queries of the block being
 * denoised attend to the first P rows of the cached encoder KV (the clean prefix) and to
 * the K/V of their own block, in one call.  Split-KV over the prefix; GQA rows packed.
 *   q_blk [batch][q_heads][S][d]; k_cache, v_cache [batch][kv_heads][capacity][d] (rows
 *   P..capacity-1 are never read); k_blk, v_blk [batch][kv_heads][S][d];
 *   out [batch][q_heads][S][d]; lse [batch][q_heads][S] or NULL.
 *   Requires 0 <= P <= capacity and ws_bytes >= e2d2_attn_decoder_sample_workspace().
 */
E2D2_API e2d2_status e2d2_attn_decoder_sample(const void* q_blk, const void* k_cache, const void* v_cache,
                                     int capacity, int P, const void* k_blk, const void* v_blk,
                                     void* out, float* lse, e2d2_dims dims, int S, void* workspace,
                                     size_t ws_bytes, cudaStream_t stream);

/*
 * Work plan of a sampling call (e2d2_attn_decoder_sample, _noalloc and
 * e2d2_attn_encoder_block_step) for these dims, block size S and prefix length P on a GPU with
 * num_sms SMs (the calls use the current device's count).  Needs no GPU; launches nothing.  The
 * calls cut the work into units of (batch entry, kv head, query tile), each a stream of
 * tiles_per_unit tiles of 128 keys (ceil(P/128) prefix tiles + ceil(S/128) own-block tiles).
 * With U units and G = min(num_sms, 256) CTAs, floor(U/G)*G units are taken whole, one CTA each,
 * after the split phase; the other split_units units are cut into equal contiguous tile ranges
 * over split_ctas CTAs, whose fp32 partials the last CTA to finish a unit merges in CTA order.
 *   kernel: 0 = the generic kernel, 16/32/64 = the kernel with keys on the tensor-memory lanes
 *   and that many packed query columns (head_dim 128 and G*S <= 64).
 * The environment variable E2D2_SPLITS=n (read once per process) sets the split phase's CTA count
 * to n, clamped to [split_units, min(grid, split_units * tiles_per_unit)], in this plan and in the
 * calls alike: a test knob for split-count independence.
 * Returns E2D2_ERR_INVALID_ARG for a NULL plan, bad dims, S <= 0, P < 0 or num_sms <= 0.
 */
typedef struct {
    int kernel;         /* 0 generic; 16, 32, 64: keys-on-lanes kernel with N query columns */
    int units;          /* work units: batch * kv_heads * query tiles per kv head            */
    int tiles_per_unit; /* 128-key tiles per unit                                             */
    int split_units;    /* units cut over the split phase's CTAs                              */
    int split_ctas;     /* CTAs of the split phase                                            */
    int whole_units;    /* units taken whole, one CTA each                                    */
    int grid;           /* CTAs launched                                                      */
} e2d2_sample_plan;

E2D2_API e2d2_status e2d2_attn_decoder_sample_plan(e2d2_dims dims, int S, int P, int num_sms,
                                                   e2d2_sample_plan* plan);

/*
 * Work order of a train call (host only, no GPU needed): which CTA takes each work item of
 * e2d2_attn_encoder_blockcausal (decoder = 0) or e2d2_attn_decoder_train (decoder = 1) on a
 * device with num_sms SMs.  A work item is a pair of 128-row query tiles of one (batch, head):
 * item k covers rows 256 * (n_pairs - 1 - k / (batch * q_heads)) .. of head k mod (batch * q_heads),
 * n_pairs = ceil(L / 256), so items = batch * q_heads * n_pairs.  The call's grid is
 * min(items, num_sms).  Items are placed longest processing time first: by decreasing key-tile
 * count (plus one for the epilogue), each on the CTA with the least work so far; with more than
 * 1152 items or 160 CTAs the order is round robin instead (item k on CTA k mod grid).
 *   cta_of_item: host array of `items` ints, written with the CTA of each item (may be NULL);
 *   *items_out, *grid_out: written when non-NULL; *balanced_out: 1 if the balanced order is used.
 * The CTA runs its items in the order listed.  Returns E2D2_ERR_INVALID_ARG for bad dims, L <= 0,
 * S <= 0 or num_sms <= 0.
 */
E2D2_API e2d2_status e2d2_attn_train_order(int decoder, e2d2_dims dims, int L, int S, int num_sms, int* cta_of_item,
                                           int* items_out, int* grid_out, int* balanced_out);

/*
 * Sampling step that allocates nothing: same arguments and result as e2d2_attn_decoder_sample
 * minus the workspace.  The paper has no counterpart; this exists for callers that cannot
 * allocate device memory (an engine that gives all of HBM to its own pool and no allocator to
 * plugins, or a hot path that may not call cudaMalloc because it can synchronise the device).
 * The split-KV scratch is a file-scope device array of E2D2_SAMPLE_NOALLOC_MAX_BYTES (32 MiB),
 * reserved on every GPU that loads the library until the process exits.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 *     once per device, with that device current); make that first call before any stream
 *     capture.
 *   - Shapes whose e2d2_attn_decoder_sample_workspace() exceeds the array are rejected with
 *     E2D2_ERR_WORKSPACE before anything is launched.
 *   - Every call shares the array: the ticket words are cleared (cudaMemsetAsync) on `stream`
 *     before each launch.  Calls that overlap on the GPU race; serialise them (one stream).
 *   - Calls no cudaMalloc, cudaFree or allocating library routine.
 */
E2D2_API e2d2_status e2d2_attn_decoder_sample_noalloc(const void* q_blk, const void* k_cache,
                                             const void* v_cache, int capacity, int P,
                                             const void* k_blk, const void* v_blk, void* out,
                                             float* lse, e2d2_dims dims, int S, cudaStream_t stream);

/*
 * Encoder incremental block step ([E2D2 notes, sec. 3]: a finished block goes through the
 * encoder, which updates the KV cache; sec. 4: the encoder's block-causal mask): the S clean
 * queries of block b attend to the cached prefix (rows 0..P-1, P = bS) and, bidirectionally, to
 * their own block -- the same rows of e2d2_attn_encoder_blockcausal over the whole sequence --
 * and the block's K/V (k_blk, v_blk) are written to cache rows P..P+S-1 in the same launch.
 *   Same layouts, workspace and errors as e2d2_attn_decoder_sample; requires P + S <= capacity
 *   (else E2D2_ERR_CAPACITY, nothing launched).  Cache rows other than P..P+S-1 are not written.
 *   The caller sets P += S after E2D2_OK.
 */
E2D2_API e2d2_status e2d2_attn_encoder_block_step(const void* q_blk, void* k_cache, void* v_cache, int capacity,
                                                  int P, const void* k_blk, const void* v_blk, void* out,
                                                  float* lse, e2d2_dims dims, int S, void* workspace,
                                                  size_t ws_bytes, cudaStream_t stream);

/*
 * Sampling step with ragged prefixes: as e2d2_attn_decoder_sample, but batch entry b has decoded
 * its own number of clean tokens, P_dev[b] ([E2D2 notes, sec. 3]: the cache grows per decoded
 * block; "Block Diffusion: Interpolating Between Autoregressive and Diffusion Language Models",
 * sec. 3: sequences of any length, so entries of one batch sit at different block boundaries, or
 * off them after prompts of different lengths).  Entry b's S queries attend to rows
 * 0..P_dev[b]-1 of its own cache and to its own block.
 *   P_dev: DEVICE array of batch ints (4-byte aligned), read by the kernel; each value is clamped
 *   to [0, capacity].  Cache rows at or past P_dev[b] are never used (they may hold anything).
 *   Other arguments, layouts and the workspace as for e2d2_attn_decoder_sample; batch <= 256
 *   (E2D2_ERR_SHAPE otherwise); a NULL P_dev is E2D2_ERR_INVALID_ARG.
 *   Work split: the key tiles of every (entry, kv head, query tile) unit form one stream cut into
 *   equal contiguous ranges over up to min(SMs, 256) CTAs (entry b's units take
 *   ceil(S/128) + ceil(P_dev[b]/128) tiles each); partials of units that straddle CTAs are merged
 *   as in the single-prefix call.
 */
E2D2_API e2d2_status e2d2_attn_decoder_sample_ragged(const void* q_blk, const void* k_cache, const void* v_cache,
                                                     int capacity, const int* P_dev, const void* k_blk,
                                                     const void* v_blk, void* out, float* lse, e2d2_dims dims, int S,
                                                     void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * Work plan of a ragged sampling call for host copies of the prefix lengths (P_host, batch ints)
 * on a GPU with num_sms SMs.  Needs no GPU; launches nothing.
 *   kernel: as in e2d2_sample_plan; units = batch * units_per_entry; total_tiles = the length of
 *   the stream (sum over entries of units_per_entry * (ceil(S/128) + ceil(P/128)), P clamped to
 *   [0, capacity]); grid = CTAs launched = min(num_sms, 256).  The stream is cut over
 *   stream_ctas = min(grid, total_tiles, max(units, total_tiles / 3)) CTAs (at least one per unit,
 *   about three tiles each beyond that, at least one tile each), CTA c < stream_ctas taking stream
 *   tiles [c * total / stream_ctas, (c + 1) * total / stream_ctas); the other CTAs take nothing.
 * Returns E2D2_ERR_INVALID_ARG for NULL pointers, bad dims, S <= 0, capacity < 0 or num_sms <= 0,
 * E2D2_ERR_SHAPE for batch > 256.
 */
typedef struct {
    int kernel;
    int units;
    int units_per_entry;
    long long total_tiles;
    int grid;
    int stream_ctas;
} e2d2_ragged_plan;

E2D2_API e2d2_status e2d2_attn_decoder_sample_ragged_plan(e2d2_dims dims, int S, const int* P_host, int capacity,
                                                          int num_sms, e2d2_ragged_plan* plan);

/*
 * KV-cache append ([E2D2 notes, sec. 3]: after a block is decoded the encoder absorbs it and
 * the cache grows by that block): rows P..P+S_new-1 of every (batch, kv head) cache take the
 * rows of k_new / v_new, bit for bit.  k_new, v_new [batch][kv_heads][S_new][d].  The cache
 * length is tracked by the caller (P += S_new after E2D2_OK).  Requires P + S_new <= capacity.
 */
E2D2_API e2d2_status e2d2_kv_cache_append(void* k_cache, void* v_cache, int capacity, int P,
                                 const void* k_new, const void* v_new, int S_new, e2d2_dims dims,
                                 cudaStream_t stream);

/*
 * KV-cache append with ragged lengths: as e2d2_kv_cache_append, but batch entry b's new rows go
 * to rows P_dev[b]..P_dev[b]+S_new-1 of its own caches (P_dev: DEVICE array of batch ints,
 * 4-byte aligned, read by the kernel; each value clamped to [0, capacity]).  Rows that would land
 * at or past capacity are not written (keep P_dev[b] + S_new <= capacity).  The lengths stay with
 * the caller, on the device: the call does not advance P_dev.  A NULL P_dev is
 * E2D2_ERR_INVALID_ARG.  With P_dev on the device, a sequence of sampling and append calls can be
 * captured once in a CUDA graph and replayed for every block.
 */
E2D2_API e2d2_status e2d2_kv_cache_append_ragged(void* k_cache, void* v_cache, int capacity, const int* P_dev,
                                                 const void* k_new, const void* v_new, int S_new, e2d2_dims dims,
                                                 cudaStream_t stream);

/* Human-readable name of a status code (static string). */
E2D2_API const char* e2d2_status_string(e2d2_status status);

/*
 * Synchronises `stream`, then reads and clears the device error word of the current device:
 * E2D2_OK; E2D2_ERR_DEVICE_CHECK if, in the debug library (built with E2D2_DEBUG, loaded by the
 * Python binding when the environment variable E2D2_DEBUG=1), a device-side bounds check on a
 * TMA coordinate or a work-unit index failed; else E2D2_ERR_TIMEOUT if a bounded device-side wait
 * gave up since the last read.  After either, outputs of the affected calls are undefined and
 * sampling workspaces must be zero-filled again.
 */
E2D2_API e2d2_status e2d2_last_device_error(cudaStream_t stream);

/*
 * Test hook for the failure path, not for production use.  On the current device, pipeline waits
 * of later launches give up after wait_limit_ns (default 2 s) and every kernel's load producer
 * first sleeps for producer_delay_ns (default 0), so that a test can make the bounded waits run
 * out without any fault: the kernels then unwind (waits that guard freeing tensor memory or copies
 * in flight keep the 2 s limit), return, and e2d2_last_device_error() reports E2D2_ERR_TIMEOUT.
 * (0, 0) restores the defaults.  Synchronous; returns E2D2_ERR_CUDA if the device is unusable.
 */
E2D2_API e2d2_status e2d2_debug_set_wait_test(unsigned long long wait_limit_ns,
                                              unsigned long long producer_delay_ns);

/* Library version, major * 10000 + minor * 100 + patch. */
E2D2_API int e2d2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* E2D2_ATTN_H_ */
