/*
 * libropeattn: exact causal scaled-dot-product attention with RoPE and grouped-query
 * key/value sharing, for NVIDIA B200 (sm_100a).
 *
 * C ABI. Every tensor argument is a plain pointer to caller-owned DEVICE memory holding
 * bf16 values (IEEE bfloat16, 2 bytes) in contiguous BHSD layout
 * [batch][heads][seq][head_dim], head_dim innermost. Pointers must be 16-byte aligned;
 * outputs must not overlap inputs. All calls are asynchronous with respect to the host:
 * they validate the arguments, enqueue work on `stream` (NULL = legacy default stream)
 * and return. A non-RA_OK return means nothing was enqueued (argument errors) or a CUDA
 * launch/allocation failed (RA_ERR_CUDA). Errors found by the kernels themselves (a wait
 * that ran out) are sticky and read with rope_attn_get_device_status().
 *
 * The positions follow the bottom-right alignment used throughout: query row i sits at
 * absolute position pos_offset + (Sk - Sq) + i, key row j at pos_offset + j, and under the
 * causal mask key j is visible to query i iff its position is not after the query's.
 *
 * Temporary device memory (the rotated keys and the RoPE table of rope_attn_fwd, the
 * per-split partials of rope_attn_decode) is taken stream-ordered on `stream` from a memory
 * pool that the library creates on each device at its first call there, and released to it
 * on the same stream before the call returns. The pool keeps up to 512 MiB cached across
 * stream synchronisations, so calls after a synchronisation find their workspace ready
 * (with the device's default pool every synchronisation returned the memory, and the next
 * call waited to map it again). rope_attn_decode_noalloc takes no memory at all.
 */
#ifndef ROPEATTN_H_
#define ROPEATTN_H_

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define RA_API __attribute__((visibility("default")))
#else
#define RA_API
#endif

struct CUstream_st; /* the same handle type as cudaStream_t / CUstream */
typedef struct CUstream_st* ra_stream_t;

typedef enum {
  RA_OK = 0,
  RA_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, bad size, aliasing, Hq % Hkv != 0 ... */
  RA_ERR_UNSUPPORTED = 2,    /* valid request outside what the kernels implement (D not 64/128) */
  RA_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed; see rope_attn_last_cuda_error */
  RA_ERR_DEVICE_TIMEOUT = 4  /* a kernel gave up waiting on one of its own barriers */
} ra_status;

/*
 * Prefill / full-sequence attention.
 *
 *   out[b,h,i,:] = sum_j softmax_j( <R(p_q(i)) q[b,h,i,:], R(p_k(j)) k[b,h/G,j,:]> / sqrt(D) + M_ij )
 *                  * v[b,h/G,j,:]
 *
 * Scaled dot-product attention softmax(QK^T/sqrt(d_k))V as defined in "Transformer
 * Architecture & Self-Attention Mechanics" (devthesis.com), §1, with the causal -inf upper
 * triangle of "Multi-Head Attention & Rotary Position Embeddings (RoPE)" (learnllm.online,
 * its scaled_dot_product_attention code), the rotary embedding of devthesis §3 "Rotary
 * Position Embeddings (RoPE)" (pairs (x_2i, x_2i+1) turned by m*base^(-2i/D)), and the
 * grouped-query sharing of "Transformer internals: attention without the mysticism"
 * (ninaddeshpande.com, "The KV cache and the memory wall"): G = Hq/Hkv query heads share
 * one key/value head, query head h reading kv head h / G.
 *
 *   q    [B, Hq,  Sq, D] bf16 (read)          k, v [B, Hkv, Sk, D] bf16 (read)
 *   out  [B, Hq,  Sq, D] bf16 (written)
 *   D in {64, 128}; Hq % Hkv == 0; all sizes >= 1; causal requires Sq <= Sk.
 *   rope_base > 0 and finite; pos_offset >= 0 (absolute position of key row 0).
 *   causal: nonzero = apply the causal mask; zero = attend all Sk keys.
 * Returns RA_OK, RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED or RA_ERR_CUDA.
 */
RA_API ra_status rope_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int Hq,
                        int Hkv, int Sq, int Sk, int D, float rope_base, int pos_offset,
                        int causal, ra_stream_t stream);

/*
 * One block of ring attention: a slice of queries against one block of keys and values,
 * with the result merged into a running accumulator ("Building Self-Attention and
 * Transformer Engines" (codingpancake.com), §6.6 "Ring Attention": each GPU holds a slice of
 * Q, K and V and attends its queries to the K/V blocks passed around the ring). The page
 * leaves the combination of the blocks open; this call takes the exact one. Each block gives
 * O_blk = softmax-weighted V over its allowed keys and LSE_blk = ln sum_j exp(s_ij), with
 * s_ij = <R(q_pos0+i) q_i, k_rot_j> / sqrt(D). Two blocks over disjoint keys then combine
 * as LSE = ln(e^LSE_a + e^LSE_b) and O = e^(LSE_a-LSE) O_a + e^(LSE_b-LSE) O_b.
 *
 *   q      [B, Hq,  Sq, D] bf16 (read), NOT rotated: row i is rotated to q_pos0 + i here.
 *   k_rot  [B, Hkv, Sk, D] bf16 (read), keys already rotated to k_pos0 + j (for example by
 *          rope_attn_rotate with pos_offset = k_pos0).   v [B, Hkv, Sk, D] bf16 (read).
 *   o_acc  [B, Hq, Sq, D] fp32 and lse_acc [B, Hq, Sq] fp32 (natural log): the running
 *          result, normalised (O, not O times the sum).
 *   accumulate: bit RA_PARTIAL_ACCUMULATE clear: o_acc / lse_acc are overwritten with this
 *          block's result; set: merged with their contents (an lse_acc entry of -inf marks an
 *          empty accumulator row). Bit RA_PARTIAL_CHAINED: the caller guarantees that q,
 *          k_rot and v were complete before the previous kernel on the stream started (for
 *          example consecutive blocks of a ring whose keys were rotated before the first
 *          block). The launch then runs alongside that kernel's last wave and waits for it
 *          only before merging into o_acc / lse_acc / out. Without the guarantee the bit
 *          gives wrong results; leave it clear on a block that follows the kernel which
 *          produced its inputs.
 *   out    [B, Hq, Sq, D] bf16 or NULL: when given, also receives the merged result
 *          (pass it on the last block).
 *   causal: key j is allowed to query row i iff k_pos0 + j <= q_pos0 + i; requires
 *   q_pos0 >= k_pos0, so that every row sees at least the block's first key. zero: all keys.
 *   q_pos0, k_pos0 >= 0; q_pos0 + Sq and k_pos0 + Sk at most 2^30.
 * Views into longer sequences: q_rows, kv_rows and acc_rows are the numbers of rows between
 * consecutive heads of q, of k_rot and v, and of o_acc / lse_acc / out (0 = packed: Sq, Sk,
 * Sq; otherwise at least Sq, Sk, Sq). Head (b, h) of q then starts (b*H + h) * q_rows * D
 * elements after q, and so on. This lets a call read rows [a, a+Sq) of a [B, H, S_alloc, D]
 * tensor (pointer advanced by a*D elements, rows = S_alloc) and merge into the matching rows
 * of an accumulator.
 * Two query segments: with 0 < q_split < Sq, rows i >= q_split sit at q_pos1 + (i - q_split)
 * instead of q_pos0 + i (two separate slices of one sequence in one launch); q_pos1 >= 0 and
 * q_pos1 + (Sq - q_split) at most 2^30. With causal, the mask uses each row's own position,
 * q_pos1 >= k_pos0 is required too, and q_split must be a multiple of 128 (of 256 when
 * Hq / Hkv is odd). q_split = 0 means one segment.
 * o_acc, lse_acc and out must not overlap the inputs or each other; o_acc is 16-byte
 * aligned, lse_acc 4-byte aligned. D in {64, 128}, Hq % Hkv == 0, sizes >= 1. Runs the
 * prefill kernel of rope_attn_fwd with its fp32 epilogue (one launch, plus the RoPE table of
 * the Sq query positions). Returns RA_OK, RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED or
 * RA_ERR_CUDA.
 */
#define RA_PARTIAL_ACCUMULATE 1
#define RA_PARTIAL_CHAINED 2
RA_API ra_status rope_attn_fwd_partial(const void* q, const void* k_rot, const void* v,
                                       float* o_acc, float* lse_acc, void* out, int B, int Hq,
                                       int Hkv, int Sq, int Sk, int D, float rope_base,
                                       int q_pos0, int k_pos0, int causal, int accumulate,
                                       int q_rows, int kv_rows, int acc_rows, int q_split,
                                       int q_pos1, ra_stream_t stream);

/*
 * Prefill with a sliding window and/or straight into a KV cache (chunked prefill).
 *
 * window W > 0 (causal only): key j is visible to query row i iff
 *   p_q(i) - W < p_k(j) <= p_q(i), i.e. the W positions ending at the query's own
 * ("Building Self-Attention and Transformer Engines" (codingpancake.com), §6.4 "Sliding
 * Window Attention (SWA) in Mistral 7B" and FAQ Q10). W = 0: no window. KV tiles wholly
 * outside every row's window are skipped.
 *
 * k_cache_rot == v_cache == NULL: the same attention as rope_attn_fwd (S_cache ignored).
 * Otherwise the two caches [B, Hkv, S_cache, D] bf16 (read and written) hold the context:
 * rows 0 .. pos_offset-1 carry the earlier tokens' rotated keys and values. The call rotates
 * the chunk's keys k [B, Hkv, Sk, D] to positions pos_offset + j and stores them, and v,
 * at rows pos_offset + j (j < Sk); then the Sq queries, at positions
 * pos_offset + Sk - Sq + i, attend all T = pos_offset + Sk cache rows under the mask. With
 * pos_offset = 0 the result equals rope_attn_fwd and the caches are ready for
 * rope_attn_decode / rope_attn_decode_step ("Transformer internals: attention without the
 * mysticism", "The KV cache and the memory wall"). Cache rows >= T are neither read nor
 * written. Requires T <= S_cache, causal => Sq <= T; the caches must not overlap q, k, v,
 * out or each other. Other arguments and errors as rope_attn_fwd.
 */
RA_API ra_status rope_attn_prefill(const void* q, const void* k, const void* v, void* out,
                                   void* k_cache_rot, void* v_cache, int S_cache, int B, int Hq,
                                   int Hkv, int Sq, int Sk, int D, float rope_base,
                                   int pos_offset, int causal, int window, ra_stream_t stream);

/*
 * RoPE rotation of a whole tensor (builds a pre-rotated key cache for rope_attn_decode).
 *
 *   x_rot[b,h,s,2i]   = x[b,h,s,2i] cos(m theta_i) - x[b,h,s,2i+1] sin(m theta_i)
 *   x_rot[b,h,s,2i+1] = x[b,h,s,2i] sin(m theta_i) + x[b,h,s,2i+1] cos(m theta_i)
 *   m = pos_offset + s, theta_i = rope_base^(-2i/D)
 *
 * devthesis.com §3 "Rotary Position Embeddings (RoPE)"; the base is a parameter as in
 * ninaddeshpande.com "Rotary positional embeddings (RoPE)".
 *   x, x_rot [B, H, S, D] bf16; x_rot may equal x (in place) but not overlap it otherwise.
 *   D even, 8 <= D <= 256 and D % 8 == 0; pos_offset >= 0. Angles are formed in fp64.
 * Returns RA_OK, RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED (B * H above 2^31 - 1) or RA_ERR_CUDA.
 */
RA_API ra_status rope_attn_rotate(const void* x, void* x_rot, int B, int H, int S, int D,
                           float rope_base, int pos_offset, ra_stream_t stream);

/*
 * rope_attn_rotate on views into longer sequences: x_rows and out_rows are the numbers of rows
 * between consecutive heads of x and of x_rot (0 = S, packed; otherwise at least S). This
 * rotates rows [a, a+S) of a [B, H, S_alloc, D] tensor in place, or into the matching rows of
 * another, at positions pos_offset + s. In place (x == x_rot) requires x_rows == out_rows;
 * otherwise the two extents must not overlap. Other arguments and errors as rope_attn_rotate.
 */
RA_API ra_status rope_attn_rotate_rows(const void* x, void* x_rot, int B, int H, int S, int D,
                                       float rope_base, int pos_offset, int x_rows, int out_rows,
                                       ra_stream_t stream);

/*
 * One decode step over a pre-rotated KV cache (split-KV with a log-sum-exp combine).
 *
 * The query of each head, at absolute position `pos`, is rotated by R(pos) and attends
 * cache rows j = 0 .. L-1, L = min(Sk, pos + 1), which hold keys already rotated to their
 * own positions (as written by rope_attn_rotate) and their values:
 *   out[b,h,0,:] = sum_{j<L} softmax_j(<R(pos) q[b,h,0,:], k_cache_rot[b,h/G,j,:]> / sqrt(D))
 *                  * v_cache[b,h/G,j,:]
 * ("Transformer internals: attention without the mysticism", "The KV cache and the memory
 * wall": decoding keeps the past keys and values and reads all of them every step.)
 *   q [B, Hq, 1, D] bf16; k_cache_rot, v_cache [B, Hkv, Sk, D] bf16; out [B, Hq, 1, D].
 *   D in {64, 128}; Hq % Hkv == 0; pos >= 0; n_splits = 0 picks the split count, otherwise
 *   the number of key ranges (clamped to what L allows).
 */
RA_API ra_status rope_attn_decode(const void* q, const void* k_cache_rot, const void* v_cache,
                           void* out, int B, int Hq, int Hkv, int Sk, int D, float rope_base,
                           int pos, int n_splits, ra_stream_t stream);

/*
 * rope_attn_decode without any device allocation. No counterpart in the paper: this is a
 * deployment variant of rope_attn_decode for callers that may not allocate device memory at
 * call time, for example an inference server that reserves the GPU's memory for its own
 * pool up front and forbids libraries from taking memory behind its back, or a step that
 * must not risk an allocation failing (or waiting on the allocator) half-way through.
 *
 * Same arguments, layouts and result as rope_attn_decode. The per-split partials go to one
 * fixed array of 16 MiB (16777216 bytes) that the library keeps in device memory on every
 * GPU that loads it, until the process exits; the caller still provides q, the caches and
 * out. Partials take B*Hq*splits*(D*4 + 8) bytes (plus up to 255 of padding): with
 * n_splits = 0 the split count is lowered until they fit; an explicit n_splits whose
 * partials do not fit, or sizes that do not fit even with one split, return
 * RA_ERR_UNSUPPORTED without enqueuing anything (the reason is in
 * rope_attn_last_cuda_error).
 *
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress)
 * with that device current; make that first call before any stream capture. All calls, on
 * every stream, share the one array and it keeps the last call's contents: calls whose work
 * overlaps on the GPU race with each other, so serialise them (one stream, or events).
 * Nothing in the array needs clearing: every partial is written before it is read.
 */
RA_API ra_status rope_attn_decode_noalloc(const void* q, const void* k_cache_rot,
                                          const void* v_cache, void* out, int B, int Hq, int Hkv,
                                          int Sk, int D, float rope_base, int pos, int n_splits,
                                          ra_stream_t stream);

/*
 * One decode step of a batch whose sequences sit at their own positions, with the step's
 * new token appended to the cache inside the call (varlen batch).
 *
 *   pos [B] int32, DEVICE memory: sequence b's new token is at absolute position pos[b]
 *   (cache rows 0 .. pos[b]-1 hold its earlier tokens, keys rotated).
 *   k_new, v_new [B, Hkv, 1, D] bf16 (keys NOT rotated), or both NULL to attend the cache
 *   as it is (row pos[b] must then already hold the token).
 *   k_cache_rot, v_cache [B, Hkv, S_cache, D] bf16: with k_new, row pos[b] of each is
 *   overwritten with R(pos[b]) k_new and v_new before it is read; no other row is written.
 *   out[b,h,0,:] = sum_{lo<=j<=pos[b]} softmax_j(<R(pos[b]) q[b,h,0,:], k[b,h/G,j,:]>/sqrt(D))
 *                  * v[b,h/G,j,:],   lo = max(0, pos[b]-W+1) with window W > 0, else 0.
 *   max_pos: an upper bound on every pos[b], 0 <= max_pos < S_cache; the launch is sized
 *   for it (fewer rows, fewer CTAs). A pos[b] outside [0, max_pos] is found by the kernel:
 *   that sequence is not computed and rope_attn_get_device_status() returns
 *   RA_ERR_INVALID_ARG.
 * KV-cache decode of "Transformer internals: attention without the mysticism" ("The KV
 * cache and the memory wall"); window as in rope_attn_prefill. The caches must not overlap
 * q, k_new, v_new, out or each other. Other arguments and errors as rope_attn_decode.
 */
RA_API ra_status rope_attn_decode_step(const void* q, const void* k_new, const void* v_new,
                                       void* k_cache_rot, void* v_cache, void* out,
                                       const int* pos, int B, int Hq, int Hkv, int S_cache, int D,
                                       float rope_base, int max_pos, int window, int n_splits,
                                       ra_stream_t stream);

/*
 * rope_attn_decode_step over a paged cache ("Building Self-Attention and Transformer
 * Engines" (codingpancake.com), §6.2 "PagedAttention": the cache is cut into fixed-size
 * physical blocks, 16 tokens each there, that a sequence reaches through its block table).
 *
 *   k_pool_rot, v_pool [num_blocks, Hkv, page_size, D] bf16: block n holds page_size
 *   consecutive rows of one sequence for every KV head.
 *   block_table [B, max_blocks_per_seq] int32, DEVICE memory: row j of sequence b is row
 *   j % page_size of block block_table[b][j / page_size].
 *   page_size in {8, 16, 32, 64}; every pos[b] <= max_pos < max_blocks_per_seq * page_size.
 * Entries for the pages of rows lo .. pos[b] must name blocks in [0, num_blocks); an entry
 * out of range reads as zeros, and for the page receiving the appended token it is reported
 * as RA_ERR_INVALID_ARG by rope_attn_get_device_status() (nothing is written then). Entries
 * of other pages are never dereferenced. Everything else as rope_attn_decode_step.
 */
RA_API ra_status rope_attn_decode_paged(const void* q, const void* k_new, const void* v_new,
                                        void* k_pool_rot, void* v_pool, const int* block_table,
                                        void* out, const int* pos, int B, int Hq, int Hkv, int D,
                                        int page_size, int max_blocks_per_seq, int num_blocks,
                                        float rope_base, int max_pos, int window, int n_splits,
                                        ra_stream_t stream);

/* Split count rope_attn_decode uses for these sizes when n_splits == 0. */
RA_API int rope_attn_decode_auto_splits(int B, int Hq, int Hkv, int Sk, int D, int pos);

/*
 * Synchronises `stream`, returns the sticky device status of the current device and clears
 * it: RA_OK, RA_ERR_DEVICE_TIMEOUT, RA_ERR_INVALID_ARG if a kernel found a per-sequence
 * position or block-table entry out of range, or RA_ERR_CUDA if the sync failed or a kernel
 * found its shared-memory base misaligned (it then did no work; see
 * rope_attn_last_cuda_error).
 */
RA_API ra_status rope_attn_get_device_status(ra_stream_t stream);

/*
 * Polls each kernel wait makes before it gives up and reports RA_ERR_DEVICE_TIMEOUT
 * (default 1<<26). A test knob: 0 makes every wait give up at once, without polling, so the
 * timeout path runs while the kernels still exit cleanly. Returns the previous value;
 * limit < 0 only queries.
 */
RA_API long long rope_attn_set_wait_limit(long long limit);

/*
 * Kernel timing for profiling. While enabled, every rope_attn_fwd call records a pair of
 * CUDA events on its stream around its attention kernel, and every rope_attn_decode call
 * around its split kernel. rope_attn_profile_read(which = 0: prefill attention kernel,
 * 1: decode split kernel) waits for the recorded events, returns the summed kernel time in
 * milliseconds and the number of launches, and starts a new count. Enabling (or disabling)
 * also starts a new count. Enabling creates, on the current device, the event pairs of the
 * first 1024 launches of each kind (so that profiled calls only record events; more are made
 * as needed) and returns RA_ERR_CUDA if that fails. Meant for one device at a time; not for
 * concurrent callers.
 *
 * rope_attn_profile_pause(1) stops the recording without ending the session: calls made
 * while paused record nothing and run exactly as they do with profiling off (the event pairs
 * sit between a call's kernels, where they hold back the programmatic overlap of one
 * kernel's start with the previous kernel's end). rope_attn_profile_pause(0) resumes; the
 * pairs recorded before the pause are kept for rope_attn_profile_read. Returns
 * RA_ERR_INVALID_ARG when profiling is not enabled. Enabling clears the pause.
 */
RA_API ra_status rope_attn_profile_enable(int enable);
RA_API ra_status rope_attn_profile_pause(int pause);
RA_API ra_status rope_attn_profile_read(int which, double* total_ms, int* launches);

/* Text of a status code; the last CUDA error string for RA_ERR_CUDA. */
RA_API const char* rope_attn_status_string(int status);
RA_API const char* rope_attn_last_cuda_error(void);

/* ABI version of this header (major * 100 + minor). */
RA_API int rope_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ROPEATTN_H_ */
