/*
 * videomla.h -- C ABI of the B200 (sm_100a) VideoMLA latent-KV hot path.
 *
 * Implements the two inference-time steps of "VideoMLA: Low-Rank Latent KV
 * Cache for Minute-Scale Autoregressive Video Diffusion" (arXiv 2605.30351):
 *
 *   videomla_cache_write  -- project new video tokens into the latent ring
 *                            cache: c^KV = RMSNorm(W_dkv x) (Sec. 3.1 Eq. 1,
 *                            App. D.2) and the head-shared, unrotated RoPE key
 *                            k^R = W_kr x (Sec. 3.2 Eq. 5), FIFO ring of frames
 *                            (App. D.4).
 *   videomla_attention    -- multi-head latent attention of a query chunk over
 *                            the sliding window of that cache, in the absorbed
 *                            inference form (App. E Eq. 8-12): scores
 *                            (W_uk,h^T q^nope) . c_j + RoPE3D(q^R) . RoPE3D(k^R_j),
 *                            divided by sqrt(d_nope + d_rope) (Sec. 3.3 Eq. 7),
 *                            softmax over the whole window, o_h = W_uv,h sum_j p_j c_j
 *                            (Eq. 10 without W_O).  Keys and queries get
 *                            window-local (t, h, w) positions (App. D.5).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers (cudaMalloc / torch CUDA memory)
 *     on the current device, contiguous row-major, 16-byte aligned.  bf16 means
 *     IEEE bfloat16 stored as 16-bit words.  The caller owns every buffer and the
 *     stream; the library allocates no device memory per call and never
 *     synchronises the stream.  ``stream`` is a cudaStream_t (NULL = legacy
 *     default stream).
 *   - Calls are asynchronous: a return of VIDEOMLA_OK means the work was
 *     validated and enqueued.  A kernel whose bounded device-side wait ran out
 *     records VIDEOMLA_ETIMEOUT in a device status word, read with
 *     videomla_device_status().
 *   - Stream order holds as for any kernel.  The attention, its window pre-pass
 *     and the projection GEMMs are launched with programmatic stream
 *     serialisation: their CTAs may start (barriers, tensor memory, query
 *     loads) while the previous kernel of the stream drains, and they wait for
 *     that kernel to finish before reading anything it may have written or
 *     writing anything.
 *   - Errors are returned as negative codes (below); no exception crosses the
 *     ABI and nothing is printed.  videomla_strerror() names a code.
 *   - Thread safety: calls may be made from several host threads; the only
 *     shared state is a per-device cache of kernel attributes.
 */
#ifndef VIDEOMLA_H
#define VIDEOMLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VIDEOMLA_OK             0
#define VIDEOMLA_EINVAL        -1  /* null pointer, bad size, bad window, misaligned  */
#define VIDEOMLA_EUNSUPPORTED  -2  /* geometry with no compiled kernel instance      */
#define VIDEOMLA_ECUDA         -3  /* CUDA runtime / driver error at launch          */
#define VIDEOMLA_ETIMEOUT      -4  /* a bounded device-side wait gave up             */
#define VIDEOMLA_ENODEVICE     -5  /* no sm_100 device is current                    */

/* Flags of videomla_cache_write. */
#define VIDEOMLA_CACHE_RAW_LATENT 1u /* cache W_dkv x without the RMSNorm            */

/*
 * Layer geometry.  d_model = d, n_heads = n_h; d_c = latent width; d_rope =
 * decoupled RoPE width; d_nope = per-head content width (d_nope + d_rope is the
 * per-head key width, Sec. 3.2); d_v = per-head value width.  A latent frame is
 * a grid_h x grid_w patch grid (T_f = grid_h * grid_w tokens, row-major).
 * pairs_t + pairs_h + pairs_w = d_rope / 2 complex pairs over (t, h, w), laid
 * out t first, interleaved (2p, 2p+1) (App. D.3: (6, 5, 5) for d_rope = 32).
 * Pair k of an axis that owns D_a dims of a full (d_nope + d_rope)-dim head
 * rotates by pos * rope_base^(-2k / D_a) (the highest-frequency bands).
 * rms_eps is the RMSNorm epsilon.
 */
typedef struct videomla_dims {
    int d_model, n_heads, d_c, d_rope, d_nope, d_v;
    int grid_h, grid_w;
    int pairs_t, pairs_h, pairs_w;
    float rope_base;
    float rms_eps;
} videomla_dims;

/*
 * The attention window over the ring cache (App. D.4-D.5).  The ring holds
 * ``slots`` frames; logical frame j (0 = oldest valid, 0 <= j < n_valid) lives
 * in slot (oldest_slot + j) mod slots and gets local temporal coordinate t = j.
 */
typedef struct videomla_window {
    int slots;
    int oldest_slot;
    int n_valid;
} videomla_window;

/*
 * videomla_cache_write -- write the latent cache rows of a chunk of new tokens.
 *   x      [batch, n_tok, d_model] bf16: token activations (n_tok a multiple of
 *          T_f; token t of the chunk belongs to frame t / T_f of the chunk).
 *   W_dkv  [d_c, d_model]    bf16: KV down-projection (Eq. 1).
 *   W_kr   [d_rope, d_model] bf16: shared RoPE-key projection (Eq. 5).
 *   gamma  [d_c] fp32 RMSNorm gain, or NULL for unit gain.
 *   cache  [batch, slots * T_f, d_c + d_rope] bf16 ring (in/out): frame f of
 *          the chunk is written to slot (first_slot + f) mod slots; row p of a
 *          slot holds token p of its frame as [RMSNorm(c) | k^R] (k^R unrotated
 *          and unnormalised).  Rows of other slots are untouched.
 *   flags  VIDEOMLA_CACHE_RAW_LATENT to skip the RMSNorm, else 0.
 * One launch on ``stream``: a chunk of few 128-token tiles (fewer than half the
 * SMs) spreads each tile's d_model range over a thread-block cluster; more
 * tiles stream through a persistent kernel (one CTA per SM).  No workspace.
 * Arithmetic: bf16 inputs, fp32 accumulation and normalisation, bf16 RNE output.
 * Errors: EINVAL (null, n_tok not a whole number of frames, first_slot out of
 * range, n_tok / T_f > slots, misaligned), EUNSUPPORTED (d_c + d_rope or d_model
 * without a kernel instance), ECUDA.
 */
int videomla_cache_write(const videomla_dims* dims, const void* x, int batch, int n_tok,
                         const void* W_dkv, const void* W_kr, const float* gamma,
                         void* cache, int slots, int first_slot, unsigned flags,
                         void* stream);

/*
 * Bytes of the workspace that videomla_attention needs for this window and
 * batch: the window's rotated RoPE keys, batch * slots * T_f * d_rope fp16
 * values.  0 for invalid arguments.
 */
size_t videomla_attention_workspace_size(const videomla_dims* dims, const videomla_window* window, int batch);

/*
 * Bytes of a workspace that also holds the split-KV partials of the split the
 * library prefers for this call: when the (query tile, head, batch) units do not
 * fill the GPU's SMs in whole waves, the key tiles of each unit are shared by up
 * to 4 CTAs, each storing an unnormalised partial (fp32 O plus the per-row max
 * and sum) that the last of them merges.  A workspace between
 * videomla_attention_workspace_size() (or the sink variant's) and this size makes
 * the call use the largest split that fits; results agree to rounding.
 * 0 for invalid arguments.
 */
size_t videomla_attention_workspace_size_split(const videomla_dims* dims, const videomla_window* window, int n_sink,
                                               int batch, int n_query);

/*
 * videomla_attention -- latent attention of the newest n_query tokens of the
 * window over all n_valid * T_f keys of the window (no mask inside it).
 *   q_nope [batch, n_query, n_heads, d_nope] bf16: per-head content queries (Eq. 4).
 *   q_rope [batch, n_query, n_heads, d_rope] bf16: per-head UNROTATED q^R (Eq. 6);
 *          the kernel rotates query i by the position of logical token
 *          n_valid * T_f - n_query + i of the window.
 *   W_uk   [n_heads * d_nope, d_c] bf16: key up-projection, head-major row blocks.
 *   W_uv   [n_heads * d_v, d_c]    bf16: value up-projection, head-major row blocks.
 *   cache  [batch, slots * T_f, d_c + d_rope] bf16, as written by videomla_cache_write.
 *   out    [batch, n_query, n_heads, d_v] bf16: per-head outputs W_uv,h (sum_j p_j c_j).
 *   lse    [batch, n_query, n_heads] fp32 natural-log softmax denominator of the
 *          scaled scores, or NULL.
 *   workspace  device scratch of at least videomla_attention_workspace_size()
 *          bytes, 16-byte aligned, owned by the caller; its contents on entry do
 *          not matter and are overwritten (the window's rotated RoPE keys,
 *          App. D.5: rotation applied when the active window is formed; with
 *          videomla_attention_workspace_size_split() bytes also the split-KV
 *          partials).  Calls that run concurrently need distinct workspaces.
 * Two launches on ``stream``: the window pre-pass, then the attention kernel.
 * The kernel's CTAs take 128 query rows each: of one head (split-KV when those
 * units leave SMs idle), or 128 consecutive rows of the head-major (head, query)
 * order when that needs fewer waves (videomla_set_attention_tiling).  The d_c = 96
 * instance, when it runs neither split-KV nor head-packed tiles, uses two softmax
 * warpgroups on alternate 96-key tiles, merged exactly at the end.
 * Arithmetic: tcgen05 tensor cores with fp32 accumulation; the latent part of
 * the scores uses bf16 operands (q_abs rounded to bf16), the RoPE part fp16
 * operands (rotated q^R and k^R), the probabilities are rounded to bf16 before
 * the sum over latents; fp32 online softmax.
 * Errors: EINVAL (null, window out of range, n_query > n_valid * T_f, small
 * workspace, misaligned), EUNSUPPORTED (geometry without a kernel instance), ECUDA.
 */
int videomla_attention(const videomla_dims* dims, const void* q_nope, const void* q_rope,
                       const void* W_uk, const void* W_uv, const void* cache,
                       const videomla_window* window, int batch, int n_query,
                       void* out, float* lse, void* workspace, size_t workspace_bytes,
                       void* stream);

/* Largest number of pinned sink frames videomla_attention_sink accepts. */
#define VIDEOMLA_MAX_SINK_FRAMES 8

/*
 * Bytes of the workspace that videomla_attention_sink needs: the rotated RoPE
 * keys of the ring and of the sink frames, batch * (slots + n_sink) * T_f *
 * d_rope fp16 values.  0 for invalid arguments.
 */
size_t videomla_attention_sink_workspace_size(const videomla_dims* dims, const videomla_window* window, int n_sink,
                                              int batch);

/*
 * videomla_attention_sink -- videomla_attention over a sink-plus-window cache
 * ("VideoMLA: Low-Rank Latent KV Cache for Minute-Scale Autoregressive Video
 * Diffusion", App. D.4: one pinned sink latent frame plus a FIFO of the last
 * frames; App. D.5: keys re-indexed to local temporal coordinates of that
 * context).  The keys are the n_sink * T_f rows of ``sink_cache`` plus the
 * n_valid * T_f valid rows of the ring ``cache``.  Local frame index: sink frame
 * s is t = s, ring frame j (j frames after the oldest valid one) is
 * t = n_sink + j; query i is logical token (n_sink + n_valid) * T_f - n_query + i.
 *   sink_cache [batch, n_sink * T_f, d_c + d_rope] bf16, written like a ring of
 *          n_sink slots by videomla_cache_write; may be NULL when n_sink == 0.
 *   n_sink     0 .. VIDEOMLA_MAX_SINK_FRAMES (0 gives exactly videomla_attention).
 *   workspace  at least videomla_attention_sink_workspace_size() bytes.
 * Every other argument, the arithmetic and the launches are those of
 * videomla_attention.
 * Errors: EINVAL (as videomla_attention, plus n_sink out of range, sink_cache
 * NULL or misaligned while n_sink > 0, n_query > (n_sink + n_valid) * T_f),
 * EUNSUPPORTED, ECUDA.
 */
int videomla_attention_sink(const videomla_dims* dims, const void* q_nope, const void* q_rope,
                            const void* W_uk, const void* W_uv, const void* cache,
                            const videomla_window* window, const void* sink_cache, int n_sink,
                            int batch, int n_query, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * videomla_dense_attention -- the dense multi-head attention baseline that the
 * latent cache replaces ("VideoMLA", App. C.1: per-head keys and values cached
 * for every token, 2 n_h d_h = 3072 scalars per token and layer; Sec. 3.3 Eq. 7),
 * for same-box comparisons of speed and memory traffic with videomla_attention.
 * The window's keys are given in logical order (oldest frame first) and the
 * queries are its newest n_query tokens, with the window-local (t, h, w)
 * positions of videomla_attention.
 *   q_nope [batch, n_query, n_heads, d_nope] bf16, q_rope [batch, n_query, n_heads,
 *          d_rope] bf16 UNROTATED (rotated in the kernel by the query's position).
 *   k      [batch, n_keys, n_heads, 128] bf16: [k^nope_h | RoPE3D(k^R)], the RoPE part
 *          already rotated by the key's window-local position.
 *   v      [batch, n_keys, n_heads, 128] bf16.
 *   out    [batch, n_query, n_heads, 128] bf16: softmax(q k^T / sqrt(128)) v per head.
 * Requires d_nope + d_rope == 128, d_v == 128 and n_keys a whole number of frames.
 * One launch on ``stream``; tcgen05 tensor cores, fp32 online softmax, P as bf16.
 * Errors: EINVAL (null, sizes, misaligned), EUNSUPPORTED (head widths), ECUDA.
 */
int videomla_dense_attention(const videomla_dims* dims, const void* q_nope, const void* q_rope, const void* k,
                             const void* v, int batch, int n_query, int n_keys, void* out, void* stream);

/*
 * Bytes of the workspace videomla_query_projection needs: per token, up to
 * ceil(d_q / 128) fp32 partial sums of squares of the query latent (one per
 * column tile of the first GEMM), and the latent times its gain in bf16, for
 * batch * n_tok tokens.  0 for invalid arguments.
 */
size_t videomla_query_projection_workspace_size(const videomla_dims* dims, int d_q, int batch, int n_tok);

/*
 * videomla_query_projection -- per-head queries of new tokens ("VideoMLA",
 * Sec. 3.1 Eq. 3-4, Sec. 3.2 Eq. 6, App. D.2):
 *   c^Q = W_dq x (fp32), RMSNorm with gain gamma_q and dims->rms_eps (App. D.2),
 *   q_nope = W_uq c^Q and q_rope = W_qr c^Q (unrotated; videomla_attention rotates it).
 *   The RMSNorm is carried by the GEMMs: the first stores gamma_q (.) c^Q in bf16 and,
 *   for each of its column tiles, the sum of each token's squares of c^Q in fp32; the
 *   second adds a token's partial sums (in tile order, so the result does not depend
 *   on scheduling) and scales its output rows by 1 / sqrt(mean square + rms_eps)
 *   before rounding them to bf16.
 *   x       [batch, n_tok, d_model] bf16
 *   W_dq    [d_q, d_model] bf16; gamma_q [d_q] fp32 or NULL (unit gain)
 *   W_uq    [n_heads * d_nope, d_q] bf16, W_qr [n_heads * d_rope, d_q] bf16
 *   q_nope  [batch, n_tok, n_heads, d_nope] bf16, q_rope [batch, n_tok, n_heads, d_rope] bf16
 *   workspace  at least videomla_query_projection_workspace_size() bytes, 16-byte aligned.
 * Two persistent tcgen05 GEMM launches (the second writes both up-projections) on
 * ``stream``; the workspace needs no initialisation.
 * Errors: EINVAL (null, d_q or d_model not a multiple of 64, n_heads * d_nope or
 * n_heads * d_rope not a multiple of 8, small workspace, misaligned), ECUDA.
 */
int videomla_query_projection(const videomla_dims* dims, int d_q, const void* x, int batch, int n_tok,
                              const void* W_dq, const float* gamma_q, const void* W_uq, const void* W_qr,
                              void* q_nope, void* q_rope, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * videomla_output_projection -- layer output y = W_O [o_1 .. o_H] of the per-head
 * attention outputs (the output projection whose per-head slices W_O,h Eq. 10-11
 * fold into B_h = W_O,h W_uv,h; applied after W_uv here, which costs fewer flops
 * than B_h when d_c > d_v).
 *   o    [batch, n_query, n_heads, d_v] bf16 (videomla_attention's out)
 *   W_O  [d_model, n_heads * d_v] bf16
 *   y    [batch, n_query, d_model] bf16
 * One tcgen05 GEMM launch on ``stream``.
 * Errors: EINVAL (null, n_heads * d_v not a multiple of 64, misaligned), ECUDA.
 */
int videomla_output_projection(const videomla_dims* dims, const void* o, int batch, int n_query, const void* W_O,
                               void* y, void* stream);

/*
 * Bytes of the library's built-in scratch array used by
 * videomla_attention_static_workspace (16 MiB per device that loads the library).
 */
#define VIDEOMLA_STATIC_WORKSPACE_BYTES (16u << 20)

/*
 * videomla_attention_static_workspace -- videomla_attention without a caller
 * workspace.  (No counterpart in the paper: this is an integration aid.)
 *
 * For callers that cannot allocate device memory themselves -- for example a
 * host framework whose memory is owned by a pool or arena it does not expose,
 * code running where cudaMalloc is not allowed or would break a capture, or a
 * plug-in that may only use the buffers it is handed.  The call's scratch lives
 * in a fixed array compiled into the library (VIDEOMLA_STATIC_WORKSPACE_BYTES
 * per device, held from library load until process exit): the window's rotated
 * RoPE keys and, when they fit beside them, the split-KV partials and arrival
 * counters of videomla_attention_workspace_size_split().  The function itself
 * allocates nothing and frees nothing.
 *
 * Arguments, results and arithmetic are those of videomla_attention.
 * - Sizes: if videomla_attention_workspace_size(dims, window, batch) exceeds
 *   VIDEOMLA_STATIC_WORKSPACE_BYTES the call returns VIDEOMLA_EINVAL and
 *   launches nothing.  When the preferred split's partials do not fit beside
 *   the RoPE keys the call runs with the largest split that fits, or unsplit,
 *   or on head-packed tiles (videomla_set_attention_tiling) where those need
 *   fewer waves: the 1560-query Wan frame step (156 per-head units) runs on
 *   147 head-packed CTAs here as in videomla_attention; a few query tiles
 *   against a long window (e.g. 128 queries, 12 heads, 21 Wan frames: 4.8 MB
 *   of partials) keep their split.  Results agree with videomla_attention to
 *   rounding either way.
 * - Set-up: every call looks up the device address of the scratch array in the
 *   current context (cudaGetSymbolAddress); the first such lookup on a device
 *   may load the library's kernels, so make the first call before any stream
 *   capture.
 * - Sharing: every call on a device uses the same scratch array and leaves the
 *   last call's contents in it.  Nothing in it needs to start at zero: each call
 *   rewrites every RoPE row it reads, and the window pre-pass of each call zeroes
 *   the split counters before the attention kernel uses them.  Calls whose
 *   kernels can overlap on the GPU (different streams without ordering between
 *   them) race on the array; issue them on one stream or order them.
 */
int videomla_attention_static_workspace(const videomla_dims* dims, const void* q_nope, const void* q_rope,
                                        const void* W_uk, const void* W_uv, const void* cache,
                                        const videomla_window* window, int batch, int n_query,
                                        void* out, float* lse, void* stream);

/* Name of an error code (static string, never NULL). */
const char* videomla_strerror(int code);

/*
 * Device status word of the current device: VIDEOMLA_OK, or VIDEOMLA_ETIMEOUT if
 * a kernel gave up a bounded wait since the last reset.  Synchronises the device.
 * reset != 0 clears the word.  Returns ECUDA if it cannot be read.
 */
int videomla_device_status(int reset);

/*
 * Upper bound, in nanoseconds, of every device-side wait of later launches on
 * this process (default 2e9).  A wait that runs out makes its kernel record
 * VIDEOMLA_ETIMEOUT, release its tensor memory and return.  0 restores the
 * default.  Returns the previous value.
 */
uint64_t videomla_set_wait_timeout_ns(uint64_t ns);

/*
 * How videomla_attention / videomla_attention_sink assign query rows to CTAs.
 * Every head attends the same latent keys, so a 128-row tile may hold queries of
 * two heads: the CTA applies W_uk,h / W_uv,h of each row's own head in its
 * prologue and epilogue.
 *   VIDEOMLA_TILING_AUTO         (default) per call, the choice with fewer
 *                                wave-quantised key-tile times per SM
 *   VIDEOMLA_TILING_PER_HEAD     one CTA per (128-query tile, head, batch
 *                                element), key tiles split over up to 4 CTAs
 *                                when the units leave SMs idle (split-KV)
 *   VIDEOMLA_TILING_HEAD_PACKED  one CTA per 128 consecutive rows of the
 *                                head-major (head, query) order of a batch
 *                                element, never split: 1560 queries x 12 heads
 *                                take 147 CTAs instead of 156.  Used only where
 *                                n_query >= 128 and Q stays in tensor memory
 *                                (d_c + 128 + 64 + (d_c + d_rope) / 2 <= 512);
 *                                elsewhere the call runs per head.
 * Process-wide, read at each call.  Every mode computes the same attention; a
 * row's arithmetic does not depend on the tile that holds it, except that
 * split-KV merges partial sums.  Returns the previous mode, or VIDEOMLA_EINVAL
 * (nothing changed) for an unknown mode.
 */
#define VIDEOMLA_TILING_AUTO 0
#define VIDEOMLA_TILING_PER_HEAD 1
#define VIDEOMLA_TILING_HEAD_PACKED 2
int videomla_set_attention_tiling(int mode);

/*
 * Self-test of the failure-detection path: launches one CTA that waits, with the
 * same bounded wait the kernels use, on a shared-memory barrier that nothing
 * ever completes.  After ``timeout_ns`` the wait gives up, records
 * VIDEOMLA_ETIMEOUT in the device status word and the kernel returns normally;
 * the context stays usable.  Returns the launch status (VIDEOMLA_OK once
 * enqueued); read the outcome with videomla_device_status().
 */
int videomla_selftest_wait_timeout(uint64_t timeout_ns, void* stream);

/* Library version, major * 10000 + minor * 100 + patch. */
int videomla_version(void);

#ifdef __cplusplus
}
#endif
#endif /* VIDEOMLA_H */
