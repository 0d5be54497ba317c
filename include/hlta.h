/*
 * hlta.h - C ABI of the B200 (sm_100a) Hybrid Linear Temporal Attention library.
 *
 * The operator (Kairos abstract, chatpaper.ai page, item (2); zhichai.net blog, section 2.2
 * "Maintain the world"; researchpapers.dev summary, "How hybrid linear temporal attention
 * suppresses drift") runs three branches over a frame-major video token sequence:
 *   - SWA:  block-causal sliding-window softmax attention over the last w latent frames
 *           ("sliding-window attention captures local dynamics");
 *   - DSWA: dilated sliding-window softmax attention over frames f, f-r, ..., f-r(w-1)
 *           ("dilated sliding windows capture mid-range dependencies");
 *   - GDN:  gated linear attention with the delta rule, the persistent global memory
 *           ("gated linear attention maintains persistent global memory"; decay term
 *           S_t = alpha_t S_{t-1} + ... in the zhaifeiyue.github.io related-papers analysis,
 *           erase-then-write in the llm-atlas long-context explainer, section 06), here
 *           S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,  o_t = S_t q_t.
 *
 * Conventions shared by every call
 * --------------------------------
 * Token l of a clip is l = f*N + n: frame f, token n of that frame (patch raster order).
 * Tensors are dense row-major. q, k, v, o: [B, H, L, d] with L = T*N. Gates a, b: [B, H, L]
 * float32 (GDN heads only). State S: [B, H, d, d] float32, S[i][j] with i the value index
 * and j the key index, so o = S q.
 * Pointers passed to compute calls are DEVICE pointers (cudaMalloc / torch tensors on the
 * GPU), owned by the caller, 16-byte aligned; the library never frees them. Element type:
 * HLTA_BF16 (bf16 in/out, fp32 accumulation and fp32 state) or HLTA_FP32 (fp32 in/out,
 * fp32 arithmetic throughout, no tensor-core rounding).
 * `stream` is a cudaStream_t (NULL: the legacy default stream). Calls are asynchronous:
 * they validate arguments on the host, enqueue kernels on `stream` and return; they never
 * synchronize the stream.
 * Concurrency: the bf16 and E4M3 window attention kernels are persistent (one CTA per SM,
 * taking work from a counter in device memory). Outside the streaming cache, whose steps use
 * the cache's own counter, the library takes the next of 64 counters per device for each
 * launch, so at most 64 such launches may be in flight at once. That includes replays of
 * captured CUDA graphs, whose launches keep the counter they were captured with.
 * Softmax scale: `scale <= 0` selects 1/sqrt(d).
 *
 * Errors: every call returns hlta_status. Argument errors are detected before any launch
 * (nothing is enqueued). HLTA_ERR_CUDA reports a launch or runtime failure (asynchronous
 * faults from earlier work surface at a later call). HLTA_ERR_TIMEOUT is reported by
 * hlta_device_status() when a kernel's bounded wait expired and the kernel stopped early.
 * hlta_last_error() returns a thread-local description of the last non-OK status.
 * No C++ exception crosses this interface.
 *
 * Supported shapes: d = 128 for HLTA_BF16; 1 <= d <= 128 for HLTA_FP32. N >= 1, T >= 1,
 * w >= 1, r >= 1, chunk = 64 (the GDN chunk length; results do not depend on it beyond
 * rounding).
 */
#ifndef HLTA_H
#define HLTA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HLTA_OK = 0,
    HLTA_ERR_INVALID_ARG = 1,
    HLTA_ERR_UNSUPPORTED = 2,
    HLTA_ERR_CUDA = 3,
    HLTA_ERR_TIMEOUT = 4
} hlta_status;

typedef enum { HLTA_BF16 = 0, HLTA_FP32 = 1 } hlta_dtype;

/* Library ABI version (major*10000 + minor*100 + patch). */
int hlta_version(void);

/* Thread-local message describing the last non-OK status returned on this thread. */
const char *hlta_last_error(void);

/*
 * Block-causal sliding-window attention (SWA).
 * For every query token in frame f: softmax over the scaled dot products with every token
 * of frames max(0, f-w+1) .. f (all N tokens of each, including later tokens of frame f),
 * then the weighted sum of their values. Defined by the Kairos abstract's "sliding-window
 * attention captures local dynamics" read as: window = the last w latent frames, the
 * current one included; bidirectional inside a frame, causal across frames.
 * q, k, v, o: [B, H, T*N, d] device, element type `dt`. o is written in full.
 */
hlta_status hlta_swa_fwd(const void *q, const void *k, const void *v, void *o,
                         int B, int H, int T, int N, int d, int w, float scale,
                         hlta_dtype dt, void *stream);

/*
 * Dilated sliding-window attention (DSWA). As hlta_swa_fwd, but the key frames of a query
 * in frame f are f - r*i for i = 0 .. w-1, dropping taps below frame 0 (Kairos abstract:
 * "dilated sliding windows capture mid-range dependencies"). r = 1 gives SWA.
 */
hlta_status hlta_dswa_fwd(const void *q, const void *k, const void *v, void *o,
                          int B, int H, int T, int N, int d, int w, int r, float scale,
                          hlta_dtype dt, void *stream);

/*
 * FP8 (E4M3) window attention: the related-papers analysis (zhaifeiyue.github.io, row C1 and
 * the paragraphs on deployment quantisation) reports that the deployed model quantises
 * attention to FP8 without giving the method; this is one. Codes are OCP 8-bit floating
 * point E4M3 (bias 7, largest finite 448) with fp32 scales, x ~ code * scale:
 *   queries: one scale per 128-row block of each head's T*N rows,
 *   keys:    one scale per 64-row run of each frame (ceil(N/64) runs per frame; the last run
 *            of a frame is short when N % 64 != 0),
 *   values:  one scale per channel of each head.
 * hlta_fp8_quantize_rows / hlta_fp8_quantize_channels produce these from bf16 tensors.
 *
 * Row-block quantisation of x [B, H, L, d] bf16 (device), d = 128: each head is cut into
 * frames of frame_rows rows (the last one may be short), each frame into runs of block_rows
 * rows (1 <= block_rows <= 128; the last run of a frame may be short). Per block:
 * amax = max |x - shift| (fp32), codes = E4M3 round-to-nearest-even, saturating, of
 * (x - shift) * (448 / amax), scale = amax / 448 (0 and all-zero codes for amax = 0); each of
 * the fp32 operations is one IEEE rounding. shift: [B, H, d] float32 subtracted from every
 * row first (e.g. the per-channel mean of K, which leaves softmax attention unchanged), or
 * NULL. x8: [B, H, L, d] bytes; scales: [B, H, ceil(L/frame_rows), ceil(frame_rows/block_rows)]
 * float32. For the attention: q with frame_rows = T*N, block_rows = 128; k with
 * frame_rows = N, block_rows = 64. All pointers device, 16-byte aligned, caller-owned;
 * enqueued on `stream`. Bad shapes or pointers: HLTA_ERR_INVALID_ARG / HLTA_ERR_UNSUPPORTED.
 */
hlta_status hlta_fp8_quantize_rows(const void *x, const float *shift, int B, int H, long L,
                                   int d, long frame_rows, int block_rows, void *x8,
                                   float *scales, void *stream);

/*
 * Per-channel quantisation of x [B, H, L, d] bf16 (device), d = 128: per (head, channel)
 * amax over the L rows, codes and scale as above. x8: [B, H, L, d] bytes; scales: [B, H, d]
 * float32 (also used as scratch while the maxima are gathered). Enqueues four operations on
 * `stream`.
 */
hlta_status hlta_fp8_quantize_channels(const void *x, int B, int H, long L, int d, void *x8,
                                       float *scales, void *stream);

/*
 * Window attention of E4M3 inputs (SWA for r = 1, DSWA otherwise; windows as hlta_dswa_fwd).
 * q8, k8, v8: [B, H, T*N, d] E4M3 codes (device, d = 128); q_scales [B, H, ceil(T*N/128)],
 * k_scales [B, H, T, ceil(N/64)], v_scales [B, H, d] float32 as produced above; o:
 * [B, H, T*N, d] bf16. The result approximates the attention of the dequantised inputs:
 * both products run on E4M3 tensor-core operands with fp32 accumulation, and the softmax
 * weights are rounded to E4M3 (relative error <= 2^-4 each) before they multiply V.
 * scale <= 0 selects 1/sqrt(d). Errors as hlta_swa_fwd.
 */
hlta_status hlta_window_fp8_fwd(const void *q8, const float *q_scales, const void *k8,
                                const float *k_scales, const void *v8, const float *v_scales,
                                void *o, int B, int H, int T, int N, int d, int w, int r,
                                float scale, void *stream);

/*
 * Training pair of the windowed attention (the backbone is trained from scratch: related-papers
 * analysis, row E). hlta_window_fwd_lse is hlta_dswa_fwd (bf16, d = 128; r = 1 gives SWA) that
 * also writes lse [B, H, T*N] float32 (device): the natural log-sum-exp of each query row's
 * scaled scores over its window keys, the softmax normaliser the backward pass reuses.
 */
hlta_status hlta_window_fwd_lse(const void *q, const void *k, const void *v, void *o,
                                float *lse, int B, int H, int T, int N, int d, int w, int r,
                                float scale, void *stream);

/* Workspace bytes of hlta_window_bwd: one float per query row (B*H*T*N*4, 256-byte rounded). */
size_t hlta_window_bwd_workspace_bytes(int B, int H, int T, int N);

/*
 * Backward pass of the windowed attention: the reverse-mode derivative of o = softmax(scale
 * q k^T over the window) v for the upstream gradient dO:
 *   D_i = dO_i . o_i,  p_ij = exp(scale q_i.k_j - lse_i),  dS_ij = p_ij (dO_i.v_j - D_i),
 *   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,  dv_j = sum_i p_ij dO_i.
 * q, k, v, o, dO, dq, dk, dv: [B, H, T*N, d] bf16 device (d = 128); o and lse as written by
 * hlta_window_fwd_lse with the same q, k, v, w, r, scale. dq, dk, dv are overwritten.
 * workspace: device scratch of at least hlta_window_bwd_workspace_bytes(...), caller-owned,
 * 16-byte aligned. Enqueued on `stream` (three launches). Errors as hlta_swa_fwd, plus
 * HLTA_ERR_INVALID_ARG for a short workspace.
 */
hlta_status hlta_window_bwd(const void *q, const void *k, const void *v, const void *o,
                            const float *lse, const void *dO, void *dq, void *dk, void *dv,
                            int B, int H, int T, int N, int d, int w, int r, float scale,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * Rotary position embedding of the softmax heads' q and k, in place: the prologue of the SWA /
 * DSWA branches (llm-atlas long-context explainer, position-encoding section: RoPE turns a
 * position into a rotation of Q and K, so their dot product depends on the relative position;
 * Kairos gives RoPE the local position and leaves the global one to the linear path,
 * related-papers analysis row B1). The pair (x_{2i}, x_{2i+1}) of a token at position p turns
 * by the angle p * base^(-2i/d), clockwise for inverse != 0 (the inverse rotation, which is
 * also the map of the gradient, so the backward pass calls the same entry point).
 * p = l mod N, the token's index inside its frame, for pos_mode 0 (the local position; a
 * streaming step's frame index does not enter); p = l, the index in the sequence, for
 * pos_mode 1.
 * q, k: [B, H, L, d] device, element type `dt`, either may be NULL (skipped), not overlapping
 * each other (the same rows passed as both would turn twice); heads
 * [h0, h0 + Hr) are rotated, the others untouched (so the softmax heads of a hybrid tensor
 * can be rotated in place). d even, 2 <= d <= 128; base > 1 finite (10000 is the usual
 * value); N >= 1. The angle is reduced in double precision before a single-precision sine and
 * cosine; the result is rounded to `dt` once. One launch on `stream`. Errors:
 * HLTA_ERR_INVALID_ARG for bad shapes, ranges, base, pos_mode or misaligned (16-byte)
 * pointers.
 */
hlta_status hlta_rope(void *q, void *k, int B, int H, int h0, int Hr, long L, int N, int d,
                      float base, int pos_mode, int inverse, hlta_dtype dt, void *stream);

/* Workspace bytes of hlta_gdn_chunk_bwd (chunk = 64, d = 128): about 0.9 MB per 64-token
 * chunk of every (batch, head) (fp32 chunk intermediates plus the forward's bf16 chunk
 * products); 0 for unsupported arguments. */
size_t hlta_gdn_bwd_workspace_bytes(int B, int H, long L, int d, int chunk);

/*
 * Backward pass of the gated delta rule (training: related-papers analysis, row E): the
 * reverse-mode derivative of hlta_gdn_chunk_fwd's recurrence for the upstream gradients dO of
 * every output and dS_final of the final state (NULL for zero). Computed in chunk form with
 * the chunk start states recomputed from S0 (NULL for zero): a forward pass over the chunks
 * storing each start state, a backward pass over the chunks carrying the state gradient
 * (dS_start = dS_end (gamma I - Kt^T W) + dO^T Qt with the forward's chunk products), and the
 * gradients of every chunk in parallel. fp32 tensors: fp32 arithmetic throughout. bf16
 * tensors: the two passes over the chunks run on the tensor cores from the forward's bf16 chunk
 * products (state and state gradient carried in fp32), side by side on the library's
 * high-priority streams (joined back into `stream` before the gradient launch), and the chunk
 * products take bf16-rounded operands with fp32 accumulation.
 * q, k, v, dO, dq, dk, dv: [B, H, L, d] device, element type `dt` (d = 128); a, b, da, db:
 * [B, H, L] float32 (a > 0); S0, dS_final, dS0: [B, H, d, d] float32 (dS0 NULL to skip).
 * workspace: device scratch of at least hlta_gdn_bwd_workspace_bytes(...), caller-owned, 16-byte
 * aligned. Enqueued on `stream` (four launches for fp32, five for bf16). Errors as
 * hlta_gdn_chunk_fwd.
 */
hlta_status hlta_gdn_chunk_bwd(const void *q, const void *k, const void *v, const float *a,
                               const float *b, const float *S0, const void *dO,
                               const float *dS_final, void *dq, void *dk, void *dv, float *da,
                               float *db, float *dS0, int B, int H, long L, int d, int chunk,
                               void *workspace, size_t workspace_bytes, hlta_dtype dt,
                               void *stream);

/*
 * Workspace size in bytes needed by hlta_gdn_chunk_fwd for B*H heads of L tokens: the chunk
 * products of every 64-token chunk, and for bf16 heads long enough to be split into
 * segments (see hlta_gdn_chunk_fwd) each segment's fp32 state map and start state.
 */
size_t hlta_gdn_workspace_bytes(int B, int H, long L, int d, int chunk, hlta_dtype dt);

/*
 * Gated delta rule in chunkwise form (UT transform within 64-token chunks, state passed
 * between chunks; llm-atlas long-context explainer, sections 06 and 09: "parallel within a
 * block, recurrent across blocks"). Result equals the token recurrence
 *   S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S_t q_t
 * in sequence order l = 0 .. L-1 for each (batch, head), up to rounding.
 * q, k, v, o: [B, H, L, d] device (type `dt`); a, b: [B, H, L] float32 device, with
 * a in (0, 1] and b in [0, 1] (values outside are not rejected; the result is then the
 * same algebra without the contraction guarantee).
 * S0: [B, H, d, d] float32 initial state, or NULL for zero. S_out: final state or NULL;
 * S_out may equal S0 (in-place update).
 * workspace: device scratch of at least hlta_gdn_workspace_bytes(...) bytes, 256-byte
 * aligned, owned by the caller; its contents on entry are ignored.
 */
hlta_status hlta_gdn_chunk_fwd(const void *q, const void *k, const void *v,
                               const float *a, const float *b, void *o,
                               const float *S0, float *S_out,
                               int B, int H, long L, int d, int chunk,
                               void *workspace, size_t ws_bytes,
                               hlta_dtype dt, void *stream);

/*
 * hlta_gdn_chunk_fwd with the GDN heads' prologue fused into the chunk preparation, for
 * callers holding raw projections. The delta rule contracts only for unit keys and gates in
 * range (researchpapers.dev summary, Theorem 2: ||I - b k k^T|| <= 1 for ||k|| = 1, b in
 * [0, 1]); here the library establishes that itself: q and k of every token are scaled to
 * unit L2 norm (a zero vector stays zero), and the gates are
 *   a = exp(-c * softplus(x)) in (0, 1],   b = sigmoid(y) in (0, 1),
 * so the result equals hlta_gdn_chunk_fwd on (q/|q|, k/|k|, v, a, b) up to rounding.
 * q, k: raw [B, H, L, d] (type `dt`); x, y: [B, H, L] float32 device; c: finite, >= 0 (the
 * decay strength; c = 0 gives a = 1). The normalised q, k never reach device memory:
 * the preparation normalises its staged copy and rounds it to `dt` once. Other arguments
 * and errors as hlta_gdn_chunk_fwd; an invalid c is HLTA_ERR_INVALID_ARG.
 */
hlta_status hlta_gdn_chunk_fwd_raw(const void *q, const void *k, const void *v,
                                   const float *x, const float *y, float c, void *o,
                                   const float *S0, float *S_out,
                                   int B, int H, long L, int d, int chunk,
                                   void *workspace, size_t ws_bytes,
                                   hlta_dtype dt, void *stream);

/*
 * hlta_gdn_chunk_fwd for callers that cannot allocate device memory (no counterpart on the
 * pages: an interface addition of this library). Some callers may not allocate: code embedded
 * in a host application that owns the device-memory budget and passes in only inputs and
 * outputs, or a latency-critical loop that must never enter the allocator. This entry point
 * takes no workspace; its scratch is a fixed array of HLTA_STATIC_SCRATCH_BYTES compiled into
 * the library, which every GPU that uses the library keeps reserved until the process exits.
 * It calls no allocator (no cudaMalloc / cudaFree, no allocating library routine).
 * Arguments and results are those of hlta_gdn_chunk_fwd (same kernels). Problems whose
 * hlta_gdn_workspace_bytes() exceeds HLTA_STATIC_SCRATCH_BYTES are rejected with
 * HLTA_ERR_INVALID_ARG before anything is enqueued.
 * The first call on a device looks up the scratch's device address (cudaGetSymbolAddress);
 * make that first call before any stream capture on that device.
 * Every call on a device shares the one scratch array, and the array keeps the last call's
 * contents (nothing in it needs to start at zero). Calls whose GPU work overlaps in time (on
 * different streams, or from different host threads without ordering) race on the scratch and
 * give wrong results; order them on one stream.
 */
#define HLTA_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)
hlta_status hlta_gdn_chunk_fwd_static(const void *q, const void *k, const void *v,
                                      const float *a, const float *b, void *o,
                                      const float *S0, float *S_out,
                                      int B, int H, long L, int d, int chunk,
                                      hlta_dtype dt, void *stream);

/* Workspace size in bytes for hlta_hybrid_fwd. */
size_t hlta_hybrid_workspace_bytes(int B, int Hg, int T, int N, int d, int chunk,
                                   hlta_dtype dt);

/*
 * The hybrid operator: heads [0, Hs) run SWA(w_swa), heads [Hs, Hs+Hd) run DSWA(w_dswa, r),
 * heads [Hs+Hd, H) run the gated delta rule; outputs are concatenated on the head axis
 * (each branch writes its own head range of o, in place).
 * q, k, v, o: [B, H, T*N, d] with H = Hs + Hd + Hg; a, b: [B, Hg, T*N] float32.
 * S0 / S_out: [B, Hg, d, d] float32 or NULL (as hlta_gdn_chunk_fwd).
 * The GDN branch runs on a library-owned stream of the highest priority, ordered after
 * `stream` by an event, so the branches overlap. bf16: the SWA and DSWA heads run as one
 * persistent attention launch on `stream`, started after the GDN chunk preparation, leaving
 * the GDN chain its SMs; a second launch of the same kernel queued behind the chain on the GDN
 * stream takes the units still left. fp32: the DSWA branch runs on a second library-owned
 * stream beside the SWA branch. The call still completes, in stream order, on `stream` (later
 * work on `stream` sees every output).
 */
hlta_status hlta_hybrid_fwd(const void *q, const void *k, const void *v,
                            const float *a, const float *b, void *o,
                            const float *S0, float *S_out,
                            int B, int Hs, int Hd, int Hg, int T, int N, int d,
                            int w_swa, int w_dswa, int r, int chunk, float scale,
                            void *workspace, size_t ws_bytes,
                            hlta_dtype dt, void *stream);

/*
 * hlta_hybrid_fwd with raw GDN inputs: the GDN heads' q, k are scaled to unit L2 norm per
 * token and their gates computed from x, y as in hlta_gdn_chunk_fwd_raw (x, y: [B, Hg, T*N]
 * float32; c >= 0). The softmax heads are unchanged (their q, k are used as given).
 */
hlta_status hlta_hybrid_fwd_raw(const void *q, const void *k, const void *v,
                                const float *x, const float *y, float c, void *o,
                                const float *S0, float *S_out,
                                int B, int Hs, int Hd, int Hg, int T, int N, int d,
                                int w_swa, int w_dswa, int r, int chunk, float scale,
                                void *workspace, size_t ws_bytes,
                                hlta_dtype dt, void *stream);

/*
 * Streaming rollout (zhichai.net blog, section 2.3: the "streaming token" design generates
 * incrementally without waiting for the whole sequence). A cache holds, for B independent
 * rollouts advancing in lockstep, the K/V of the last w_swa frames of the SWA heads, of the
 * last r*(w_dswa-1)+1 frames of the DSWA heads, and the fp32 state of the GDN heads.
 * Each step appends one frame of N tokens per rollout; its output equals the last frame of
 * hlta_hybrid_fwd over all frames appended so far (up to rounding).
 */
typedef struct hlta_stream *hlta_stream_t;

/* Allocates the cache on the current CUDA device (the only call that allocates). S0:
 * [B, Hg, d, d] float32 device initial state or NULL for zero. Starts at frame 0. */
hlta_status hlta_stream_create(hlta_stream_t *out, int B, int Hs, int Hd, int Hg, int N,
                               int d, int w_swa, int w_dswa, int r, int chunk, float scale,
                               hlta_dtype dt, const float *S0);

/* hlta_stream_create for steps that append up to max_step_frames frames per rollout at once
 * (hlta_stream_step_frames): the rings keep w_swa - 1 (SWA) and r*(w_dswa-1) (DSWA) earlier
 * frames plus max_step_frames new ones, and the GDN workspace covers max_step_frames * N
 * tokens. max_step_frames in [1, 4096]; hlta_stream_create is this call with 1. */
hlta_status hlta_stream_create_ex(hlta_stream_t *out, int B, int Hs, int Hd, int Hg, int N,
                                  int d, int w_swa, int w_dswa, int r, int chunk, float scale,
                                  int max_step_frames, hlta_dtype dt, const float *S0);

/* One step. q_new, k_new, v_new, o_new: [B, H, N, d] device; a_new, b_new: [B, Hg, N]
 * float32 device. Appends the new K/V to the rings, advances the frame counter. */
hlta_status hlta_stream_step(hlta_stream_t c, const void *q_new, const void *k_new,
                             const void *v_new, const float *a_new, const float *b_new,
                             void *o_new, void *stream);

/* F frames per rollout in one step (a rollout of F frames whose inputs are all known, e.g. the
 * conditioning frames): q, k, v, o: [B, H, F*N, d] device; a, b: [B, Hg, F*N] float32. The
 * result equals F successive hlta_stream_step calls on the frame slices (up to rounding): the
 * new frames attend to each other exactly as to cached ones (block-causal windows), and the
 * GDN state advances over the F*N tokens. 1 <= F <= the cache's max_step_frames, else
 * HLTA_ERR_INVALID_ARG. */
hlta_status hlta_stream_step_frames(hlta_stream_t c, const void *q, const void *k,
                                    const void *v, const float *a, const float *b, void *o,
                                    int F, void *stream);

/* Device pointer to the carried GDN state [B, Hg, d, d] (owned by the cache) and the
 * number of frames appended so far by the calls made on the host. */
hlta_status hlta_stream_state(hlta_stream_t c, float **S_dev, int *frames_done);

/*
 * Replaying steps (the rollout part of deployment: the pages' streaming-token design runs the
 * same step frame after frame). A step's frame index lives in a device counter owned by the
 * cache: the ring appends and the attention kernels read it when they run, and every step
 * ends by advancing it by F in stream order. A step captured into a CUDA graph (stream capture
 * on `stream`, whose library-internal branch streams join the capture through events) can
 * therefore be replayed for successive frames, with the new frame's inputs written into the
 * captured input buffers before each replay; the host-side count of hlta_stream_state then
 * counts calls, not replays. The cache creates the library's per-device helpers, so no step
 * needs to do so during a capture. *f_dev receives the counter's device address (an int,
 * owned by the cache): the number of frames appended so far, replays included.
 */
hlta_status hlta_stream_frame_counter(hlta_stream_t c, int **f_dev);

/*
 * Checkpoint and resume of a streaming cache (a rollout paused and continued later, in this
 * process or another one). A checkpoint is a flat byte image: a 64-byte header (magic
 * "HLTC", format version 1, the cache's geometry, scale and element type, the frames a step
 * may append (which fix the ring slot counts) and the number of frames appended, replays
 * included) followed by the carried GDN state
 * [B, Hg, d, d] float32 and the four rings (SWA K, SWA V, DSWA K, DSWA V, in the cache's
 * layout). A cache resumed from it continues exactly as the saved one would have: the next
 * steps give bit-identical outputs.
 *
 * hlta_stream_checkpoint_bytes: the image size of this cache (0 for a NULL cache).
 * hlta_stream_save: writes the image to `dst` (host memory, pageable or pinned, at least
 *   hlta_stream_checkpoint_bytes bytes, owned by the caller) after the work already enqueued
 *   on `stream` (NULL: the legacy default stream); returns when the image is complete.
 * hlta_stream_load: replaces the cache's state, rings and frame count with the image in
 *   `src` (host memory, `bytes` long), in order on `stream`; returns when the copies are done.
 *   HLTA_ERR_INVALID_ARG for a wrong magic, version or size, or an image of a cache created
 *   with other arguments (the cache is then left unchanged).
 * Neither call allocates device memory; both return HLTA_ERR_CUDA if a copy fails.
 */
size_t hlta_stream_checkpoint_bytes(hlta_stream_t c);
hlta_status hlta_stream_save(hlta_stream_t c, void *dst, size_t bytes, void *stream);
hlta_status hlta_stream_load(hlta_stream_t c, const void *src, size_t bytes, void *stream);

/* Frees the cache. Synchronizes the device first. */
hlta_status hlta_stream_destroy(hlta_stream_t c);

/*
 * Profiling hook for hlta_hybrid_fwd(_raw) and the streaming steps (measurement, not needed
 * for results). `events` is NULL (off) or an array of 5 cudaEvent_t created by the caller on
 * the current device. While set, each hybrid call or streaming step records events[0] where
 * the softmax branches start (on the caller's stream, before their first kernel; with bf16 GDN
 * heads, after the wait for the GDN chunk preparation), events[1] after the SWA kernel
 * (caller's stream), events[2] after the DSWA kernel (on the stream it ran on; with bf16 both
 * branches share one attention launch, and events[2] follows its late CTAs on the GDN stream
 * when there are any), events[3] before and events[4] after the GDN kernels (on the GDN
 * stream). The array is
 * copied; the setting is process-wide and stays until changed.
 */
hlta_status hlta_set_profile_events(void *const *events);

/*
 * Measurement hook: the number of kernels this library has enqueued in this process so far
 * (all devices, all host threads; replays of a captured CUDA graph are not calls and are not
 * counted). The difference over a region is the number of the library's kernel launches in it.
 */
unsigned long long hlta_kernel_launches(void);

/* Bits of the device error word (hlta_device_status): the kernel kind whose bounded wait
 * expired. */
#define HLTA_DEVERR_ATTN_WAIT 0x1u  /* a window-attention kernel (forward or backward) */
#define HLTA_DEVERR_GDN_WAIT 0x2u   /* a gated-delta-rule kernel */
#define HLTA_DEVERR_SELFTEST 0x4u   /* hlta_wait_expiry_selftest */

/*
 * Synchronizes `stream`, then reads and clears the library's device error word.
 * *code receives the raw word (0: no kernel stopped early; otherwise HLTA_DEVERR_* bits).
 * Returns HLTA_ERR_TIMEOUT if a bounded wait expired in any kernel since the last call,
 * HLTA_ERR_CUDA on a CUDA error.
 */
hlta_status hlta_device_status(void *stream, unsigned int *code);

/*
 * Failure-detection self-test (no counterpart on the pages: it exercises this library's own
 * bounded-wait protocol). Every pipelined kernel of the library waits on its mbarriers with a
 * cycle limit, after which it records its HLTA_DEVERR_* bit in the device error word, stops
 * its roles and returns, so a lost arrival ends in an error status instead of a hung GPU.
 * This call enqueues on `stream` one single-thread kernel that makes such a wait run out: it
 * waits on a fresh shared-memory mbarrier that nothing arrives at, through the same bounded
 * wait, for `cycles` SM clock cycles (1 <= cycles <= 2^32; 2^24 is about 9 ms at 1.9 GHz),
 * then ORs HLTA_DEVERR_SELFTEST into the word and returns. No copy or tensor-core operation is
 * in flight, so the context stays usable: the next hlta_device_status() reports
 * HLTA_ERR_TIMEOUT with that bit and clears it. A `cycles` outside the range is
 * HLTA_ERR_INVALID_ARG (nothing enqueued).
 */
hlta_status hlta_wait_expiry_selftest(unsigned long long cycles, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HLTA_H */
