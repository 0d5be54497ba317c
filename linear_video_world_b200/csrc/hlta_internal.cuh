// Internal declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include "hlta.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace hlta {

// Windowed softmax attention over frames. One description covers SWA (r = 1), DSWA and the
// streaming step: queries are rows of a [B][q_Htot][q_rows][d] tensor (this branch's heads
// start at q_h0); query row n lies in frame fq0 + n / N. Keys and values are rows of a
// [B][kv_Htot][kv_rows][d] tensor; key frame fk occupies rows (fk % kv_slots) * N ...
// (a clip when kv_slots covers every frame, a ring of frame slots when streaming).
// The key frames of query frame f are f - r*i for i in [0, w), kept when >= 0.
struct AttnArgs {
    const void *q, *k, *v;
    void *o;
    int B, Hbr;
    int q_Htot, q_h0;
    long q_rows;
    int kv_Htot, kv_h0;
    long kv_rows;
    int kv_slots;
    int N, d, w, r;
    int fq0;
    const int *fq0_dev = nullptr;   // if set, fq0 is read from this device int when the kernel runs
    float scale;
    unsigned int *err;   // device error word (bounded waits that expired)
    // E4M3 inputs only: fp32 scales of the query blocks ([B*q_Htot][ceil(q_rows/128)]), the
    // key tiles ([B*kv_Htot][kv_slots][ceil(N/64)]) and the value channels ([B*kv_Htot][d])
    const float *qs = nullptr, *ks = nullptr, *vs = nullptr;
    // bf16 kernel only: per query row log-sum-exp (natural log) of the scaled scores
    // ([B*q_Htot][q_rows] float32), written when non-null
    float *lse = nullptr;
    // bf16 / E4M3 kernel: the launch's work counter (two device ints, zero between launches,
    // used by one launch at a time), or null for one of the library's 64 shared counters
    int *sched = nullptr;
};

// Gated delta rule over [B][Htot][L][d] tensors, this branch's heads at h0 .. h0 + Hg.
// Gates a, b: [B][Hg][L]. State: [B][Hg][d][d] (S[i][j], i value index, j key index).
struct GdnArgs {
    const void *q, *k, *v;
    const float *a, *b;         // gates; with `raw` the raw gate inputs x, y instead
    int raw;                    // 1: q, k raw (scaled to unit L2 norm per token inside the
                                //    chunk preparation), a = exp(-raw_c softplus(x)), b = sigmoid(y)
    float raw_c;
    void *o;
    int B, Hg, Htot, h0;
    long L;
    int d, chunk;
    const float *S0;
    float *S_out;
    void *ws;
    size_t ws_bytes;
    unsigned int *err;
    // optional (bf16 state pass): each chunk's start state, [d][d] fp32 at
    // S_chunks + (bh * nchunks + c) * S_chunk_stride; with o null the outputs are skipped
    float *S_chunks;
    long S_chunk_stride;
    // bf16 pass over the chunks: segments per head of the two-level scan (0: as many as keep
    // the latency low; 1: one serial chain per head on as few SMs as possible, for a branch
    // that runs beside other work); at most the count the workspace was sized for
    int scan_segments;
    // bf16: when set, recorded on the launch stream after the chunk preparation (work that
    // holds SMs for long, such as the persistent attention launch, waits for it)
    cudaEvent_t prep_done = nullptr;
};

// Chunk workspace (per GDN head, per chunk of C tokens; elements of type E):
//   W  = T diag(b e^g) K,   Up = T diag(b) V,   Op = P Up,
//   Qt = diag(e^g) Q - P W, Kt = diag(e^{g_C - g}) K        each [C][d]
//   gam = e^{g_C}                               one float per chunk, in a 16-byte slot
// laid out as five arrays [BHg][nchunks][C][d] followed by gam [BHg][nchunks][4]; the bf16
// path stores Up and Op of a chunk transposed, [d][C] (state row by token).
struct GdnWorkspace {
    void *W, *Up, *Op, *Qt, *Kt;
    float *gam;
};

__host__ __device__ inline long gdn_num_chunks(long L, int C) { return (L + C - 1) / C; }
// the layout above (the fp32 path, and the bf16 chunk products the backward pass uses)
size_t gdn_rowmajor_bytes(long BH, long L, int d, int C, bool bf16);
GdnWorkspace gdn_workspace_carve(void *base, long BH, long L, int d, int C, bool bf16);
// workspace of hlta_gdn_chunk_fwd: the layout above for fp32, GdnWs2 for bf16
size_t gdn_workspace_bytes(long BH, long L, int d, int C, bool bf16);

// Chunk workspace of the bf16 forward (d = 128, C = 64), per chunk of a head, every array
// [BHg * nchunks][128][64] bf16 (state row, or key index, by token):
//   Wt = W^T, Qt = Qt^T, Ut = Up^T, Ot = Op^T,
//   scal: GDN_SCAL floats, gam = e^{g_n} at 0, ek_t = e^{g_n - g_t} (times 1/|k_t| for raw
//         inputs, 0 past the chunk's end) at 4 + t,
// then the segment scan's fp32 maps and start states (gdn_scan_bytes).
constexpr int GDN_SCAL = 68;
struct GdnWs2 {
    void *Wt, *Qt, *Ut, *Ot;
    float *scal;
    float *scan;
};
GdnWs2 gdn_ws2_carve(void *base, long BH, long L);

// Records the thread-local message returned by hlta_last_error() and returns `st`.
int record_error_impl(int st, const char *fmt, ...);
#define record_error(st, ...) ((hlta_status)::hlta::record_error_impl((int)(st), __VA_ARGS__))

// 2-D TMA tensor map over a row-major [rows][cols] bf16 tensor with a box of
// box_rows x box_cols, 128-byte swizzle or none.
cudaError_t make_tmap_2d_bf16(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                              uint32_t box_cols, uint32_t box_rows, bool swizzle128);
// The same over fp32 (box_cols * 4 <= 128 with the swizzle).
cudaError_t make_tmap_2d_f32(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                             uint32_t box_cols, uint32_t box_rows, bool swizzle128);
// The same over bytes (E4M3 codes), always with the 128-byte swizzle (box_cols <= 128).
cudaError_t make_tmap_2d_u8(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                            uint32_t box_cols, uint32_t box_rows);

// Launchers. Return cudaGetLastError() of their launches.
cudaError_t launch_attn_f32(const AttnArgs &a, cudaStream_t s);
// bf16 window attention: 128-key tiles, two query sub-tiles, P staged in shared memory; a
// persistent launch of one CTA per SM (attn_tc2.cu)
cudaError_t launch_attn_bf16_tc2(const AttnArgs &a, cudaStream_t s);
// The same over one or two branches in one launch (the branches share q, o, B, q_rows, N, d,
// fq0, scale and err; cudaErrorInvalidValue otherwise), leaving `reserve_sms` SMs (at most
// half) to kernels that run beside it on `s_fill`; with `s_fill` set, a second launch of that
// many CTAs, queued on `s_fill` behind them, takes the remaining units from the same counter
cudaError_t launch_attn_bf16_tc2_multi(const AttnArgs *br, int nbr, int reserve_sms, cudaStream_t s,
                                       cudaStream_t s_fill);
// the same two-tile design on E4M3 codes (attn_tc2.cu)
cudaError_t launch_attn_fp8_tc2(const AttnArgs &a, cudaStream_t s);
// E4M3 quantisation (bf16 input, d = 128): row blocks inside frames, and value channels
cudaError_t launch_fp8_quantize_rows(const void *x, const float *shift, long BH, long L,
                                     long frame_rows, int block_rows, void *x8, float *scales,
                                     cudaStream_t s);
cudaError_t launch_fp8_quantize_channels(const void *x, long BH, long L, void *x8,
                                         float *scales, cudaStream_t s);
// Window attention backward (bf16, d = 128): D = rowsum(dO o O) into `Dws` ([BH][L] fp32),
// then dq (query-tile major) and dk, dv (key-tile major).
struct AttnBwdArgs {
    const void *q, *k, *v, *o, *dO;
    const float *lse;
    void *dq, *dk, *dv;
    float *Dws;
    int BH, T, N, w, r;
    float scale;
};
cudaError_t launch_attn_bwd(const AttnBwdArgs &a, cudaStream_t s);
cudaError_t launch_attn_bwd_tc(const AttnBwdArgs &a, cudaStream_t s);
// Gated delta rule backward (chunk form, fp32 arithmetic, d = 128): q, k, v, dO, dq, dk, dv
// [B][H][L][d] (bf16 when `bf16`, else fp32); a, b, da, db [B][H][L]; S0, dS_final, dS0
// [B][H][d][d] fp32 (S0 / dS_final null for zero, dS0 null to skip).
struct GdnBwdArgs {
    const void *q, *k, *v, *dO;
    const float *a, *b, *S0, *dS_final;
    void *dq, *dk, *dv;
    float *da, *db, *dS0;
    void *ws;
    int B, H, d;
    long L;
    bool bf16;
    unsigned int *err;
};
size_t gdn_bwd_workspace_bytes(long BH, long L);
// Two side streams and four events for running the bf16 backward's serial state passes
// beside its parallel chunk preparation (null: everything on the caller's stream)
struct SideStreams {
    cudaStream_t a, b;
    cudaEvent_t fork, mid, join_a, join_b;
};
// The two state passes of the bf16 backward on the tensor cores, from the forward's bf16
// chunk products (g.ws: a bf16 forward workspace; g.o null): the forward pass storing each
// chunk's start state (g.S_chunks), and the backward pass over the chunks storing each chunk's
// end-state gradient at dS_chunks + (bh * nchunks + c) * g.S_chunk_stride and the initial
// state's gradient in dS0 (null to skip); dS_final null for zero.
// The forward preparation and state pass run on `s`, the state-gradient pass on `s2` after
// the preparation (event `mid`, recorded on `s`; unused when s2 == s).
cudaError_t launch_gdn_bf16_bwd_states(const GdnArgs &g, const void *dO, const float *dS_final,
                                       float *dS_chunks, float *dS0, cudaStream_t s,
                                       cudaStream_t s2, cudaEvent_t mid);
cudaError_t launch_gdn_bwd(const GdnBwdArgs &a, cudaStream_t s, const SideStreams *side);
cudaError_t launch_gdn_f32(const GdnArgs &g, cudaStream_t s);
// The bf16 pass over the chunks as a two-level segment scan (gdn_scan.cu): segment length in
// chunks, the fp32 scratch it needs after the chunk workspace (0 for a single segment), and
// the launches (segment maps, their composition, the replay with outputs) after the prep.
int gdn_scan_segment_len(long BH, long nch);
// segments per head for a GDN branch running beside softmax work of `attn_flop` (the fewest
// whose serial chain still ends within that work's estimated time)
int gdn_scan_segments_beside(long BH, long nch, double attn_flop);
size_t gdn_scan_bytes(long BH, long nch);
cudaError_t launch_gdn_bf16_scan(const GdnArgs &g, const GdnWs2 &ws, cudaStream_t s);
// the bf16 forward: the tensor-core chunk preparation, then the segment scan
cudaError_t launch_gdn_bf16_v2(const GdnArgs &g, cudaStream_t s);
// f0: the first new frame's index, read from f0_dev when that is set (streaming steps keep
// their frame counter on the device so that a captured step can be replayed)
cudaError_t launch_ring_append(const void *src, int B, int Htot, int h0, int Hbr, int N, int d,
                               size_t elem, int F, void *ring, int slots, int f0,
                               const int *f0_dev, cudaStream_t s);
// *f += F on the device (one thread), in stream order
cudaError_t launch_frame_advance(int *f, int F, cudaStream_t s);

// Rotary embedding of heads [h0, h0 + Hr) of q and k ([B][Htot][L][d], either may be null),
// in place; sign -1 for the inverse rotation
cudaError_t launch_rope(void *q, void *k, bool bf16, int B, int Htot, int h0, int Hr, long L,
                        int N, int d, double base, int pos_mode, int sign, cudaStream_t s);

// Device error word: kernels OR a code into it when a bounded wait expires (the bits are the
// HLTA_DEVERR_* values of hlta.h).
enum : unsigned int {
    DEVERR_ATTN_WAIT = 1u << 0,
    DEVERR_GDN_WAIT = 1u << 1,
    DEVERR_SELFTEST = 1u << 2,
};
static_assert(DEVERR_ATTN_WAIT == HLTA_DEVERR_ATTN_WAIT && DEVERR_GDN_WAIT == HLTA_DEVERR_GDN_WAIT &&
                  DEVERR_SELFTEST == HLTA_DEVERR_SELFTEST,
              "device error bits must match hlta.h");

// Counts one kernel launch enqueued by the library (hlta_kernel_launches); every launch site
// appends it to its launch statement.
void note_launch();

// The bounded-wait self-test kernel: waits `cycles` on an mbarrier nothing arrives at.
cudaError_t launch_wait_selftest(unsigned int *err, long long cycles, cudaStream_t s);
unsigned int *device_error_word();  // device address of the word (current device)

}  // namespace hlta
