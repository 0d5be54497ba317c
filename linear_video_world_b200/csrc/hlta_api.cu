// C ABI of the library: argument validation, dispatch to the kernels, the hybrid operator's
// branch fork/join, the streaming cache and the device error word. Declarations and the
// contract of every entry point are in include/hlta.h.
#include "hlta.h"
#include "hlta_internal.cuh"

#include <algorithm>
#include <atomic>
#include <math.h>
#include <mutex>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

namespace hlta {

__device__ unsigned int g_device_error;

namespace {

thread_local char t_msg[512] = "";

hlta_status fail(hlta_status st, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_msg, sizeof t_msg, fmt, ap);
    va_end(ap);
    return st;
}

hlta_status cuda_fail(cudaError_t e, const char *where)
{
    return fail(HLTA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Per-device helpers: the device error word's address and an auxiliary stream plus two
// events for the hybrid operator's fork/join. Created once per device, kept until exit.
struct DeviceCtx {
    bool ready = false;
    unsigned int *err = nullptr;
    cudaStream_t aux = nullptr;     // GDN branch (highest priority)
    cudaStream_t aux2 = nullptr;    // DSWA branch of the hybrid (default priority)
    cudaStream_t aux3 = nullptr;    // second serial pass of the GDN backward (highest priority)
    cudaEvent_t fork = nullptr, join = nullptr, join2 = nullptr, mid = nullptr;
    cudaEvent_t prep = nullptr;     // the GDN branch's chunk preparation done (bf16)
};
constexpr int kMaxDevices = 64;
DeviceCtx g_ctx[kMaxDevices];
std::mutex g_ctx_mu;
std::mutex g_fork_mu;   // the per-device fork/join events are shared by all host threads
cudaEvent_t g_prof[5];  // profiling events of hlta_set_profile_events (guarded by g_fork_mu)
bool g_prof_on = false;

void prof_record(int i, cudaStream_t s)
{
    if (g_prof_on && g_prof[i]) cudaEventRecord(g_prof[i], s);
}

hlta_status device_ctx(DeviceCtx **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(HLTA_ERR_UNSUPPORTED, "device %d", dev);
    std::lock_guard<std::mutex> lk(g_ctx_mu);
    DeviceCtx &c = g_ctx[dev];
    if (!c.ready) {
        if ((e = cudaGetSymbolAddress((void **)&c.err, g_device_error)) != cudaSuccess)
            return cuda_fail(e, "cudaGetSymbolAddress(error word)");
        // The GDN branch (a short parallel prep, then a long serial chain on a few SMs) runs
        // on this stream at the highest priority: its CTAs are dispatched ahead of the
        // softmax branches' whenever SMs free up, so the serial chain starts right after its
        // prep and the softmax kernels fill the remaining SMs around it.
        int least = 0, greatest = 0;
        if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess)
            return cuda_fail(e, "cudaDeviceGetStreamPriorityRange");
        if ((e = cudaStreamCreateWithPriority(&c.aux, cudaStreamNonBlocking, greatest)) != cudaSuccess)
            return cuda_fail(e, "cudaStreamCreateWithPriority");
        if ((e = cudaEventCreateWithFlags(&c.fork, cudaEventDisableTiming)) != cudaSuccess)
            return cuda_fail(e, "cudaEventCreate");
        if ((e = cudaEventCreateWithFlags(&c.join, cudaEventDisableTiming)) != cudaSuccess)
            return cuda_fail(e, "cudaEventCreate");
        // the hybrid's DSWA launch runs beside its SWA launch, so neither waits for the
        // other's last wave of CTAs
        if ((e = cudaStreamCreateWithPriority(&c.aux2, cudaStreamNonBlocking, least)) != cudaSuccess)
            return cuda_fail(e, "cudaStreamCreateWithPriority");
        if ((e = cudaEventCreateWithFlags(&c.join2, cudaEventDisableTiming)) != cudaSuccess)
            return cuda_fail(e, "cudaEventCreate");
        if ((e = cudaStreamCreateWithPriority(&c.aux3, cudaStreamNonBlocking, greatest)) != cudaSuccess)
            return cuda_fail(e, "cudaStreamCreateWithPriority");
        if ((e = cudaEventCreateWithFlags(&c.mid, cudaEventDisableTiming)) != cudaSuccess)
            return cuda_fail(e, "cudaEventCreate");
        if ((e = cudaEventCreateWithFlags(&c.prep, cudaEventDisableTiming)) != cudaSuccess)
            return cuda_fail(e, "cudaEventCreate");
        c.ready = true;
    }
    *out = &c;
    return HLTA_OK;
}

hlta_status check_dtype_d(hlta_dtype dt, int d)
{
    if (dt == HLTA_BF16) {
        if (d != 128) return fail(HLTA_ERR_UNSUPPORTED, "bf16 path supports d = 128 only (got %d)", d);
    } else if (dt == HLTA_FP32) {
        if (d < 1 || d > 128) return fail(HLTA_ERR_UNSUPPORTED, "fp32 path supports 1 <= d <= 128 (got %d)", d);
    } else {
        return fail(HLTA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    }
    return HLTA_OK;
}

hlta_status check_window(int w, int r)
{
    if (w < 1) return fail(HLTA_ERR_INVALID_ARG, "window w must be >= 1 (got %d)", w);
    if (r < 1) return fail(HLTA_ERR_INVALID_ARG, "dilation r must be >= 1 (got %d)", r);
    if ((long)r * (w - 1) > (1L << 24)) return fail(HLTA_ERR_INVALID_ARG, "r*(w-1) too large");
    return HLTA_OK;
}

hlta_status attn_status(cudaError_t e)
{
    if (e == cudaErrorNotSupported) return fail(HLTA_ERR_UNSUPPORTED, "window attention: unsupported shape");
    if (e != cudaSuccess) return cuda_fail(e, "window attention launch");
    return HLTA_OK;
}

// `reserve_sms`: SMs the bf16 kernel (persistent, one CTA per SM) leaves free for the kernels
// queued on `s_fill` (the GDN branch's chain); as many more of its CTAs start behind them
hlta_status run_attn(const AttnArgs &a, hlta_dtype dt, cudaStream_t s, int reserve_sms = 0,
                     cudaStream_t s_fill = nullptr)
{
    if (a.B * a.Hbr == 0 || a.q_rows == 0) return HLTA_OK;
    return attn_status(dt == HLTA_FP32 ? launch_attn_f32(a, s)
                                       : launch_attn_bf16_tc2_multi(&a, 1, reserve_sms, s, s_fill));
}

// The SWA and DSWA branches: on bf16 one persistent launch takes both branches' units (no
// tail between two launches); fp32 launches them one after the other on `s`
hlta_status run_attn_pair(const AttnArgs &a0, const AttnArgs &a1, hlta_dtype dt, cudaStream_t s,
                          int reserve_sms, cudaStream_t s_fill)
{
    if (dt != HLTA_BF16) {
        hlta_status st = run_attn(a0, dt, s);
        return st != HLTA_OK ? st : run_attn(a1, dt, s);
    }
    const AttnArgs br[2] = {a0, a1};
    return attn_status(launch_attn_bf16_tc2_multi(br, 2, reserve_sms, s, s_fill));
}

hlta_status run_gdn(const GdnArgs &g, hlta_dtype dt, cudaStream_t s)
{
    if (g.B * g.Hg == 0) return HLTA_OK;
    cudaError_t e = dt == HLTA_FP32 ? launch_gdn_f32(g, s) : launch_gdn_bf16_v2(g, s);
    if (e == cudaErrorNotSupported) return fail(HLTA_ERR_UNSUPPORTED, "gated delta rule: unsupported shape");
    if (e != cudaSuccess) return cuda_fail(e, "gated delta rule launch");
    return HLTA_OK;
}

AttnArgs clip_attn_args(const void *q, const void *k, const void *v, void *o, int B, int Htot,
                        int h0, int Hbr, int T, int N, int d, int w, int r, float scale,
                        unsigned int *err)
{
    AttnArgs a;
    a.q = q; a.k = k; a.v = v; a.o = o;
    a.B = B; a.Hbr = Hbr;
    a.q_Htot = Htot; a.q_h0 = h0; a.q_rows = (long)T * N;
    a.kv_Htot = Htot; a.kv_h0 = h0; a.kv_rows = (long)T * N; a.kv_slots = T;
    a.N = N; a.d = d; a.w = w; a.r = r; a.fq0 = 0;
    a.scale = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
    a.err = err;
    return a;
}

hlta_status window_fwd(const void *q, const void *k, const void *v, void *o, int B, int H,
                       int T, int N, int d, int w, int r, float scale, hlta_dtype dt,
                       void *stream)
{
    hlta_status st;
    if (!q || !k || !v || !o) return fail(HLTA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(HLTA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (B < 0 || H < 0 || T < 1 || N < 1) return fail(HLTA_ERR_INVALID_ARG, "bad shape B=%d H=%d T=%d N=%d", B, H, T, N);
    if ((long)T * N > (1L << 30)) return fail(HLTA_ERR_INVALID_ARG, "T*N too large");
    if ((st = check_dtype_d(dt, d)) != HLTA_OK) return st;
    if ((st = check_window(w, r)) != HLTA_OK) return st;
    DeviceCtx *ctx;
    if ((st = device_ctx(&ctx)) != HLTA_OK) return st;
    AttnArgs a = clip_attn_args(q, k, v, o, B, H, 0, H, T, N, d, w, r, scale, ctx->err);
    return run_attn(a, dt, (cudaStream_t)stream);
}

hlta_status check_gdn_common(const void *q, const void *k, const void *v, const float *a,
                             const float *b, const void *o, const float *S0, const float *S_out,
                             int d, int chunk, hlta_dtype dt)
{
    hlta_status st;
    if (!q || !k || !v || !a || !b || !o) return fail(HLTA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(a) ||
        !aligned16(b) || (S0 && !aligned16(S0)) || (S_out && !aligned16(S_out)))
        return fail(HLTA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (chunk != 64) return fail(HLTA_ERR_UNSUPPORTED, "chunk must be 64 (got %d)", chunk);
    if ((st = check_dtype_d(dt, d)) != HLTA_OK) return st;
    return HLTA_OK;
}

hlta_status check_raw_c(float c)
{
    if (!(c >= 0.f) || !(c <= 1e30f)) return fail(HLTA_ERR_INVALID_ARG, "decay constant c must be finite and >= 0 (got %g)", (double)c);
    return HLTA_OK;
}

}  // namespace

size_t gdn_rowmajor_bytes(long BH, long L, int d, int C, bool bf16)
{
    const size_t el = bf16 ? 2 : 4;
    const size_t nch = (size_t)gdn_num_chunks(L, C);
    const size_t arr = ((size_t)BH * nch * C * d * el + 255) & ~(size_t)255;
    return 5 * arr + (((size_t)BH * nch * 4 * sizeof(float) + 255) & ~(size_t)255);
}

namespace {
size_t ws2_arr(long BH, long L) { return ((size_t)BH * gdn_num_chunks(L, 64) * 128 * 64 * 2 + 255) & ~(size_t)255; }
size_t ws2_scal(long BH, long L) { return ((size_t)BH * gdn_num_chunks(L, 64) * GDN_SCAL * 4 + 255) & ~(size_t)255; }
}  // namespace

size_t gdn_workspace_bytes(long BH, long L, int d, int C, bool bf16)
{
    if (!bf16 || d != 128 || C != 64) return gdn_rowmajor_bytes(BH, L, d, C, bf16);
    return 4 * ws2_arr(BH, L) + ws2_scal(BH, L) + gdn_scan_bytes(BH, gdn_num_chunks(L, 64));
}

GdnWs2 gdn_ws2_carve(void *base, long BH, long L)
{
    char *p = (char *)base;
    const size_t arr = ws2_arr(BH, L), sc = ws2_scal(BH, L);
    GdnWs2 w;
    w.Wt = p; w.Qt = p + arr; w.Ut = p + 2 * arr; w.Ot = p + 3 * arr;
    w.scal = (float *)(p + 4 * arr);
    w.scan = gdn_scan_bytes(BH, gdn_num_chunks(L, 64)) ? (float *)(p + 4 * arr + sc) : nullptr;
    return w;
}

GdnWorkspace gdn_workspace_carve(void *base, long BH, long L, int d, int C, bool bf16)
{
    const size_t el = bf16 ? 2 : 4;
    const size_t nch = (size_t)gdn_num_chunks(L, C);
    const size_t arr = ((size_t)BH * nch * C * d * el + 255) & ~(size_t)255;
    char *p = (char *)base;
    GdnWorkspace w;
    w.W = p; w.Up = p + arr; w.Op = p + 2 * arr; w.Qt = p + 3 * arr; w.Kt = p + 4 * arr;
    w.gam = (float *)(p + 5 * arr);
    return w;
}

int record_error_impl(int st, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_msg, sizeof t_msg, fmt, ap);
    va_end(ap);
    return st;
}

namespace {
std::atomic<unsigned long long> g_launches{0};
}

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

unsigned int *device_error_word()
{
    DeviceCtx *c = nullptr;
    return device_ctx(&c) == HLTA_OK ? c->err : nullptr;
}

}  // namespace hlta

using namespace hlta;

// ------------------------------------------------------------------------------------
// Streaming cache
// ------------------------------------------------------------------------------------
struct hlta_stream {
    int device;
    int B, Hs, Hd, Hg, N, d, w_swa, w_dswa, r, chunk;
    float scale;
    hlta_dtype dt;
    int max_frames;           // frames one step may append
    int slots_s, slots_d;     // ring slots: SWA w_swa-1, DSWA r*(w_dswa-1) earlier frames plus
                              // max_frames new ones
    void *ks, *vs, *kd, *vd;  // rings [B][Hs][slots_s][N][d], [B][Hd][slots_d][N][d]
    float *S;                 // [B][Hg][d][d]
    void *ws;                 // GDN workspace for max_frames * N tokens
    size_t ws_bytes;
    int frames;               // steps' frames appended, counted on the host per call
    int *fdev;                // the same count on the device: the kernels read it and each step
                              // advances it in stream order, so a captured step can be replayed;
                              // fdev[2..3] are the cache's own work counter of its attention
                              // launch (a captured step then shares no counter with other work)
};

extern "C" {

int hlta_version(void) { return 100; }

const char *hlta_last_error(void) { return t_msg; }

hlta_status hlta_swa_fwd(const void *q, const void *k, const void *v, void *o, int B, int H,
                         int T, int N, int d, int w, float scale, hlta_dtype dt, void *stream)
{
    return window_fwd(q, k, v, o, B, H, T, N, d, w, 1, scale, dt, stream);
}

hlta_status hlta_dswa_fwd(const void *q, const void *k, const void *v, void *o, int B, int H,
                          int T, int N, int d, int w, int r, float scale, hlta_dtype dt,
                          void *stream)
{
    return window_fwd(q, k, v, o, B, H, T, N, d, w, r, scale, dt, stream);
}

hlta_status hlta_fp8_quantize_rows(const void *x, const float *shift, int B, int H, long L,
                                   int d, long frame_rows, int block_rows, void *x8,
                                   float *scales, void *stream)
{
    if (!x || !x8 || !scales) return fail(HLTA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(x) || !aligned16(x8) || !aligned16(scales) || (shift && !aligned16(shift)))
        return fail(HLTA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (B < 0 || H < 0 || L < 0) return fail(HLTA_ERR_INVALID_ARG, "bad shape B=%d H=%d L=%ld", B, H, L);
    if (d != 128) return fail(HLTA_ERR_UNSUPPORTED, "FP8 quantisation supports d = 128 only (got %d)", d);
    if (frame_rows < 1 || block_rows < 1 || block_rows > 128)
        return fail(HLTA_ERR_INVALID_ARG, "need frame_rows >= 1 and 1 <= block_rows <= 128 (got %ld, %d)", frame_rows, block_rows);
    cudaError_t e = launch_fp8_quantize_rows(x, shift, (long)B * H, L, frame_rows, block_rows, x8,
                                             scales, (cudaStream_t)stream);
    if (e == cudaErrorNotSupported) return fail(HLTA_ERR_UNSUPPORTED, "FP8 quantisation: too many blocks");
    if (e != cudaSuccess) return cuda_fail(e, "FP8 row quantisation launch");
    return HLTA_OK;
}

hlta_status hlta_fp8_quantize_channels(const void *x, int B, int H, long L, int d, void *x8,
                                       float *scales, void *stream)
{
    if (!x || !x8 || !scales) return fail(HLTA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(x) || !aligned16(x8) || !aligned16(scales))
        return fail(HLTA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (B < 0 || H < 0 || L < 0) return fail(HLTA_ERR_INVALID_ARG, "bad shape B=%d H=%d L=%ld", B, H, L);
    if (d != 128) return fail(HLTA_ERR_UNSUPPORTED, "FP8 quantisation supports d = 128 only (got %d)", d);
    cudaError_t e = launch_fp8_quantize_channels(x, (long)B * H, L, x8, scales, (cudaStream_t)stream);
    if (e == cudaErrorNotSupported) return fail(HLTA_ERR_UNSUPPORTED, "FP8 quantisation: too many heads");
    if (e != cudaSuccess) return cuda_fail(e, "FP8 channel quantisation launch");
    return HLTA_OK;
}

hlta_status hlta_window_fp8_fwd(const void *q8, const float *q_scales, const void *k8,
                                const float *k_scales, const void *v8, const float *v_scales,
                                void *o, int B, int H, int T, int N, int d, int w, int r,
                                float scale, void *stream)
{
    hlta_status st;
    if (!q8 || !k8 || !v8 || !o || !q_scales || !k_scales || !v_scales)
        return fail(HLTA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) ||
        !aligned16(q_scales) || !aligned16(k_scales) || !aligned16(v_scales))
        return fail(HLTA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (B < 0 || H < 0 || T < 1 || N < 1) return fail(HLTA_ERR_INVALID_ARG, "bad shape B=%d H=%d T=%d N=%d", B, H, T, N);
    if ((long)T * N > (1L << 30)) return fail(HLTA_ERR_INVALID_ARG, "T*N too large");
    if (d != 128) return fail(HLTA_ERR_UNSUPPORTED, "FP8 attention supports d = 128 only (got %d)", d);
    if ((st = check_window(w, r)) != HLTA_OK) return st;
    DeviceCtx *ctx;
    if ((st = device_ctx(&ctx)) != HLTA_OK) return st;
    AttnArgs a = clip_attn_args(q8, k8, v8, o, B, H, 0, H, T, N, d, w, r, scale, ctx->err);
    a.qs = q_scales;
    a.ks = k_scales;
    a.vs = v_scales;
    if (B * H == 0) return HLTA_OK;
    cudaError_t e = launch_attn_fp8_tc2(a, (cudaStream_t)stream);
    if (e == cudaErrorNotSupported) return fail(HLTA_ERR_UNSUPPORTED, "FP8 window attention: unsupported shape");
    if (e != cudaSuccess) return cuda_fail(e, "FP8 window attention launch");
    return HLTA_OK;
}

hlta_status hlta_window_fwd_lse(const void *q, const void *k, const void *v, void *o,
                                float *lse, int B, int H, int T, int N, int d, int w, int r,
                                float scale, void *stream)
{
    hlta_status st;
    if (!lse || !aligned16(lse)) return fail(HLTA_ERR_INVALID_ARG, "lse must be a 16-byte aligned device pointer");
    if (!q || !k || !v || !o) return fail(HLTA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(HLTA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (B < 0 || H < 0 || T < 1 || N < 1) return fail(HLTA_ERR_INVALID_ARG, "bad shape B=%d H=%d T=%d N=%d", B, H, T, N);
    if ((long)T * N > (1L << 30)) return fail(HLTA_ERR_INVALID_ARG, "T*N too large");
    if (d != 128) return fail(HLTA_ERR_UNSUPPORTED, "training attention supports bf16, d = 128 only (got %d)", d);
    if ((st = check_window(w, r)) != HLTA_OK) return st;
    DeviceCtx *ctx;
    if ((st = device_ctx(&ctx)) != HLTA_OK) return st;
    AttnArgs a = clip_attn_args(q, k, v, o, B, H, 0, H, T, N, d, w, r, scale, ctx->err);
    a.lse = lse;
    return run_attn(a, HLTA_BF16, (cudaStream_t)stream);
}

size_t hlta_window_bwd_workspace_bytes(int B, int H, int T, int N)
{
    if (B < 0 || H < 0 || T < 0 || N < 0) return 0;
    return (((size_t)B * H * T * N * sizeof(float)) + 255) & ~(size_t)255;
}

hlta_status hlta_window_bwd(const void *q, const void *k, const void *v, const void *o,
                            const float *lse, const void *dO, void *dq, void *dk, void *dv,
                            int B, int H, int T, int N, int d, int w, int r, float scale,
                            void *workspace, size_t workspace_bytes, void *stream)
{
    hlta_status st;
    const void *ptrs[] = {q, k, v, o, lse, dO, dq, dk, dv, workspace};
    for (const void *p : ptrs) {
        if (!p) return fail(HLTA_ERR_INVALID_ARG, "null tensor pointer");
        if (!aligned16(p)) return fail(HLTA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    }
    if (B < 0 || H < 0 || T < 1 || N < 1) return fail(HLTA_ERR_INVALID_ARG, "bad shape B=%d H=%d T=%d N=%d", B, H, T, N);
    if ((long)T * N > (1L << 30)) return fail(HLTA_ERR_INVALID_ARG, "T*N too large");
    if (d != 128) return fail(HLTA_ERR_UNSUPPORTED, "attention backward supports bf16, d = 128 only (got %d)", d);
    if ((st = check_window(w, r)) != HLTA_OK) return st;
    if (workspace_bytes < hlta_window_bwd_workspace_bytes(B, H, T, N))
        return fail(HLTA_ERR_INVALID_ARG, "workspace too small (%zu < %zu bytes)", workspace_bytes,
                    hlta_window_bwd_workspace_bytes(B, H, T, N));
    if (B * H == 0) return HLTA_OK;
    AttnBwdArgs a;
    a.q = q; a.k = k; a.v = v; a.o = o; a.dO = dO; a.lse = lse;
    a.dq = dq; a.dk = dk; a.dv = dv;
    a.Dws = (float *)workspace;
    a.BH = B * H; a.T = T; a.N = N; a.w = w; a.r = r;
    a.scale = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
    cudaError_t e = launch_attn_bwd(a, (cudaStream_t)stream);
    if (e == cudaErrorNotSupported) return fail(HLTA_ERR_UNSUPPORTED, "attention backward: unsupported shape");
    if (e != cudaSuccess) return cuda_fail(e, "attention backward launch");
    return HLTA_OK;
}

hlta_status hlta_rope(void *q, void *k, int B, int H, int h0, int Hr, long L, int N, int d,
                      float base, int pos_mode, int inverse, hlta_dtype dt, void *stream)
{
    if (dt != HLTA_BF16 && dt != HLTA_FP32) return fail(HLTA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    if (B < 0 || H < 0 || L < 0 || N < 1) return fail(HLTA_ERR_INVALID_ARG, "bad shape B=%d H=%d L=%ld N=%d", B, H, L, N);
    if (d < 2 || d > 128 || d % 2) return fail(HLTA_ERR_INVALID_ARG, "d must be even, 2 <= d <= 128 (got %d)", d);
    if (h0 < 0 || Hr < 0 || h0 + Hr > H) return fail(HLTA_ERR_INVALID_ARG, "head range [%d, %d) outside [0, %d)", h0, h0 + Hr, H);
    if (!(base > 1.f) || !(base < 1e30f)) return fail(HLTA_ERR_INVALID_ARG, "base must be finite and > 1 (got %g)", (double)base);
    if (pos_mode != 0 && pos_mode != 1) return fail(HLTA_ERR_INVALID_ARG, "pos_mode must be 0 or 1 (got %d)", pos_mode);
    if ((q && !aligned16(q)) || (k && !aligned16(k)))
        return fail(HLTA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    cudaError_t e = launch_rope(q, k, dt == HLTA_BF16, B, H, h0, Hr, L, N, d, (double)base, pos_mode,
                                inverse ? -1 : 1, (cudaStream_t)stream);
    if (e == cudaErrorNotSupported) return fail(HLTA_ERR_UNSUPPORTED, "rotary embedding: shape too large");
    if (e != cudaSuccess) return cuda_fail(e, "rotary embedding launch");
    return HLTA_OK;
}

size_t hlta_gdn_bwd_workspace_bytes(int B, int H, long L, int d, int chunk)
{
    if (B < 0 || H < 0 || L < 0 || d != 128 || chunk != 64) return 0;
    return gdn_bwd_workspace_bytes((long)B * H, L);
}

hlta_status hlta_gdn_chunk_bwd(const void *q, const void *k, const void *v, const float *a,
                               const float *b, const float *S0, const void *dO,
                               const float *dS_final, void *dq, void *dk, void *dv, float *da,
                               float *db, float *dS0, int B, int H, long L, int d, int chunk,
                               void *workspace, size_t workspace_bytes, hlta_dtype dt,
                               void *stream)
{
    const void *req[] = {q, k, v, a, b, dO, dq, dk, dv, da, db, workspace};
    for (const void *p : req) {
        if (!p) return fail(HLTA_ERR_INVALID_ARG, "null tensor pointer");
        if (!aligned16(p)) return fail(HLTA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    }
    const void *opt[] = {S0, dS_final, dS0};
    for (const void *p : opt)
        if (p && !aligned16(p)) return fail(HLTA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (dt != HLTA_BF16 && dt != HLTA_FP32) return fail(HLTA_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    if (B < 0 || H < 0 || L < 0) return fail(HLTA_ERR_INVALID_ARG, "bad shape B=%d H=%d L=%ld", B, H, L);
    if (chunk != 64) return fail(HLTA_ERR_UNSUPPORTED, "chunk must be 64 (got %d)", chunk);
    if (d != 128) return fail(HLTA_ERR_UNSUPPORTED, "gated delta rule backward supports d = 128 only (got %d)", d);
    const size_t need = hlta_gdn_bwd_workspace_bytes(B, H, L, d, chunk);
    if (workspace_bytes < need)
        return fail(HLTA_ERR_INVALID_ARG, "workspace too small (%zu < %zu bytes)", workspace_bytes, need);
    DeviceCtx *ctx;
    hlta_status st;
    if ((st = device_ctx(&ctx)) != HLTA_OK) return st;
    GdnBwdArgs g;
    g.err = ctx->err;
    g.q = q; g.k = k; g.v = v; g.dO = dO; g.a = a; g.b = b; g.S0 = S0; g.dS_final = dS_final;
    g.dq = dq; g.dk = dk; g.dv = dv; g.da = da; g.db = db; g.dS0 = dS0;
    g.ws = workspace; g.B = B; g.H = H; g.d = d; g.L = L; g.bf16 = dt == HLTA_BF16;
    if ((long)B * H == 0 || L == 0) {
        // no tokens: the state gradient passes through unchanged
        if (dS0 && (long)B * H > 0) {
            cudaError_t e = dS_final ? cudaMemcpyAsync(dS0, dS_final, (size_t)B * H * d * d * sizeof(float), cudaMemcpyDeviceToDevice, (cudaStream_t)stream)
                                     : cudaMemsetAsync(dS0, 0, (size_t)B * H * d * d * sizeof(float), (cudaStream_t)stream);
            if (e != cudaSuccess) return cuda_fail(e, "dS0 copy");
        }
        return HLTA_OK;
    }
    // the bf16 path's two serial state passes run on the library's high-priority side
    // streams, beside the chunk preparation (the per-device events are shared: hold them
    // until the joins are enqueued)
    std::unique_lock<std::mutex> lk(g_fork_mu, std::defer_lock);
    SideStreams side = {ctx->aux, ctx->aux3, ctx->fork, ctx->mid, ctx->join, ctx->join2};
    if (g.bf16) lk.lock();
    cudaError_t e = launch_gdn_bwd(g, (cudaStream_t)stream, g.bf16 ? &side : nullptr);
    if (e == cudaErrorNotSupported) return fail(HLTA_ERR_UNSUPPORTED, "gated delta rule backward: unsupported shape");
    if (e != cudaSuccess) return cuda_fail(e, "gated delta rule backward launch");
    return HLTA_OK;
}

size_t hlta_gdn_workspace_bytes(int B, int H, long L, int d, int chunk, hlta_dtype dt)
{
    if (B < 0 || H < 0 || L < 0 || d < 1 || chunk != 64) return 0;
    return gdn_workspace_bytes((long)B * H, L, d, chunk, dt == HLTA_BF16);
}

namespace {
hlta_status gdn_fwd_impl(const void *q, const void *k, const void *v, const float *a,
                         const float *b, int raw, float raw_c, void *o, const float *S0,
                         float *S_out, int B, int H, long L, int d, int chunk, void *workspace,
                         size_t ws_bytes, hlta_dtype dt, void *stream)
{
    hlta_status st = check_gdn_common(q, k, v, a, b, o, S0, S_out, d, chunk, dt);
    if (st == HLTA_OK && raw) st = check_raw_c(raw_c);
    if (st != HLTA_OK) return st;
    if (B < 0 || H < 0 || L < 1 || L > (1L << 30)) return fail(HLTA_ERR_INVALID_ARG, "bad shape B=%d H=%d L=%ld", B, H, L);
    size_t need = gdn_workspace_bytes((long)B * H, L, d, chunk, dt == HLTA_BF16);
    if (!workspace || ws_bytes < need)
        return fail(HLTA_ERR_INVALID_ARG, "workspace too small: need %zu bytes, got %zu", need, ws_bytes);
    if (((uintptr_t)workspace & 255u) != 0) return fail(HLTA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    DeviceCtx *ctx;
    if ((st = device_ctx(&ctx)) != HLTA_OK) return st;
    GdnArgs g = {};
    g.q = q; g.k = k; g.v = v; g.a = a; g.b = b; g.o = o; g.raw = raw; g.raw_c = raw_c;
    g.B = B; g.Hg = H; g.Htot = H; g.h0 = 0; g.L = L; g.d = d; g.chunk = chunk;
    g.S0 = S0; g.S_out = S_out; g.ws = workspace; g.ws_bytes = ws_bytes; g.err = ctx->err;
    return run_gdn(g, dt, (cudaStream_t)stream);
}
}  // namespace

hlta_status hlta_gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *a,
                               const float *b, void *o, const float *S0, float *S_out, int B,
                               int H, long L, int d, int chunk, void *workspace,
                               size_t ws_bytes, hlta_dtype dt, void *stream)
{
    return gdn_fwd_impl(q, k, v, a, b, 0, 0.f, o, S0, S_out, B, H, L, d, chunk, workspace,
                        ws_bytes, dt, stream);
}

hlta_status hlta_gdn_chunk_fwd_raw(const void *q, const void *k, const void *v, const float *x,
                                   const float *y, float c, void *o, const float *S0,
                                   float *S_out, int B, int H, long L, int d, int chunk,
                                   void *workspace, size_t ws_bytes, hlta_dtype dt, void *stream)
{
    return gdn_fwd_impl(q, k, v, x, y, 1, c, o, S0, S_out, B, H, L, d, chunk, workspace,
                        ws_bytes, dt, stream);
}

size_t hlta_hybrid_workspace_bytes(int B, int Hg, int T, int N, int d, int chunk, hlta_dtype dt)
{
    if (B < 0 || Hg < 0 || T < 1 || N < 1 || d < 1 || chunk != 64) return 0;
    return gdn_workspace_bytes((long)B * Hg, (long)T * N, d, chunk, dt == HLTA_BF16);
}

namespace {
hlta_status hybrid_fwd_impl(const void *q, const void *k, const void *v, const float *a,
                            const float *b, int raw, float raw_c, void *o, const float *S0,
                            float *S_out, int B, int Hs, int Hd, int Hg, int T, int N, int d,
                            int w_swa, int w_dswa, int r, int chunk, float scale,
                            void *workspace, size_t ws_bytes, hlta_dtype dt, void *stream)
{
    hlta_status st;
    if (B < 0 || Hs < 0 || Hd < 0 || Hg < 0 || T < 1 || N < 1)
        return fail(HLTA_ERR_INVALID_ARG, "bad shape");
    if ((long)T * N > (1L << 30)) return fail(HLTA_ERR_INVALID_ARG, "T*N too large");
    const int H = Hs + Hd + Hg;
    if (!q || !k || !v || !o) return fail(HLTA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(HLTA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if ((st = check_dtype_d(dt, d)) != HLTA_OK) return st;
    if (Hs && (st = check_window(w_swa, 1)) != HLTA_OK) return st;
    if (Hd && (st = check_window(w_dswa, r)) != HLTA_OK) return st;
    const long L = (long)T * N;
    if (Hg) {
        if ((st = check_gdn_common(q, k, v, a, b, o, S0, S_out, d, chunk, dt)) != HLTA_OK) return st;
        if (raw && (st = check_raw_c(raw_c)) != HLTA_OK) return st;
        size_t need = gdn_workspace_bytes((long)B * Hg, L, d, chunk, dt == HLTA_BF16);
        if (!workspace || ws_bytes < need)
            return fail(HLTA_ERR_INVALID_ARG, "workspace too small: need %zu bytes, got %zu", need, ws_bytes);
        if (((uintptr_t)workspace & 255u) != 0) return fail(HLTA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    }
    DeviceCtx *ctx;
    if ((st = device_ctx(&ctx)) != HLTA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    std::lock_guard<std::mutex> lk(g_fork_mu);
    // the GDN branch runs on a library stream ordered after everything already on `s` (one
    // fork event), and `s` waits for it at the end; bf16 SWA and DSWA heads share one launch,
    // fp32 runs DSWA on a second library stream beside SWA
    const bool pair = Hd && Hs && dt == HLTA_BF16;
    const bool split_d = Hd && Hs && !pair;
    int reserve = 0;
    cudaStream_t s_fill = nullptr;  // bf16 with GDN heads: the attention's late CTAs follow the chain
    if (Hg || split_d) {
        if ((e = cudaEventRecord(ctx->fork, s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    }
    // GDN heads on the high-priority auxiliary stream
    if (Hg) {
        if ((e = cudaStreamWaitEvent(ctx->aux, ctx->fork, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
        GdnArgs g = {};
        g.q = q; g.k = k; g.v = v; g.a = a; g.b = b; g.o = o; g.raw = raw; g.raw_c = raw_c;
        g.B = B; g.Hg = Hg; g.Htot = H; g.h0 = Hs + Hd; g.L = L; g.d = d; g.chunk = chunk;
        g.S0 = S0; g.S_out = S_out; g.ws = workspace; g.ws_bytes = ws_bytes; g.err = ctx->err;
        // the GDN branch runs beside the softmax branches: its chain needs to end only within
        // their time, so it takes as few segments (and SMs) as that allows
        double pairs = 0.0;
        for (int f = 0; f < T; ++f) {
            for (int i = 0; i < w_swa && Hs; ++i) pairs += f - i >= 0 ? (double)Hs : 0.0;
            for (int i = 0; i < w_dswa && Hd; ++i) pairs += f - (long)r * i >= 0 ? (double)Hd : 0.0;
        }
        pairs *= (double)B * N * N;
        g.scan_segments = gdn_scan_segments_beside((long)B * Hg, gdn_num_chunks(L, chunk), 4.0 * d * pairs);
        // the chain's kernels take one SM per (head, segment) at most: the softmax launch
        // leaves those to it
        reserve = (int)std::min<long>((long)B * Hg * std::max(g.scan_segments, 1), 1L << 20);
        // the persistent attention launch holds its SMs to the end: it starts after the
        // preparation (which takes the whole GPU for a short time), beside the chain
        if (dt == HLTA_BF16) g.prep_done = ctx->prep;
        prof_record(3, ctx->aux);
        st = run_gdn(g, dt, ctx->aux);
        prof_record(4, ctx->aux);
        cudaEventRecord(ctx->join, ctx->aux);
        if (st != HLTA_OK) {
            cudaStreamWaitEvent(s, ctx->join, 0);   // `s` never runs ahead of enqueued work
            return st;
        }
        if (dt == HLTA_BF16 && (e = cudaStreamWaitEvent(s, ctx->prep, 0)) != cudaSuccess) {
            cudaStreamWaitEvent(s, ctx->join, 0);
            return cuda_fail(e, "cudaStreamWaitEvent");
        }
        if (dt == HLTA_BF16) s_fill = ctx->aux;
    }
    prof_record(0, s);      // the softmax branches start here (bf16: after the preparation)
    if (pair) {
        AttnArgs a1 = clip_attn_args(q, k, v, o, B, H, 0, Hs, T, N, d, w_swa, 1, scale, ctx->err);
        AttnArgs a2 = clip_attn_args(q, k, v, o, B, H, Hs, Hd, T, N, d, w_dswa, r, scale, ctx->err);
        st = run_attn_pair(a2, a1, dt, s, reserve, s_fill);
        prof_record(2, s_fill ? s_fill : s);        // after the late CTAs, if any
    }
    // DSWA on the second library stream (beside SWA) when both softmax branches are present
    if (Hd && !pair) {
        cudaStream_t sd = split_d ? ctx->aux2 : s;
        if (split_d && (e = cudaStreamWaitEvent(sd, ctx->fork, 0)) != cudaSuccess)
            st = cuda_fail(e, "cudaStreamWaitEvent");
        if (st == HLTA_OK) {
            AttnArgs a2 = clip_attn_args(q, k, v, o, B, H, Hs, Hd, T, N, d, w_dswa, r, scale, ctx->err);
            st = run_attn(a2, dt, sd, reserve, s_fill);
        }
        prof_record(2, sd);
        if (split_d) cudaEventRecord(ctx->join2, sd);
    }
    if (Hs && !pair && st == HLTA_OK) {
        AttnArgs a1 = clip_attn_args(q, k, v, o, B, H, 0, Hs, T, N, d, w_swa, 1, scale, ctx->err);
        st = run_attn(a1, dt, s, reserve, s_fill);
    }
    prof_record(1, s);
    // join: work enqueued on `s` after this call sees every branch's outputs (the GDN stream
    // also carries the attention's late CTAs)
    if (split_d) cudaStreamWaitEvent(s, ctx->join2, 0);
    if (s_fill) cudaEventRecord(ctx->join, ctx->aux);
    if (Hg) cudaStreamWaitEvent(s, ctx->join, 0);
    return st;
}
}  // namespace

hlta_status hlta_hybrid_fwd(const void *q, const void *k, const void *v, const float *a,
                            const float *b, void *o, const float *S0, float *S_out, int B,
                            int Hs, int Hd, int Hg, int T, int N, int d, int w_swa,
                            int w_dswa, int r, int chunk, float scale, void *workspace,
                            size_t ws_bytes, hlta_dtype dt, void *stream)
{
    return hybrid_fwd_impl(q, k, v, a, b, 0, 0.f, o, S0, S_out, B, Hs, Hd, Hg, T, N, d, w_swa,
                           w_dswa, r, chunk, scale, workspace, ws_bytes, dt, stream);
}

hlta_status hlta_hybrid_fwd_raw(const void *q, const void *k, const void *v, const float *x,
                                const float *y, float c, void *o, const float *S0, float *S_out,
                                int B, int Hs, int Hd, int Hg, int T, int N, int d, int w_swa,
                                int w_dswa, int r, int chunk, float scale, void *workspace,
                                size_t ws_bytes, hlta_dtype dt, void *stream)
{
    return hybrid_fwd_impl(q, k, v, x, y, 1, c, o, S0, S_out, B, Hs, Hd, Hg, T, N, d, w_swa,
                           w_dswa, r, chunk, scale, workspace, ws_bytes, dt, stream);
}

hlta_status hlta_stream_create(hlta_stream_t *out, int B, int Hs, int Hd, int Hg, int N, int d,
                               int w_swa, int w_dswa, int r, int chunk, float scale,
                               hlta_dtype dt, const float *S0)
{
    return hlta_stream_create_ex(out, B, Hs, Hd, Hg, N, d, w_swa, w_dswa, r, chunk, scale, 1, dt, S0);
}

hlta_status hlta_stream_create_ex(hlta_stream_t *out, int B, int Hs, int Hd, int Hg, int N, int d,
                                  int w_swa, int w_dswa, int r, int chunk, float scale,
                                  int max_step_frames, hlta_dtype dt, const float *S0)
{
    hlta_status st;
    if (!out) return fail(HLTA_ERR_INVALID_ARG, "null output handle");
    *out = nullptr;
    if (B < 1 || Hs < 0 || Hd < 0 || Hg < 0 || N < 1) return fail(HLTA_ERR_INVALID_ARG, "bad shape");
    if (max_step_frames < 1 || max_step_frames > 4096 || (long)max_step_frames * N > (1L << 30))
        return fail(HLTA_ERR_INVALID_ARG, "max_step_frames must be in [1, 4096] (got %d)", max_step_frames);
    if ((st = check_dtype_d(dt, d)) != HLTA_OK) return st;
    if (Hs && (st = check_window(w_swa, 1)) != HLTA_OK) return st;
    if (Hd && (st = check_window(w_dswa, r)) != HLTA_OK) return st;
    if (Hg && chunk != 64) return fail(HLTA_ERR_UNSUPPORTED, "chunk must be 64");
    if (S0 && !aligned16(S0)) return fail(HLTA_ERR_INVALID_ARG, "S0 must be 16-byte aligned");
    DeviceCtx *ctx;   // the device helpers (library streams, events) exist before any capture
    if ((st = device_ctx(&ctx)) != HLTA_OK) return st;
    hlta_stream *c = new (std::nothrow) hlta_stream();
    if (!c) return fail(HLTA_ERR_CUDA, "host allocation failed");
    cudaGetDevice(&c->device);
    c->B = B; c->Hs = Hs; c->Hd = Hd; c->Hg = Hg; c->N = N; c->d = d;
    c->w_swa = w_swa; c->w_dswa = w_dswa; c->r = r; c->chunk = chunk; c->dt = dt;
    c->scale = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
    c->max_frames = max_step_frames;
    c->slots_s = Hs ? w_swa - 1 + max_step_frames : 0;
    c->slots_d = Hd ? r * (w_dswa - 1) + max_step_frames : 0;
    const size_t el = dt == HLTA_BF16 ? 2 : 4;
    const size_t frame = (size_t)N * d * el;
    size_t bs = (size_t)B * Hs * c->slots_s * frame, bd = (size_t)B * Hd * c->slots_d * frame;
    c->ws_bytes = Hg ? gdn_workspace_bytes((long)B * Hg, (long)max_step_frames * N, d, chunk, dt == HLTA_BF16) : 0;
    cudaError_t e = cudaSuccess;
    if (bs && e == cudaSuccess) e = cudaMalloc(&c->ks, bs);
    if (bs && e == cudaSuccess) e = cudaMalloc(&c->vs, bs);
    if (bd && e == cudaSuccess) e = cudaMalloc(&c->kd, bd);
    if (bd && e == cudaSuccess) e = cudaMalloc(&c->vd, bd);
    if (Hg && e == cudaSuccess) e = cudaMalloc((void **)&c->S, (size_t)B * Hg * d * d * sizeof(float));
    if (Hg && e == cudaSuccess) e = cudaMalloc(&c->ws, c->ws_bytes);
    if (e == cudaSuccess) e = cudaMalloc((void **)&c->fdev, 4 * sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(c->fdev, 0, 4 * sizeof(int));
    if (e == cudaSuccess && Hg) {
        if (S0) e = cudaMemcpy(c->S, S0, (size_t)B * Hg * d * d * sizeof(float), cudaMemcpyDeviceToDevice);
        else e = cudaMemset(c->S, 0, (size_t)B * Hg * d * d * sizeof(float));
    }
    if (e != cudaSuccess) {
        hlta_stream_destroy(c);
        return cuda_fail(e, "stream cache allocation");
    }
    c->frames = 0;
    *out = c;
    return HLTA_OK;
}

hlta_status hlta_stream_step(hlta_stream_t c, const void *q_new, const void *k_new,
                             const void *v_new, const float *a_new, const float *b_new,
                             void *o_new, void *stream)
{
    return hlta_stream_step_frames(c, q_new, k_new, v_new, a_new, b_new, o_new, 1, stream);
}

hlta_status hlta_stream_step_frames(hlta_stream_t c, const void *q_new, const void *k_new,
                                    const void *v_new, const float *a_new, const float *b_new,
                                    void *o_new, int F, void *stream)
{
    if (!c) return fail(HLTA_ERR_INVALID_ARG, "null cache");
    if (F < 1 || F > c->max_frames)
        return fail(HLTA_ERR_INVALID_ARG, "frames per step must be in [1, %d] (got %d)", c->max_frames, F);
    if (!q_new || !k_new || !v_new || !o_new) return fail(HLTA_ERR_INVALID_ARG, "null tensor pointer");
    if (c->Hg && (!a_new || !b_new)) return fail(HLTA_ERR_INVALID_ARG, "null gate pointer");
    if (!aligned16(q_new) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(o_new) ||
        (c->Hg && (!aligned16(a_new) || !aligned16(b_new))))
        return fail(HLTA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    int dev = -1;
    cudaGetDevice(&dev);
    if (dev != c->device) return fail(HLTA_ERR_INVALID_ARG, "cache lives on device %d, current device is %d", c->device, dev);
    hlta_status st;
    DeviceCtx *ctx;
    if ((st = device_ctx(&ctx)) != HLTA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    const int H = c->Hs + c->Hd + c->Hg;
    const int f = c->frames;
    const size_t el = c->dt == HLTA_BF16 ? 2 : 4;
    // the fork/join events are shared per device: hold them until the joins are enqueued.
    // GDN runs on the high-priority library stream; bf16 SWA and DSWA heads share one
    // attention launch on `s`, fp32 runs the DSWA branch (ring append and attention) on the
    // second library stream when SWA heads are present too
    std::unique_lock<std::mutex> lk(g_fork_mu, std::defer_lock);
    const bool pair = c->Hd && c->Hs && c->dt == HLTA_BF16;
    const bool split_d = c->Hd && c->Hs && !pair;
    int reserve = 0;
    cudaStream_t s_fill = nullptr;  // bf16 with GDN heads: the attention's late CTAs follow the chain
    lk.lock();
    if (c->Hg || split_d) {
        if ((e = cudaEventRecord(ctx->fork, s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    }
    if (c->Hg) {
        if ((e = cudaStreamWaitEvent(ctx->aux, ctx->fork, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
        prof_record(3, ctx->aux);
        GdnArgs g = {};
        g.q = q_new; g.k = k_new; g.v = v_new; g.a = a_new; g.b = b_new; g.o = o_new;
        g.B = c->B; g.Hg = c->Hg; g.Htot = H; g.h0 = c->Hs + c->Hd; g.L = (long)F * c->N; g.d = c->d;
        g.chunk = c->chunk; g.S0 = c->S; g.S_out = c->S; g.ws = c->ws; g.ws_bytes = c->ws_bytes;
        g.err = ctx->err;
        // the chain takes one SM per (head, segment): the softmax launch leaves those to it
        const long nch = gdn_num_chunks(g.L, g.chunk), BHg = (long)c->B * c->Hg;
        const long seg = gdn_scan_segment_len(BHg, nch);
        reserve = (int)std::min<long>(BHg * ((nch + seg - 1) / seg), 1L << 20);
        // the persistent attention launch starts after the preparation, beside the chain
        if (c->dt == HLTA_BF16) g.prep_done = ctx->prep;
        st = run_gdn(g, c->dt, ctx->aux);
        prof_record(4, ctx->aux);
        cudaEventRecord(ctx->join, ctx->aux);
        if (st != HLTA_OK) {
            cudaStreamWaitEvent(s, ctx->join, 0);
            return st;
        }
        if (c->dt == HLTA_BF16) s_fill = ctx->aux;
    }
    // the ring appends run beside the preparation; the attention waits for it (bf16 with GDN
    // heads). events[0] marks where the attention starts.
    bool started = false;
    auto attn_start = [&](cudaStream_t sa) -> hlta_status {
        if (started) return HLTA_OK;
        started = true;
        if (s_fill) {
            cudaError_t e2 = cudaStreamWaitEvent(sa, ctx->prep, 0);
            if (e2 != cudaSuccess) return cuda_fail(e2, "cudaStreamWaitEvent");
        }
        prof_record(0, sa);
        return HLTA_OK;
    };
    struct Branch { int h0, Hbr, slots, w, r; void *rk, *rv; } br[2] = {
        {0, c->Hs, c->slots_s, c->w_swa, 1, c->ks, c->vs},
        {c->Hs, c->Hd, c->slots_d, c->w_dswa, c->r, c->kd, c->vd}};
    if (split_d && (e = cudaStreamWaitEvent(ctx->aux2, ctx->fork, 0)) != cudaSuccess) {
        cudaStreamWaitEvent(s, ctx->join, 0);
        return cuda_fail(e, "cudaStreamWaitEvent");
    }
    AttnArgs pa[2];
    for (int bi = 1; bi >= 0; --bi) {                  // DSWA first: it goes to its own stream
        const Branch &x = br[bi];
        if (!x.Hbr) continue;
        cudaStream_t s = (bi == 1 && split_d) ? ctx->aux2 : (cudaStream_t)stream;
        if ((e = launch_ring_append(k_new, c->B, H, x.h0, x.Hbr, c->N, c->d, el, F, x.rk, x.slots, f, c->fdev, s)) != cudaSuccess ||
            (e = launch_ring_append(v_new, c->B, H, x.h0, x.Hbr, c->N, c->d, el, F, x.rv, x.slots, f, c->fdev, s)) != cudaSuccess) {
            st = cuda_fail(e, "ring append");
            break;
        }
        AttnArgs a;
        a.q = q_new; a.k = x.rk; a.v = x.rv; a.o = o_new;
        a.B = c->B; a.Hbr = x.Hbr;
        a.q_Htot = H; a.q_h0 = x.h0; a.q_rows = (long)F * c->N;
        a.kv_Htot = x.Hbr; a.kv_h0 = 0; a.kv_rows = (long)x.slots * c->N; a.kv_slots = x.slots;
        a.N = c->N; a.d = c->d; a.w = x.w; a.r = x.r; a.fq0 = f; a.fq0_dev = c->fdev; a.scale = c->scale;
        a.err = ctx->err;
        a.sched = c->fdev + 2;
        if (pair) {
            pa[1 - bi] = a;                            // launched below, DSWA's units first
            continue;
        }
        if ((st = attn_start(s)) != HLTA_OK || (st = run_attn(a, c->dt, s, reserve, s_fill)) != HLTA_OK) break;
        prof_record(bi == 1 ? 2 : 1, s);
    }
    if (pair && st == HLTA_OK && (st = attn_start((cudaStream_t)stream)) == HLTA_OK) {
        st = run_attn_pair(pa[0], pa[1], c->dt, (cudaStream_t)stream, reserve, s_fill);
        prof_record(2, s_fill ? s_fill : (cudaStream_t)stream);     // after the late CTAs, if any
        prof_record(1, (cudaStream_t)stream);
    }
    // join the other branches after the softmax launches were enqueued, so they overlap
    if (split_d) {
        cudaEventRecord(ctx->join2, ctx->aux2);
        cudaStreamWaitEvent(s, ctx->join2, 0);
    }
    if (s_fill) cudaEventRecord(ctx->join, ctx->aux);
    if (c->Hg) cudaStreamWaitEvent(s, ctx->join, 0);
    if (st != HLTA_OK) return st;
    if ((e = launch_frame_advance(c->fdev, F, s)) != cudaSuccess) return cuda_fail(e, "frame counter");
    c->frames = f + F;
    return HLTA_OK;
}

hlta_status hlta_stream_frame_counter(hlta_stream_t c, int **f_dev)
{
    if (!c || !f_dev) return fail(HLTA_ERR_INVALID_ARG, "null argument");
    *f_dev = c->fdev;
    return HLTA_OK;
}

hlta_status hlta_stream_state(hlta_stream_t c, float **S_dev, int *frames_done)
{
    if (!c) return fail(HLTA_ERR_INVALID_ARG, "null cache");
    if (S_dev) *S_dev = c->S;
    if (frames_done) *frames_done = c->frames;
    return HLTA_OK;
}

}  // extern "C"

namespace {
// the checkpoint image's header: 64 bytes, then the state and the four rings
struct CkptHeader {
    char magic[4];
    int32_t version;
    int32_t B, Hs, Hd, Hg, N, d, w_swa, w_dswa, r, chunk, dt, max_frames;
    int32_t frames;
    float scale;
};
static_assert(sizeof(CkptHeader) == 64, "checkpoint header is 64 bytes");
constexpr char CKPT_MAGIC[4] = {'H', 'L', 'T', 'C'};

struct CkptPart { void *p; size_t bytes; };

// the device buffers of a cache in image order (absent branches have 0 bytes)
void ckpt_parts(const hlta_stream *c, CkptPart (&parts)[5])
{
    const size_t el = c->dt == HLTA_BF16 ? 2 : 4;
    const size_t frame = (size_t)c->N * c->d * el;
    const size_t bs = (size_t)c->B * c->Hs * c->slots_s * frame, bd = (size_t)c->B * c->Hd * c->slots_d * frame;
    parts[0] = {c->S, c->Hg ? (size_t)c->B * c->Hg * c->d * c->d * sizeof(float) : 0};
    parts[1] = {c->ks, bs};
    parts[2] = {c->vs, bs};
    parts[3] = {c->kd, bd};
    parts[4] = {c->vd, bd};
}

CkptHeader ckpt_header(const hlta_stream *c, int frames)
{
    CkptHeader h;
    memcpy(h.magic, CKPT_MAGIC, 4);
    h.version = 1;
    h.B = c->B; h.Hs = c->Hs; h.Hd = c->Hd; h.Hg = c->Hg; h.N = c->N; h.d = c->d;
    h.w_swa = c->w_swa; h.w_dswa = c->w_dswa; h.r = c->r; h.chunk = c->chunk; h.dt = (int32_t)c->dt;
    h.max_frames = c->max_frames; h.frames = frames; h.scale = c->scale;
    return h;
}

hlta_status ckpt_device(const hlta_stream *c)
{
    int dev = -1;
    cudaGetDevice(&dev);
    if (dev != c->device) return fail(HLTA_ERR_INVALID_ARG, "cache lives on device %d, current device is %d", c->device, dev);
    return HLTA_OK;
}
}  // namespace

extern "C" {

size_t hlta_stream_checkpoint_bytes(hlta_stream_t c)
{
    if (!c) return 0;
    CkptPart parts[5];
    ckpt_parts(c, parts);
    size_t n = sizeof(CkptHeader);
    for (const CkptPart &pt : parts) n += pt.bytes;
    return n;
}

hlta_status hlta_stream_save(hlta_stream_t c, void *dst, size_t bytes, void *stream)
{
    if (!c || !dst) return fail(HLTA_ERR_INVALID_ARG, "null argument");
    const size_t need = hlta_stream_checkpoint_bytes(c);
    if (bytes < need) return fail(HLTA_ERR_INVALID_ARG, "checkpoint buffer too small: need %zu bytes, got %zu", need, bytes);
    hlta_status st;
    if ((st = ckpt_device(c)) != HLTA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    int frames = 0;
    cudaError_t e = cudaMemcpyAsync(&frames, c->fdev, sizeof(int), cudaMemcpyDeviceToHost, s);
    CkptPart parts[5];
    ckpt_parts(c, parts);
    size_t off = sizeof(CkptHeader);
    for (const CkptPart &pt : parts) {
        if (e == cudaSuccess && pt.bytes) e = cudaMemcpyAsync((char *)dst + off, pt.p, pt.bytes, cudaMemcpyDeviceToHost, s);
        off += pt.bytes;
    }
    const cudaError_t es = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = es;
    if (e != cudaSuccess) return cuda_fail(e, "checkpoint copy");
    const CkptHeader h = ckpt_header(c, frames);
    memcpy(dst, &h, sizeof h);
    return HLTA_OK;
}

hlta_status hlta_stream_load(hlta_stream_t c, const void *src, size_t bytes, void *stream)
{
    if (!c || !src) return fail(HLTA_ERR_INVALID_ARG, "null argument");
    const size_t need = hlta_stream_checkpoint_bytes(c);
    if (bytes != need) return fail(HLTA_ERR_INVALID_ARG, "checkpoint size %zu does not match this cache's %zu bytes", bytes, need);
    CkptHeader h;
    memcpy(&h, src, sizeof h);
    if (memcmp(h.magic, CKPT_MAGIC, 4) != 0 || h.version != 1)
        return fail(HLTA_ERR_INVALID_ARG, "not a streaming-cache checkpoint (magic or version)");
    const CkptHeader mine = ckpt_header(c, h.frames);
    if (memcmp(&h, &mine, sizeof h) != 0 || h.frames < 0)
        return fail(HLTA_ERR_INVALID_ARG, "checkpoint of a cache created with other arguments");
    hlta_status st;
    if ((st = ckpt_device(c)) != HLTA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const int frames = h.frames;
    cudaError_t e = cudaMemcpyAsync(c->fdev, &frames, sizeof(int), cudaMemcpyHostToDevice, s);
    CkptPart parts[5];
    ckpt_parts(c, parts);
    size_t off = sizeof(CkptHeader);
    for (const CkptPart &pt : parts) {
        if (e == cudaSuccess && pt.bytes) e = cudaMemcpyAsync(pt.p, (const char *)src + off, pt.bytes, cudaMemcpyHostToDevice, s);
        off += pt.bytes;
    }
    const cudaError_t es = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = es;
    if (e != cudaSuccess) return cuda_fail(e, "checkpoint copy");
    c->frames = frames;
    return HLTA_OK;
}

hlta_status hlta_stream_destroy(hlta_stream_t c)
{
    if (!c) return HLTA_OK;
    int prev = -1;
    cudaGetDevice(&prev);
    cudaSetDevice(c->device);
    cudaDeviceSynchronize();
    void *bufs[] = {c->ks, c->vs, c->kd, c->vd, c->S, c->ws, c->fdev};
    for (void *p : bufs)
        if (p) cudaFree(p);
    if (prev >= 0) cudaSetDevice(prev);
    delete c;
    return HLTA_OK;
}

hlta_status hlta_set_profile_events(void *const *events)
{
    std::lock_guard<std::mutex> lk(g_fork_mu);
    g_prof_on = events != nullptr;
    for (int i = 0; i < 5; ++i) g_prof[i] = events ? (cudaEvent_t)events[i] : nullptr;
    return HLTA_OK;
}

unsigned long long hlta_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

hlta_status hlta_wait_expiry_selftest(unsigned long long cycles, void *stream)
{
    if (cycles < 1 || cycles > (1ull << 32))
        return fail(HLTA_ERR_INVALID_ARG, "cycles must be in [1, 2^32] (got %llu)", cycles);
    hlta_status st;
    DeviceCtx *ctx;
    if ((st = device_ctx(&ctx)) != HLTA_OK) return st;
    cudaError_t e = launch_wait_selftest(ctx->err, (long long)cycles, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "wait self-test launch");
    return HLTA_OK;
}

hlta_status hlta_device_status(void *stream, unsigned int *code)
{
    hlta_status st;
    DeviceCtx *ctx;
    if ((st = device_ctx(&ctx)) != HLTA_OK) return st;
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int word = 0, zero = 0;
    if ((e = cudaMemcpy(&word, ctx->err, sizeof word, cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "read device error word");
    if ((e = cudaMemcpy(ctx->err, &zero, sizeof zero, cudaMemcpyHostToDevice)) != cudaSuccess)
        return cuda_fail(e, "clear device error word");
    if (code) *code = word;
    if (word) return fail(HLTA_ERR_TIMEOUT, "a kernel's bounded wait expired (device error word 0x%x)", word);
    return HLTA_OK;
}

}  // extern "C"
