// Windowed softmax attention (SWA / DSWA / streaming step), fp32 in, fp32 out, fp32
// arithmetic on the CUDA cores. This is the HLTA_FP32 element type's path: it keeps full
// single precision (no tensor-core operand rounding), which the fp32 workloads need.
//
// Online (running-max) softmax over 32-key tiles, exact up to fp32 rounding (llm-atlas
// long-context explainer, section 03: tiled exact attention with a running normaliser
// reaches the same result as the full softmax).
#include "hlta_internal.cuh"

#include <math.h>

namespace hlta {
namespace {

constexpr int QB = 16;   // query rows per block
constexpr int KT = 32;   // keys per tile
constexpr int THREADS = 128;

__device__ __forceinline__ bool is_tap(int fq, int fk, int w, int r)
{
    int dist = fq - fk;
    return dist >= 0 && dist <= r * (w - 1) && (dist % r) == 0;
}

__device__ __forceinline__ float warp_max(float x)
{
    for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x)
{
    for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__global__ void __launch_bounds__(THREADS) attn_f32_kernel(AttnArgs p)
{
    extern __shared__ float smem[];
    const int d = p.d;
    const int dp = d + 1;
    float *Qs = smem;                    // [QB][d]
    float *Ks = Qs + QB * d;             // [KT][d+1]
    float *Vs = Ks + KT * dp;            // [KT][d]

    const int bh = blockIdx.y;
    const int b = bh / p.Hbr, h = bh % p.Hbr;
    const long l0 = (long)blockIdx.x * QB;
    const float *q = (const float *)p.q + ((long)(b * p.q_Htot + p.q_h0 + h) * p.q_rows) * d;
    float *o = (float *)p.o + ((long)(b * p.q_Htot + p.q_h0 + h) * p.q_rows) * d;
    const float *kb = (const float *)p.k + ((long)(b * p.kv_Htot + p.kv_h0 + h) * p.kv_rows) * d;
    const float *vb = (const float *)p.v + ((long)(b * p.kv_Htot + p.kv_h0 + h) * p.kv_rows) * d;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long nrows = min((long)QB, p.q_rows - l0);
    for (int e = tid; e < QB * d; e += THREADS) {
        int rr = e / d, c = e % d;
        Qs[e] = rr < nrows ? q[(l0 + rr) * d + c] : 0.f;
    }

    const int fq0 = p.fq0_dev ? *p.fq0_dev : p.fq0;
    const int fa = fq0 + (int)(l0 / p.N);
    const int fb = fq0 + (int)((l0 + nrows - 1) / p.N);
    const int span = p.r * (p.w - 1);

    // per warp: rows warp*4 .. warp*4+3; per row running max m, sum l, output dims per lane
    float m[4], l[4], acc[4][4];
    int fq[4];
    bool valid[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int rr = warp * 4 + i;
        valid[i] = rr < nrows;
        fq[i] = fq0 + (int)((l0 + rr) / p.N);
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    }

    for (int fk = max(0, fa - span); fk <= fb; ++fk) {
        bool needed = false;
        for (int f = fa; f <= fb && !needed; ++f) needed = is_tap(f, fk, p.w, p.r);
        if (!needed) continue;
        const long krow0 = (long)(fk % p.kv_slots) * p.N;
        for (int n0 = 0; n0 < p.N; n0 += KT) {
            __syncthreads();
            for (int e = tid; e < KT * d; e += THREADS) {
                int j = e / d, c = e % d;
                bool ok = n0 + j < p.N;
                Ks[j * dp + c] = ok ? kb[(krow0 + n0 + j) * d + c] : 0.f;
                Vs[j * d + c] = ok ? vb[(krow0 + n0 + j) * d + c] : 0.f;
            }
            __syncthreads();
            const bool key_ok = n0 + lane < p.N;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (!valid[i] || !is_tap(fq[i], fk, p.w, p.r)) continue;
                const float *qr = Qs + (warp * 4 + i) * d;
                float s = 0.f;
                for (int c = 0; c < d; ++c) s = fmaf(qr[c], Ks[lane * dp + c], s);
                s = key_ok ? s * p.scale : -INFINITY;
                float mt = warp_max(s);
                float mn = fmaxf(m[i], mt);
                float alpha = expf(m[i] - mn);   // m = -inf on the first tile: alpha = 0
                float pj = key_ok ? expf(s - mn) : 0.f;
                l[i] = l[i] * alpha + warp_sum(pj);
                m[i] = mn;
#pragma unroll
                for (int jd = 0; jd < 4; ++jd) acc[i][jd] *= alpha;
                for (int j = 0; j < KT; ++j) {
                    float pb = __shfl_sync(0xffffffffu, pj, j);
#pragma unroll
                    for (int jd = 0; jd < 4; ++jd) {
                        int c = lane + 32 * jd;
                        if (c < d) acc[i][jd] = fmaf(pb, Vs[j * d + c], acc[i][jd]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (!valid[i]) continue;
        long row = l0 + warp * 4 + i;
        float inv = 1.f / l[i];
#pragma unroll
        for (int jd = 0; jd < 4; ++jd) {
            int c = lane + 32 * jd;
            if (c < d) o[row * d + c] = acc[i][jd] * inv;
        }
    }
}

}  // namespace

cudaError_t launch_attn_f32(const AttnArgs &a, cudaStream_t s)
{
    size_t smem = sizeof(float) * ((size_t)QB * a.d + (size_t)KT * (a.d + 1) + (size_t)KT * a.d);
    // d <= 128: at most 41 KB, inside the default dynamic shared memory limit
    dim3 grid((unsigned)((a.q_rows + QB - 1) / QB), (unsigned)(a.B * a.Hbr));
    attn_f32_kernel<<<grid, THREADS, smem, s>>>(a), note_launch();
    return cudaGetLastError();
}

}  // namespace hlta
