// Gated delta rule, chunkwise form, fp32 in / fp32 out, fp32 arithmetic on the CUDA cores
// (the HLTA_FP32 element type's path). Same two-kernel structure as the bf16 path:
//
//   prep  (parallel over every chunk of every head): the UT transform of the chunk and the
//         products that do not depend on the incoming state;
//   state (serial over the chunks of a head, parallel over row blocks of the state):
//         passes the state from chunk to chunk and writes the outputs.
//
// Chunk algebra (derived from S_t = a_t S_{t-1}(I - b_t k_t k_t^T) + b_t v_t k_t^T; the
// chunkwise split itself is the "parallel within a block, recurrent across blocks" form of
// the llm-atlas long-context explainer, sections 06 and 09). For a chunk of n tokens with
// incoming state S0 and g_t = sum_{s<=t} log a_s (within the chunk):
//   A_ti = b_t e^{g_t-g_i} k_t.k_i (i < t),  T = (I + A)^{-1}
//   W  = T diag(b e^g) K,  Up = T diag(b) V,  P_ti = e^{g_t-g_i} q_t.k_i (i <= t)
//   Op = P Up,  Qt = diag(e^g) Q - P W,  Kt = diag(e^{g_n - g}) K,  gam = e^{g_n}
// and then, with the state:
//   U = Up - W S0^T,  O = Op + Qt S0^T,  S_n = gam S0 + U^T Kt.
// Only decays e^{g_t - g_i} with t >= i (exponent <= 0) are ever formed.
#include "hlta_internal.cuh"

#include <math.h>

namespace hlta {
namespace {

constexpr int C = 64;          // chunk length
constexpr int PREP_THREADS = 256;
constexpr int STATE_THREADS = 256;
constexpr int R = 16;          // state rows per block in the state pass

__global__ void __launch_bounds__(PREP_THREADS) gdn_prep_f32(GdnArgs p, GdnWorkspace ws)
{
    extern __shared__ float sm[];
    const int d = p.d, dp = d + 1, cp = C + 1;
    float *Qc = sm;                 // [C][d+1]
    float *Kc = Qc + C * dp;        // [C][d+1]
    float *VW = Kc + C * dp;        // [C][d+1]  V, later W
    float *Uc = VW + C * dp;        // [C][d+1]  Up
    float *Am = Uc + C * dp;        // [C][C+1]  A
    float *Tm = Am + C * cp;        // [C][C+1]  T
    float *Pm = Tm + C * cp;        // [C][C+1]  P
    float *g = Pm + C * cp;         // [C]
    float *bb = g + C;              // [C]

    const int chunk = blockIdx.x, bh = blockIdx.y;
    const int b = bh / p.Hg, h = bh % p.Hg;
    const long nch = gdn_num_chunks(p.L, C);
    const long t0 = (long)chunk * C;
    const int n = (int)min((long)C, p.L - t0);
    const long head = (long)(b * p.Htot + p.h0 + h) * p.L;
    const float *q = (const float *)p.q + (head + t0) * d;
    const float *k = (const float *)p.k + (head + t0) * d;
    const float *v = (const float *)p.v + (head + t0) * d;
    const float *ag = p.a + (long)bh * p.L + t0;
    const float *bg = p.b + (long)bh * p.L + t0;
    const int tid = threadIdx.x;

    for (int e = tid; e < C * d; e += PREP_THREADS) {
        int t = e / d, c = e % d;
        bool ok = t < n;
        Qc[t * dp + c] = ok ? q[(long)t * d + c] : 0.f;
        Kc[t * dp + c] = ok ? k[(long)t * d + c] : 0.f;
        VW[t * dp + c] = ok ? v[(long)t * d + c] : 0.f;
    }
    if (tid == 0) {
        // log of the decay gate: log a, or with raw inputs -c softplus(x); the write
        // strength b, or sigmoid(y)
        float acc = 0.f;
        for (int t = 0; t < C; ++t) {
            if (t < n) acc += p.raw ? -p.raw_c * (ag[t] > 20.f ? ag[t] : log1pf(expf(ag[t]))) : logf(ag[t]);
            g[t] = acc;
            bb[t] = t < n ? (p.raw ? 1.f / (1.f + expf(-bg[t])) : bg[t]) : 0.f;
        }
    }
    __syncthreads();
    // raw inputs: q and k of every token scaled to unit L2 norm (rows of zeros stay zero)
    if (p.raw) {
        if (tid < 2 * C) {
            float *row = (tid < C ? Qc : Kc) + (tid & (C - 1)) * dp;
            float ss = 0.f;
            for (int c = 0; c < d; ++c) ss = fmaf(row[c], row[c], ss);
            const float sc = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
            for (int c = 0; c < d; ++c) row[c] *= sc;
        }
        __syncthreads();
    }

    // A (strictly lower) and P (lower, diagonal included)
    for (int e = tid; e < C * C; e += PREP_THREADS) {
        int t = e / C, i = e % C;
        float kk = 0.f, qk = 0.f;
        if (i <= t && t < n) {
            for (int c = 0; c < d; ++c) {
                kk = fmaf(Kc[t * dp + c], Kc[i * dp + c], kk);
                qk = fmaf(Qc[t * dp + c], Kc[i * dp + c], qk);
            }
        }
        float dec = (i <= t && t < n) ? expf(g[t] - g[i]) : 0.f;
        Am[t * cp + i] = i < t ? bb[t] * dec * kk : 0.f;
        Pm[t * cp + i] = dec * qk;
    }
    __syncthreads();

    // T = (I + A)^{-1}: column j by forward substitution (one thread per column)
    if (tid < C) {
        const int j = tid;
        for (int t = 0; t < C; ++t) Tm[t * cp + j] = t == j ? 1.f : 0.f;
        for (int t = j + 1; t < C; ++t) {
            float s = 0.f;
            for (int i = j; i < t; ++i) s = fmaf(Am[t * cp + i], Tm[i * cp + j], s);
            Tm[t * cp + j] = -s;
        }
    }
    __syncthreads();

    // Up = T diag(b) V ; rows t >= n are zero because b is zero there and T is unit lower
    for (int e = tid; e < C * d; e += PREP_THREADS) {
        int t = e / d, c = e % d;
        float s = 0.f;
        for (int i = 0; i <= t; ++i) s = fmaf(Tm[t * cp + i] * bb[i], VW[i * dp + c], s);
        Uc[t * dp + c] = t < n ? s : 0.f;
    }
    __syncthreads();
    // W = T diag(b e^g) K, written over V
    for (int e = tid; e < C * d; e += PREP_THREADS) {
        int t = e / d, c = e % d;
        float s = 0.f;
        for (int i = 0; i <= t; ++i)
            s = fmaf(Tm[t * cp + i] * bb[i] * expf(g[i]), Kc[i * dp + c], s);
        VW[t * dp + c] = t < n ? s : 0.f;
    }
    __syncthreads();

    const long base = ((long)bh * nch + chunk) * C * d;
    float *Wo = (float *)ws.W + base, *Uo = (float *)ws.Up + base, *Oo = (float *)ws.Op + base;
    float *Qo = (float *)ws.Qt + base, *Ko = (float *)ws.Kt + base;
    const float gn = g[n - 1];
    for (int e = tid; e < C * d; e += PREP_THREADS) {
        int t = e / d, c = e % d;
        float op = 0.f, pw = 0.f;
        for (int i = 0; i <= t; ++i) {
            op = fmaf(Pm[t * cp + i], Uc[i * dp + c], op);
            pw = fmaf(Pm[t * cp + i], VW[i * dp + c], pw);
        }
        bool ok = t < n;
        Wo[e] = VW[t * dp + c];
        Uo[e] = Uc[t * dp + c];
        Oo[e] = ok ? op : 0.f;
        Qo[e] = ok ? expf(g[t]) * Qc[t * dp + c] - pw : 0.f;
        Ko[e] = ok ? expf(gn - g[t]) * Kc[t * dp + c] : 0.f;
    }
    if (tid == 0) ws.gam[((long)bh * nch + chunk) * 4] = expf(gn);
}

__global__ void __launch_bounds__(STATE_THREADS) gdn_state_f32(GdnArgs p, GdnWorkspace ws)
{
    extern __shared__ float sm[];
    const int d = p.d, dp = d + 1;
    float *S = sm;                  // [R][d+1]
    float *Wc = S + R * dp;         // [C][d]
    float *Qt = Wc + C * d;         // [C][d]
    float *Kt = Qt + C * d;         // [C][d]
    float *Uc = Kt + C * d;         // [C][R]
    const int i0 = blockIdx.x * R, bh = blockIdx.y;
    const int b = bh / p.Hg, h = bh % p.Hg;
    const long nch = gdn_num_chunks(p.L, C);
    const int tid = threadIdx.x;
    float *o = (float *)p.o + (long)(b * p.Htot + p.h0 + h) * p.L * d;

    for (int e = tid; e < R * d; e += STATE_THREADS) {
        int i = e / d, j = e % d;
        float s0 = 0.f;
        if (p.S0 && i0 + i < d) s0 = p.S0[((long)bh * d + i0 + i) * d + j];
        S[i * dp + j] = s0;
    }
    for (long c = 0; c < nch; ++c) {
        const long base = ((long)bh * nch + c) * C * d;
        const float *W = (const float *)ws.W + base, *Up = (const float *)ws.Up + base;
        const float *Op = (const float *)ws.Op + base, *Q = (const float *)ws.Qt + base;
        const float *K = (const float *)ws.Kt + base;
        const float gam = ws.gam[((long)bh * nch + c) * 4];
        __syncthreads();
        for (int e = tid; e < C * d; e += STATE_THREADS) {
            Wc[e] = W[e];
            Qt[e] = Q[e];
            Kt[e] = K[e];
        }
        __syncthreads();
        const long t0 = c * C;
        for (int e = tid; e < C * R; e += STATE_THREADS) {
            int t = e / R, i = e % R;
            float x = 0.f, y = 0.f;
            if (i0 + i < d) {
                for (int j = 0; j < d; ++j) {
                    float s = S[i * dp + j];
                    x = fmaf(Wc[t * d + j], s, x);
                    y = fmaf(Qt[t * d + j], s, y);
                }
                Uc[t * R + i] = Up[(long)t * d + i0 + i] - x;
                if (t0 + t < p.L) o[(t0 + t) * d + i0 + i] = Op[(long)t * d + i0 + i] + y;
            } else {
                Uc[t * R + i] = 0.f;
            }
        }
        __syncthreads();
        for (int e = tid; e < R * d; e += STATE_THREADS) {
            int i = e / d, j = e % d;
            float s = gam * S[i * dp + j];
            for (int t = 0; t < C; ++t) s = fmaf(Uc[t * R + i], Kt[t * d + j], s);
            S[i * dp + j] = s;
        }
    }
    __syncthreads();
    if (p.S_out) {
        for (int e = tid; e < R * d; e += STATE_THREADS) {
            int i = e / d, j = e % d;
            if (i0 + i < d) p.S_out[((long)bh * d + i0 + i) * d + j] = S[i * dp + j];
        }
    }
}

}  // namespace

cudaError_t launch_gdn_f32(const GdnArgs &g, cudaStream_t s)
{
    const int d = g.d;
    const long nch = gdn_num_chunks(g.L, C);
    GdnWorkspace ws = gdn_workspace_carve(g.ws, (long)g.B * g.Hg, g.L, d, C, false);
    size_t smem_prep = sizeof(float) * (4 * (size_t)C * (d + 1) + 3 * (size_t)C * (C + 1) + 2 * C);
    size_t smem_state = sizeof(float) * ((size_t)R * (d + 1) + 3 * (size_t)C * d + (size_t)C * R);
    cudaError_t e = cudaFuncSetAttribute(gdn_prep_f32, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_prep);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gdn_state_f32, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_state);
    if (e != cudaSuccess) return e;
    gdn_prep_f32<<<dim3((unsigned)nch, (unsigned)(g.B * g.Hg)), PREP_THREADS, smem_prep, s>>>(g, ws), note_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    gdn_state_f32<<<dim3((unsigned)((d + R - 1) / R), (unsigned)(g.B * g.Hg)), STATE_THREADS,
                    smem_state, s>>>(g, ws), note_launch();
    return cudaGetLastError();
}

}  // namespace hlta
