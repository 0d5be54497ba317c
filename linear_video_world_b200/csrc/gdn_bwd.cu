// Backward pass of the gated delta rule in chunk form (bf16 or fp32 inputs and gradients;
// d = 128, chunks of 64 tokens; fp32 accumulation throughout).
//
// The derivative of the chunk form of the forward pass, term by term. Per chunk, with start
// state S0, end-state gradient dS_C, g the running sum of log a, R = diag(b)(V - diag(e^g) K S0^T),
// U = T R, Qt = diag(e^g) Q - P W and Kt = diag(e^{g_C - g}) K as in the forward:
//   across chunks, last to first:  dS0 = dS_C (gamma I - Kt^T W) + dO^T Qt
//   inside a chunk:  dU = P^T dO + Kt dS_C^T,  dR = T^T dU,  dP = dO U^T (s <= t),
//                    dA = -dR U^T (s < t),  M = dA o b_t e^{g_t - g_s}
//     dQ = diag(e^g) dO S0 + (dP o Gam) K
//     dK = (dP o Gam)^T Q + diag(e^{g_C - g}) U dS_C + M K + M^T K - diag(b e^g) dR S0
//     dV = diag(b) dR
//     db = rowsum(dA o e^{g_t - g_s} o K K^T) + rowsum(dR o (V - diag(e^g) K S0^T))
//     dg = rowsum - colsum of (dP o P) and (dA o A) + e^g o rowsum(Q o dO S0)
//          - b e^g o rowsum(dR o K S0^T) - e^{g_C - g} o rowsum(U o K dS_C^T)
//          + on the last token: gamma <dS_C, S0> + sum_s e^{g_C - g_s} rowsum(U o K dS_C^T)_s
//     d(log a) = reverse running sum of dg inside the chunk,  da = d(log a) / a
// (Gam: e^{g_t - g_s} on s <= t; only such decays, with non-positive exponents, are formed.)
//
// Launches: prep (every chunk in parallel: inputs to fp32, the chunk's A, T, P, W, Up, Qt,
// Kt), the forward state pass storing each chunk's start state, the backward state pass
// storing each chunk's end-state gradient (both serial over chunks, parallel over rows of the
// state), and the gradient kernel (every chunk in parallel). The per-chunk products go through
// one block GEMM routine on the fp32 operands in the workspace: on the CUDA cores for fp32
// tensors, on the tensor cores (mma.sync, operands rounded to bf16, fp32 accumulation) for
// bf16 ones. With bf16 tensors the two state passes are the tensor-core kernels of gdn_tc.cu
// (after the forward's chunk preparation), run on side streams beside this file's prep.
#include "hlta_internal.cuh"

#include <math.h>

namespace hlta {
namespace {

constexpr int C = 64;
constexpr int D = 128;
constexpr int THREADS = 256;
constexpr int R = 8;                // state rows per CTA in the state passes
constexpr int CD = C * D, CC = C * C, DD = D * D;
static_assert(D == 128, "the gradient kernel's row sums take four columns a lane");
constexpr int DS = D + 4;           // staged row stride: 16-byte rows, no bank conflicts
constexpr int CDS = C * DS;
constexpr int TS = 68;              // row stride of the block GEMM's staged tiles
constexpr int AP = C + 4;           // row stride of the prep's A scratch (16-byte rows)

// per chunk-head scratch (floats)
enum : long {
    O_Q = 0, O_K = O_Q + CD, O_V = O_K + CD, O_G = O_V + CD, O_W = O_G + CD, O_UP = O_W + CD,
    O_QT = O_UP + CD, O_KT = O_QT + CD, O_U = O_KT + CD, O_DU = O_U + CD, O_DR = O_DU + CD,
    O_DS = O_DR + CD, O_RS = O_DS + CD, O_UD = O_RS + CD, O_KS = O_UD + CD, O_KD = O_KS + CD,
    O_DQ = O_KD + CD, O_DK = O_DQ + CD,
    O_T = O_DK + CD, O_P = O_T + CC, O_A = O_P + CC, O_KK = O_A + CC, O_DP = O_KK + CC,
    O_DA = O_DP + CC,
    O_S0 = O_DA + CC, O_DSC = O_S0 + DD,
    O_VEC = O_DSC + DD,                 // g, b, a, b e^g, dg (C each), gamma and n
    CHUNK_FLOATS = O_VEC + 6 * C
};

struct BwdP {
    const void *q, *k, *v, *dO;
    const float *a, *b, *S0, *dSL;
    void *dq, *dk, *dv;
    float *da, *db, *dS0;
    float *ws;
    long L;
    int BH, nch;
};

// four consecutive elements (i a multiple of 4, the row 16-byte aligned)
template <typename E> __device__ __forceinline__ float4 ld4(const E *p, long i);
template <> __device__ __forceinline__ float4 ld4<float>(const float *p, long i) { return *reinterpret_cast<const float4 *>(p + i); }
template <> __device__ __forceinline__ float4 ld4<__nv_bfloat16>(const __nv_bfloat16 *p, long i)
{
    const uint2 u = *reinterpret_cast<const uint2 *>(p + i);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}
template <typename E> __device__ __forceinline__ void st4(E *p, long i, float4 v);
template <> __device__ __forceinline__ void st4<float>(float *p, long i, float4 v) { *reinterpret_cast<float4 *>(p + i) = v; }
template <> __device__ __forceinline__ void st4<__nv_bfloat16>(__nv_bfloat16 *p, long i, float4 v)
{
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p + i) = u;
}
__device__ __forceinline__ float4 f4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ void f4st(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ float4 scale4(float a, float4 x) { return make_float4(a * x.x, a * x.y, a * x.z, a * x.w); }


// O[M][N] = alpha * sum_k opA(m, k) s(k) opB(k, n) + beta * O[m][n]; opA(m, k) = A[m][k] or,
// transposed, A[k][m] (leading dimension lda); opB likewise; s an optional per-k scale.
// M, N multiples of 64 and K of 32; 256 threads, each a 4 x 4 block of the 64 x 64 tile read
// as two float4 per k (tile rows padded to 68 floats). O must not alias A or B.
// `sm`: 2 * 32 * 68 floats of shared memory, 16-byte aligned.
__device__ void bgemm(float *O, int ldo, const float *A, int lda, bool tA, const float *B, int ldb,
                      bool tB, const float *s, int M, int N, int K, float alpha, float beta, float *sm)
{
    float *As = sm, *Bs = sm + 32 * TS;            // [k][m], [k][n]
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    // element e of a 32 x 64 operand tile; consecutive threads walk the contiguous index
    auto a_at = [&](int m0, int k0, int e, int &kk, int &mm) -> float {
        if (tA) { kk = e >> 6; mm = e & 63; return A[(long)(k0 + kk) * lda + m0 + mm]; }
        kk = e & 31; mm = e >> 5;
        return A[(long)(m0 + mm) * lda + k0 + kk];
    };
    auto b_at = [&](int n0, int k0, int e, int &kb, int &nb) -> float {
        if (tB) { kb = e & 31; nb = e >> 5; return B[(long)(n0 + nb) * ldb + k0 + kb]; }
        kb = e >> 6; nb = e & 63;
        return B[(long)(k0 + kb) * ldb + n0 + nb];
    };
    constexpr int PER = 32 * 64 / THREADS;          // elements of each tile per thread
    for (int m0 = 0; m0 < M; m0 += 64)
        for (int n0 = 0; n0 < N; n0 += 64) {
            float acc[4][4] = {};
            float ra[PER], rb[PER];
            int dummy0, dummy1;
#pragma unroll
            for (int r = 0; r < PER; ++r) {             // loads of the first k-step
                ra[r] = a_at(m0, 0, threadIdx.x + r * THREADS, dummy0, dummy1);
                rb[r] = b_at(n0, 0, threadIdx.x + r * THREADS, dummy0, dummy1);
            }
            for (int k0 = 0; k0 < K; k0 += 32) {
                __syncthreads();
#pragma unroll
                for (int r = 0; r < PER; ++r) {
                    const int e = threadIdx.x + r * THREADS;
                    int kk, mm, kb, nb;
                    if (tA) { kk = e >> 6; mm = e & 63; } else { kk = e & 31; mm = e >> 5; }
                    if (tB) { kb = e & 31; nb = e >> 5; } else { kb = e >> 6; nb = e & 63; }
                    As[kk * TS + mm] = ra[r];
                    Bs[kb * TS + nb] = (s ? s[k0 + kb] : 1.f) * rb[r];
                }
                __syncthreads();
                if (k0 + 32 < K) {                      // next k-step's loads, in flight meanwhile
#pragma unroll
                    for (int r = 0; r < PER; ++r) {
                        ra[r] = a_at(m0, k0 + 32, threadIdx.x + r * THREADS, dummy0, dummy1);
                        rb[r] = b_at(n0, k0 + 32, threadIdx.x + r * THREADS, dummy0, dummy1);
                    }
                }
#pragma unroll 8
                for (int kk = 0; kk < 32; ++kk) {
                    const float4 xa = *reinterpret_cast<const float4 *>(As + kk * TS + ty * 4);
                    const float4 yb = *reinterpret_cast<const float4 *>(Bs + kk * TS + tx * 4);
                    const float x[4] = {xa.x, xa.y, xa.z, xa.w}, y[4] = {yb.x, yb.y, yb.z, yb.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(x[i], y[j], acc[i][j]);
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float *o = O + (long)(m0 + ty * 4 + i) * ldo + n0 + tx * 4 + j;
                    *o = alpha * acc[i][j] + (beta != 0.f ? beta * *o : 0.f);
                }
        }
    __syncthreads();
}

// The same product on the tensor cores (mma.sync m16n8k16, fp32 accumulation) with A and B
// rounded to bf16 as their fragments are formed: the bf16 path's block GEMM. The fp32 operand
// tiles of every (64 x 64 output tile, 32-wide k-step) stream into shared memory by cp.async
// through a three-stage ring that runs across output tiles, so the loads of later steps are
// in flight while a step computes. Eight warps, each a 16 x 32 piece of the output tile.
// Staged tiles keep the source layout: [64][32] with 40-float rows when k is the contiguous
// index, [32][64] with 68-float rows otherwise (both conflict-free for the fragment reads).
// M, N multiples of 64, K of 32; operand pointers and leading dimensions 16-byte aligned;
// same conventions as bgemm. `smf`: TC_SMEM_FLOATS floats of shared memory, 16-byte aligned.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ void cp_async16(float *dst, const float *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src) : "memory");
}

constexpr int TC_NSTG = 3;                  // stages of the operand ring with two A operands
constexpr int TC_SK = 40;                   // row stride of [64][32] tiles (floats)
constexpr int TC_SN = 68;                   // row stride of [32][64] tiles
constexpr int TC_TILE = 64 * TC_SK;         // floats reserved per operand tile (>= 32 * TC_SN)
constexpr int TC_MAXA = 2;                  // products sharing one B operand per pass
constexpr int TC_SMEM_FLOATS = TC_NSTG * (TC_MAXA + 1) * TC_TILE;
static_assert(32 * TC_SN <= TC_TILE, "a [32][64] tile must fit the reservation");

// NA products O_a = alpha_a A_a opB + beta_a O_a (a < NA) sharing B, tA, lda, ldo and the shape:
// each B tile is staged once for all of them
template <int NA>
__device__ void bgemm_tc_n(float *const (&O)[NA], int ldo, const float *const (&A)[NA], int lda, bool tA,
                           const float *B, int ldb, bool tB, const float *s, int M, int N, int K,
                           const float (&alpha)[NA], const float (&beta)[NA], float *smf)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wm = warp & 3, wn = warp >> 2, g = lane >> 2, tg = lane & 3;
    const int nk = K / 32, ntn = N / 64, steps = (M / 64) * ntn * nk;
    constexpr int STAGE = (NA + 1) * TC_TILE;
    // as many stages as the staging area holds: four with one A operand, three with two
    constexpr int NSTG = TC_SMEM_FLOATS / STAGE;
    static_assert(NSTG >= 3, "at least three stages");
    // step st: output tile st / nk, k-step st % nk, into stage st % NSTG (16-byte copies,
    // two per thread and operand tile)
    auto issue = [&](int st) {
        if (st < steps) {
            const int tile = st / nk, k0 = (st % nk) * 32;
            const int m0 = (tile / ntn) * 64, n0 = (tile % ntn) * 64;
            float *sa = smf + (st % NSTG) * STAGE, *sb = sa + NA * TC_TILE;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int e = tid + r * THREADS;
#pragma unroll
                for (int ia = 0; ia < NA; ++ia) {
                    if (!tA) cp_async16(sa + ia * TC_TILE + (e >> 3) * TC_SK + (e & 7) * 4, A[ia] + (long)(m0 + (e >> 3)) * lda + k0 + (e & 7) * 4);
                    else     cp_async16(sa + ia * TC_TILE + (e >> 4) * TC_SN + (e & 15) * 4, A[ia] + (long)(k0 + (e >> 4)) * lda + m0 + (e & 15) * 4);
                }
                if (tB) cp_async16(sb + (e >> 3) * TC_SK + (e & 7) * 4, B + (long)(n0 + (e >> 3)) * ldb + k0 + (e & 7) * 4);
                else    cp_async16(sb + (e >> 4) * TC_SN + (e & 15) * 4, B + (long)(k0 + (e >> 4)) * ldb + n0 + (e & 15) * 4);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");   // empty groups past the end keep the count uniform
    };
    __syncthreads();                                // the caller's operand stores are visible
#pragma unroll
    for (int st = 0; st < NSTG - 1; ++st) issue(st);
    float acc[NA][4][4] = {};
    for (int st = 0; st < steps; ++st) {
        asm volatile("cp.async.wait_group %0;" ::"n"(NSTG - 2) : "memory");
        __syncthreads();                            // step st landed for all; stage st - 1 is free
        issue(st + NSTG - 1);
        const float *sa = smf + (st % NSTG) * STAGE, *sb = sa + NA * TC_TILE;
        const int k0 = (st % nk) * 32;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const int kb = ks * 16 + 2 * tg;        // this lane's k pairs: kb, kb + 1 and kb + 8, kb + 9
            const int r0 = 16 * wm + g;
            uint32_t a[NA][4];
#pragma unroll
            for (int ia = 0; ia < NA; ++ia) {
                const float *t = sa + ia * TC_TILE;
                if (!tA) {
                    const float2 x0 = *reinterpret_cast<const float2 *>(t + r0 * TC_SK + kb);
                    const float2 x1 = *reinterpret_cast<const float2 *>(t + (r0 + 8) * TC_SK + kb);
                    const float2 x2 = *reinterpret_cast<const float2 *>(t + r0 * TC_SK + kb + 8);
                    const float2 x3 = *reinterpret_cast<const float2 *>(t + (r0 + 8) * TC_SK + kb + 8);
                    a[ia][0] = pack_bf16x2(x0.x, x0.y);
                    a[ia][1] = pack_bf16x2(x1.x, x1.y);
                    a[ia][2] = pack_bf16x2(x2.x, x2.y);
                    a[ia][3] = pack_bf16x2(x3.x, x3.y);
                } else {
                    a[ia][0] = pack_bf16x2(t[kb * TC_SN + r0], t[(kb + 1) * TC_SN + r0]);
                    a[ia][1] = pack_bf16x2(t[kb * TC_SN + r0 + 8], t[(kb + 1) * TC_SN + r0 + 8]);
                    a[ia][2] = pack_bf16x2(t[(kb + 8) * TC_SN + r0], t[(kb + 9) * TC_SN + r0]);
                    a[ia][3] = pack_bf16x2(t[(kb + 8) * TC_SN + r0 + 8], t[(kb + 9) * TC_SN + r0 + 8]);
                }
            }
            float s0 = 1.f, s1 = 1.f, s8 = 1.f, s9 = 1.f;
            if (s) {
                s0 = s[k0 + kb];
                s1 = s[k0 + kb + 1];
                s8 = s[k0 + kb + 8];
                s9 = s[k0 + kb + 9];
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int cn = 32 * wn + 8 * nt + g;
                float b0, b1, b8, b9;
                if (tB) {
                    const float2 y0 = *reinterpret_cast<const float2 *>(sb + cn * TC_SK + kb);
                    const float2 y1 = *reinterpret_cast<const float2 *>(sb + cn * TC_SK + kb + 8);
                    b0 = y0.x; b1 = y0.y; b8 = y1.x; b9 = y1.y;
                } else {
                    b0 = sb[kb * TC_SN + cn];
                    b1 = sb[(kb + 1) * TC_SN + cn];
                    b8 = sb[(kb + 8) * TC_SN + cn];
                    b9 = sb[(kb + 9) * TC_SN + cn];
                }
                const uint32_t bp0 = pack_bf16x2(b0 * s0, b1 * s1), bp1 = pack_bf16x2(b8 * s8, b9 * s9);
#pragma unroll
                for (int ia = 0; ia < NA; ++ia) mma_bf16_16816(acc[ia][nt], a[ia], bp0, bp1);
            }
        }
        if (st % nk == nk - 1) {                    // the output tile's last k-step
            const int tile = st / nk;
            const int m0 = (tile / ntn) * 64, n0 = (tile % ntn) * 64;
#pragma unroll
            for (int ia = 0; ia < NA; ++ia)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float2 *o = reinterpret_cast<float2 *>(O[ia] + (long)(m0 + 16 * wm + g + 8 * hh) * ldo + n0 + 32 * wn + 8 * nt + 2 * tg);
                        float2 v = make_float2(alpha[ia] * acc[ia][nt][2 * hh], alpha[ia] * acc[ia][nt][2 * hh + 1]);
                        if (beta[ia] != 0.f) {
                            const float2 old = *o;
                            v.x = fmaf(beta[ia], old.x, v.x);
                            v.y = fmaf(beta[ia], old.y, v.y);
                        }
                        *o = v;
                        acc[ia][nt][2 * hh] = acc[ia][nt][2 * hh + 1] = 0.f;
                    }
        }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
}

__device__ __forceinline__ void bgemm_tc(float *O, int ldo, const float *A, int lda, bool tA, const float *B, int ldb,
                                         bool tB, const float *s, int M, int N, int K, float alpha, float beta, float *smf)
{
    float *const o1[1] = {O};
    const float *const a1[1] = {A};
    const float al[1] = {alpha}, be[1] = {beta};
    bgemm_tc_n<1>(o1, ldo, a1, lda, tA, B, ldb, tB, s, M, N, K, al, be, smf);
}

template <typename E>
constexpr int gemm_smem_bytes() { return (int)sizeof(float) * (sizeof(E) == 2 ? TC_SMEM_FLOATS : 2 * 32 * TS); }
static_assert(C * AP <= 2 * 32 * TS, "the prep kernel's A scratch aliases the GEMM staging");

// two products sharing B (and tA, lda, ldo, the shape): B staged once on the tensor-core path
template <typename E>
__device__ __forceinline__ void gemm2(float *O1, float *O2, int ldo, const float *A1, const float *A2, int lda,
                                      bool tA, const float *B, int ldb, bool tB, int M, int N, int K,
                                      float alpha1, float beta1, float alpha2, float beta2, float *sm)
{
    if constexpr (sizeof(E) == 2) {
        float *const o[2] = {O1, O2};
        const float *const a[2] = {A1, A2};
        const float al[2] = {alpha1, alpha2}, be[2] = {beta1, beta2};
        bgemm_tc_n<2>(o, ldo, a, lda, tA, B, ldb, tB, nullptr, M, N, K, al, be, sm);
    } else {
        bgemm(O1, ldo, A1, lda, tA, B, ldb, tB, nullptr, M, N, K, alpha1, beta1, sm);
        bgemm(O2, ldo, A2, lda, tA, B, ldb, tB, nullptr, M, N, K, alpha2, beta2, sm);
    }
}

template <typename E>
__device__ __forceinline__ void gemm(float *O, int ldo, const float *A, int lda, bool tA, const float *B, int ldb,
                                     bool tB, const float *s, int M, int N, int K, float alpha, float beta, float *sm)
{
    if constexpr (sizeof(E) == 2) bgemm_tc(O, ldo, A, lda, tA, B, ldb, tB, s, M, N, K, alpha, beta, sm);
    else bgemm(O, ldo, A, lda, tA, B, ldb, tB, s, M, N, K, alpha, beta, sm);
}

// ----------------------------------------------------------------------------------------
// prep: one CTA per (chunk, head)
template <typename E>
__global__ void __launch_bounds__(THREADS, 2) gdn_bwd_prep(BwdP p)
{
    extern __shared__ __align__(16) float sm[];        // the block GEMM's staging (gemm_smem_bytes)
    float *At = sm;                                     // [C][AP] between GEMMs only
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    float *w = p.ws + ((long)bh * p.nch + c) * CHUNK_FLOATS;
    const long t0 = (long)c * C;
    const int n = (int)min((long)C, p.L - t0);
    const long base = ((long)bh * p.L + t0) * D;
    float *g = w + O_VEC, *bb = g + C, *aa = bb + C, *bg = aa + C;
    for (int e = 4 * tid; e < CD; e += 4 * THREADS) {  // four elements of one token a thread
        const bool ok = e / D < n;
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        f4st(w + O_Q + e, ok ? ld4((const E *)p.q, base + e) : z);
        f4st(w + O_K + e, ok ? ld4((const E *)p.k, base + e) : z);
        f4st(w + O_V + e, ok ? ld4((const E *)p.v, base + e) : z);
        f4st(w + O_G + e, ok ? ld4((const E *)p.dO, base + e) : z);
    }
    if (tid < 32) {
        // g_t = running sum of log a over the chunk (tokens past n add nothing): two tokens a
        // lane, then a warp scan
        const int lane = tid, t = 2 * lane;
        const long gi = (long)bh * p.L + t0 + t;
        const float a0 = t < n ? p.a[gi] : 1.f, a1 = t + 1 < n ? p.a[gi + 1] : 1.f;
        const float l0 = t < n ? logf(a0) : 0.f, l1 = t + 1 < n ? logf(a1) : 0.f;
        const float pair = l0 + l1;
        float x = pair;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        const float gt0 = x - pair + l0, gt1 = x;
        const float b0 = t < n ? p.b[gi] : 0.f, b1 = t + 1 < n ? p.b[gi + 1] : 0.f;
        g[t] = gt0;
        g[t + 1] = gt1;
        bb[t] = b0;
        bb[t + 1] = b1;
        aa[t] = a0;
        aa[t + 1] = a1;
        bg[t] = b0 * expf(gt0);
        bg[t + 1] = b1 * expf(gt1);
        if (lane == 31) w[O_VEC + 5 * C] = expf(gt1);   // gamma = e^{g of the last token}
        if (lane == 0) w[O_VEC + 5 * C + 1] = (float)n;
    }
    __syncthreads();
    gemm<E>(w + O_KK, C, w + O_K, D, false, w + O_K, D, true, nullptr, C, C, D, 1.f, 0.f, sm);
    gemm<E>(w + O_P, C, w + O_Q, D, false, w + O_K, D, true, nullptr, C, C, D, 1.f, 0.f, sm);
    for (int e = 4 * tid; e < CC; e += 4 * THREADS) {  // columns s .. s + 3 of row t
        const int t = e / C, s0 = e % C;
        const float gt = g[t], bt = bb[t];
        const float4 gs = f4(g + s0), kk = f4(w + O_KK + e), pp = f4(w + O_P + e);
        const float gsv[4] = {gs.x, gs.y, gs.z, gs.w}, kkv[4] = {kk.x, kk.y, kk.z, kk.w};
        const float ppv[4] = {pp.x, pp.y, pp.z, pp.w};
        float av[4], pv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int s = s0 + u;
            const float dec = (s <= t && t < n) ? expf(gt - gsv[u]) : 0.f;
            av[u] = s < t ? bt * dec * kkv[u] : 0.f;
            pv[u] = dec * ppv[u];
        }
        const float4 a4 = make_float4(av[0], av[1], av[2], av[3]);
        f4st(w + O_A + e, a4);
        f4st(At + t * AP + s0, a4);
        f4st(w + O_P + e, make_float4(pv[0], pv[1], pv[2], pv[3]));
    }
    __syncthreads();
    if (tid < C) {
        // T = (I + A)^{-1} by forward substitution, column j = tid in registers:
        // T_tj = -sum_{i<t} A_ti T_ij (0 above the diagonal, 1 on it); rows of A read as
        // float4 broadcasts into four partial sums
        const int j = tid;
        float tc[C];
#pragma unroll
        for (int t = 0; t < C; ++t) {
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            const float4 *ar = reinterpret_cast<const float4 *>(At + t * AP);
#pragma unroll
            for (int i4 = 0; i4 < t / 4; ++i4) {
                const float4 av = ar[i4];
                a0 = fmaf(av.x, tc[4 * i4], a0);
                a1 = fmaf(av.y, tc[4 * i4 + 1], a1);
                a2 = fmaf(av.z, tc[4 * i4 + 2], a2);
                a3 = fmaf(av.w, tc[4 * i4 + 3], a3);
            }
#pragma unroll
            for (int i = (t / 4) * 4; i < t; ++i) a0 = fmaf(At[t * AP + i], tc[i], a0);
            tc[t] = t < j ? 0.f : (t == j ? 1.f : -((a0 + a1) + (a2 + a3)));
        }
#pragma unroll
        for (int t = 0; t < C; ++t) w[O_T + t * C + j] = tc[t];
    }
    __syncthreads();
    gemm<E>(w + O_W, D, w + O_T, C, false, w + O_K, D, false, bg, C, D, C, 1.f, 0.f, sm);
    gemm<E>(w + O_UP, D, w + O_T, C, false, w + O_V, D, false, bb, C, D, C, 1.f, 0.f, sm);
    const float gC = g[C - 1];
    for (int e = 4 * tid; e < CD; e += 4 * THREADS) {
        const int t = e / D;
        f4st(w + O_QT + e, scale4(t < n ? expf(g[t]) : 0.f, f4(w + O_Q + e)));
        f4st(w + O_KT + e, scale4(t < n ? expf(gC - g[t]) : 0.f, f4(w + O_K + e)));
    }
    gemm<E>(w + O_QT, D, w + O_P, C, false, w + O_W, D, false, nullptr, C, D, C, -1.f, 1.f, sm);
}

// ----------------------------------------------------------------------------------------
// State passes: one CTA per R rows of one head's state, serial over the chunks; each chunk's
// C x d products are staged in shared memory (coalesced float4 copies) before use.
// a C x D fp32 array into shared memory rows of DS floats
__device__ __forceinline__ void stage(float *dst, const float *src, int n)
{
    const uint32_t d0 = (uint32_t)__cvta_generic_to_shared(dst);
    for (int e = threadIdx.x; e < n / 4; e += THREADS) {
        const int t = e / (D / 4), c4 = e % (D / 4);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d0 + 4u * (uint32_t)(t * DS + 4 * c4)),
                     "l"(src + 4 * e)
                     : "memory");
    }
}
__device__ __forceinline__ void stage_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void stage_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Register-blocked inner products of the state passes (R = 8 rows per CTA):
//   dot:    thread (token tq, lane quarter q) sums x_i = sum_j X[tq][j] S[i][j] over the
//           columns j = 4 jj + q for all eight rows (the rows of S at one column are one 32-byte
//           line of ST, read as two broadcast float4), then the four quarters are added by
//           shuffles;
//   update: thread (column j, rows h4 .. h4+3) keeps its four state values in registers and
//           adds the C rank-one terms, reading the per-row coefficients as broadcast float4.
static_assert(R == 8, "state passes are written for 8 rows per CTA");

__device__ __forceinline__ void dot8(float (&x)[8], const float *Xrow, const float *ST, int q)
{
    const float4 *ST4 = reinterpret_cast<const float4 *>(ST);
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = 0.f;
#pragma unroll 8
    for (int jj = 0; jj < D / 4; ++jj) {
        const int jx = 4 * jj + q;
        const float wv = Xrow[jx];
        const float4 a = ST4[2 * jx], b = ST4[2 * jx + 1];
        x[0] = fmaf(wv, a.x, x[0]); x[1] = fmaf(wv, a.y, x[1]);
        x[2] = fmaf(wv, a.z, x[2]); x[3] = fmaf(wv, a.w, x[3]);
        x[4] = fmaf(wv, b.x, x[4]); x[5] = fmaf(wv, b.y, x[5]);
        x[6] = fmaf(wv, b.z, x[6]); x[7] = fmaf(wv, b.w, x[7]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[i] += __shfl_xor_sync(0xffffffffu, x[i], 1);
        x[i] += __shfl_xor_sync(0xffffffffu, x[i], 2);
    }
}

// forward: stores every chunk's start state (rows of this CTA)
__global__ void __launch_bounds__(THREADS) gdn_bwd_fwdstate(BwdP p)
{
    extern __shared__ __align__(16) float dsm[];
    float *buf = dsm;                               // two stages of W, Kt: [2][2][C][DS]
    float *ST = dsm + 4 * CDS;                      // [D][R] the state, column-major
    float *Uc = ST + D * R;                         // [C][R] U on this slice
    float *Ups = Uc + C * R;                        // [C][R] this slice's columns of Up
    const int i0 = blockIdx.x * R, bh = blockIdx.y, tid = threadIdx.x;
    const int j = tid & (D - 1), h4 = (tid >> 7) * 4;
    const int q = tid & 3, tq = tid >> 2;
    float sv[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        sv[r] = p.S0 ? p.S0[((long)bh * D + i0 + h4 + r) * D + j] : 0.f;
        ST[j * R + h4 + r] = sv[r];
    }
    {
        const float *w0 = p.ws + (long)bh * p.nch * CHUNK_FLOATS;
        stage(buf, w0 + O_W, CD);
        stage(buf + CDS, w0 + O_KT, CD);
        stage_commit();
    }
    for (int c = 0; c < p.nch; ++c) {
        float *w = p.ws + ((long)bh * p.nch + c) * CHUNK_FLOATS;
        const float *Wc = buf + (c & 1) * 2 * CDS, *Kc = Wc + CDS;
        const float gam = w[O_VEC + 5 * C];
        __syncthreads();                            // the other stage and Uc are free again
        if (c + 1 < p.nch) {
            const float *wn = w + CHUNK_FLOATS;
            stage(buf + ((c + 1) & 1) * 2 * CDS, wn + O_W, CD);
            stage(buf + ((c + 1) & 1) * 2 * CDS + CDS, wn + O_KT, CD);
        }
        stage_commit();
#pragma unroll
        for (int r = 0; r < 4; ++r) w[O_S0 + (long)(i0 + h4 + r) * D + j] = sv[r];
        for (int e = tid; e < C * R; e += THREADS) Ups[e] = w[O_UP + (e / R) * D + i0 + e % R];
        stage_wait_prev();
        __syncthreads();
        float x[8];                                 // U = Up - W S0^T on this slice
        dot8(x, Wc + tq * DS, ST, q);
        if (q == 0)
#pragma unroll
            for (int i = 0; i < 8; ++i) Uc[tq * R + i] = Ups[tq * R + i] - x[i];
        __syncthreads();
        const float4 *U4 = reinterpret_cast<const float4 *>(Uc);
#pragma unroll
        for (int r = 0; r < 4; ++r) sv[r] *= gam;   // S = gamma S + U^T Kt
#pragma unroll 8
        for (int t = 0; t < C; ++t) {
            const float kv = Kc[t * DS + j];
            const float4 u = U4[t * 2 + h4 / 4];
            sv[0] = fmaf(u.x, kv, sv[0]); sv[1] = fmaf(u.y, kv, sv[1]);
            sv[2] = fmaf(u.z, kv, sv[2]); sv[3] = fmaf(u.w, kv, sv[3]);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) ST[j * R + h4 + r] = sv[r];
    }
}

// backward: dS <- dS (gamma I - Kt^T W) + dO^T Qt from the last chunk to the first; stores
// every chunk's end-state gradient and writes dS0
__global__ void __launch_bounds__(THREADS) gdn_bwd_bwdstate(BwdP p)
{
    extern __shared__ __align__(16) float dsm[];
    float *buf = dsm;                               // two stages of W, Kt, Qt: [2][3][C][DS]
    float *ST = dsm + 6 * CDS;                      // [D][R] the state gradient, column-major
    float *Y = ST + D * R;                          // [C][R] Kt dS^T on this slice
    float *Gs = Y + C * R;                          // [C][R] this slice's columns of dO
    const int i0 = blockIdx.x * R, bh = blockIdx.y, tid = threadIdx.x;
    const int j = tid & (D - 1), h4 = (tid >> 7) * 4;
    const int q = tid & 3, tq = tid >> 2;
    float sv[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        sv[r] = p.dSL ? p.dSL[((long)bh * D + i0 + h4 + r) * D + j] : 0.f;
        ST[j * R + h4 + r] = sv[r];
    }
    {
        const float *wl = p.ws + ((long)bh * p.nch + p.nch - 1) * CHUNK_FLOATS;
        stage(buf, wl + O_W, CD);
        stage(buf + CDS, wl + O_KT, CD);
        stage(buf + 2 * CDS, wl + O_QT, CD);
        stage_commit();
    }
    for (int c = p.nch - 1; c >= 0; --c) {
        float *w = p.ws + ((long)bh * p.nch + c) * CHUNK_FLOATS;
        const int sl = (p.nch - 1 - c) & 1;
        const float *Wc = buf + sl * 3 * CDS, *Kc = Wc + CDS, *Qc = Kc + CDS;
        const float gam = w[O_VEC + 5 * C];
        __syncthreads();                            // the other stage, Y and Gs are free again
        if (c > 0) {
            const float *wn = w - CHUNK_FLOATS;
            float *nb = buf + (sl ^ 1) * 3 * CDS;
            stage(nb, wn + O_W, CD);
            stage(nb + CDS, wn + O_KT, CD);
            stage(nb + 2 * CDS, wn + O_QT, CD);
        }
        stage_commit();
#pragma unroll
        for (int r = 0; r < 4; ++r) w[O_DSC + (long)(i0 + h4 + r) * D + j] = sv[r];
        for (int e = tid; e < C * R; e += THREADS) Gs[e] = w[O_G + (e / R) * D + i0 + e % R];
        stage_wait_prev();
        __syncthreads();
        float x[8];                                 // Y = Kt dS^T on this slice
        dot8(x, Kc + tq * DS, ST, q);
        if (q == 0)
#pragma unroll
            for (int i = 0; i < 8; ++i) Y[tq * R + i] = x[i];
        __syncthreads();
        const float4 *Y4 = reinterpret_cast<const float4 *>(Y), *G4 = reinterpret_cast<const float4 *>(Gs);
#pragma unroll
        for (int r = 0; r < 4; ++r) sv[r] *= gam;
#pragma unroll 4
        for (int t = 0; t < C; ++t) {
            const float qv = Qc[t * DS + j], wv = Wc[t * DS + j];
            const float4 gg = G4[t * 2 + h4 / 4], yy = Y4[t * 2 + h4 / 4];
            sv[0] = fmaf(gg.x, qv, fmaf(-yy.x, wv, sv[0]));
            sv[1] = fmaf(gg.y, qv, fmaf(-yy.y, wv, sv[1]));
            sv[2] = fmaf(gg.z, qv, fmaf(-yy.z, wv, sv[2]));
            sv[3] = fmaf(gg.w, qv, fmaf(-yy.w, wv, sv[3]));
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) ST[j * R + h4 + r] = sv[r];
    }
    if (p.dS0)
#pragma unroll
        for (int r = 0; r < 4; ++r) p.dS0[((long)bh * D + i0 + h4 + r) * D + j] = sv[r];
}

// ----------------------------------------------------------------------------------------
// gradients of one chunk
template <typename E>
__global__ void __launch_bounds__(THREADS, 2) gdn_bwd_grad(BwdP p)
{
    extern __shared__ __align__(16) float sm[];        // the block GEMM's staging (gemm_smem_bytes)
    __shared__ float red[THREADS / 32];
    __shared__ float rowv[6][C];
    __shared__ float colp[THREADS / C][C], cola[THREADS / C][C];
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    float *w = p.ws + ((long)bh * p.nch + c) * CHUNK_FLOATS;
    const float *g = w + O_VEC, *bb = g + C, *aa = bb + C;
    float *dg = w + O_VEC + 4 * C;
    const float gam = w[O_VEC + 5 * C];
    const int n = (int)w[O_VEC + 5 * C + 1];
    const float gC = g[C - 1];
    const float *S0 = w + O_S0, *dSC = w + O_DSC;
    // U = Up - W S0^T and K S0^T
    for (int e = 4 * tid; e < CD; e += 4 * THREADS) f4st(w + O_U + e, f4(w + O_UP + e));
    gemm2<E>(w + O_U, w + O_KS, D, w + O_W, w + O_K, D, false, S0, D, true, C, D, D, -1.f, 1.f, 1.f, 0.f, sm);
    // dU = Kt dS_C^T + P^T dO (and K dS_C^T);  dR = T^T dU
    gemm2<E>(w + O_DU, w + O_KD, D, w + O_KT, w + O_K, D, false, dSC, D, true, C, D, D, 1.f, 0.f, 1.f, 0.f, sm);
    gemm<E>(w + O_DU, D, w + O_P, C, true, w + O_G, D, false, nullptr, C, D, C, 1.f, 1.f, sm);
    gemm<E>(w + O_DR, D, w + O_T, C, true, w + O_DU, D, false, nullptr, C, D, C, 1.f, 0.f, sm);
    // C x C: dP = dO U^T, dA' = dR U^T
    gemm2<E>(w + O_DP, w + O_DA, C, w + O_G, w + O_DR, D, false, w + O_U, D, true, C, C, D, 1.f, 0.f, 1.f, 0.f, sm);
    // products with the d x d states: dO S0, dR S0, U dS_C
    gemm2<E>(w + O_DS, w + O_RS, D, w + O_G, w + O_DR, D, false, S0, D, false, C, D, D, 1.f, 0.f, 1.f, 0.f, sm);
    gemm<E>(w + O_UD, D, w + O_U, D, false, dSC, D, false, nullptr, C, D, D, 1.f, 0.f, sm);
    // per-row sums over the C x C products and the C x d ones: warp w takes rows 8w .. 8w + 7,
    // its lanes the columns (coalesced), combined by butterfly shuffles
    const int warp = tid >> 5, lane = tid & 31;
    for (int rr = 0; rr < C / 8; ++rr) {
        const int t = warp * (C / 8) + rr;
        const bool ok = t < n;
        float pp = 0.f, ap = 0.f, db1 = 0.f;
        for (int s = lane; s < C; s += 32) {
            const bool inc = s <= t && ok, low = s < t && ok;
            const float dpv = inc ? w[O_DP + t * C + s] : 0.f;
            const float dav = low ? -w[O_DA + t * C + s] : 0.f;
            pp += dpv * w[O_P + t * C + s];
            ap += dav * w[O_A + t * C + s];
            db1 += low ? dav * expf(g[t] - g[s]) * w[O_KK + t * C + s] : 0.f;
        }
        const float eg = expf(g[t]);
        float qds = 0.f, drk = 0.f, ukd = 0.f, drv = 0.f;
        {
            const int j = 4 * lane;                         // D = 128: four columns a lane
            const float4 ks = f4(w + O_KS + t * D + j), dr = f4(w + O_DR + t * D + j);
            const float4 qq = f4(w + O_Q + t * D + j), ds = f4(w + O_DS + t * D + j);
            const float4 uu = f4(w + O_U + t * D + j), kd = f4(w + O_KD + t * D + j);
            const float4 vv = f4(w + O_V + t * D + j);
            qds = fmaf(qq.x, ds.x, fmaf(qq.y, ds.y, fmaf(qq.z, ds.z, qq.w * ds.w)));
            drk = fmaf(dr.x, ks.x, fmaf(dr.y, ks.y, fmaf(dr.z, ks.z, dr.w * ks.w)));
            ukd = fmaf(uu.x, kd.x, fmaf(uu.y, kd.y, fmaf(uu.z, kd.z, uu.w * kd.w)));
            drv = fmaf(dr.x, vv.x - eg * ks.x, fmaf(dr.y, vv.y - eg * ks.y,
                  fmaf(dr.z, vv.z - eg * ks.z, dr.w * (vv.w - eg * ks.w))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            pp += __shfl_xor_sync(0xffffffffu, pp, o);
            ap += __shfl_xor_sync(0xffffffffu, ap, o);
            db1 += __shfl_xor_sync(0xffffffffu, db1, o);
            qds += __shfl_xor_sync(0xffffffffu, qds, o);
            drk += __shfl_xor_sync(0xffffffffu, drk, o);
            ukd += __shfl_xor_sync(0xffffffffu, ukd, o);
            drv += __shfl_xor_sync(0xffffffffu, drv, o);
        }
        if (lane == 0) {
            rowv[0][t] = pp;
            rowv[1][t] = ap;
            rowv[2][t] = db1;
            dg[t] = ok ? eg * qds - bb[t] * eg * drk - expf(gC - g[t]) * ukd : 0.f;
            rowv[5][t] = ok ? expf(gC - g[t]) * ukd : 0.f;  // for the last token's term
            w[O_DU + t] = drv;                               // (dU is free now) db part 2
        }
    }
    // column sums of the same C x C products: column s = tid % C, rows t = tid / C + 4i
    {
        const int sc = tid & (C - 1), q4 = tid >> 6;
        float pp = 0.f, ap = 0.f;
        for (int t = q4; t < n; t += THREADS / C) {
            if (t < sc) continue;
            pp += w[O_DP + t * C + sc] * w[O_P + t * C + sc];
            if (t > sc) ap += -w[O_DA + t * C + sc] * w[O_A + t * C + sc];
        }
        colp[q4][sc] = pp;
        cola[q4][sc] = ap;
    }
    // <dS_C, S0>
    float sd = 0.f;
    for (int e = 4 * tid; e < DD; e += 4 * THREADS) {
        const float4 x = f4(dSC + e), y = f4(S0 + e);
        sd = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, fmaf(x.w, y.w, sd))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sd += __shfl_xor_sync(0xffffffffu, sd, o);
    if (lane == 0) red[warp] = sd;
    __syncthreads();
    if (warp == 0) {
        // d(log a)_t = sum over t' >= t (t' < n) of v_t': a reverse running sum, two tokens a lane
        float tot = 0.f;
#pragma unroll
        for (int i = 0; i < THREADS / 32; ++i) tot += red[i];
        float su = (lane < n ? rowv[5][lane] : 0.f) + (lane + 32 < n ? rowv[5][lane + 32] : 0.f);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) su += __shfl_xor_sync(0xffffffffu, su, o);
        float v[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int t = lane + 32 * hh;
            float cs = 0.f, ca = 0.f;
#pragma unroll
            for (int i = 0; i < THREADS / C; ++i) {
                cs += colp[i][t];
                ca += cola[i][t];
            }
            float x = dg[t] + rowv[0][t] - cs + rowv[1][t] - ca;
            if (t == n - 1) x += gam * tot + su;
            v[hh] = t < n ? x : 0.f;
        }
        // suffix sums: the upper half within itself, the lower half plus the upper total
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, v[hh], o);
                if (lane + o < 32) v[hh] += y;
            }
        v[0] += __shfl_sync(0xffffffffu, v[1], 0);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int t = lane + 32 * hh;
            if (t < n) {
                const long gi = (long)bh * p.L + (long)c * C + t;
                p.da[gi] = v[hh] / aa[t];
                p.db[gi] = rowv[2][t] + w[O_DU + t];
            }
        }
    }
    // M = dA o b_t e^{g_t - g_s} (s < t) into O_DA;  dP o Gam into O_DP
    for (int e = 4 * tid; e < CC; e += 4 * THREADS) {  // columns s .. s + 3 of row t
        const int t = e / C, s0 = e % C;
        const float gt = g[t], bt = bb[t];
        const float4 gs = f4(g + s0), da = f4(w + O_DA + e), dp = f4(w + O_DP + e);
        const float gsv[4] = {gs.x, gs.y, gs.z, gs.w}, dav[4] = {da.x, da.y, da.z, da.w};
        const float dpv[4] = {dp.x, dp.y, dp.z, dp.w};
        float mo[4], po[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int s = s0 + u;
            const bool inc = s <= t && t < n, low = s < t && t < n;
            const float dec = inc ? expf(gt - gsv[u]) : 0.f;
            mo[u] = low ? -dav[u] * bt * dec : 0.f;
            po[u] = inc ? dpv[u] * dec : 0.f;
        }
        f4st(w + O_DA + e, make_float4(mo[0], mo[1], mo[2], mo[3]));
        f4st(w + O_DP + e, make_float4(po[0], po[1], po[2], po[3]));
    }
    __syncthreads();
    // dQ = diag(e^g) dO S0 + (dP o Gam) K
    for (int e = 4 * tid; e < CD; e += 4 * THREADS) f4st(w + O_DQ + e, scale4(expf(g[e / D]), f4(w + O_DS + e)));
    gemm<E>(w + O_DQ, D, w + O_DP, C, false, w + O_K, D, false, nullptr, C, D, C, 1.f, 1.f, sm);
    // dK = diag(e^{g_C - g}) U dS_C - diag(b e^g) dR S0 + (dP o Gam)^T Q + M K + M^T K
    for (int e = 4 * tid; e < CD; e += 4 * THREADS) {
        const int t = e / D;
        const float cu = t < n ? expf(gC - g[t]) : 0.f, cr = t < n ? -bb[t] * expf(g[t]) : 0.f;
        const float4 ud = f4(w + O_UD + e), rs = f4(w + O_RS + e);
        f4st(w + O_DK + e, make_float4(fmaf(cu, ud.x, cr * rs.x), fmaf(cu, ud.y, cr * rs.y),
                                       fmaf(cu, ud.z, cr * rs.z), fmaf(cu, ud.w, cr * rs.w)));
    }
    gemm<E>(w + O_DK, D, w + O_DP, C, true, w + O_Q, D, false, nullptr, C, D, C, 1.f, 1.f, sm);
    gemm<E>(w + O_DK, D, w + O_DA, C, false, w + O_K, D, false, nullptr, C, D, C, 1.f, 1.f, sm);
    gemm<E>(w + O_DK, D, w + O_DA, C, true, w + O_K, D, false, nullptr, C, D, C, 1.f, 1.f, sm);
    const long base = ((long)bh * p.L + (long)c * C) * D;
    for (int e = 4 * tid; e < n * D; e += 4 * THREADS) {
        st4((E *)p.dq, base + e, f4(w + O_DQ + e));
        st4((E *)p.dk, base + e, f4(w + O_DK + e));
        st4((E *)p.dv, base + e, scale4(bb[e / D], f4(w + O_DR + e)));
    }
}

template <typename E>
cudaError_t set_gemm_smem()
{
    cudaError_t e = cudaFuncSetAttribute(gdn_bwd_prep<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem_bytes<E>());
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(gdn_bwd_grad<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem_bytes<E>());
}

template <typename E>
cudaError_t launch_typed(const BwdP &p, cudaStream_t s)
{
    const dim3 gc((unsigned)p.nch, (unsigned)p.BH), gs((unsigned)(D / R), (unsigned)p.BH);
    const int sm_f = (int)sizeof(float) * (4 * CDS + D * R + 2 * C * R);
    const int sm_b = (int)sizeof(float) * (6 * CDS + D * R + 2 * C * R);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(gdn_bwd_fwdstate, cudaFuncAttributeMaxDynamicSharedMemorySize, sm_f)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(gdn_bwd_bwdstate, cudaFuncAttributeMaxDynamicSharedMemorySize, sm_b)) != cudaSuccess) return e;
    if ((e = set_gemm_smem<E>()) != cudaSuccess) return e;
    gdn_bwd_prep<E><<<gc, THREADS, gemm_smem_bytes<E>(), s>>>(p), note_launch();
    gdn_bwd_fwdstate<<<gs, THREADS, sm_f, s>>>(p), note_launch();
    gdn_bwd_bwdstate<<<gs, THREADS, sm_b, s>>>(p), note_launch();
    gdn_bwd_grad<E><<<gc, THREADS, gemm_smem_bytes<E>(), s>>>(p), note_launch();
    return cudaGetLastError();
}

// fp32 chunk scratch, then the bf16 forward's chunk products (the bf16 path's state passes
// run on the tensor cores from those)
size_t bwd_f32_bytes(long BH, long L)
{
    return ((size_t)BH * (size_t)gdn_num_chunks(L, C) * (size_t)CHUNK_FLOATS * sizeof(float) + 255) & ~(size_t)255;
}

}  // namespace

size_t gdn_bwd_workspace_bytes(long BH, long L)
{
    return bwd_f32_bytes(BH, L) + gdn_rowmajor_bytes(BH, L, D, C, true);
}

cudaError_t launch_gdn_bwd(const GdnBwdArgs &a, cudaStream_t s, const SideStreams *side)
{
    if (a.d != D) return cudaErrorNotSupported;
    if (a.B * a.H == 0 || a.L == 0) return cudaSuccess;
    const long nch = gdn_num_chunks(a.L, C);
    if (nch >= (1L << 31) || (long)a.B * a.H > 65535) return cudaErrorNotSupported;
    BwdP p;
    p.q = a.q; p.k = a.k; p.v = a.v; p.dO = a.dO;
    p.a = a.a; p.b = a.b; p.S0 = a.S0; p.dSL = a.dS_final;
    p.dq = a.dq; p.dk = a.dk; p.dv = a.dv; p.da = a.da; p.db = a.db; p.dS0 = a.dS0;
    p.ws = (float *)a.ws;
    p.L = a.L;
    p.BH = a.B * a.H;
    p.nch = (int)nch;
    if (!a.bf16) return launch_typed<float>(p, s);
    // bf16: the state passes on the tensor cores, from the forward's bf16 chunk products.
    // With side streams they run there (each a serial chain on a few SMs, dispatched first),
    // beside the chunk preparation on the caller's stream; the gradient kernel needs both.
    cudaError_t e;
    const cudaStream_t sa = side ? side->a : s, sb = side ? side->b : s;
    if (side) {
        if ((e = cudaEventRecord(side->fork, s)) != cudaSuccess) return e;
        if ((e = cudaStreamWaitEvent(sa, side->fork, 0)) != cudaSuccess) return e;
    }
    GdnArgs g = {};
    g.q = a.q; g.k = a.k; g.v = a.v; g.a = a.a; g.b = a.b;
    g.o = nullptr;
    g.B = a.B; g.Hg = a.H; g.Htot = a.H; g.h0 = 0; g.L = a.L; g.d = D; g.chunk = C;
    g.S0 = a.S0;
    g.ws = (char *)a.ws + bwd_f32_bytes(p.BH, a.L);
    g.ws_bytes = gdn_rowmajor_bytes(p.BH, a.L, D, C, true);
    g.err = a.err;
    g.S_chunks = p.ws + O_S0;
    g.S_chunk_stride = CHUNK_FLOATS;
    const cudaError_t es = launch_gdn_bf16_bwd_states(g, a.dO, a.dS_final, p.ws + O_DSC, a.dS0, sa, sb,
                                                      side ? side->mid : nullptr);
    e = set_gemm_smem<__nv_bfloat16>();
    if (e == cudaSuccess) {
        gdn_bwd_prep<__nv_bfloat16><<<dim3((unsigned)nch, (unsigned)p.BH), THREADS,
                                      gemm_smem_bytes<__nv_bfloat16>(), s>>>(p), note_launch();
        e = cudaGetLastError();
    }
    if (side) {
        // join whatever was enqueued on the side streams, also after a failed launch
        cudaEventRecord(side->join_a, sa);
        cudaEventRecord(side->join_b, sb);
        cudaStreamWaitEvent(s, side->join_a, 0);
        cudaStreamWaitEvent(s, side->join_b, 0);
    }
    if (es != cudaSuccess) return es;
    if (e != cudaSuccess) return e;
    gdn_bwd_grad<__nv_bfloat16><<<dim3((unsigned)nch, (unsigned)p.BH), THREADS,
                                  gemm_smem_bytes<__nv_bfloat16>(), s>>>(p), note_launch();
    return cudaGetLastError();
}

}  // namespace hlta
