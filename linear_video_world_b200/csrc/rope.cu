// Rotary position embedding of the softmax heads' q and k, in place (the prologue of the
// SWA / DSWA branches): the pair (x_{2i}, x_{2i+1}) of a token at position p is rotated by
// p * base^(-2i/d) (llm-atlas long-context explainer, position-encoding section: RoPE turns
// position into a rotation of Q and K; Kairos gives it the local position, the related-papers
// analysis, row B1). p is the token's index inside its frame (pos_mode 0) or in the sequence
// (pos_mode 1); sign -1 applies the inverse rotation (the map of the gradient).
//
// One thread per (batch, token, pair): the angle is formed and reduced to [-pi, pi] in double
// precision (positions reach tens of thousands of radians), its sine and cosine taken once in
// single precision, and the rotation applied to that pair of every head in the range, q and
// k; the kernel is HBM-bound (each element read and written once). Rows of 16-byte multiples
// take the vector form below (one 16-byte chunk per thread); other d the pair form.
#include "hlta_internal.cuh"

#include <math.h>

namespace hlta {
namespace {

template <typename E> struct Pair;
template <> struct Pair<__nv_bfloat16> {
    using T = __nv_bfloat162;
    static __device__ __forceinline__ float2 ld(const T *p) { return __bfloat1622float2(*p); }
    static __device__ __forceinline__ void st(T *p, float2 v) { *p = __floats2bfloat162_rn(v.x, v.y); }
};
template <> struct Pair<float> {
    using T = float2;
    static __device__ __forceinline__ float2 ld(const T *p) { return *p; }
    static __device__ __forceinline__ void st(T *p, float2 v) { *p = v; }
};

template <typename E>
__global__ void __launch_bounds__(256)
rope_kernel(E *q, E *k, int Htot, int h0, int Hr, long L, int N, int d, double log2_base,
            int pos_mode, int sign, long total)
{
    using P = Pair<E>;
    const long gid = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= total) return;
    const int half = d >> 1;
    const int i = (int)(gid % half);
    const long bl = gid / half;
    const long l = bl % L, b = bl / L;
    const double p = pos_mode ? (double)l : (double)(l % N);
    const double two_pi = 6.283185307179586476925287;
    double ang = sign * p * exp2(-2.0 * i / d * log2_base);
    ang -= two_pi * rint(ang / two_pi);
    float s, c;
    sincosf((float)ang, &s, &c);
    for (int h = h0; h < h0 + Hr; ++h) {
        const long off = ((b * Htot + h) * L + l) * d + 2 * i;
        if (q) {
            typename P::T *pq = reinterpret_cast<typename P::T *>(q + off);
            const float2 x = P::ld(pq);
            P::st(pq, make_float2(x.x * c - x.y * s, x.x * s + x.y * c));
        }
        if (k) {
            typename P::T *pk = reinterpret_cast<typename P::T *>(k + off);
            const float2 x = P::ld(pk);
            P::st(pk, make_float2(x.x * c - x.y * s, x.x * s + x.y * c));
        }
    }
}

// The same with one 16-byte chunk per thread (V pairs: 4 in bf16, 2 in fp32) when d is a
// multiple of the chunk: a warp then moves 512 contiguous bytes per head and tensor, and the
// head loop is unrolled so several heads' loads are in flight at once.
template <typename E>
__global__ void __launch_bounds__(256)
rope_kernel_v(E *__restrict__ q, E *__restrict__ k, int Htot, int h0, int Hr, long L, int N, int d,
              double log2_base, int pos_mode, int sign, long total)
{
    constexpr int V = 16 / (2 * (int)sizeof(E));          // pairs per 16-byte chunk
    const long gid = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= total) return;
    const int chunks = d / (2 * V);
    const int ch = (int)(gid % chunks);
    const long bl = gid / chunks;
    const long l = bl % L, b = bl / L;
    const double p = pos_mode ? (double)l : (double)(l % N);
    const double two_pi = 6.283185307179586476925287;
    float cs[V], sn[V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const int i = ch * V + j;
        double ang = sign * p * exp2(-2.0 * i / d * log2_base);
        ang -= two_pi * rint(ang / two_pi);
        sincosf((float)ang, &sn[j], &cs[j]);
    }
    auto rot = [&](E *base) {
        uint4 *ptr = reinterpret_cast<uint4 *>(base);
        uint4 u = *ptr;
        if constexpr (sizeof(E) == 2) {
            __nv_bfloat162 *h2 = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const float2 x = __bfloat1622float2(h2[j]);
                h2[j] = __floats2bfloat162_rn(x.x * cs[j] - x.y * sn[j], x.x * sn[j] + x.y * cs[j]);
            }
        } else {
            float2 *f2 = reinterpret_cast<float2 *>(&u);
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const float2 x = f2[j];
                f2[j] = make_float2(x.x * cs[j] - x.y * sn[j], x.x * sn[j] + x.y * cs[j]);
            }
        }
        *ptr = u;
    };
#pragma unroll 4
    for (int h = h0; h < h0 + Hr; ++h) {
        const long off = ((b * Htot + h) * L + l) * d + ch * 2 * V;
        if (q) rot(q + off);
        if (k) rot(k + off);
    }
}

}  // namespace

cudaError_t launch_rope(void *q, void *k, bool bf16, int B, int Htot, int h0, int Hr, long L,
                        int N, int d, double base, int pos_mode, int sign, cudaStream_t s)
{
    const long total = (long)B * L * (d / 2);
    if (total == 0 || Hr == 0 || (!q && !k)) return cudaSuccess;
    const long blocks = (total + 255) / 256;
    if (blocks > 0x7fffffffL) return cudaErrorNotSupported;
    const double lb = log2(base);
    const int per16 = bf16 ? 8 : 4;                       // elements per 16-byte chunk
    if (d % per16 == 0) {
        const long tv = (long)B * L * (d / per16);
        const unsigned bv = (unsigned)((tv + 255) / 256);
        if (bf16)
            rope_kernel_v<__nv_bfloat16><<<bv, 256, 0, s>>>((__nv_bfloat16 *)q, (__nv_bfloat16 *)k, Htot, h0,
                                                            Hr, L, N, d, lb, pos_mode, sign, tv), note_launch();
        else
            rope_kernel_v<float><<<bv, 256, 0, s>>>((float *)q, (float *)k, Htot, h0, Hr, L, N, d, lb,
                                                    pos_mode, sign, tv), note_launch();
        return cudaGetLastError();
    }
    if (bf16)
        rope_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
            (__nv_bfloat16 *)q, (__nv_bfloat16 *)k, Htot, h0, Hr, L, N, d, lb, pos_mode, sign, total), note_launch();
    else
        rope_kernel<float><<<(unsigned)blocks, 256, 0, s>>>((float *)q, (float *)k, Htot, h0, Hr, L, N,
                                                            d, lb, pos_mode, sign, total), note_launch();
    return cudaGetLastError();
}

}  // namespace hlta
