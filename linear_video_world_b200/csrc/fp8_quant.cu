// E4M3 quantisation of bf16 tensors [BH][L][128] for the FP8 window attention.
//
// OCP 8-bit floating point, E4M3 encoding (bias 7, largest finite 448, subnormals below
// 2^-6). One fp32 scale per block: amax = largest |x| of the block (x minus an optional
// per-channel shift), code = E4M3 nearest to x * (448 / amax) (round to nearest even,
// saturating), scale = amax / 448. The three fp32 operations are single IEEE roundings
// (__fdiv_rn, __fmul_rn), so the codes are reproducible bit for bit.
//
// Row blocks: each head is cut into frames of frame_rows rows and each frame into runs of
// block_rows rows (the last run of a frame, and the last frame, may be short): the attention
// kernel takes Q in 128-row blocks of the whole head and K in 64-key runs of each frame (two
// runs per 128-key tile).
// Value channels: one scale per (head, channel) over all rows.
//
// HBM-bound: 2 bytes read and 1 byte written per element (the row kernel holds its block in
// registers between the max and the conversion; the channel path reads x twice).
#include "hlta_internal.cuh"

namespace hlta {
namespace {

constexpr int D = 128;
constexpr int QTHREADS = 256;       // 16 threads per row (8 channels each), 16 rows per pass
constexpr int MAX_PASSES = 8;       // row blocks of up to 128 rows
constexpr int CH_ROWS = 256;        // rows per CTA of the per-channel kernels

__device__ __forceinline__ uint32_t e4m3x4(float p0, float p1, float p2, float p3)
{
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(r)
        : "f"(p0), "f"(p1), "f"(p2), "f"(p3));
    return r;
}

__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8])
{
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void store8(uint8_t *p, const float (&v)[8], float inv)
{
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = __fmul_rn(v[i], inv);
    *reinterpret_cast<uint2 *>(p) = make_uint2(e4m3x4(y[0], y[1], y[2], y[3]), e4m3x4(y[4], y[5], y[6], y[7]));
}

__device__ __forceinline__ float block_max(float m, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int i = 1; i < QTHREADS / 32; ++i) m = fmaxf(m, red[i]);
    return m;
}

// one CTA per block (head, frame, run)
__global__ void __launch_bounds__(QTHREADS)
fp8_rows_kernel(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ shift, long L,
                long frame_rows, int block_rows, int nf, int nb, uint8_t *__restrict__ x8,
                float *__restrict__ scales)
{
    __shared__ float red[QTHREADS / 32];
    const long blk = blockIdx.x;
    const long bh = blk / ((long)nf * nb);
    const int f = (int)((blk / nb) % nf), j = (int)(blk % nb);
    const long fr0 = (long)f * frame_rows, fr1 = min(fr0 + frame_rows, L);
    const long r0 = fr0 + (long)j * block_rows;
    const int nr = r0 >= fr1 ? 0 : (int)min((long)block_rows, fr1 - r0);
    const int tr = threadIdx.x >> 4, tc = (threadIdx.x & 15) * 8;
    float sh[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) sh[i] = shift ? __ldg(shift + bh * D + tc + i) : 0.f;
    const __nv_bfloat16 *xb = x + (bh * L + r0) * D + tc;
    float v[MAX_PASSES][8];
    float amax = 0.f;
#pragma unroll
    for (int ps = 0; ps < MAX_PASSES; ++ps) {
        const int row = ps * 16 + tr;
        if (row < nr) {
            load8(xb + (long)row * D, v[ps]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                v[ps][i] = __fsub_rn(v[ps][i], sh[i]);
                amax = fmaxf(amax, fabsf(v[ps][i]));
            }
        }
    }
    amax = block_max(amax, red);
    const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
    uint8_t *ob = x8 + (bh * L + r0) * D + tc;
#pragma unroll
    for (int ps = 0; ps < MAX_PASSES; ++ps) {
        const int row = ps * 16 + tr;
        if (row < nr) store8(ob + (long)row * D, v[ps], inv);
    }
    if (threadIdx.x == 0) scales[blk] = __fdiv_rn(amax, 448.f);
}

// per-channel maxima of CH_ROWS rows, merged into amax_bits[bh][128] (non-negative floats
// order like their bit patterns, so an integer atomic max is exact and order-independent)
__global__ void __launch_bounds__(QTHREADS)
fp8_channel_max_kernel(const __nv_bfloat16 *__restrict__ x, long L, unsigned int *amax_bits)
{
    __shared__ float part[16][D];
    const long bh = blockIdx.y;
    const long rb = (long)blockIdx.x * CH_ROWS;
    const int tr = threadIdx.x >> 4, tc = (threadIdx.x & 15) * 8;
    float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const long rend = min(rb + CH_ROWS, L);
    for (long row = rb + tr; row < rend; row += 16) {
        float v[8];
        load8(x + (bh * L + row) * D + tc, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], fabsf(v[i]));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) part[tr][tc + i] = m[i];
    __syncthreads();
    if (threadIdx.x < D) {
        float mm = 0.f;
#pragma unroll
        for (int t = 0; t < 16; ++t) mm = fmaxf(mm, part[t][threadIdx.x]);
        atomicMax(amax_bits + bh * D + threadIdx.x, __float_as_uint(mm));
    }
}

__global__ void __launch_bounds__(QTHREADS)
fp8_channel_quant_kernel(const __nv_bfloat16 *__restrict__ x, long L,
                         const unsigned int *__restrict__ amax_bits, uint8_t *__restrict__ x8)
{
    const long bh = blockIdx.y;
    const long rb = (long)blockIdx.x * CH_ROWS;
    const int tr = threadIdx.x >> 4, tc = (threadIdx.x & 15) * 8;
    float inv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float a = __uint_as_float(amax_bits[bh * D + tc + i]);
        inv[i] = a > 0.f ? __fdiv_rn(448.f, a) : 0.f;
    }
    const long rend = min(rb + CH_ROWS, L);
    for (long row = rb + tr; row < rend; row += 16) {
        float v[8];
        load8(x + (bh * L + row) * D + tc, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], inv[i]);
        *reinterpret_cast<uint2 *>(x8 + (bh * L + row) * D + tc) =
            make_uint2(e4m3x4(v[0], v[1], v[2], v[3]), e4m3x4(v[4], v[5], v[6], v[7]));
    }
}

// amax bits -> scale = amax / 448, in place
__global__ void fp8_channel_scale_kernel(float *scales, long n)
{
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) scales[i] = __fdiv_rn(__uint_as_float(reinterpret_cast<unsigned int *>(scales)[i]), 448.f);
}

}  // namespace

cudaError_t launch_fp8_quantize_rows(const void *x, const float *shift, long BH, long L,
                                     long frame_rows, int block_rows, void *x8, float *scales,
                                     cudaStream_t s)
{
    if (block_rows < 1 || block_rows > 16 * MAX_PASSES || frame_rows < 1) return cudaErrorNotSupported;
    const long nf = (L + frame_rows - 1) / frame_rows;
    const long nb = (frame_rows + block_rows - 1) / block_rows;
    const long blocks = BH * nf * nb;
    if (blocks == 0) return cudaSuccess;
    if (blocks >= (1L << 31) || nf >= (1L << 31) || nb >= (1L << 31)) return cudaErrorNotSupported;
    fp8_rows_kernel<<<(unsigned)blocks, QTHREADS, 0, s>>>((const __nv_bfloat16 *)x, shift, L,
                                                         frame_rows, block_rows, (int)nf, (int)nb,
                                                         (uint8_t *)x8, scales), note_launch();
    return cudaGetLastError();
}

cudaError_t launch_fp8_quantize_channels(const void *x, long BH, long L, void *x8,
                                         float *scales, cudaStream_t s)
{
    if (BH == 0) return cudaSuccess;
    if (BH > 65535) return cudaErrorNotSupported;
    cudaError_t e = cudaMemsetAsync(scales, 0, (size_t)BH * D * sizeof(float), s);
    if (e != cudaSuccess) return e;
    if (L > 0) {
        const dim3 grid((unsigned)((L + CH_ROWS - 1) / CH_ROWS), (unsigned)BH);
        fp8_channel_max_kernel<<<grid, QTHREADS, 0, s>>>((const __nv_bfloat16 *)x, L, (unsigned int *)scales), note_launch();
        fp8_channel_quant_kernel<<<grid, QTHREADS, 0, s>>>((const __nv_bfloat16 *)x, L, (const unsigned int *)scales,
                                                           (uint8_t *)x8), note_launch();
    }
    const long n = BH * D;
    fp8_channel_scale_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(scales, n), note_launch();
    return cudaGetLastError();
}

}  // namespace hlta
