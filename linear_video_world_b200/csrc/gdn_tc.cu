// Gated delta rule, chunkwise form, bf16 in / bf16 out, fp32 accumulation and fp32 state.
//
// Chunk algebra (derived from S_t = a_t S_{t-1}(I - b_t k_t k_t^T) + b_t v_t k_t^T; the
// chunkwise split is the "parallel within a block, recurrent across blocks" form of the
// llm-atlas long-context explainer, sections 06 and 09). For a chunk of n <= 64 tokens with
// incoming state S0 and g_t = sum_{s<=t} log a_s within the chunk (the kernels carry g in
// log2 units, so e^{g_t - g_i} is a single 2^x):
//   A_ti = b_t e^{g_t-g_i} k_t.k_i (i < t),    T = (I + A)^{-1}          (UT transform)
//   W  = T diag(b e^g) K,  Up = T diag(b) V,   P_ti = e^{g_t-g_i} q_t.k_i (i <= t)
//   Op = P Up,  Qt = diag(e^g) Q - P W,  Kt = diag(e^{g_n-g}) K,  gam = e^{g_n}
//   U = Up - W S0^T,   O = Op + Qt S0^T,   S_n = gam S0 + U^T Kt.
// Only decays e^{g_t-g_i} with t >= i are formed, so nothing overflows.
//
// Two kernels:
//   prep   one CTA per (chunk, head), every chunk in parallel: Q, K, V of the chunk arrive
//          by TMA as 128B-swizzled boxes; KK^T, QK^T, T in 32 x 32 blocks (fp32: forward
//          substitution of the diagonal blocks, a column per thread, then two block products),
//          then W, Up, Op, Qt on mma.sync bf16 tensor cores;
//          writes W, Qt, Kt, and Up, Op transposed (bf16), and gam (fp32) to the workspace.
//   state  serial over the chunks of a head; the 128 state rows are split into 16-row blocks
//          (rows of S evolve independently), one warp per block, four per CTA, two CTAs per
//          head. A warp keeps its rows of S in registers over all key columns, in the layout
//          of m16n8k16 accumulator tiles, which is also the A-operand layout of the next
//          product: per chunk S [Qt; W]^T, then S <- gam S + U Kt with U taken straight from
//          the first product's accumulators, without a round trip through shared memory.
//          A producer warp streams the chunk operands in by TMA through a 3-stage ring
//          (stage release counted over the four state warps); waits are bounded
//          (DEVERR_GDN_WAIT).
// The serial chain is latency-bound (two dependent 64x16x128-class products per chunk), so
// it uses register-resident warp MMAs rather than a TMEM round trip per dependent step.
// These kernels serve the backward pass (its recomputed chunk preparation, the chunk start
// states, and the state-gradient pass built the same way); the forward runs the tcgen05
// chunk preparation of gdn_prep_tc.cu and the segment scan of gdn_scan.cu.
#include "hlta_internal.cuh"
#include "sm100_ptx.cuh"

#include <math.h>

namespace hlta {
namespace {

constexpr int C = 64;             // chunk length
constexpr int D = 128;            // head dim
constexpr int SC = C + 8;         // padded smem row stride of [.][64] bf16 tiles
constexpr int AP = C + 4;         // fp32 row stride of A: 16-byte aligned rows

using ptx::smem_u32;
using ptx::sw128_off;

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// d += a * b (m16n8k16, bf16 operands, fp32 accumulate)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragment (16x16) of a row-major [M][K] bf16 tile with row stride `ld` (elements)
__device__ __forceinline__ void frag_a(uint32_t (&r)[4], const __nv_bfloat16 *base, int ld, int m0,
                                       int k0, int lane)
{
    const int q = lane >> 3, rr = lane & 7;
    ldsm_x4(r, smem_u32(base + (m0 + (q & 1) * 8 + rr) * ld + k0 + (q >> 1) * 8));
}

// Fragment loaders on a [64][128] bf16 tile in the 128B-swizzled two-half layout
// (byte offsets from ptx::sw128_off); every ldmatrix row address is one 16-byte chunk.
__device__ __forceinline__ void frag_a_sw(uint32_t (&r)[4], const uint8_t *tile, int m0, int k0, int lane)
{
    const int q = lane >> 3, rr = lane & 7;
    ldsm_x4(r, smem_u32(tile + sw128_off(m0 + (q & 1) * 8 + rr, k0 + (q >> 1) * 8, C)));
}
__device__ __forceinline__ void frag_b_nk_sw(uint32_t (&r)[4], const uint8_t *tile, int n0, int k0, int lane)
{
    ldsm_x4(r, smem_u32(tile + sw128_off(n0 + (lane >> 4) * 8 + (lane & 7), k0 + ((lane >> 3) & 1) * 8, C)));
}
__device__ __forceinline__ void frag_b_kn_sw(uint32_t (&r)[4], const uint8_t *tile, int k0, int n0, int lane)
{
    ldsm_x4_t(r, smem_u32(tile + sw128_off(k0 + ((lane >> 3) & 1) * 8 + (lane & 7), n0 + (lane >> 4) * 8, C)));
}

__device__ __forceinline__ float fast_lg2(float x)
{
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float fast_ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log2 of the decay gate a of a token: from a itself, or with raw inputs from x as
// log2 exp(-c softplus(x)) = -c softplus(x) / ln 2 (softplus(x) = log(1 + e^x), taken as x
// itself where e^-x is below float resolution)
__device__ __forceinline__ float log2_gate(const GdnArgs &p, float v)
{
    if (!p.raw) return fast_lg2(v);
    const float sp = v > 20.f ? v : log1pf(__expf(v));
    return -p.raw_c * sp * 1.4426950408889634f;
}
// the write strength b of a token: b itself, or with raw inputs sigmoid(y)
__device__ __forceinline__ float beta_gate(const GdnArgs &p, float v)
{
    return p.raw ? 1.f / (1.f + __expf(-v)) : v;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}


// -----------------------------------------------------------------------------------------
// prep
// -----------------------------------------------------------------------------------------
constexpr int PREP_THREADS = 256;
constexpr uint32_t SWT = C * D * 2;        // one swizzled [64][128] bf16 tile: 16 KB

// Shared memory of the prep kernel (about 92 KB: two CTAs per SM). Q, K, V arrive by TMA as
// swizzled tiles; regions are reused once their contents are dead:
//   R1: A (fp32 [64][68]) -> T (in place) -> T1, T2 (bf16 [64][72] each) -> Op (swizzled tile)
//   R2: W (swizzled tile)
//   V:  V -> Up          Q:  Q -> Qt (in place)
// T = (I + A)^{-1} is formed over A in place (fp32) before T1, T2 replace both.
struct PrepSmem {
    alignas(1024) uint8_t Q[SWT];
    alignas(1024) uint8_t K[SWT];
    alignas(1024) uint8_t V[SWT];
    alignas(1024) uint8_t R2[SWT];
    alignas(16) uint8_t R1[2 * C * SC * 2];
    __nv_bfloat16 P[C * SC];
    float g[C], eg[C], ek[C], bb[C];
    alignas(8) uint64_t bar;
    int abort_flag;
};
static_assert(sizeof(float) * C * AP <= 2 * C * SC * 2, "A must fit in R1");
static_assert(SWT <= 2 * C * SC * 2, "Op must fit in R1");

// One warp's 16 rows x (NT*8) columns of X = Am ([64][lda] row-major, padded) times a
// swizzled [K][N] tile, k-steps 0 .. ksteps-1, columns n0 ...
template <int NT>
__device__ __forceinline__ void gemm_rows_kn(float (&acc)[NT][4], const __nv_bfloat16 *Am, int lda,
                                             const uint8_t *Bt, int m0, int n0, int ksteps, int lane)
{
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
        acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    for (int kk = 0; kk < ksteps; ++kk) {
        uint32_t a[4];
        frag_a(a, Am, lda, m0, kk * 16, lane);
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
            uint32_t b[4];
            frag_b_kn_sw(b, Bt, kk * 16, n0 + np * 16, lane);
            mma16816(acc[2 * np], a, b[0], b[1]);
            mma16816(acc[2 * np + 1], a, b[2], b[3]);
        }
    }
}

// accumulator fragment -> swizzled bf16 tile
template <int NT>
__device__ __forceinline__ void store_acc_sw(uint8_t *tile, const float (&acc)[NT][4], int m0, int n0,
                                             int lane)
{
    const int g8 = lane >> 2, tg = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int c = n0 + nt * 8 + 2 * tg;
        *reinterpret_cast<uint32_t *>(tile + sw128_off(m0 + g8, c, C)) = pack2(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<uint32_t *>(tile + sw128_off(m0 + g8 + 8, c, C)) = pack2(acc[nt][2], acc[nt][3]);
    }
}

struct PrepMaps {
    CUtensorMap q, k, v;          // [B*Htot*L][128] bf16, boxes 64 rows x 64 columns, swizzled
};

__global__ void __launch_bounds__(PREP_THREADS, 2)
gdn_prep_bf16(const __grid_constant__ PrepMaps maps, GdnArgs p, GdnWorkspace ws)
{
    extern __shared__ uint8_t smem_raw[];
    PrepSmem &s = *reinterpret_cast<PrepSmem *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float *A = reinterpret_cast<float *>(s.R1);            // [64][68]
    __nv_bfloat16 *T1 = reinterpret_cast<__nv_bfloat16 *>(s.R1);
    __nv_bfloat16 *T2 = T1 + C * SC;
    uint8_t *Op = s.R1;
    uint8_t *W = s.R2;

    const int chunk = blockIdx.x, bh = blockIdx.y;
    const int b = bh / p.Hg, h = bh % p.Hg;
    const long nch = gdn_num_chunks(p.L, C);
    const long t0 = (long)chunk * C;
    const int n = (int)min((long)C, p.L - t0);
    const long head = (long)(b * p.Htot + p.h0 + h) * p.L;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g8 = lane >> 2, tg = lane & 3;
    const int rb = warp & 3, ch = warp >> 2;               // 16-row block, column half
    const int m0 = rb * 16;
    const uint32_t bar = smem_u32(&s.bar);

    // ---- Q, K, V of the chunk by TMA (two 64-column boxes each)
    if (tid == 0) {
        s.abort_flag = 0;
        ptx::mbar_init(bar, 1);
        ptx::mbar_init_fence();
        ptx::mbar_expect_tx(bar, 3 * SWT);
        const int row = (int)(head + t0);
        for (int hf = 0; hf < 2; ++hf) {
            ptx::tma_load_2d(smem_u32(s.Q + hf * (SWT / 2)), &maps.q, hf * 64, row, bar);
            ptx::tma_load_2d(smem_u32(s.K + hf * (SWT / 2)), &maps.k, hf * 64, row, bar);
            ptx::tma_load_2d(smem_u32(s.V + hf * (SWT / 2)), &maps.v, hf * 64, row, bar);
        }
    }
    if (warp == 1) {
        // inclusive prefix sum of log2 a over 64 entries (decays are then 2^(g_t - g_i), one
        // ex2 each): two per lane, then a warp scan
        const int t = 2 * lane;
        const float l0 = t < n ? log2_gate(p, p.a[(long)bh * p.L + t0 + t]) : 0.f;
        const float l1 = t + 1 < n ? log2_gate(p, p.a[(long)bh * p.L + t0 + t + 1]) : 0.f;
        float pair = l0 + l1, x = pair;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        s.g[t] = x - pair + l0;
        s.g[t + 1] = x;
        s.bb[t] = t < n ? beta_gate(p, p.b[(long)bh * p.L + t0 + t]) : 0.f;
        s.bb[t + 1] = t + 1 < n ? beta_gate(p, p.b[(long)bh * p.L + t0 + t + 1]) : 0.f;
    }
    __syncthreads();                                       // barrier initialised, g, bb ready
    if (tid < C) {
        const float gn = s.g[n - 1];
        s.eg[tid] = tid < n ? fast_ex2(s.g[tid]) : 0.f;
        s.ek[tid] = tid < n ? fast_ex2(gn - s.g[tid]) : 0.f;
    }
    const bool landed = ptx::mbar_wait(bar, 0, (volatile int *)&s.abort_flag, p.err, DEVERR_GDN_WAIT);
    if (!__syncthreads_and(landed)) {
        // a bounded wait expired: give the three copies a last bounded chance to land
        if (tid == 0) {
            const long long t0 = clock64();
            while (!ptx::mbar_try(bar, 0) && clock64() - t0 < (1LL << 31)) {}
        }
        return;
    }
    // a ragged last chunk: the box rows past the chunk belong to the next head (or are past
    // the tensor); zero them so no stray value reaches a product
    if (n < C) {
        for (int e = tid; e < (C - n) * 16; e += PREP_THREADS) {
            const int t = n + (e >> 4), cc = e & 15;
            const uint32_t off = (cc >> 3) * (SWT / 2) + t * 128 + (cc & 7) * 16;
            *reinterpret_cast<uint4 *>(s.Q + off) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(s.K + off) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(s.V + off) = make_uint4(0, 0, 0, 0);
        }
        __syncthreads();
    }
    // raw inputs: scale the staged q and k of every token to unit L2 norm (two threads per
    // row, 64 columns each; rows of zeros stay zero)
    if (p.raw) {
        const int row = tid >> 1, half = tid & 1;          // rows 0..63: Q, 64..127: K
        uint8_t *tile = row < C ? s.Q : s.K;
        const int t = row & (C - 1);
        float ss = 0.f;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
            const uint4 u = *reinterpret_cast<const uint4 *>(tile + sw128_off(t, (half * 8 + c8) * 8, C));
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
            }
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        const float sc = ss > 0.f ? rsqrtf(ss) : 0.f;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
            uint4 *pu = reinterpret_cast<uint4 *>(tile + sw128_off(t, (half * 8 + c8) * 8, C));
            uint4 u = *pu;
            __nv_bfloat162 *h2 = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                h2[e] = __floats2bfloat162_rn(f.x * sc, f.y * sc);
            }
            *pu = u;
        }
        __syncthreads();
    }

    // ---- KK^T and QK^T: this warp's 16 rows, 32 columns; columns above the diagonal block
    //      are zero and not computed
    {
        const int n0 = ch * 32;
        const bool live = n0 <= m0 + 15;
        float kk[4][4], qk[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) kk[nt][e] = qk[nt][e] = 0.f;
        if (live) {
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t ak[4], aq[4];
                frag_a_sw(ak, s.K, m0, ks * 16, lane);
                frag_a_sw(aq, s.Q, m0, ks * 16, lane);
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    uint32_t bk[4];
                    frag_b_nk_sw(bk, s.K, n0 + np * 16, ks * 16, lane);
                    mma16816(kk[2 * np], ak, bk[0], bk[1]);
                    mma16816(kk[2 * np + 1], ak, bk[2], bk[3]);
                    mma16816(qk[2 * np], aq, bk[0], bk[1]);
                    mma16816(qk[2 * np + 1], aq, bk[2], bk[3]);
                }
            }
        }
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = m0 + g8 + (e >> 1) * 8;
                const int i = n0 + nt * 8 + 2 * tg + (e & 1);
                const bool lower = i <= t && t < n;
                const float dec = lower ? fast_ex2(s.g[t] - s.g[i]) : 0.f;
                A[t * AP + i] = (i < t && t < n) ? s.bb[t] * dec * kk[nt][e] : 0.f;
                s.P[t * SC + i] = __float2bfloat16_rn(lower ? dec * qk[nt][e] : 0.f);
            }
        }
    }
    __syncthreads();

    // ---- T = (I + A)^{-1} (A strictly lower triangular, so T is unit lower triangular), in
    //      two levels of 32 x 32 blocks, written over A in place:
    //        T00 = (I + A00)^-1, T11 = (I + A11)^-1  forward substitution, a column per thread
    //                                               (T_tj = -sum_{i<t} A_ti T_ij inside a block)
    //        T10 = -T11 A10 T00                     two 32 x 32 products, four columns a thread
    //      (T01 = 0 = A01). Then T1 = T diag(b e^g) and T2 = T diag(b) in bf16 over R1.
    {
        if (tid < C) {
            const int base = (tid >> 5) * 32, jj = tid & 31;
            float tc[32];
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                const float *ar = A + (base + t) * AP + base;
                const float4 *ar4 = reinterpret_cast<const float4 *>(ar);
#pragma unroll
                for (int i4 = 0; i4 < t / 4; ++i4) {
                    const float4 av = ar4[i4];
                    a0 = fmaf(av.x, tc[4 * i4], a0);
                    a1 = fmaf(av.y, tc[4 * i4 + 1], a1);
                    a2 = fmaf(av.z, tc[4 * i4 + 2], a2);
                    a3 = fmaf(av.w, tc[4 * i4 + 3], a3);
                }
#pragma unroll
                for (int i = (t / 4) * 4; i < t; ++i) a0 = fmaf(ar[i], tc[i], a0);
                tc[t] = t < jj ? 0.f : (t == jj ? 1.f : -((a0 + a1) + (a2 + a3)));
            }
            __syncwarp();
            // every column of this block is in registers once all threads of the block (one
            // warp) are here: the diagonal block of A is dead
#pragma unroll
            for (int t = 0; t < 32; ++t) A[(base + t) * AP + base + jj] = tc[t];
        }
        __syncthreads();
        const int r = tid >> 3, c4 = (tid & 7) * 4;         // a row of the 32 x 32 block, 4 columns
        float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {                   // Y = A10 T00
            const float a = A[(32 + r) * AP + kk];
            const float4 t4 = *reinterpret_cast<const float4 *>(A + kk * AP + c4);
            y.x = fmaf(a, t4.x, y.x); y.y = fmaf(a, t4.y, y.y);
            y.z = fmaf(a, t4.z, y.z); y.w = fmaf(a, t4.w, y.w);
        }
        __syncthreads();                                    // A10 is read: Y takes its place
        *reinterpret_cast<float4 *>(A + (32 + r) * AP + c4) = y;
        __syncthreads();
        float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {                   // T10 = -T11 Y
            const float tk = A[(32 + r) * AP + 32 + kk];
            const float4 y4 = *reinterpret_cast<const float4 *>(A + (32 + kk) * AP + c4);
            z.x = fmaf(-tk, y4.x, z.x); z.y = fmaf(-tk, y4.y, z.y);
            z.z = fmaf(-tk, y4.z, z.z); z.w = fmaf(-tk, y4.w, z.w);
        }
        __syncthreads();
        *reinterpret_cast<float4 *>(A + (32 + r) * AP + c4) = z;
        __syncthreads();
        float tcol[C];
        if (tid < C)
#pragma unroll
            for (int t = 0; t < C; ++t) tcol[t] = A[t * AP + tid];
        __syncthreads();                                   // T is in registers: A is dead
        if (tid < C) {
            const int j = tid;
            const float s1 = s.bb[j] * s.eg[j], s2 = s.bb[j];
#pragma unroll
            for (int t = 0; t < C; ++t) {
                T1[t * SC + j] = __float2bfloat16_rn(tcol[t] * s1);
                T2[t * SC + j] = __float2bfloat16_rn(tcol[t] * s2);
            }
        }
        __syncthreads();
    }

    // ---- W = T1 K, Up = T2 V (lower-triangular T: k-steps 0 .. rb)
    const int nc0 = ch * 64;
    {
        float w[8][4], u[8][4];
        gemm_rows_kn<8>(w, T1, SC, s.K, m0, nc0, rb + 1, lane);
        gemm_rows_kn<8>(u, T2, SC, s.V, m0, nc0, rb + 1, lane);
        __syncthreads();                                   // T, T1, T2 and V are dead now
        store_acc_sw<8>(W, w, m0, nc0, lane);
        store_acc_sw<8>(s.V, u, m0, nc0, lane);
    }
    __syncthreads();
    // ---- Op = P Up (into R1), Qt = diag(e^g) Q - P W (in place over Q)
    {
        float op[8][4], pw[8][4];
        gemm_rows_kn<8>(op, s.P, SC, s.V, m0, nc0, rb + 1, lane);
        gemm_rows_kn<8>(pw, s.P, SC, W, m0, nc0, rb + 1, lane);
        store_acc_sw<8>(Op, op, m0, nc0, lane);
        const int ta = m0 + g8, tb = ta + 8;
        const float ea = s.eg[ta], eb = s.eg[tb];          // zero for rows >= n
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int c = nc0 + nt * 8 + 2 * tg;
            uint32_t *qa = reinterpret_cast<uint32_t *>(s.Q + sw128_off(ta, c, C));
            uint32_t *qb = reinterpret_cast<uint32_t *>(s.Q + sw128_off(tb, c, C));
            const float2 fa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(qa));
            const float2 fb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(qb));
            *qa = pack2(ta < n ? ea * fa.x - pw[nt][0] : 0.f, ta < n ? ea * fa.y - pw[nt][1] : 0.f);
            *qb = pack2(tb < n ? eb * fb.x - pw[nt][2] : 0.f, tb < n ? eb * fb.y - pw[nt][3] : 0.f);
        }
    }
    __syncthreads();

    // ---- write W, Qt, Kt (row-major [64 t][128] per chunk), Up and Op transposed
    //      ([128 i][64 t] per chunk: the state pass reads them in its accumulator layout, state
    //      row i by token t) and gam
    const long base = ((long)bh * nch + chunk) * C * D;
    uint4 *oW = reinterpret_cast<uint4 *>((__nv_bfloat16 *)ws.W + base);
    uint4 *oU = reinterpret_cast<uint4 *>((__nv_bfloat16 *)ws.Up + base);
    uint4 *oO = reinterpret_cast<uint4 *>((__nv_bfloat16 *)ws.Op + base);
    uint4 *oQ = reinterpret_cast<uint4 *>((__nv_bfloat16 *)ws.Qt + base);
    uint4 *oK = reinterpret_cast<uint4 *>((__nv_bfloat16 *)ws.Kt + base);
    for (int e = tid; e < D * (C / 8); e += PREP_THREADS) {
        // lanes run over the state row i (consecutive 2-byte columns of the staged tiles),
        // each gathering 8 consecutive tokens
        const int i = e & (D - 1), t8 = e >> 7;
        uint32_t up[4], op[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int t = t8 * 8 + 2 * u;
            const uint16_t u0 = *reinterpret_cast<const uint16_t *>(s.V + sw128_off(t, i, C));
            const uint16_t u1 = *reinterpret_cast<const uint16_t *>(s.V + sw128_off(t + 1, i, C));
            const uint16_t o0 = *reinterpret_cast<const uint16_t *>(Op + sw128_off(t, i, C));
            const uint16_t o1 = *reinterpret_cast<const uint16_t *>(Op + sw128_off(t + 1, i, C));
            up[u] = (uint32_t)u0 | ((uint32_t)u1 << 16);
            op[u] = (uint32_t)o0 | ((uint32_t)o1 << 16);
        }
        oU[i * (C / 8) + t8] = make_uint4(up[0], up[1], up[2], up[3]);
        oO[i * (C / 8) + t8] = make_uint4(op[0], op[1], op[2], op[3]);
    }
    for (int e = tid; e < C * (D / 8); e += PREP_THREADS) {
        const int t = e >> 4, c8 = e & 15;
        const uint32_t so = sw128_off(t, c8 * 8, C);
        oW[e] = *reinterpret_cast<const uint4 *>(W + so);
        oQ[e] = *reinterpret_cast<const uint4 *>(s.Q + so);
        const float dk = s.ek[t];
        uint4 kv = *reinterpret_cast<const uint4 *>(s.K + so);
        __nv_bfloat162 *k2 = reinterpret_cast<__nv_bfloat162 *>(&kv);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float2 f = __bfloat1622float2(k2[u]);
            k2[u] = __floats2bfloat162_rn(f.x * dk, f.y * dk);
        }
        oK[e] = kv;
    }
    if (tid < 4) ws.gam[((long)bh * nch + chunk) * 4 + tid] = tid == 0 ? fast_ex2(s.g[n - 1]) : 0.f;
}

// -----------------------------------------------------------------------------------------
// state pass
// -----------------------------------------------------------------------------------------
// Two CTAs per head, four warps each; a warp owns 16 rows i of the state S (rows evolve
// independently) and keeps them in registers as m16n8k16 accumulator tiles over all 128 key
// columns j. Per chunk, with U, O, D laid out state row by token:
//   D = S [W; Qt]^T   (A operand: S itself, repacked to bf16 pairs; B: the W and Qt tiles)
//   O = Op^T + D_Qt,  U = Up^T - D_W
//   S <- gam S + U Kt  (A operand: U, repacked straight from D's accumulator tiles; B: Kt)
// An m16n8 accumulator tile holds rows (g, g+8) and column pairs (2t, 2t+1) of each lane,
// which is exactly the A fragment of the next m16n8k16 product over those columns, so
// neither S nor U goes through shared memory. The chunk operands (swizzled W, Qt, Kt tiles,
// the CTA's 64 rows of Up^T and Op^T, gam) stream in by TMA through a 3-stage mbarrier ring,
// two chunks ahead; outputs leave through a double-buffered shared staging tile.
constexpr int NSTAGE = 3;                  // chunk operand buffers of the state pass
constexpr int SWARPS = 4;                  // state warps per CTA, 16 state rows each
constexpr int STATE_THREADS = (SWARPS + 1) * 32;   // plus one TMA producer warp
constexpr int CW = SWARPS * 16;            // state rows per CTA: 64
constexpr uint32_t SLICE = CW * C * 2;     // the CTA's rows of Up^T or Op^T: [64 i][64 t], 8 KB
constexpr uint32_t STAGE_TX = 3 * SWT + 2 * SLICE + 16;
constexpr int OSI = 16 + 8;                // staging row stride of a warp's [64 t][16 i] outputs

struct StateBuf {
    alignas(1024) uint8_t W[SWT];          // W  [64 t][128 j], two 128B-swizzled halves
    alignas(1024) uint8_t Q[SWT];          // Qt
    alignas(1024) uint8_t K[SWT];          // Kt
    alignas(1024) uint8_t U[SLICE];        // Up^T rows of this CTA [64 i][64 t], 128B swizzle
    alignas(1024) uint8_t O[SLICE];        // Op^T rows of this CTA
    alignas(16) float gam[4];              // gam of the chunk (element 0)
};
struct StateSmem {
    StateBuf buf[NSTAGE];
    alignas(16) __nv_bfloat16 Ost[SWARPS][C * OSI];   // per warp: its outputs of a chunk, [t][i]
    alignas(8) uint64_t full[NSTAGE];
    alignas(8) uint64_t empty[NSTAGE];     // every warp is done with the stage (count SWARPS)
    int abort_flag;
};

struct StateMaps {
    CUtensorMap W, Q, K;                   // [BHg*nch*64][128]: 64x64 swizzled boxes
    CUtensorMap U, O;                      // [BHg*nch*128][64]: 64x64 swizzled boxes
};

__device__ __forceinline__ void issue_chunk(StateSmem &s, const StateMaps &maps, const GdnWorkspace &ws,
                                            int bh, long nch, long c, int c0)
{
    StateBuf &bf = s.buf[c % NSTAGE];
    const uint32_t bar = smem_u32(&s.full[c % NSTAGE]);
    ptx::mbar_expect_tx(bar, STAGE_TX);
    const int row = (int)(((long)bh * nch + c) * C);
    for (int hf = 0; hf < 2; ++hf) {
        ptx::tma_load_2d(smem_u32(bf.W + hf * (SWT / 2)), &maps.W, hf * 64, row, bar);
        ptx::tma_load_2d(smem_u32(bf.Q + hf * (SWT / 2)), &maps.Q, hf * 64, row, bar);
        ptx::tma_load_2d(smem_u32(bf.K + hf * (SWT / 2)), &maps.K, hf * 64, row, bar);
    }
    const int trow = (int)(((long)bh * nch + c) * D + c0);
    ptx::tma_load_2d(smem_u32(bf.U), &maps.U, 0, trow, bar);
    ptx::tma_load_2d(smem_u32(bf.O), &maps.O, 0, trow, bar);
    ptx::bulk_load(smem_u32(bf.gam), ws.gam + ((long)bh * nch + c) * 4, 16, bar);
}

__device__ __forceinline__ uint32_t pack_acc(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// four 8x8 bf16 matrices from the accumulator-fragment layout (lane: row lane/4, column pair
// lane%4) stored transposed; lanes 8k..8k+7 give the 16-byte row addresses of matrix k
__device__ __forceinline__ void stsm_x4_t(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3)
{
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};"
                 ::"r"(addr), "r"(r0), "r"(r1), "r"(r2), "r"(r3) : "memory");
}

// DQ[nt] = S Qt^T and DW[nt] = S W^T (nt < 8: tokens 8nt..8nt+7) for this warp's 16 rows, in
// one pass over the key columns: each A fragment of S is packed to bf16 once for both
__device__ __forceinline__ void state_times_tiles(float (&dq)[8][4], float (&dw)[8][4], const float (&st)[16][4],
                                                  const uint8_t *qt, const uint8_t *wt, int lane)
{
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) dq[nt][e] = dw[nt][e] = 0.f;
#pragma unroll
    for (int kb = 0; kb < D / 16; ++kb) {
        uint32_t a[4];
        a[0] = pack_acc(st[2 * kb][0], st[2 * kb][1]);
        a[1] = pack_acc(st[2 * kb][2], st[2 * kb][3]);
        a[2] = pack_acc(st[2 * kb + 1][0], st[2 * kb + 1][1]);
        a[3] = pack_acc(st[2 * kb + 1][2], st[2 * kb + 1][3]);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
            uint32_t bq[4], bw[4];
            frag_b_nk_sw(bq, qt, np * 16, kb * 16, lane);     // tile rows = tokens (n), cols = j (k)
            frag_b_nk_sw(bw, wt, np * 16, kb * 16, lane);
            mma16816(dq[2 * np], a, bq[0], bq[1]);
            mma16816(dq[2 * np + 1], a, bq[2], bq[3]);
            mma16816(dw[2 * np], a, bw[0], bw[1]);
            mma16816(dw[2 * np + 1], a, bw[2], bw[3]);
        }
    }
}

// a warp's 16 state rows (accumulator tiles over the 128 key columns) to a row-major
// [128][128] fp32 matrix at `dst` (rows i0 .. i0 + 15)
__device__ __forceinline__ void store_rows(float *dst, const float (&st)[16][4], int i0, int lane)
{
    const int g8 = lane >> 2, tg = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
            *reinterpret_cast<float2 *>(dst + (long)(i0 + g8 + hh * 8) * D + nt * 8 + 2 * tg) =
                make_float2(st[nt][2 * hh], st[nt][2 * hh + 1]);
}

__global__ void __launch_bounds__(STATE_THREADS, 1)
gdn_state_bf16(const __grid_constant__ StateMaps maps, GdnArgs p, GdnWorkspace ws)
{
    extern __shared__ uint8_t smem_raw[];
    StateSmem &s = *reinterpret_cast<StateSmem *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int bh = blockIdx.y;
    const int b = bh / p.Hg, h = bh % p.Hg;
    const long nch = gdn_num_chunks(p.L, C);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g8 = lane >> 2, tg = lane & 3;
    const int c0 = blockIdx.x * CW;                        // first state row of this CTA
    const int r0 = warp * 16;                              // first row of this warp in the CTA
    __nv_bfloat16 *o = (__nv_bfloat16 *)p.o + (long)(b * p.Htot + p.h0 + h) * p.L * D;

    if (tid == 0) {
        for (int i = 0; i < NSTAGE; ++i) {
            ptx::mbar_init(smem_u32(&s.full[i]), 1);
            ptx::mbar_init(smem_u32(&s.empty[i]), SWARPS);
        }
        s.abort_flag = 0;
        ptx::mbar_init_fence();
    }
    volatile int *abort_flag = (volatile int *)&s.abort_flag;
    if (warp == SWARPS) {
        // ------------------------------ TMA producer --------------------------------------
        // chunk c goes into stage c % NSTAGE once every state warp released chunk c - NSTAGE
        __syncthreads();
        if (lane == 0) {
            long c = 0;
            for (; c < nch; ++c) {
                if (c >= NSTAGE) {
                    const uint32_t eb = smem_u32(&s.empty[c % NSTAGE]);
                    const uint32_t ep = (uint32_t)((c - NSTAGE) / NSTAGE) & 1u;
                    if (!(ptx::mbar_try(eb, ep) || ptx::mbar_wait(eb, ep, abort_flag, p.err, DEVERR_GDN_WAIT))) break;
                }
                issue_chunk(s, maps, ws, bh, nch, c, c0);
            }
            if (*abort_flag) {
                // a bounded wait expired somewhere: let the copies this CTA issued land before
                // it exits (the last NSTAGE chunks issued, each on its own stage and phase)
                const long long tw = clock64();
                for (long cc = c - 1; cc >= 0 && cc >= c - NSTAGE; --cc) {
                    const uint32_t bar = smem_u32(&s.full[cc % NSTAGE]);
                    while (!ptx::mbar_try(bar, (uint32_t)(cc / NSTAGE) & 1u) && clock64() - tw < (1LL << 31)) {}
                }
            }
        }
        return;
    }
    // the state rows of this warp: st[nt] holds (i = g8, g8 + 8) x (j = 8 nt + 2 tg, +1)
    float st[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = c0 + r0 + g8 + (e >> 1) * 8;
            const int j = nt * 8 + 2 * tg + (e & 1);
            st[nt][e] = p.S0 ? p.S0[((long)bh * D + i) * D + j] : 0.f;
        }
    __syncthreads();

    // this warp's outputs of a chunk: staged transposed ([t][i], stmatrix) and written out as
    // 32-byte runs of its 16 state rows per token
    __nv_bfloat16 *stage = s.Ost[warp];
    const uint32_t stage_a = smem_u32(stage);

    for (long c = 0; c < nch; ++c) {
        if (p.S_chunks) store_rows(p.S_chunks + ((long)bh * nch + c) * p.S_chunk_stride, st, c0 + r0, lane);
        StateBuf &cur = s.buf[c % NSTAGE];
        const uint32_t fb = smem_u32(&s.full[c % NSTAGE]), fp = (uint32_t)(c / NSTAGE) & 1u;
        if (!__all_sync(0xffffffffu, ptx::mbar_try(fb, fp) || ptx::mbar_wait(fb, fp, abort_flag, p.err, DEVERR_GDN_WAIT)))
            return;                                        // the producer waits for its copies
        const float gam = cur.gam[0];
        const long t0 = c * C;
        float dq[8][4], dw[8][4];
        state_times_tiles(dq, dw, st, cur.Q, cur.W, lane);
        // O = Op^T + S Qt^T (old S); skipped when only the chunk states are wanted
        if (p.o) {
            uint32_t ov[8][2];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int il = r0 + g8 + hh * 8, t = nt * 8 + 2 * tg;
                    const float2 of = __bfloat1622float2(
                        *reinterpret_cast<const __nv_bfloat162 *>(cur.O + ptx::sw128_off(il, t, CW)));
                    ov[nt][hh] = pack_acc(of.x + dq[nt][2 * hh], of.y + dq[nt][2 * hh + 1]);
                }
            __syncwarp();                                  // the previous chunk's run reads are done
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                // matrices (rows i 0-7 | 8-15) x (tokens 16np .. +7 | +8 .. +15)
                const int k = lane >> 3, r = lane & 7;
                const int t = np * 16 + (k >> 1) * 8 + r, ib = (k & 1) * 8;
                stsm_x4_t(stage_a + (uint32_t)(t * OSI + ib) * 2u, ov[2 * np][0], ov[2 * np][1],
                          ov[2 * np + 1][0], ov[2 * np + 1][1]);
            }
            __syncwarp();
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int t = u * 32 + lane;
                if (t0 + t < p.L) {
                    const uint4 *srow = reinterpret_cast<const uint4 *>(stage + t * OSI);
                    uint4 *drow = reinterpret_cast<uint4 *>(o + (t0 + t) * D + c0 + r0);
                    drow[0] = srow[0];
                    drow[1] = srow[1];
                }
            }
        }
        // U = Up^T - S W^T, as the A fragments of the update product
        uint32_t ua[4][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int il = r0 + g8 + hh * 8, t = nt * 8 + 2 * tg;
                const float2 uf = __bfloat1622float2(
                    *reinterpret_cast<const __nv_bfloat162 *>(cur.U + ptx::sw128_off(il, t, CW)));
                ua[nt >> 1][(nt & 1) * 2 + hh] = pack_acc(uf.x - dw[nt][2 * hh], uf.y - dw[nt][2 * hh + 1]);
            }
        // S <- gam S + U Kt
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) st[nt][e] *= gam;
#pragma unroll
        for (int kb = 0; kb < C / 16; ++kb) {
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t bk[4];
                frag_b_kn_sw(bk, cur.K, kb * 16, np * 16, lane);      // Kt rows = tokens (k), cols = j (n)
                mma16816(st[2 * np], ua[kb], bk[0], bk[1]);
                mma16816(st[2 * np + 1], ua[kb], bk[2], bk[3]);
            }
        }
        // this warp no longer reads the stage (its shared loads have completed: their values
        // fed the products above)
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(smem_u32(&s.empty[c % NSTAGE]));
    }
    if (p.S_out)
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = c0 + r0 + g8 + (e >> 1) * 8;
                const int j = nt * 8 + 2 * tg + (e & 1);
                p.S_out[((long)bh * D + i) * D + j] = st[nt][e];
            }
}

// -----------------------------------------------------------------------------------------
// backward state pass (training)
// -----------------------------------------------------------------------------------------
// The state gradient carried from the last chunk to the first. With S_end = gam S + U^T Kt,
// U = Up - W S^T and O = Op + Qt S^T, the gradient of the chunk's start state S is
//   dS = gam dS_end - (dS_end Kt^T) W + dO^T Qt.
// Rows i of dS evolve independently, so the layout is the forward pass's: two CTAs per head,
// four warps of 16 rows each, kept in registers as accumulator tiles over the key columns j.
// Per chunk (last to first): X = dS_end Kt^T (A operand: dS_end repacked to bf16; B: Kt),
// then dS = gam dS_end + [-X | dO^T] [W; Qt] (A operands: -X straight from X's accumulator
// tiles, dO^T by transposing ldmatrix from the chunk's dO rows; B: W, Qt). Each chunk's
// end-state gradient is stored before the chunk is processed.
struct DStateBuf {
    alignas(1024) uint8_t W[SWT];          // W  [64 t][128 j]
    alignas(1024) uint8_t Q[SWT];          // Qt
    alignas(1024) uint8_t K[SWT];          // Kt
    alignas(1024) uint8_t G[SLICE];        // dO [64 t][64 i] on this CTA's state rows
    alignas(16) float gam[4];
};
struct DStateSmem {
    DStateBuf buf[NSTAGE];
    alignas(8) uint64_t full[NSTAGE];
    alignas(8) uint64_t empty[NSTAGE];     // count SWARPS
    int abort_flag;
};
constexpr uint32_t DSTAGE_TX = 3 * SWT + SLICE + 16;

struct DStateMaps {
    CUtensorMap W, Q, K;                   // [BHg*nch*64][128]: 64x64 swizzled boxes
    CUtensorMap G;                         // dO [B*Htot*L][128]: 64x64 swizzled boxes
};

// A fragment (16 rows x 16 k) of A = B^T from a swizzled tile holding B row-major ([k][m]):
// four transposed 8x8 matrices (m 0-7 | 8-15) x (k 0-7 | 8-15)
__device__ __forceinline__ void frag_a_t_sw(uint32_t (&r)[4], const uint8_t *tile, int m0, int k0, int lane)
{
    const int q = lane >> 3;
    ldsm_x4_t(r, smem_u32(tile + sw128_off(k0 + (q >> 1) * 8 + (lane & 7), m0 + (q & 1) * 8, C)));
}

// the k-th chunk processed (chunk c = nch - 1 - k) into stage k % NSTAGE
__device__ __forceinline__ void issue_dchunk(DStateSmem &s, const DStateMaps &maps, const GdnWorkspace &ws,
                                             int bh, long nch, long c, long k, long g_row, int c0)
{
    DStateBuf &bf = s.buf[k % NSTAGE];
    const uint32_t bar = smem_u32(&s.full[k % NSTAGE]);
    ptx::mbar_expect_tx(bar, DSTAGE_TX);
    const int row = (int)(((long)bh * nch + c) * C);
    for (int hf = 0; hf < 2; ++hf) {
        ptx::tma_load_2d(smem_u32(bf.W + hf * (SWT / 2)), &maps.W, hf * 64, row, bar);
        ptx::tma_load_2d(smem_u32(bf.Q + hf * (SWT / 2)), &maps.Q, hf * 64, row, bar);
        ptx::tma_load_2d(smem_u32(bf.K + hf * (SWT / 2)), &maps.K, hf * 64, row, bar);
    }
    ptx::tma_load_2d(smem_u32(bf.G), &maps.G, c0, (int)(g_row + c * C), bar);
    ptx::bulk_load(smem_u32(bf.gam), ws.gam + ((long)bh * nch + c) * 4, 16, bar);
}

__global__ void __launch_bounds__(STATE_THREADS, 1)
gdn_dstate_bf16(const __grid_constant__ DStateMaps maps, GdnArgs p, GdnWorkspace ws,
                const float *dS_final, float *dS_chunks, float *dS0)
{
    extern __shared__ uint8_t smem_raw[];
    DStateSmem &s = *reinterpret_cast<DStateSmem *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int bh = blockIdx.y;
    const int b = bh / p.Hg, h = bh % p.Hg;
    const long nch = gdn_num_chunks(p.L, C);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g8 = lane >> 2, tg = lane & 3;
    const int c0 = blockIdx.x * CW;
    const int r0 = warp * 16;

    if (tid == 0) {
        for (int i = 0; i < NSTAGE; ++i) {
            ptx::mbar_init(smem_u32(&s.full[i]), 1);
            ptx::mbar_init(smem_u32(&s.empty[i]), SWARPS);
        }
        s.abort_flag = 0;
        ptx::mbar_init_fence();
    }
    volatile int *abort_flag = (volatile int *)&s.abort_flag;
    if (warp == SWARPS) {
        // ------------------------------ TMA producer --------------------------------------
        __syncthreads();
        if (lane == 0) {
            const long g_row = (long)(b * p.Htot + p.h0 + h) * p.L;
            long k = 0;
            for (; k < nch; ++k) {
                if (k >= NSTAGE) {
                    const uint32_t eb = smem_u32(&s.empty[k % NSTAGE]);
                    const uint32_t ep = (uint32_t)((k - NSTAGE) / NSTAGE) & 1u;
                    if (!(ptx::mbar_try(eb, ep) || ptx::mbar_wait(eb, ep, abort_flag, p.err, DEVERR_GDN_WAIT))) break;
                }
                issue_dchunk(s, maps, ws, bh, nch, nch - 1 - k, k, g_row, c0);
            }
            if (*abort_flag) {
                const long long tw = clock64();
                for (long kk = k - 1; kk >= 0 && kk >= k - NSTAGE; --kk) {
                    const uint32_t bar = smem_u32(&s.full[kk % NSTAGE]);
                    while (!ptx::mbar_try(bar, (uint32_t)(kk / NSTAGE) & 1u) && clock64() - tw < (1LL << 31)) {}
                }
            }
        }
        return;
    }
    // this warp's rows of the state gradient: ds[nt] holds (i = g8, g8 + 8) x (j = 8 nt + 2 tg, +1)
    float ds[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = c0 + r0 + g8 + (e >> 1) * 8;
            const int j = nt * 8 + 2 * tg + (e & 1);
            ds[nt][e] = dS_final ? dS_final[((long)bh * D + i) * D + j] : 0.f;
        }
    __syncthreads();

    for (long k = 0; k < nch; ++k) {
        const long c = nch - 1 - k;
        if (dS_chunks) store_rows(dS_chunks + ((long)bh * nch + c) * p.S_chunk_stride, ds, c0 + r0, lane);
        DStateBuf &cur = s.buf[k % NSTAGE];
        const uint32_t fb = smem_u32(&s.full[k % NSTAGE]), fp = (uint32_t)(k / NSTAGE) & 1u;
        if (!__all_sync(0xffffffffu, ptx::mbar_try(fb, fp) || ptx::mbar_wait(fb, fp, abort_flag, p.err, DEVERR_GDN_WAIT)))
            return;                                        // the producer waits for its copies
        const float gam = cur.gam[0];
        // X = dS_end Kt^T (tokens 8 nt .. 8 nt + 7)
        float x[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) x[nt][e] = 0.f;
#pragma unroll
        for (int kb = 0; kb < D / 16; ++kb) {
            uint32_t a[4];
            a[0] = pack_acc(ds[2 * kb][0], ds[2 * kb][1]);
            a[1] = pack_acc(ds[2 * kb][2], ds[2 * kb][3]);
            a[2] = pack_acc(ds[2 * kb + 1][0], ds[2 * kb + 1][1]);
            a[3] = pack_acc(ds[2 * kb + 1][2], ds[2 * kb + 1][3]);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bk[4];
                frag_b_nk_sw(bk, cur.K, np * 16, kb * 16, lane);      // Kt rows = tokens (n), cols = j (k)
                mma16816(x[2 * np], a, bk[0], bk[1]);
                mma16816(x[2 * np + 1], a, bk[2], bk[3]);
            }
        }
        // -X as the A fragments of the update product (tokens as k)
        uint32_t xa[4][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                xa[nt >> 1][(nt & 1) * 2 + hh] = pack_acc(-x[nt][2 * hh], -x[nt][2 * hh + 1]);
        // dS = gam dS_end - X W + dO^T Qt
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) ds[nt][e] *= gam;
#pragma unroll
        for (int kb = 0; kb < C / 16; ++kb) {
            uint32_t ga[4];
            frag_a_t_sw(ga, cur.G, r0, kb * 16, lane);                 // dO^T: rows i, k = tokens
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t bw[4], bq[4];
                frag_b_kn_sw(bw, cur.W, kb * 16, np * 16, lane);      // rows = tokens (k), cols = j (n)
                frag_b_kn_sw(bq, cur.Q, kb * 16, np * 16, lane);
                mma16816(ds[2 * np], xa[kb], bw[0], bw[1]);
                mma16816(ds[2 * np + 1], xa[kb], bw[2], bw[3]);
                mma16816(ds[2 * np], ga, bq[0], bq[1]);
                mma16816(ds[2 * np + 1], ga, bq[2], bq[3]);
            }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(smem_u32(&s.empty[k % NSTAGE]));
    }
    if (dS0) store_rows(dS0 + (long)bh * D * D, ds, c0 + r0, lane);
}

}  // namespace

cudaError_t launch_gdn_bf16_bwd_states(const GdnArgs &g, const void *dO, const float *dS_final,
                                       float *dS_chunks, float *dS0, cudaStream_t s,
                                       cudaStream_t s2, cudaEvent_t mid)
{
    if (g.d != D || g.o != nullptr || !g.S_chunks) return cudaErrorNotSupported;
    const long nch = gdn_num_chunks(g.L, C);
    const long BH = (long)g.B * g.Hg;
    const long in_rows = (long)g.B * g.Htot * g.L;
    const long ws_rows = BH * nch * C;
    if (nch > 0x7fffffffL || in_rows + C >= (1L << 31) || ws_rows >= (1L << 31))
        return cudaErrorNotSupported;
    GdnWorkspace ws = gdn_workspace_carve(g.ws, BH, g.L, D, C, true);
    cudaError_t e;
    PrepMaps pm;
    if ((e = make_tmap_2d_bf16(&pm.q, g.q, in_rows, D, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&pm.k, g.k, in_rows, D, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&pm.v, g.v, in_rows, D, 64, C, true)) != cudaSuccess) return e;
    StateMaps sm;
    if ((e = make_tmap_2d_bf16(&sm.W, ws.W, ws_rows, D, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&sm.Q, ws.Qt, ws_rows, D, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&sm.K, ws.Kt, ws_rows, D, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&sm.U, ws.Up, ws_rows * 2, C, 64, CW, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&sm.O, ws.Op, ws_rows * 2, C, 64, CW, true)) != cudaSuccess) return e;
    DStateMaps dm;
    dm.W = sm.W;
    dm.Q = sm.Q;
    dm.K = sm.K;
    if ((e = make_tmap_2d_bf16(&dm.G, dO, in_rows, D, 64, C, true)) != cudaSuccess) return e;
    const size_t smem_prep = sizeof(PrepSmem) + 1024;
    const size_t smem_state = sizeof(StateSmem) + 1024;
    const size_t smem_dstate = sizeof(DStateSmem) + 1024;
    if ((e = cudaFuncSetAttribute(gdn_prep_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_prep)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(gdn_state_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_state)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(gdn_dstate_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dstate)) != cudaSuccess) return e;
    gdn_prep_bf16<<<dim3((unsigned)nch, (unsigned)BH), PREP_THREADS, smem_prep, s>>>(pm, g, ws), note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (s2 != s) {
        // the two state passes are independent of each other: side by side
        if ((e = cudaEventRecord(mid, s)) != cudaSuccess) return e;
        if ((e = cudaStreamWaitEvent(s2, mid, 0)) != cudaSuccess) return e;
    }
    gdn_dstate_bf16<<<dim3(D / CW, (unsigned)BH), STATE_THREADS, smem_dstate, s2>>>(dm, g, ws, dS_final, dS_chunks, dS0), note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    gdn_state_bf16<<<dim3(D / CW, (unsigned)BH), STATE_THREADS, smem_state, s>>>(sm, g, ws), note_launch();
    return cudaGetLastError();
}

}  // namespace hlta
