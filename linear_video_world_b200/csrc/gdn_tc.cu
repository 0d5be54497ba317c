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
//          by TMA as 128B-swizzled boxes; KK^T, QK^T, the blocked inversion for T (fp32),
//          then W, Up, Op, Qt on mma.sync bf16 tensor cores; writes W, Up, Op, Qt, Kt (bf16)
//          and gam (fp32) to the workspace.
//   state  serial over the chunks of a head; the 128 state rows are split into 16-row blocks
//          (rows of S evolve independently), four blocks per CTA, two CTAs per head. A
//          block's state lives in registers as the accumulator fragments of the S update;
//          each chunk does two dependent small GEMMs ([W;Qt] S^T, then U^T Kt) on mma.sync.
//          The chunk operands (swizzled W/Qt/Kt boxes, the CTA's 64 columns of Up/Op, gam)
//          stream in by TMA through a 3-stage mbarrier ring shared by the four blocks, two
//          chunks ahead; waits are bounded (DEVERR_GDN_WAIT).
// The serial chain is latency-bound (two dependent 64x16x128-class products per chunk), so
// it uses register-resident warp MMAs rather than a TMEM round trip per dependent step.
#include "hlta_internal.cuh"
#include "sm100_ptx.cuh"

#include <math.h>

namespace hlta {
namespace {

constexpr int C = 64;             // chunk length
constexpr int D = 128;            // head dim
constexpr int SD = D + 8;         // padded smem row stride (elements) of [.][128] bf16 tiles
constexpr int SC = C + 8;         // padded smem row stride of [.][64] bf16 tiles
constexpr int AP = C + 4;         // fp32 row stride of A: 16-byte aligned rows
constexpr int THREADS = 128;
constexpr int RB = 16;            // state rows per CTA in the state pass

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

// B fragments of two adjacent n-tiles (k16 x n16) from a [N][K] row-major tile:
// r[0], r[1] = n-tile n0, r[2], r[3] = n-tile n0 + 8
__device__ __forceinline__ void frag_b_nk(uint32_t (&r)[4], const __nv_bfloat16 *base, int ld,
                                          int n0, int k0, int lane)
{
    ldsm_x4(r, smem_u32(base + (n0 + (lane >> 4) * 8 + (lane & 7)) * ld + k0 + ((lane >> 3) & 1) * 8));
}

// The same four loaders on a [64][128] bf16 tile in the 128B-swizzled two-half layout
// (byte offsets from ptx::sw128_off); every ldmatrix row address is one 16-byte chunk.
__device__ __forceinline__ void frag_a_sw(uint32_t (&r)[4], const uint8_t *tile, int m0, int k0, int lane)
{
    const int q = lane >> 3, rr = lane & 7;
    ldsm_x4(r, smem_u32(tile + sw128_off(m0 + (q & 1) * 8 + rr, k0 + (q >> 1) * 8, C)));
}
__device__ __forceinline__ void frag_a_t_sw(uint32_t (&r)[4], const uint8_t *tile, int m0, int k0, int lane)
{
    const int q = lane >> 3, rr = lane & 7;
    ldsm_x4_t(r, smem_u32(tile + sw128_off(k0 + (q >> 1) * 8 + rr, m0 + (q & 1) * 8, C)));
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
//   R1: A (fp32 [64][68]) -> T1, T2 (bf16 [64][72] each) -> Op (swizzled tile)
//   R2: W (swizzled tile)
//   V:  V -> Up          Q:  Q -> Qt (in place)
// T = (I + A)^{-1} itself never reaches shared memory: its columns live in registers.
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

    // ---- T = (I + A)^{-1} (A strictly lower triangular, so T is unit lower triangular) by
    //      forward substitution, one column per thread held in registers:
    //      T_tj = -sum_{i<t} A_ti T_ij (T_tj = 0 above the diagonal, 1 on it), the row of A
    //      read as float4 broadcasts and summed in four partial sums. Then T1 = T diag(b e^g)
    //      and T2 = T diag(b) in bf16, written over A once every column is done.
    {
        float tc[C];
        if (tid < C) {
            const int j = tid;
#pragma unroll
            for (int t = 0; t < C; ++t) {
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                const float4 *ar = reinterpret_cast<const float4 *>(A + t * AP);
#pragma unroll
                for (int i4 = 0; i4 < t / 4; ++i4) {
                    const float4 av = ar[i4];
                    a0 = fmaf(av.x, tc[4 * i4], a0);
                    a1 = fmaf(av.y, tc[4 * i4 + 1], a1);
                    a2 = fmaf(av.z, tc[4 * i4 + 2], a2);
                    a3 = fmaf(av.w, tc[4 * i4 + 3], a3);
                }
#pragma unroll
                for (int i = (t / 4) * 4; i < t; ++i) a0 = fmaf(A[t * AP + i], tc[i], a0);
                const float acc = (a0 + a1) + (a2 + a3);
                tc[t] = t < j ? 0.f : (t == j ? 1.f : -acc);
            }
        }
        __syncthreads();                                   // every column done: A is dead
        if (tid < C) {
            const int j = tid;
            const float s1 = s.bb[j] * s.eg[j], s2 = s.bb[j];
#pragma unroll
            for (int t = 0; t < C; ++t) {
                T1[t * SC + j] = __float2bfloat16_rn(tc[t] * s1);
                T2[t * SC + j] = __float2bfloat16_rn(tc[t] * s2);
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

    // ---- write W, Up, Op, Qt, Kt (row-major [64][128] per chunk) and gam
    const long base = ((long)bh * nch + chunk) * C * D;
    uint4 *oW = reinterpret_cast<uint4 *>((__nv_bfloat16 *)ws.W + base);
    uint4 *oU = reinterpret_cast<uint4 *>((__nv_bfloat16 *)ws.Up + base);
    uint4 *oO = reinterpret_cast<uint4 *>((__nv_bfloat16 *)ws.Op + base);
    uint4 *oQ = reinterpret_cast<uint4 *>((__nv_bfloat16 *)ws.Qt + base);
    uint4 *oK = reinterpret_cast<uint4 *>((__nv_bfloat16 *)ws.Kt + base);
    for (int e = tid; e < C * (D / 8); e += PREP_THREADS) {
        const int t = e >> 4, c8 = e & 15;
        const uint32_t so = sw128_off(t, c8 * 8, C);
        oW[e] = *reinterpret_cast<const uint4 *>(W + so);
        oU[e] = *reinterpret_cast<const uint4 *>(s.V + so);
        oO[e] = *reinterpret_cast<const uint4 *>(Op + so);
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
// Two CTAs per head; each CTA holds four 16-row blocks of the state (one group of four warps
// per block) that share one ring of chunk operands, so a head occupies two SMs.
constexpr int NSTAGE = 3;                  // chunk operand buffers of the state pass
constexpr int GROUPS = 4;                  // 16-row blocks per CTA
constexpr int STATE_THREADS = GROUPS * THREADS;
constexpr int CW = GROUPS * RB;            // state rows (= Up/Op columns) per CTA: 64
constexpr uint32_t SLICE = C * CW * 2;     // the CTA's 64 columns of Up or Op: 8 KB
constexpr uint32_t STAGE_TX = 3 * SWT + 2 * SLICE + 16;

struct StateBuf {
    alignas(1024) uint8_t W[SWT];
    alignas(1024) uint8_t Q[SWT];          // Qt
    alignas(1024) uint8_t K[SWT];          // Kt
    alignas(128) __nv_bfloat16 U[C * CW];  // Up[:, c0:c0+64], row-major [64][64]
    alignas(128) __nv_bfloat16 O[C * CW];  // Op[:, c0:c0+64]
    alignas(16) float gam[4];              // gam of the chunk (element 0)
};
struct StateGroup {
    __nv_bfloat16 Sb[RB * SD];             // state slice as bf16 [i][j]
    __nv_bfloat16 Ut[RB * SC];             // U^T slice [i][t]
};
struct StateSmem {
    StateBuf buf[NSTAGE];
    StateGroup grp[GROUPS];
    alignas(8) uint64_t full[NSTAGE];
    int abort_flag;
};

struct StateMaps {
    CUtensorMap W, Q, K;                   // workspace [BHg*nch*64][128]: 64x64 swizzled boxes
    CUtensorMap U, O;                      // workspace [BHg*nch*64][128]: 64 rows x 64 columns
};

__device__ __forceinline__ void issue_chunk(StateSmem &s, const StateMaps &maps, const GdnWorkspace &ws,
                                            int bh, long nch, long c, int c0)
{
    StateBuf &bf = s.buf[c % NSTAGE];
    const uint32_t bar = smem_u32(&s.full[c % NSTAGE]);
    const int row = (int)(((long)bh * nch + c) * C);
    ptx::mbar_expect_tx(bar, STAGE_TX);
    for (int hf = 0; hf < 2; ++hf) {
        ptx::tma_load_2d(smem_u32(bf.W + hf * (SWT / 2)), &maps.W, hf * 64, row, bar);
        ptx::tma_load_2d(smem_u32(bf.Q + hf * (SWT / 2)), &maps.Q, hf * 64, row, bar);
        ptx::tma_load_2d(smem_u32(bf.K + hf * (SWT / 2)), &maps.K, hf * 64, row, bar);
    }
    ptx::tma_load_2d(smem_u32(bf.U), &maps.U, c0, row, bar);
    ptx::tma_load_2d(smem_u32(bf.O), &maps.O, c0, row, bar);
    ptx::bulk_load(smem_u32(bf.gam), ws.gam + ((long)bh * nch + c) * 4, 16, bar);
}

__device__ __forceinline__ void group_sync(int g)
{
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "r"(THREADS) : "memory");
}

__global__ void __launch_bounds__(STATE_THREADS, 1)
gdn_state_bf16(const __grid_constant__ StateMaps maps, GdnArgs p, GdnWorkspace ws)
{
    extern __shared__ uint8_t smem_raw[];
    StateSmem &s = *reinterpret_cast<StateSmem *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int bh = blockIdx.y;
    const int b = bh / p.Hg, h = bh % p.Hg;
    const long nch = gdn_num_chunks(p.L, C);
    const int tid = threadIdx.x, lane = tid & 31;
    const int g = tid / THREADS, warp = (tid / 32) % 4;    // row-block group, warp in group
    const int g8 = lane >> 2, tg = lane & 3;
    const int c0 = blockIdx.x * CW;                        // first state row of this CTA
    const int i0 = c0 + g * RB;                            // first state row of this group
    StateGroup &sg = s.grp[g];
    __nv_bfloat16 *o = (__nv_bfloat16 *)p.o + (long)(b * p.Htot + p.h0 + h) * p.L * D;

    if (tid == 0) {
        s.abort_flag = 0;
        for (int st = 0; st < NSTAGE; ++st) ptx::mbar_init(smem_u32(&s.full[st]), 1);
        ptx::mbar_init_fence();
    }
    // state fragments: this warp owns key columns j in [32w, 32w+32) of S^T = D[m=j][n=i]
    float st[2][2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = warp * 32 + mt * 16 + g8 + (e >> 1) * 8;
                const int i = nt * 8 + 2 * tg + (e & 1);
                st[mt][nt][e] = p.S0 ? p.S0[((long)bh * D + i0 + i) * D + j] : 0.f;
                sg.Sb[i * SD + j] = __float2bfloat16_rn(st[mt][nt][e]);
            }
    __syncthreads();
    if (tid == 0)
        for (long c = 0; c < NSTAGE - 1 && c < nch; ++c) issue_chunk(s, maps, ws, bh, nch, c, c0);

    bool ok = true;
    long c_fail = 0;
    for (long c = 0; c < nch; ++c) {
        StateBuf &cur = s.buf[c % NSTAGE];
        const bool landed = ptx::mbar_wait(smem_u32(&s.full[c % NSTAGE]), (uint32_t)(c / NSTAGE) & 1u,
                                           (volatile int *)&s.abort_flag, p.err, DEVERR_GDN_WAIT);
        // chunk c has landed for every thread; every group's Sb holds its incoming state
        if (!__syncthreads_and(landed)) { ok = false; c_fail = c; break; }
        // the stage of chunk c-1 is free again (every thread passed the barrier above)
        if (tid == 0 && c + NSTAGE - 1 < nch) issue_chunk(s, maps, ws, bh, nch, c + NSTAGE - 1, c0);
        const float gam = cur.gam[0];
        const long t0 = c * C;

        // GEMM 1: rows [W; Qt] (warps 0-1 of the group: W rows, warps 2-3: Qt rows) times S^T
        {
            const uint8_t *Am = warp < 2 ? cur.W : cur.Q;
            const int mb = (warp & 1) * 32;
            float acc[2][2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t bsf[4];
                frag_b_nk(bsf, sg.Sb, SD, 0, ks * 16, lane);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    uint32_t a[4];
                    frag_a_sw(a, Am, mb + mt * 16, ks * 16, lane);
                    mma16816(acc[mt][0], a, bsf[0], bsf[1]);
                    mma16816(acc[mt][1], a, bsf[2], bsf[3]);
                }
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int t = mb + mt * 16 + g8 + hh * 8;
                        const int i = nt * 8 + 2 * tg;
                        const float a0 = acc[mt][nt][2 * hh], a1 = acc[mt][nt][2 * hh + 1];
                        if (warp < 2) {
                            const float u0 = __bfloat162float(cur.U[t * CW + g * RB + i]) - a0;
                            const float u1 = __bfloat162float(cur.U[t * CW + g * RB + i + 1]) - a1;
                            sg.Ut[i * SC + t] = __float2bfloat16_rn(u0);
                            sg.Ut[(i + 1) * SC + t] = __float2bfloat16_rn(u1);
                        } else if (t0 + t < p.L) {
                            const float v0 = __bfloat162float(cur.O[t * CW + g * RB + i]) + a0;
                            const float v1 = __bfloat162float(cur.O[t * CW + g * RB + i + 1]) + a1;
                            *reinterpret_cast<uint32_t *>(o + (t0 + t) * D + i0 + i) = pack2(v0, v1);
                        }
                    }
        }
        group_sync(g);                         // this group's Ut is complete

        // GEMM 2: S^T <- gam S^T + Kt^T U   (D[m=j][n=i] = sum_t Kt[t][j] U[t][i])
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) st[mt][nt][e] *= gam;
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks) {
            uint32_t bu[4];
            frag_b_nk(bu, sg.Ut, SC, 0, ks * 16, lane);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                uint32_t a[4];
                frag_a_t_sw(a, cur.K, warp * 32 + mt * 16, ks * 16, lane);
                mma16816(st[mt][0], a, bu[0], bu[1]);
                mma16816(st[mt][1], a, bu[2], bu[3]);
            }
        }
        // bf16 copy of the new state for the next chunk's GEMM 1 (made visible by the
        // barrier at the top of the loop)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = warp * 32 + mt * 16 + g8 + (e >> 1) * 8;
                    const int i = nt * 8 + 2 * tg + (e & 1);
                    sg.Sb[i * SD + j] = __float2bfloat16_rn(st[mt][nt][e]);
                }
    }
    if (!ok) {
        // a bounded wait expired: let the copies this CTA issued and never consumed land
        // before it exits (chunks c .. issued-1, each on its own stage and phase)
        if (tid == 0) {
            const long long tw = clock64();
            for (long cc = c_fail; cc < c_fail + NSTAGE - 1 && cc < nch; ++cc) {
                const uint32_t bar = smem_u32(&s.full[cc % NSTAGE]);
                while (!ptx::mbar_try(bar, (uint32_t)(cc / NSTAGE) & 1u) && clock64() - tw < (1LL << 31)) {}
            }
        }
        return;
    }
    if (p.S_out) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = warp * 32 + mt * 16 + g8 + (e >> 1) * 8;
                    const int i = nt * 8 + 2 * tg + (e & 1);
                    p.S_out[((long)bh * D + i0 + i) * D + j] = st[mt][nt][e];
                }
    }
}

}  // namespace

cudaError_t launch_gdn_bf16(const GdnArgs &g, cudaStream_t s)
{
    if (g.d != D) return cudaErrorNotSupported;
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
    if ((e = make_tmap_2d_bf16(&sm.U, ws.Up, ws_rows, D, CW, C, false)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&sm.O, ws.Op, ws_rows, D, CW, C, false)) != cudaSuccess) return e;
    const size_t smem_prep = sizeof(PrepSmem) + 1024;
    const size_t smem_state = sizeof(StateSmem) + 1024;
    e = cudaFuncSetAttribute(gdn_prep_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_prep);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gdn_state_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_state);
    if (e != cudaSuccess) return e;
    gdn_prep_bf16<<<dim3((unsigned)nch, (unsigned)BH), PREP_THREADS, smem_prep, s>>>(pm, g, ws);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    gdn_state_bf16<<<dim3(D / CW, (unsigned)BH), STATE_THREADS, smem_state, s>>>(sm, g, ws);
    return cudaGetLastError();
}

}  // namespace hlta
