// Backward pass of the windowed softmax attention (SWA / DSWA), bf16 inputs, d = 128.
//
// With the forward's per-row log-sum-exp (natural log) lse_i, the weights are
// p_ij = exp(scale q_i.k_j - lse_i) over row i's window keys, and for the upstream gradient dO:
//   D_i = dO_i . o_i (= sum_j p_ij dP_ij),  dP_ij = dO_i . v_j,  dS_ij = p_ij (dP_ij - D_i),
//   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,  dv_j = sum_i p_ij dO_i
// (the reverse-mode derivative of exact attention; the llm-atlas long-context explainer, section
// 03, is the tiled forward this inverts). Three launches:
//   attn_bwd_dot   D per row (fp32 workspace)
//   attn_bwd_dq    one CTA per 64-row query tile of a frame: walks the key tiles of the row's
//                  window frames (as the forward), recomputes S and dP, accumulates dq
//   attn_bwd_dkv   one CTA per 64-key tile of a frame: walks the query tiles of the frames
//                  that see it (f = g + r i), recomputes S^T and dP^T, accumulates dk, dv
// Tiles are 64 rows because every row of a frame-local tile shares its window: the mask is
// only the ragged end of a frame. Products on mma.sync m16n8k16 (bf16 in, fp32 accumulate);
// each warp owns 16 rows of the tile it accumulates, so a product's accumulator fragments
// feed the next product as its A operand without leaving registers. K/V (dq) and Q/dO (dkv)
// tiles stream through a two-stage cp.async ring with a row-swizzled shared layout.
#include "hlta_internal.cuh"

namespace hlta {
namespace {

constexpr int D = 128;
constexpr int BT = 64;                          // rows per tile (query or key)
constexpr int THREADS = 128;                    // four warps, 16 rows each
constexpr uint32_t TILE = BT * D * 2;           // 16 KB

// [64][128] bf16 tile, 16-byte chunks XOR-swizzled with the row (conflict-free ldmatrix)
__device__ __forceinline__ uint32_t toff(int r, int chunk) { return (uint32_t)(r * 256 + ((chunk ^ (r & 7)) << 4)); }

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

// rows r0 .. r0+63 of a [rows][128] bf16 tensor; rows at or past rend read as zeros
__device__ __forceinline__ void load_tile(uint32_t dst, const __nv_bfloat16 *base, long r0, long rend)
{
    for (int i = threadIdx.x; i < BT * 16; i += THREADS) {
        const int r = i >> 4, c = i & 15;
        const long gr = r0 + r;
        const bool ok = gr < rend;
        const __nv_bfloat16 *src = base + (ok ? gr * D + c * 8 : 0);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst + toff(r, c)), "l"(src),
                     "r"(ok ? 16 : 0)
                     : "memory");
    }
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// C[16 x 64] = A[rows m0.., 128] . B[64 rows, 128]^T, A and B both row-major tiles (B's rows are
// the output columns): 8 k-steps x 8 n-tiles
__device__ __forceinline__ void gemm_abt(float (&c)[8][4], uint32_t sa, int m0, uint32_t sb)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
        c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(sa + toff(m0 + (lane & 15), 2 * kk + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
            const int mid = lane >> 3;
            uint32_t b0, b1, b2, b3;
            ldsm_x4(sb + toff(8 * (2 * np + (mid >> 1)) + (lane & 7), 2 * kk + (mid & 1)), b0, b1, b2, b3);
            mma16816(c[2 * np], a0, a1, a2, a3, b0, b1);
            mma16816(c[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
    }
}

// acc[16 x 128] += X[16 x 64] . B[64 rows, 128], X given as bf16 A fragments of four k-steps
// (the accumulator layout of a 16 x 64 product), B a row-major tile (k = its rows)
__device__ __forceinline__ void gemm_xb(float (&acc)[16][4], const uint32_t (&x)[4][4], uint32_t sb)
{
    const int lane = threadIdx.x & 31;
    const int mid = lane >> 3;
#pragma unroll
    for (int kk = 0; kk < BT / 16; ++kk) {
#pragma unroll
        for (int np = 0; np < 8; ++np) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(sb + toff(16 * kk + 8 * (mid & 1) + (lane & 7), 2 * np + (mid >> 1)), b0, b1, b2, b3);
            mma16816(acc[2 * np], x[kk][0], x[kk][1], x[kk][2], x[kk][3], b0, b1);
            mma16816(acc[2 * np + 1], x[kk][0], x[kk][1], x[kk][2], x[kk][3], b2, b3);
        }
    }
}

// bf16 A fragments (k-step kk = columns 16kk..16kk+15) of a 16 x 64 fp32 accumulator
__device__ __forceinline__ void to_afrag(const float (&c)[8][4], uint32_t (&x)[4][4])
{
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        x[kk][0] = pack2(c[2 * kk][0], c[2 * kk][1]);
        x[kk][1] = pack2(c[2 * kk][2], c[2 * kk][3]);
        x[kk][2] = pack2(c[2 * kk + 1][0], c[2 * kk + 1][1]);
        x[kk][3] = pack2(c[2 * kk + 1][2], c[2 * kk + 1][3]);
    }
}

__device__ __forceinline__ void store_rows(__nv_bfloat16 *dst, long r0, int nrows, int m0,
                                           const float (&acc)[16][4], float mul)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int rr = m0 + g + 8 * half;
        if (rr >= nrows) continue;
        __nv_bfloat16 *row = dst + (r0 + rr) * D;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
            *reinterpret_cast<uint32_t *>(row + 8 * nt + 2 * t) =
                pack2(acc[nt][2 * half] * mul, acc[nt][2 * half + 1] * mul);
    }
}

__device__ __forceinline__ bool frame_sees(int f, int g, int w, int r)
{
    const int dist = f - g;
    return dist >= 0 && dist <= r * (w - 1) && dist % r == 0;
}

// ----------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
attn_bwd_dot(const __nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ dO,
             float *__restrict__ Dws, long rows)
{
    const long row = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const uint2 a = *reinterpret_cast<const uint2 *>(o + row * D + 4 * lane);
    const uint2 b = *reinterpret_cast<const uint2 *>(dO + row * D + 4 * lane);
    const uint32_t aw[2] = {a.x, a.y}, bw[2] = {b.x, b.y};
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        s = fmaf(__uint_as_float(aw[i] << 16), __uint_as_float(bw[i] << 16), s);
        s = fmaf(__uint_as_float(aw[i] & 0xFFFF0000u), __uint_as_float(bw[i] & 0xFFFF0000u), s);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) Dws[row] = s;
}

struct BwdParams {
    const __nv_bfloat16 *q, *k, *v, *dO;
    const float *lse, *Dws;
    __nv_bfloat16 *dq, *dk, *dv;
    int T, N, w, r, tpf;
    float sl2, scale;
};

// ----------------------------------------------------------------------------------------
// dq: one CTA per (head, frame f, 64-row query tile u)
__global__ void __launch_bounds__(THREADS, 2)
attn_bwd_dq(const BwdParams p)
{
    extern __shared__ __align__(128) uint8_t sm[];
    const uint32_t sQ = smem_addr(sm), sdO = sQ + TILE, sK0 = sQ + 2 * TILE;   // K0 V0 K1 V1
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const long L = (long)p.T * p.N;
    const long bh = blockIdx.y;
    const int f = blockIdx.x / p.tpf, u = blockIdx.x % p.tpf;
    const long r0 = (long)f * p.N + (long)u * BT;
    const int nq = min(BT, p.N - u * BT);
    const __nv_bfloat16 *Qh = p.q + bh * L * D, *Kh = p.k + bh * L * D, *Vh = p.v + bh * L * D;
    const long fend = (long)(f + 1) * p.N;
    load_tile(sQ, Qh, r0, fend);
    load_tile(sdO, p.dO + bh * L * D, r0, fend);
    cp_commit();
    // per-row softmax constants of this thread's two rows (16w + g, +8)
    float lse2[2], Dr[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int rr = 16 * warp + g + 8 * hf;
        const bool ok = rr < nq;
        lse2[hf] = ok ? p.lse[bh * L + r0 + rr] * 1.4426950408889634f : INFINITY;
        Dr[hf] = ok ? p.Dws[bh * L + r0 + rr] : 0.f;
    }
    // key tiles: frames f - r i (i < w, >= 0) from the oldest, 64-key tiles of each
    const int nframes = min(p.w, f / p.r + 1);
    const int ntiles = nframes * p.tpf;
    auto tile_src = [&](int it, long &k0, int &nv) {
        const int fk = f - p.r * (nframes - 1 - it / p.tpf), jt = it % p.tpf;
        k0 = (long)fk * p.N + (long)jt * BT;
        nv = min(BT, p.N - jt * BT);
    };
    {
        long k0;
        int nv;
        tile_src(0, k0, nv);
        load_tile(sK0, Kh, k0, L);
        load_tile(sK0 + TILE, Vh, k0, L);
        cp_commit();
    }
    float acc[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    for (int it = 0; it < ntiles; ++it) {
        const uint32_t sK = sK0 + (uint32_t)(it & 1) * 2 * TILE, sV = sK + TILE;
        if (it + 1 < ntiles) {
            long k0;
            int nv;
            tile_src(it + 1, k0, nv);
            const uint32_t nK = sK0 + (uint32_t)((it + 1) & 1) * 2 * TILE;
            load_tile(nK, Kh, k0, L);
            load_tile(nK + TILE, Vh, k0, L);
        }
        cp_commit();
        cp_wait<1>();
        __syncthreads();
        long k0;
        int nv;
        tile_src(it, k0, nv);
        float s[8][4], dp[8][4];
        gemm_abt(s, sQ, 16 * warp, sK);
        gemm_abt(dp, sdO, 16 * warp, sV);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int col = 8 * nt + 2 * t + (e & 1), hf = e >> 1;
                const float pv = col < nv ? exp2f(fmaf(s[nt][e], p.sl2, -lse2[hf])) : 0.f;
                s[nt][e] = pv * (dp[nt][e] - Dr[hf]);           // dS
            }
        uint32_t x[4][4];
        to_afrag(s, x);
        gemm_xb(acc, x, sK);
        __syncthreads();                                        // before the ring slot is refilled
    }
    store_rows(p.dq + bh * L * D, r0, nq, 16 * warp, acc, p.scale);
}

// ----------------------------------------------------------------------------------------
// dk, dv: one CTA per (head, key frame g, 64-key tile jt)
__global__ void __launch_bounds__(THREADS, 2)
attn_bwd_dkv(const BwdParams p)
{
    extern __shared__ __align__(128) uint8_t sm[];
    const uint32_t sK = smem_addr(sm), sV = sK + TILE, sQ0 = sK + 2 * TILE;   // Q0 dO0 Q1 dO1
    float *sL = reinterpret_cast<float *>(sm + 6 * TILE);                      // [2][64] lse2
    float *sD = sL + 2 * BT;                                                   // [2][64] D
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const long L = (long)p.T * p.N;
    const long bh = blockIdx.y;
    const int gk = blockIdx.x / p.tpf, jt = blockIdx.x % p.tpf;
    const long k0 = (long)gk * p.N + (long)jt * BT;
    const int nv = min(BT, p.N - jt * BT);
    const __nv_bfloat16 *Qh = p.q + bh * L * D, *Gh = p.dO + bh * L * D;
    load_tile(sK, p.k + bh * L * D, k0, (long)(gk + 1) * p.N);
    load_tile(sV, p.v + bh * L * D, k0, (long)(gk + 1) * p.N);
    cp_commit();
    // query tiles: frames f = gk + r i (i < w, f < T), 64-row tiles of each
    const int nframes = min(p.w, (p.T - 1 - gk) / p.r + 1);
    const int ntiles = nframes * p.tpf;
    auto tile_src = [&](int it, long &q0, int &nq) {
        const int fq = gk + p.r * (it / p.tpf), u = it % p.tpf;
        q0 = (long)fq * p.N + (long)u * BT;
        nq = min(BT, p.N - u * BT);
    };
    auto load_q = [&](int it, int slot) {
        long q0;
        int nq;
        tile_src(it, q0, nq);
        const uint32_t dQ = sQ0 + (uint32_t)slot * 2 * TILE;
        const long qend = q0 + nq;
        load_tile(dQ, Qh, q0, qend);
        load_tile(dQ + TILE, Gh, q0, qend);
        if (threadIdx.x < BT) {
            const int rr = threadIdx.x;
            const bool ok = rr < nq;
            sL[slot * BT + rr] = ok ? p.lse[bh * L + q0 + rr] * 1.4426950408889634f : INFINITY;
            sD[slot * BT + rr] = ok ? p.Dws[bh * L + q0 + rr] : 0.f;
        }
    };
    load_q(0, 0);
    cp_commit();
    float dk[16][4], dv[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;
    for (int it = 0; it < ntiles; ++it) {
        const int slot = it & 1;
        const uint32_t sQ = sQ0 + (uint32_t)slot * 2 * TILE, sG = sQ + TILE;
        if (it + 1 < ntiles) load_q(it + 1, slot ^ 1);
        cp_commit();
        cp_wait<1>();
        __syncthreads();
        // S^T and dP^T: rows = this warp's 16 keys, columns = the tile's 64 queries
        float s[8][4], dp[8][4];
        gemm_abt(s, sK, 16 * warp, sQ);
        gemm_abt(dp, sV, 16 * warp, sG);
        uint32_t xp[4][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int col = 8 * nt + 2 * t + (e & 1);
                const float pv = exp2f(fmaf(s[nt][e], p.sl2, -sL[slot * BT + col]));   // 0 past the tile's rows
                s[nt][e] = pv;
                dp[nt][e] = pv * (dp[nt][e] - sD[slot * BT + col]);                    // dS^T
            }
        to_afrag(s, xp);
        gemm_xb(dv, xp, sG);
        to_afrag(dp, xp);
        gemm_xb(dk, xp, sQ);
        __syncthreads();
    }
    (void)g;
    store_rows(p.dk + bh * L * D, k0, nv, 16 * warp, dk, p.scale);
    store_rows(p.dv + bh * L * D, k0, nv, 16 * warp, dv, 1.f);
}

}  // namespace

cudaError_t launch_attn_bwd(const AttnBwdArgs &a, cudaStream_t s)
{
    const long L = (long)a.T * a.N;
    const long rows = (long)a.BH * L;
    if (rows == 0) return cudaSuccess;
    BwdParams p;
    p.q = (const __nv_bfloat16 *)a.q; p.k = (const __nv_bfloat16 *)a.k; p.v = (const __nv_bfloat16 *)a.v;
    p.dO = (const __nv_bfloat16 *)a.dO;
    p.lse = a.lse; p.Dws = a.Dws;
    p.dq = (__nv_bfloat16 *)a.dq; p.dk = (__nv_bfloat16 *)a.dk; p.dv = (__nv_bfloat16 *)a.dv;
    p.T = a.T; p.N = a.N; p.w = a.w; p.r = a.r;
    p.tpf = (a.N + BT - 1) / BT;
    p.scale = a.scale;
    p.sl2 = a.scale * 1.4426950408889634f;
    const long tiles = (long)a.T * p.tpf;
    if (tiles >= (1L << 31) || a.BH > 65535 || rows >= (1L << 40)) return cudaErrorNotSupported;
    attn_bwd_dot<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>((const __nv_bfloat16 *)a.o, p.dO, a.Dws, rows);
    cudaError_t e;
    const int smem_dq = 6 * TILE, smem_dkv = 6 * TILE + 4 * BT * sizeof(float);
    if ((e = cudaFuncSetAttribute(attn_bwd_dq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dq)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(attn_bwd_dkv, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_dkv)) != cudaSuccess) return e;
    const dim3 grid((unsigned)tiles, (unsigned)a.BH);
    attn_bwd_dq<<<grid, THREADS, smem_dq, s>>>(p);
    attn_bwd_dkv<<<grid, THREADS, smem_dkv, s>>>(p);
    return cudaGetLastError();
}

}  // namespace hlta
