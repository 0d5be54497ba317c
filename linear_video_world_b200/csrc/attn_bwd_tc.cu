// Gradients of the windowed attention on the sm_100a tensor cores (bf16, d = 128): dK and dV
// (one kernel, key-tile major) and dQ (one kernel, query-tile major), with the forward's per-row
// log-sum-exp to recompute p = exp(s scale - lse) and D = rowsum(dO o O) from the first launch.
//
// dK / dV: one CTA per 128-key tile of one key frame g; it walks the 64-row query tiles of every
// frame that sees g (f = g + r i, i < w, f < T) and keeps dK and dV of its keys in tensor memory.
// Per query tile j:
//   S^T  = K Q_j^T,  dP^T = V dO_j^T                   (128 x 64 each; shared-memory operands)
//   P^T  = exp2(S^T sl2 - lse2_j),  dS^T = P^T o (dP^T - D_j)     (elementwise warps)
//   dV  += P^T dO_j,  dK += dS^T Q_j                   (P^T and dS^T read from tensor memory)
// dQ: the same with queries and keys exchanged (one CTA per 128-row query tile of a frame,
// walking the 64-key tiles of its window; dQ += dS K_j).
// The roles follow the first forward design (64-key tiles, P in tensor memory): the CTA's own
// 128-row tile takes the place of its query sub-tile, the other side's tiles stream through a
// TMA ring like its key tiles,
// P^T / dS are written over their fp32 buffers as bf16 pairs (each half of the columns into the
// first 16 of its own 32 fp32 columns, so the two warps of a lane quadrant never overwrite each
// other's unread scores), and
// products of one issuing thread execute in issue order, so S of tile j+1 is issued into the
// buffers that the same thread's accumulating products of tile j-1 read without a wait (dQ's S
// buffer, which only the elementwise warps read, is reissued after their arrival).
// Threads: warps 0..7 elementwise (one row of the CTA's tile per lane, the warp's TMEM lane
// quadrant; warps w and w + 4 split the 64 columns), warp 8 TMA producer, warps 9 and 10 MMA
// issuers (one thread issues at a limited rate, so the products are split over two; warp 9 owns
// TMEM). Tensor memory: per buffer
// b (two) S at 128 b and dP at 128 b + 64; accumulators at 256 (dV or dQ) and 384 (dK). Every
// mbarrier wait is bounded.
#include "hlta_internal.cuh"
#include "sm100_ptx.cuh"
#include "tc_ptx.cuh"

#include <math.h>

namespace hlta {
namespace {

using namespace ptx;
using namespace tc;

constexpr int BK = 128;                 // keys per CTA (the products' M)
constexpr int BQ = 64;                  // queries per tile (N of S^T, K of the accumulations)
constexpr int D = 128;
constexpr int NS = 3;                   // Q / dO ring stages
constexpr int THREADS = 352;
constexpr int WARP_TMA = 8, WARP_MMA = 9;   // issuers: warp 9 (A, owns TMEM) and warp 10 (B)
constexpr int EW_THREADS = 256;             // elementwise: 8 warps, two per TMEM lane quadrant
constexpr uint32_t KHALF = BK * 128;    // [128 rows][64 cols] bf16: 16 KB
constexpr uint32_t KTILE = 2 * KHALF;
constexpr uint32_t QHALF = BQ * 128;    // [64 rows][64 cols]: 8 KB
constexpr uint32_t QTILE = 2 * QHALF;
constexpr uint32_t SM_K = 0, SM_V = KTILE;
__host__ __device__ constexpr uint32_t SM_Q(int st) { return 2 * KTILE + (uint32_t)st * 2 * QTILE; }
__host__ __device__ constexpr uint32_t SM_G(int st) { return SM_Q(st) + QTILE; }
constexpr uint32_t SM_LD = 2 * KTILE + NS * 2 * QTILE;       // per elementwise warp: lse2[32] | D[32]
constexpr uint32_t SM_BAR = SM_LD + 8 * 64 * 4;
enum { B_KV = 0, B_QFULL = 1, B_EMPTY = B_QFULL + NS, B_SFULL = B_EMPTY + NS, B_PFULL = B_SFULL + 2,
       B_ODONE = B_PFULL + 2, NBARS = B_ODONE + 1 };
constexpr uint32_t SM_TMEMSLOT = SM_BAR + 8 * NBARS;
constexpr uint32_t SM_ABORT = SM_TMEMSLOT + 4;
constexpr size_t SMEM_BYTES = SM_ABORT + 4 + 1024;
constexpr uint32_t TM_ST(int b) { return (uint32_t)b * 128u; }
constexpr uint32_t TM_DPT(int b) { return (uint32_t)b * 128u + 64u; }
constexpr uint32_t TM_DV = 256, TM_DK = 384;

struct Params {
    const float *lse, *Dws;
    __nv_bfloat16 *dk, *dv;
    long L;
    int T, N, w, r, tpk, tpq;   // key tiles (128) and query tiles (64) per frame
    float sl2, scale;
    unsigned int *err;
};

constexpr uint32_t ODONE_DKV = 2, ODONE_DQ = 1;

__global__ void __launch_bounds__(THREADS, 1)
attn_bwd_dkv_tc(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tg,
                const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    auto BAR = [&](int i) { return sbase + SM_BAR + 8u * (uint32_t)i; };
    volatile int *abort_flag = (volatile int *)(smem + SM_ABORT);
    uint32_t *tmem_slot = (uint32_t *)(smem + SM_TMEMSLOT);
    float *LD = (float *)(smem + SM_LD);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long bh = blockIdx.y;
    const int g = blockIdx.x / p.tpk, jt = blockIdx.x % p.tpk;
    const long k0 = (long)g * p.N + (long)jt * BK;
    const int nv = min(BK, p.N - jt * BK);
    const long head = bh * p.L;
    const int nframes = min(p.w, (p.T - 1 - g) / p.r + 1);
    const int ntiles = nframes * p.tpq;
    auto qrow0 = [&](int j) { return head + (long)(g + p.r * (j / p.tpq)) * p.N + (long)(j % p.tpq) * BQ; };
    auto qcount = [&](int j) { return min(BQ, p.N - (j % p.tpq) * BQ); };

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_KV), 1);
        for (int st = 0; st < NS; ++st) {
            mbar_init(BAR(B_QFULL + st), 1);
            mbar_init(BAR(B_EMPTY + st), 2);            // both issuers' products on the stage
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(B_SFULL + b), 2);             // S and dP, one from each issuer
            mbar_init(BAR(B_PFULL + b), EW_THREADS);
        }
        mbar_init(BAR(B_ODONE), ODONE_DKV);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == WARP_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == WARP_TMA) {
        if (lane == 0) {
            mbar_expect_tx(BAR(B_KV), 2 * KTILE);
            const int kr = (int)(head + k0);
            tma_load_2d(sbase + SM_K, &tk, 0, kr, BAR(B_KV));
            tma_load_2d(sbase + SM_K + KHALF, &tk, 64, kr, BAR(B_KV));
            tma_load_2d(sbase + SM_V, &tv, 0, kr, BAR(B_KV));
            tma_load_2d(sbase + SM_V + KHALF, &tv, 64, kr, BAR(B_KV));
            int j = 0;
            for (; j < ntiles; ++j) {
                const int st = j % NS;
                if (j >= NS && !mbar_wait(BAR(B_EMPTY + st), (uint32_t)((j / NS) + 1) & 1u, abort_flag, p.err, DEVERR_ATTN_WAIT)) break;
                mbar_expect_tx(BAR(B_QFULL + st), 2 * QTILE);
                const int qr = (int)qrow0(j);
                tma_load_2d(sbase + SM_Q(st), &tq, 0, qr, BAR(B_QFULL + st));
                tma_load_2d(sbase + SM_Q(st) + QHALF, &tq, 64, qr, BAR(B_QFULL + st));
                tma_load_2d(sbase + SM_G(st), &tg, 0, qr, BAR(B_QFULL + st));
                tma_load_2d(sbase + SM_G(st) + QHALF, &tg, 64, qr, BAR(B_QFULL + st));
            }
            if (*abort_flag) {
                // let this CTA's copies in flight land before the CTA may exit
                const long long t0 = clock64();
                while (!mbar_try(BAR(B_KV), 0) && clock64() - t0 < (1LL << 31)) {}
                for (int jj = j - 1; jj >= 0 && jj >= j - NS; --jj)
                    while (!mbar_try(BAR(B_QFULL + jj % NS), (uint32_t)(jj / NS) & 1u) && clock64() - t0 < (1LL << 31)) {}
            }
        }
    } else if (warp == WARP_MMA || warp == WARP_MMA + 1) {
        // Issuer A: S^T = K Q^T and dV += P^T dO (buffer ST); issuer B: dP^T = V dO^T and
        // dK += dS^T Q (buffer DPT). Each issuer reuses only its own buffers, in issue order.
        if (lane == 0) {
            const bool A = warp == WARP_MMA;
            constexpr uint32_t IDESC_S = idesc_bf16(BK, BQ, false, false);   // K / V and Q / dO K-major
            constexpr uint32_t IDESC_A = idesc_bf16(BK, D, false, true);     // P^T, dS^T from TMEM; dO, Q MN-major
            const uint64_t da_ = sw128_desc(sbase + (A ? SM_K : SM_V), 16, 1024);
            auto wait_bar = [&](uint32_t bar, uint32_t parity) -> bool {
                return mbar_try(bar, parity) || mbar_wait(bar, parity, abort_flag, p.err, DEVERR_ATTN_WAIT);
            };
            auto issue_s = [&](int j) -> bool {
                const int st = j % NS, b = j & 1;
                if (!wait_bar(BAR(B_QFULL + st), (uint32_t)(j / NS) & 1u)) return false;
                fence_after_sync();
                const uint64_t db_ = sw128_desc(sbase + (A ? SM_Q(st) : SM_G(st)), 16, 1024);
                const uint32_t dst = tmem + (A ? TM_ST(b) : TM_DPT(b));
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t aoff = ((kk >> 2) * KHALF + (kk & 3) * 32) >> 4;
                    const uint32_t boff = ((kk >> 2) * QHALF + (kk & 3) * 32) >> 4;
                    umma_bf16(dst, da_ + aoff, db_ + boff, IDESC_S, kk > 0 ? 1u : 0u);
                }
                umma_commit(BAR(B_SFULL + b));
                return true;
            };
            bool ok = wait_bar(BAR(B_KV), 0) && issue_s(0);
            for (int j = 0; ok && j < ntiles; ++j) {
                if (j + 1 < ntiles && !(ok = issue_s(j + 1))) break;
                const int st = j % NS, b = j & 1;
                if (!(ok = wait_bar(BAR(B_PFULL + b), (uint32_t)(j >> 1) & 1u))) break;
                fence_after_sync();
                // dV += P^T dO_j (A) or dK += dS^T Q_j (B): 64 queries in 4 steps of 16
                const uint64_t dbm = sw128_desc(sbase + (A ? SM_G(st) : SM_Q(st)), QHALF, 1024);
                const uint32_t acc = tmem + (A ? TM_DV : TM_DK), src = tmem + (A ? TM_ST(b) : TM_DPT(b));
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk)
                    umma_bf16_ts(acc, src + (kk >> 1) * 32 + (kk & 1) * 8, dbm + (uint64_t)((kk * 2048) >> 4), IDESC_A,
                                 (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(BAR(B_EMPTY + st));
            }
            if (ok) umma_commit(BAR(B_ODONE));
        }
    } else {
        // ----------- elementwise: one key row per lane, query columns split over two warps ----
        // Warps q4 and q4 + 4 share TMEM lanes 32 q4 ..; warp half h takes query columns
        // 32 h .. 32 h + 31 and writes its bf16 pairs over the first 16 of its own 32 fp32
        // columns (columns 0..15 and 32..47), which the accumulating products read as A.
        const int q4 = warp & 3, h = warp >> 2;
        const int kr = q4 * 32 + lane;
        const uint32_t tlane = tmem + ((uint32_t)(q4 * 32) << 16);
        bool ok = true;
        float *LDw = LD + warp * 64;                // this warp's lse2 | D (no wait across warps)
        for (int j = 0; j < ntiles; ++j) {
            const int b = j & 1;
            // this tile's lse2 (log2 units) and D of the warp's columns; past the frame: +inf, 0
            {
                const long q0 = qrow0(j);
                const int nq = qcount(j);
                const int c = 32 * h + lane;
                __syncwarp();
                LDw[lane] = c < nq ? p.lse[q0 + c] * 1.4426950408889634f : INFINITY;
                LDw[32 + lane] = c < nq ? p.Dws[q0 + c] : 0.f;
                __syncwarp();
            }
            const uint32_t sbar = BAR(B_SFULL + b), spar = (uint32_t)(j >> 1) & 1u;
            if (!__all_sync(0xffffffffu, mbar_try(sbar, spar) || mbar_wait(sbar, spar, abort_flag, p.err, DEVERR_ATTN_WAIT))) { ok = false; break; }
            fence_after_sync();
            uint32_t sr[32], dr[32];
            tmem_ld32(tlane + TM_ST(b) + 32 * h, sr);
            tmem_ld32(tlane + TM_DPT(b) + 32 * h, dr);
            const float4 *L4 = reinterpret_cast<const float4 *>(LDw);
            uint32_t pk[16], gk[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 l = L4[i], dd = L4[8 + i];
                const int col = 4 * i;
                const float p0 = ex2(fmaf(__uint_as_float(sr[col]), p.sl2, -l.x));
                const float p1 = ex2(fmaf(__uint_as_float(sr[col + 1]), p.sl2, -l.y));
                const float p2 = ex2(fmaf(__uint_as_float(sr[col + 2]), p.sl2, -l.z));
                const float p3 = ex2(fmaf(__uint_as_float(sr[col + 3]), p.sl2, -l.w));
                pk[2 * i] = pack_bf16(p0, p1);
                pk[2 * i + 1] = pack_bf16(p2, p3);
                gk[2 * i] = pack_bf16(p0 * (__uint_as_float(dr[col]) - dd.x), p1 * (__uint_as_float(dr[col + 1]) - dd.y));
                gk[2 * i + 1] = pack_bf16(p2 * (__uint_as_float(dr[col + 2]) - dd.z), p3 * (__uint_as_float(dr[col + 3]) - dd.w));
            }
            tmem_st16(tlane + TM_ST(b) + 32 * h, pk);
            tmem_st16(tlane + TM_DPT(b) + 32 * h, gk);
            tmem_wait_st();
            fence_before_sync();
            mbar_arrive(BAR(B_PFULL + b));
        }
        // epilogue: dK (times the softmax scale) and dV of this thread's key, columns 64 h ..
        const bool fin = ok && __all_sync(0xffffffffu, mbar_wait(BAR(B_ODONE), 0u, abort_flag, p.err, DEVERR_ATTN_WAIT));
        if (fin) {
            fence_after_sync();
            const long row = head + k0 + kr;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                __nv_bfloat16 *dst = (which ? p.dv : p.dk) + row * D;
                const float mul = which ? 1.f : p.scale;
#pragma unroll
                for (int c = 2 * h; c < 2 * h + 2; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tlane + (which ? TM_DV : TM_DK) + c * 32, v);
                    if (kr < nv) {
                        uint32_t pk2[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pk2[i] = pack_bf16(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul);
                        uint4 *d4 = reinterpret_cast<uint4 *>(dst + c * 32);
#pragma unroll
                        for (int q4_ = 0; q4_ < 4; ++q4_)
                            d4[q4_] = make_uint4(pk2[4 * q4_], pk2[4 * q4_ + 1], pk2[4 * q4_ + 2], pk2[4 * q4_ + 3]);
                    }
                }
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == WARP_MMA) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    }
}

// ----------------------------------------------------------------------------------------
// dQ: one CTA per 128-row query tile of one frame f; walks the 64-key tiles of the frame's
// window (f - r i, i < w, >= 0). Per key tile j:
//   S = Q K_j^T,  dP = dO V_j^T,  dS = exp2(S sl2 - lse2) o (dP - D)   (row constants)
//   dQ += dS K_j                                                      (dS from tensor memory)
// Same roles and barrier protocol as the dK / dV kernel with queries and keys exchanged.
__global__ void __launch_bounds__(THREADS, 1)
attn_bwd_dq_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tg,
               const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
               const Params p, __nv_bfloat16 *dq)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    auto BAR = [&](int i) { return sbase + SM_BAR + 8u * (uint32_t)i; };
    volatile int *abort_flag = (volatile int *)(smem + SM_ABORT);
    uint32_t *tmem_slot = (uint32_t *)(smem + SM_TMEMSLOT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long bh = blockIdx.y;
    const int f = blockIdx.x / p.tpk, ut = blockIdx.x % p.tpk;
    const long q0 = (long)f * p.N + (long)ut * BK;
    const int nq = min(BK, p.N - ut * BK);
    const long head = bh * p.L;
    const int nframes = min(p.w, f / p.r + 1);
    const int ntiles = nframes * p.tpq;
    // key frames from the oldest
    auto krow0 = [&](int j) { return head + (long)(f - p.r * (nframes - 1 - j / p.tpq)) * p.N + (long)(j % p.tpq) * BQ; };
    auto kcount = [&](int j) { return min(BQ, p.N - (j % p.tpq) * BQ); };

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_KV), 1);
        for (int st = 0; st < NS; ++st) {
            mbar_init(BAR(B_QFULL + st), 1);
            mbar_init(BAR(B_EMPTY + st), 2);            // both issuers' products on the stage
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(B_SFULL + b), 2);             // S and dP, one from each issuer
            mbar_init(BAR(B_PFULL + b), EW_THREADS);
        }
        mbar_init(BAR(B_ODONE), ODONE_DQ);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == WARP_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == WARP_TMA) {
        if (lane == 0) {
            // the query tile's Q and dO (128 rows) in the slots of K and V of the other kernel
            mbar_expect_tx(BAR(B_KV), 2 * KTILE);
            const int qr = (int)(head + q0);
            tma_load_2d(sbase + SM_K, &tq, 0, qr, BAR(B_KV));
            tma_load_2d(sbase + SM_K + KHALF, &tq, 64, qr, BAR(B_KV));
            tma_load_2d(sbase + SM_V, &tg, 0, qr, BAR(B_KV));
            tma_load_2d(sbase + SM_V + KHALF, &tg, 64, qr, BAR(B_KV));
            int j = 0;
            for (; j < ntiles; ++j) {
                const int st = j % NS;
                if (j >= NS && !mbar_wait(BAR(B_EMPTY + st), (uint32_t)((j / NS) + 1) & 1u, abort_flag, p.err, DEVERR_ATTN_WAIT)) break;
                mbar_expect_tx(BAR(B_QFULL + st), 2 * QTILE);
                const int kr = (int)krow0(j);
                tma_load_2d(sbase + SM_Q(st), &tk, 0, kr, BAR(B_QFULL + st));
                tma_load_2d(sbase + SM_Q(st) + QHALF, &tk, 64, kr, BAR(B_QFULL + st));
                tma_load_2d(sbase + SM_G(st), &tv, 0, kr, BAR(B_QFULL + st));
                tma_load_2d(sbase + SM_G(st) + QHALF, &tv, 64, kr, BAR(B_QFULL + st));
            }
            if (*abort_flag) {
                const long long t0 = clock64();
                while (!mbar_try(BAR(B_KV), 0) && clock64() - t0 < (1LL << 31)) {}
                for (int jj = j - 1; jj >= 0 && jj >= j - NS; --jj)
                    while (!mbar_try(BAR(B_QFULL + jj % NS), (uint32_t)(jj / NS) & 1u) && clock64() - t0 < (1LL << 31)) {}
            }
        }
    } else if (warp == WARP_MMA || warp == WARP_MMA + 1) {
        // Issuer A: S = Q K^T (buffer ST; it waits until the elementwise warps have read the S
        // it overwrites); issuer B: dP = dO V^T and dQ += dS K (buffer DPT, reused in issue order).
        if (lane == 0) {
            const bool A = warp == WARP_MMA;
            constexpr uint32_t IDESC_S = idesc_bf16(BK, BQ, false, false);   // Q / dO and K / V K-major
            constexpr uint32_t IDESC_A = idesc_bf16(BK, D, false, true);     // dS from TMEM; K MN-major
            const uint64_t da_ = sw128_desc(sbase + (A ? SM_K : SM_V), 16, 1024);
            auto wait_bar = [&](uint32_t bar, uint32_t parity) -> bool {
                return mbar_try(bar, parity) || mbar_wait(bar, parity, abort_flag, p.err, DEVERR_ATTN_WAIT);
            };
            auto issue_s = [&](int j) -> bool {
                const int st = j % NS, b = j & 1;
                if (!wait_bar(BAR(B_QFULL + st), (uint32_t)(j / NS) & 1u)) return false;
                if (A && j >= 2 && !wait_bar(BAR(B_PFULL + b), (uint32_t)((j - 2) >> 1) & 1u)) return false;
                fence_after_sync();
                const uint64_t db_ = sw128_desc(sbase + (A ? SM_Q(st) : SM_G(st)), 16, 1024);
                const uint32_t dst = tmem + (A ? TM_ST(b) : TM_DPT(b));
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t aoff = ((kk >> 2) * KHALF + (kk & 3) * 32) >> 4;
                    const uint32_t boff = ((kk >> 2) * QHALF + (kk & 3) * 32) >> 4;
                    umma_bf16(dst, da_ + aoff, db_ + boff, IDESC_S, kk > 0 ? 1u : 0u);
                }
                umma_commit(BAR(B_SFULL + b));
                if (A) umma_commit(BAR(B_EMPTY + st));   // A reads the stage's K only here
                return true;
            };
            bool ok = wait_bar(BAR(B_KV), 0) && issue_s(0);
            for (int j = 0; ok && j < ntiles; ++j) {
                if (j + 1 < ntiles && !(ok = issue_s(j + 1))) break;
                if (A) continue;
                const int st = j % NS, b = j & 1;
                if (!(ok = wait_bar(BAR(B_PFULL + b), (uint32_t)(j >> 1) & 1u))) break;
                fence_after_sync();
                // dQ += dS K_j: 64 keys in 4 steps of 16 (8 TMEM columns each), K MN-major
                const uint64_t dkm = sw128_desc(sbase + SM_Q(st), QHALF, 1024);
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk)
                    umma_bf16_ts(tmem + TM_DV, tmem + TM_DPT(b) + (kk >> 1) * 32 + (kk & 1) * 8, dkm + (uint64_t)((kk * 2048) >> 4), IDESC_A,
                                 (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(BAR(B_EMPTY + st));
            }
            if (ok && !A) umma_commit(BAR(B_ODONE));
        }
    } else {
        // ----------- elementwise: one query row per lane, key columns split over two warps ----
        const int q4 = warp & 3, h = warp >> 2;
        const int qrw = q4 * 32 + lane;
        const uint32_t tlane = tmem + ((uint32_t)(q4 * 32) << 16);
        const bool rv = qrw < nq;
        const float lse2 = rv ? p.lse[head + q0 + qrw] * 1.4426950408889634f : INFINITY;
        const float Dr = rv ? p.Dws[head + q0 + qrw] : 0.f;
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            const int b = j & 1;
            const int nv = kcount(j) - 32 * h;      // valid key columns of this warp's half
            const uint32_t sbar = BAR(B_SFULL + b), spar = (uint32_t)(j >> 1) & 1u;
            if (!__all_sync(0xffffffffu, mbar_try(sbar, spar) || mbar_wait(sbar, spar, abort_flag, p.err, DEVERR_ATTN_WAIT))) { ok = false; break; }
            fence_after_sync();
            uint32_t sr[32], dr[32];
            tmem_ld32(tlane + TM_ST(b) + 32 * h, sr);
            tmem_ld32(tlane + TM_DPT(b) + 32 * h, dr);
            uint32_t gk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int col = 2 * i;
                const float p0 = col < nv ? ex2(fmaf(__uint_as_float(sr[col]), p.sl2, -lse2)) : 0.f;
                const float p1 = col + 1 < nv ? ex2(fmaf(__uint_as_float(sr[col + 1]), p.sl2, -lse2)) : 0.f;
                gk[i] = pack_bf16(p0 * (__uint_as_float(dr[col]) - Dr), p1 * (__uint_as_float(dr[col + 1]) - Dr));
            }
            tmem_st16(tlane + TM_DPT(b) + 32 * h, gk);
            tmem_wait_st();
            fence_before_sync();
            mbar_arrive(BAR(B_PFULL + b));
        }
        const bool fin = ok && __all_sync(0xffffffffu, mbar_wait(BAR(B_ODONE), 0u, abort_flag, p.err, DEVERR_ATTN_WAIT));
        if (fin) {
            fence_after_sync();
            __nv_bfloat16 *dst = dq + (head + q0 + qrw) * D;
#pragma unroll
            for (int c = 2 * h; c < 2 * h + 2; ++c) {
                uint32_t v[32];
                tmem_ld32(tlane + TM_DV + c * 32, v);
                if (rv) {
                    uint32_t pk2[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk2[i] = pack_bf16(__uint_as_float(v[2 * i]) * p.scale, __uint_as_float(v[2 * i + 1]) * p.scale);
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst + c * 32);
#pragma unroll
                    for (int q4_ = 0; q4_ < 4; ++q4_)
                        d4[q4_] = make_uint4(pk2[4 * q4_], pk2[4 * q4_ + 1], pk2[4 * q4_ + 2], pk2[4 * q4_ + 3]);
                }
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == WARP_MMA) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    }
}

}  // namespace

cudaError_t launch_attn_bwd_tc(const AttnBwdArgs &a, cudaStream_t s)
{
    const long L = (long)a.T * a.N;
    const long rows = (long)a.BH * L;
    if (rows + BK >= (1L << 31)) return cudaErrorNotSupported;
    CUtensorMap mk, mv, mq, mg;
    cudaError_t e;
    if ((e = make_tmap_2d_bf16(&mk, a.k, rows, D, 64, BK, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&mv, a.v, rows, D, 64, BK, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&mq, a.q, rows, D, 64, BQ, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&mg, a.dO, rows, D, 64, BQ, true)) != cudaSuccess) return e;
    Params p;
    p.lse = a.lse; p.Dws = a.Dws;
    p.dk = (__nv_bfloat16 *)a.dk; p.dv = (__nv_bfloat16 *)a.dv;
    p.L = L; p.T = a.T; p.N = a.N; p.w = a.w; p.r = a.r;
    p.tpk = (a.N + BK - 1) / BK;
    p.tpq = (a.N + BQ - 1) / BQ;
    p.scale = a.scale;
    p.sl2 = a.scale * 1.4426950408889634f;
    p.err = device_error_word();
    if (!p.err) return cudaErrorUnknown;
    if ((e = cudaFuncSetAttribute(attn_bwd_dkv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES)) != cudaSuccess)
        return e;
    const dim3 grid((unsigned)((long)a.T * p.tpk), (unsigned)a.BH);
    attn_bwd_dkv_tc<<<grid, THREADS, SMEM_BYTES, s>>>(mk, mv, mq, mg, p), note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // dQ: query tiles of 128 rows (the maps of the other kernel with the boxes exchanged)
    CUtensorMap mq2, mg2, mk2, mv2;
    if ((e = make_tmap_2d_bf16(&mq2, a.q, rows, D, 64, BK, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&mg2, a.dO, rows, D, 64, BK, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&mk2, a.k, rows, D, 64, BQ, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&mv2, a.v, rows, D, 64, BQ, true)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(attn_bwd_dq_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES)) != cudaSuccess)
        return e;
    attn_bwd_dq_tc<<<grid, THREADS, SMEM_BYTES, s>>>(mq2, mg2, mk2, mv2, p, (__nv_bfloat16 *)a.dq), note_launch();
    return cudaGetLastError();
}

}  // namespace hlta
