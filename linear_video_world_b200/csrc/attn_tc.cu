// Windowed softmax attention (SWA / DSWA / streaming step) on the sm_100a tensor cores.
// bf16 q/k/v/o, head dim 128, fp32 accumulation in tensor memory.
//
// Exact attention by tiles with a running max and normaliser (llm-atlas long-context
// explainer, section 03 "Flash Attention": the score matrix never leaves the chip and the
// result equals the full softmax). The key set of a query tile is the union of the key
// frames of its rows' frames (sliding window: frames f-w+1..f; dilated: f, f-r, ...,
// f-r(w-1); Kairos abstract, item (2)); each key frame is walked in 128-token tiles and a
// per-element mask (row frame vs. key frame, ragged frame end) removes what a row must not
// see.
//
// One CTA = two 128-row query sub-tiles (256 consecutive query rows) of one head; 18 warps:
//   warps 0..7    softmax of sub-tile 0, warps 8..15 softmax of sub-tile 1: each query row is
//                 shared by two threads (same TMEM lane, warps w and w+4), one per 64-key half
//                 of every S tile; they agree on the row max through shared memory once per
//                 tile and keep partial row sums until the end
//   warp 16       TMA producer: Q (both sub-tiles) once, then K and V tiles into a 2-stage
//                 ring (128B swizzle); the sub-tiles share every K/V tile
//   warp 17       TMEM owner and MMA issuer (tcgen05.mma kind::f16): S_q = Q_q K_j^T into TMEM,
//                 O_q += P_q V_j with P_q read from TMEM (written there by the softmax over the
//                 first 64 columns of S_q) and V_j an MN-major shared-memory operand; order
//                 S_0(j) S_1(j) | PV_0(j) S_0(j+1) PV_1(j) S_1(j+1) | ...; same-thread tcgen05.mma
//                 execute in issue order, so the next S follows the PV that reads P directly
// The running max lives per row (O rescaled in TMEM only when it grows by more than 2^8), P is
// bf16 in TMEM, and the final normalisation combines the two partial row sums.
// A key tile that no row of a sub-tile may see is skipped for that sub-tile (no MMA, no
// softmax). Every mbarrier wait is bounded; on expiry the kernel records DEVERR_ATTN_WAIT in
// the device error word, every role stops, and the TMEM allocation is released.
#include "hlta_internal.cuh"
#include "sm100_ptx.cuh"

#include <math.h>

namespace hlta {
namespace {

using namespace ptx;

constexpr int BM = 128;                 // query rows per sub-tile
constexpr int QT = 2;                   // query sub-tiles per CTA
constexpr int BN = 128;                 // keys per tile
constexpr int D = 128;                  // head dim
constexpr int NS = 2;                   // K/V ring stages
constexpr int THREADS = 576;           // 16 softmax warps, TMA warp, MMA warp
constexpr int WARP_TMA = 16, WARP_MMA = 17;
constexpr int SOFTMAX_THREADS = 256;   // per sub-tile: 128 rows x 2 column halves
constexpr uint32_t HALF = 16384;        // one [128 rows][64 cols] bf16 half tile
constexpr uint32_t TILE = 2 * HALF;     // [128][128] bf16
constexpr uint32_t TMEM_COLS = 512;     // S_0 @0, S_1 @128, O_0 @256, O_1 @384
__host__ __device__ constexpr uint32_t TM_S(int q) { return (uint32_t)q * 128u; }
__host__ __device__ constexpr uint32_t TM_O(int q) { return 256u + (uint32_t)q * 128u; }

// shared memory map (offsets from a 1024-byte aligned base)
__host__ __device__ constexpr uint32_t SM_Q(int q) { return (uint32_t)q * TILE; }
__host__ __device__ constexpr uint32_t SM_K(int st) { return QT * TILE + (uint32_t)st * 2 * TILE; }
__host__ __device__ constexpr uint32_t SM_V(int st) { return SM_K(st) + TILE; }
constexpr uint32_t SM_BAR = SM_K(NS);
// barriers (8 bytes each)
enum {
    B_QFULL = 0,
    B_KFULL = 1,                // + stage
    B_VFULL = B_KFULL + NS,
    B_KEMPTY = B_VFULL + NS,
    B_VEMPTY = B_KEMPTY + NS,
    B_SFULL = B_VEMPTY + NS,    // + sub-tile
    B_PFULL = B_SFULL + QT,
    B_PVDONE = B_PFULL + QT,
    NBARS = B_PVDONE + QT
};
constexpr uint32_t SM_TMEMSLOT = SM_BAR + 8 * NBARS;
constexpr uint32_t SM_ABORT = SM_TMEMSLOT + 4;
// row-max exchange between the two column halves: [sub-tile][tile parity][half][row] floats
constexpr uint32_t SM_XCH = (SM_ABORT + 4 + 15) & ~15u;
constexpr uint32_t SM_TOTAL = SM_XCH + QT * 2 * 2 * BM * 4;
constexpr size_t SMEM_BYTES = SM_TOTAL + 1024;          // slack for the 1024-byte alignment

struct TcParams {
    int Hbr, q_Htot, q_h0, kv_Htot, kv_h0, kv_slots;
    long q_rows, kv_rows;
    int N, w, r, fq0;
    float sl2;                  // softmax scale * log2(e)
    __nv_bfloat16 *o;
    unsigned int *err;
};

// ---------------------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void fence_before_sync()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Same with the A operand read from tensor memory (M lanes x K bf16 packed in pairs per column)
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), sm_100 version bit.
// lbo / sbo in bytes: K-major operands use sbo = 1024 (8 rows of 128 B) and an unused lbo;
// MN-major operands use lbo = distance between 64-element column blocks, sbo = 1024.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor for kind::f16: bf16 A and B, fp32 accumulator, M x N tile.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

#define TMEM_REGS32(x)                                                                      \
    "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3]), "=r"(x[4]), "=r"(x[5]), "=r"(x[6]),     \
        "=r"(x[7]), "=r"(x[8]), "=r"(x[9]), "=r"(x[10]), "=r"(x[11]), "=r"(x[12]),          \
        "=r"(x[13]), "=r"(x[14]), "=r"(x[15]), "=r"(x[16]), "=r"(x[17]), "=r"(x[18]),       \
        "=r"(x[19]), "=r"(x[20]), "=r"(x[21]), "=r"(x[22]), "=r"(x[23]), "=r"(x[24]),       \
        "=r"(x[25]), "=r"(x[26]), "=r"(x[27]), "=r"(x[28]), "=r"(x[29]), "=r"(x[30]),       \
        "=r"(x[31])
#define TMEM_SRC32(x)                                                                        \
    "r"(x[0]), "r"(x[1]), "r"(x[2]), "r"(x[3]), "r"(x[4]), "r"(x[5]), "r"(x[6]), "r"(x[7]), \
        "r"(x[8]), "r"(x[9]), "r"(x[10]), "r"(x[11]), "r"(x[12]), "r"(x[13]), "r"(x[14]),    \
        "r"(x[15]), "r"(x[16]), "r"(x[17]), "r"(x[18]), "r"(x[19]), "r"(x[20]), "r"(x[21]),  \
        "r"(x[22]), "r"(x[23]), "r"(x[24]), "r"(x[25]), "r"(x[26]), "r"(x[27]), "r"(x[28]),  \
        "r"(x[29]), "r"(x[30]), "r"(x[31])

// 32 consecutive fp32 columns of this thread's TMEM lane (warp w reads lanes 32*(w%4)..).
// The load and its wait sit in one asm statement, so no use of the registers can be
// scheduled between them.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&x)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : TMEM_REGS32(x)
        : "r"(taddr)
        : "memory");
}

// 64 consecutive fp32 columns, load and wait in one statement
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&x)[64])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {"
        "%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
        "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
        "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, "
        "[%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : TMEM_REGS32(x), TMEM_REGS32((x + 32))
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&x)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(x[0]), "r"(x[1]), "r"(x[2]), "r"(x[3]), "r"(x[4]), "r"(x[5]), "r"(x[6]), "r"(x[7]),
        "r"(x[8]), "r"(x[9]), "r"(x[10]), "r"(x[11]), "r"(x[12]), "r"(x[13]), "r"(x[14]), "r"(x[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&x)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        TMEM_SRC32(x)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// ---------------------------------------------------------------------------------------
// key-tile walk shared by every role (all roles must visit the same sequence)
// ---------------------------------------------------------------------------------------
// frame fk is a key frame of some query frame in [fa, fb]
__device__ __forceinline__ bool frame_needed(int fk, int fa, int fb, int w, int r)
{
    const int i0 = fa > fk ? (fa - fk + r - 1) / r : 0;
    return i0 < w && fk + r * i0 <= fb;
}

struct Walk {
    int fa, fb, w, r, tpf;
    __device__ __forceinline__ bool needed(int fk) const { return frame_needed(fk, fa, fb, w, r); }
    // advance (fk, jt) to the next tile; false when done
    __device__ __forceinline__ bool next(int &fk, int &jt) const
    {
        if (++jt < tpf) return true;
        for (++fk; fk <= fb; ++fk)
            if (needed(fk)) {
                jt = 0;
                return true;
            }
        return false;
    }
};

__device__ __forceinline__ bool is_tap(int fq, int fk, int w, int r)
{
    int dist = fq - fk;
    return dist >= 0 && dist <= r * (w - 1) && (dist % r) == 0;
}

__global__ void __launch_bounds__(THREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, const TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + SM_BAR;
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    volatile int *abort_flag = (volatile int *)(smem + SM_ABORT);
    uint32_t *tmem_slot = (uint32_t *)(smem + SM_TMEMSLOT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int b = bh / p.Hbr, h = bh % p.Hbr;
    const long l0 = (long)blockIdx.x * (QT * BM);
    const long q_head = (long)(b * p.q_Htot + p.q_h0 + h) * p.q_rows;
    const long kv_head = (long)(b * p.kv_Htot + p.kv_h0 + h) * p.kv_rows;
    // frame ranges of the two sub-tiles (sub-tile 1 may be empty in the last CTA of a head)
    int sfa[QT], sfb[QT];
    bool svalid[QT];
#pragma unroll
    for (int q = 0; q < QT; ++q) {
        const long r0 = l0 + q * BM;
        svalid[q] = r0 < p.q_rows;
        const long r1 = min(r0 + BM, p.q_rows) - 1;
        sfa[q] = p.fq0 + (int)(r0 / p.N);
        sfb[q] = svalid[q] ? p.fq0 + (int)(r1 / p.N) : sfa[q];
    }
    Walk wk;
    wk.fa = sfa[0];
    wk.fb = svalid[1] ? sfb[1] : sfb[0];
    wk.w = p.w;
    wk.r = p.r;
    wk.tpf = (p.N + BN - 1) / BN;
    const int fstart = max(0, wk.fa - p.r * (p.w - 1));
    auto active = [&](int q, int fk) {
        return svalid[q] && frame_needed(fk, sfa[q], sfb[q], p.w, p.r);
    };

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_QFULL), 1);
        for (int st = 0; st < NS; ++st) {
            mbar_init(BAR(B_KFULL + st), 1);
            mbar_init(BAR(B_VFULL + st), 1);
            mbar_init(BAR(B_KEMPTY + st), 1);
            mbar_init(BAR(B_VEMPTY + st), 1);
        }
        for (int q = 0; q < QT; ++q) {
            mbar_init(BAR(B_SFULL + q), 1);
            mbar_init(BAR(B_PFULL + q), SOFTMAX_THREADS);
            mbar_init(BAR(B_PVDONE + q), 1);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == WARP_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == WARP_TMA) {
        // ------------------------------- TMA producer -----------------------------------
        if (lane == 0) {
            mbar_expect_tx(BAR(B_QFULL), QT * TILE);
            for (int q = 0; q < QT; ++q) {
                const int qrow = (int)(q_head + l0 + q * BM);
                tma_load_2d(sbase + SM_Q(q), &tq, 0, qrow, BAR(B_QFULL));
                tma_load_2d(sbase + SM_Q(q) + HALF, &tq, 64, qrow, BAR(B_QFULL));
            }
            int fk = fstart - 1, jt = wk.tpf - 1, j = 0;
            while (wk.next(fk, jt)) {
                const int st = j % NS;
                const uint32_t ph = (uint32_t)((j / NS) + 1) & 1u;
                const int krow = (int)(kv_head + (long)(fk % p.kv_slots) * p.N + (long)jt * BN);
                if (j >= NS && !mbar_wait(BAR(B_KEMPTY + st), ph, abort_flag, p.err, DEVERR_ATTN_WAIT)) break;
                mbar_expect_tx(BAR(B_KFULL + st), TILE);
                tma_load_2d(sbase + SM_K(st), &tk, 0, krow, BAR(B_KFULL + st));
                tma_load_2d(sbase + SM_K(st) + HALF, &tk, 64, krow, BAR(B_KFULL + st));
                if (j >= NS && !mbar_wait(BAR(B_VEMPTY + st), ph, abort_flag, p.err, DEVERR_ATTN_WAIT)) break;
                mbar_expect_tx(BAR(B_VFULL + st), TILE);
                tma_load_2d(sbase + SM_V(st), &tv, 0, krow, BAR(B_VFULL + st));
                tma_load_2d(sbase + SM_V(st) + HALF, &tv, 64, krow, BAR(B_VFULL + st));
                ++j;
            }
            if (*abort_flag) {
                // let this CTA's copies in flight land before the CTA may exit
                const long long t0 = clock64();
                for (int jj = j - 1; jj >= 0 && jj >= j - NS; --jj) {
                    const int st = jj % NS;
                    const uint32_t ph = (uint32_t)(jj / NS) & 1u;
                    while (!mbar_try(BAR(B_KFULL + st), ph) && clock64() - t0 < (1LL << 31)) {}
                    while (!mbar_try(BAR(B_VFULL + st), ph) && clock64() - t0 < (1LL << 31)) {}
                }
                while (!mbar_try(BAR(B_QFULL), 0) && clock64() - t0 < (1LL << 31)) {}
            }
        }
    } else if (warp == WARP_MMA) {
        // ------------------------------- MMA issuer -------------------------------------
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16(BM, BN, false, false);   // Q, K K-major
            constexpr uint32_t IDESC_O = idesc_bf16(BM, D, false, true);     // P (TMEM), V MN-major
            int n_pv[QT] = {0, 0};
            bool ok = mbar_wait(BAR(B_QFULL), 0, abort_flag, p.err, DEVERR_ATTN_WAIT);
            // S_q = Q_q K^T. It overwrites the TMEM columns the previous PV of this sub-tile
            // reads P_q from; tcgen05.mma operations issued by one thread execute in issue
            // order, so it is issued right behind that PV without waiting for it.
            auto issue_s = [&](int q, int st) -> bool {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
                    umma_bf16(tmem + TM_S(q), sw128_desc(sbase + SM_Q(q) + off, 16, 1024),
                              sw128_desc(sbase + SM_K(st) + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
                }
                umma_commit(BAR(B_SFULL + q));
                return true;
            };
            // O_q += P_q V, P_q from TMEM (bf16 pairs in the first 64 columns of S_q)
            auto issue_pv = [&](int q, int st) -> bool {
                if (!mbar_wait(BAR(B_PFULL + q), (uint32_t)n_pv[q] & 1u, abort_flag, p.err, DEVERR_ATTN_WAIT)) return false;
                fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    umma_bf16_ts(tmem + TM_O(q), tmem + TM_S(q) + kk * 8,
                                 sw128_desc(sbase + SM_V(st) + kk * 2048, HALF, 1024), IDESC_O,
                                 (n_pv[q] > 0 || kk > 0) ? 1u : 0u);
                umma_commit(BAR(B_PVDONE + q));
                ++n_pv[q];
                return true;
            };
            int fk = fstart - 1, jt = wk.tpf - 1, j = 0;
            bool have = ok && wk.next(fk, jt);
            if (have) {
                ok = mbar_wait(BAR(B_KFULL + 0), 0, abort_flag, p.err, DEVERR_ATTN_WAIT);
                for (int q = 0; q < QT && ok; ++q)
                    if (active(q, fk)) ok = issue_s(q, 0);
                if (ok) umma_commit(BAR(B_KEMPTY + 0));
            }
            while (ok && have) {
                const int st = j % NS, fk_cur = fk;
                int fk_n = fk, jt_n = jt;
                const bool have_n = wk.next(fk_n, jt_n);
                const int stn = (j + 1) % NS;
                if (!mbar_wait(BAR(B_VFULL + st), (uint32_t)(j / NS) & 1u, abort_flag, p.err, DEVERR_ATTN_WAIT)) { ok = false; break; }
                bool k_ready = false;                   // K of the next tile, waited for once
                for (int q = 0; q < QT && ok; ++q) {
                    if (active(q, fk_cur)) ok = issue_pv(q, st);
                    if (ok && have_n && active(q, fk_n)) {
                        if (!k_ready)
                            ok = k_ready = mbar_wait(BAR(B_KFULL + stn), (uint32_t)((j + 1) / NS) & 1u, abort_flag, p.err, DEVERR_ATTN_WAIT);
                        if (ok) ok = issue_s(q, stn);
                    }
                }
                if (!ok) break;
                if (have_n) umma_commit(BAR(B_KEMPTY + stn));
                umma_commit(BAR(B_VEMPTY + st));
                fk = fk_n;
                jt = jt_n;
                have = have_n;
                ++j;
            }
        }
    } else if (warp < 16) {
        // ------------------------------- softmax ----------------------------------------
        const int q = warp >> 3;                        // sub-tile of this warp
        const int hf = (warp >> 2) & 1;                 // 64-key half of every S tile
        const int quad = warp & 3;                      // TMEM lane quadrant of this warp
        const int row = quad * 32 + lane;
        const long lrow = l0 + q * BM + row;
        const bool row_valid = lrow < p.q_rows;
        const int fq = p.fq0 + (int)(lrow / p.N);
        const uint32_t tlane = tmem + ((uint32_t)(quad * 32) << 16);
        float *xch = (float *)(smem + SM_XCH) + q * (2 * 2 * BM);   // [parity][half][row]
        auto pair_sync = [&]() {                        // the 256 threads of this sub-tile
            asm volatile("bar.sync %0, %1;" ::"r"(1 + q), "r"(SOFTMAX_THREADS) : "memory");
        };
        // a barrier over the sub-tile's 256 threads that is true only if `v` is true for all:
        // a bounded wait that expired makes every thread of the sub-tile leave the loop at
        // the same tile, so the pairing barriers below stay matched
        auto pair_all = [&](bool v) -> bool {
            uint32_t r;
            asm volatile(
                "{\n\t.reg .pred pi, po;\n\t"
                "setp.ne.u32 pi, %1, 0;\n\t"
                "bar.red.and.pred po, %2, %3, pi;\n\t"
                "selp.u32 %0, 1, 0, po;\n\t}"
                : "=r"(r)
                : "r"((uint32_t)v), "r"(1 + q), "r"(SOFTMAX_THREADS)
                : "memory");
            return r != 0;
        };
        float m = -INFINITY, lsum = 0.f;                // lsum: this half's partial row sum
        bool ok = true;
        int fk = fstart - 1, jt = wk.tpf - 1, k = 0;
        while (wk.next(fk, jt)) {
            if (!active(q, fk)) continue;               // uniform over the sub-tile
            if (!pair_all(mbar_wait(BAR(B_SFULL + q), (uint32_t)k & 1u, abort_flag, p.err, DEVERR_ATTN_WAIT))) { ok = false; break; }
            fence_after_sync();
            const int nv = min(BN, p.N - jt * BN);
            const int nvh = min(64, max(0, nv - hf * 64));            // valid keys of this half
            const bool rok = row_valid && is_tap(fq, fk, p.w, p.r);
            const bool full = rok && nvh == 64;
            // this half of the S row in one TMEM round trip
            uint32_t sr[64];
            tmem_ld64(tlane + TM_S(q) + hf * 64, sr);
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (full) {
#pragma unroll
                for (int i = 0; i < 64; ++i) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(sr[i]));
            } else if (rok) {
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    mx[i & 3] = fmaxf(mx[i & 3], i < nvh ? __uint_as_float(sr[i]) : -INFINITY);
            }
            // agree on the row max with the other half (double-buffered by tile parity: a
            // slot is rewritten two tiles later, after the partner passed the next barrier)
            float *slot = xch + (k & 1) * (2 * BM);
            slot[hf * BM + row] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            pair_sync();                                // both halves also finished reading S
            const float mt = fmaxf(slot[row], slot[BM + row]);
            const float mnew = rok ? fmaxf(m, mt * p.sl2) : m;
            // grow the reference max only when it rose by more than 2^8 (lazy rescale)
            const bool need = rok && mnew > m + 8.f;
            const float muse = need ? mnew : m;
            const float alpha = (need && m != -INFINITY) ? ex2(m - mnew) : 1.f;
            // exponentials 32 keys at a time; bf16 pairs (key 2i in the low half) go to P
            // columns 32*hf + 16c .. +15 of S_q (S columns both halves have read). `full` and
            // `rok` differ between lanes whose rows straddle a frame boundary, so only the
            // arithmetic branches on them; every tcgen05.ld / st stays warp-uniform.
            float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t pk[16];
                if (full) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float p0 = ex2(fmaf(__uint_as_float(sr[c * 32 + 2 * i]), p.sl2, -muse));
                        const float p1 = ex2(fmaf(__uint_as_float(sr[c * 32 + 2 * i + 1]), p.sl2, -muse));
                        ps[i & 3] += p0 + p1;
                        pk[i] = pack_bf16(p0, p1);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int col = c * 32 + 2 * i;
                        float p0 = 0.f, p1 = 0.f;
                        if (rok) {
                            p0 = col < nvh ? ex2(fmaf(__uint_as_float(sr[col]), p.sl2, -muse)) : 0.f;
                            p1 = col + 1 < nvh ? ex2(fmaf(__uint_as_float(sr[col + 1]), p.sl2, -muse)) : 0.f;
                        }
                        ps[i & 3] += p0 + p1;
                        pk[i] = pack_bf16(p0, p1);
                    }
                }
                __syncwarp();                           // reconverge before .sync.aligned
                tmem_st16(tlane + TM_S(q) + hf * 32 + c * 16, pk);
            }
            // S_FULL completes only when every MMA issued before it has, so the previous PV
            // of this sub-tile is done: this half's columns of O may be rescaled (warp-wide
            // TMEM traffic, so the warp takes the branch together)
            if (k >= 1 && __any_sync(0xffffffffu, need && m != -INFINITY)) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t orow[32];
                    tmem_ld32(tlane + TM_O(q) + hf * 64 + c * 32, orow);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
                    tmem_st32(tlane + TM_O(q) + hf * 64 + c * 32, orow);
                }
            }
            lsum = lsum * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
            m = muse;
            tmem_wait_st();
            fence_before_sync();
            mbar_arrive(BAR(B_PFULL + q));
            ++k;
        }
        // final: both halves combine their partial sums and normalise their 64 columns of O
        const bool fin = ok && k >= 1 &&
                         __all_sync(0xffffffffu, mbar_wait(BAR(B_PVDONE + q), (uint32_t)(k - 1) & 1u, abort_flag, p.err, DEVERR_ATTN_WAIT));
        float *sums = xch + (k & 1) * (2 * BM);         // a slot no one reads any more
        sums[hf * BM + row] = lsum;
        pair_sync();
        if (fin) {
            fence_after_sync();
            const float tot = sums[row] + sums[BM + row];
            const float inv = tot > 0.f ? 1.f / tot : 0.f;
            __nv_bfloat16 *orow = p.o + (q_head + lrow) * D + hf * 64;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t ov[32];
                __syncwarp();
                tmem_ld32(tlane + TM_O(q) + hf * 64 + c * 32, ov);
                if (row_valid) {
                    uint32_t pk2[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk2[i] = pack_bf16(__uint_as_float(ov[2 * i]) * inv, __uint_as_float(ov[2 * i + 1]) * inv);
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[q4] = make_uint4(pk2[4 * q4], pk2[4 * q4 + 1], pk2[4 * q4 + 2], pk2[4 * q4 + 3]);
                }
            }
        }
    }

    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == WARP_MMA) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
}  // namespace

cudaError_t launch_attn_bf16_tc(const AttnArgs &a, cudaStream_t s)
{
    if (a.d != D) return cudaErrorNotSupported;
    cudaError_t e;
    const long q_total = (long)a.B * a.q_Htot * a.q_rows;
    const long kv_total = (long)a.B * a.kv_Htot * a.kv_rows;
    if (q_total + QT * BM >= (1L << 31) || kv_total + BN >= (1L << 31)) return cudaErrorNotSupported;
    CUtensorMap mq, mk, mv;
    // [rows][128] bf16 views, boxes of 128 rows x 64 columns, 128-byte swizzle
    if ((e = make_tmap_2d_bf16(&mq, a.q, q_total, D, 64, BM, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&mk, a.k, kv_total, D, 64, BN, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&mv, a.v, kv_total, D, 64, BN, true)) != cudaSuccess) return e;
    TcParams p;
    p.Hbr = a.Hbr; p.q_Htot = a.q_Htot; p.q_h0 = a.q_h0; p.kv_Htot = a.kv_Htot; p.kv_h0 = a.kv_h0;
    p.kv_slots = a.kv_slots; p.q_rows = a.q_rows; p.kv_rows = a.kv_rows;
    p.N = a.N; p.w = a.w; p.r = a.r; p.fq0 = a.fq0;
    p.sl2 = a.scale * 1.4426950408889634f;
    p.o = (__nv_bfloat16 *)a.o;
    p.err = a.err;
    e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((a.q_rows + QT * BM - 1) / (QT * BM)), (unsigned)(a.B * a.Hbr));
    attn_tc_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

}  // namespace hlta
