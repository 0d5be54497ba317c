// Windowed softmax attention (SWA / DSWA) on the sm_100a tensor cores, E4M3 operands: the
// kernel behind hlta_window_fp8_fwd. Head dim 128, fp32 accumulation in tensor memory.
// The design below was first built for bf16 and is written for both element types (template
// flag F8); only the E4M3 instantiation is launched: the bf16 entry points run attn_tc2.cu,
// whose 128-key tiles with P staged in shared memory measured faster in bf16.
//
// Exact attention by tiles with a running max and normaliser (llm-atlas long-context
// explainer, section 03 "Flash Attention": the score matrix never leaves the chip and the
// result equals the full softmax). The key set of a query tile is the union of the key
// frames of its rows' frames (sliding window: frames f-w+1..f; dilated: f, f-r, ...,
// f-r(w-1); Kairos abstract, item (2)); each key frame is walked in 64-token tiles and a
// per-element mask (row frame vs. key frame, ragged frame end) removes what a row must not
// see.
//
// One CTA = two 128-row query sub-tiles (256 consecutive query rows) of one head; 11 warps:
//   warps 0..3   softmax of sub-tile 0, warps 4..7 softmax of sub-tile 1, one thread per
//                query row (the warp's TMEM lane quadrant)
//   warp 8       TMA producer: Q (both sub-tiles) once, then 64-key K and V tiles into two
//                4-stage rings (128B swizzle), K two tiles ahead of V; the sub-tiles share
//                every K/V tile, and a stage is refilled once both sub-tiles released it
//   warps 9, 10  MMA issuers (tcgen05.mma kind::f16) of sub-tile 0 and 1; warp 9 owns the
//                TMEM allocation. One thread issues products at a limited rate (tens of
//                cycles each), so each sub-tile has its own issuing thread.
// Tensor memory: per sub-tile two S buffers of 64 columns and O (128 columns), 512 in all.
// S being double-buffered is what keeps the tensor pipe and the softmax apart: the MMA warp
// issues S_q for the sub-tile's next tile into the other buffer while the softmax works on the
// current one, so the softmax of consecutive tiles runs back to back. Per tile and sub-tile:
//   softmax: S_q[b] -> registers (one 64-column load), row max, P = 2^(s*scale*log2e - m) as
//            bf16 pairs written over the first 32 columns of S_q[b], P_FULL
//   MMA:     O_q += P_q[b] V_j (P read from tensor memory, V an MN-major smem operand),
//            then S_q for the tile two ahead into the same buffer (tcgen05.mma operations of
//            one thread execute in issue order, so the overwrite of P needs no wait)
// The running max lives per row (O rescaled in TMEM only when it grows by more than 2^8,
// after the previous P V of the sub-tile has completed). A key tile that no row of a
// sub-tile may see is skipped for that sub-tile. Every mbarrier wait is bounded; on expiry
// the kernel records DEVERR_ATTN_WAIT in the device error word, every role stops, and the
// TMEM allocation is released.
//
// E4M3 variant (template flag F8): q, k, v arrive as OCP E4M3 codes with fp32 scales: one per
// 128-row block of the head's query rows, one per 64-key tile of each key frame (the tiles
// the walk visits), one per value channel. Both products run as tcgen05.mma kind::f8f6f4
// (32 keys or head channels per instruction instead of 16): S from the codes, the softmax
// scales each tile's scores by sl2 * s_q * s_k (one multiply it already does), P is written
// as E4M3 codes (four per TMEM column) and the channel scales of V multiply the normalised
// output. P = 2^(x - m + 4) with the running max grown once it rose by more than 2^4, so P
// stays in [0, 256] (E4M3 reaches 448) and keeps normal precision down to 2^-6 of the max.
#include "hlta_internal.cuh"
#include "sm100_ptx.cuh"

#include <math.h>

namespace hlta {
namespace {

using namespace ptx;

constexpr int BM = 128;                 // query rows per sub-tile
constexpr int QT = 2;                   // query sub-tiles per CTA
constexpr int BN = 64;                  // keys per tile
constexpr int D = 128;                  // head dim
constexpr int NS = 4;                   // stages of each of the K and V rings
constexpr int LOOKAHEAD = 2;            // S is issued up to two tiles ahead of P V
constexpr int THREADS = 352;            // 8 softmax warps, TMA warp, two MMA warps
constexpr int WARP_TMA = 8, WARP_MMA = 9;   // MMA warps 9 (sub-tile 0, owns TMEM) and 10 (sub-tile 1)
constexpr int SOFTMAX_THREADS = 128;    // per sub-tile: one thread per query row
constexpr uint32_t QHALF = BM * 128;    // [128 rows][64 cols] bf16: 16 KB
constexpr uint32_t QTILE = 2 * QHALF;   // [128][128]
constexpr uint32_t KHALF = BN * 128;    // [64 rows][64 cols] bf16: 8 KB
constexpr uint32_t KTILE = 2 * KHALF;   // [64][128]
// bytes of one Q sub-tile and of one K or V tile as loaded: an E4M3 row is one 128-byte
// swizzle row, a bf16 row two 64-column halves. The shared-memory slots are sized for bf16.
template <bool F8> constexpr uint32_t q_bytes() { return F8 ? (uint32_t)BM * 128u : QTILE; }
template <bool F8> constexpr uint32_t kv_bytes() { return F8 ? (uint32_t)BN * 128u : KTILE; }
constexpr uint32_t TMEM_COLS = 512;     // S_0[0] @0, S_0[1] @64, S_1[0] @128, S_1[1] @192, O_0 @256, O_1 @384
__host__ __device__ constexpr uint32_t TM_S(int q, int b) { return (uint32_t)q * 128u + (uint32_t)b * 64u; }
__host__ __device__ constexpr uint32_t TM_O(int q) { return 256u + (uint32_t)q * 128u; }

// shared memory map (offsets from a 1024-byte aligned base)
__host__ __device__ constexpr uint32_t SM_Q(int q) { return (uint32_t)q * QTILE; }
__host__ __device__ constexpr uint32_t SM_K(int st) { return QT * QTILE + (uint32_t)st * KTILE; }
__host__ __device__ constexpr uint32_t SM_V(int st) { return QT * QTILE + (uint32_t)(NS + st) * KTILE; }
constexpr uint32_t SM_BAR = QT * QTILE + 2 * NS * KTILE;
// barriers (8 bytes each)
enum {
    B_QFULL = 0,
    B_KFULL = 1,                // + stage
    B_VFULL = B_KFULL + NS,     // + stage
    B_EMPTY = B_VFULL + NS,     // + stage: K and V of the stage consumed by both MMA warps
    B_SFULL = B_EMPTY + NS,     // + 2 * sub-tile + buffer
    B_PFULL = B_SFULL + 2 * QT, // + 2 * sub-tile + buffer (per buffer: the softmax may finish
                                //   the next tile before the MMA warp consumed this one)
    B_PVDONE = B_PFULL + 2 * QT, // + sub-tile
    B_ODONE = B_PVDONE + QT,    // + sub-tile: every product of the sub-tile has completed
    NBARS = B_ODONE + QT
};
constexpr uint32_t SM_TMEMSLOT = SM_BAR + 8 * NBARS;
constexpr uint32_t SM_ABORT = SM_TMEMSLOT + 4;
constexpr uint32_t SM_TOTAL = SM_ABORT + 4;
constexpr size_t SMEM_BYTES = SM_TOTAL + 1024;          // slack for the 1024-byte alignment

struct TcParams {
    int Hbr, q_Htot, q_h0, kv_Htot, kv_h0, kv_slots;
    long q_rows, kv_rows;
    int N, w, r, fq0;
    const int *fq0_dev;         // if set, the frame of query row 0 is read here (streaming steps)
    float sl2;                  // softmax scale * log2(e)
    const float *qs, *ks, *vs;  // E4M3 scales: [heads][nqb], [heads][nkb], [heads][128]
    int nqb, nkb;               // per head: query blocks of 128 rows, key tiles (slot * tpf + tile)
    float *lse;                 // per query row log-sum-exp (natural log) of its scores, or null
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

// kind::f8f6f4 forms (both operands E4M3 here; 32 elements of K per instruction)
__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
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

// Instruction descriptor for kind::f8f6f4: E4M3 A and B (format code 0), fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn, bool b_mn)
{
    return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
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

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&x)[8])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
        "r"(x[0]), "r"(x[1]), "r"(x[2]), "r"(x[3]), "r"(x[4]), "r"(x[5]), "r"(x[6]), "r"(x[7])
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


// packed fp32 pairs (sm_100 f32x2 instructions): half the issue slots of two scalar ops
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 pa, pb, pc, pd;\n\tmov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
        "mov.b64 pc, {%6, %7};\n\tfma.rn.f32x2 pd, pa, pb, pc;\n\tmov.b64 {%0, %1}, pd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 pa, pb, pd;\n\tmov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
        "add.rn.f32x2 pd, pa, pb;\n\tmov.b64 {%0, %1}, pd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// four E4M3 codes in one word, p0 in the lowest byte (the K order of a TMEM A operand);
// round to nearest even, saturating at 448
__device__ __forceinline__ uint32_t pack_e4m3x4(float p0, float p1, float p2, float p3)
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

// ---------------------------------------------------------------------------------------
// key-tile walk shared by every role (all roles must visit the same sequence)
// ---------------------------------------------------------------------------------------
// frame fk is a key frame of some query frame in [fa, fb]
__device__ __forceinline__ bool frame_needed(int fk, int fa, int fb, int w, int r)
{
    const int i0 = fa > fk ? (fa - fk + r - 1) / r : 0;
    return i0 < w && fk + r * i0 <= fb;
}

// The key-tile walk of a CTA: every 64-key tile of every frame some row of the CTA needs,
// frame by frame. A position carries the frame's sub-tile mask (bit q: sub-tile q needs the
// frame), computed once per frame, so stepping through the tiles of a frame costs an
// increment and a compare: the MMA warp's issue loop is serial code on one thread, and every
// instruction it spends between products is time the tensor pipe may run dry.
struct Walk {
    int fa0, fb0, fa1, fb1, fb, w, r, tpf;
    bool valid1;
    __device__ __forceinline__ int mask_of(int fk) const
    {
        return (frame_needed(fk, fa0, fb0, w, r) ? 1 : 0) |
               (valid1 && frame_needed(fk, fa1, fb1, w, r) ? 2 : 0);
    }
};
struct Pos {
    int fk, jt, mask, j;        // frame, tile in the frame, sub-tile mask, global tile index
    bool valid;
};
__device__ __forceinline__ Pos walk_start(const Walk &wk, int fstart)
{
    Pos c;
    c.fk = fstart - 1;
    c.jt = wk.tpf - 1;
    c.mask = 0;
    c.j = -1;
    c.valid = true;
    return c;
}
// the next tile of the walk (any sub-tile); false when done
__device__ __forceinline__ bool walk_step(const Walk &wk, Pos &c)
{
    ++c.j;
    if (++c.jt < wk.tpf) return true;
    for (++c.fk; c.fk <= wk.fb; ++c.fk) {
        const int m = wk.mask_of(c.fk);
        if (m) {
            c.mask = m;
            c.jt = 0;
            return true;
        }
    }
    return c.valid = false;
}
// the next tile of the walk whose frame sub-tile `want` (a mask bit) needs; false when done
__device__ __forceinline__ bool walk_next(const Walk &wk, Pos &c, int want)
{
    while (walk_step(wk, c)) {
        if (c.mask & want) return true;
        c.j += wk.tpf - 1 - c.jt;   // skip the rest of a frame this sub-tile does not need
        c.jt = wk.tpf - 1;
    }
    return false;
}

__device__ __forceinline__ bool is_tap(int fq, int fk, int w, int r)
{
    int dist = fq - fk;
    return dist >= 0 && dist <= r * (w - 1) && (dist % r) == 0;
}

// The kernel body of both variants; the tensor maps stay in the kernel's parameter space.
template <bool F8>
__device__ __forceinline__ void attn_body(const CUtensorMap &tq, const CUtensorMap &tk,
                                          const CUtensorMap &tv, const TcParams &p)
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
    // frame ranges of the two sub-tiles (sub-tile 1 may be empty in the last CTA of a head);
    // scalars, not arrays indexed by the sub-tile, so nothing lands in local memory
    const long r1_0 = min(l0 + BM, p.q_rows) - 1;
    const int fq0 = p.fq0_dev ? *p.fq0_dev : p.fq0;
    const int fa0 = fq0 + (int)(l0 / p.N), fb0 = fq0 + (int)(r1_0 / p.N);
    const bool valid1 = l0 + BM < p.q_rows;
    const int fa1 = valid1 ? fq0 + (int)((l0 + BM) / p.N) : fa0;
    const int fb1 = valid1 ? fq0 + (int)((min(l0 + 2 * BM, p.q_rows) - 1) / p.N) : fa1;
    Walk wk;
    wk.fa0 = fa0;
    wk.fb0 = fb0;
    wk.fa1 = fa1;
    wk.fb1 = fb1;
    wk.valid1 = valid1;
    wk.fb = valid1 ? fb1 : fb0;
    wk.w = p.w;
    wk.r = p.r;
    wk.tpf = (p.N + BN - 1) / BN;
    const int fstart = max(0, fa0 - p.r * (p.w - 1));
    // row of the K/V tensor maps where tile (fk, jt) starts
    auto kv_row = [&](int fk, int jt) {
        return (int)(kv_head + (long)(fk % p.kv_slots) * p.N + (long)jt * BN);
    };

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_QFULL), 1);
        for (int st = 0; st < NS; ++st) {
            mbar_init(BAR(B_KFULL + st), 1);
            mbar_init(BAR(B_VFULL + st), 1);
            mbar_init(BAR(B_EMPTY + st), 2);
        }
        for (int q = 0; q < QT; ++q) {
            mbar_init(BAR(B_SFULL + 2 * q), 1);
            mbar_init(BAR(B_SFULL + 2 * q + 1), 1);
            mbar_init(BAR(B_PFULL + 2 * q), SOFTMAX_THREADS);
            mbar_init(BAR(B_PFULL + 2 * q + 1), SOFTMAX_THREADS);
            mbar_init(BAR(B_PVDONE + q), 1);
            mbar_init(BAR(B_ODONE + q), 1);
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
        // step s loads K(s) and V(s - LOOKAHEAD): the MMA warp consumes K up to LOOKAHEAD
        // tiles ahead of V
        if (lane == 0) {
            mbar_expect_tx(BAR(B_QFULL), QT * q_bytes<F8>());
            for (int q = 0; q < QT; ++q) {
                const int qrow = (int)(q_head + l0 + q * BM);
                tma_load_2d(sbase + SM_Q(q), &tq, 0, qrow, BAR(B_QFULL));
                if (!F8) tma_load_2d(sbase + SM_Q(q) + QHALF, &tq, 64, qrow, BAR(B_QFULL));
            }
            Pos kp = walk_start(wk, fstart), vp = kp;
            int nk = 0, nv = 0;                     // K and V tiles issued
            bool more_k = true, more_v = true, ok = true;
            while (ok && (more_k || more_v)) {
                if (more_k && (more_k = walk_step(wk, kp))) {
                    const int st = nk % NS;
                    if (nk >= NS && !mbar_wait(BAR(B_EMPTY + st), (uint32_t)((nk / NS) + 1) & 1u, abort_flag, p.err, DEVERR_ATTN_WAIT)) { ok = false; break; }
                    mbar_expect_tx(BAR(B_KFULL + st), kv_bytes<F8>());
                    const int row = kv_row(kp.fk, kp.jt);
                    tma_load_2d(sbase + SM_K(st), &tk, 0, row, BAR(B_KFULL + st));
                    if (!F8) tma_load_2d(sbase + SM_K(st) + KHALF, &tk, 64, row, BAR(B_KFULL + st));
                    ++nk;
                }
                if (nv < nk - LOOKAHEAD || (!more_k && nv < nk)) {
                    more_v = walk_step(wk, vp);
                    const int st = nv % NS;
                    // the same release as K of this tile: complete already (the stage's next
                    // release needs this V, so the phase cannot have moved on)
                    if (nv >= NS && !mbar_wait(BAR(B_EMPTY + st), (uint32_t)((nv / NS) + 1) & 1u, abort_flag, p.err, DEVERR_ATTN_WAIT)) { ok = false; break; }
                    mbar_expect_tx(BAR(B_VFULL + st), kv_bytes<F8>());
                    const int row = kv_row(vp.fk, vp.jt);
                    tma_load_2d(sbase + SM_V(st), &tv, 0, row, BAR(B_VFULL + st));
                    if (!F8) tma_load_2d(sbase + SM_V(st) + KHALF, &tv, 64, row, BAR(B_VFULL + st));
                    ++nv;
                } else if (!more_k) {
                    more_v = false;
                }
            }
            if (*abort_flag) {
                // let this CTA's copies in flight land before the CTA may exit
                const long long t0 = clock64();
                for (int jj = nk - 1; jj >= 0 && jj >= nk - NS; --jj)
                    while (!mbar_try(BAR(B_KFULL + jj % NS), (uint32_t)(jj / NS) & 1u) && clock64() - t0 < (1LL << 31)) {}
                for (int jj = nv - 1; jj >= 0 && jj >= nv - NS; --jj)
                    while (!mbar_try(BAR(B_VFULL + jj % NS), (uint32_t)(jj / NS) & 1u) && clock64() - t0 < (1LL << 31)) {}
                while (!mbar_try(BAR(B_QFULL), 0) && clock64() - t0 < (1LL << 31)) {}
            }
        }
    } else if (warp == WARP_MMA || warp == WARP_MMA + 1) {
        // ------------------------------- MMA issuers ------------------------------------
        // One warp per sub-tile: a single thread issues tcgen05.mma at a limited rate, so the
        // two sub-tiles' products come from two threads. Each walks every tile of the CTA
        // (the release of a K/V stage needs both) and works on its sub-tile's tiles.
        if (lane == 0) {
            const int q = warp - WARP_MMA;
            const int want = 1 << q;
            // Q, K K-major; P (TMEM), V MN-major
            constexpr uint32_t IDESC_S = F8 ? idesc_e4m3(BM, BN, false, false) : idesc_bf16(BM, BN, false, false);
            constexpr uint32_t IDESC_O = F8 ? idesc_e4m3(BM, D, false, true) : idesc_bf16(BM, D, false, true);
            // Shared-memory descriptors built once; each product only adds a compile-time
            // offset (and the ring stage's) to the 14-bit start-address field.
            const uint64_t dq = sw128_desc(sbase + SM_Q(q), 16, 1024);
            const uint64_t dk0 = sw128_desc(sbase + SM_K(0), 16, 1024);
            const uint64_t dv0 = sw128_desc(sbase + SM_V(0), KHALF, 1024);
            const uint32_t s_tm = tmem + TM_S(q, 0), o_tm = tmem + TM_O(q);
            // waits that find their phase complete cost one try_wait, no call
            auto wait_bar = [&](uint32_t bar, uint32_t parity) -> bool {
                return mbar_try(bar, parity) || mbar_wait(bar, parity, abort_flag, p.err, DEVERR_ATTN_WAIT);
            };
            int ns = 0, npv = 0;                    // S and P V products issued
            Pos c = walk_start(wk, fstart);         // the next tile whose S is not issued yet
            walk_next(wk, c, want);
            // S = Q K^T for cursor tiles up to global index jmax while an S buffer is free
            // (at most two S ahead of P V; K of a tile more than LOOKAHEAD ahead of the walk
            // may wait on a stage this warp has not released yet)
            auto topup = [&](int jmax) -> bool {
                while (c.valid && c.j <= jmax && ns - npv < 2) {
                    const int st = c.j & (NS - 1);
                    if (!wait_bar(BAR(B_KFULL + st), (uint32_t)(c.j / NS) & 1u)) return false;
                    const int bf = ns & 1;
                    const uint64_t dk = dk0 + (uint64_t)((st * KTILE) >> 4);
                    if constexpr (F8) {
                        // 32 channels (32 bytes of the swizzle row) per instruction
#pragma unroll
                        for (int kk = 0; kk < D / 32; ++kk)
                            umma_f8(s_tm + bf * 64, dq + (uint64_t)(kk * 2), dk + (uint64_t)(kk * 2), IDESC_S, kk > 0 ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t qoff = ((kk >> 2) * QHALF + (kk & 3) * 32) >> 4;
                            const uint32_t koff = ((kk >> 2) * KHALF + (kk & 3) * 32) >> 4;
                            umma_bf16(s_tm + bf * 64, dq + qoff, dk + koff, IDESC_S, kk > 0 ? 1u : 0u);
                        }
                    }
                    umma_commit(BAR(B_SFULL + 2 * q + bf));
                    ++ns;
                    walk_next(wk, c, want);
                }
                return true;
            };
            bool ok = wait_bar(BAR(B_QFULL), 0);
            Pos t = walk_start(wk, fstart);
            while (ok && walk_step(wk, t)) {
                const int j = t.j, st = j & (NS - 1);
                ok = topup(j + LOOKAHEAD) && wait_bar(BAR(B_VFULL + st), (uint32_t)(j / NS) & 1u);
                if (!ok) break;
                if (t.mask & want) {
                    // O += P V with P in the first 32 (bf16) or 16 (E4M3) columns of the S buffer
                    const int bf = npv & 1;
                    if (!(ok = wait_bar(BAR(B_PFULL + 2 * q + bf), (uint32_t)(npv >> 1) & 1u))) break;
                    fence_after_sync();
                    const uint64_t dv = dv0 + (uint64_t)((st * KTILE) >> 4);
                    const uint32_t acc0 = npv > 0 ? 1u : 0u;
                    if constexpr (F8) {
                        // 32 keys per instruction: 8 TMEM columns of P, 32 V rows of 128 B
#pragma unroll
                        for (int kk = 0; kk < BN / 32; ++kk)
                            umma_f8_ts(o_tm, s_tm + bf * 64 + kk * 8, dv + (uint64_t)((kk * 4096) >> 4), IDESC_O,
                                       kk > 0 ? 1u : acc0);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < BN / 16; ++kk)
                            umma_bf16_ts(o_tm, s_tm + bf * 64 + kk * 8, dv + (uint64_t)((kk * 2048) >> 4), IDESC_O,
                                         kk > 0 ? 1u : acc0);
                    }
                    umma_commit(BAR(B_PVDONE + q));
                    ++npv;
                    // the buffer P V just read takes the S two tiles ahead (issue order)
                    if (!(ok = topup(j + LOOKAHEAD))) break;
                    // K_j (read by an S issued earlier) and V_j are consumed once these complete
                    umma_commit(BAR(B_EMPTY + st));
                } else {
                    // a tile only the other sub-tile needs: V_j has landed, so this stage's
                    // previous release is complete and the arrival belongs to this tile
                    mbar_arrive(BAR(B_EMPTY + st));
                }
            }
            if (ok) umma_commit(BAR(B_ODONE + q));
        }
    } else {
        // ------------------------------- softmax ----------------------------------------
        const int q = warp >> 2;                        // sub-tile of this warp
        const int quad = warp & 3;                      // TMEM lane quadrant of this warp
        const int row = quad * 32 + lane;
        const long lrow = l0 + q * BM + row;
        const bool row_valid = lrow < p.q_rows;
        const int fq = fq0 + (int)(lrow / p.N);
        const uint32_t tlane = tmem + ((uint32_t)(quad * 32) << 16);
        // E4M3: scores carry the Q block's scale (per sub-tile) and the K tile's (per tile);
        // sub-tile 1 of a head's last CTA may lie past the last query block
        const int kvh = b * p.kv_Htot + p.kv_h0 + h;
        const long qblk = l0 / BM + q;
        const float sl2q = !F8 ? p.sl2
                         : qblk < p.nqb ? p.sl2 * __ldg(p.qs + (long)(b * p.q_Htot + p.q_h0 + h) * p.nqb + qblk)
                                        : 0.f;
        constexpr float LAZY = F8 ? 4.f : 8.f;          // log2 growth of the max before a rescale
        constexpr float PBIAS = F8 ? 4.f : 0.f;         // P = 2^(x - m + PBIAS)
        float m = -INFINITY, lsum = 0.f;
        bool ok = true;
        int k = 0;
        Pos c = walk_start(wk, fstart);
        while (walk_next(wk, c, 1 << q)) {              // this sub-tile's tiles (uniform per warp)
            const int fk = c.fk, jt = c.jt;
            const int bf = k & 1;
            // the K tile's scale, fetched before the wait so its latency hides behind it
            const float sl2 = F8 ? sl2q * __ldg(p.ks + (long)kvh * p.nkb + (long)(fk % p.kv_slots) * wk.tpf + jt) : sl2q;
            const uint32_t sbar = BAR(B_SFULL + 2 * q + bf), spar = (uint32_t)(k >> 1) & 1u;
            if (!__all_sync(0xffffffffu, mbar_try(sbar, spar) || mbar_wait(sbar, spar, abort_flag, p.err, DEVERR_ATTN_WAIT))) { ok = false; break; }
            fence_after_sync();
            const int nv = min(BN, p.N - jt * BN);
            const bool rok = row_valid && is_tap(fq, fk, p.w, p.r);
            const bool full = rok && nv == BN;
            uint32_t sr[64];
            tmem_ld64(tlane + TM_S(q, bf), sr);
            // E4M3 fast path, taken when every row of the warp has a full tile and a reference
            // max already: the exponentials run against the reference max while the tile max
            // is taken in the same pass. A tile whose max rose more than 2^LAZY above the
            // reference (after a row's first tiles, rare) is redone by the general path below,
            // which grows the reference and rescales O; its P stores overwrite these. (With
            // E4M3 products the softmax is the longer side of the S -> P -> P V -> S cycle, so
            // the pass saved shows; the bf16 kernel is bound by the product issue and keeps
            // the two-pass form, measured no slower.)
            bool done = false;
            if (F8 && __all_sync(0xffffffffu, full && m != -INFINITY)) {
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                float2 ps2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                const float2 sl2x2 = make_float2(sl2, sl2), nm2 = make_float2(PBIAS - m, PBIAS - m);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    if constexpr (F8) {
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int col = c * 32 + 4 * i;
                            mx[i & 1] = fmax3(mx[i & 1], __uint_as_float(sr[col]), __uint_as_float(sr[col + 1]));
                            mx[2 + (i & 1)] = fmax3(mx[2 + (i & 1)], __uint_as_float(sr[col + 2]), __uint_as_float(sr[col + 3]));
                            const float2 xa = ffma2(make_float2(__uint_as_float(sr[col]), __uint_as_float(sr[col + 1])), sl2x2, nm2);
                            const float2 xb = ffma2(make_float2(__uint_as_float(sr[col + 2]), __uint_as_float(sr[col + 3])), sl2x2, nm2);
                            const float2 pa = make_float2(ex2(xa.x), ex2(xa.y));
                            const float2 pb = make_float2(ex2(xb.x), ex2(xb.y));
                            ps2[0] = fadd2(ps2[0], pa);
                            ps2[1] = fadd2(ps2[1], pb);
                            pk[i] = pack_e4m3x4(pa.x, pa.y, pb.x, pb.y);
                        }
                        tmem_st8(tlane + TM_S(q, bf) + c * 8, pk);
                    } else {
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int col = c * 32 + 2 * i;
                            mx[i & 3] = fmax3(mx[i & 3], __uint_as_float(sr[col]), __uint_as_float(sr[col + 1]));
                            const float2 x = ffma2(make_float2(__uint_as_float(sr[col]), __uint_as_float(sr[col + 1])), sl2x2, nm2);
                            const float2 pp = make_float2(ex2(x.x), ex2(x.y));
                            ps2[i & 1] = fadd2(ps2[i & 1], pp);
                            pk[i] = pack_bf16(pp.x, pp.y);
                        }
                        tmem_st16(tlane + TM_S(q, bf) + c * 16, pk);
                    }
                }
                const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                done = __all_sync(0xffffffffu, !(mt * sl2 > m + LAZY));
                if (done) lsum += (ps2[0].x + ps2[0].y) + (ps2[1].x + ps2[1].y);
            }
            if (!done) {
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if (full) {
    #pragma unroll
                    for (int i = 0; i < 32; ++i)
                        mx[i & 3] = fmax3(mx[i & 3], __uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]));
                } else if (rok) {
    #pragma unroll
                    for (int i = 0; i < 64; ++i)
                        mx[i & 3] = fmaxf(mx[i & 3], i < nv ? __uint_as_float(sr[i]) : -INFINITY);
                }
                const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                const float mnew = rok ? fmaxf(m, mt * sl2) : m;
                // grow the reference max only when it rose by more than 2^LAZY (lazy rescale)
                const bool need = rok && mnew > m + LAZY;
                const float muse = need ? mnew : m;
                const float alpha = (need && m != -INFINITY) ? ex2(m - mnew) : 1.f;
                // rescale O (warp-wide TMEM traffic, so the warp takes the branch together) once
                // the previous P V of this sub-tile, which accumulates into O, has completed. The
                // one before it has: S of this tile was issued behind it and has completed, so
                // the phase awaited here is the current or the next one, never older.
                if (k >= 1 && __any_sync(0xffffffffu, need && m != -INFINITY)) {
                    if (!__all_sync(0xffffffffu, mbar_wait(BAR(B_PVDONE + q), (uint32_t)(k - 1) & 1u, abort_flag, p.err, DEVERR_ATTN_WAIT))) { ok = false; break; }
                    fence_after_sync();
    #pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t orow[32];
                        tmem_ld32(tlane + TM_O(q) + c * 32, orow);
    #pragma unroll
                        for (int i = 0; i < 32; ++i)
                            orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
                        tmem_st32(tlane + TM_O(q) + c * 32, orow);
                    }
                }
                // exponentials 32 keys at a time; bf16 pairs (key 2i in the low half) or E4M3
                // quads (key 4i in the low byte) go to the first 32 or 16 columns of the S buffer.
                // `full` and `rok` differ between lanes whose rows straddle a frame boundary, so
                // only the arithmetic branches on them; every tcgen05.ld / st stays warp-uniform.
                float ps[4] = {0.f, 0.f, 0.f, 0.f};
                float2 ps2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                const float2 sl2x2 = make_float2(sl2, sl2), nm2 = make_float2(PBIAS - muse, PBIAS - muse);
    #pragma unroll
                for (int c = 0; c < 2; ++c) {
                    if constexpr (F8) {
                        uint32_t pk[8];
                        if (full) {
    #pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int col = c * 32 + 4 * i;
                                const float2 xa = ffma2(make_float2(__uint_as_float(sr[col]), __uint_as_float(sr[col + 1])), sl2x2, nm2);
                                const float2 xb = ffma2(make_float2(__uint_as_float(sr[col + 2]), __uint_as_float(sr[col + 3])), sl2x2, nm2);
                                const float2 pa = make_float2(ex2(xa.x), ex2(xa.y));
                                const float2 pb = make_float2(ex2(xb.x), ex2(xb.y));
                                ps2[0] = fadd2(ps2[0], pa);
                                ps2[1] = fadd2(ps2[1], pb);
                                pk[i] = pack_e4m3x4(pa.x, pa.y, pb.x, pb.y);
                            }
                        } else {
    #pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                float pv[4];
    #pragma unroll
                                for (int t = 0; t < 4; ++t) {
                                    const int col = c * 32 + 4 * i + t;
                                    pv[t] = rok && col < nv ? ex2(fmaf(__uint_as_float(sr[col]), sl2, PBIAS - muse)) : 0.f;
                                }
                                ps[i & 3] += (pv[0] + pv[1]) + (pv[2] + pv[3]);
                                pk[i] = pack_e4m3x4(pv[0], pv[1], pv[2], pv[3]);
                            }
                        }
                        __syncwarp();                       // reconverge before .sync.aligned
                        tmem_st8(tlane + TM_S(q, bf) + c * 8, pk);
                    } else {
                        uint32_t pk[16];
                        if (full) {
    #pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const float2 x = ffma2(make_float2(__uint_as_float(sr[c * 32 + 2 * i]), __uint_as_float(sr[c * 32 + 2 * i + 1])), sl2x2, nm2);
                                const float2 pp = make_float2(ex2(x.x), ex2(x.y));
                                ps2[i & 1] = fadd2(ps2[i & 1], pp);
                                pk[i] = pack_bf16(pp.x, pp.y);
                            }
                        } else {
    #pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int col = c * 32 + 2 * i;
                                float p0 = 0.f, p1 = 0.f;
                                if (rok) {
                                    p0 = col < nv ? ex2(fmaf(__uint_as_float(sr[col]), sl2, -muse)) : 0.f;
                                    p1 = col + 1 < nv ? ex2(fmaf(__uint_as_float(sr[col + 1]), sl2, -muse)) : 0.f;
                                }
                                ps[i & 3] += p0 + p1;
                                pk[i] = pack_bf16(p0, p1);
                            }
                        }
                        __syncwarp();                       // reconverge before .sync.aligned
                        tmem_st16(tlane + TM_S(q, bf) + c * 16, pk);
                    }
                }
                lsum = lsum * alpha + (((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps2[0].x + ps2[0].y) + (ps2[1].x + ps2[1].y)));
                m = muse;
            }
            tmem_wait_st();
            fence_before_sync();
            mbar_arrive(BAR(B_PFULL + 2 * q + bf));
            ++k;
        }
        // final: once every product of the sub-tile has completed (a one-phase barrier its MMA
        // warp commits after its last issue; the last two P V of this sub-tile may both still
        // run, so a parity wait on P_V_DONE would be ambiguous), normalise O and store it
        const bool fin = ok && k >= 1 &&
                         __all_sync(0xffffffffu, mbar_wait(BAR(B_ODONE + q), 0u, abort_flag, p.err, DEVERR_ATTN_WAIT));
        if (fin) {
            fence_after_sync();
            const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
            // the softmax normaliser for the backward pass: scores s, P = 2^(s sl2 - m) / lsum,
            // so log sum exp(s scale) = (m + log2(lsum)) ln 2 (the bf16 kernel only: PBIAS = 0)
            if (!F8 && p.lse && row_valid) p.lse[q_head + lrow] = (m + log2f(lsum)) * 0.69314718055994531f;
            __nv_bfloat16 *orow = p.o + (q_head + lrow) * D;
            const float4 *vsc = F8 ? reinterpret_cast<const float4 *>(p.vs + (long)kvh * D) : nullptr;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t ov[32];
                __syncwarp();
                tmem_ld32(tlane + TM_O(q) + c * 32, ov);
                if (row_valid) {
                    if constexpr (F8) {
                        // the value channels' scales (the same 32 floats for every lane)
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float4 sv = __ldg(vsc + c * 8 + i);
                            ov[4 * i] = __float_as_uint(__uint_as_float(ov[4 * i]) * sv.x);
                            ov[4 * i + 1] = __float_as_uint(__uint_as_float(ov[4 * i + 1]) * sv.y);
                            ov[4 * i + 2] = __float_as_uint(__uint_as_float(ov[4 * i + 2]) * sv.z);
                            ov[4 * i + 3] = __float_as_uint(__uint_as_float(ov[4 * i + 3]) * sv.w);
                        }
                    }
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

__global__ void __launch_bounds__(THREADS, 1)
attn_fp8_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const TcParams p)
{
    attn_body<true>(tq, tk, tv, p);
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------

template <bool F8>
cudaError_t launch_attn_tc(const AttnArgs &a, cudaStream_t s)
{
    if (a.d != D) return cudaErrorNotSupported;
    cudaError_t e;
    const long q_total = (long)a.B * a.q_Htot * a.q_rows;
    const long kv_total = (long)a.B * a.kv_Htot * a.kv_rows;
    if (q_total + QT * BM >= (1L << 31) || kv_total + BN >= (1L << 31)) return cudaErrorNotSupported;
    CUtensorMap mq, mk, mv;
    // [rows][128] views with 128-byte swizzle: bf16 in boxes of 64 columns, E4M3 in boxes of
    // the whole 128-byte row; 128 rows for Q, 64 for K and V
    if (F8) {
        if ((e = make_tmap_2d_u8(&mq, a.q, q_total, D, D, BM)) != cudaSuccess) return e;
        if ((e = make_tmap_2d_u8(&mk, a.k, kv_total, D, D, BN)) != cudaSuccess) return e;
        if ((e = make_tmap_2d_u8(&mv, a.v, kv_total, D, D, BN)) != cudaSuccess) return e;
    } else {
        if ((e = make_tmap_2d_bf16(&mq, a.q, q_total, D, 64, BM, true)) != cudaSuccess) return e;
        if ((e = make_tmap_2d_bf16(&mk, a.k, kv_total, D, 64, BN, true)) != cudaSuccess) return e;
        if ((e = make_tmap_2d_bf16(&mv, a.v, kv_total, D, 64, BN, true)) != cudaSuccess) return e;
    }
    TcParams p;
    p.Hbr = a.Hbr; p.q_Htot = a.q_Htot; p.q_h0 = a.q_h0; p.kv_Htot = a.kv_Htot; p.kv_h0 = a.kv_h0;
    p.kv_slots = a.kv_slots; p.q_rows = a.q_rows; p.kv_rows = a.kv_rows;
    p.N = a.N; p.w = a.w; p.r = a.r; p.fq0 = a.fq0; p.fq0_dev = a.fq0_dev;
    p.sl2 = a.scale * 1.4426950408889634f;
    p.qs = a.qs; p.ks = a.ks; p.vs = a.vs;
    p.lse = a.lse;
    p.nqb = (int)((a.q_rows + BM - 1) / BM);
    p.nkb = a.kv_slots * ((a.N + BN - 1) / BN);
    p.o = (__nv_bfloat16 *)a.o;
    p.err = a.err;
    if (F8 && (!p.qs || !p.ks || !p.vs)) return cudaErrorInvalidValue;
    static_assert(F8, "the bf16 entry points run attn_tc2.cu");
    auto kern = attn_fp8_kernel;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((a.q_rows + QT * BM - 1) / (QT * BM)), (unsigned)(a.B * a.Hbr));
    kern<<<grid, THREADS, SMEM_BYTES, s>>>(mq, mk, mv, p), note_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fp8_tc(const AttnArgs &a, cudaStream_t s) { return launch_attn_tc<true>(a, s); }

}  // namespace hlta
