// Windowed softmax attention (SWA / DSWA / streaming step), head dim 128, on the sm_100a
// tensor cores: 128-key tiles, two query sub-tiles per CTA, S decoupled from P. bf16 operands,
// or E4M3 codes with fp32 scales (template flag F8, below).
//
// Exact attention by tiles with a running max and normaliser (llm-atlas long-context
// explainer, section 03 "Flash Attention"); the key set of a query tile is the union of the
// key frames of its rows' frames (sliding window: frames f-w+1..f; dilated: f, f-r, ...,
// f-r(w-1); Kairos abstract, item (2)), walked frame by frame in tiles of up to 128 keys (the
// last tile of a frame holds N mod 128 keys; its products shrink to match), with a
// per-element mask (row frame vs. key frame, frame end).
//
// Why this shape. At d = 128 a (query, key) pair costs 4 d = 512 tensor FLOP and one
// exponential, and an SM runs 8192 bf16 FLOP and 16 exponentials per cycle, so the softmax
// of one tile takes as long as its two products; the products of tile t+1 must run while the
// softmax works on tile t. Here the scores S live in tensor memory and the probabilities P go
// to shared memory (the A operand of P V), so S of the next tile is issued as soon as the
// softmax has read this tile's scores into registers, not after P V: per sub-tile the softmax
// then runs tile after tile with its next scores already computed. 128-key tiles give every S
// product N = 128, which halves the products one issuing thread sends per key compared with
// 64-key tiles (one thread issues a tcgen05.mma in roughly a hundred cycles).
//
// Persistent: one CTA per SM (at most), each taking units of work from a launch-wide counter
// until none is left. A unit is two 128-row query sub-tiles (256 consecutive query rows) of
// one head of one of up to two branches (the hybrid's SWA and DSWA heads share one launch);
// units go head by head, the latest query rows of a head first (the longest key sets), so the
// last units handed out are the shortest. 11 warps:
//   warps 0-3 / 4-7  softmax of sub-tile 0 / 1, one thread per query row (its TMEM lane)
//   warp 8           TMA producer: takes the units and publishes each in shared memory; per
//                    unit Q, then K and V tiles of 128 keys through one ring of three 32 KB
//                    slots, in the order K0, K1, V0, K2, V1, ... (the order the MMA warps
//                    consume them); the ring runs on from one unit to the next
//   warps 9, 10      MMA issuers of sub-tile 0 / 1 (warp 9 owns the TMEM allocation). Each
//                    walks every tile in the ring's order: for K of a tile its sub-tile needs,
//                    S = Q K^T once the softmax freed the S buffer; for V, O += P V once P is in
//                    shared memory, committed in two halves of 64 keys so that the softmax can
//                    store the next tile's first half of P while it forms the second; a slot is
//                    released by both warps
// Tensor memory: per sub-tile S (128 columns) and O (128). Shared memory: Q (64 KB), the ring
// (96 KB), P per sub-tile ([128 rows][128 keys] bf16, 128-byte swizzle, 64 KB).
// O is rescaled in TMEM only when a row's max grows by more than 2^8 (exact: numerator and
// denominator use the same stale max). One pair in four of a tile's exponentials runs on the
// FMA pipe (a range-reduced cubic) instead of the exponential unit, which the remaining three
// keep busy: the unit and the issue slots are then closer to balanced.
// From one unit to the next: the producer loads the next Q once both issuers' last S of the
// unit completed; an issuer's first P V of a unit (which overwrites O) waits until its softmax
// read the previous unit's O; S, P and the ring's barriers keep counting across units. A
// second launch of the same kernel may share the counter (CTAs that start late, on SMs another
// kernel held); the last CTA to finish resets the counter.
//
// E4M3 instantiation (hlta_window_fp8_fwd): q, k, v arrive as OCP E4M3 codes, one 128-byte
// swizzled row per token, with fp32 scales: one per 128-row block of a head's query rows (one
// per sub-tile), one per 64-key run of each key frame (two per 128-key tile), one per value
// channel. Both products run as tcgen05.mma kind::f8f6f4, 32 elements of K per instruction
// (four products per S and per P V instead of eight); Q, the ring tiles and P take half the
// bytes, so the ring holds six tiles. The softmax scales each half of a tile's scores by
// sl2 * s_q * s_k of its run, forms P = 2^(x - m + 4) with the reference max grown once it
// rose by more than 2^4 (so P stays within [0, 256], inside E4M3's 448), rounds P to E4M3 codes
// (four a word, key order), and the value channels' scales multiply the normalised output.
//
// Every mbarrier wait is bounded; on expiry the kernel records DEVERR_ATTN_WAIT, every role
// stops, and the TMEM allocation is released.
#include "hlta_internal.cuh"
#include "sm100_ptx.cuh"
#include "tc_ptx.cuh"

#include <math.h>
#include <algorithm>
#include <atomic>

namespace hlta {
namespace {

using namespace ptx;

constexpr int BM = 128;                 // query rows per sub-tile
constexpr int QT = 2;                   // query sub-tiles per CTA
constexpr int BN = 128;                 // keys per tile
constexpr int D = 128;                  // head dim
constexpr int THREADS = 352;            // 8 softmax warps, TMA warp, two MMA warps
constexpr int WARP_TMA = 8, WARP_MMA = 9;
constexpr int SOFTMAX_THREADS = 128;    // per sub-tile
constexpr int UNIT_READERS = 2 + 8;     // the two MMA warps and the eight softmax warps
constexpr uint32_t QHALF = BM * 128;    // [128 rows][64 cols] bf16: 16 KB
constexpr uint32_t KHALF = BN * 128;    // [128 keys][64 cols] bf16: 16 KB
constexpr uint32_t PHALF = BM * 128;    // P: [128 rows][64 keys] bf16: 16 KB
constexpr uint32_t TMEM_COLS = 512;     // S_0 @0, S_1 @128, O_0 @256, O_1 @384
__host__ __device__ constexpr uint32_t TM_S(int q) { return (uint32_t)q * 128u; }
__host__ __device__ constexpr uint32_t TM_O(int q) { return 256u + (uint32_t)q * 128u; }

// Shared-memory layout per element type. bf16: a Q sub-tile, a K or V tile and a P sub-tile
// are two 128B-swizzled halves of 64 columns (32 KB); E4M3: one swizzled 128-byte row per
// token or query row (16 KB), and the ring holds twice as many tiles.
template <bool F8> struct Lay {
    static constexpr uint32_t QTILE = F8 ? BM * 128u : 2 * QHALF;
    static constexpr uint32_t KTILE = F8 ? BN * 128u : 2 * KHALF;
    static constexpr uint32_t PTILE = F8 ? BM * 128u : 2 * PHALF;
    static constexpr int NSLOT = F8 ? 6 : 3;    // ring slots (K and V tiles in consumption order)
    static constexpr uint32_t SM_Q(int q) { return (uint32_t)q * QTILE; }
    static constexpr uint32_t SM_SLOT(int i) { return QT * QTILE + (uint32_t)i * KTILE; }
    static constexpr uint32_t SM_P(int q) { return QT * QTILE + NSLOT * KTILE + (uint32_t)q * PTILE; }
    static constexpr uint32_t SM_BAR = QT * QTILE + NSLOT * KTILE + QT * PTILE;
    static constexpr int B_QFULL = 0;
    static constexpr int B_FULL = 1;                    // + slot
    static constexpr int B_EMPTY = B_FULL + NSLOT;      // + slot: both MMA warps done with it (count 2)
    static constexpr int B_SFULL = B_EMPTY + NSLOT;     // + sub-tile
    static constexpr int B_SFREE = B_SFULL + QT;        // + sub-tile: its softmax read S (count SOFTMAX_THREADS)
    static constexpr int B_PFULL = B_SFREE + QT;        // + sub-tile: P in shared memory (count SOFTMAX_THREADS)
    static constexpr int B_PVDONE = B_PFULL + QT;       // + sub-tile: P V complete
    static constexpr int B_ODONE = B_PVDONE + QT;       // + sub-tile: every product of the sub-tile has completed
    static constexpr int B_PVA = B_ODONE + QT;          // + sub-tile: the first half of P V (keys 0-63) complete
    static constexpr int B_QFREE = B_PVA + QT;          // both issuers' last S of a unit done (count 2)
    static constexpr int B_OFREE = B_QFREE + 1;         // + sub-tile: its epilogue read O (count SOFTMAX_THREADS)
    static constexpr int B_UFULL = B_OFREE + QT;        // + unit slot: the next unit published (count 1)
    static constexpr int B_UEMPTY = B_UFULL + 2;        // + unit slot: every role read it (count UNIT_READERS)
    static constexpr int NBARS = B_UEMPTY + 2;
    static constexpr uint32_t SM_UNIT = SM_BAR + 8 * NBARS;   // two published unit indices
    static constexpr uint32_t SM_TMEMSLOT = SM_UNIT + 8;
    static constexpr uint32_t SM_ABORT = SM_TMEMSLOT + 4;
    static constexpr uint32_t SM_TOTAL = SM_ABORT + 4;
    static constexpr size_t SMEM_BYTES = SM_TOTAL + 1024;
    static_assert(SMEM_BYTES <= 232448, "shared memory of one CTA");
};

// One branch of a launch: its heads (queries at q_h0.. of the query tensor, keys and values at
// kv_h0.. of its own key/value tensors), window and dilation.
struct BranchP {
    int Hbr, q_h0, kv_Htot, kv_h0, kv_slots, w, r;
    int nkb;                    // E4M3: key runs of 64 per head (kv_slots * ceil(N / 64))
    long kv_rows;
    const float *ks, *vs;       // E4M3 scales: [heads][nkb], [heads][128]
};
struct Params {
    BranchP br[2];
    int nbr, B, Hsum;           // branches; batch; heads over the branches
    int q_Htot;
    long q_rows;
    int N, fq0;
    const int *fq0_dev;
    float sl2;                  // softmax scale * log2(e)
    const float *qs;            // E4M3 query scales: [heads][nqb]
    int nqb;                    // E4M3: query blocks of 128 rows
    int nqt, nunits;            // query tiles of 256 rows per head; units = nqt * B * Hsum
    int *sched;                 // this launch's work counter: [0] next unit, [1] CTAs finished
    int ctas_total;             // CTAs over the launches sharing the counter
    float *lse;
    __nv_bfloat16 *o;
    unsigned int *err;
};

// packed fp32 pairs (sm_100 f32x2 instructions)
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

// kind::f8f6f4 product with both operands E4M3 in shared memory (32 elements of K per
// instruction), and its instruction descriptor (E4M3 = format code 0, fp32 accumulator)
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
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn, bool b_mn)
{
    return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// four E4M3 codes in one word, p0 in the lowest byte (key order along the row); round to
// nearest even, saturating at 448
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


// 2^x for a pair of values on the FMA pipe instead of the exponential unit (Cody-Waite range
// reduction and a polynomial): x + 1.5 * 2^23 rounds x to the nearest integer n in the low
// mantissa bits, f = x - n lies in [-1/2, 1/2], 2^f is a cubic fitted for minimum relative
// error on that interval (7.5e-5, below bf16's rounding of P), and n is added to the result's
// exponent bits. x is clamped below at -125 (masked -inf included) so the exponent stays normal.
constexpr float EXP2_C0 = 0.9999280571937561f, EXP2_C1 = 0.6932609677314758f;
constexpr float EXP2_C2 = 0.2426111400127411f, EXP2_C3 = 0.0551716573536396f;
__device__ __forceinline__ float2 exp2_fma2(float2 x)
{
    x.x = fmaxf(x.x, -125.f);
    x.y = fmaxf(x.y, -125.f);
    constexpr float SH = 12582912.f;                            // 1.5 * 2^23
    const float2 t = fadd2(x, make_float2(SH, SH));
    const float2 n = fadd2(t, make_float2(-SH, -SH));
    const float2 f = ffma2(n, make_float2(-1.f, -1.f), x);
    float2 q = ffma2(make_float2(EXP2_C3, EXP2_C3), f, make_float2(EXP2_C2, EXP2_C2));
    q = ffma2(q, f, make_float2(EXP2_C1, EXP2_C1));
    q = ffma2(q, f, make_float2(EXP2_C0, EXP2_C0));
    return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// ---------------------------------------------------------------------------------------
// key-tile walk shared by every role (all roles visit the same sequence)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ bool frame_needed(int fk, int fa, int fb, int w, int r)
{
    const int i0 = fa > fk ? (fa - fk + r - 1) / r : 0;
    return i0 < w && fk + r * i0 <= fb;
}
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
__device__ __forceinline__ bool is_tap(int fq, int fk, int w, int r)
{
    const int dist = fq - fk;
    return dist >= 0 && dist <= r * (w - 1) && (dist % r) == 0;
}

// Work counters of the persistent launches whose caller passes none, one pair per launch slot,
// used in turn: [0] the next unit to take, [1] the CTAs that finished. The last CTA of a launch
// to finish puts both back to zero for the counter's next launch, so a slot serves any launch
// that starts after the one SCHED_SLOTS launches earlier has finished.
constexpr int SCHED_SLOTS = 64;
__device__ int g_attn_sched[SCHED_SLOTS][2];

// One unit of work: 256 consecutive query rows (two sub-tiles) of one (rollout, head).
struct Unit {
    long l0, q_head, kv_head;
    int bi, qh, kvh;            // branch; query head and key/value head (rollout included)
    int fa0, fb0, fa1, fb1, fstart;
    bool valid1;
    Walk wk;
};
__device__ __forceinline__ Unit unit_of(const Params &p, int u, int fq0)
{
    Unit c;
    const int bh = u / p.nqt;
    const int b = bh / p.Hsum;
    int h = bh % p.Hsum;
    c.bi = p.nbr > 1 && h >= p.br[0].Hbr ? 1 : 0;
    if (c.bi) h -= p.br[0].Hbr;
    const BranchP &br = p.br[c.bi];
    c.l0 = (long)(p.nqt - 1 - u % p.nqt) * (QT * BM);
    c.qh = b * p.q_Htot + br.q_h0 + h;
    c.kvh = b * br.kv_Htot + br.kv_h0 + h;
    c.q_head = (long)c.qh * p.q_rows;
    c.kv_head = (long)c.kvh * br.kv_rows;
    const long r1_0 = min(c.l0 + BM, p.q_rows) - 1;
    c.fa0 = fq0 + (int)(c.l0 / p.N);
    c.fb0 = fq0 + (int)(r1_0 / p.N);
    c.valid1 = c.l0 + BM < p.q_rows;
    c.fa1 = c.valid1 ? fq0 + (int)((c.l0 + BM) / p.N) : c.fa0;
    c.fb1 = c.valid1 ? fq0 + (int)((min(c.l0 + 2 * BM, p.q_rows) - 1) / p.N) : c.fa1;
    c.wk.fa0 = c.fa0;
    c.wk.fb0 = c.fb0;
    c.wk.fa1 = c.fa1;
    c.wk.fb1 = c.fb1;
    c.wk.valid1 = c.valid1;
    c.wk.fb = c.valid1 ? c.fb1 : c.fb0;
    c.wk.w = br.w;
    c.wk.r = br.r;
    c.wk.tpf = (p.N + BN - 1) / BN;
    c.fstart = max(0, c.fa0 - br.r * (br.w - 1));
    return c;
}

template <bool F8>
__global__ void __launch_bounds__(THREADS, 1)
attn_tc2_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk0,
                const __grid_constant__ CUtensorMap tv0, const __grid_constant__ CUtensorMap tk1,
                const __grid_constant__ CUtensorMap tv1, const __grid_constant__ Params p)
{
    using LY = Lay<F8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + LY::SM_BAR;
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    volatile int *abort_flag = (volatile int *)(smem + LY::SM_ABORT);
    uint32_t *tmem_slot = (uint32_t *)(smem + LY::SM_TMEMSLOT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int fq0 = p.fq0_dev ? *p.fq0_dev : p.fq0;
    volatile int *unit_slot = (volatile int *)(smem + LY::SM_UNIT);
    auto kv_row = [&](const Unit &c, int fk, int jt) {
        return (int)(c.kv_head + (long)(fk % p.br[c.bi].kv_slots) * p.N + (long)jt * BN);
    };
    auto nkeys = [&](int jt) { return min(BN, p.N - jt * BN); };

    if (threadIdx.x == 0) {
        mbar_init(BAR(LY::B_QFULL), 1);
        for (int i = 0; i < LY::NSLOT; ++i) {
            mbar_init(BAR(LY::B_FULL + i), 1);
            mbar_init(BAR(LY::B_EMPTY + i), 2);
        }
        for (int q = 0; q < QT; ++q) {
            mbar_init(BAR(LY::B_SFULL + q), 1);
            mbar_init(BAR(LY::B_SFREE + q), SOFTMAX_THREADS);
            mbar_init(BAR(LY::B_PFULL + q), SOFTMAX_THREADS);
            mbar_init(BAR(LY::B_PVDONE + q), 1);
            mbar_init(BAR(LY::B_PVA + q), 1);
            mbar_init(BAR(LY::B_ODONE + q), 1);
            mbar_init(BAR(LY::B_OFREE + q), SOFTMAX_THREADS);
        }
        mbar_init(BAR(LY::B_QFREE), 2);
        for (int i = 0; i < 2; ++i) {
            mbar_init(BAR(LY::B_UFULL + i), 1);
            mbar_init(BAR(LY::B_UEMPTY + i), UNIT_READERS);
        }
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == WARP_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    auto wait_bar = [&](uint32_t bar, uint32_t parity) -> bool {
        return mbar_try(bar, parity) || mbar_wait(bar, parity, abort_flag, p.err, DEVERR_ATTN_WAIT);
    };
    // The ring's items in order: K of tile 0, then K of tile j + 1 and V of tile j for j = 0, 1,
    // ...; item i sits in slot i % NSLOT. K(j) is item 2j - 1 (j >= 1), V(j) is item 2j + 2
    // (2j + 1 when tile j + 1 does not exist, i.e. for the last tile).

    if (warp == WARP_TMA) {
        // ------------------------------- TMA producer -----------------------------------
        // Takes the units of this CTA from the launch's work counter and publishes each in a
        // shared slot (two, used in turn); then loads the unit's Q (once both issuers' last S
        // of the previous unit completed) and streams its K and V tiles into the ring, which
        // runs on from one unit to the next.
        if (lane == 0) {
            int it = 0;                                  // ring items issued
            int nq = 0;                                  // Q loads issued
            bool ok = true;
            auto load = [&](const CUtensorMap *map, int row) -> bool {
                const int sl = it % LY::NSLOT;
                if (it >= LY::NSLOT && !wait_bar(BAR(LY::B_EMPTY + sl), (uint32_t)((it / LY::NSLOT) + 1) & 1u)) return false;
                mbar_expect_tx(BAR(LY::B_FULL + sl), LY::KTILE);
                tma_load_2d(sbase + LY::SM_SLOT(sl), map, 0, row, BAR(LY::B_FULL + sl));
                if constexpr (!F8) tma_load_2d(sbase + LY::SM_SLOT(sl) + KHALF, map, 64, row, BAR(LY::B_FULL + sl));
                ++it;
                return true;
            };
            for (int i = 0; ok; ++i) {
                const int us = i & 1;
                if (i >= 2 && !(ok = wait_bar(BAR(LY::B_UEMPTY + us), (uint32_t)((i - 2) >> 1) & 1u))) break;
                const int u0 = atomicAdd(&p.sched[0], 1);
                const int u = u0 < p.nunits ? u0 : -1;
                unit_slot[us] = u;
                mbar_arrive(BAR(LY::B_UFULL + us));
                if (u < 0) break;
                const Unit c = unit_of(p, u, fq0);
                if (i >= 1 && !(ok = wait_bar(BAR(LY::B_QFREE), (uint32_t)(i - 1) & 1u))) break;
                mbar_expect_tx(BAR(LY::B_QFULL), QT * LY::QTILE);
                for (int q = 0; q < QT; ++q) {
                    const int qrow = (int)(c.q_head + c.l0 + q * BM);
                    tma_load_2d(sbase + LY::SM_Q(q), &tq, 0, qrow, BAR(LY::B_QFULL));
                    if constexpr (!F8) tma_load_2d(sbase + LY::SM_Q(q) + QHALF, &tq, 64, qrow, BAR(LY::B_QFULL));
                }
                ++nq;
                const CUtensorMap *tk = c.bi ? &tk1 : &tk0, *tv = c.bi ? &tv1 : &tv0;
                Pos kp = walk_start(c.wk, c.fstart), vp = kp;
                if (walk_step(c.wk, kp)) ok = load(tk, kv_row(c, kp.fk, kp.jt));
                while (ok && walk_step(c.wk, vp)) {
                    if (walk_step(c.wk, kp) && !(ok = load(tk, kv_row(c, kp.fk, kp.jt)))) break;
                    if (!(ok = load(tv, kv_row(c, vp.fk, vp.jt)))) break;
                }
            }
            if (*abort_flag) {
                // a bounded wait expired somewhere: let the copies this CTA issued land
                const long long t0 = clock64();
                for (int ii = it - 1; ii >= 0 && ii >= it - LY::NSLOT; --ii)
                    while (!mbar_try(BAR(LY::B_FULL + ii % LY::NSLOT), (uint32_t)(ii / LY::NSLOT) & 1u) && clock64() - t0 < (1LL << 31)) {}
                if (nq > 0)
                    while (!mbar_try(BAR(LY::B_QFULL), (uint32_t)(nq - 1) & 1u) && clock64() - t0 < (1LL << 31)) {}
            }
        }
    } else if (warp == WARP_MMA || warp == WARP_MMA + 1) {
        // ------------------------------- MMA issuers ------------------------------------
        if (lane == 0) {
            const int q = warp - WARP_MMA;
            Walk wk;
            const int want = 1 << q;
            constexpr uint32_t IDESC_S0 = (F8 ? idesc_e4m3(BM, 16, false, false) : tc::idesc_bf16(BM, 16, false, false)) & ~(0x3Fu << 17);
            constexpr uint32_t IDESC_O = F8 ? idesc_e4m3(BM, D, false, true) : tc::idesc_bf16(BM, D, false, true);
            const uint64_t dq = tc::sw128_desc(sbase + LY::SM_Q(q), 16, 1024);
            const uint64_t dsl0 = tc::sw128_desc(sbase + LY::SM_SLOT(0), 16, 1024);        // K-major (K)
            const uint64_t dvl0 = tc::sw128_desc(sbase + LY::SM_SLOT(0), KHALF, 1024);     // MN-major (V)
            const uint64_t dp = tc::sw128_desc(sbase + LY::SM_P(q), 16, 1024);
            const uint32_t s_tm = tmem + TM_S(q), o_tm = tmem + TM_O(q);
            int it = 0, ns = 0, npv = 0;
            int npv0 = 0;                   // P V products issued before the current unit
            bool ok = true;
            int ui = 0;                     // units taken
            // the first P V of a unit overwrites O: the previous unit's epilogue must have read it
            auto ofree = [&]() -> bool {
                return ui < 1 || wait_bar(BAR(LY::B_OFREE + q), (uint32_t)(ui - 1) & 1u);
            };
            // K of tile u (ring item `it`): S = Q K^T once this sub-tile's softmax read the
            // previous S (N = the tile's keys rounded up to 16), then the slot released
            auto handle_k = [&](const Pos &u) -> bool {
                const int sl = it % LY::NSLOT;
                if (!wait_bar(BAR(LY::B_FULL + sl), (uint32_t)(it / LY::NSLOT) & 1u)) return false;
                if (u.mask & want) {
                    if (ns > 0 && !wait_bar(BAR(LY::B_SFREE + q), (uint32_t)(ns - 1) & 1u)) return false;
                    tc::fence_after_sync();
                    const int n16 = (nkeys(u.jt) + 15) & ~15;
                    const uint32_t idesc = IDESC_S0 | ((uint32_t)(n16 >> 3) << 17);
                    const uint64_t dk = dsl0 + (uint64_t)((sl * LY::KTILE) >> 4);
                    if constexpr (F8) {
                        // 32 channels (32 bytes of the swizzled row) per instruction
#pragma unroll
                        for (int kk = 0; kk < D / 32; ++kk)
                            umma_f8(s_tm, dq + (uint64_t)(kk * 2), dk + (uint64_t)(kk * 2), idesc, kk > 0 ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t off = (uint64_t)((((kk >> 2) * QHALF + (kk & 3) * 32) >> 4));
                            const uint64_t koff = (uint64_t)((((kk >> 2) * KHALF + (kk & 3) * 32) >> 4));
                            tc::umma_bf16(s_tm, dq + off, dk + koff, idesc, kk > 0 ? 1u : 0u);
                        }
                    }
                    tc::umma_commit(BAR(LY::B_SFULL + q));
                    tc::umma_commit(BAR(LY::B_EMPTY + sl));
                    ++ns;
                } else {
                    mbar_arrive(BAR(LY::B_EMPTY + sl));
                }
                ++it;
                return true;
            };
            // V of tile t: O += P V once P is in shared memory, then the slot released
            auto handle_v = [&](const Pos &t) -> bool {
                const int sl = it % LY::NSLOT;
                if (!wait_bar(BAR(LY::B_FULL + sl), (uint32_t)(it / LY::NSLOT) & 1u)) return false;
                if (t.mask & want) {
                    if (!wait_bar(BAR(LY::B_PFULL + q), (uint32_t)npv & 1u)) return false;
                    if (npv == npv0 && !ofree()) return false;
                    tc::fence_after_sync();
                    const uint64_t dv = dvl0 + (uint64_t)((sl * LY::KTILE) >> 4);
                    if constexpr (F8) {
                        // 32 keys per instruction: 32 bytes of each P row, 32 V rows of 128 B
                        const int ksteps = (nkeys(t.jt) + 31) >> 5;
                        for (int kk = 0; kk < ksteps; ++kk) {
                            umma_f8(o_tm, dp + (uint64_t)(kk * 2), dv + (uint64_t)((kk * 4096) >> 4), IDESC_O,
                                    (npv > npv0 || kk > 0) ? 1u : 0u);
                            if (kk == 1 && ksteps == BN / 32) tc::umma_commit(BAR(LY::B_PVA + q));
                        }
                        if (ksteps < BN / 32) tc::umma_commit(BAR(LY::B_PVA + q));
                    } else {
                    const int ksteps = (nkeys(t.jt) + 15) >> 4;
                    if (ksteps == BN / 16 && npv > npv0) {
                        // the first half of P (keys 0-63) is released once its products are
                        // done, so the softmax can store the next tile's first half early
#pragma unroll
                        for (int kk = 0; kk < BN / 16; ++kk) {
                            const uint64_t poff = (uint64_t)((((kk >> 2) * PHALF + (kk & 3) * 32) >> 4));
                            tc::umma_bf16(o_tm, dp + poff, dv + (uint64_t)((kk * 2048) >> 4), IDESC_O, 1u);
                            if (kk == BN / 32 - 1) tc::umma_commit(BAR(LY::B_PVA + q));
                        }
                    } else {
                        for (int kk = 0; kk < ksteps; ++kk) {
                            const uint64_t poff = (uint64_t)((((kk >> 2) * PHALF + (kk & 3) * 32) >> 4));
                            tc::umma_bf16(o_tm, dp + poff, dv + (uint64_t)((kk * 2048) >> 4), IDESC_O,
                                          (npv > npv0 || kk > 0) ? 1u : 0u);
                        }
                        tc::umma_commit(BAR(LY::B_PVA + q));
                    }
                    }
                    tc::umma_commit(BAR(LY::B_PVDONE + q));
                    tc::umma_commit(BAR(LY::B_EMPTY + sl));
                    ++npv;
                } else {
                    mbar_arrive(BAR(LY::B_EMPTY + sl));
                }
                ++it;
                return true;
            };
            for (; ok; ++ui) {
                const int us = ui & 1;
                if (!(ok = wait_bar(BAR(LY::B_UFULL + us), (uint32_t)(ui >> 1) & 1u))) break;
                const int un = unit_slot[us];
                mbar_arrive(BAR(LY::B_UEMPTY + us));
                if (un < 0) break;
                const Unit c = unit_of(p, un, fq0);
                wk = c.wk;
                if (!(ok = wait_bar(BAR(LY::B_QFULL), (uint32_t)ui & 1u))) break;
                tc::fence_after_sync();
                npv0 = npv;
                Pos t = walk_start(wk, c.fstart);
                bool have = walk_step(wk, t);
                if (have) ok = handle_k(t);
                else tc::umma_commit(BAR(LY::B_QFREE));       // a unit without tiles
                while (ok && have) {
                    Pos u = t;
                    const bool next = walk_step(wk, u);
                    if (next) ok = handle_k(u);           // K(t + 1) before V(t)
                    else tc::umma_commit(BAR(LY::B_QFREE));   // the unit's last S was issued
                    if (!ok) break;
                    if (!(ok = handle_v(t))) break;
                    have = next;
                    t = u;
                }
                if (!ok) break;
                // a unit without a P V of this sub-tile still waits for the previous epilogue,
                // so that its completion below never runs two units ahead of the softmax
                if (npv == npv0 && !(ok = ofree())) break;
                tc::umma_commit(BAR(LY::B_ODONE + q));
            }
        }
    } else {
        // ------------------------------- softmax ----------------------------------------
        // The loop keeps little besides the 128 scores of a row: its own walk over the
        // sub-tile's key frames (frame, tile), the running max and sum, and 32-bit addresses.
        const int q = warp >> 2;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t tlane = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t prow = sbase + LY::SM_P(q) + (uint32_t)row * 128u;
        const uint32_t rx = (uint32_t)(row & 7);
        const int tpf64 = (p.N + 63) / 64;
        // log2 growth of the max before a rescale; E4M3: P = 2^(x - m + 4) stays within 2^8
        constexpr float LAZY = F8 ? 4.f : 8.f;
        constexpr float PBIAS = F8 ? 4.f : 0.f;
        bool ok = true;
        int k = 0;                      // tiles of this sub-tile over every unit so far
        for (int ui = 0; ok; ++ui) {
        const int us = ui & 1;
        if (!__all_sync(0xffffffffu, wait_bar(BAR(LY::B_UFULL + us), (uint32_t)(ui >> 1) & 1u))) { ok = false; break; }
        const int un = unit_slot[us];
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(LY::B_UEMPTY + us));
        if (un < 0) break;
        const Unit c = unit_of(p, un, fq0);
        const Walk &wk = c.wk;
        const long lrow = c.l0 + q * BM + row;
        const bool row_valid = lrow < p.q_rows;
        const int fq = fq0 + (int)(lrow / p.N);
        // E4M3: the scores carry the Q block's scale (one per sub-tile; sub-tile 1 of a head's
        // last unit may lie past the last query block) and each 64-key run's K scale
        const BranchP &br = p.br[c.bi];
        float sl2 = p.sl2;
        if constexpr (F8) {
            const long qblk = c.l0 / BM + q;
            sl2 = qblk < p.nqb ? p.sl2 * __ldg(p.qs + (long)c.qh * p.nqb + qblk) : 0.f;
        }
        const int faq = q == 0 ? c.fa0 : c.fa1, fbq = q == 0 ? c.fb0 : c.fb1;
        const bool qvalid = q == 0 || c.valid1;
        float m = -INFINITY, lsum = 0.f;
        const int k0 = k;
        int fk = c.fstart - 1, jt = wk.tpf - 1;
        while (qvalid) {
            // the next tile of this sub-tile: the same frames and order as the MMA warp's walk
            if (++jt >= wk.tpf) {
                for (++fk; fk <= fbq && !frame_needed(fk, faq, fbq, wk.w, wk.r); ++fk) {}
                if (fk > fbq) break;
                jt = 0;
            }
            float sla = sl2, slb = sl2;          // the scales of keys 0-63 and 64-127
            if constexpr (F8) {
                const long kb = (long)c.kvh * br.nkb + (long)(fk % br.kv_slots) * tpf64 + 2 * jt;
                sla = sl2 * __ldg(br.ks + kb);
                slb = 2 * jt + 1 < tpf64 ? sl2 * __ldg(br.ks + kb + 1) : sla;
            }
            if (!__all_sync(0xffffffffu, wait_bar(BAR(LY::B_SFULL + q), (uint32_t)k & 1u))) { ok = false; break; }
            tc::fence_after_sync();
            const int nv = nkeys(jt);
            const bool rok = row_valid && is_tap(fq, fk, wk.w, wk.r);
            // the tile's scores into registers, then the S buffer is free for the next tile
            uint32_t sa[64], sb[64];
            tc::tmem_ld64(tlane + TM_S(q), sa);
            tc::tmem_ld64(tlane + TM_S(q) + 64, sb);
            tc::fence_before_sync();
            mbar_arrive(BAR(LY::B_SFREE + q));
            // masked keys (past the frame's end, or a frame this row does not attend) become
            // -inf, so the exponentials below serve full, partial and masked tiles alike (the
            // warp takes the masking branch together: rok differs between rows only where the
            // sub-tile straddles a frame)
            const int lim = rok ? nv : 0;
            if (__any_sync(0xffffffffu, lim < BN)) {
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    if (i >= lim) sa[i] = __float_as_uint(-INFINITY);
                    if (64 + i >= lim) sb[i] = __float_as_uint(-INFINITY);
                }
            }
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                mx0 = fmax3(mx0, __uint_as_float(sa[2 * i]), __uint_as_float(sa[2 * i + 1]));
                mx1 = fmax3(mx1, __uint_as_float(sb[2 * i]), __uint_as_float(sb[2 * i + 1]));
            }
            float mt;
            if constexpr (F8) mt = fmaxf(mx0 * sla, mx1 * slb);
            else mt = fmaxf(mx0, mx1) * sl2;
            const float mnew = rok ? fmaxf(m, mt) : m;
            const bool need = rok && mnew > m + LAZY;
            const float muse = need ? mnew : m;
            const float alpha = (need && m != -INFINITY) ? tc::ex2(m - mnew) : 1.f;
            // P = 2^(s sl2 - m) as bf16 pairs, first into registers: the shared P tile is still
            // the A operand of the previous tile's P V until that product completes
            const float negm = muse == -INFINITY ? 0.f : PBIAS - muse;
            const float2 sl2x2 = make_float2(sla, sla), nm2 = make_float2(negm, negm);
            float2 ps2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            uint32_t pk[64];
            if constexpr (F8) {
                // E4M3 codes, four keys a word: keys 0-63 in words 0-15 (the first four 16-byte
                // chunks of the row), keys 64-127 in words 16-31
                const float2 slb2 = make_float2(slb, slb);
                auto store_half8 = [&](int half) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int ch = half * 4 + c;
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                                         prow + ((((uint32_t)ch) ^ rx) << 4)),
                                     "r"(pk[ch * 4]), "r"(pk[ch * 4 + 1]), "r"(pk[ch * 4 + 2]), "r"(pk[ch * 4 + 3])
                                     : "memory");
                    }
                };
                // the second pair of every other quad on the FMA pipe (one pair in four; its
                // floor of 2^-125 rounds to an E4M3 zero)
                auto quad8 = [&](const uint32_t *sv, int i, float2 scl) {
                    const float2 xa = ffma2(make_float2(__uint_as_float(sv[4 * i]), __uint_as_float(sv[4 * i + 1])), scl, nm2);
                    const float2 xb = ffma2(make_float2(__uint_as_float(sv[4 * i + 2]), __uint_as_float(sv[4 * i + 3])), scl, nm2);
                    const float2 pa = make_float2(tc::ex2(xa.x), tc::ex2(xa.y));
                    const float2 pb = (i & 1) ? exp2_fma2(xb) : make_float2(tc::ex2(xb.x), tc::ex2(xb.y));
                    ps2[0] = fadd2(ps2[0], pa);
                    ps2[1] = fadd2(ps2[1], pb);
                    return pack_e4m3x4(pa.x, pa.y, pb.x, pb.y);
                };
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = quad8(sa, i, sl2x2);
                const bool resc = k >= 1 && __any_sync(0xffffffffu, need && m != -INFINITY);
                if (k >= 1 && !__all_sync(0xffffffffu, wait_bar(BAR(LY::B_PVA + q), (uint32_t)(k - 1) & 1u))) { ok = false; break; }
                if (!resc) store_half8(0);
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[16 + i] = quad8(sb, i, slb2);
                if (k >= 1 && !__all_sync(0xffffffffu, wait_bar(BAR(LY::B_PVDONE + q), (uint32_t)(k - 1) & 1u))) { ok = false; break; }
                tc::fence_after_sync();
                if (resc) {
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t orow[32];
                        tc::tmem_ld32(tlane + TM_O(q) + cc * 32, orow);
#pragma unroll
                        for (int i = 0; i < 32; ++i) orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
                        tc::tmem_st32(tlane + TM_O(q) + cc * 32, orow);
                    }
                    tc::tmem_wait_st();
                    tc::fence_before_sync();
                    store_half8(0);
                }
                store_half8(1);
                lsum = lsum * alpha + ((ps2[0].x + ps2[0].y) + (ps2[1].x + ps2[1].y));
                m = muse;
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(BAR(LY::B_PFULL + q));
                ++k;
                continue;
            }
            auto store_half = [&](int half) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                                     prow + (uint32_t)half * PHALF + ((((uint32_t)ch) ^ rx) << 4)),
                                 "r"(pk[half * 32 + ch * 4]), "r"(pk[half * 32 + ch * 4 + 1]),
                                 "r"(pk[half * 32 + ch * 4 + 2]), "r"(pk[half * 32 + ch * 4 + 3])
                                 : "memory");
            };
#pragma unroll
            // one pair in four on the FMA pipe (it floors 2^x at 2^-125, a masked key's -inf
            // included: negligible beside the row sum, which is at least 1 once the row has met
            // a key it attends)
            for (int i = 0; i < 32; ++i) {
                const float2 x = ffma2(make_float2(__uint_as_float(sa[2 * i]), __uint_as_float(sa[2 * i + 1])), sl2x2, nm2);
                const float2 pp = ((i & 3) == 3) ? exp2_fma2(x) : make_float2(tc::ex2(x.x), tc::ex2(x.y));
                ps2[i & 1] = fadd2(ps2[i & 1], pp);
                pk[i] = tc::pack_bf16(pp.x, pp.y);
            }
            // the first half of the previous P V has completed: this tile's first half of P
            // may go over it while the second half is formed (unless O needs rescaling first)
            const bool resc = k >= 1 && __any_sync(0xffffffffu, need && m != -INFINITY);
            if (k >= 1 && !__all_sync(0xffffffffu, wait_bar(BAR(LY::B_PVA + q), (uint32_t)(k - 1) & 1u))) { ok = false; break; }
            if (!resc) store_half(0);
#pragma unroll
            for (int i = 32; i < 64; ++i) {
                const int j = i & 31;
                const float2 x = ffma2(make_float2(__uint_as_float(sb[2 * j]), __uint_as_float(sb[2 * j + 1])), sl2x2, nm2);
                const float2 pp = ((i & 3) == 3) ? exp2_fma2(x) : make_float2(tc::ex2(x.x), tc::ex2(x.y));
                ps2[i & 1] = fadd2(ps2[i & 1], pp);
                pk[i] = tc::pack_bf16(pp.x, pp.y);
            }
            // the previous P V has completed (it read the P tile and accumulated into O)
            if (k >= 1 && !__all_sync(0xffffffffu, wait_bar(BAR(LY::B_PVDONE + q), (uint32_t)(k - 1) & 1u))) { ok = false; break; }
            tc::fence_after_sync();
            if (resc) {
                // the running max grew by more than 2^LAZY: rescale O before P V of this tile
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t orow[32];
                    tc::tmem_ld32(tlane + TM_O(q) + cc * 32, orow);
#pragma unroll
                    for (int i = 0; i < 32; ++i) orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
                    tc::tmem_st32(tlane + TM_O(q) + cc * 32, orow);
                }
                tc::tmem_wait_st();
                tc::fence_before_sync();
            }
            // this row of the shared P tile (128-byte swizzle: the 16-byte chunk index XORed
            // with the row mod 8); masked keys give 0
            if (resc) store_half(0);
            store_half(1);
            lsum = lsum * alpha + ((ps2[0].x + ps2[0].y) + (ps2[1].x + ps2[1].y));
            m = muse;
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(BAR(LY::B_PFULL + q));
            ++k;
        }
        if (!ok) break;
        // the unit's end: every product of the sub-tile has completed (its MMA warp commits
        // once per unit after its last issue); normalise O and store it, then hand O back
        if (!__all_sync(0xffffffffu, wait_bar(BAR(LY::B_ODONE + q), (uint32_t)ui & 1u))) { ok = false; break; }
        tc::fence_after_sync();
        if (k > k0) {
            const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
            if (!F8 && p.lse && row_valid) p.lse[c.q_head + lrow] = (m + log2f(lsum)) * 0.69314718055994531f;
            __nv_bfloat16 *orow = p.o + (c.q_head + lrow) * D;
            const float4 *vsc = F8 ? reinterpret_cast<const float4 *>(br.vs + (long)c.kvh * D) : nullptr;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t ov[32];
                __syncwarp();
                tc::tmem_ld32(tlane + TM_O(q) + cc * 32, ov);
                if (row_valid) {
                    if constexpr (F8) {
                        // the value channels' scales (the same 32 floats for every lane)
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float4 sv = __ldg(vsc + cc * 8 + i);
                            ov[4 * i] = __float_as_uint(__uint_as_float(ov[4 * i]) * sv.x);
                            ov[4 * i + 1] = __float_as_uint(__uint_as_float(ov[4 * i + 1]) * sv.y);
                            ov[4 * i + 2] = __float_as_uint(__uint_as_float(ov[4 * i + 2]) * sv.z);
                            ov[4 * i + 3] = __float_as_uint(__uint_as_float(ov[4 * i + 3]) * sv.w);
                        }
                    }
                    uint32_t pk2[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk2[i] = tc::pack_bf16(__uint_as_float(ov[2 * i]) * inv, __uint_as_float(ov[2 * i + 1]) * inv);
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + cc * 32);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[q4] = make_uint4(pk2[4 * q4], pk2[4 * q4 + 1], pk2[4 * q4 + 2], pk2[4 * q4 + 3]);
                }
            }
        }
        tc::fence_before_sync();
        mbar_arrive(BAR(LY::B_OFREE + q));
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == WARP_MMA) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
    // every path reaches this point once per CTA, after this CTA's last ticket; the last CTA
    // (of every launch sharing the counter) to arrive leaves the slot at zero for its next use
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&p.sched[1], 1) == p.ctas_total - 1) {
            atomicExch(&p.sched[0], 0);
            atomicExch(&p.sched[1], 0);
        }
    }
}

// Branches sharing one launch share the query and output tensors, the batch, the query rows,
// frame size, first query frame, scale and error word; their heads, windows and key/value
// tensors may differ.
bool same_launch(const AttnArgs &a, const AttnArgs &b)
{
    return a.q == b.q && a.o == b.o && a.B == b.B && a.q_Htot == b.q_Htot && a.q_rows == b.q_rows &&
           a.N == b.N && a.d == b.d && a.fq0 == b.fq0 && a.fq0_dev == b.fq0_dev && a.scale == b.scale &&
           a.err == b.err && a.qs == b.qs && a.lse == b.lse && a.sched == b.sched;
}

template <bool F8>
cudaError_t launch_attn_tc2(const AttnArgs *br, int nbr, int reserve_sms, cudaStream_t s,
                            cudaStream_t s_fill)
{
    using LY = Lay<F8>;
    cudaError_t e;
    if (nbr < 1 || nbr > 2) return cudaErrorInvalidValue;
    if (nbr == 2 && !same_launch(br[0], br[1])) return cudaErrorInvalidValue;
    const AttnArgs &a = br[0];
    if (a.d != D) return cudaErrorNotSupported;
    const long q_total = (long)a.B * a.q_Htot * a.q_rows;
    if (q_total + QT * BM >= (1L << 31)) return cudaErrorNotSupported;
    CUtensorMap mq, mk[2], mv[2];
    if (F8) {
        // E4M3 codes: one 128-byte row per token, one box covers the row
        if ((e = make_tmap_2d_u8(&mq, a.q, q_total, D, D, BM)) != cudaSuccess) return e;
    } else {
        if ((e = make_tmap_2d_bf16(&mq, a.q, q_total, D, 64, BM, true)) != cudaSuccess) return e;
    }
    Params p = {};
    int Hsum = 0;
    for (int i = 0; i < nbr; ++i) {
        const AttnArgs &x = br[i];
        const long kv_total = (long)x.B * x.kv_Htot * x.kv_rows;
        if (kv_total + BN >= (1L << 31)) return cudaErrorNotSupported;
        if (F8) {
            if ((e = make_tmap_2d_u8(&mk[i], x.k, kv_total, D, D, BN)) != cudaSuccess) return e;
            if ((e = make_tmap_2d_u8(&mv[i], x.v, kv_total, D, D, BN)) != cudaSuccess) return e;
            if (!x.qs || !x.ks || !x.vs) return cudaErrorInvalidValue;
        } else {
            if ((e = make_tmap_2d_bf16(&mk[i], x.k, kv_total, D, 64, BN, true)) != cudaSuccess) return e;
            if ((e = make_tmap_2d_bf16(&mv[i], x.v, kv_total, D, 64, BN, true)) != cudaSuccess) return e;
        }
        BranchP &b = p.br[i];
        b.Hbr = x.Hbr; b.q_h0 = x.q_h0; b.kv_Htot = x.kv_Htot; b.kv_h0 = x.kv_h0;
        b.kv_slots = x.kv_slots; b.w = x.w; b.r = x.r;
        b.nkb = x.kv_slots * ((x.N + 63) / 64);
        b.kv_rows = x.kv_rows;
        b.ks = x.ks; b.vs = x.vs;
        Hsum += x.Hbr;
    }
    if (nbr == 1) { mk[1] = mk[0]; mv[1] = mv[0]; }
    p.nbr = nbr; p.B = a.B; p.Hsum = Hsum;
    p.q_Htot = a.q_Htot; p.q_rows = a.q_rows;
    p.N = a.N; p.fq0 = a.fq0; p.fq0_dev = a.fq0_dev;
    p.sl2 = a.scale * 1.4426950408889634f;
    p.qs = a.qs;
    p.nqb = (int)((a.q_rows + BM - 1) / BM);
    p.lse = a.lse;
    p.o = (__nv_bfloat16 *)a.o;
    p.err = a.err;
    // persistent: one CTA per SM at most (less the SMs left to a kernel running beside it),
    // each taking 256-row units from the slot's counter; with `s_fill`, as many more CTAs as
    // SMs were left start behind the work on that stream and take units from the same counter
    const long nqt = (a.q_rows + QT * BM - 1) / (QT * BM);
    const long nunits = nqt * a.B * Hsum;
    if (nunits <= 0) return cudaSuccess;
    if (nunits >= (1L << 30)) return cudaErrorNotSupported;
    p.nqt = (int)nqt;
    p.nunits = (int)nunits;
    int dev = 0, nsm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (a.sched) {
        p.sched = a.sched;
    } else {
        static std::atomic<unsigned> next_slot{0};
        int *base = nullptr;
        if ((e = cudaGetSymbolAddress((void **)&base, g_attn_sched)) != cudaSuccess) return e;
        p.sched = base + 2 * (int)(next_slot.fetch_add(1u) % (unsigned)SCHED_SLOTS);
    }
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    nsm = std::max(nsm, 1);
    const int ctas = std::max(nsm - std::max(reserve_sms, 0), (nsm + 1) / 2);
    e = cudaFuncSetAttribute(attn_tc2_kernel<F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LY::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<long>(nunits, ctas);
    const int fill = s_fill ? (int)std::min<long>(nunits - grid, nsm - ctas) : 0;
    p.ctas_total = grid + fill;
    attn_tc2_kernel<F8><<<grid, THREADS, LY::SMEM_BYTES, s>>>(mq, mk[0], mv[0], mk[1], mv[1], p), note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess || fill <= 0) return e;
    attn_tc2_kernel<F8><<<fill, THREADS, LY::SMEM_BYTES, s_fill>>>(mq, mk[0], mv[0], mk[1], mv[1], p), note_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bf16_tc2(const AttnArgs &a, cudaStream_t s) { return launch_attn_tc2<false>(&a, 1, 0, s, nullptr); }
cudaError_t launch_attn_bf16_tc2_multi(const AttnArgs *br, int nbr, int reserve_sms, cudaStream_t s,
                                       cudaStream_t s_fill)
{
    return launch_attn_tc2<false>(br, nbr, reserve_sms, s, s_fill);
}
cudaError_t launch_attn_fp8_tc2(const AttnArgs &a, cudaStream_t s) { return launch_attn_tc2<true>(&a, 1, 0, s, nullptr); }

}  // namespace hlta
