// Gated delta rule, bf16: the pass over the chunks as a two-level scan on the sm_100a tensor
// cores (tcgen05.mma with tensor-memory accumulators).
//
// The chunk preparation (gdn_prep_tc.cu) leaves per 64-token chunk c of a head the bf16
// products W^T, Qt^T ([128 j][64 t]), Up^T, Op^T ([128 i][64 t]), gam = e^{g_n} and
// ek_t = e^{g_n - g_t}; with Kt = diag(ek) K and a chunk start state S (S[i][j], i value
// index, j key index) the recurrence is
//   U = Up - S W^T,   O = Op + S Qt^T,   S_end = gam S + U Kt = gam S + (U diag(ek)) K,
// i.e. for every row s of S (with up the matching row of Up^T): s_end = s (gam I - W^T Kt) +
// up Kt. The rows of S evolve independently and the map over a chunk is affine in S. Over a
// segment of consecutive chunks the composition is affine too, S_end = S_start A_p + B_p, where
// A_p is what the chain does to the rows of the identity with Up = 0 and B_p what it does to
// zero rows with Up. That is the "state passing is a composition of multiplicative
// transitions" of the llm-atlas long-context explainer (sections 06 and 09: chunkwise =
// parallel within a block, recurrent across blocks); the scan applies it at two levels:
//   1. segmap  (every segment but the last, A and B parts in separate CTAs of one launch, all
//              in parallel): the chain over the segment's chunks from I (A part) or 0 (B
//              part), no output;
//   2. compose (serial over segments, rows split over CTAs, fp32 on the CUDA cores):
//              S_0 = S0, S_{p+1} = S_p A_p + B_p;
//   3. replay  (every segment in parallel): the chain from S_p with the outputs O, the last
//              segment also writing the final state.
// A head whose chunks fit one segment runs only the replay (from S0).
//
// The chain kernel (one CTA per segment, 192 threads):
//   warps 0-3  chain: thread i holds row i of the state (fp32, registers); per chunk it stores
//              the row as bf16 pairs into tensor memory (the A operand of S [Qt; W]^T, whose
//              B operand is [Qt^T | W^T] read MN-major), takes D_W, forms U diag(ek) =
//              (Up - D_W) diag(ek) as bf16 pairs (the A operand of the product with K, read
//              from the input, MN-major), and while that runs on the tensor pipe writes its
//              outputs O = Op + D_Q (replay); then it takes U Kt and updates
//              s <- gam s + (U Kt)_i
//   warp 4     TMA producer: the chunk operands through a two-stage ring
//   warp 5     tensor-memory owner and MMA issuer (one thread)
// Tensor memory (512 columns allocated): S bf16 [0, 64), U bf16 [64, 96), D = [D_Q | D_W] at
// 128 (replay; D_W alone at 192 in the segment maps), U Kt at 256.
// Every mbarrier wait is bounded (DEVERR_GDN_WAIT); on expiry every role stops, the producer
// lets its copies land, and the tensor memory is released.
#include "hlta_internal.cuh"
#include "sm100_ptx.cuh"
#include "tc_ptx.cuh"

namespace hlta {
namespace {

constexpr int C = 64;                  // chunk length
constexpr int D = 128;                 // head dim (state is D x D)
constexpr int NSTG = 2;                // stages of the operand ring
constexpr int WARP_TMA = 4, WARP_MMA = 5;
constexpr int THREADS = 192;
constexpr int ROWS = 128;              // chain threads = state rows

constexpr uint32_t SLICE = 128 * 128;      // [128 rows][64 t] bf16: 16 KB
constexpr uint32_t KT_HALF = 64 * 128;     // [64 t][64 j] bf16: 8 KB

enum Mode { SEGMAP = 0, REPLAY = 2 };

// Tensor-memory columns. Replay: S bf16 [0, 64), U bf16 [64, 96), D = [D_Q | D_W] at 128, U Kt
// at 256 (512 allocated). Segment maps (no outputs, two CTAs per SM): D_W and U Kt share the
// columns at 128, since U Kt is issued after the chain threads read D_W and the next D_W after
// they read U Kt (256 allocated).
template <int MODE> struct Tm {
    static constexpr uint32_t S = 0, U = 64;
    static constexpr uint32_t D1 = 128;                           // target of S [Qt; W]^T
    static constexpr uint32_t DW = MODE == REPLAY ? 192 : 128;    // D_W
    static constexpr uint32_t DL = MODE == REPLAY ? 256 : 128;    // U Kt
    static constexpr uint32_t COLS = MODE == REPLAY ? 512 : 256;
};

template <int MODE> struct Stage {
    // replay: Qt^T then W^T; segment maps: W^T alone; each [128 j][64 t]
    static constexpr uint32_t W_OFF = MODE == REPLAY ? SLICE : 0;
    alignas(1024) uint8_t QW[(MODE == REPLAY ? 2 : 1) * SLICE];
    alignas(1024) uint8_t Kt[2 * KT_HALF];   // K [64 t][128 j] (the input) as two 64-column halves
    alignas(1024) uint8_t Up[SLICE];         // Up^T [128 i][64 t]
    alignas(1024) uint8_t Op[MODE == REPLAY ? SLICE : 16];   // Op^T (replay)
    alignas(16) float scal[GDN_SCAL];        // gam, then ek_t at 4 + t
};
template <int MODE> struct ChainSmem {
    Stage<MODE> st[NSTG];
    alignas(8) uint64_t full[NSTG];
    alignas(8) uint64_t empty[NSTG];       // MMA commit (+ chain threads done with Op, replay)
    alignas(8) uint64_t s_ready;           // chain threads stored S (count ROWS)
    alignas(8) uint64_t u_ready;           // chain threads stored U (count ROWS)
    alignas(8) uint64_t d_full;            // S [Qt; W]^T complete
    alignas(8) uint64_t dl_full;           // U Kt complete
    uint32_t tmem_slot;
    int abort_flag;
};

struct ChainMaps {
    CUtensorMap W, Q, U, O;                // [BH*nch*128][64]: 64 cols x 128 rows, swizzled
    CUtensorMap K;                         // the input k [B*Htot*L][128]: 64x64 swizzled boxes
};

struct ChainArgs {
    GdnArgs g;
    GdnWs2 ws;
    long nch;
    int seg, nseg;
    // [BH][nseg][D][D] fp32 each, every matrix stored transposed ([j][i]: element (i, j) at
    // j * D + i), so that a warp's 32 rows i read or write one 128-byte line per column j
    float *Amap, *Bmap, *Sseg;
};

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                         unsigned int *err)
{
    return ptx::mbar_try(bar, parity) || ptx::mbar_wait(bar, parity, abort_flag, err, DEVERR_GDN_WAIT);
}

// element (i, t) of a [128 i][64 t] bf16 tile staged by a 128B-swizzled TMA box: 16-byte chunk
// t/8 of row i sits at chunk (t/8) ^ (i % 8)
__device__ __forceinline__ const uint4 *slice_chunk(const uint8_t *tile, int i, int c8)
{
    return reinterpret_cast<const uint4 *>(tile + i * 128 + ((c8 ^ (i & 7)) << 4));
}

template <int MODE>
__global__ void __launch_bounds__(THREADS, MODE == SEGMAP ? 2 : 1)
gdn_chain_bf16(const __grid_constant__ ChainMaps maps, const ChainArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    using TM = Tm<MODE>;
    using Stg = Stage<MODE>;
    ChainSmem<MODE> &s = *reinterpret_cast<ChainSmem<MODE> *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const GdnArgs &p = a.g;
    const int seg = blockIdx.x, bh = blockIdx.y;
    // the segment maps: part A (blockIdx.z 0) runs the chain from the identity with Up = 0,
    // part B (blockIdx.z 1) from zero with Up; both in one launch
    const bool segA = MODE == SEGMAP && blockIdx.z == 0;
    const bool segB = MODE == SEGMAP && blockIdx.z == 1;
    const int b = bh / p.Hg, h = bh % p.Hg;
    const long c_begin = (long)seg * a.seg;
    const long c_end = min(a.nch, c_begin + a.seg);
    const int nc = (int)(c_end - c_begin);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int *abort_flag = (volatile int *)&s.abort_flag;
    const uint32_t FULL0 = ptx::smem_u32(&s.full[0]), EMPTY0 = ptx::smem_u32(&s.empty[0]);
    const uint32_t S_READY = ptx::smem_u32(&s.s_ready), U_READY = ptx::smem_u32(&s.u_ready);
    const uint32_t D_FULL = ptx::smem_u32(&s.d_full), DL_FULL = ptx::smem_u32(&s.dl_full);

    if (tid == 0) {
        for (int i = 0; i < NSTG; ++i) {
            ptx::mbar_init(FULL0 + 8 * i, 1);
            ptx::mbar_init(EMPTY0 + 8 * i, MODE == REPLAY ? 1 + ROWS : 1);
        }
        ptx::mbar_init(S_READY, ROWS);
        ptx::mbar_init(U_READY, ROWS);
        ptx::mbar_init(D_FULL, 1);
        ptx::mbar_init(DL_FULL, 1);
        s.abort_flag = 0;
        ptx::mbar_init_fence();
    }
    if (warp == WARP_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         ptx::smem_u32(&s.tmem_slot)),
                     "r"(TM::COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = s.tmem_slot;

    if (warp == WARP_TMA) {
        // ------------------------------ TMA producer --------------------------------------
        if (lane == 0) {
            const uint32_t TX = (MODE == REPLAY ? 2 * SLICE : SLICE) + 2 * KT_HALF +
                                (segA ? 0 : SLICE) + (MODE == REPLAY ? SLICE : 0) + GDN_SCAL * 4;
            const long krow0 = (long)(b * p.Htot + p.h0 + h) * p.L;
            int k = 0;
            for (; k < nc; ++k) {
                const int st = k % NSTG;
                if (k >= NSTG && !wait_bar(EMPTY0 + 8 * st, (uint32_t)((k - NSTG) / NSTG) & 1u, abort_flag, p.err)) break;
                Stg &sg = s.st[st];
                const uint32_t full = FULL0 + 8 * st;
                ptx::mbar_expect_tx(full, TX);
                const long c = c_begin + k;
                const int trow = (int)(((long)bh * a.nch + c) * D);
                if (MODE == REPLAY) ptx::tma_load_2d(ptx::smem_u32(sg.QW), &maps.Q, 0, trow, full);
                ptx::tma_load_2d(ptx::smem_u32(sg.QW + Stg::W_OFF), &maps.W, 0, trow, full);
                // K rows past a ragged last chunk belong to the next head (or are zero-filled
                // past the tensor): U diag(ek) is zero there, so they add nothing
                const int krow = (int)(krow0 + c * C);
                for (int hf = 0; hf < 2; ++hf)
                    ptx::tma_load_2d(ptx::smem_u32(sg.Kt + hf * KT_HALF), &maps.K, hf * 64, krow, full);
                if (!segA) ptx::tma_load_2d(ptx::smem_u32(sg.Up), &maps.U, 0, trow, full);
                if (MODE == REPLAY) ptx::tma_load_2d(ptx::smem_u32(sg.Op), &maps.O, 0, trow, full);
                ptx::bulk_load(ptx::smem_u32(sg.scal), a.ws.scal + ((long)bh * a.nch + c) * GDN_SCAL,
                               GDN_SCAL * 4, full);
            }
            if (*abort_flag) {
                // a bounded wait expired somewhere: let the copies this CTA issued land
                const long long t0 = clock64();
                for (int kk = k - 1; kk >= 0 && kk >= k - NSTG; --kk)
                    while (!ptx::mbar_try(FULL0 + 8 * (kk % NSTG), (uint32_t)(kk / NSTG) & 1u) &&
                           clock64() - t0 < (1LL << 31)) {}
            }
        }
    } else if (warp == WARP_MMA) {
        // ------------------------------ MMA issuer ----------------------------------------
        if (lane == 0) {
            // S [Qt; W]^T: A = S (tensor memory), B = [Qt^T | W^T], MN-major (token t along N);
            // replay N = 128 tokens (Qt then W), segmap N = 64 (W only, into the D_W half)
            constexpr int N1 = MODE == REPLAY ? 128 : 64;
            constexpr uint32_t IDESC1 = tc::idesc_bf16(128, N1, false, true);
            // U Kt: A = U (tensor memory), B = Kt, MN-major (key j along N)
            constexpr uint32_t IDESC2 = tc::idesc_bf16(128, 128, false, true);
            bool ok = true;
            for (int k = 0; k < nc && ok; ++k) {
                const int st = k % NSTG;
                Stg &sg = s.st[st];
                ok = wait_bar(FULL0 + 8 * st, (uint32_t)(k / NSTG) & 1u, abort_flag, p.err) &&
                     wait_bar(S_READY, (uint32_t)k & 1u, abort_flag, p.err);
                if (!ok) break;
                tc::fence_after_sync();
                const uint64_t d1 = tc::sw128_desc(ptx::smem_u32(sg.QW), SLICE, 1024);
                const uint32_t dcol = tmem + (MODE == REPLAY ? TM::D1 : TM::DW);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tc::umma_bf16_ts(dcol, tmem + TM::S + kk * 8, d1 + (uint64_t)((kk * 2048) >> 4), IDESC1, kk > 0 ? 1u : 0u);
                tc::umma_commit(D_FULL);
                if (!(ok = wait_bar(U_READY, (uint32_t)k & 1u, abort_flag, p.err))) break;
                tc::fence_after_sync();
                const uint64_t d2 = tc::sw128_desc(ptx::smem_u32(sg.Kt), KT_HALF, 1024);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    tc::umma_bf16_ts(tmem + TM::DL, tmem + TM::U + kk * 8, d2 + (uint64_t)((kk * 2048) >> 4),
                                     IDESC2, kk > 0 ? 1u : 0u);
                tc::umma_commit(DL_FULL);
                tc::umma_commit(EMPTY0 + 8 * st);
            }
        }
    } else if (warp < 4) {
        // ------------------------------ chain (state rows) --------------------------------
        const int i = warp * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
        __nv_bfloat16 *o = MODE == REPLAY ? (__nv_bfloat16 *)p.o + (long)(b * p.Htot + p.h0 + h) * p.L * D + i : nullptr;
        float sr[D];
        if (segA) {
#pragma unroll
            for (int j = 0; j < D; ++j) sr[j] = j == i ? 1.f : 0.f;
        } else if (segB) {
#pragma unroll
            for (int j = 0; j < D; ++j) sr[j] = 0.f;
        } else {
            // segment 0 starts from S0 (or zero) when it is the only one; otherwise every
            // segment starts from its composed start state (stored transposed)
            const float *src = a.nseg > 1 ? nullptr : (p.S0 ? p.S0 + ((long)bh * D + i) * D : nullptr);
            if (a.nseg > 1) {
                const float *st_t = a.Sseg + ((long)bh * a.nseg + seg) * D * D + i;
#pragma unroll
                for (int j = 0; j < D; ++j) sr[j] = st_t[(long)j * D];
            } else if (src) {
                const float4 *s4 = reinterpret_cast<const float4 *>(src);
#pragma unroll
                for (int j4 = 0; j4 < D / 4; ++j4) {
                    const float4 v = s4[j4];
                    sr[4 * j4] = v.x; sr[4 * j4 + 1] = v.y; sr[4 * j4 + 2] = v.z; sr[4 * j4 + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < D; ++j) sr[j] = 0.f;
            }
        }
        bool ok = true;
        for (int k = 0; k < nc; ++k) {
            const int st = k % NSTG;
            const Stg &sg = s.st[st];
            // the state row as bf16 pairs: A operand of S [Qt; W]^T
#pragma unroll
            for (int qt = 0; qt < 4; ++qt) {
                uint32_t pk[16];
#pragma unroll
                for (int m = 0; m < 16; ++m) pk[m] = tc::pack_bf16(sr[qt * 32 + 2 * m], sr[qt * 32 + 2 * m + 1]);
                tc::tmem_st16(tl + TM::S + qt * 16, pk);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            ptx::mbar_arrive(S_READY);
            // U = Up - S W^T, as bf16 pairs: A operand of U Kt (the stage's gam is read here
            // too: the stage may be refilled as soon as U is handed over)
            if (!__all_sync(0xffffffffu, wait_bar(D_FULL, (uint32_t)k & 1u, abort_flag, p.err) &&
                                             wait_bar(FULL0 + 8 * st, (uint32_t)(k / NSTG) & 1u, abort_flag, p.err))) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const float gam = sg.scal[0];
            // in quarters of 16 tokens, to keep few registers live beside the state row
#pragma unroll
            for (int qt = 0; qt < 4; ++qt) {
                uint32_t dw[16];
                tc::tmem_ld16(tl + TM::DW + qt * 16, dw);
                uint32_t pk[8];
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    const float4 ea = *reinterpret_cast<const float4 *>(&sg.scal[4 + qt * 16 + c2 * 8]);
                    const float4 eb = *reinterpret_cast<const float4 *>(&sg.scal[4 + qt * 16 + c2 * 8 + 4]);
                    const float ek[8] = {ea.x, ea.y, ea.z, ea.w, eb.x, eb.y, eb.z, eb.w};
                    uint32_t uw[4] = {0u, 0u, 0u, 0u};    // Up = 0 for the A part of the maps
                    if (!segA) {
                        const uint4 u = *slice_chunk(sg.Up, i, qt * 2 + c2);
                        uw[0] = u.x; uw[1] = u.y; uw[2] = u.z; uw[3] = u.w;
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&uw[e]));
                        pk[c2 * 4 + e] = tc::pack_bf16(ek[2 * e] * (f.x - __uint_as_float(dw[c2 * 8 + 2 * e])),
                                                       ek[2 * e + 1] * (f.y - __uint_as_float(dw[c2 * 8 + 2 * e + 1])));
                    }
                }
                tc::tmem_st8(tl + TM::U + qt * 8, pk);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            ptx::mbar_arrive(U_READY);
            if (MODE == REPLAY) {
                // while U Kt runs: O = Op + S Qt^T of this chunk, row i of every token
                const long t0 = (c_begin + k) * C;
                const int n = (int)min((long)C, p.L - t0);
                __nv_bfloat16 *orow = o + t0 * D;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t dq[32];
                    tc::tmem_ld32(tl + TM::D1 + hf * 32, dq);
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const uint4 u = *slice_chunk(sg.Op, i, hf * 4 + c4);
                        const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&uw[e]));
                            const int t = hf * 32 + c4 * 8 + 2 * e;
                            if (t < n) orow[(long)t * D] = __float2bfloat16_rn(f.x + __uint_as_float(dq[c4 * 8 + 2 * e]));
                            if (t + 1 < n) orow[(long)(t + 1) * D] = __float2bfloat16_rn(f.y + __uint_as_float(dq[c4 * 8 + 2 * e + 1]));
                        }
                    }
                }
                // Op of this stage is read (the MMA commit releases the rest of it)
                ptx::mbar_arrive(EMPTY0 + 8 * st);
            }
            // s <- gam s + (U Kt)_i
            if (!__all_sync(0xffffffffu, wait_bar(DL_FULL, (uint32_t)k & 1u, abort_flag, p.err))) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uint32_t dl[16];
                tc::tmem_ld16(tl + TM::DL + q * 16, dl);
#pragma unroll
                for (int j = 0; j < 16; ++j) sr[q * 16 + j] = fmaf(gam, sr[q * 16 + j], __uint_as_float(dl[j]));
            }
        }
        if (ok) {
            float *dst = nullptr;
            if (segA || segB) {
                // the map transposed (A_p^T is then the K-major operand of the composition's
                // products); consecutive rows i make each store of a warp one 128-byte line
                float *mt = (segA ? a.Amap : a.Bmap) + ((long)bh * a.nseg + seg) * D * D + i;
#pragma unroll
                for (int j = 0; j < D; ++j) mt[(long)j * D] = sr[j];
            } else if (seg == a.nseg - 1 && p.S_out) dst = p.S_out + ((long)bh * D + i) * D;
            if (dst) {
                float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
                for (int j4 = 0; j4 < D / 4; ++j4)
                    d4[j4] = make_float4(sr[4 * j4], sr[4 * j4 + 1], sr[4 * j4 + 2], sr[4 * j4 + 3]);
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == WARP_MMA) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TM::COLS)
                     : "memory");
    }
}

// -----------------------------------------------------------------------------------------
// compose: S_0 = S0, S_{p+1} = S_p A_p + B_p on the tensor cores, one CTA per head.
// S_p stays in tensor memory in fp32 and is the A operand of the next product directly
// (kind::tf32, A from tensor memory); A_p arrives by TMA as the K-major B operand (the segment
// maps store it transposed, [j][k]); the accumulator is set to B_p first (tcgen05.st), so the
// product adds onto it. Two column regions of 128 alternate: S_p in one, S_{p+1} built in the
// other. Each S_{p+1} is copied out to the start states the replay reads while the next
// product runs. Warps 0-3: thread i owns row i (TMEM lane i); warp 4: TMEM owner, TMA
// producer and MMA issuer (one thread).
// -----------------------------------------------------------------------------------------
constexpr int COMPOSE_THREADS = 160;
constexpr uint32_t AT_BOX = 128 * 128;           // [128 j][32 k] fp32, 128-byte swizzle: 16 KB
struct ComposeSmem {
    alignas(1024) uint8_t At[2][4 * AT_BOX];     // A_p^T, K-major (k along the 128-byte rows)
    alignas(8) uint64_t full[2];                 // A_p^T landed
    alignas(8) uint64_t empty[2];                // its product completed
    alignas(8) uint64_t b_ready;                 // B_p stored into the accumulator (count 128)
    alignas(8) uint64_t d_full;                  // S_{p+1} complete
    uint32_t tmem_slot;
    int abort_flag;
};

__global__ void __launch_bounds__(COMPOSE_THREADS, 1)
gdn_compose_tc(const __grid_constant__ CUtensorMap mat, const ChainArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    ComposeSmem &s = *reinterpret_cast<ComposeSmem *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const GdnArgs &p = a.g;
    const int bh = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nmaps = a.nseg - 1;                // the launch has nseg > 1
    volatile int *abort_flag = (volatile int *)&s.abort_flag;
    const uint32_t FULL0 = ptx::smem_u32(&s.full[0]), EMPTY0 = ptx::smem_u32(&s.empty[0]);
    const uint32_t B_READY = ptx::smem_u32(&s.b_ready), D_FULL = ptx::smem_u32(&s.d_full);
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(FULL0 + 8 * i, 1);
            ptx::mbar_init(EMPTY0 + 8 * i, 1);
        }
        ptx::mbar_init(B_READY, ROWS);
        ptx::mbar_init(D_FULL, 1);
        s.abort_flag = 0;
        ptx::mbar_init_fence();
    }
    if (warp == 4) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         ptx::smem_u32(&s.tmem_slot)),
                     "r"(256)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = s.tmem_slot;
    const long map0 = (long)bh * a.nseg;         // this head's first map / start state

    if (warp == 4) {
        if (lane == 0) {
            // A_p^T of map p: rows (map0 + p) * 128 .. of the [BH * nseg * 128][128] view
            auto load = [&](int mp) {
                const uint32_t full = FULL0 + 8 * (mp & 1);
                ptx::mbar_expect_tx(full, 4 * AT_BOX);
                for (int q = 0; q < 4; ++q)
                    ptx::tma_load_2d(ptx::smem_u32(s.At[mp & 1]) + q * AT_BOX, &mat, 32 * q,
                                     (int)((map0 + mp) * D), full);
            };
            load(0);
            if (nmaps > 1) load(1);
            int issued = nmaps > 1 ? 2 : 1;
            constexpr uint32_t ID = tc::idesc_tf32(128, 128);
            bool ok = true;
            for (int mp = 0; mp < nmaps && ok; ++mp) {
                const int st = mp & 1;
                ok = wait_bar(FULL0 + 8 * st, (uint32_t)(mp >> 1) & 1u, abort_flag, p.err) &&
                     wait_bar(B_READY, (uint32_t)mp & 1u, abort_flag, p.err);
                if (!ok) break;
                tc::fence_after_sync();
                const uint32_t a_col = tmem + (uint32_t)(mp & 1) * 128u;         // S_p
                const uint32_t d_col = tmem + (uint32_t)((mp + 1) & 1) * 128u;   // B_p, then S_{p+1}
                const uint64_t bd = tc::sw128_desc(ptx::smem_u32(s.At[st]), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 8; ++kk)
                    tc::umma_tf32_ts(d_col, a_col + kk * 8,
                                     bd + (uint64_t)(((kk >> 2) * AT_BOX + (kk & 3) * 32) >> 4), ID, 1u);
                tc::umma_commit(D_FULL);
                tc::umma_commit(EMPTY0 + 8 * st);
                if (mp + 2 < nmaps) {
                    // the stage is free once this product completed
                    if (!(ok = wait_bar(EMPTY0 + 8 * st, (uint32_t)(mp >> 1) & 1u, abort_flag, p.err))) break;
                    load(mp + 2);
                    issued = mp + 3;
                }
            }
            if (*abort_flag) {
                // a bounded wait expired somewhere: let the copies this CTA issued land
                const long long t0 = clock64();
                for (int mp = issued - 1; mp >= 0 && mp >= issued - 2; --mp)
                    while (!ptx::mbar_try(FULL0 + 8 * (mp & 1), (uint32_t)(mp >> 1) & 1u) &&
                           clock64() - t0 < (1LL << 31)) {}
            }
        }
    } else {
        const int i = tid;                       // row i of S (TMEM lane i)
        const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
        // start states, B maps: transposed, element (i, j) of matrix m at m * D * D + j * D + i
        float *sseg = a.Sseg + map0 * D * D + i;
        const float *bmap = a.Bmap + map0 * D * D + i;
        // S_0: S0 or zero, into the start states and into columns [0, 128)
        {
            const float *src = p.S0 ? p.S0 + ((long)bh * D + i) * D : nullptr;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float4 v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    v[e] = src ? reinterpret_cast<const float4 *>(src)[4 * q + e] : make_float4(0.f, 0.f, 0.f, 0.f);
                uint32_t u[16];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    u[4 * e] = __float_as_uint(v[e].x); u[4 * e + 1] = __float_as_uint(v[e].y);
                    u[4 * e + 2] = __float_as_uint(v[e].z); u[4 * e + 3] = __float_as_uint(v[e].w);
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) sseg[(long)(16 * q + e) * D] = __uint_as_float(u[e]);
                tc::tmem_st16(tl + q * 16, u);
            }
        }
        // B_0's row i
        float bnext[D];
#pragma unroll
        for (int j = 0; j < D; ++j) bnext[j] = bmap[(long)j * D];
        for (int mp = 0; mp < nmaps; ++mp) {
            // B_p into the accumulator columns (they held S_{p-1}, whose product completed)
            const uint32_t dcol = tl + (uint32_t)((mp + 1) & 1) * 128u;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                uint32_t u[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) u[e] = __float_as_uint(bnext[16 * q + e]);
                tc::tmem_st16(dcol + q * 16, u);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            ptx::mbar_arrive(B_READY);
            // the next map's row loads while the product runs
            if (mp + 1 < nmaps) {
                const float *bn = bmap + (long)(mp + 1) * D * D;
#pragma unroll
                for (int j = 0; j < D; ++j) bnext[j] = bn[(long)j * D];
            }
            if (!__all_sync(0xffffffffu, wait_bar(D_FULL, (uint32_t)mp & 1u, abort_flag, p.err))) break;
            tc::fence_after_sync();
            // S_{p+1} out to the start states (it stays in tensor memory for the next product)
            float *dst = sseg + (long)(mp + 1) * D * D;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t v[32];
                tc::tmem_ld32(dcol + q * 32, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) dst[(long)(32 * q + e) * D] = __uint_as_float(v[e]);
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 4) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256)
                     : "memory");
    }
}

}  // namespace

int gdn_scan_segment_len(long BH, long nch)
{
    // about 128 replay CTAs in all (one per SM, the rest of the GPU left to the softmax
    // branches running beside), never segments shorter than 32 chunks: below that the
    // segment maps and their composition cost more than the shorter chain saves
    const long per_head = BH >= 128 ? 1 : 128 / BH;
    const long seg = (nch + per_head - 1) / per_head;
    return (int)(seg < 32 ? 32 : seg);
}

int gdn_scan_segments_beside(long BH, long nch, double attn_flop)
{
    // Estimates from measurements on the B200 at 480P: the softmax launches run at about
    // 8e8 FLOP per microsecond; one chunk step of the chain takes about 2 us when the chains
    // of few heads run beside them. One segment is a single pass over the chunks; s > 1
    // segments are two passes over ceil(nch / s) chunks (the maps, then the replay) plus s
    // composition steps of about 3 us. The fewest segments whose chain ends within
    // the softmax branches' time beside the GDN branch (about 1.15 times their time alone,
    // measured: they share the SMs with the chunk preparation and the chain) are taken: every
    // extra segment occupies more SMs the softmax branches could use.
    const long seg_lat = gdn_scan_segment_len(BH, nch);
    const long max_seg = (nch + seg_lat - 1) / seg_lat;
    const double attn_us = 1.15 * attn_flop / 8.0e8, chunk_us = 2.0, compose_us = 3.0;
    for (long s = 1; s < max_seg; ++s) {
        const double lat = s == 1 ? chunk_us * (double)nch
                                  : 2.0 * chunk_us * (double)((nch + s - 1) / s) + compose_us * (double)s;
        if (lat <= attn_us) return (int)s;
    }
    return (int)max_seg;
}

size_t gdn_scan_bytes(long BH, long nch)
{
    const long seg = gdn_scan_segment_len(BH, nch);
    const long nseg = (nch + seg - 1) / seg;
    if (nseg <= 1) return 0;
    return (size_t)3 * BH * nseg * D * D * sizeof(float);
}

cudaError_t launch_gdn_bf16_scan(const GdnArgs &g, const GdnWs2 &ws, cudaStream_t s)
{
    const long nch = gdn_num_chunks(g.L, C);
    const long BH = (long)g.B * g.Hg;
    const long out_rows = BH * nch * D;
    const long in_rows = (long)g.B * g.Htot * g.L;
    float *scan_ws = ws.scan;
    ChainArgs a;
    a.g = g;
    a.ws = ws;
    a.nch = nch;
    a.seg = gdn_scan_segment_len(BH, nch);
    a.nseg = (int)((nch + a.seg - 1) / a.seg);
    if (g.scan_segments > 0 && g.scan_segments < a.nseg) {
        // fewer, longer segments than the latency-oriented split (the workspace holds more)
        a.seg = (int)((nch + g.scan_segments - 1) / g.scan_segments);
        a.nseg = (int)((nch + a.seg - 1) / a.seg);
    }
    a.Amap = scan_ws;
    a.Bmap = scan_ws ? scan_ws + BH * a.nseg * D * D : nullptr;
    a.Sseg = scan_ws ? scan_ws + 2 * BH * a.nseg * D * D : nullptr;
    if (a.nseg > 1 && !scan_ws) return cudaErrorInvalidValue;
    if (BH > 65535) return cudaErrorNotSupported;
    cudaError_t e;
    ChainMaps m;
    if ((e = make_tmap_2d_bf16(&m.W, ws.Wt, out_rows, C, 64, D, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&m.Q, ws.Qt, out_rows, C, 64, D, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&m.U, ws.Ut, out_rows, C, 64, D, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&m.O, ws.Ot, out_rows, C, 64, D, true)) != cudaSuccess) return e;
    if ((e = make_tmap_2d_bf16(&m.K, g.k, in_rows, D, 64, C, true)) != cudaSuccess) return e;
    // the segment maps' A parts, transposed: [BH * nseg * 128 j][128 k] fp32, boxes of 32 k
    CUtensorMap mat;
    if (a.nseg > 1 &&
        (e = make_tmap_2d_f32(&mat, a.Amap, (uint64_t)BH * a.nseg * D, D, 32, D, true)) != cudaSuccess)
        return e;
    const size_t smem_map = sizeof(ChainSmem<SEGMAP>) + 1024, smem = sizeof(ChainSmem<REPLAY>) + 1024;
    static_assert(2 * (sizeof(ChainSmem<SEGMAP>) + 2048) <= 228 * 1024, "two segment-map CTAs per SM");
    if ((e = cudaFuncSetAttribute(gdn_chain_bf16<SEGMAP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_map)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(gdn_chain_bf16<SEGMAP>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  (int)cudaSharedmemCarveoutMaxShared)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(gdn_chain_bf16<REPLAY>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
    const size_t csmem = sizeof(ComposeSmem) + 1024;
    if ((e = cudaFuncSetAttribute(gdn_compose_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csmem)) != cudaSuccess) return e;
    if (a.nseg > 1) {
        // the maps of every segment but the last, then their composition
        const dim3 gm((unsigned)(a.nseg - 1), (unsigned)BH, 2);
        gdn_chain_bf16<SEGMAP><<<gm, THREADS, smem_map, s>>>(m, a), note_launch();
        gdn_compose_tc<<<(unsigned)BH, COMPOSE_THREADS, csmem, s>>>(mat, a), note_launch();
    }
    gdn_chain_bf16<REPLAY><<<dim3((unsigned)a.nseg, (unsigned)BH), THREADS, smem, s>>>(m, a), note_launch();
    return cudaGetLastError();
}

}  // namespace hlta
