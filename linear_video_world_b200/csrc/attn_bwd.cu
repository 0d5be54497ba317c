// Backward pass of the windowed softmax attention (SWA / DSWA), bf16 inputs, d = 128.
//
// With the forward's per-row log-sum-exp (natural log) lse_i, the weights are
// p_ij = exp(scale q_i.k_j - lse_i) over row i's window keys, and for the upstream gradient dO:
//   D_i = dO_i . o_i (= sum_j p_ij dP_ij),  dP_ij = dO_i . v_j,  dS_ij = p_ij (dP_ij - D_i),
//   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,  dv_j = sum_i p_ij dO_i
// (the reverse-mode derivative of exact attention; the llm-atlas long-context explainer, section
// 03, is the tiled forward this inverts). Three launches: D per row (this file), then dK / dV
// and dQ on the tensor cores (attn_bwd_tc.cu).
#include "hlta_internal.cuh"

namespace hlta {
namespace {

constexpr int D = 128;

// D_i = dO_i . o_i, one warp per row
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

}  // namespace

cudaError_t launch_attn_bwd(const AttnBwdArgs &a, cudaStream_t s)
{
    const long L = (long)a.T * a.N;
    const long rows = (long)a.BH * L;
    if (rows == 0) return cudaSuccess;
    if (a.BH > 65535 || rows >= (1L << 40)) return cudaErrorNotSupported;
    attn_bwd_dot<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>((const __nv_bfloat16 *)a.o,
                                                            (const __nv_bfloat16 *)a.dO, a.Dws, rows), note_launch();
    cudaError_t e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_attn_bwd_tc(a, s);
}

}  // namespace hlta
