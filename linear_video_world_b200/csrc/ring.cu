// Ring append for the streaming cache: copies F new frames' K (or V) of one branch's heads
// from a [B][H][F*N][d] tensor into slots (f0 + i) mod slots of a [B][Hbr][slots][N][d] ring;
// and the in-stream advance of the cache's device-side frame counter.
#include "hlta_internal.cuh"

namespace hlta {
namespace {

__global__ void ring_append_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ ring,
                                   int Htot, int h0, int Hbr, long frame_vec, int F, int slots,
                                   int f0, const int *f0_dev)
{
    if (f0_dev) f0 = *f0_dev;
    const int bh = blockIdx.y, i = blockIdx.z;
    const int b = bh / Hbr, h = bh % Hbr;
    const uint4 *s = src + (((long)b * Htot + h0 + h) * F + i) * frame_vec;
    uint4 *dst = ring + ((long)bh * slots + (f0 + i) % slots) * frame_vec;
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < frame_vec;
         i += (long)gridDim.x * blockDim.x)
        dst[i] = s[i];
}

__global__ void frame_advance_kernel(int *f, int F) { *f += F; }

}  // namespace

cudaError_t launch_frame_advance(int *f, int F, cudaStream_t s)
{
    frame_advance_kernel<<<1, 1, 0, s>>>(f, F), note_launch();
    return cudaGetLastError();
}

cudaError_t launch_ring_append(const void *src, int B, int Htot, int h0, int Hbr, int N, int d,
                               size_t elem, int F, void *ring, int slots, int f0,
                               const int *f0_dev, cudaStream_t s)
{
    const size_t bytes = (size_t)N * d * elem;
    if (bytes % 16) return cudaErrorNotSupported;   // d*elem is a multiple of 16 for d % 8 == 0
    if (F < 1 || F > slots || F > 65535) return cudaErrorInvalidValue;
    const long frame_vec = (long)(bytes / 16);
    const unsigned gx = (unsigned)((frame_vec + 255) / 256 < 64 ? (frame_vec + 255) / 256 : 64);
    ring_append_kernel<<<dim3(gx, (unsigned)(B * Hbr), (unsigned)F), 256, 0, s>>>(
        (const uint4 *)src, (uint4 *)ring, Htot, h0, Hbr, frame_vec, F, slots, f0, f0_dev), note_launch();
    return cudaGetLastError();
}

}  // namespace hlta
