// Self-test of the failure-detection path: one thread waits, through the same bounded mbarrier
// wait every pipelined kernel of the library uses, on a barrier phase that nothing completes.
// The wait expires after the given number of cycles, ORs DEVERR_SELFTEST into the device error
// word and the kernel returns. No copy and no tensor-core operation is in flight, so the
// context stays usable; the host reads the word with hlta_device_status.
#include "hlta_internal.cuh"
#include "sm100_ptx.cuh"

namespace hlta {
namespace {

__global__ void wait_selftest_kernel(unsigned int *err, long long cycles)
{
    __shared__ alignas(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    abort_flag = 0;
    const uint32_t b = ptx::smem_u32(&bar);
    ptx::mbar_init(b, 1);           // expects one arrival; none is ever made
    ptx::mbar_init_fence();
    ptx::mbar_wait(b, 0, (volatile int *)&abort_flag, err, DEVERR_SELFTEST, cycles);
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(b) : "memory");
}

}  // namespace

cudaError_t launch_wait_selftest(unsigned int *err, long long cycles, cudaStream_t s)
{
    wait_selftest_kernel<<<1, 32, 0, s>>>(err, cycles), note_launch();
    return cudaGetLastError();
}

}  // namespace hlta
