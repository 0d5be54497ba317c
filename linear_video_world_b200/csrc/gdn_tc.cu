#include "hlta_internal.cuh"
namespace hlta {
cudaError_t launch_gdn_bf16(const GdnArgs &, cudaStream_t) { return cudaErrorNotSupported; }
}
