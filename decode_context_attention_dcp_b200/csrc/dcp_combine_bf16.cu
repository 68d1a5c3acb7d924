// dcp_combine_bf16.cu -- the combine kernel instances for bf16 data (compiled on its
// own so that the library's translation units build in parallel).
#include "dcp_combine_launch.cuh"

namespace dcp_host {

int32_t dispatch_combine_bf16(const dcp::CombineArgs &a, bool packed, cudaStream_t stream) {
    return packed ? dispatch_combine<dcp::Bf16, true>(a, stream) : dispatch_combine<dcp::Bf16, false>(a, stream);
}

}  // namespace dcp_host
