// dcp_combine_fp16.cu -- the combine kernel instances for fp16 data (compiled on its
// own so that the library's translation units build in parallel).
#include "dcp_combine_launch.cuh"

namespace dcp_host {

int32_t dispatch_combine_fp16(const dcp::CombineArgs &a, bool packed, cudaStream_t stream) {
    return packed ? dispatch_combine<dcp::Fp16, true>(a, stream) : dispatch_combine<dcp::Fp16, false>(a, stream);
}

}  // namespace dcp_host
