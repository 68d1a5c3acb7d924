// dcp_combine_fp32.cu -- the packed-layout combine kernel instances for fp32 data (each
// element type and layout is compiled on its own so that the library builds in parallel).
#include "dcp_combine_launch.cuh"

namespace dcp_host {

int32_t dispatch_combine_fp32(const dcp::CombineArgs &a, bool packed, cudaStream_t stream) {
    return packed ? dispatch_packed<dcp::Fp32>(a, stream) : dispatch_split_fp32(a, stream);
}

}  // namespace dcp_host
