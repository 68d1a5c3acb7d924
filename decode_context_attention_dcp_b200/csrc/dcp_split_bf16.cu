// dcp_split_bf16.cu -- the split-layout combine kernel instances for bf16 data (plain,
// strided, variable-length and fused-pack).
#include "dcp_combine_launch.cuh"

namespace dcp_host {

int32_t dispatch_split_bf16(const dcp::CombineArgs &a, cudaStream_t stream) { return dispatch_split<dcp::Bf16>(a, stream); }

}  // namespace dcp_host
