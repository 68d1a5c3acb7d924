// dcp_split_fp32.cu -- the split-layout combine kernel instances for fp32 data (plain,
// strided, variable-length and fused-pack).
#include "dcp_combine_launch.cuh"

namespace dcp_host {

int32_t dispatch_split_fp32(const dcp::CombineArgs &a, cudaStream_t stream) { return dispatch_split<dcp::Fp32>(a, stream); }

}  // namespace dcp_host
