#include "conv_tc.cuh"

namespace sige {

bool tc_supported(const sige_conv_desc *, int) { return false; }
size_t tc_workspace_bytes(const sige_conv_desc *, int, int) { return 0; }
int launch_conv_tc(const ConvParams &, cudaStream_t) { return SIGE_ERR_UNSUPPORTED; }

} // namespace sige
