// Tensor-core (tcgen05) conv kernel: interface used by the ABI layer.
#pragma once

#include "conv_common.cuh"

namespace sige {

bool tc_supported(const sige_conv_desc *cd, int dtype);
size_t tc_workspace_bytes(const sige_conv_desc *cd, int batch, int ntiles);
int launch_conv_tc(const ConvParams &p, cudaStream_t stream);
int tc_schedule(const sige_conv_desc *cd, int tiles, int grid, int csize, int32_t *out, int n_out);

// 3x3 stride-1 layers on 8x8 tiles (pixels as the MMA's M, C_out as N).
bool conv8_supported(const sige_conv_desc *cd, int dtype);
int launch_conv8(const ConvParams &p, cudaStream_t stream);

// 1x1 and 3x3 "same" stride-1 layers on any tile size: a GEMM over the
// tiles' pixels, one tap-shifted copy of the tile per K chunk, K split across
// a cluster when the units are few.
bool tile_gemm_supported(const sige_conv_desc *cd, int dtype, bool dense);
int launch_tile_gemm(const ConvParams &p, cudaStream_t stream);
// A 3x3 layer with an input transform: the transform of the pixels its tiles
// read, once, into `scratch` (tile_gemm_scratch_bytes), then the tile GEMM on
// that copy without a transform.
size_t tile_gemm_scratch_bytes(const sige_conv_desc *cd, int batch, int in_h, int in_w);
int launch_tile_gemm_pre(const ConvParams &p, uint8_t *scratch, cudaStream_t stream);

} // namespace sige
