// tcgen05 / TMA decode kernel for the DeepSeek-V2 head shape (internal).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace mla {

struct DecodeParams;

bool sm100_supports(int n_h, int d_c, int d_r);
size_t sm100_workspace_bytes(int n_h, int d_c, int B, int T_q);
int sm100_launches(int B, int T_q, int max_splits);
cudaError_t launch_decode_sm100(const DecodeParams& P, void* ws, int max_splits, cudaStream_t stream);

}  // namespace mla
