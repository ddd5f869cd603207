// tcgen05 / TMA per-head projection kernels (internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

bool sm100_absorb_supports(int d_h, int d_c);
bool sm100_up_v_supports(int d_h, int d_c);
cudaError_t launch_absorb_q_sm100(const uint16_t* q_c, const uint16_t* w_uk, uint16_t* q_abs, int n_tok, int n_h,
                                  int d_h, int d_c, int32_t* status, cudaStream_t stream);
cudaError_t launch_up_v_sm100(const uint16_t* latent, const uint16_t* w_uv, uint16_t* out, int n_tok, int n_h,
                              int d_h, int d_c, int32_t* status, cudaStream_t stream);

}  // namespace mla
