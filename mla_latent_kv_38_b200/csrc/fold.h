// Folded projections (internal): the weight fold on CUDA cores and the two
// folded products on the tcgen05 tensor cores.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mla {

// F_i = W^UK_i^T W^UQ_i -> w_fold_q (n_h, d_c, d_cq) and G_i = W^O_i W^UV_i ->
// w_fold_o (d_model, n_h, d_c), fp32 sums rounded to bf16; either output may be null.
cudaError_t launch_fold_weights(const uint16_t* w_uq, const uint16_t* w_uk, const uint16_t* w_uv,
                                const uint16_t* w_o, uint16_t* w_fold_q, uint16_t* w_fold_o, int n_h, int d_h,
                                int d_c, int d_cq, int d_model, cudaStream_t stream);

bool fold_q_supports(int d_c, int d_cq);
bool fold_o_supports(int n_h, int d_c, int d_model);

// q_abs[n, i, :] = F_i c_q[n]
cudaError_t launch_q_folded(const uint16_t* c_q, const uint16_t* w_fold_q, uint16_t* q_abs, int n_tok, int n_h,
                            int d_c, int d_cq, int32_t* status, cudaStream_t stream);

// u[n] = sum_i G_i latent[n, i, :], split over K with fp32 partials in the workspace
size_t o_folded_workspace_bytes(int n_h, int d_c, int d_model, int n_tok);
cudaError_t launch_o_folded(const uint16_t* latent, const uint16_t* w_fold_o, uint16_t* u, int n_tok, int n_h,
                            int d_c, int d_model, void* workspace, int32_t* status, cudaStream_t stream);

}  // namespace mla
