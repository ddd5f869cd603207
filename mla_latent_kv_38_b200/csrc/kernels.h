// Internal launchers (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "mla.h"

namespace mla {

// Host-side argument checks shared by every entry point: MLA_OK or the
// MLA_ERR_* code for an unsupported configuration, and the score scale that
// cfg->scale selects (1/sqrt(d_h + d_r) when it is <= 0).
int check_config(const mla_config_t* cfg);
float effective_scale(const mla_config_t* cfg);

struct DecodeParams;

// pool: bf16 rows of d_c + d_r values, or (e4m3) rows in the layout of
// mla_e4m3_row_bytes
cudaError_t launch_rope_append(uint16_t* q_r, const uint16_t* k_r, const uint16_t* c_kv,
                               const int32_t* positions, const float* table, int max_pos,
                               const int32_t* block_table, int max_blocks, void* pool, bool e4m3,
                               int num_blocks, int n_tok, int T_q, int n_h, int d_c, int d_r,
                               int block_size, int32_t* status, cudaStream_t stream);

size_t simt_smem_bytes(int d_c, int d_r, bool e4m3);
cudaError_t launch_decode_simt(const DecodeParams& P, cudaStream_t stream);
cudaError_t launch_merge(const float* part_o, const float* part_lse, uint16_t* out_latent,
                         float* out_lse, int rows, int d_c, int splits, cudaStream_t stream);

cudaError_t launch_absorb_q_simt(const uint16_t* q_c, const uint16_t* w_uk, uint16_t* q_abs,
                                 int n_tok, int n_h, int d_h, int d_c, cudaStream_t stream);
cudaError_t launch_up_v_simt(const uint16_t* latent, const uint16_t* w_uv, uint16_t* out,
                             int n_tok, int n_h, int d_h, int d_c, cudaStream_t stream);

}  // namespace mla
