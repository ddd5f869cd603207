// tcgen05 / TMA decode kernel for the DeepSeek-V2 head shape (internal).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mla {

struct DecodeParams;

bool sm100_supports(int n_h, int d_c, int d_r);
size_t sm100_workspace_bytes(int n_h, int d_c, int B, int T_q);
int sm100_launches(int B, int T_q, int n_h);
// Byte offset, inside the tcgen05 workspace region, of the per-unit metadata
// (int4 {kv_len, first cluster, parts, sequence} per unit).
size_t sm100_unit_meta_offset(int n_h, int B, int T_q);
// The next launch never issues one load and bounds every wait by wait_limit_ns.
void sm100_arm_timeout_test(uint64_t wait_limit_ns);
cudaError_t launch_decode_sm100(const DecodeParams& P, void* ws, int max_splits, cudaStream_t stream);

}  // namespace mla
