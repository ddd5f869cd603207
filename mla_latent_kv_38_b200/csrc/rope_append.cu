// Decoupled RoPE on q^R / k^R and the paged append of c^KV || k^R.
//
// "DeepSeek-V2 review" 2.3 and "Техотчёт DeepSeek-V2 (2024): MLA и экономика
// инференса", "Идея 2: отделённый RoPE": the RoPE key k^R is one vector per
// token shared by all heads and is cached after rotation; the query keeps one
// RoPE part per head.  "MLA(Multi-head Latent Attention): DeepSeek-V2
// 논문정리", "MLA 코드 구현": half-split rotate_half pairing, new tokens take
// absolute positions past_len .. T_total-1, and the cache is the latent
// concatenated with the rotated key.
//
// One warp per token.  The latent row is a 16-byte vector copy (bit exact);
// RoPE is float32 multiply / add with explicit round-to-nearest intrinsics so
// that no fused multiply-add changes the bits, then bf16 round to nearest even.

#include "common.cuh"
#include "kernels.h"

namespace mla {

__device__ __forceinline__ void rope_pair(uint16_t x1b, uint16_t x2b, float c, float s,
                                          uint16_t* y1, uint16_t* y2) {
    const float x1 = bf2f(x1b), x2 = bf2f(x2b);
    const float a = __fsub_rn(__fmul_rn(x1, c), __fmul_rn(x2, s));
    const float b = __fadd_rn(__fmul_rn(x2, c), __fmul_rn(x1, s));
    *y1 = f2bf(a);
    *y2 = f2bf(b);
}

__global__ void __launch_bounds__(256)
rope_append_kernel(uint16_t* __restrict__ q_r, const uint16_t* __restrict__ k_r,
                   const uint16_t* __restrict__ c_kv, const int32_t* __restrict__ positions,
                   const float* __restrict__ table, int max_pos,
                   const int32_t* __restrict__ block_table, int max_blocks,
                   uint16_t* __restrict__ pool, int num_blocks, int n_tok, int T_q,
                   int n_h, int d_c, int d_r, int block_size, int32_t* status) {
    const int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (n >= n_tok) return;
    const int b = n / T_q;
    const int p = positions[n];
    if (p < 0 || p >= max_pos || p / block_size >= max_blocks) {
        if (lane == 0) raise_status(status, MLA_STATUS_BAD_POSITION);
        return;
    }
    const int h = d_r >> 1;
    const float* cs = table + static_cast<size_t>(p) * d_r;

    // query RoPE, every head, in place
    if (q_r != nullptr) {
        uint16_t* q = q_r + static_cast<size_t>(n) * n_h * d_r;
        for (int e = lane; e < n_h * h; e += 32) {
            const int i = e / h, m = e - i * h;
            uint16_t* qi = q + i * d_r;
            rope_pair(qi[m], qi[m + h], cs[m], cs[h + m], &qi[m], &qi[m + h]);
        }
    }

    const int blk = block_table[static_cast<size_t>(b) * max_blocks + p / block_size];
    if (blk < 0 || blk >= num_blocks) {
        if (lane == 0) raise_status(status, MLA_STATUS_BAD_BLOCK);
        return;
    }
    const int row_elems = d_c + d_r;
    uint16_t* row = pool + (static_cast<size_t>(blk) * block_size + (p % block_size)) * row_elems;

    // latent: bit copy in 16-byte vectors
    const uint4* src = reinterpret_cast<const uint4*>(c_kv + static_cast<size_t>(n) * d_c);
    uint4* dst = reinterpret_cast<uint4*>(row);
    for (int v = lane; v < (d_c >> 3); v += 32) dst[v] = src[v];

    // shared RoPE key
    const uint16_t* kr = k_r + static_cast<size_t>(n) * d_r;
    for (int m = lane; m < h; m += 32) {
        rope_pair(kr[m], kr[m + h], cs[m], cs[h + m], &row[d_c + m], &row[d_c + m + h]);
    }
}

cudaError_t launch_rope_append(uint16_t* q_r, const uint16_t* k_r, const uint16_t* c_kv,
                               const int32_t* positions, const float* table, int max_pos,
                               const int32_t* block_table, int max_blocks, uint16_t* pool,
                               int num_blocks, int n_tok, int T_q, int n_h, int d_c, int d_r,
                               int block_size, int32_t* status, cudaStream_t stream) {
    const int warps = 8;
    const int grid = (n_tok + warps - 1) / warps;
    rope_append_kernel<<<grid, warps * 32, 0, stream>>>(q_r, k_r, c_kv, positions, table, max_pos,
                                                        block_table, max_blocks, pool, num_blocks,
                                                        n_tok, T_q, n_h, d_c, d_r, block_size,
                                                        status);
    return cudaGetLastError();
}

}  // namespace mla
