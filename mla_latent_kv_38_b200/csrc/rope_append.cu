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
// The latent row is a 16-byte vector copy (bit exact), or, into an e4m3 pool,
// its 64-column groups quantised to OCP FP8 E4M3 codes with a float32 scale
// each (layout and rounding in include/mla.h; the pages quote a ~6-bit cache,
// "DeepSeek-V2 review", 4.2 "Inference efficiency", and give no format).
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

// Blocks [0, q_blocks) rotate the queries: one thread per (token, head, four
// consecutive pairs m .. m+3), with 8-byte loads of both halves of the head's
// RoPE part and 16-byte loads of the cos / sin rows.  The remaining blocks do
// the cache append, one warp per token.
// One warp quantises a latent row of d_c <= 512 values: lane l takes values
// 16 l .. 16 l + 15, four lanes make a 64-column group.  All 32 lanes take
// part in the group maxima (lanes past d_c / 16 hold zeros).
__device__ __forceinline__ void quantize_row_e4m3(const uint16_t* __restrict__ src, unsigned char* row, int d_c,
                                                  int scale_off, int lane) {
    const bool active = 16 * lane < d_c;
    float x[16];
    if (active) {
        const uint4* s4 = reinterpret_cast<const uint4*>(src + 16 * lane);
        unpack8(s4[0], x);
        unpack8(s4[1], x + 8);
    } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) x[k] = 0.f;
    }
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(x[k]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    if (!active) return;
    const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t a = e4m3x2_from_f32(__fmul_rn(x[4 * k], inv), __fmul_rn(x[4 * k + 1], inv));
        const uint32_t b = e4m3x2_from_f32(__fmul_rn(x[4 * k + 2], inv), __fmul_rn(x[4 * k + 3], inv));
        w[k] = a | (b << 16);
    }
    *reinterpret_cast<uint4*>(row + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
    if ((lane & 3) == 0)
        *reinterpret_cast<float*>(row + scale_off + 4 * (lane >> 2)) = amax > 0.f ? __fdiv_rn(amax, 448.f) : 0.f;
}

// kE4m3: the pool holds e4m3 rows (row_bytes each, scales at scale_off, the
// bf16 key at kr_off); otherwise bf16 rows of d_c + d_r values.
template <bool kE4m3>
__global__ void __launch_bounds__(256)
rope_append_kernel(uint16_t* __restrict__ q_r, const uint16_t* __restrict__ k_r,
                   const uint16_t* __restrict__ c_kv, const int32_t* __restrict__ positions,
                   const float* __restrict__ table, int max_pos,
                   const int32_t* __restrict__ block_table, int max_blocks,
                   unsigned char* __restrict__ pool, int num_blocks, int n_tok, int T_q,
                   int n_h, int d_c, int d_r, int block_size, int q_blocks, int32_t* status) {
    griddep_launch_dependents();
    griddep_wait();   // q_r, the pool and the status word may be in use by earlier kernels
    const int h = d_r >> 1;
    if (static_cast<int>(blockIdx.x) < q_blocks) {
        // ---- query RoPE, in place
        const int quads = h >> 2;
        const long g = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
        if (g >= static_cast<long>(n_tok) * n_h * quads) return;
        const int m = static_cast<int>(g % quads) * 4;
        const long ni = g / quads;                      // token * n_h + head
        const int n = static_cast<int>(ni / n_h);
        const int p = positions[n];
        if (p < 0 || p >= max_pos || p / block_size >= max_blocks) return;   // flagged by the append
        uint16_t* q = q_r + ni * d_r;
        const float4 c = *reinterpret_cast<const float4*>(table + static_cast<size_t>(p) * d_r + m);
        const float4 sn = *reinterpret_cast<const float4*>(table + static_cast<size_t>(p) * d_r + h + m);
        const uint2 x1 = *reinterpret_cast<const uint2*>(q + m);
        const uint2 x2 = *reinterpret_cast<const uint2*>(q + h + m);
        const float cc[4] = {c.x, c.y, c.z, c.w}, ss[4] = {sn.x, sn.y, sn.z, sn.w};
        const uint32_t a_in[2] = {x1.x, x1.y}, b_in[2] = {x2.x, x2.y};
        uint32_t a_out[2], b_out[2];
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            uint16_t y1[2], y2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e)
                rope_pair(static_cast<uint16_t>(a_in[w] >> (16 * e)), static_cast<uint16_t>(b_in[w] >> (16 * e)),
                          cc[2 * w + e], ss[2 * w + e], &y1[e], &y2[e]);
            a_out[w] = y1[0] | (static_cast<uint32_t>(y1[1]) << 16);
            b_out[w] = y2[0] | (static_cast<uint32_t>(y2[1]) << 16);
        }
        *reinterpret_cast<uint2*>(q + m) = make_uint2(a_out[0], a_out[1]);
        *reinterpret_cast<uint2*>(q + h + m) = make_uint2(b_out[0], b_out[1]);
        return;
    }

    // ---- cache append, one warp per token
    const int n = (blockIdx.x - q_blocks) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (n >= n_tok) return;
    const int b = n / T_q;
    const int p = positions[n];
    if (p < 0 || p >= max_pos || p / block_size >= max_blocks) {
        if (lane == 0) raise_status(status, MLA_STATUS_BAD_POSITION);
        return;
    }
    const float* cs = table + static_cast<size_t>(p) * d_r;
    const int blk = block_table[static_cast<size_t>(b) * max_blocks + p / block_size];
    if (blk < 0 || blk >= num_blocks) {
        if (lane == 0) raise_status(status, MLA_STATUS_BAD_BLOCK);
        return;
    }
    const size_t slot = static_cast<size_t>(blk) * block_size + (p % block_size);
    uint16_t* key;   // the row's RoPE key (bf16)
    if constexpr (kE4m3) {
        const E4m3Row L = e4m3_row(d_c, d_r);
        unsigned char* row = pool + slot * L.bytes;
        quantize_row_e4m3(c_kv + static_cast<size_t>(n) * d_c, row, d_c, L.scale_off, lane);
        // padding bytes are zero
        for (int o = L.scale_off + 4 * (d_c / MLA_E4M3_GROUP) + lane; o < L.kr_off; o += 32) row[o] = 0;
        for (int o = L.kr_off + 2 * d_r + lane; o < L.bytes; o += 32) row[o] = 0;
        key = reinterpret_cast<uint16_t*>(row + L.kr_off);
    } else {
        uint16_t* row = reinterpret_cast<uint16_t*>(pool) + slot * (d_c + d_r);
        // latent: bit copy in 16-byte vectors
        const uint4* src = reinterpret_cast<const uint4*>(c_kv + static_cast<size_t>(n) * d_c);
        uint4* dst = reinterpret_cast<uint4*>(row);
        for (int v = lane; v < (d_c >> 3); v += 32) dst[v] = src[v];
        key = row + d_c;
    }

    // shared RoPE key
    const uint16_t* kr = k_r + static_cast<size_t>(n) * d_r;
    for (int m = lane; m < h; m += 32) {
        rope_pair(kr[m], kr[m + h], cs[m], cs[h + m], &key[m], &key[m + h]);
    }
}

cudaError_t launch_rope_append(uint16_t* q_r, const uint16_t* k_r, const uint16_t* c_kv,
                               const int32_t* positions, const float* table, int max_pos,
                               const int32_t* block_table, int max_blocks, void* pool, bool e4m3,
                               int num_blocks, int n_tok, int T_q, int n_h, int d_c, int d_r,
                               int block_size, int32_t* status, cudaStream_t stream) {
    const int threads = 256, warps = threads / 32;
    const long q_threads = q_r != nullptr ? static_cast<long>(n_tok) * n_h * (d_r / 8) : 0;
    const long q_blocks = (q_threads + threads - 1) / threads;
    const long a_blocks = (n_tok + warps - 1) / warps;
    if (q_blocks + a_blocks > 0x7fffffffL) return cudaErrorInvalidValue;
    const dim3 grid(static_cast<unsigned>(q_blocks + a_blocks));
    unsigned char* p = static_cast<unsigned char*>(pool);
    if (e4m3)
        return launch_pdl(rope_append_kernel<true>, grid, dim3(threads), 0, stream, q_r, k_r, c_kv, positions, table,
                          max_pos, block_table, max_blocks, p, num_blocks, n_tok, T_q, n_h, d_c, d_r, block_size,
                          static_cast<int>(q_blocks), status);
    return launch_pdl(rope_append_kernel<false>, grid, dim3(threads), 0, stream, q_r, k_r, c_kv, positions, table,
                      max_pos, block_table, max_blocks, p, num_blocks, n_tok, T_q, n_h, d_c, d_r, block_size,
                      static_cast<int>(q_blocks), status);
}

}  // namespace mla
