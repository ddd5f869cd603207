// Portable absorbed-MLA decode (CUDA cores, float32), any supported head shape,
// plus the split-KV log-sum-exp merge used by every decode kernel.
//
// Scores follow DeepSeek-V3 report notes eq. (10) with the absorbed query of
// "MLA(Multi-head Latent Attention): DeepSeek-V2 논문정리", "Key에 대한 수식
// 전개": s_j = scale * (q_abs . c_j + q^R . k^R_j); the output is the
// probability-weighted latent sum of "Value에 대한 수식 전개" (W^UV is applied
// afterwards by mla_up_v).  The causal limit of query t is
// seq_len - T_q + t ("MLA 코드 구현", generalised causal mask).
//
// Layout of the work: grid (split, token, head group of 32).  Each warp owns
// four heads, so a staged key row is read from shared memory once for all of
// them; the 8 warps share each 32-row key tile staged in shared memory with
// 16-byte loads.  The query rows stay bf16 in shared memory (the score scale
// multiplies each finished dot product), which with at most 128 registers a
// thread keeps two CTAs on an SM.  Online softmax in the exp2 domain.
//
// With an e4m3 pool (the low-bit cache of include/mla.h) the tile is staged as
// float32: each latent value is e4m3(code) * its group's scale, the RoPE key
// is widened from bf16; the rest of the kernel is the same.

#include "common.cuh"
#include "kernels.h"

namespace mla {

constexpr int kHeadsPerWarp = 4;
constexpr int kSimtHeads = 8 * kHeadsPerWarp;   // heads per CTA
constexpr int kSimtKeys = 32;

// Eight consecutive values of staged key row `row` from value 8 v on.
template <bool kE4m3>
__device__ __forceinline__ void load8(const unsigned char* tile, int row_stride, int row, int v, float* f) {
    if constexpr (kE4m3) {
        const float4* p = reinterpret_cast<const float4*>(tile + static_cast<size_t>(row) * row_stride) + 2 * v;
        const float4 a = p[0], b = p[1];
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else {
        unpack8(reinterpret_cast<const uint4*>(tile + static_cast<size_t>(row) * row_stride)[v], f);
    }
}

// Bytes of one staged key row: bf16 values plus 16 bytes, or float32 values
// plus 16 bytes (the padding spreads the rows over the shared-memory banks).
__host__ __device__ __forceinline__ int staged_row_bytes(int D, bool e4m3) { return (e4m3 ? 4 : 2) * D + 16; }

template <bool kE4m3>
__global__ void __launch_bounds__(256, 2)
decode_simt_kernel(DecodeParams P) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int D = P.d_c + P.d_r;
    const int row_bytes = staged_row_bytes(D, kE4m3);
    unsigned char* tile = smem_raw;                                          // [32][row_bytes]
    uint16_t* Qs = reinterpret_cast<uint16_t*>(smem_raw + kSimtKeys * row_bytes);  // [heads][D] bf16

    const int split = blockIdx.x, n = blockIdx.y, hg = blockIdx.z;
    const int b = n / P.T_q, t = n - b * P.T_q;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int head0 = hg * kSimtHeads + warp * kHeadsPerWarp;   // this warp's heads: head0, head0 + 1
    const bool warp_ok = head0 < P.n_h;

    int L = P.seq_lens[b];
    const bool len_ok = L >= P.T_q && L <= P.max_blocks * P.block_size;
    if (!len_ok && threadIdx.x == 0 && split == 0 && hg == 0 && t == 0)
        raise_status(P.status, MLA_STATUS_BAD_SEQ_LEN);
    const int kv_len = len_ok ? L - P.T_q + t + 1 : 0;
    const int ntiles = (kv_len + kSimtKeys - 1) / kSimtKeys;
    const int per = (ntiles + P.splits - 1) / P.splits;
    const int tile0 = split * per;
    const int tile1 = min(ntiles, tile0 + per);

    // stage the query rows as bf16 (the score scale is applied to each dot product)
    for (int e = threadIdx.x; e < kSimtHeads * D; e += blockDim.x) {
        const int w = e / D, c = e - w * D;
        const int hh = hg * kSimtHeads + w;
        uint16_t v = 0;
        if (hh < P.n_h) {
            v = c < P.d_c ? P.q_abs[(static_cast<size_t>(n) * P.n_h + hh) * P.d_c + c]
                          : P.q_r[(static_cast<size_t>(n) * P.n_h + hh) * P.d_r + (c - P.d_c)];
        }
        Qs[e] = v;
    }

    const int nchunk = P.d_c >> 3;                      // 8-column latent chunks
    float o[kHeadsPerWarp][2][8];
    float m_run[kHeadsPerWarp], l_run[kHeadsPerWarp];
#pragma unroll
    for (int h = 0; h < kHeadsPerWarp; ++h) {
        m_run[h] = -INFINITY;
        l_run[h] = 0.f;
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int k = 0; k < 8; ++k) o[h][u][k] = 0.f;
    }
    const uint16_t* q = Qs + warp * kHeadsPerWarp * D;  // the warp's query rows, one after the other

    for (int kt = tile0; kt < tile1; ++kt) {
        __syncthreads();
        // cooperative load of 32 cache rows through the block table
        if constexpr (kE4m3) {
            // work item: 16 latent codes (with their group's scale) or 8 RoPE-key values
            const E4m3Row L = e4m3_row(P.d_c, P.d_r);
            const int per_row = P.d_c / 16 + P.d_r / 8;
            for (int e = threadIdx.x; e < kSimtKeys * per_row; e += blockDim.x) {
                const int j = e / per_row, v = e - j * per_row;
                const int key = kt * kSimtKeys + j;
                const unsigned char* src = nullptr;
                if (key < kv_len) {
                    const int blk = P.block_table[static_cast<size_t>(b) * P.max_blocks + key / P.block_size];
                    if (blk >= 0 && blk < P.num_blocks)
                        src = P.pool8 + (static_cast<size_t>(blk) * P.block_size + key % P.block_size) * L.bytes;
                    else if (v == 0)
                        raise_status(P.status, MLA_STATUS_BAD_BLOCK);
                }
                float4* dst = reinterpret_cast<float4*>(tile + static_cast<size_t>(j) * row_bytes);
                if (v < P.d_c / 16) {
                    float f[16];
                    if (src != nullptr) {
                        const uint4 c = reinterpret_cast<const uint4*>(src)[v];
                        const float sc = reinterpret_cast<const float*>(src + L.scale_off)[v >> 2];
                        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float2 lo = e4m3x2_to_f32(static_cast<uint16_t>(w[k] & 0xFFFFu));
                            const float2 hi = e4m3x2_to_f32(static_cast<uint16_t>(w[k] >> 16));
                            f[4 * k] = lo.x * sc;
                            f[4 * k + 1] = lo.y * sc;
                            f[4 * k + 2] = hi.x * sc;
                            f[4 * k + 3] = hi.y * sc;
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < 16; ++k) f[k] = 0.f;
                    }
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        dst[4 * v + k] = make_float4(f[4 * k], f[4 * k + 1], f[4 * k + 2], f[4 * k + 3]);
                } else {
                    const int r = v - P.d_c / 16;   // 8 key values from column d_c + 8 r
                    float f[8];
                    if (src != nullptr) {
                        unpack8(reinterpret_cast<const uint4*>(src + L.kr_off)[r], f);
                    } else {
#pragma unroll
                        for (int k = 0; k < 8; ++k) f[k] = 0.f;
                    }
                    dst[P.d_c / 4 + 2 * r] = make_float4(f[0], f[1], f[2], f[3]);
                    dst[P.d_c / 4 + 2 * r + 1] = make_float4(f[4], f[5], f[6], f[7]);
                }
            }
        } else {
            for (int e = threadIdx.x; e < kSimtKeys * (D / 8); e += blockDim.x) {
                const int j = e / (D / 8), v = e - j * (D / 8);
                const int key = kt * kSimtKeys + j;
                uint4 val = make_uint4(0, 0, 0, 0);
                if (key < kv_len) {
                    const int blk = P.block_table[static_cast<size_t>(b) * P.max_blocks + key / P.block_size];
                    if (blk >= 0 && blk < P.num_blocks) {
                        const uint4* src = reinterpret_cast<const uint4*>(
                            P.pool + (static_cast<size_t>(blk) * P.block_size + key % P.block_size) * D);
                        val = src[v];
                    } else if (v == 0) {
                        raise_status(P.status, MLA_STATUS_BAD_BLOCK);
                    }
                }
                reinterpret_cast<uint4*>(tile + static_cast<size_t>(j) * row_bytes)[v] = val;
            }
        }
        __syncthreads();
        if (!warp_ok) continue;

        // scores: lane j scores key j against both of the warp's heads
        const int key = kt * kSimtKeys + lane;
        float s[kHeadsPerWarp];
#pragma unroll
        for (int h = 0; h < kHeadsPerWarp; ++h) s[h] = 0.f;
        for (int v = 0; v < D / 8; ++v) {
            float kf[8];
            load8<kE4m3>(tile, row_bytes, lane, v, kf);
#pragma unroll
            for (int h = 0; h < kHeadsPerWarp; ++h) {
                float qf[8];
                unpack8(*reinterpret_cast<const uint4*>(q + h * D + 8 * v), qf);
                float a = s[h];
#pragma unroll
                for (int k = 0; k < 8; ++k) a = fmaf(qf[k], kf[k], a);
                s[h] = a;
            }
        }
#pragma unroll
        for (int h = 0; h < kHeadsPerWarp; ++h) s[h] *= P.scale_log2;
        float p[kHeadsPerWarp];
#pragma unroll
        for (int h = 0; h < kHeadsPerWarp; ++h) {
            if (key >= kv_len) s[h] = -INFINITY;
            const float m_new = fmaxf(m_run[h], warp_max(s[h]));   // finite: key kt * 32 is visible
            const float alpha = ex2(m_run[h] - m_new);
            p[h] = ex2(s[h] - m_new);
            l_run[h] = l_run[h] * alpha + warp_sum(p[h]);
            m_run[h] = m_new;
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int k = 0; k < 8; ++k) o[h][u][k] *= alpha;
        }
        for (int j = 0; j < kSimtKeys; ++j) {
            float pj[kHeadsPerWarp];
            bool any = false;
#pragma unroll
            for (int h = 0; h < kHeadsPerWarp; ++h) {
                pj[h] = __shfl_sync(0xffffffffu, p[h], j);
                any = any || pj[h] != 0.f;
            }
            if (!any) continue;   // warp-uniform
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int ch = lane + 32 * u;
                if (ch < nchunk) {
                    float vf[8];
                    load8<kE4m3>(tile, row_bytes, j, ch, vf);
#pragma unroll
                    for (int h = 0; h < kHeadsPerWarp; ++h)
#pragma unroll
                        for (int k = 0; k < 8; ++k) o[h][u][k] = fmaf(pj[h], vf[k], o[h][u][k]);
                }
            }
        }
    }

#pragma unroll
    for (int h = 0; h < kHeadsPerWarp; ++h) {
        const int head = head0 + h;
        if (head >= P.n_h) break;
        const size_t row = static_cast<size_t>(n) * P.n_h + head;
        const bool empty = l_run[h] == 0.f;
        const float inv_l = empty ? 0.f : 1.f / l_run[h];
        const float lse = empty ? -INFINITY : (m_run[h] + __log2f(l_run[h])) * kLn2;
        if (P.splits == 1) {
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int ch = lane + 32 * u;
                if (ch < nchunk) {
                    uint4 w;
                    w.x = pack_bf16x2(o[h][u][0] * inv_l, o[h][u][1] * inv_l);
                    w.y = pack_bf16x2(o[h][u][2] * inv_l, o[h][u][3] * inv_l);
                    w.z = pack_bf16x2(o[h][u][4] * inv_l, o[h][u][5] * inv_l);
                    w.w = pack_bf16x2(o[h][u][6] * inv_l, o[h][u][7] * inv_l);
                    reinterpret_cast<uint4*>(P.out_latent + row * P.d_c)[ch] = w;
                }
            }
            if (lane == 0) P.out_lse[row] = lse;
        } else {
            float* po = P.part_o + (static_cast<size_t>(split) * P.n_tok * P.n_h + row) * P.d_c;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int ch = lane + 32 * u;
                if (ch < nchunk) {
                    float4* d = reinterpret_cast<float4*>(po + 8 * ch);
                    d[0] = make_float4(o[h][u][0] * inv_l, o[h][u][1] * inv_l, o[h][u][2] * inv_l,
                                       o[h][u][3] * inv_l);
                    d[1] = make_float4(o[h][u][4] * inv_l, o[h][u][5] * inv_l, o[h][u][6] * inv_l,
                                       o[h][u][7] * inv_l);
                }
            }
            if (lane == 0) P.part_lse[static_cast<size_t>(split) * P.n_tok * P.n_h + row] = lse;
        }
    }
}

// Split-KV merge: o = sum_s w_s o_s / sum_s w_s, lse = max + log sum_s w_s with
// w_s = exp(lse_s - max).  One block per (token, head).
__global__ void __launch_bounds__(128)
merge_splits_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                    uint16_t* __restrict__ out_latent, float* __restrict__ out_lse,
                    int rows, int d_c, int splits) {
    const int row = blockIdx.x;
    float m = -INFINITY;
    for (int s = 0; s < splits; ++s) m = fmaxf(m, part_lse[static_cast<size_t>(s) * rows + row]);
    float z = 0.f;
    for (int s = 0; s < splits; ++s) {
        const float ls = part_lse[static_cast<size_t>(s) * rows + row];
        z += (ls == -INFINITY) ? 0.f : ex2((ls - m) * kLog2e);
    }
    const float inv_z = z > 0.f ? 1.f / z : 0.f;
    for (int c = threadIdx.x * 4; c < d_c; c += blockDim.x * 4) {
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        for (int s = 0; s < splits; ++s) {
            const float ls = part_lse[static_cast<size_t>(s) * rows + row];
            if (ls == -INFINITY) continue;
            const float w = ex2((ls - m) * kLog2e) * inv_z;
            const float4 v = *reinterpret_cast<const float4*>(
                part_o + (static_cast<size_t>(s) * rows + row) * d_c + c);
            a0 = fmaf(w, v.x, a0); a1 = fmaf(w, v.y, a1);
            a2 = fmaf(w, v.z, a2); a3 = fmaf(w, v.w, a3);
        }
        uint2 pk;
        pk.x = pack_bf16x2(a0, a1);
        pk.y = pack_bf16x2(a2, a3);
        *reinterpret_cast<uint2*>(out_latent + static_cast<size_t>(row) * d_c + c) = pk;
    }
    if (threadIdx.x == 0) out_lse[row] = z > 0.f ? m + logf(z) : -INFINITY;
}

size_t simt_smem_bytes(int d_c, int d_r, bool e4m3) {
    const int D = d_c + d_r;
    return static_cast<size_t>(kSimtKeys) * staged_row_bytes(D, e4m3) + static_cast<size_t>(kSimtHeads) * D * 2;
}

cudaError_t launch_decode_simt(const DecodeParams& P, cudaStream_t stream) {
    const bool e4m3 = P.pool8 != nullptr;
    const size_t smem = simt_smem_bytes(P.d_c, P.d_r, e4m3);
    auto kernel = e4m3 ? decode_simt_kernel<true> : decode_simt_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(P.splits, P.n_tok, (P.n_h + kSimtHeads - 1) / kSimtHeads);
    kernel<<<grid, 256, smem, stream>>>(P);
    e = cudaGetLastError();
    if (e != cudaSuccess || P.splits == 1) return e;
    return launch_merge(P.part_o, P.part_lse, P.out_latent, P.out_lse, P.n_tok * P.n_h, P.d_c,
                        P.splits, stream);
}

cudaError_t launch_merge(const float* part_o, const float* part_lse, uint16_t* out_latent,
                         float* out_lse, int rows, int d_c, int splits, cudaStream_t stream) {
    merge_splits_kernel<<<rows, 128, 0, stream>>>(part_o, part_lse, out_latent, out_lse, rows, d_c,
                                                  splits);
    return cudaGetLastError();
}

}  // namespace mla
