// Per-head projections around the absorbed decode, CUDA-core float32 version.
//
//   absorb_q: q_abs[n,i,:] = W^UK_i^T q^C[n,i,:]   ("MLA(Multi-head Latent
//             Attention): DeepSeek-V2 논문정리", "Key에 대한 수식 전개")
//   up_v:     o[n,i,:]     = W^UV_i latent[n,i,:]  (same page, "Value에 대한
//             수식 전개")
// W^UK_i and W^UV_i are the (d_h x d_c) slices w[i] of the (n_h, d_h, d_c)
// weight tensors.  Both calls read their 16 MiB (V2) weight once per launch.

#include "common.cuh"
#include "kernels.h"

namespace mla {

constexpr int kAbsCols = 128;   // latent columns per block (one per thread)
constexpr int kAbsTok = 16;     // tokens staged per pass

// grid (n_h, ceil(d_c / 128)); 128 threads; thread = one latent column.
__global__ void __launch_bounds__(128)
absorb_q_simt_kernel(const uint16_t* __restrict__ q_c, const uint16_t* __restrict__ w_uk,
                     uint16_t* __restrict__ q_abs, int n_tok, int n_h, int d_h, int d_c) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint16_t* Ws = reinterpret_cast<uint16_t*>(smem_raw);                   // [d_h][128]
    float* Qs = reinterpret_cast<float*>(Ws + static_cast<size_t>(d_h) * kAbsCols);  // [16][d_h]
    const int i = blockIdx.x;
    const int c = blockIdx.y * kAbsCols + threadIdx.x;
    const bool col_ok = c < d_c;
    const uint16_t* wi = w_uk + static_cast<size_t>(i) * d_h * d_c;
    for (int k = 0; k < d_h; ++k) Ws[k * kAbsCols + threadIdx.x] = col_ok ? wi[static_cast<size_t>(k) * d_c + c] : 0;
    for (int n0 = 0; n0 < n_tok; n0 += kAbsTok) {
        const int nt = min(kAbsTok, n_tok - n0);
        __syncthreads();
        for (int e = threadIdx.x; e < nt * d_h; e += blockDim.x) {
            const int tt = e / d_h, k = e - tt * d_h;
            Qs[e] = bf2f(q_c[(static_cast<size_t>(n0 + tt) * n_h + i) * d_h + k]);
        }
        __syncthreads();
        float acc[kAbsTok];
#pragma unroll
        for (int tt = 0; tt < kAbsTok; ++tt) acc[tt] = 0.f;
        for (int k = 0; k < d_h; ++k) {
            const float w = bf2f(Ws[k * kAbsCols + threadIdx.x]);
#pragma unroll
            for (int tt = 0; tt < kAbsTok; ++tt) acc[tt] = fmaf(Qs[tt * d_h + k], w, acc[tt]);
        }
        if (col_ok) {
            for (int tt = 0; tt < nt; ++tt)
                q_abs[(static_cast<size_t>(n0 + tt) * n_h + i) * d_c + c] = f2bf(acc[tt]);
        }
    }
}

// grid (n_h, ceil(d_h / 8)); 256 threads; warp = one output row k of head i,
// lanes split the d_c reduction in 16-byte chunks.
__global__ void __launch_bounds__(256)
up_v_simt_kernel(const uint16_t* __restrict__ latent, const uint16_t* __restrict__ w_uv,
                 uint16_t* __restrict__ out, int n_tok, int n_h, int d_h, int d_c) {
    const int i = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k = blockIdx.y * 8 + warp;
    if (k >= d_h) return;
    const int nchunk = d_c >> 3;
    float w[2][8];
    const uint4* wrow = reinterpret_cast<const uint4*>(w_uv + (static_cast<size_t>(i) * d_h + k) * d_c);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int ch = lane + 32 * u;
        if (ch < nchunk) unpack8(wrow[ch], w[u]);
        else
#pragma unroll
            for (int e = 0; e < 8; ++e) w[u][e] = 0.f;
    }
    for (int n = 0; n < n_tok; ++n) {
        const uint4* x = reinterpret_cast<const uint4*>(latent + (static_cast<size_t>(n) * n_h + i) * d_c);
        float s = 0.f;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int ch = lane + 32 * u;
            if (ch < nchunk) {
                float xf[8];
                unpack8(x[ch], xf);
#pragma unroll
                for (int e = 0; e < 8; ++e) s = fmaf(w[u][e], xf[e], s);
            }
        }
        s = warp_sum(s);
        if (lane == 0) out[(static_cast<size_t>(n) * n_h + i) * d_h + k] = f2bf(s);
    }
}

cudaError_t launch_absorb_q_simt(const uint16_t* q_c, const uint16_t* w_uk, uint16_t* q_abs,
                                 int n_tok, int n_h, int d_h, int d_c, cudaStream_t stream) {
    const size_t smem = static_cast<size_t>(d_h) * kAbsCols * 2 + static_cast<size_t>(kAbsTok) * d_h * 4;
    cudaError_t e = cudaFuncSetAttribute(absorb_q_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(n_h, (d_c + kAbsCols - 1) / kAbsCols);
    absorb_q_simt_kernel<<<grid, kAbsCols, smem, stream>>>(q_c, w_uk, q_abs, n_tok, n_h, d_h, d_c);
    return cudaGetLastError();
}

cudaError_t launch_up_v_simt(const uint16_t* latent, const uint16_t* w_uv, uint16_t* out,
                             int n_tok, int n_h, int d_h, int d_c, cudaStream_t stream) {
    dim3 grid(n_h, (d_h + 7) / 8);
    up_v_simt_kernel<<<grid, 256, 0, stream>>>(latent, w_uv, out, n_tok, n_h, d_h, d_c);
    return cudaGetLastError();
}

}  // namespace mla
