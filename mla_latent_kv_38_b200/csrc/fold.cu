// Folded projections on either side of the absorbed decode.
//
// "MLA(Multi-head Latent Attention): DeepSeek-V2 논문정리", "Key에 대한 수식
// 전개" (W^UK folds into the query projection) and "Value에 대한 수식 전개"
// (W^UV folds into the output projection); "Техотчёт DeepSeek-V2 (2024)",
// "Идея 1":
//
//   F_i = W^UK_i^T W^UQ_i   (d_c x d'_c per head)   q_abs[n, i, :] = F_i c^Q[n]
//   G_i = W^O_i W^UV_i      (d_model x d_c per head) u[n] = sum_i G_i latent[n, i, :]
//
// so the query side is one product from the query latent c^Q to q_abs, and the
// output side one product with K = n_h d_c from the decode's latent output to
// the model width.  The fold itself runs once per weight set (CUDA cores, fp32
// sums, bf16 results).  The two products stream their weights once through a
// ring of TMA stages into cta_group::1 MMAs (M = 128 weight rows, N = a token
// tile, K in chunks of 64): every weight byte is read once per call, which is
// what bounds them at decode sizes (F is 3 x the bytes of W^UQ + W^UK, G 3.6 x
// those of W^O + W^UV at the DeepSeek-V2 shape).  The output side splits K over
// CTAs and adds the fp32 partials in a second kernel.

#include <cuda.h>

#include "common.cuh"
#include "fold.h"
#include "sm100_ptx.cuh"
#include "tensor_map.h"

namespace mla {
namespace {

// ---------------------------------------------------------------------------
// The fold: C[b][r][c] = sum_k A[b][k][r] B[b][k][c], strided operands, fp32
// accumulation, bf16 (round to nearest even) results.  64 x 64 outputs per
// block, 4 x 4 per thread, K in steps of 16 through shared memory.
// ---------------------------------------------------------------------------

struct FoldMM {
    const uint16_t* A;
    const uint16_t* B;
    uint16_t* C;
    long sAb, sAk, sAr;   // A element (b, k, r) at b sAb + k sAk + r sAr
    long sBb, sBk, sBc;   // B element (b, k, c)
    long sCb, sCr, sCc;   // C element (b, r, c)
    int R, Cn, K;
};

__global__ void __launch_bounds__(256) fold_mm_kernel(const FoldMM p) {
    __shared__ float As[16][64 + 4];
    __shared__ float Bs[16][64 + 4];
    const long b = blockIdx.z;
    const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    // consecutive threads read along whichever index of A is contiguous
    const bool a_k_fast = p.sAk == 1;
    for (int k0 = 0; k0 < p.K; k0 += 16) {
        for (int e = threadIdx.x; e < 16 * 64; e += 256) {
            const int kk = a_k_fast ? (e & 15) : (e >> 6), j = a_k_fast ? (e >> 4) : (e & 63);
            const int k = k0 + kk, r = r0 + j;
            As[kk][j] = (k < p.K && r < p.R) ? bf2f(p.A[b * p.sAb + k * p.sAk + r * p.sAr]) : 0.f;
        }
        for (int e = threadIdx.x; e < 16 * 64; e += 256) {
            const int kk = e >> 6, j = e & 63;
            const int k = k0 + kk, c = c0 + j;
            Bs[kk][j] = (k < p.K && c < p.Cn) ? bf2f(p.B[b * p.sBb + k * p.sBk + c * p.sBc]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bb[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = r0 + ty * 4 + i;
        if (r >= p.R) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = c0 + tx * 4 + j;
            if (c < p.Cn) p.C[b * p.sCb + r * p.sCr + c * p.sCc] = f2bf(acc[i][j]);
        }
    }
}

cudaError_t launch_fold_mm(const FoldMM& p, int batch, cudaStream_t stream) {
    const dim3 grid((p.Cn + 63) / 64, (p.R + 63) / 64, batch);
    fold_mm_kernel<<<grid, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fold_weights(const uint16_t* w_uq, const uint16_t* w_uk, const uint16_t* w_uv,
                                const uint16_t* w_o, uint16_t* w_fold_q, uint16_t* w_fold_o, int n_h, int d_h,
                                int d_c, int d_cq, int d_model, cudaStream_t stream) {
    if (w_fold_q) {
        // F[i][c][d] = sum_k W^UK[i][k][c] W^UQ[i][k][d]
        FoldMM p;
        p.A = w_uk;
        p.sAb = static_cast<long>(d_h) * d_c, p.sAk = d_c, p.sAr = 1;
        p.B = w_uq;
        p.sBb = static_cast<long>(d_h) * d_cq, p.sBk = d_cq, p.sBc = 1;
        p.C = w_fold_q;
        p.sCb = static_cast<long>(d_c) * d_cq, p.sCr = d_cq, p.sCc = 1;
        p.R = d_c, p.Cn = d_cq, p.K = d_h;
        const cudaError_t e = launch_fold_mm(p, n_h, stream);
        if (e != cudaSuccess) return e;
    }
    if (w_fold_o) {
        // G[m][i][c] = sum_k W^O[m][i][k] W^UV[i][k][c]
        FoldMM p;
        p.A = w_o;
        p.sAb = d_h, p.sAk = 1, p.sAr = static_cast<long>(n_h) * d_h;
        p.B = w_uv;
        p.sBb = static_cast<long>(d_h) * d_c, p.sBk = d_c, p.sBc = 1;
        p.C = w_fold_o;
        p.sCb = d_c, p.sCr = static_cast<long>(n_h) * d_c, p.sCc = 1;
        p.R = d_model, p.Cn = d_c, p.K = d_h;
        const cudaError_t e = launch_fold_mm(p, n_h, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}


namespace {

// ---------------------------------------------------------------------------
// K-streamed product on tcgen05: D[row][token] = sum_k A[row][k] B[token][k]
// for 128 rows of A (TMEM lanes) and a tile of nt tokens (TMEM columns), A and
// B K-major bf16 read by TMA in 64-column chunks through a ring of stages.
// Grid (row tiles, slices, token tiles); a slice is a head (query side: A
// rows and output columns move with it) or a K range (output side: A and B
// columns move with it, output rows go to the slice's partial block).
// ---------------------------------------------------------------------------

constexpr int kThreads = 128;
constexpr int kRows = 128;                 // A rows per CTA (MMA M)
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint32_t kABytes = kRows * 128;  // one 64-column chunk of 128 rows (16 KB)
constexpr size_t kRingLimit = 200 * 1024;
constexpr int kMaxStages = 4;                 // two CTAs an SM at decode token counts

struct KGemm {
    CUtensorMap tm_a;      // A [rows][K] bf16, boxes 64 x 128
    CUtensorMap tm_b;      // B [tokens][K] bf16, boxes 64 x nt
    CUtensorMap tm_out;    // bf16 [tokens][cols] boxes 64 x nt, or fp32 [rows][cols] boxes 32 x nt
    int32_t* status;
    int n_tok, nt, k_chunks, stages;
    int a_rows_per_slice, a_k_per_slice, b_k_per_slice;
    int out_cols_per_slice, out_rows_per_slice;
    uint32_t idesc, tmem_cols;
};

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::global_timer_ns();
    while (!ptx::mbar_try_wait_suspend(bar, parity, 100000)) {
        if (*abort_flag) return false;
        if (ptx::global_timer_ns() - t0 > kTimeoutNs) {
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

template <bool kF32Out>
__global__ void __launch_bounds__(kThreads, 1) fold_gemm_kernel(const __grid_constant__ KGemm p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                           ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const int nt = p.nt, S = p.stages;
    const uint32_t b_bytes = static_cast<uint32_t>(nt) * 128;       // 64 columns x nt tokens
    const uint32_t stage_bytes = kABytes + b_bytes;
    const uint32_t bars = sbase + S * stage_bytes;
    auto full = [&](int s) { return bars + 8 * s; };
    auto empty = [&](int s) { return bars + 8 * (S + s); };
    const uint32_t done = bars + 8 * (2 * S);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + (bars - sbase) + 8 * (2 * S + 1));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + (bars - sbase) + 8 * (2 * S + 1) + 4);

    __shared__ int s_go;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slice = blockIdx.y;
    const int a_row0 = slice * p.a_rows_per_slice + blockIdx.x * kRows;
    const int a_k0 = slice * p.a_k_per_slice, b_k0 = slice * p.b_k_per_slice;
    const int n0 = blockIdx.z * nt;

    griddep_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(full(s), 1);
            ptx::mbar_init(empty(s), 1);
        }
        ptx::mbar_init(done, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&p.tm_a);
        ptx::prefetch_tmap(&p.tm_b);
        ptx::prefetch_tmap(&p.tm_out);
    }
    if (warp == 1) {
        ptx::tmem_alloc1(ptx::smem_u32(tmem_slot), p.tmem_cols);
        ptx::tmem_relinquish1();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_wait();   // the activations come from earlier kernels; the output may still be read by them

    if (warp == 0) {
        // producer: chunk c into stage c mod S, issued by lane c mod 8 (a
        // thread's copies run one after another, so consecutive stages come
        // from different threads)
        for (int c = 0; c < p.k_chunks; ++c) {
            const int s = c % S;
            bool ok = true;
            if (lane == (c & 7)) {
                ok = wait_bounded(empty(s), ((c / S) & 1) ^ 1, abort_flag);
                if (ok) {
                    const uint32_t st = sbase + s * stage_bytes;
                    ptx::mbar_arrive_expect_tx(full(s), stage_bytes);
                    ptx::tma_load_2d(st, &p.tm_a, a_k0 + 64 * c, a_row0, full(s));
                    ptx::tma_load_2d(st + kABytes, &p.tm_b, b_k0 + 64 * c, n0, full(s));
                }
            }
            if (!__all_sync(0xffffffffu, ok)) break;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            bool ok = true;
            for (int c = 0; c < p.k_chunks && ok; ++c) {
                const int s = c % S;
                ok = wait_bounded(full(s), (c / S) & 1, abort_flag);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t st = sbase + s * stage_bytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t a = ptx::smem_desc_sw128(st + kk * 32, 16, 1024);
                    const uint64_t b = ptx::smem_desc_sw128(st + kABytes + kk * 32, 16, 1024);
                    ptx::mma1_ss(tmem, a, b, p.idesc, (c | kk) ? 1u : 0u);
                }
                ptx::mma1_commit(empty(s));
            }
            // completes when every MMA issued above has (also on the abort path)
            ptx::mma1_commit(done);
        }
    }
    __syncwarp();
    wait_bounded(done, 0, abort_flag);
    // one decision for the whole CTA (the flag may be raised while others read it)
    __syncthreads();
    if (threadIdx.x == 0) {
        s_go = *abort_flag ? 0 : 1;
        if (!s_go) raise_status(p.status, MLA_STATUS_TIMEOUT);
    }
    __syncthreads();
    // the ring is idle now: its first bytes hold the output tile
    if (s_go) {
        ptx::tc_fence_after();
        const int f = threadIdx.x;   // the TMEM lane: row a_row0 + f of the product
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const int nvalid = min(nt, p.n_tok - n0);
        for (int j0 = 0; j0 < nvalid; j0 += 16) {
            uint32_t r[16];
            ptx::tmem_ld16(t_lane + j0, r);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int row = j0 + j;   // token
                if (kF32Out) {
                    // 4 boxes of 32 fp32 columns: box f / 32, chunk (f % 32) / 4, element f % 4
                    *reinterpret_cast<float*>(smem + (f >> 5) * (nt * 128) + row * 128 +
                                              (((((f & 31) >> 2)) ^ (row & 7)) * 16) + (f & 3) * 4) =
                        __uint_as_float(r[j]);
                } else {
                    // 2 boxes of 64 bf16 columns: box f / 64, chunk (f % 64) / 8, element f % 8
                    *reinterpret_cast<uint16_t*>(smem + (f >> 6) * (nt * 128) + row * 128 +
                                                 ((((f & 63) >> 3) ^ (row & 7)) * 16) + (f & 7) * 2) =
                        f2bf(__uint_as_float(r[j]));
                }
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            const int col = slice * p.out_cols_per_slice + blockIdx.x * kRows;
            const int row = slice * p.out_rows_per_slice + n0;
            if (kF32Out) {
                for (int q = 0; q < 4; ++q) ptx::tma_store_2d(&p.tm_out, sbase + q * (nt * 128), col + 32 * q, row);
            } else {
                for (int q = 0; q < 2; ++q) ptx::tma_store_2d(&p.tm_out, sbase + q * (nt * 128), col + 64 * q, row);
            }
            ptx::bulk_commit_group();
            ptx::bulk_wait_all();
        }
    } else {
        // give copies in flight time to land before shared memory is released
        const uint64_t t0 = ptx::global_timer_ns();
        while (ptx::global_timer_ns() - t0 < 200000ull) {
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc1(tmem, p.tmem_cols);
}

// u[n][m] = sum_s part[s][n][m] -> bf16; part rows of split s start at s * rows_pad.
__global__ void __launch_bounds__(256) fold_reduce_kernel(const float* __restrict__ part, uint16_t* __restrict__ u,
                                                          int n_tok, int d_model, int splits, int rows_pad) {
    griddep_launch_dependents();
    griddep_wait();
    const long quads = static_cast<long>(n_tok) * (d_model / 4);
    for (long g = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; g < quads;
         g += static_cast<long>(gridDim.x) * blockDim.x) {
        const long n = g / (d_model / 4), m4 = g - n * (d_model / 4);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < splits; ++s) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(part + (static_cast<long>(s) * rows_pad + n) *
                                                                        d_model) + m4);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        uint2 o;
        o.x = pack_bf16x2(acc.x, acc.y);
        o.y = pack_bf16x2(acc.z, acc.w);
        reinterpret_cast<uint2*>(u + n * d_model)[m4] = o;
    }
}

uint32_t tmem_cols_for(int nt) {
    uint32_t c = 32;
    while (c < static_cast<uint32_t>(nt)) c <<= 1;
    return c;
}

int token_tile(int n_tok) {
    const int want = (n_tok + 15) / 16 * 16;
    return want < 256 ? want : 256;
}

// As many stages as fit (at most kMaxStages; at least 2), leaving the first stage's
// bytes for the output tile (bf16: nt x 256 B, fp32: nt x 512 B).
int ring_stages(int nt, bool f32_out) {
    const size_t stage = kABytes + static_cast<size_t>(nt) * 128;
    int s = static_cast<int>(kRingLimit / stage);
    if (s > kMaxStages) s = kMaxStages;
    const size_t out_bytes = static_cast<size_t>(nt) * (f32_out ? 512 : 256);
    while (static_cast<size_t>(s) * stage < out_bytes) ++s;
    return s < 2 ? 2 : s;
}

template <bool kF32Out>
cudaError_t launch_gemm(KGemm& p, dim3 grid, cudaStream_t stream) {
    p.tmem_cols = tmem_cols_for(p.nt);
    p.idesc = ptx::idesc_bf16_f32(kRows, p.nt, 0, 0);
    const size_t smem = static_cast<size_t>(p.stages) * (kABytes + static_cast<size_t>(p.nt) * 128) + 1024 +
                        8 * (2 * p.stages + 1) + 16;
    static std::atomic<uint64_t> smem_set{0};
    cudaError_t e = allow_smem_once(fold_gemm_kernel<kF32Out>, static_cast<int>(kRingLimit + 4096), smem_set);
    if (e != cudaSuccess) return e;
    return launch_pdl(fold_gemm_kernel<kF32Out>, grid, dim3(kThreads), smem, stream, p);
}

// K split of the output side: slices of a whole number of 64-column chunks,
// at least 8 chunks each, about 8 CTAs per SM over the whole grid.
int o_splits(int n_h, int d_c, int d_model) {
    const int chunks = n_h * d_c / 64;
    const int m_tiles = d_model / kRows;
    int s = 1;
    while (s * 2 <= chunks / 8 && chunks % (s * 2) == 0 && m_tiles * s * 2 <= 8 * 148) s *= 2;
    return s;
}

}  // namespace

bool fold_q_supports(int d_c, int d_cq) { return d_c % kRows == 0 && d_cq % 64 == 0; }

bool fold_o_supports(int n_h, int d_c, int d_model) {
    return d_model % kRows == 0 && (static_cast<long>(n_h) * d_c) % 64 == 0;
}

cudaError_t launch_q_folded(const uint16_t* c_q, const uint16_t* w_fold_q, uint16_t* q_abs, int n_tok, int n_h,
                            int d_c, int d_cq, int32_t* status, cudaStream_t stream) {
    KGemm p;
    p.status = status;
    p.n_tok = n_tok;
    p.nt = token_tile(n_tok);
    p.k_chunks = d_cq / 64;
    p.stages = ring_stages(p.nt, false);
    p.a_rows_per_slice = d_c;          // slice = head: rows i d_c .. of F viewed as [n_h d_c][d_cq]
    p.a_k_per_slice = 0;
    p.b_k_per_slice = 0;               // every head reads the same c^Q
    p.out_cols_per_slice = d_c;        // q_abs viewed as [n_tok][n_h d_c]
    p.out_rows_per_slice = 0;
    const uint64_t rows = static_cast<uint64_t>(n_h) * d_c;
    if (!make_map_2d(&p.tm_a, w_fold_q, d_cq, rows, static_cast<uint64_t>(d_cq) * 2, 64, kRows) ||
        !make_map_2d(&p.tm_b, c_q, d_cq, n_tok, static_cast<uint64_t>(d_cq) * 2, 64, p.nt) ||
        !make_map_2d(&p.tm_out, q_abs, rows, n_tok, rows * 2, 64, p.nt))
        return cudaErrorInvalidValue;
    const dim3 grid(d_c / kRows, n_h, (n_tok + p.nt - 1) / p.nt);
    return launch_gemm<false>(p, grid, stream);
}

size_t o_folded_workspace_bytes(int n_h, int d_c, int d_model, int n_tok) {
    const int nt = token_tile(n_tok);
    const size_t rows_pad = static_cast<size_t>((n_tok + nt - 1) / nt) * nt;
    return static_cast<size_t>(o_splits(n_h, d_c, d_model)) * rows_pad * d_model * 4;
}

cudaError_t launch_o_folded(const uint16_t* latent, const uint16_t* w_fold_o, uint16_t* u, int n_tok, int n_h,
                            int d_c, int d_model, void* workspace, int32_t* status, cudaStream_t stream) {
    const int splits = o_splits(n_h, d_c, d_model);
    const int K = n_h * d_c;
    KGemm p;
    p.status = status;
    p.n_tok = n_tok;
    p.nt = token_tile(n_tok);
    const int rows_pad = (n_tok + p.nt - 1) / p.nt * p.nt;
    p.k_chunks = K / 64 / splits;
    p.stages = ring_stages(p.nt, true);
    p.a_rows_per_slice = 0;
    p.a_k_per_slice = p.k_chunks * 64;  // slice = a K range of G viewed as [d_model][n_h d_c]
    p.b_k_per_slice = p.k_chunks * 64;  // and of the latent viewed as [n_tok][n_h d_c]
    p.out_cols_per_slice = 0;
    p.out_rows_per_slice = rows_pad;    // partials [splits][rows_pad][d_model] fp32
    float* part = static_cast<float*>(workspace);
    if (!make_map_2d(&p.tm_a, w_fold_o, K, d_model, static_cast<uint64_t>(K) * 2, 64, kRows) ||
        !make_map_2d(&p.tm_b, latent, K, n_tok, static_cast<uint64_t>(K) * 2, 64, p.nt) ||
        !make_map_2d_f32(&p.tm_out, part, d_model, static_cast<uint64_t>(splits) * rows_pad,
                         static_cast<uint64_t>(d_model) * 4, 32, p.nt))
        return cudaErrorInvalidValue;
    const dim3 grid(d_model / kRows, splits, (n_tok + p.nt - 1) / p.nt);
    cudaError_t e = launch_gemm<true>(p, grid, stream);
    if (e != cudaSuccess) return e;
    const long quads = static_cast<long>(n_tok) * (d_model / 4);
    const int blocks = static_cast<int>((quads + 255) / 256 < 148 * 8 ? (quads + 255) / 256 : 148 * 8);
    return launch_pdl(fold_reduce_kernel, dim3(blocks), dim3(256), 0, stream, static_cast<const float*>(part), u,
                      n_tok, d_model, splits, rows_pad);
}

}  // namespace mla
