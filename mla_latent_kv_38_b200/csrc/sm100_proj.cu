// Per-head projections around the absorbed decode on the tcgen05 tensor cores.
//
//   absorb_q: q_abs[n,i,:] = W^UK_i^T q^C[n,i,:]   ("MLA(Multi-head Latent
//             Attention): DeepSeek-V2 논문정리", "Key에 대한 수식 전개")
//   up_v:     o[n,i,:]     = W^UV_i latent[n,i,:]  (same page, "Value에 대한
//             수식 전개")
//
// Both are, per head i, a product D = A . B^T with the head's weight slice as
// A (M = 128 output features per CTA) and the tokens' activations as B
// (N = tokens, K = the contracted feature):
//
//   absorb_q: A = W^UK_i^T  (M = latent column c, K = d_h), stored [k][c], so A
//             is read MN-major; B = q^C[:, i, :] (K-major).
//   up_v:     A = W^UV_i    (M = head feature k, K = d_c), stored [k][c], so A
//             is K-major;  B = latent[:, i, :]  (K-major).
//
// With the few tokens of a decode step (N = 32 for 32 sequences) the weights
// dominate the bytes (2 x 16 MiB at the DeepSeek-V2 shape) and both calls are
// bound by HBM: each CTA loads its weight tile once with TMA, keeps it in
// shared memory and runs every token tile of its head against it.  One thread
// issues the MMAs (cta_group::1, M = 128, N = token tile <= 256) into tensor
// memory; four warps read the fp32 accumulator back (one TMEM lane per thread,
// i.e. one output feature per thread) into a bf16 tile in shared memory that
// TMA bulk tensor stores write out.

#include <cuda.h>

#include "common.cuh"
#include "sm100_proj.h"
#include "sm100_ptx.cuh"
#include "tensor_map.h"

namespace mla {
namespace {

constexpr int kThreads = 128;
constexpr int kM = 128;                       // output features per CTA
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr size_t kSmemLimit = 216 * 1024;     // A + one or two activation buffers per CTA
constexpr size_t kSmemPerSm = 233472;         // shared memory of one SM (228 KB)
constexpr size_t kSmemAttr = kSmemLimit + 4096;   // dynamic shared-memory limit set on the kernel (>= every launch)

struct ProjParams {
    CUtensorMap tm_a;   // weights, [n_h * d_h][d_c], 64-column boxes
    CUtensorMap tm_b;   // activations, [n_tok][n_h * K], boxes of 64 x nt
    CUtensorMap tm_out; // output, [n_tok][n_h * m_total], boxes of 64 x nt (stores)
    int32_t* status;    // device status word (may be null): MLA_STATUS_TIMEOUT
    int n_tok, n_h, d_h, d_c;
    int K;              // contracted length: d_h (absorb_q) or d_c (up_v)
    int m_total;        // output features per head: d_c (absorb_q) or d_h (up_v)
    int nt;             // token tile (multiple of 16, <= 256)
    int nbuf;           // activation buffers (1 or 2)
    uint32_t idesc;
    uint32_t tmem_cols;
};

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::global_timer_ns();
    while (!ptx::mbar_try_wait_suspend(bar, parity, 100000))
        if (ptx::global_timer_ns() - t0 > kTimeoutNs) return false;
    return true;
}

// grid (m_total / 128, n_h); 128 threads.  kAbsorb selects the A layout.
//
// Token tiles: with nbuf = 2 the activations of tile t + 1 are requested at
// the start of tile t, into the buffer tile t - 1 used, so that they land
// while tile t's MMAs and epilogue run.  The epilogue converts the
// accumulator (one output feature per thread, one token per column) to bf16
// in a [token][feature] tile laid out as a TMA store box (128-byte swizzle)
// in the buffer of the tile's own activations, which its MMAs no longer need,
// and writes it with two bulk tensor stores (64 features each); rows past the
// last token are clipped by the store.
template <bool kAbsorb>
__global__ void __launch_bounds__(kThreads, 1) mla_proj_sm100_kernel(const __grid_constant__ ProjParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                           ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const int K = p.K, nt = p.nt, nbuf = p.nbuf;
    const uint32_t a_bytes = static_cast<uint32_t>(kM) * K * 2;
    const uint32_t b_box = static_cast<uint32_t>(nt) * 128;      // 64 columns x nt rows
    const int kchunks = K / 64;
    const uint32_t b_bytes = kchunks * b_box;
    const uint32_t buf_bytes = b_bytes > 2 * b_box ? b_bytes : 2 * b_box;   // activations, later the staging tile
    const uint32_t sA = sbase, sB0 = sbase + a_bytes;
    const uint32_t bars = sB0 + nbuf * buf_bytes;                 // A full, B full x2, MMA done
    const uint32_t barA = bars, barD = bars + 8;
    auto barB = [&](int i) { return bars + 16 + 8 * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + (bars - sbase) + 32);
    __shared__ int s_ok;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int head = blockIdx.y;
    const int m0 = blockIdx.x * kM;
    const int n_tiles = (p.n_tok + nt - 1) / nt;

    griddep_launch_dependents();
    if (threadIdx.x == 0) {
        ptx::mbar_init(barA, 1);
        ptx::mbar_init(barD, 1);
        for (int i = 0; i < 2; ++i) ptx::mbar_init(barB(i), 1);
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

    // Boxes are issued by the lanes of warp 0 in parallel (one box each).
    auto load_b = [&](int t) {   // warp 0: token tile t into buffer t mod nbuf
        const int buf = t % nbuf;
        if (lane == 0) ptx::mbar_arrive_expect_tx(barB(buf), b_bytes);
        __syncwarp();
        if (lane < kchunks)
            ptx::tma_load_2d(sB0 + buf * buf_bytes + lane * b_box, &p.tm_b, head * K + 64 * lane, t * nt, barB(buf));
    };

    // The weights are read-only inputs no kernel writes: fetch them while the
    // previous kernel finishes, then wait for it before touching activations.
    if (warp == 0) {
        if (lane == 0) ptx::mbar_arrive_expect_tx(barA, a_bytes);
        __syncwarp();
        if (kAbsorb) {
            // two boxes of 64 latent columns x d_h rows: [mh][k][64 c]
            if (lane < 2) ptx::tma_load_2d(sA + lane * (K * 128), &p.tm_a, m0 + 64 * lane, head * p.d_h, barA);
        } else {
            // d_c / 64 boxes of 64 latent columns x 128 rows: [kc][k][64 c]
            if (lane < kchunks) ptx::tma_load_2d(sA + lane * (kM * 128), &p.tm_a, 64 * lane, head * p.d_h + m0, barA);
        }
    }
    griddep_wait();
    if (warp == 0) load_b(0);

    const int f = threadIdx.x;                    // this thread's output feature (TMEM lane) in the tile
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    // staging address of (token row r, feature f): half f / 64, 16-byte chunk
    // (f % 64) / 8 at position chunk ^ (r & 7), element f % 8
    const int half = f >> 6, chunk = (f & 63) >> 3, elem = f & 7;
    for (int t = 0; t < n_tiles; ++t) {
        const int buf = t % nbuf;
        if (warp == 0) {
            // the buffer of tile t - 1 holds its staging tile until its stores have read it
            if (lane == 0) ptx::bulk_wait_read_all();
            __syncwarp();
            if (nbuf == 2 && t + 1 < n_tiles) load_b(t + 1);
        }
        if (threadIdx.x == 0) {
            bool ok = (t > 0 || wait_bounded(barA, 0)) && wait_bounded(barB(buf), (t / nbuf) & 1);
            if (ok) {
                ptx::tc_fence_after();
                const uint32_t sB = sB0 + buf * buf_bytes;
                for (int s = 0; s < K / 16; ++s) {
                    uint64_t a, b;
                    if (kAbsorb) {
                        // MN-major: 8-row (k) atoms 1 KB apart, the two 64-column halves K*128 B apart
                        a = ptx::smem_desc_sw128(sA + s * 2048, K * 128, 1024);
                    } else {
                        a = ptx::smem_desc_sw128(sA + (s >> 2) * (kM * 128) + (s & 3) * 32, 16, 1024);
                    }
                    b = ptx::smem_desc_sw128(sB + (s >> 2) * b_box + (s & 3) * 32, 16, 1024);
                    ptx::mma1_ss(tmem, a, b, p.idesc, s > 0 ? 1u : 0u);
                }
                ptx::mma1_commit(barD);
                ok = wait_bounded(barD, t & 1);
            }
            if (!ok) raise_status(p.status, MLA_STATUS_TIMEOUT);
            s_ok = ok;
        }
        __syncthreads();
        if (!s_ok) break;
        ptx::tc_fence_after();
        unsigned char* stage = smem + (sB0 - sbase) + buf * buf_bytes;
        const int n0 = t * nt;
        const int nvalid = min(nt, p.n_tok - n0);
        for (int j0 = 0; j0 < nvalid; j0 += 16) {
            uint32_t r[16];
            ptx::tmem_ld16(t_lane + j0, r);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int row = j0 + j;
                *reinterpret_cast<uint16_t*>(stage + half * (nt * 128) + row * 128 + ((chunk ^ (row & 7)) * 16) +
                                             elem * 2) = f2bf(__uint_as_float(r[j]));
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            const uint32_t st = sB0 + buf * buf_bytes;
            const int x = head * p.m_total + m0;
            ptx::tma_store_2d(&p.tm_out, st, x, n0);
            ptx::tma_store_2d(&p.tm_out, st + nt * 128, x + 64, n0);
            ptx::bulk_commit_group();
        }
        // single buffer: the next tile's activations go where this staging tile is
        if (nbuf == 1 && t + 1 < n_tiles && warp == 0) {
            if (lane == 0) ptx::bulk_wait_read_all();
            __syncwarp();
            load_b(t + 1);
        }
    }
    if (threadIdx.x == 0) ptx::bulk_wait_all();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc1(tmem, p.tmem_cols);
}

uint32_t tmem_cols_for(int nt) {
    uint32_t c = 32;
    while (c < static_cast<uint32_t>(nt)) c <<= 1;
    return c;
}

// Bytes of one activation buffer (it later holds the nt x 128 staging tile).
size_t buf_bytes_for(int K, int nt) {
    const size_t b = static_cast<size_t>(K) * 2 * nt, st = static_cast<size_t>(nt) * 256;
    return b > st ? b : st;
}

// Token tile and buffer count: one buffer holding every token when they fit;
// otherwise two buffers (the next tile's activations load during this tile)
// if that still leaves tiles of 64 tokens or more, else one buffer of as many
// tokens as fit (fewer, larger tiles: fewer small MMAs).
void choose_tiles(int n_tok, int K, int* nt, int* nbuf) {
    const size_t a_bytes = static_cast<size_t>(kM) * K * 2;
    const size_t room = kSmemLimit - 2048 - a_bytes;
    auto cap_for = [&](int bufs) {
        int c = 256;
        while (c > 16 && bufs * buf_bytes_for(K, c) > room) c -= 16;
        return c;
    };
    const int want = (n_tok + 15) / 16 * 16;
    const int single = cap_for(1), dbl = cap_for(2);
    if (want <= single) {
        *nt = want;
        *nbuf = 1;
    } else if (dbl >= 64) {
        *nt = dbl;
        *nbuf = 2;
    } else {
        *nt = single;
        *nbuf = 1;
    }
}

template <bool kAbsorb>
cudaError_t launch_proj(ProjParams& p, cudaStream_t stream) {
    size_t smem = static_cast<size_t>(kM) * p.K * 2 + p.nbuf * buf_bytes_for(p.K, p.nt) + 1024 + 64;
    p.tmem_cols = tmem_cols_for(p.nt);
    // no more CTAs per SM than the 512 tensor-memory columns hold, so that no
    // allocation has to wait for another CTA to finish
    const size_t max_ctas = 512 / p.tmem_cols;
    const size_t min_smem = kSmemPerSm / (max_ctas + 1) - 1024 + 16;
    if (max_ctas < 16 && smem < min_smem) smem = min_smem;
    static std::atomic<uint64_t> smem_set{0};
    cudaError_t e = allow_smem_once(mla_proj_sm100_kernel<kAbsorb>, static_cast<int>(kSmemAttr), smem_set);
    if (e != cudaSuccess) return e;
    p.idesc = ptx::idesc_bf16_f32(kM, p.nt, kAbsorb ? 1 : 0, 0);
    dim3 grid(p.m_total / kM, p.n_h);
    return launch_pdl(mla_proj_sm100_kernel<kAbsorb>, grid, dim3(kThreads), smem, stream, p);
}

}  // namespace

bool sm100_absorb_supports(int d_h, int d_c) { return d_h % 64 == 0 && d_h <= 256 && d_c % kM == 0; }

bool sm100_up_v_supports(int d_h, int d_c) { return d_h % kM == 0 && d_c % 64 == 0 && d_c <= 512; }

cudaError_t launch_absorb_q_sm100(const uint16_t* q_c, const uint16_t* w_uk, uint16_t* q_abs, int n_tok, int n_h,
                                  int d_h, int d_c, int32_t* status, cudaStream_t stream) {
    ProjParams p;
    p.status = status;
    p.n_tok = n_tok;
    p.n_h = n_h;
    p.d_h = d_h;
    p.d_c = d_c;
    p.K = d_h;
    p.m_total = d_c;
    choose_tiles(n_tok, d_h, &p.nt, &p.nbuf);
    const uint64_t hk = static_cast<uint64_t>(n_h) * d_h;
    const uint64_t hm = static_cast<uint64_t>(n_h) * d_c;
    if (!make_map_2d(&p.tm_a, w_uk, d_c, hk, static_cast<uint64_t>(d_c) * 2, 64, d_h) ||
        !make_map_2d(&p.tm_b, q_c, hk, n_tok, hk * 2, 64, p.nt) ||
        !make_map_2d(&p.tm_out, q_abs, hm, n_tok, hm * 2, 64, p.nt))
        return cudaErrorInvalidValue;
    return launch_proj<true>(p, stream);
}

cudaError_t launch_up_v_sm100(const uint16_t* latent, const uint16_t* w_uv, uint16_t* out, int n_tok, int n_h,
                              int d_h, int d_c, int32_t* status, cudaStream_t stream) {
    ProjParams p;
    p.status = status;
    p.n_tok = n_tok;
    p.n_h = n_h;
    p.d_h = d_h;
    p.d_c = d_c;
    p.K = d_c;
    p.m_total = d_h;
    choose_tiles(n_tok, d_c, &p.nt, &p.nbuf);
    const uint64_t hk = static_cast<uint64_t>(n_h) * d_c;
    const uint64_t hm = static_cast<uint64_t>(n_h) * d_h;
    if (!make_map_2d(&p.tm_a, w_uv, d_c, static_cast<uint64_t>(n_h) * d_h, static_cast<uint64_t>(d_c) * 2, 64,
                     kM) ||
        !make_map_2d(&p.tm_b, latent, hk, n_tok, hk * 2, 64, p.nt) ||
        !make_map_2d(&p.tm_out, out, hm, n_tok, hm * 2, 64, p.nt))
        return cudaErrorInvalidValue;
    return launch_proj<false>(p, stream);
}

}  // namespace mla
