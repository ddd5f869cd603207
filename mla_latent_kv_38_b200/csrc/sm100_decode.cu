// Absorbed MLA decode on the 5th-generation tensor cores (tcgen05), DeepSeek-V2
// head shape: d_c = 512 latent columns + d_r = 64 RoPE columns per cache row,
// heads in blocks of 128.
//
// What is computed (DeepSeek-V3 report notes eq. (10) with the absorbed query
// of "MLA(Multi-head Latent Attention): DeepSeek-V2 논문정리", "Key에 대한 수식
// 전개" / "Value에 대한 수식 전개"):
//   S = [q_abs ; q^R] . [c ; k^R]^T * scale   (M = 128 heads, K = 576)
//   causal mask, online softmax (exp2 domain)
//   O = P . c                                  (M = 128 heads, N = 512, K = keys)
// Every head reads every cache row, so both products are dense contractions
// with M = heads; the cache is streamed from HBM once.
//
// Mapping onto B200:
//  * A cluster of two CTAs (two SMs) issues cta_group::2 MMAs with M = 128: CTA
//    r owns heads [64r, 64r+64).  In the paired 128-row layout each SM's tensor
//    memory holds its 64 rows spread over all 128 lanes, so the 128 x 512 fp32
//    accumulator O needs 256 columns per SM and S (N = 64 keys) 32 columns;
//    one CTA alone could not hold O (512 columns) and S together.
//  * Per 64-row cache block (one page) each CTA loads by TMA (128-byte swizzle)
//    its 32 keys x 576 columns for S (the pair's B operand is split by keys)
//    and all 64 keys of the latent columns it contributes to P.V (the B
//    operand of P.V is split by latent columns): CTA 0 columns [0,128) and
//    [256,384), CTA 1 columns [128,256) and [384,512).
//  * Warp roles per CTA: warp 0 issues TMA, warp 1 allocates tensor memory
//    and (CTA 0 only) issues the MMAs, warps 2-5 run the softmax and the
//    epilogue, one thread per tensor-memory lane.  S is double buffered so the
//    softmax of block j overlaps P.V of block j-1.  The running max is
//    rescaled lazily (only when it grows by more than 2^8).
//  * Work: the key blocks of all (sequence, token, head block) units are laid
//    end to end and cut into equal contiguous ranges, one per cluster
//    (persistent, 74 clusters on 148 SMs).  A unit covered by one cluster is
//    written directly in bf16; otherwise each cluster writes an fp32 partial
//    and its log-sum-exp, merged by a reduction kernel.
//  * Every mbarrier wait is bounded by the global timer: on expiry the kernel
//    sets MLA_STATUS_TIMEOUT and unwinds instead of hanging.

#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "sm100_decode.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kThreads = 192;
constexpr int kClusters = 74;                     // 148 SMs / 2
constexpr int kDc = 512, kDr = 64, kRow = 576;    // row = c^KV || k^R
constexpr int kPage = 64;                         // cache rows per page
constexpr int kTile = 32;                         // keys per tile (half a page)
constexpr int kStages = 4;                        // TMA ring depth
constexpr int kSBuf = 4;                          // S accumulators in tensor memory
constexpr int kPBuf = 2;                          // P operand buffers

constexpr uint32_t kQChunk = 8192;                // 64 heads x 128 B
constexpr uint32_t kQBytes = 9 * kQChunk;         // 64 heads x 576 columns
constexpr uint32_t kSChunk = 2048;                // 16 keys x 128 B
constexpr uint32_t kSRegion = 9 * kSChunk;        // this CTA's 16 keys x 576
constexpr uint32_t kVSlot = 4096;                 // 32 keys x 128 B
constexpr uint32_t kVRegion = 4 * kVSlot;         // 32 keys x 256 latent columns
constexpr uint32_t kStageBytes = kSRegion + kVRegion;
constexpr uint32_t kPBytes = 4096;                // 64 heads x 32 keys bf16 (64-byte swizzle)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffStage = kOffQ + kQBytes;
constexpr uint32_t kOffP = kOffStage + kStages * kStageBytes;
constexpr uint32_t kOffXmax = kOffP + kPBuf * kPBytes;   // 2 x 128 floats
constexpr uint32_t kOffXsum = kOffXmax + 1024;           // 128 floats
constexpr uint32_t kOffBar = kOffXsum + 512;
constexpr uint32_t kOffMisc = kOffBar + 8 * 32;          // tmem base, abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;    // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

enum {
    BAR_Q_FULL = 0,
    BAR_Q_EMPTY = 1,
    BAR_KV_FULL = 2,                     // + stage
    BAR_KV_EMPTY = BAR_KV_FULL + kStages,
    BAR_S_FULL = BAR_KV_EMPTY + kStages, // + S buffer
    BAR_S_FREE = BAR_S_FULL + kSBuf,
    BAR_P_FULL = BAR_S_FREE + kSBuf,     // + P buffer
    BAR_P_FREE = BAR_P_FULL + kPBuf,
    BAR_DRAIN = BAR_P_FREE + kPBuf,
    NUM_BARS = BAR_DRAIN + 1
};
static_assert(NUM_BARS <= 32, "barrier area");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;                    // 2 x 128 columns (paired layout)
constexpr uint32_t kTmemS = 256;                  // kSBuf x 16 columns

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, kTile, 0, 0);
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, 256, 0, 1);

constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleThreshold = 8.0f;         // log2 units

struct Sm100Params {
    CUtensorMap tm_pool_s;    // pool as [rows][576], box 64 cols x 16 rows
    CUtensorMap tm_pool_v;    // pool as [rows][576], box 64 cols x 32 rows
    CUtensorMap tm_qa;        // q_abs as [n_tok*n_h][512], box 64 x 64
    CUtensorMap tm_qr;        // q_r   as [n_tok*n_h][64],  box 64 x 64
    const int32_t* block_table;
    const int32_t* prefix;    // (U + 1) exclusive prefix of tiles per unit
    const int4* unit_meta;    // (U) {kv_len, first cluster, parts, batch index}
    uint16_t* out_latent;
    float* out_lse;
    float* part_o;            // (C + U) slots x 128 rows x 512
    float* part_lse;          // (C + U) slots x 128
    int32_t* status;
    int n_h, n_hb, T_q, U, C, num_blocks, max_blocks;
    float scale_log2;
};

__device__ __forceinline__ bool wait_bar(uint32_t addr, uint32_t parity, volatile int* abort_flag,
                                         int32_t* status) {
    if (ptx::mbar_try_wait(addr, parity)) return true;
    const uint64_t t0 = ptx::global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (ptx::mbar_try_wait(addr, parity)) return true;
        if (*abort_flag) return false;
        if (ptx::global_timer_ns() - t0 > kTimeoutNs) {
            *abort_flag = 1;
            raise_status(status, MLA_STATUS_TIMEOUT);
            return false;
        }
    }
}

// Unit whose tile range contains global tile g (prefix is non-decreasing).
__device__ __forceinline__ int find_unit(const int32_t* prefix, int U, int g) {
    int lo = 0, hi = U - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= g) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Walks a cluster's tiles [g0, g1) unit by unit.
struct TileCursor {
    const int32_t* prefix;
    int g, g0, g1, u;
    __device__ void init(const int32_t* pf, int U, int g0_, int g1_) {
        prefix = pf;
        g = g0_;
        g0 = g0_;
        g1 = g1_;
        u = g0_ < g1_ ? find_unit(pf, U, g0_) : 0;
        skip();
    }
    __device__ void skip() {
        while (g < g1 && prefix[u + 1] <= g) ++u;
    }
    __device__ bool done() const { return g >= g1; }
    __device__ int j() const { return g - prefix[u]; }   // tile index within the unit
    __device__ bool seg_first() const { return g == g0 || g == prefix[u]; }
    __device__ bool seg_last() const { return g + 1 == g1 || g + 1 == prefix[u + 1]; }
    __device__ void next() {
        ++g;
        skip();
    }
};

// latent column chunk (64 wide) that V-region slot i of CTA `rank` holds:
// P.V instruction h takes N columns [0,128) from CTA 0 and [128,256) from CTA 1
__device__ __forceinline__ int owned_chunk(uint32_t rank, int i) {
    return 4 * (i >> 1) + 2 * static_cast<int>(rank) + (i & 1);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
mla_decode_sm100_kernel(const __grid_constant__ Sm100Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t rank = ptx::cluster_rank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cluster = blockIdx.x >> 1;

    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    auto bar = [&](int i) { return sbase + kOffBar + 8u * static_cast<uint32_t>(i); };
    auto leader_bar = [&](int i) { return ptx::map_to_rank(bar(i), 0); };

    if (threadIdx.x == 0) {
        ptx::mbar_init(bar(BAR_Q_FULL), 1);
        ptx::mbar_init(bar(BAR_Q_EMPTY), 1);
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(bar(BAR_KV_FULL + s), 1);
            ptx::mbar_init(bar(BAR_KV_EMPTY + s), 1);
        }
        for (int b = 0; b < kSBuf; ++b) {
            ptx::mbar_init(bar(BAR_S_FULL + b), 1);
            ptx::mbar_init(bar(BAR_S_FREE + b), 8);   // 4 softmax warps x 2 CTAs
        }
        for (int b = 0; b < kPBuf; ++b) {
            ptx::mbar_init(bar(BAR_P_FULL + b), 8);
            ptx::mbar_init(bar(BAR_P_FREE + b), 1);
        }
        ptx::mbar_init(bar(BAR_DRAIN), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&p.tm_pool_s);
        ptx::prefetch_tmap(&p.tm_pool_v);
        ptx::prefetch_tmap(&p.tm_qa);
        ptx::prefetch_tmap(&p.tm_qr);
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), kTmemCols);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // this cluster's contiguous range of global tiles; with fewer tiles than
    // clusters only the first `total` clusters work, so no range is empty
    const int total = p.prefix[p.U];
    const int Ce = min(p.C, total);
    const int g0 = cluster < Ce ? static_cast<int>((static_cast<long long>(cluster) * total) / Ce) : 0;
    const int g1 = cluster < Ce ? static_cast<int>((static_cast<long long>(cluster + 1) * total) / Ce) : 0;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && g0 < g1) {
            const uint64_t pol_stream = ptx::l2_policy_evict_first();
            const uint64_t pol_q = ptx::l2_policy_evict_last();
            TileCursor c;
            c.init(p.prefix, p.U, g0, g1);
            int it = 0, uc = 0;
            for (; !c.done(); ++it) {
                const int u = c.u, j = c.j();
                const int b = p.unit_meta[u].w;
                if (c.seg_first()) {
                    const int bt = u / p.n_hb, hb = u - bt * p.n_hb;
                    const int qrow = bt * p.n_h + hb * 128 + 64 * static_cast<int>(rank);
                    if (!wait_bar(bar(BAR_Q_EMPTY), (uc & 1) ^ 1, abort_flag, p.status)) break;
                    if (rank == 0) ptx::mbar_arrive_expect_tx(bar(BAR_Q_FULL), 2 * kQBytes);
                    const uint32_t qf = leader_bar(BAR_Q_FULL);
                    for (int cc = 0; cc < 8; ++cc)
                        ptx::tma_load_2d_pair(sbase + kOffQ + cc * kQChunk, &p.tm_qa, 64 * cc, qrow, qf, pol_q);
                    ptx::tma_load_2d_pair(sbase + kOffQ + 8 * kQChunk, &p.tm_qr, 0, qrow, qf, pol_q);
                }
                const int st = it % kStages;
                if (!wait_bar(bar(BAR_KV_EMPTY + st), ((it / kStages) & 1) ^ 1, abort_flag, p.status)) break;
                if (rank == 0) ptx::mbar_arrive_expect_tx(bar(BAR_KV_FULL + st), 2 * kStageBytes);
                int blk = p.block_table[static_cast<size_t>(b) * p.max_blocks + (j >> 1)];
                if (blk < 0 || blk >= p.num_blocks) {
                    raise_status(p.status, MLA_STATUS_BAD_BLOCK);
                    blk = 0;
                }
                const uint32_t kf = leader_bar(BAR_KV_FULL + st);
                const uint32_t stage = sbase + kOffStage + st * kStageBytes;
                const int row0 = blk * kPage + kTile * (j & 1);
                const int row_s = row0 + 16 * static_cast<int>(rank);
                for (int cc = 0; cc < 9; ++cc)
                    ptx::tma_load_2d_pair(stage + cc * kSChunk, &p.tm_pool_s, 64 * cc, row_s, kf, pol_stream);
                for (int i = 0; i < 4; ++i)
                    ptx::tma_load_2d_pair(stage + kSRegion + i * kVSlot, &p.tm_pool_v,
                                          64 * owned_chunk(rank, i), row0, kf, pol_stream);
                if (c.seg_last()) ++uc;
                c.next();
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (rank == 0 && lane == 0 && g0 < g1) {
            TileCursor cs, cp;
            cs.init(p.prefix, p.U, g0, g1);
            cp.init(p.prefix, p.U, g0, g1);
            int its = 0, itp = 0, ucs = 0;
            bool ok = true;
            uint64_t last = ptx::global_timer_ns();
            while (!cp.done()) {
                bool progress = false;
                // S(its) = Q K^T once its keys have landed and its accumulator is free
                if (!cs.done()) {
                    const int st = its % kStages, sb = its % kSBuf;
                    bool ready = !cs.seg_first() || ptx::mbar_test_wait(bar(BAR_Q_FULL), ucs & 1);
                    ready = ready && ptx::mbar_test_wait(bar(BAR_KV_FULL + st), (its / kStages) & 1);
                    ready = ready && ptx::mbar_test_wait(bar(BAR_S_FREE + sb), ((its / kSBuf) & 1) ^ 1);
                    if (ready) {
                        ptx::tc_fence_after();
                        const uint32_t sreg = sbase + kOffStage + st * kStageBytes;
                        const uint64_t a0 = ptx::smem_desc_sw128(sbase + kOffQ, 16, 1024);
                        const uint64_t b0 = ptx::smem_desc_sw128(sreg, 16, 1024);
#pragma unroll 4
                        for (int kk = 0; kk < 36; ++kk) {
                            const int c = kk >> 2, k4 = kk & 3;
                            // descriptor start addresses advance in 16-byte units
                            const uint64_t a = a0 + static_cast<uint64_t>((c * kQChunk + 32 * k4) >> 4);
                            const uint64_t bd = b0 + static_cast<uint64_t>((c * kSChunk + 32 * k4) >> 4);
                            ptx::mma_pair_ss(tmem_base + kTmemS + 16 * sb, a, bd, kIdescS, kk > 0 ? 1u : 0u);
                        }
                        ptx::mma_commit_pair(bar(BAR_S_FULL + sb), 0x3);
                        if (cs.seg_last()) {
                            ptx::mma_commit_pair(bar(BAR_Q_EMPTY), 0x3);
                            ++ucs;
                        }
                        ++its;
                        cs.next();
                        progress = true;
                    }
                }
                // O (+)= P V once the softmax has written P(itp)
                if (itp < its) {
                    const int pb = itp % kPBuf;
                    if (ptx::mbar_test_wait(bar(BAR_P_FULL + pb), (itp / kPBuf) & 1)) {
                        ptx::tc_fence_after();
                        const bool first = cp.seg_first();
                        const uint32_t vbase = sbase + kOffStage + (itp % kStages) * kStageBytes + kSRegion;
                        const uint64_t a0 = ptx::smem_desc_sw64(sbase + kOffP + pb * kPBytes, 16, 512);
                        const uint64_t b0 = ptx::smem_desc_sw128(vbase, kVSlot, 1024);
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int kk = 0; kk < 2; ++kk) {
                                const uint64_t a = a0 + static_cast<uint64_t>((32 * kk) >> 4);
                                const uint64_t bd = b0 + static_cast<uint64_t>((8192 * h + 2048 * kk) >> 4);
                                ptx::mma_pair_ss(tmem_base + kTmemO + 128 * h, a, bd, kIdescPV,
                                                 (first && kk == 0) ? 0u : 1u);
                            }
                        ptx::mma_commit_pair(bar(BAR_KV_EMPTY + itp % kStages), 0x3);
                        ptx::mma_commit_pair(bar(BAR_P_FREE + pb), 0x3);
                        ++itp;
                        cp.next();
                        progress = true;
                    }
                }
                if (progress) {
                    last = ptx::global_timer_ns();
                } else {
                    if (*abort_flag) { ok = false; break; }
                    if (ptx::global_timer_ns() - last > kTimeoutNs) {
                        *abort_flag = 1;
                        raise_status(p.status, MLA_STATUS_TIMEOUT);
                        ok = false;
                        break;
                    }
                }
            }
            if (!ok) {
                // let every issued MMA finish before the teardown frees anything
                ptx::mma_commit_pair(bar(BAR_DRAIN), 0x1);
                const uint64_t t0 = ptx::global_timer_ns();
                while (!ptx::mbar_try_wait(bar(BAR_DRAIN), 0) && ptx::global_timer_ns() - t0 < kTimeoutNs) {
                }
            }
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int wq = warp & 3;                     // tensor-memory lane quadrant
        const int l = wq * 32 + lane;                // lane = (row, half)
        const bool hi = l >= 64;
        const int m = l & 63;
        const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(wq * 32) << 16);
        float* xmax = reinterpret_cast<float*>(smem + kOffXmax);
        float* xsum = reinterpret_cast<float*>(smem + kOffXsum);
        TileCursor c;
        c.init(p.prefix, p.U, g0, g1);
        int it = 0;
        bool ok = true;
        while (!c.done() && ok) {
            const int u = c.u;
            const int4 meta = p.unit_meta[u];
            const int kv_len = meta.x;
            const int jfirst = c.j();
            float m_used = -INFINITY, l_part = 0.f;
            bool seg_last = false;
            do {
                const int j = c.j();
                const int sb = it % kSBuf;
                ok = wait_bar(bar(BAR_S_FULL + sb), (it / kSBuf) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                ptx::tc_fence_after();
                uint32_t r[16];
                ptx::tmem_ld16(t_lane + kTmemS + 16 * sb, r);
                ptx::tmem_wait_ld();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive_cluster(leader_bar(BAR_S_FREE + sb));

                const int key0 = j * kTile + (hi ? 16 : 0);
                float s[16];
                float mx = -INFINITY;
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    s[q] = (key0 + q < kv_len) ? __uint_as_float(r[q]) * p.scale_log2 : -INFINITY;
                    mx = fmaxf(mx, s[q]);
                }
                float* xb = xmax + (it & 1) * 128;
                xb[l] = mx;
                ptx::named_bar_sync(1, 128);
                mx = fmaxf(mx, xb[l ^ 64]);
                float new_m = m_used;
                bool resc = false;
                if (mx > m_used + kRescaleThreshold) {
                    new_m = mx;
                    resc = j > jfirst;
                }
                const float alpha = ex2(m_used - new_m);
                m_used = new_m;
                uint32_t pk[8];
                float ps = 0.f;
#pragma unroll
                for (int q = 0; q < 16; q += 2) {
                    const float p0 = ex2(s[q] - m_used), p1 = ex2(s[q + 1] - m_used);
                    ps += p0 + p1;
                    pk[q >> 1] = pack_bf16x2(p0, p1);
                }
                l_part = l_part * alpha + ps;

                const int pb = it % kPBuf;
                // P buffer pb is free once P.V(it - 2) has completed
                ok = wait_bar(bar(BAR_P_FREE + pb), ((it / kPBuf) & 1) ^ 1, abort_flag, p.status);
                // a rescale of O needs P.V(it - 1) complete as well
                if (ok && resc)
                    ok = wait_bar(bar(BAR_P_FREE + (pb ^ 1)), ((it - 1) / kPBuf) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                ptx::tc_fence_after();
                if (resc) {
#pragma unroll 1
                    for (int q = 0; q < 8; ++q) {
                        uint32_t o[32];
                        ptx::tmem_ld32(t_lane + kTmemO + 32 * q, o);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        ptx::tmem_st32(t_lane + kTmemO + 32 * q, o);
                    }
                    ptx::tmem_wait_st();
                }
                // keys past the end hold stale rows: zero this CTA's P.V operand
                // rows for them (their P is zero already)
                const int valid = kv_len - j * kTile;
                if (valid < kTile) {
                    const int bad = kTile - valid;
                    uint4* vreg = reinterpret_cast<uint4*>(smem + kOffStage + (it % kStages) * kStageBytes + kSRegion);
                    for (int e = l; e < 4 * bad * 8; e += 128) {
                        const int slot = e / (bad * 8), rem = e - slot * bad * 8;
                        const int row = valid + (rem >> 3), ch = rem & 7;
                        vreg[(slot * kVSlot + row * 128) / 16 + ch] = make_uint4(0, 0, 0, 0);
                    }
                }
                // P row m, keys (hi ? 16 : 0) + [0, 16): K-major, 64-byte rows,
                // 64-byte swizzle (16-byte chunk index XOR (row >> 1) & 3)
                unsigned char* Pb = smem + kOffP + pb * kPBytes;
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    const int chunk = (hi ? 2 : 0) + q2;
                    const int phys = chunk ^ ((m >> 1) & 3);
                    *reinterpret_cast<uint4*>(Pb + m * 64 + phys * 16) =
                        make_uint4(pk[4 * q2], pk[4 * q2 + 1], pk[4 * q2 + 2], pk[4 * q2 + 3]);
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive_cluster(leader_bar(BAR_P_FULL + pb));
                seg_last = c.seg_last();
                ++it;
                c.next();
            } while (!seg_last);
            if (!ok) break;

            // ---- epilogue of this unit segment: wait for P.V of its last tile
            const int e = it - 1;
            ok = wait_bar(bar(BAR_P_FREE + e % kPBuf), (e / kPBuf) & 1, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            ptx::tc_fence_after();
            xsum[l] = l_part;
            ptx::named_bar_sync(1, 128);
            const float lsum = l_part + xsum[l ^ 64];
            const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
            const float lse = lsum > 0.f ? (m_used + __log2f(lsum)) * kLn2 : -INFINITY;
            const int bt = u / p.n_hb, hb = u - bt * p.n_hb;
            const int head_in_unit = 64 * static_cast<int>(rank) + m;
            const bool whole = meta.z == 1;
            const size_t grow = static_cast<size_t>(bt) * p.n_h + hb * 128 + head_in_unit;
            const size_t slot = static_cast<size_t>(cluster) + u;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                const int col0 = 256 * h + (hi ? 128 : 0);
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    uint32_t o[32];
                    ptx::tmem_ld32(t_lane + kTmemO + 128 * h + 32 * q, o);
                    ptx::tmem_wait_ld();
                    const int col = col0 + 32 * q;
                    if (whole) {
                        uint4* dst = reinterpret_cast<uint4*>(p.out_latent + grow * kDc + col);
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            uint4 w;
                            w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
                            w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
                            w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
                            w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
                            dst[v] = w;
                        }
                    } else {
                        float4* dst = reinterpret_cast<float4*>(p.part_o + (slot * 128 + head_in_unit) * kDc + col);
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv, __uint_as_float(o[4 * v + 1]) * inv,
                                                 __uint_as_float(o[4 * v + 2]) * inv, __uint_as_float(o[4 * v + 3]) * inv);
                    }
                }
            }
            if (!hi) {
                if (whole) p.out_lse[grow] = lse;
                else p.part_lse[slot * 128 + head_in_unit] = lse;
            }
            ptx::tc_fence_before();
        }
    }

    // ---------------------------------------------------------------- teardown
    if (*abort_flag) {
        // give copies still in flight time to land before shared memory is released
        const uint64_t t0 = ptx::global_timer_ns();
        while (ptx::global_timer_ns() - t0 < 200000ull) {
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc_pair(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------
// Work schedule: tiles per unit, exclusive prefix, first cluster and number of
// clusters per unit.  One block of 1024 threads.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
mla_sm100_schedule_kernel(const int32_t* __restrict__ seq_lens, int B, int T_q, int n_hb,
                          int max_blocks, int C, int32_t* __restrict__ prefix,
                          int4* __restrict__ unit_meta, int32_t* status) {
    __shared__ int warp_tot[32];
    __shared__ int carry;
    const int U = B * T_q * n_hb;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < U; base += 1024) {
        const int u = base + threadIdx.x;
        int tiles = 0, kv = 0, b = 0;
        if (u < U) {
            const int bt = u / n_hb;
            b = bt / T_q;
            const int t = bt - b * T_q;
            const int L = seq_lens[b];
            if (L >= T_q && L <= max_blocks * kPage) {
                kv = L - T_q + t + 1;
                tiles = (kv + kTile - 1) / kTile;
            } else if (t == 0 && (u % n_hb) == 0) {
                raise_status(status, MLA_STATUS_BAD_SEQ_LEN);
            }
            unit_meta[u] = make_int4(kv, 0, 0, b);
        }
        // block exclusive scan of `tiles`
        int v = tiles;
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        if (lane == 31) warp_tot[w] = v;
        __syncthreads();
        if (w == 0) {
            int t = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            warp_tot[lane] = t;
        }
        __syncthreads();
        const int incl = v + (w > 0 ? warp_tot[w - 1] : 0) + carry;
        if (u < U) prefix[u + 1] = incl;
        if (u == 0) prefix[0] = 0;
        __syncthreads();
        if (threadIdx.x == 1023) carry = incl;
        __syncthreads();
    }
    __syncthreads();
    const long long T = carry;
    const long long Ce = T < C ? T : C;   // clusters that get work (all non-empty ranges)
    for (int u = threadIdx.x; u < U; u += 1024) {
        const int a = prefix[u], e = prefix[u + 1];
        if (e > a) {
            // cluster c covers tiles [floor(c T / Ce), floor((c+1) T / Ce)); tile g
            // lies in cluster floor(((g + 1) Ce - 1) / T)
            const int c0 = static_cast<int>(((static_cast<long long>(a) + 1) * Ce - 1) / T);
            const int c1 = static_cast<int>((static_cast<long long>(e) * Ce - 1) / T);
            unit_meta[u].y = c0;
            unit_meta[u].z = c1 - c0 + 1;
        }
    }
}

// LSE merge of the partial slots of every unit covered by more than one
// cluster; grid (128 rows, U units), 128 threads x 4 columns.
__global__ void __launch_bounds__(128)
mla_sm100_merge_kernel(const int4* __restrict__ unit_meta, const float* __restrict__ part_o,
                       const float* __restrict__ part_lse, uint16_t* __restrict__ out_latent,
                       float* __restrict__ out_lse, int n_h, int n_hb) {
    const int row = blockIdx.x, u = blockIdx.y;
    const int4 meta = unit_meta[u];
    const int bt = u / n_hb, hb = u - bt * n_hb;
    const size_t grow = static_cast<size_t>(bt) * n_h + hb * 128 + row;
    if (meta.x == 0) {   // invalid sequence length: defined output
        reinterpret_cast<uint2*>(out_latent + grow * kDc)[threadIdx.x] = make_uint2(0, 0);
        if (threadIdx.x == 0) out_lse[grow] = -INFINITY;
        return;
    }
    if (meta.z <= 1) return;
    float mx = -INFINITY;
    for (int i = 0; i < meta.z; ++i)
        mx = fmaxf(mx, part_lse[static_cast<size_t>(meta.y + i + u) * 128 + row]);
    float z = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = 0; i < meta.z; ++i) {
        const size_t slot = static_cast<size_t>(meta.y + i + u);
        const float ls = part_lse[slot * 128 + row];
        const float w = ls == -INFINITY ? 0.f : ex2((ls - mx) * kLog2e);
        z += w;
        const float4 v = reinterpret_cast<const float4*>(part_o + (slot * 128 + row) * kDc)[threadIdx.x];
        acc.x = fmaf(w, v.x, acc.x); acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z); acc.w = fmaf(w, v.w, acc.w);
    }
    const float inv = z > 0.f ? 1.f / z : 0.f;
    uint2 pk;
    pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(out_latent + grow * kDc)[threadIdx.x] = pk;
    if (threadIdx.x == 0) out_lse[grow] = z > 0.f ? mx + logf(z) : -INFINITY;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

bool make_map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                 uint32_t box_cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t r256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Sm100Ws {
    size_t prefix, meta, part_lse, part_o, total;
};

Sm100Ws sm100_ws(int U) {
    Sm100Ws w;
    w.prefix = 0;
    w.meta = w.prefix + r256(static_cast<size_t>(U + 1) * 4);
    w.part_lse = w.meta + r256(static_cast<size_t>(U) * 16);
    w.part_o = w.part_lse + r256(static_cast<size_t>(kClusters + U) * 128 * 4);
    w.total = w.part_o + r256(static_cast<size_t>(kClusters + U) * 128 * kDc * 4);
    return w;
}

}  // namespace

bool sm100_supports(int n_h, int d_c, int d_r) { return d_c == kDc && d_r == kDr && n_h % 128 == 0; }

size_t sm100_workspace_bytes(int n_h, int d_c, int B, int T_q) {
    if (n_h % 128 != 0 || d_c != kDc) return 0;
    return sm100_ws(B * T_q * (n_h / 128)).total;
}

int sm100_launches(int, int, int) { return 3; }

cudaError_t launch_decode_sm100(const DecodeParams& P, void* ws, int /*max_splits*/, cudaStream_t stream) {
    const int n_hb = P.n_h / 128;
    const int U = P.B * P.T_q * n_hb;
    if (U > 65535) return cudaErrorInvalidValue;
    const Sm100Ws w = sm100_ws(U);
    char* base = static_cast<char*>(ws);
    Sm100Params k;
    const uint64_t pool_rows = static_cast<uint64_t>(P.num_blocks) * P.block_size;
    const uint64_t q_rows = static_cast<uint64_t>(P.n_tok) * P.n_h;
    if (!make_map_2d(&k.tm_pool_s, P.pool, kRow, pool_rows, kRow * 2, 64, 16) ||
        !make_map_2d(&k.tm_pool_v, P.pool, kRow, pool_rows, kRow * 2, 64, 32) ||
        !make_map_2d(&k.tm_qa, P.q_abs, kDc, q_rows, kDc * 2, 64, 64) ||
        !make_map_2d(&k.tm_qr, P.q_r, kDr, q_rows, kDr * 2, 64, 64))
        return cudaErrorInvalidValue;
    k.block_table = P.block_table;
    k.prefix = reinterpret_cast<const int32_t*>(base + w.prefix);
    k.unit_meta = reinterpret_cast<const int4*>(base + w.meta);
    k.out_latent = P.out_latent;
    k.out_lse = P.out_lse;
    k.part_o = reinterpret_cast<float*>(base + w.part_o);
    k.part_lse = reinterpret_cast<float*>(base + w.part_lse);
    k.status = P.status;
    k.n_h = P.n_h;
    k.n_hb = n_hb;
    k.T_q = P.T_q;
    k.U = U;
    k.C = kClusters;
    k.num_blocks = P.num_blocks;
    k.max_blocks = P.max_blocks;
    k.scale_log2 = P.scale_log2;

    mla_sm100_schedule_kernel<<<1, 1024, 0, stream>>>(P.seq_lens, P.B, P.T_q, n_hb, P.max_blocks, kClusters,
                                                      reinterpret_cast<int32_t*>(base + w.prefix),
                                                      reinterpret_cast<int4*>(base + w.meta), P.status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(mla_decode_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    mla_decode_sm100_kernel<<<2 * kClusters, kThreads, kSmemBytes, stream>>>(k);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 mgrid(128, U);
    mla_sm100_merge_kernel<<<mgrid, 128, 0, stream>>>(k.unit_meta, k.part_o, k.part_lse, P.out_latent, P.out_lse,
                                                      P.n_h, n_hb);
    return cudaGetLastError();
}

}  // namespace mla
