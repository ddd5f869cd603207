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
//    r owns heads [64r, 64r+64).  In the paired layout each SM's tensor memory
//    holds its 64 rows spread over all 128 lanes (lanes 0-63 take the first
//    half of N, lanes 64-127 the second), so O (64 heads x 512, fp32) takes 256
//    columns per SM and one S buffer (N = 256 keys) 128 columns; O and two S
//    buffers fill the 512 columns.
//  * A tile is 4 cache pages (256 keys).  S = [q_abs ; q^R] . K^T runs as 9 MMA
//    groups of K = 64 columns, N = 256: the pair's B operand is split by keys,
//    so each CTA loads its own 2 pages (128 keys x 576 columns).  O += P . V
//    runs as 2 x N = 256 per 16 keys: the B operand is split by latent
//    columns, so each CTA loads all 4 pages of its 256 latent columns (these
//    second reads hit L2).
//  * All operands arrive by TMA (128-byte swizzle) in two rings, each with one
//    producer warp and one in-order MMA consumer: S entries of 24 KB (one
//    column chunk of the CTA's 2 pages plus the same chunk of its 64 query
//    rows, re-read from L2 each tile so that no 72 KB query buffer has to stay
//    resident) and V entries of 32 KB (the CTA's 4 latent chunks of one page,
//    one 3-D box).
//  * Warp roles per CTA: warp 0 S producer, warp 1 tensor-memory allocation
//    and (CTA 0) the S MMAs, warps 2-5 softmax and epilogue (one thread per
//    tensor-memory lane), warp 6 (CTA 0) the P.V MMAs, warp 7 V producer.  S
//    is double buffered; P is written to shared memory in two key halves, each
//    released as soon as its MMAs complete, so the next tile's softmax overlaps
//    P.V.  The running max is rescaled lazily (only when it grows by 2^8).
//  * Work: the pages of all (sequence, token, head block) units are laid end
//    to end and cut into equal contiguous ranges, one per cluster (persistent,
//    74 clusters on 148 SMs).  A unit covered by one cluster is written
//    directly in bf16; otherwise each cluster writes an fp32 partial and its
//    log-sum-exp, merged by a reduction kernel.
//  * Every mbarrier wait is bounded by the global timer: on expiry the kernel
//    sets MLA_STATUS_TIMEOUT and unwinds instead of hanging.

#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "sm100_decode.h"
#include "sm100_ptx.cuh"
#include "tensor_map.h"

namespace mla {
namespace {

constexpr int kThreads = 384;   // 12 warps: S loads, S MMAs, P.V MMAs, V loads, 8 x softmax
constexpr int kClusters = 74;                     // 148 SMs / 2
constexpr int kDc = 512, kDr = 64, kRow = 576;    // row = c^KV || k^R
constexpr int kPage = 64;                         // cache rows per page (TMA box height)
constexpr int kTilePages = 4;                     // a tile = 4 pages = 256 keys (MMA N)
constexpr int kSRing = 4;                         // 24 KB entries, S operand stream
constexpr int kVRing = 3;                         // 32 KB entries (one page), P.V operand stream

constexpr uint32_t kBox = 8192;                   // one page x 64 columns (128 B rows)
constexpr uint32_t kSEntry = 3 * kBox;            // S ring entry: a column chunk of the CTA's 2 pages + of its 64 heads' query
constexpr uint32_t kVEntry = 4 * kBox;            // V ring entry: 4 latent chunks of one page
constexpr uint32_t kPBytes = 4 * kBox;            // 64 heads x 256 keys (4 blocks of 64 keys)
constexpr uint32_t kOffSRing = 0;
constexpr uint32_t kOffVRing = kOffSRing + kSRing * kSEntry;
constexpr uint32_t kOffP = kOffVRing + kVRing * kVEntry;
constexpr uint32_t kOffXmax = kOffP + kPBytes;    // 4 x 64 floats: partial row maxima (or sums)
constexpr uint32_t kOffBar = kOffXmax + 1024;
constexpr uint32_t kOffMisc = kOffBar + 8 * 32;   // tmem base, abort flag
constexpr uint32_t kSmemUsed = kOffMisc + 16;
// Dynamic shared memory: the buffers above from a 1024-byte aligned base; what
// the alignment leaves over at the end holds a copy of the cluster's unit
// prefix when it fits.
constexpr uint32_t kSmemBytes = 232448;
static_assert(kSmemUsed + 1024 <= kSmemBytes, "shared memory budget");

enum {
    BAR_SR_FULL = 0,                         // + slot (leader: both CTAs' bytes)
    BAR_SR_EMPTY = BAR_SR_FULL + kSRing,     // + slot (each CTA, MMA commit)
    BAR_VR_FULL = BAR_SR_EMPTY + kSRing,
    BAR_VR_EMPTY = BAR_VR_FULL + kVRing,
    BAR_S_FULL = BAR_VR_EMPTY + kVRing,      // + S buffer
    BAR_S_FREE = BAR_S_FULL + 2,             // + S buffer (leader, 8 warps)
    BAR_P_FULL = BAR_S_FREE + 2,             // + P half (leader, 2 warps x 2 CTAs)
    BAR_P_FREE = BAR_P_FULL + 2,             // + P half (each CTA, MMA commit)
    BAR_TAIL_READY = BAR_P_FREE + 2,         // each CTA, MMA thread arrives remotely
    BAR_TAIL_DONE = BAR_TAIL_READY + 1,      // leader, 8 warps
    BAR_DRAIN = BAR_TAIL_DONE + 1,           // S issuer's own drain on abort
    BAR_DRAIN_PV = BAR_DRAIN + 1,            // P.V issuer's
    NUM_BARS = BAR_DRAIN_PV + 1
};
static_assert(NUM_BARS <= 32, "barrier area");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;                    // 2 x 128 columns (paired layout)
constexpr uint32_t kTmemS = 256;                  // 2 x 128 columns

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 256, 0, 0);
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, 256, 0, 1);

constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint32_t kSuspendHintNs = 100000;      // a waiting thread sleeps up to 0.1 ms per try
constexpr int kSchedSmemUnits = 8192;             // units whose prefix the schedule keeps in shared memory
constexpr float kRescaleThreshold = 8.0f;         // log2 units

struct Sm100Params {
    CUtensorMap tm_pool;      // pool as [rows][576], box 64 cols x 64 rows
    CUtensorMap tm_pool_v;    // pool as [chunk][rows][64], box 64 cols x 64 rows x 4 chunks
    CUtensorMap tm_qa;        // q_abs as [n_tok*n_h][512], box 64 x 64
    CUtensorMap tm_qr;        // q_r   as [n_tok*n_h][64],  box 64 x 64
    const uint16_t* pool;     // for L2 prefetches of whole pages
    const int32_t* block_table;
    const int32_t* prefix;    // (U + 1) exclusive prefix of pages per unit
    const int4* unit_meta;    // (U) {kv_len, first cluster, parts, batch index}
    const int4* cluster_info; // (C) {first page, end page, first unit, last unit}
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
        if (ptx::mbar_try_wait_suspend(addr, parity, kSuspendHintNs)) return true;
        if (*abort_flag) return false;
        if (ptx::global_timer_ns() - t0 > kTimeoutNs) {
            *abort_flag = 1;
            raise_status(status, MLA_STATUS_TIMEOUT);
            return false;
        }
    }
}

// Unit whose page range contains global page g (prefix is non-decreasing).

// One tile of a cluster's work: up to 4 consecutive pages of one unit.
struct Tile {
    int u;          // unit = (b T_q + t) n_hb + hb
    int bt;         // query row b T_q + t of the unit
    int hb;         // head block of the unit
    int b;          // sequence of the unit
    int page0;      // first page, within the unit
    int np;         // pages in this tile (1..4)
    bool first;     // first tile of a unit segment (new Q, O starts from zero)
    bool last;      // last tile of a unit segment (epilogue follows)
    bool unit_end;  // the unit's last page is in this tile
};

// Walks a cluster's pages [g0, g1) as tiles.  The prefix entry of unit v is
// pf[v - off] (pf: a shared-memory copy of the cluster's range of the prefix,
// or the global array with off = 0).  The unit's (query row, head block,
// sequence) are kept up to date incrementally, without divisions.
struct TileWalker {
    const int32_t* pf;
    int off, g, g0, g1, u;
    int bt, hb, b, t, n_hb, T_q;
    __device__ int prefix(int v) const { return pf[v - off]; }
    __device__ void step_unit() {
        ++u;
        if (++hb == n_hb) {
            hb = 0;
            ++bt;
            if (++t == T_q) {
                t = 0;
                ++b;
            }
        }
    }
    __device__ void init(const int32_t* pf_, int off_, int u0, int g0_, int g1_, int n_hb_, int T_q_) {
        pf = pf_;
        off = off_;
        g = g0_;
        g0 = g0_;
        g1 = g1_;
        n_hb = n_hb_;
        T_q = T_q_;
        u = u0;
        bt = u0 / n_hb;
        hb = u0 - bt * n_hb;
        b = bt / T_q;
        t = bt - b * T_q;
        while (g < g1 && prefix(u + 1) <= g) step_unit();
    }
    __device__ bool done() const { return g >= g1; }
    __device__ Tile next() {
        Tile r;
        const int ubeg = prefix(u), uend = prefix(u + 1);
        r.u = u;
        r.bt = bt;
        r.hb = hb;
        r.b = b;
        r.page0 = g - ubeg;
        r.first = (g == g0) || (g == ubeg);
        const int seg_end = min(g1, uend);   // tiles start at the segment start
        r.np = min(kTilePages, seg_end - g);
        r.last = g + r.np == seg_end;
        r.unit_end = g + r.np == uend;
        g += r.np;
        while (g < g1 && prefix(u + 1) <= g) step_unit();
        return r;
    }
};

// P.V operand split: CTA r supplies latent chunks 4r .. 4r+3 (columns
// [256r, 256r+256)); instruction h (N = 256) takes chunks 4r+2h, 4r+2h+1 from
// each CTA, so TMEM column 128h + j of lane half r holds latent column
// 256r + 128h + j.

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

    griddep_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSRing; ++s) {
            ptx::mbar_init(bar(BAR_SR_FULL + s), 1);
            ptx::mbar_init(bar(BAR_SR_EMPTY + s), 1);
        }
        for (int s = 0; s < kVRing; ++s) {
            ptx::mbar_init(bar(BAR_VR_FULL + s), 1);
            ptx::mbar_init(bar(BAR_VR_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(bar(BAR_S_FULL + b), 1);
            ptx::mbar_init(bar(BAR_S_FREE + b), 16);   // 8 softmax warps x 2 CTAs
        }
        for (int hf = 0; hf < 2; ++hf) {
            ptx::mbar_init(bar(BAR_P_FULL + hf), 8);   // 4 softmax warps x 2 CTAs
            ptx::mbar_init(bar(BAR_P_FREE + hf), 1);
        }
        ptx::mbar_init(bar(BAR_TAIL_READY), 1);
        ptx::mbar_init(bar(BAR_TAIL_DONE), 16);
        ptx::mbar_init(bar(BAR_DRAIN), 1);
        ptx::mbar_init(bar(BAR_DRAIN_PV), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&p.tm_pool);
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
    // everything below reads what the schedule kernel (and the kernels before
    // it: q_abs, q^R, the appended cache rows) wrote
    griddep_wait();

    // this cluster's contiguous range of global pages [g0, g1) and the unit of
    // page g0, precomputed by the schedule kernel (empty range: no work)
    const int4 cinfo = p.cluster_info[cluster];
    const int g0 = cinfo.x, g1 = cinfo.y, u0 = cinfo.z;
    const int n_pre = cinfo.w - u0 + 2;   // prefix entries of units u0 .. cinfo.w, + 1
    int32_t* pre_s = reinterpret_cast<int32_t*>(smem + kSmemUsed);
    const int pre_cap = static_cast<int>(
        (reinterpret_cast<uintptr_t>(smem_raw) + kSmemBytes - reinterpret_cast<uintptr_t>(pre_s)) / 4);
    const bool pre_in_smem = g0 < g1 && n_pre <= pre_cap;
    if (pre_in_smem)
        for (int k = threadIdx.x; k < n_pre; k += kThreads) pre_s[k] = p.prefix[u0 + k];
    __syncthreads();
    const int32_t* pf_base = pre_in_smem ? pre_s : p.prefix;
    const int pf_off = pre_in_smem ? u0 : 0;

    // Two load streams, each consumed in order by one MMA issuer:
    //   S ring: S(i) = 9 entries (column chunk c of this CTA's pages 2r, 2r+1)
    //   V ring: V(i) = 2 entries per page (latent chunks owned for P.V h = 0, 1)
    // Block-table entries are plain global loads.  Each producer issues them a
    // tile or two before it needs them, so that their latency overlaps the
    // ring waits of the tiles in between; an entry is validated where it is
    // used (out-of-range entries are flagged and read as block 0).
    auto load_blk = [&](const Tile& t, int pg) -> int {
        return __ldg(p.block_table + static_cast<size_t>(t.b) * p.max_blocks + t.page0 + pg);
    };
    auto blk_row = [&](int blk) -> int {
        if (blk < 0 || blk >= p.num_blocks) {
            raise_status(p.status, MLA_STATUS_BAD_BLOCK);
            blk = 0;
        }
        return blk * kPage;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ S stream
        // Entry c of a tile holds column chunk c (64 columns) of this CTA's two
        // pages (keys) and of its 64 heads' query rows: the query is re-read from
        // L2 with every tile instead of staying resident, which leaves room for
        // deeper rings.  Lanes 0 and 1 load the pages, lane 2 the query chunk;
        // lane 0 of the leader CTA arms the full barrier with both CTAs' bytes.
        // Lane l < 2 owns this CTA's page 2r + l of every tile: its block for
        // tiles i, i+1, i+2 sits in b0, b1, b2 while tile i is issued.
        const int my_pg = 2 * static_cast<int>(rank) + (lane & 1);
        TileWalker w, wa;
        w.init(pf_base, pf_off, u0, g0, g1, p.n_hb, p.T_q);
        wa.init(pf_base, pf_off, u0, g0, g1, p.n_hb, p.T_q);
        int b0 = 0, b1 = 0, b2 = 0;
        bool h0 = false, h1 = false, h2 = false;
        // (the loads are unconditional, to a valid entry, so that nothing waits
        // for them until their value is used a tile or two later)
        auto look = [&](int& b, bool& h) {
            h = false;
            if (!wa.done()) {
                const Tile t = wa.next();
                h = lane < 2 && my_pg < t.np;
                b = load_blk(t, min(my_pg, t.np - 1));
            }
        };
        look(b0, h0);
        look(b1, h1);
        look(b2, h2);
        int e = 0;
        bool ok = g0 < g1;
        while (ok && !w.done()) {
            const Tile cur = w.next();
            const int qrow = cur.bt * p.n_h + cur.hb * 128 + 64 * static_cast<int>(rank);
            const int row = h0 ? blk_row(b0) : 0;
            const uint32_t tx = static_cast<uint32_t>(cur.np + 2) * kBox;    // both CTAs' pages and query chunks
            for (int c = 0; c < 9; ++c, ++e) {
                const int slot = e % kSRing;
                const uint32_t dst = sbase + kOffSRing + slot * kSEntry;
                bool good = true;
                if (lane < 3) {
                    good = wait_bar(bar(BAR_SR_EMPTY + slot), ((e / kSRing) & 1) ^ 1, abort_flag, p.status);
                    if (good && lane == 0 && rank == 0) ptx::mbar_arrive_expect_tx(bar(BAR_SR_FULL + slot), tx);
                    // one TMA instruction for the three lanes' boxes
                    const bool q_lane = lane == 2;
                    const void* tm = q_lane ? (c < 8 ? static_cast<const void*>(&p.tm_qa) : &p.tm_qr) : &p.tm_pool;
                    const int bx = q_lane ? (c < 8 ? 64 * c : 0) : 64 * c;
                    const int by = q_lane ? qrow : row;
                    if (good && (h0 || q_lane))
                        ptx::tma_load_2d_pair_normal(dst + (q_lane ? 2 : (lane & 1)) * kBox, tm, bx, by,
                                                     leader_bar(BAR_SR_FULL + slot));
                }
                if (!__all_sync(0xffffffffu, good)) { ok = false; break; }
            }
            b0 = b1; h0 = h1;
            b1 = b2; h1 = h2;
            look(b2, h2);
        }
    } else if (warp == 3) {
        // ------------------------------------------------------------ V stream
        // Lane pg < 4 holds the block of page pg of the current tile (v0) and of
        // the next one (v1).
        const uint64_t pol_v = ptx::l2_policy_evict_first();   // last use of these lines
        TileWalker w, wa;
        w.init(pf_base, pf_off, u0, g0, g1, p.n_hb, p.T_q);
        wa.init(pf_base, pf_off, u0, g0, g1, p.n_hb, p.T_q);
        int v0 = 0, v1 = 0;
        auto look = [&](int& v) {
            if (!wa.done()) {
                const Tile t = wa.next();
                v = load_blk(t, min(lane, t.np - 1));
            }
        };
        look(v0);
        look(v1);
        int e = 0;
        bool ok = g0 < g1;
        while (ok && !w.done()) {
            const Tile cur = w.next();
            for (int pg = 0; pg < cur.np && ok; ++pg, ++e) {
                const int row = blk_row(__shfl_sync(0xffffffffu, v0, pg));
                const int slot = e % kVRing;
                bool good = true;
                if (lane == 0) {
                    good = wait_bar(bar(BAR_VR_EMPTY + slot), ((e / kVRing) & 1) ^ 1, abort_flag, p.status);
                    if (good && rank == 0) ptx::mbar_arrive_expect_tx(bar(BAR_VR_FULL + slot), 2 * kVEntry);
                    // this CTA's 4 latent chunks of the page in one box: [chunk][row][64 columns]
                    if (good)
                        ptx::tma_load_3d_pair(sbase + kOffVRing + slot * kVEntry, &p.tm_pool_v, 0, row,
                                              4 * static_cast<int>(rank), leader_bar(BAR_VR_FULL + slot), pol_v);
                }
                if (!__all_sync(0xffffffffu, good)) { ok = false; break; }
            }
            v0 = v1;
            look(v1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ S = Q K^T issuer
        // S(i) occupies entries 9 i .. 9 i + 8 of the S ring (keys as B, query as A).
        if (rank == 0 && lane == 0 && g0 < g1) {
            TileWalker w;
            w.init(pf_base, pf_off, u0, g0, g1, p.n_hb, p.T_q);
            int i = 0;
            bool ok = true;
            while (ok && !w.done()) {
                w.next();
                const int e0 = 9 * i;
                const int sb = i & 1;
                if (!(ok = wait_bar(bar(BAR_S_FREE + sb), ((i >> 1) & 1) ^ 1, abort_flag, p.status))) break;
                ptx::tc_fence_after();   // the softmax's reads of this S buffer are done
                for (int c = 0; c < 9; ++c) {
                    const int e = e0 + c;
                    if (!(ok = wait_bar(bar(BAR_SR_FULL + e % kSRing), (e / kSRing) & 1, abort_flag, p.status))) break;
                    const uint32_t ent = sbase + kOffSRing + (e % kSRing) * kSEntry;
                    const uint64_t b0 = ptx::smem_desc_sw128(ent, 16, 1024);
                    const uint64_t a0 = ptx::smem_desc_sw128(ent + 2 * kBox, 16, 1024);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const uint64_t a = a0 + static_cast<uint64_t>((32 * k4) >> 4);
                        const uint64_t bd = b0 + static_cast<uint64_t>((32 * k4) >> 4);
                        ptx::mma_pair_ss(tmem_base + kTmemS + 128 * sb, a, bd, kIdescS, (c | k4) ? 1u : 0u);
                    }
                    ptx::mma_commit_pair(bar(BAR_SR_EMPTY + e % kSRing), 0x3);
                }
                if (!ok) break;
                ptx::mma_commit_pair(bar(BAR_S_FULL + sb), 0x3);
                ++i;
            }
            if (!ok) {
                // let every MMA this thread issued finish before the teardown frees anything
                ptx::mma_commit_pair(bar(BAR_DRAIN), 0x1);
                const uint64_t t0 = ptx::global_timer_ns();
                while (!ptx::mbar_try_wait(bar(BAR_DRAIN), 0) && ptx::global_timer_ns() - t0 < kTimeoutNs) {
                }
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ O += P V issuer
        // V(i) occupies the next 2 np entries of the V ring.
        if (rank == 0 && lane == 0 && g0 < g1) {
            TileWalker w;
            w.init(pf_base, pf_off, u0, g0, g1, p.n_hb, p.T_q);
            int i = 0, tails = 0, e = 0;
            bool ok = true;
            const uint64_t a0 = ptx::smem_desc_sw128(sbase + kOffP, 16, 1024);
            while (ok && !w.done()) {
                const Tile t = w.next();
                const int kv_len = __ldg(&p.unit_meta[t.u].x);   // read before the wait hides its latency
                const bool tail = t.unit_end && (kv_len % kPage) != 0;
                // P is written in two halves: keys [0,128) (pages 0, 1) by the softmax
                // warps of TMEM lanes 0-63, keys [128,256) by those of lanes 64-127;
                // each half is released as soon as its pages' MMAs complete.
                for (int pg = 0; pg < 4 && ok; ++pg) {
                    if (pg == 0 || pg == 2) {
                        if (pg == 2) ptx::mma_commit_pair(bar(BAR_P_FREE + 0), 0x3);
                        if (!(ok = wait_bar(bar(BAR_P_FULL + (pg >> 1)), i & 1, abort_flag, p.status))) break;
                        ptx::tc_fence_after();
                    }
                    if (pg >= t.np) continue;
                    if (tail && pg == t.np - 1) {
                        // the unit's last page holds rows past the end: once its V
                        // entry has landed, the softmax warps of both CTAs zero those
                        // rows (entries are consumed in ring order, so the earlier
                        // pages' slots are already free for this load)
                        if (!(ok = wait_bar(bar(BAR_VR_FULL + e % kVRing), (e / kVRing) & 1, abort_flag, p.status)))
                            break;
                        ptx::mbar_arrive_cluster(ptx::map_to_rank(bar(BAR_TAIL_READY), 0));
                        ptx::mbar_arrive_cluster(ptx::map_to_rank(bar(BAR_TAIL_READY), 1));
                        if (!(ok = wait_bar(bar(BAR_TAIL_DONE), tails & 1, abort_flag, p.status))) break;
                        ++tails;
                    }
                    if (!(ok = wait_bar(bar(BAR_VR_FULL + e % kVRing), (e / kVRing) & 1, abort_flag, p.status))) break;
                    for (int h = 0; h < 2; ++h) {
                        const uint64_t b0 =
                            ptx::smem_desc_sw128(sbase + kOffVRing + (e % kVRing) * kVEntry + h * 2 * kBox, kBox, 1024);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t a = a0 + static_cast<uint64_t>((pg * kBox + 32 * kk) >> 4);
                            const uint64_t bd = b0 + static_cast<uint64_t>((2048 * kk) >> 4);
                            ptx::mma_pair_ss(tmem_base + kTmemO + 128 * h, a, bd, kIdescPV,
                                             (t.first && pg == 0 && kk == 0) ? 0u : 1u);
                        }
                    }
                    ptx::mma_commit_pair(bar(BAR_VR_EMPTY + e % kVRing), 0x3);
                    ++e;
                }
                if (!ok) break;
                ptx::mma_commit_pair(bar(BAR_P_FREE + 1), 0x3);
                ++i;
            }
            if (!ok) {
                ptx::mma_commit_pair(bar(BAR_DRAIN_PV), 0x1);
                const uint64_t t0 = ptx::global_timer_ns();
                while (!ptx::mbar_try_wait(bar(BAR_DRAIN_PV), 0) && ptx::global_timer_ns() - t0 < kTimeoutNs) {
                }
            }
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        // Eight warps, two per tensor-memory lane quadrant: a thread owns lane l
        // (head row m, key half hi of the S tile, latent half hi of O) and
        // column group cg (64 of the lane's 128 S columns, 128 of its 256 O
        // columns), so four threads share a head row.
        const int sw = warp - 4;                     // softmax warp 0..7
        const int wq = warp & 3;                     // tensor-memory lane quadrant
        const int cg = sw >> 2;                      // column group
        const int l = wq * 32 + lane;                // lane = (row, half)
        const bool hi = l >= 64;
        const int m = l & 63;
        const int st = sw * 32 + lane;               // 0 .. 255 over the softmax warps
        const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(wq * 32) << 16);
        float* xmax = reinterpret_cast<float*>(smem + kOffXmax);   // [cg][l]
        TileWalker w, wa;      // wa runs one tile ahead: the next tile's unit data is loaded early
        w.init(pf_base, pf_off, u0, g0, g1, p.n_hb, p.T_q);
        wa.init(pf_base, pf_off, u0, g0, g1, p.n_hb, p.T_q);
        const int u_first = g0 < g1 ? wa.next().u : 0;
        int4 meta_nxt = __ldg(&p.unit_meta[u_first]);
        int i = 0, tails = 0;
        int v_before = 0;      // V ring entries of tiles before i
        bool ok = true;
        float m_used = -INFINITY, l_part = 0.f;
        // the four partial values of row m (both key halves, both column groups)
        auto row_max4 = [&]() {
            return fmaxf(fmaxf(xmax[m], xmax[64 + m]), fmaxf(xmax[128 + m], xmax[192 + m]));
        };
        while (ok && !w.done()) {
            const Tile t = w.next();
            const int4 meta = meta_nxt;
            int u_nxt = t.u;
            if (!wa.done()) u_nxt = wa.next().u;
            meta_nxt = __ldg(&p.unit_meta[u_nxt]);
            // keys of this tile that belong to this segment
            const int key_end = min(meta.x, kPage * (t.page0 + t.np));
            if (t.first) {
                m_used = -INFINITY;
                l_part = 0.f;
            }
            const int sb = i & 1;
            ok = wait_bar(bar(BAR_S_FULL + sb), (i >> 1) & 1, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            ptx::tc_fence_after();
            // This thread's 64 scores (row m, keys key0 ..) are read from tensor
            // memory twice: once for the row maximum, once for the weights.
            const uint32_t s_col = t_lane + kTmemS + 128 * sb + 64 * cg;
            const int key0 = kPage * t.page0 + (hi ? 128 : 0) + 64 * cg;
            const int nvalid = key_end - key0;   // scores of this thread that count (<= 0 .. >= 64)
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // independent chains
            {
                uint32_t r[2][32];
                ptx::tmem_ld32(s_col, r[0]);
                ptx::tmem_ld32(s_col + 32, r[1]);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (j < nvalid) mx4[j & 3] = fmaxf(mx4[j & 3], __uint_as_float(r[j >> 5][j & 31]));
            }
            float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            mx *= p.scale_log2;   // the scale is positive
            xmax[cg * 128 + l] = mx;
            ptx::named_bar_sync(1, 256);
            mx = row_max4();
            ptx::named_bar_sync(2, 256);   // every read done before the buffer is written again
            float new_m = m_used;
            bool resc = false;
            if (mx > m_used + kRescaleThreshold) {
                new_m = mx;
                resc = !t.first;
            }
            const float alpha = ex2(m_used - new_m);
            m_used = new_m;

            // This half of the P buffer must be free (the previous tile's P.V MMAs on
            // it complete); a rescale of O needs the whole previous P.V complete.
            const int hf = hi ? 1 : 0;
            ok = wait_bar(bar(BAR_P_FREE + hf), (i & 1) ^ 1, abort_flag, p.status);
            if (ok && !hi && __any_sync(0xffffffffu, resc))
                ok = wait_bar(bar(BAR_P_FREE + 1), (i & 1) ^ 1, abort_flag, p.status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            ptx::tc_fence_after();
            if (resc) {
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    uint32_t o[32];
                    ptx::tmem_ld32(t_lane + kTmemO + 128 * cg + 32 * q, o);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    ptx::tmem_st32(t_lane + kTmemO + 128 * cg + 32 * q, o);
                }
                ptx::tmem_wait_st();
            }
            // P row m, keys key0 + [0, 64) = one 64-key block (2 hi + cg) of P:
            // K-major, 128-byte rows, 128-byte swizzle (16-byte chunk index XOR row & 7)
            float ps2[2] = {0.f, 0.f};
            const float neg_m = -m_used;
            {
                uint32_t r[2][32];
                ptx::tmem_ld32(s_col, r[0]);
                ptx::tmem_ld32(s_col + 32, r[1]);
                ptx::tmem_wait_ld();
                uint32_t pk[32];
#pragma unroll
                for (int j = 0; j < 64; j += 2) {
                    const float s0 = __uint_as_float(r[j >> 5][j & 31]), s1 = __uint_as_float(r[j >> 5][(j & 31) + 1]);
                    const float p0 = j < nvalid ? ex2(fmaf(s0, p.scale_log2, neg_m)) : 0.f;
                    const float p1 = j + 1 < nvalid ? ex2(fmaf(s1, p.scale_log2, neg_m)) : 0.f;
                    ps2[(j >> 1) & 1] += p0 + p1;
                    pk[j >> 1] = pack_bf16x2(p0, p1);
                }
                unsigned char* Pb = smem + kOffP + (2 * hf + cg) * kBox + m * 128;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4*>(Pb + ((ch ^ (m & 7)) * 16)) =
                        make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
            }
            const float ps = ps2[0] + ps2[1];
            l_part = l_part * alpha + ps;
            // both reads of the S buffer are done
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster_relaxed(leader_bar(BAR_S_FREE + sb));
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(leader_bar(BAR_P_FULL + hf));

            // V ring position of this tile's entries
            const int v_start = v_before;
            v_before += t.np;
            if (t.unit_end && (meta.x % kPage) != 0) {
                // zero rows past the end in this CTA's V entry of the last page (4 chunks)
                ok = wait_bar(bar(BAR_TAIL_READY), tails & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                ++tails;
                const int valid = meta.x - kPage * (t.page0 + t.np - 1);
                const int bad = kPage - valid;
                const int et = v_start + (t.np - 1);
                unsigned char* ent = smem + kOffVRing + (et % kVRing) * kVEntry;
                for (int x = st; x < 4 * bad * 8; x += 256) {
                    const int chunk = x / (bad * 8);
                    const int rem = x - chunk * bad * 8;
                    const int row = valid + (rem >> 3), ch = rem & 7;
                    reinterpret_cast<uint4*>(ent + chunk * kBox + row * 128)[ch] = make_uint4(0, 0, 0, 0);
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive_cluster(leader_bar(BAR_TAIL_DONE));
            }

            if (t.last) {
                // ---- epilogue of this unit segment: wait for P.V of this tile (all
                // warps' P of this tile is in, so every read of the maxima is done)
                ok = wait_bar(bar(BAR_P_FREE + 1), i & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                ptx::tc_fence_after();
                xmax[cg * 128 + l] = l_part;   // partial row sums
                ptx::named_bar_sync(1, 256);
                const float lsum = xmax[m] + xmax[64 + m] + xmax[128 + m] + xmax[192 + m];
                ptx::named_bar_sync(2, 256);
                const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
                const float lse = lsum > 0.f ? (m_used + __log2f(lsum)) * kLn2 : -INFINITY;
                const int bt = t.bt, hb = t.hb;
                const int head_in_unit = 64 * static_cast<int>(rank) + m;
                const bool whole = meta.z == 1;
                const size_t grow = static_cast<size_t>(bt) * p.n_h + hb * 128 + head_in_unit;
                const size_t slot = static_cast<size_t>(cluster) + t.u;
                // This warp's 32 rows (consecutive heads) x 32 columns go through a
                // 4 KB shared-memory tile in the free P buffer (16-byte chunks
                // swizzled by row), so that each global store instruction writes
                // whole row segments instead of 32 scattered 16-byte pieces.
                unsigned char* stage = smem + kOffP + sw * 4096;
                const size_t grow0 = grow - lane;
                const size_t prow0 = slot * 128 + head_in_unit - lane;
                const int h = cg;   // this thread's 128 O columns
                const int col0 = 128 * h + (hi ? 256 : 0);
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    uint32_t o[32];
                    ptx::tmem_ld32(t_lane + kTmemO + 128 * h + 32 * q, o);
                    ptx::tmem_wait_ld();
                    const int col = col0 + 32 * q;
                    if (whole) {
                        // 32 bf16 = 64 B per row, 4 chunks at position k ^ ((row >> 1) & 3)
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            uint4 wv;
                            wv.x = pack_bf16x2(__uint_as_float(o[8 * k + 0]) * inv, __uint_as_float(o[8 * k + 1]) * inv);
                            wv.y = pack_bf16x2(__uint_as_float(o[8 * k + 2]) * inv, __uint_as_float(o[8 * k + 3]) * inv);
                            wv.z = pack_bf16x2(__uint_as_float(o[8 * k + 4]) * inv, __uint_as_float(o[8 * k + 5]) * inv);
                            wv.w = pack_bf16x2(__uint_as_float(o[8 * k + 6]) * inv, __uint_as_float(o[8 * k + 7]) * inv);
                            *reinterpret_cast<uint4*>(stage + lane * 64 + ((k ^ ((lane >> 1) & 3)) * 16)) = wv;
                        }
                        __syncwarp();
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int row = 8 * j + (lane >> 2), k = lane & 3;
                            const uint4 wv =
                                *reinterpret_cast<const uint4*>(stage + row * 64 + ((k ^ ((row >> 1) & 3)) * 16));
                            *reinterpret_cast<uint4*>(p.out_latent + (grow0 + row) * kDc + col + 8 * k) = wv;
                        }
                        __syncwarp();
                    } else {
                        // 32 floats = 128 B per row, 8 chunks at position k ^ (row & 7)
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            *reinterpret_cast<float4*>(stage + lane * 128 + ((k ^ (lane & 7)) * 16)) =
                                make_float4(__uint_as_float(o[4 * k]) * inv, __uint_as_float(o[4 * k + 1]) * inv,
                                            __uint_as_float(o[4 * k + 2]) * inv, __uint_as_float(o[4 * k + 3]) * inv);
                        __syncwarp();
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int row = 4 * j + (lane >> 3), k = lane & 7;
                            const float4 v = *reinterpret_cast<const float4*>(stage + row * 128 + ((k ^ (row & 7)) * 16));
                            *reinterpret_cast<float4*>(p.part_o + (prow0 + row) * kDc + col + 4 * k) = v;
                        }
                        __syncwarp();
                    }
                }
                if (!hi && cg == 0) {
                    if (whole) p.out_lse[grow] = lse;
                    else p.part_lse[slot * 128 + head_in_unit] = lse;
                }
                ptx::tc_fence_before();
            }
            ++i;
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
                          int4* __restrict__ unit_meta, int4* __restrict__ cluster_info, int32_t* status) {
    __shared__ int warp_tot[32];
    __shared__ int carry;
    __shared__ int pre_s[kSchedSmemUnits + 1];   // the prefix again, for the searches below
    griddep_launch_dependents();
    griddep_wait();   // the workspace may still be read by an earlier decode call's kernels
    const int U = B * T_q * n_hb;
    const bool in_smem = U <= kSchedSmemUnits;
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
                tiles = (kv + kPage - 1) / kPage;
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
        if (u < U) {
            prefix[u + 1] = incl;
            if (in_smem) pre_s[u + 1] = incl;
        }
        if (u == 0) {
            prefix[0] = 0;
            if (in_smem) pre_s[0] = 0;
        }
        __syncthreads();
        if (threadIdx.x == 1023) carry = incl;
        __syncthreads();
    }
    __syncthreads();
    const int* pf = in_smem ? pre_s : prefix;
    const long long T = carry;
    const long long Ce = T < C ? T : C;   // clusters that get work (all non-empty ranges)
    for (int u = threadIdx.x; u < U; u += 1024) {
        const int a = pf[u], e = pf[u + 1];
        if (e > a) {
            // cluster c covers tiles [floor(c T / Ce), floor((c+1) T / Ce)); tile g
            // lies in cluster floor(((g + 1) Ce - 1) / T)
            const int c0 = static_cast<int>(((static_cast<long long>(a) + 1) * Ce - 1) / T);
            const int c1 = static_cast<int>((static_cast<long long>(e) * Ce - 1) / T);
            unit_meta[u].y = c0;
            unit_meta[u].z = c1 - c0 + 1;
        }
    }
    // per cluster: page range and the unit holding its first page
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += 1024) {
        int4 ci = make_int4(0, 0, 0, 0);
        if (c < Ce) {
            const int a = static_cast<int>((static_cast<long long>(c) * T) / Ce);
            const int e = static_cast<int>((static_cast<long long>(c + 1) * T) / Ce);
            int lo = 0, hi = U - 1;   // last unit with prefix <= a
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (pf[mid] <= a) lo = mid; else hi = mid - 1;
            }
            int lo2 = lo, hi2 = U - 1;   // last unit with prefix <= e - 1 (holds the range's last page)
            while (lo2 < hi2) {
                const int mid = (lo2 + hi2 + 1) >> 1;
                if (pf[mid] <= e - 1) lo2 = mid; else hi2 = mid - 1;
            }
            ci = make_int4(a, e, lo, lo2);
        }
        cluster_info[c] = ci;
    }
}

// LSE merge of the partial slots of every unit covered by more than one
// cluster; grid (128 rows, U units), 128 threads x 4 columns.
__global__ void __launch_bounds__(128)
mla_sm100_merge_kernel(const int4* __restrict__ unit_meta, const float* __restrict__ part_o,
                       const float* __restrict__ part_lse, uint16_t* __restrict__ out_latent,
                       float* __restrict__ out_lse, int n_h, int n_hb) {
    griddep_launch_dependents();
    griddep_wait();
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

// The pool viewed as [chunk (9)][row][64 columns]: one box loads several
// 64-column chunks of the same rows into consecutive 8 KB blocks.
bool make_map_chunks(CUtensorMap* m, const void* base, uint64_t rows) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[3] = {64, rows, 9};
    const cuuint64_t strides[2] = {kRow * 2, 128};
    const cuuint32_t box[3] = {64, 64, 4};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t r256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Sm100Ws {
    size_t prefix, meta, cinfo, part_lse, part_o, total;
};

Sm100Ws sm100_ws(int U) {
    Sm100Ws w;
    w.prefix = 0;
    w.meta = w.prefix + r256(static_cast<size_t>(U + 1) * 4);
    w.cinfo = w.meta + r256(static_cast<size_t>(U) * 16);
    w.part_lse = w.cinfo + r256(static_cast<size_t>(kClusters) * 16);
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
    if (!make_map_2d(&k.tm_pool, P.pool, kRow, pool_rows, kRow * 2, 64, 64) ||
        !make_map_chunks(&k.tm_pool_v, P.pool, pool_rows) ||
        !make_map_2d(&k.tm_qa, P.q_abs, kDc, q_rows, kDc * 2, 64, 64) ||
        !make_map_2d(&k.tm_qr, P.q_r, kDr, q_rows, kDr * 2, 64, 64))
        return cudaErrorInvalidValue;
    k.pool = P.pool;
    k.block_table = P.block_table;
    k.prefix = reinterpret_cast<const int32_t*>(base + w.prefix);
    k.unit_meta = reinterpret_cast<const int4*>(base + w.meta);
    k.cluster_info = reinterpret_cast<const int4*>(base + w.cinfo);
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

    cudaError_t e = launch_pdl(mla_sm100_schedule_kernel, dim3(1), dim3(1024), 0, stream, P.seq_lens, P.B, P.T_q,
                               n_hb, P.max_blocks, static_cast<int>(kClusters),
                               reinterpret_cast<int32_t*>(base + w.prefix), reinterpret_cast<int4*>(base + w.meta),
                               reinterpret_cast<int4*>(base + w.cinfo), P.status);
    if (e != cudaSuccess) return e;
    static std::atomic<uint64_t> smem_set{0};
    e = allow_smem_once(mla_decode_sm100_kernel, static_cast<int>(kSmemBytes), smem_set);
    if (e != cudaSuccess) return e;
    e = launch_pdl(mla_decode_sm100_kernel, dim3(2 * kClusters), dim3(kThreads), kSmemBytes, stream, k);
    if (e != cudaSuccess) return e;
    dim3 mgrid(128, U);
    return launch_pdl(mla_sm100_merge_kernel, mgrid, dim3(128), 0, stream, k.unit_meta,
                      static_cast<const float*>(k.part_o), static_cast<const float*>(k.part_lse), P.out_latent,
                      P.out_lse, P.n_h, n_hb);
}

}  // namespace mla
