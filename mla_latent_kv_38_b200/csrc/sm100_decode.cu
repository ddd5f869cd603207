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
//    producer warp and one in-order MMA consumer: 24 KB S entries (one
//    64-column chunk of the CTA's 2 pages and of its 64 query rows; the query
//    is re-read from L2 each tile, which leaves shared memory to the rings) and
//    32 KB V entries (the CTA's 4 latent chunks of one page, one 3-D box).  The
//    loads run at DRAM latency, so the bytes in flight per SM set the rate; a
//    thread's TMA copies run one after another, so every ring slot has its own
//    issuing thread.
//  * Warp roles per CTA: warp 0 S producer, warp 1 tensor-memory allocation
//    and (CTA 0) the S MMAs, warp 2 (CTA 0) the P.V MMAs, warp 3 V producer,
//    warps 4-11 softmax and epilogue (two warps per tensor-memory lane
//    quadrant).  S is double
//    buffered; P is written to shared memory in two key halves, each released
//    as soon as its MMAs complete.  The running max is rescaled lazily (only
//    when it grows by 2^8).
//  * Work: the tiles of all (sequence, token, head block) units are laid end
//    to end and cut into contiguous ranges, one per cluster (persistent, 74
//    clusters on 148 SMs).  Each CTA computes the cut from the sequence
//    lengths itself (a block-wide scan), so no separate scheduling launch
//    precedes the decode unless the unit count is very large.  A bound on the
//    parts per unit moves each cut to the next allowed split point.  A unit
//    covered by one cluster is written directly in bf16; otherwise each
//    cluster writes an fp32 partial and its log-sum-exp, merged by a
//    reduction kernel.
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
// Registers per thread: 168 at launch (65,536 / 384, rounded down to 8); then
// the load / MMA warpgroup gives registers up to the two softmax warpgroups.
constexpr uint32_t kRegsLaunch = 168;
constexpr uint32_t kRegsIssue = 64;
constexpr uint32_t kRegsSoftmax = 216;
static_assert(128 * kRegsIssue + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
constexpr int kClusters = 74;                     // 148 SMs / 2
constexpr int kDc = 512, kDr = 64, kRow = 576;    // row = c^KV || k^R
constexpr int kPage = 64;                         // cache rows per page (TMA box height)
constexpr int kTilePages = 4;                     // a tile = 4 pages = 256 keys (MMA N)
constexpr int kChunks = 9;                        // 64-column chunks of a row (8 latent + 1 RoPE)
constexpr int kSRing = 4;                         // 24 KB entries, S operand stream (query chunk + key chunks)
constexpr int kVRing = 3;                         // 32 KB entries, P.V operand stream
constexpr int kSLaneGroups = 4;                   // S ring slots are issued by this many groups of lanes in turn

constexpr uint32_t kBox = 8192;                   // one page x 64 columns (128 B rows)
constexpr uint32_t kSEntry = 3 * kBox;            // chunk c of the CTA's 2 pages (keys) and of its 64 query rows
constexpr uint32_t kVEntry = 4 * kBox;            // the CTA's 4 latent chunks of one page
constexpr uint32_t kPBytes = 4 * kBox;            // 64 heads x 256 keys (4 blocks of 64 keys)
constexpr uint32_t kOffSRing = 0;
constexpr uint32_t kOffVRing = kOffSRing + kSRing * kSEntry;
constexpr uint32_t kOffP = kOffVRing + kVRing * kVEntry;
constexpr uint32_t kOffXmax = kOffP + kPBytes;    // 4 x 64 floats: partial row maxima (or sums)
constexpr uint32_t kOffBar = kOffXmax + 1024;
constexpr uint32_t kMaxBars = 40;
constexpr uint32_t kOffMisc = kOffBar + 8 * kMaxBars;   // tmem base, abort flag
constexpr uint32_t kOffCuts = kOffMisc + 64;      // cluster boundaries (75 ints)
constexpr uint32_t kOffSlice = kOffCuts + 320;    // key counts of the cluster's units
// Dynamic shared memory: the buffers above from a 1024-byte aligned base.
constexpr uint32_t kSmemBytes = 232448;
constexpr int kSliceCap = static_cast<int>((kSmemBytes - 1024 - kOffSlice) / 4);
// Units up to which every CTA computes the schedule itself (the scan's scratch
// is the ring area).  The key counts of the cluster's units go to shared
// memory when they fit, else to the CTA's own region of the workspace.
constexpr int kInKernelUnits = 2048;
static_assert(kOffSlice + 1024 <= kSmemBytes, "shared memory budget");
static_assert(4 * (5 * kInKernelUnits + 3 + kClusters + 1 + 48) <= static_cast<int>(kOffP - kOffSRing), "schedule scratch");
static_assert(4 * (kClusters + 1) <= 320, "cut area");
static_assert(kSRing % kSLaneGroups == 0, "each lane group keeps its own ring slots");
static_assert(4 * kSLaneGroups <= 32, "lane groups of the S producer warp");
static_assert(8 * 16384 <= kOffP, "the last epilogue's staging (16 KB per softmax warp) lies in the rings");

enum {
    BAR_SR_FULL = 0,                         // + slot (leader: both CTAs' bytes)
    BAR_SR_EMPTY = BAR_SR_FULL + kSRing,     // + slot (each CTA, MMA commit)
    BAR_VR_FULL = BAR_SR_EMPTY + kSRing,
    BAR_VR_EMPTY = BAR_VR_FULL + kVRing,
    BAR_S_FULL = BAR_VR_EMPTY + kVRing,      // + S buffer
    BAR_S_FREE = BAR_S_FULL + 2,             // + S buffer (leader, 8 warps x 2 CTAs)
    BAR_P_FULL = BAR_S_FREE + 2,             // + P half (leader, 4 warps x 2 CTAs)
    BAR_P_FREE = BAR_P_FULL + 2,             // + P half (each CTA, MMA commit)
    BAR_TAIL_READY = BAR_P_FREE + 2,         // each CTA, MMA thread arrives remotely
    BAR_TAIL_DONE = BAR_TAIL_READY + 1,      // leader, 8 warps x 2 CTAs
    BAR_DRAIN = BAR_TAIL_DONE + 1,           // S issuer's own drain on abort
    BAR_DRAIN_PV = BAR_DRAIN + 1,            // P.V issuer's
    NUM_BARS = BAR_DRAIN_PV + 1
};
static_assert(NUM_BARS <= static_cast<int>(kMaxBars), "barrier area");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;                    // 2 x 128 columns (paired layout)
constexpr uint32_t kTmemS = 256;                  // 2 x 128 columns

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 256, 0, 0);
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, 256, 0, 1);

constexpr uint32_t kSuspendHintNs = 100000;      // a waiting thread sleeps up to 0.1 ms per try
constexpr float kRescaleThreshold = 8.0f;         // log2 units

struct Sm100Params {
    CUtensorMap tm_pool;      // pool as [rows][576], box 64 cols x 64 rows
    CUtensorMap tm_pool_v;    // pool as [chunk][rows][64], box 64 cols x 64 rows x 4 chunks
    CUtensorMap tm_qa;        // q_abs as [n_tok*n_h][512], box 64 x 64
    CUtensorMap tm_qr;        // q_r   as [n_tok*n_h][64],  box 64 x 64
    CUtensorMap tm_out;       // out_latent as [n_tok*n_h][512] bf16, box 64 x 32 (stores)
    CUtensorMap tm_part;      // part_o as [(C+U)*128][512] fp32, box 32 x 32 (stores)
    const int32_t* block_table;
    const int32_t* seq_lens;
    int32_t* prefix;          // (U + 1) exclusive prefix of pages per unit (schedule kernel only)
    int32_t* unit_kv;         // (U) keys per unit (schedule kernel only)
    int32_t* kv_cta;          // (148 x U) per-CTA key counts when the slice exceeds shared memory
    int4* unit_meta;          // (U) {kv_len, first cluster, parts, sequence}
    const int4* cluster_info; // (C) {first page, end page, first unit, last unit} (schedule kernel only)
    uint16_t* out_latent;
    float* out_lse;
    float* part_o;            // (C + U) slots x 128 rows x 512
    float* part_lse;          // (C + U) slots x 128
    int32_t* status;
    int n_h, n_hb, B, T_q, U, num_blocks, max_blocks, max_splits;
    int in_kernel_schedule;   // 1: each CTA computes the schedule; 0: the schedule kernel did
    int withhold_load;        // test hook: 1 = never issue the first S entry's load of CTA 0
    uint64_t timeout_ns;      // bound of every wait
    float scale_log2;
};

__device__ __forceinline__ bool wait_bar(uint32_t addr, uint32_t parity, volatile int* abort_flag,
                                         int32_t* status, uint64_t timeout_ns) {
    if (ptx::mbar_try_wait(addr, parity)) return true;
    const uint64_t t0 = ptx::global_timer_ns();
    while (true) {
        if (ptx::mbar_try_wait_suspend(addr, parity, kSuspendHintNs)) return true;
        if (*abort_flag) return false;
        if (ptx::global_timer_ns() - t0 > timeout_ns) {
            *abort_flag = 1;
            raise_status(status, MLA_STATUS_TIMEOUT);
            return false;
        }
    }
}

// ---------------------------------------------------------------------------
// Work schedule.  Units are numbered token-major: u = (t B + b) n_hb + hb
// for query token t of sequence b and head block hb, so that the T_q units
// of one sequence lie a quarter (for T_q = 4) of the work apart and run on
// different clusters at the same time, at the same relative position in the
// cache: their page reads meet in L2 instead of streaming the cache from
// HBM T_q times.  Unit u covers the keys 0 .. kv - 1 of query row (b, t),
// kv = L_b - T_q + t + 1, i.e. ceil(kv / 64) pages; a sequence whose length
// is out of range has no pages (its outputs are defined as zero / -inf by
// the merge kernel).  pf is the exclusive prefix of the page counts, T =
// pf[U] the total.
// ---------------------------------------------------------------------------

struct UnitIdx {
    int b, t, hb;
};

__device__ __forceinline__ UnitIdx unit_index(int u, int n_hb, int B) {
    const int r = u / n_hb;
    const int t = r / B;
    return UnitIdx{r - t * B, t, u - r * n_hb};
}

__device__ __forceinline__ int unit_keys(const int32_t* seq_lens, int u, int n_hb, int B, int T_q, int max_blocks) {
    const UnitIdx x = unit_index(u, n_hb, B);
    const int L = seq_lens[x.b];   // global or shared memory
    return (L >= T_q && L <= max_blocks * kPage) ? L - T_q + x.t + 1 : 0;
}

// Last unit v with pf[v] <= g (for g < T: the unit holding page g).
__device__ __forceinline__ int unit_of_page(const int32_t* pf, int U, int g) {
    int lo = 0, hi = U - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pf[mid] <= g) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Work is cut at whole tiles (4 pages, 256 keys, counted from each unit's
// start), so that a range that crosses a unit boundary carries no extra
// partial tile.  The cut balances a cost per cluster: 4 per tile (quarter
// tiles) plus kSegCost for every unit segment it starts, which stands for
// the epilogue and pipeline restart of a segment (measured at about 1.5
// tiles).  wf is the exclusive prefix of the units' costs, W = wf[U]; raw cut
// c lies at cost floor(c W / C), rounded to the nearest tile of the unit it
// falls in.  With max_splits = s > 0 it then moves up to the next allowed
// cut, where unit u's P tiles are cut into k = min(s, P) pieces at
// tf[u] + floor(j P / k), j = 0 .. k, so no unit lies in more than s ranges.
constexpr int kSegCost = 6;

__device__ __forceinline__ int unit_cost(int tiles) { return 4 * tiles + (tiles > 0 ? kSegCost : 0); }

__device__ int raw_cut_tile(int c, int Tt, const int32_t* tf, const int32_t* wf, int U, int max_splits) {
    if (c <= 0) return 0;
    if (c >= kClusters) return Tt;
    const int W = wf[U];
    const int x = static_cast<int>(static_cast<long long>(c) * W / kClusters);
    if (x >= W) return Tt;
    int u = unit_of_page(wf, U, x);           // wf[u] <= x < wf[u + 1]
    const int tiles = tf[u + 1] - tf[u];
    const int d = x - wf[u] - kSegCost;
    const int g = tf[u] + (d <= 0 ? 0 : min(tiles, (d + 2) / 4));
    if (max_splits <= 0 || g >= Tt) return g;
    u = unit_of_page(tf, U, g);
    const int a = tf[u], P = tf[u + 1] - a;   // a <= g < tf[u + 1], so P > 0
    const int k = min(max_splits, P);
    const int j = static_cast<int>((static_cast<long long>(g - a) * k + P - 1) / P);   // ceil((g-a) k / P)
    return a + static_cast<int>(static_cast<long long>(j) * P / k);
}

// First page of global tile gt (T pages, Tt tiles in all).
__device__ int tile_to_page(int gt, int Tt, int T, const int32_t* tf, const int32_t* pf, int U) {
    if (gt >= Tt) return T;
    const int u = unit_of_page(tf, U, gt);    // tf[u] <= gt < tf[u + 1]
    return pf[u] + kTilePages * (gt - tf[u]);
}

// Cluster boundaries cuts[0 .. C] in pages: the distinct raw cuts in order,
// then T repeated, so cluster c covers pages [cuts[c], cuts[c + 1]) and every
// non-empty range comes before every empty one (a unit's ranges are always
// consecutive clusters).  All threads of the block call it; tmp holds C + 1
// ints of scratch.
__device__ void compute_cuts(int* cuts, int* tmp, const int32_t* pf, const int32_t* tf, const int32_t* wf, int U,
                             int T, int Tt, int max_splits) {
    for (int c = threadIdx.x; c <= kClusters; c += blockDim.x)
        tmp[c] = tile_to_page(raw_cut_tile(c, Tt, tf, wf, U, max_splits), Tt, T, tf, pf, U);
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        constexpr int kPer = (kClusters + 1 + 31) / 32;
        int n = 0;
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int c = lane * kPer + k;
            if (c <= kClusters && (c == 0 || tmp[c] != tmp[c - 1])) ++n;
        }
        int x = n;   // inclusive warp scan of the distinct counts
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        const int total = __shfl_sync(0xffffffffu, x, 31);
        int pos = x - n;
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int c = lane * kPer + k;
            if (c <= kClusters && (c == 0 || tmp[c] != tmp[c - 1])) cuts[pos++] = tmp[c];
        }
        for (int c = total + lane; c <= kClusters; c += 32) cuts[c] = T;
    }
    __syncthreads();
}

// Cluster whose range holds page g < T (the last cluster starting at or before g).
__device__ int cluster_of_page(int g, const int* cuts) {
    int lo = 0, hi = kClusters - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cuts[mid] <= g) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Merge metadata of unit u: {kv_len, first cluster, parts, sequence}.
__device__ int4 unit_meta_of(int u, const int32_t* pf, const int* cuts, const int32_t* seq_lens, int n_hb, int B,
                             int T_q, int max_blocks) {
    const int kv = unit_keys(seq_lens, u, n_hb, B, T_q, max_blocks);
    const int b = unit_index(u, n_hb, B).b;
    const int a = pf[u], e = pf[u + 1];
    if (e <= a) return make_int4(0, 0, 0, b);
    const int c0 = cluster_of_page(a, cuts);
    const int c1 = cluster_of_page(e - 1, cuts);
    return make_int4(kv, c0, c1 - c0 + 1, b);
}

// One tile of a cluster's work: up to 4 consecutive pages of one unit.
struct Tile {
    int u;          // unit = (t B + b) n_hb + hb
    int bt;         // query row b T_q + t of the unit
    int hb;         // head block of the unit
    int b;          // sequence of the unit
    int kv;         // keys of the unit (kv_len)
    int page0;      // first page, within the unit
    int np;         // pages in this tile (1..4)
    bool first;     // first tile of a unit segment (new query, O starts from zero)
    bool last;      // last tile of a unit segment (epilogue follows)
    bool unit_end;  // the unit's last page is in this tile
    bool whole;     // the whole unit lies in this cluster's range (no partial)
};

// Walks a cluster's pages [g0, g1) as tiles.  kvs[v - off] is the key count
// of unit v (a shared-memory slice of the cluster's units, or a global array
// with off = 0); unit u0 starts at global page ubeg0.  The unit's page range
// and (query row, head block, sequence) are kept up to date incrementally.
struct TileWalker {
    const int32_t* kvs;
    int off, g, g0, g1, u, ubeg, uend, kv;
    int bt, hb, b, t, n_hb, B, T_q;
    __device__ void load_unit() {
        kv = kvs[u - off];
        uend = ubeg + (kv + kPage - 1) / kPage;
    }
    __device__ void step_unit() {
        ++u;
        ubeg = uend;
        load_unit();
        if (++hb == n_hb) {
            hb = 0;
            if (++b == B) {
                b = 0;
                ++t;
            }
            bt = b * T_q + t;
        }
    }
    __device__ void init(const int32_t* kvs_, int off_, int u0, int ubeg0, int g0_, int g1_, int n_hb_, int B_,
                         int T_q_) {
        kvs = kvs_;
        off = off_;
        g = g0_;
        g0 = g0_;
        g1 = g1_;
        n_hb = n_hb_;
        B = B_;
        T_q = T_q_;
        u = u0;
        ubeg = ubeg0;
        const UnitIdx x = unit_index(u0, n_hb, B);
        b = x.b;
        t = x.t;
        hb = x.hb;
        bt = b * T_q + t;
        if (g < g1) {
            load_unit();
            while (g < g1 && uend <= g) step_unit();
        }
    }
    __device__ bool done() const { return g >= g1; }
    __device__ Tile next() {
        Tile r;
        r.u = u;
        r.bt = bt;
        r.hb = hb;
        r.b = b;
        r.kv = kv;
        r.page0 = g - ubeg;
        r.first = (g == g0) || (g == ubeg);
        r.whole = ubeg >= g0 && uend <= g1;
        const int seg_end = min(g1, uend);   // tiles start at the segment start
        r.np = min(kTilePages, seg_end - g);
        r.last = g + r.np == seg_end;
        r.unit_end = g + r.np == uend;
        g += r.np;
        while (g < g1 && uend <= g) step_unit();
        return r;
    }
};

// Block-wide exclusive scans of the units' page counts, tile counts and cut
// costs into pf, tf, wf[0 .. U] (U <= kInKernelUnits); every thread of the
// CTA takes part; warp_tot holds 3 x 16 ints of scratch.  Returns {T, Tt}.
__device__ int2 schedule_scan(int* pf, int* tf, int* wf, int* warp_tot, const int32_t* seq_lens, int U, int n_hb,
                              int B, int T_q, int max_blocks) {
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int per = (U + kThreads - 1) / kThreads;
    const int beg = min(U, tid * per), end = min(U, beg + per);
    int loc[3] = {0, 0, 0};
    for (int u = beg; u < end; ++u) {
        const int pages = (unit_keys(seq_lens, u, n_hb, B, T_q, max_blocks) + kPage - 1) / kPage;
        const int tiles = (pages + kTilePages - 1) / kTilePages;
        pf[u + 1] = pages;
        tf[u + 1] = tiles;
        wf[u + 1] = unit_cost(tiles);
        loc[0] += pages;
        loc[1] += tiles;
        loc[2] += unit_cost(tiles);
    }
    int v[3] = {loc[0], loc[1], loc[2]};   // inclusive warp scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            const int y = __shfl_up_sync(0xffffffffu, v[q], o);
            if (lane >= o) v[q] += y;
        }
    }
    if (lane == 31)
        for (int q = 0; q < 3; ++q) warp_tot[16 * q + w] = v[q];
    __syncthreads();
    if (w == 0) {
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            int x = lane < kThreads / 32 ? warp_tot[16 * q + lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (lane < kThreads / 32) warp_tot[16 * q + lane] = x;   // inclusive over warps
        }
    }
    __syncthreads();
    int r[3];
    for (int q = 0; q < 3; ++q) r[q] = v[q] - loc[q] + (w > 0 ? warp_tot[16 * q + w - 1] : 0);
    for (int u = beg; u < end; ++u) {
        r[0] += pf[u + 1];
        pf[u + 1] = r[0];
        r[1] += tf[u + 1];
        tf[u + 1] = r[1];
        r[2] += wf[u + 1];
        wf[u + 1] = r[2];
    }
    if (tid == 0) pf[0] = tf[0] = wf[0] = 0;
    __syncthreads();
    return make_int2(pf[U], tf[U]);
}

// P.V operand split: CTA r supplies latent chunks 4r .. 4r+3 (columns
// [256r, 256r+256)); instruction h (N = 256) takes chunks 4r+2h, 4r+2h+1 from
// each CTA, so TMEM column 128h + j of lane half r holds latent column
// 256r + 128h + j.  V ring entry (page, h) holds exactly those two chunks.

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
    const uint64_t tmo = p.timeout_ns;

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
    // The sequence lengths and the block table are read first after the wait:
    // bring them into L2 now (a prefetch changes no data, and L2 is coherent
    // with the writes of a kernel still running, so it may precede the wait).
    // Each CTA takes every 148th 128-byte line.
    if (warp >= 4) {
        const char* lens_b = reinterpret_cast<const char*>(p.seq_lens);
        const char* tab_b = reinterpret_cast<const char*>(p.block_table);
        const long n_lens = (static_cast<long>(p.B) * 4 + 127) / 128;
        const long n_tab = (static_cast<long>(p.B) * p.max_blocks * 4 + 127) / 128;
        for (long k = blockIdx.x + static_cast<long>(gridDim.x) * (threadIdx.x - 128); k < n_lens + n_tab;
             k += static_cast<long>(gridDim.x) * (kThreads - 128))
            ptx::prefetch_l2_line(k < n_lens ? lens_b + 128 * k : tab_b + 128 * (k - n_lens));
    }
    // everything below reads what the kernels before this one wrote (q_abs,
    // q^R, the appended cache rows) or what an earlier decode call may still
    // read (the workspace)
    griddep_wait();

    // ---- this cluster's contiguous range of global pages [g0, g1), its first
    // unit u0 (starting at global page ubeg0) and the key counts of its units
    int32_t* kv_s = reinterpret_cast<int32_t*>(smem + kOffSlice);
    int g0 = 0, g1 = 0, u0 = 0, ubeg0 = 0;
    const int32_t* kv_base = kv_s;
    int kv_off = 0;
    if (p.in_kernel_schedule) {
        // scratch: the ring area is unused until the loads start
        int* sc = reinterpret_cast<int*>(smem + kOffSRing);          // page prefix, U + 1
        int* tfx = sc + kInKernelUnits + 1;                           // tile prefix, U + 1
        int* wfx = tfx + kInKernelUnits + 1;                          // cost prefix, U + 1
        int* ctmp = wfx + kInKernelUnits + 1;                         // cut scratch, C + 1
        int* lens = ctmp + kClusters + 1;                             // sequence lengths, B <= U
        int* wtot = lens + kInKernelUnits;                            // scan scratch, 48
        for (int b = threadIdx.x; b < p.B; b += kThreads) lens[b] = __ldg(p.seq_lens + b);
        __syncthreads();
        const int2 TT = schedule_scan(sc, tfx, wfx, wtot, lens, p.U, p.n_hb, p.B, p.T_q, p.max_blocks);
        const int T = TT.x;
        int* cuts = reinterpret_cast<int*>(smem + kOffCuts);
        compute_cuts(cuts, ctmp, sc, tfx, wfx, p.U, T, TT.y, p.max_splits);
        g0 = cuts[cluster];
        g1 = cuts[cluster + 1];
        if (g0 < g1) {
            u0 = unit_of_page(sc, p.U, g0);
            ubeg0 = sc[u0];
            const int u1 = unit_of_page(sc, p.U, g1 - 1);
            int32_t* dst = kv_s;
            if (u1 - u0 + 1 > kSliceCap) {   // only this CTA reads its region
                dst = p.kv_cta + static_cast<size_t>(blockIdx.x) * p.U;
                kv_base = dst;
            }
            for (int k = threadIdx.x; k <= u1 - u0; k += kThreads)
                dst[k] = unit_keys(lens, u0 + k, p.n_hb, p.B, p.T_q, p.max_blocks);
        }
        kv_off = u0;
        // merge metadata and length checks, spread over the grid's threads
        for (int u = blockIdx.x * kThreads + threadIdx.x; u < p.U; u += gridDim.x * kThreads) {
            const int4 m = unit_meta_of(u, sc, cuts, lens, p.n_hb, p.B, p.T_q, p.max_blocks);
            p.unit_meta[u] = m;
            if (m.x == 0 && u < p.B * p.n_hb && u % p.n_hb == 0) raise_status(p.status, MLA_STATUS_BAD_SEQ_LEN);
        }
    } else {
        const int4 cinfo = p.cluster_info[cluster];
        g0 = cinfo.x;
        g1 = cinfo.y;
        u0 = cinfo.z;
        const int n_units = cinfo.w - u0 + 1;   // units u0 .. cinfo.w
        if (g0 < g1) {
            ubeg0 = p.prefix[u0];
            if (n_units <= kSliceCap) {
                for (int k = threadIdx.x; k < n_units; k += kThreads) kv_s[k] = p.unit_kv[u0 + k];
                kv_off = u0;
            } else {
                kv_base = p.unit_kv;
                kv_off = 0;
            }
        }
    }
    ptx::fence_proxy_async_smem();   // the scan's reads of the ring area precede the loads into it
    __syncthreads();   // slice written; the scan scratch is free for the rings

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
    auto walker = [&](TileWalker& w) { w.init(kv_base, kv_off, u0, ubeg0, g0, g1, p.n_hb, p.B, p.T_q); };

    if (warp < 4) {
        // Warpgroup 0 (loads and MMA issue) needs few registers: it gives them to
        // the softmax warpgroups (setmaxnreg, per warpgroup, at the top of each
        // branch so that the compiler budgets each branch on its own).
        ptx::regs_dec<kRegsIssue>();
        if (warp == 0) {
            // ------------------------------------------------------------ S stream
            // Entry c of a tile holds column chunk c (64 columns) of this CTA's two
            // pages (keys) and of its 64 query rows, one 8 KB box each; the query is
            // re-read from L2 with every tile, which leaves the shared memory to
            // the rings (the loads run at DRAM latency, so the bytes in flight set
            // the rate).  A thread's TMA copies run one after another, so ring slot
            // s is issued by its own group of lanes 4g + {0, 1, 2}, g = s mod
            // kSLaneGroups: lane j = 0, 1 loads own page j, lane 2 the query chunk.
            // The group's lane 0 in the leader CTA arms the full barrier with both
            // CTAs' bytes.  The page lanes hold the block of their page for tiles
            // i, i+1, i+2 in b0, b1, b2.
            const int grp = lane >> 2, j = lane & 3;
            const bool active = grp < kSLaneGroups && j < 3;
            const int my_pg = 2 * static_cast<int>(rank) + (j & 1);
            TileWalker w, wa;
            walker(w);
            walker(wa);
            int b0 = 0, b1 = 0, b2 = 0;
            bool h0 = false, h1 = false, h2 = false;
            // (the loads are unconditional, to a valid entry, so that nothing waits
            // for them until their value is used a tile or two later)
            auto look = [&](int& b, bool& h) {
                h = false;
                if (!wa.done()) {
                    const Tile t = wa.next();
                    h = active && j < 2 && my_pg < t.np;
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
                const uint32_t tx = static_cast<uint32_t>(cur.np + 2) * kBox;    // both CTAs' page and query chunks
                for (int c = 0; c < kChunks; ++c, ++e) {
                    const int slot = e % kSRing;
                    bool good = true;
                    if (active && grp == slot % kSLaneGroups) {
                        good = wait_bar(bar(BAR_SR_EMPTY + slot), ((e / kSRing) & 1) ^ 1, abort_flag, p.status, tmo);
                        if (good && j == 0 && rank == 0) ptx::mbar_arrive_expect_tx(bar(BAR_SR_FULL + slot), tx);
                        const bool q_lane = j == 2;
                        const bool withheld = p.withhold_load && rank == 0 && e == 0 && j == 0;
                        if (good && (q_lane || h0) && !withheld) {
                            const void* tm = q_lane ? (c < 8 ? static_cast<const void*>(&p.tm_qa) : &p.tm_qr) : &p.tm_pool;
                            const int bx = q_lane ? (c < 8 ? 64 * c : 0) : 64 * c;
                            ptx::tma_load_2d_pair_normal(sbase + kOffSRing + slot * kSEntry + j * kBox, tm, bx,
                                                         q_lane ? qrow : row, leader_bar(BAR_SR_FULL + slot));
                        }
                    }
                    if (!__all_sync(0xffffffffu, good)) { ok = false; break; }
                }
                b0 = b1; h0 = h1;
                b1 = b2; h1 = h2;
                look(b2, h2);
            }
        } else if (warp == 3) {
            // ------------------------------------------------------------ V stream
            // Entry per page: this CTA's latent chunks 4r .. 4r+3 of the page, one
            // 3-D box, issued by lane (slot) so that consecutive copies come from
            // different threads.  Lane pg < 4 holds the block of page pg of the
            // current tile (v0) and of the next one (v1).
            const uint64_t pol_v = ptx::l2_policy_evict_first();   // last use of these lines
            TileWalker w, wa;
            walker(w);
            walker(wa);
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
                    if (lane == slot) {
                        good = wait_bar(bar(BAR_VR_EMPTY + slot), ((e / kVRing) & 1) ^ 1, abort_flag, p.status, tmo);
                        if (good && rank == 0) ptx::mbar_arrive_expect_tx(bar(BAR_VR_FULL + slot), 2 * kVEntry);
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
                walker(w);
                int i = 0;
                bool ok = true;
                while (ok && !w.done()) {
                    w.next();
                    const int e0 = kChunks * i;
                    const int sb = i & 1;
                    if (!(ok = wait_bar(bar(BAR_S_FREE + sb), ((i >> 1) & 1) ^ 1, abort_flag, p.status, tmo))) break;
                    ptx::tc_fence_after();   // the softmax's reads of this S buffer are done
                    for (int c = 0; c < kChunks; ++c) {
                        const int e = e0 + c;
                        if (!(ok = wait_bar(bar(BAR_SR_FULL + e % kSRing), (e / kSRing) & 1, abort_flag, p.status, tmo)))
                            break;
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
                    while (!ptx::mbar_try_wait(bar(BAR_DRAIN), 0) && ptx::global_timer_ns() - t0 < tmo) {
                    }
                }
            }
        } else if (warp == 2) {
            if (rank == 0) {
                // -------------------------------------------------------- O += P V issuer
                // V(i) occupies the next np entries of the V ring (one per page).
                if (lane == 0 && g0 < g1) {
                    TileWalker w;
                    walker(w);
                    int i = 0, tails = 0, e = 0;
                    bool ok = true;
                    const uint64_t a0 = ptx::smem_desc_sw128(sbase + kOffP, 16, 1024);
                    while (ok && !w.done()) {
                        const Tile t = w.next();
                        const bool tail = t.unit_end && (t.kv % kPage) != 0;
                        // P is written in two halves: keys [0,128) (pages 0, 1) by the
                        // softmax warps of TMEM lanes 0-63, keys [128,256) by those of
                        // lanes 64-127; each half is released as soon as its pages'
                        // MMAs complete.
                        for (int pg = 0; pg < 4 && ok; ++pg) {
                            if (pg == 0 || pg == 2) {
                                if (pg == 2) ptx::mma_commit_pair(bar(BAR_P_FREE + 0), 0x3);
                                if (!(ok = wait_bar(bar(BAR_P_FULL + (pg >> 1)), i & 1, abort_flag, p.status, tmo))) break;
                                ptx::tc_fence_after();
                            }
                            if (pg >= t.np) continue;
                            if (tail && pg == t.np - 1) {
                                // the unit's last page holds rows past the end: once its V
                                // entry has landed, the softmax warps of both CTAs zero those
                                // rows (entries are consumed in ring order, so the earlier
                                // pages' slots are already free for this load)
                                if (!(ok = wait_bar(bar(BAR_VR_FULL + e % kVRing), (e / kVRing) & 1, abort_flag,
                                                    p.status, tmo)))
                                    break;
                                ptx::mbar_arrive_cluster(ptx::map_to_rank(bar(BAR_TAIL_READY), 0));
                                ptx::mbar_arrive_cluster(ptx::map_to_rank(bar(BAR_TAIL_READY), 1));
                                if (!(ok = wait_bar(bar(BAR_TAIL_DONE), tails & 1, abort_flag, p.status, tmo))) break;
                                ++tails;
                            }
                            if (!(ok = wait_bar(bar(BAR_VR_FULL + e % kVRing), (e / kVRing) & 1, abort_flag, p.status, tmo)))
                                break;
                            for (int h = 0; h < 2; ++h) {
                                const uint64_t b0 = ptx::smem_desc_sw128(
                                    sbase + kOffVRing + (e % kVRing) * kVEntry + h * 2 * kBox, kBox, 1024);
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
                        while (!ptx::mbar_try_wait(bar(BAR_DRAIN_PV), 0) && ptx::global_timer_ns() - t0 < tmo) {
                        }
                    }
                }
            }
        }
    } else {
        ptx::regs_inc<kRegsSoftmax>();
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
        TileWalker w;
        walker(w);
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
            // keys of this tile that belong to this segment
            const int key_end = min(t.kv, kPage * (t.page0 + t.np));
            if (t.first) {
                m_used = -INFINITY;
                l_part = 0.f;
            }
            const int sb = i & 1;
            ok = wait_bar(bar(BAR_S_FULL + sb), (i >> 1) & 1, abort_flag, p.status, tmo);
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

            // The weights of row m, keys key0 + [0, 64): computed into registers
            // first, which ends this thread's reads of the S buffer.
            float ps2[2] = {0.f, 0.f};
            const float neg_m = -m_used;
            uint32_t pk[32];
            {
                uint32_t r[2][32];
                ptx::tmem_ld32(s_col, r[0]);
                ptx::tmem_ld32(s_col + 32, r[1]);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 64; j += 2) {
                    const float s0 = __uint_as_float(r[j >> 5][j & 31]), s1 = __uint_as_float(r[j >> 5][(j & 31) + 1]);
                    const float p0 = j < nvalid ? ex2(fmaf(s0, p.scale_log2, neg_m)) : 0.f;
                    const float p1 = j + 1 < nvalid ? ex2(fmaf(s1, p.scale_log2, neg_m)) : 0.f;
                    ps2[(j >> 1) & 1] += p0 + p1;
                    pk[j >> 1] = pack_bf16x2(p0, p1);
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster_relaxed(leader_bar(BAR_S_FREE + sb));
            const float ps = ps2[0] + ps2[1];
            l_part = l_part * alpha + ps;

            // This half of the P buffer must be free (the previous tile's P.V MMAs on
            // it complete); a rescale of O needs the whole previous P.V complete.
            const int hf = hi ? 1 : 0;
            ok = wait_bar(bar(BAR_P_FREE + hf), (i & 1) ^ 1, abort_flag, p.status, tmo);
            if (ok && !hi && __any_sync(0xffffffffu, resc))
                ok = wait_bar(bar(BAR_P_FREE + 1), (i & 1) ^ 1, abort_flag, p.status, tmo);
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
            {
                unsigned char* Pb = smem + kOffP + (2 * hf + cg) * kBox + m * 128;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4*>(Pb + ((ch ^ (m & 7)) * 16)) =
                        make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(leader_bar(BAR_P_FULL + hf));

            // V ring position of this tile's entries (one per page)
            const int v_start = v_before;
            v_before += t.np;
            if (t.unit_end && (t.kv % kPage) != 0) {
                // zero rows past the end in this CTA's V entry of the last page
                // (4 chunks of 64 rows x 128 B)
                ok = wait_bar(bar(BAR_TAIL_READY), tails & 1, abort_flag, p.status, tmo);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                ++tails;
                const int valid = t.kv - kPage * (t.page0 + t.np - 1);
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
                ok = wait_bar(bar(BAR_P_FREE + 1), i & 1, abort_flag, p.status, tmo);
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
                const bool whole = t.whole;
                const size_t grow = static_cast<size_t>(bt) * p.n_h + hb * 128 + head_in_unit;
                const size_t slot = static_cast<size_t>(cluster) + t.u;
                // This warp's 32 rows (consecutive heads) x the thread's 128
                // latent columns go out through 4 KB tiles written in the
                // 128-byte swizzled layout of a TMA store box (a thread's row of
                // 128 bytes, 16-byte chunk k at k ^ (row & 7)), each tile one
                // bulk tensor store: 4 stores of 32 fp32 columns for a partial,
                // 2 of 64 bf16 columns otherwise.  Between tiles the staging is
                // one 4 KB tile of the free P buffer per warp, reused store
                // after store; after the CTA's last tile no load or MMA touches
                // the rings any more, so every store gets its own tile there
                // and none waits for the one before.
                const bool final_tile = w.done();
                const int h = cg;   // this thread's 128 O columns
                const int col0 = 128 * h + (hi ? 256 : 0);
                const uint32_t stage_off = final_tile ? kOffSRing + sw * 16384u : kOffP + sw * 4096u;
                unsigned char* stage = smem + stage_off;
                const uint32_t stage_u = sbase + stage_off;
                const int x7 = lane & 7;
                const int row0 = whole ? static_cast<int>(grow - lane)
                                       : static_cast<int>(slot * 128 + head_in_unit - lane);
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    uint32_t o[32];
                    ptx::tmem_ld32(t_lane + kTmemO + 128 * h + 32 * q, o);
                    ptx::tmem_wait_ld();
                    const int tile_k = whole ? (q >> 1) : q;   // this round's store
                    const uint32_t tile_off = final_tile ? 4096u * tile_k : 0u;
                    unsigned char* my_row = stage + tile_off + lane * 128;
                    if (!final_tile && (!whole || (q & 1) == 0)) {
                        if (lane == 0) ptx::bulk_wait_read_all();   // the previous store has read the tile
                        __syncwarp();
                    }
                    if (whole) {
                        // columns 32q .. 32q + 31 are chunks 4 (q & 1) .. + 3 of the staged 64-column row
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            uint4 wv;
                            wv.x = pack_bf16x2(__uint_as_float(o[8 * k + 0]) * inv, __uint_as_float(o[8 * k + 1]) * inv);
                            wv.y = pack_bf16x2(__uint_as_float(o[8 * k + 2]) * inv, __uint_as_float(o[8 * k + 3]) * inv);
                            wv.z = pack_bf16x2(__uint_as_float(o[8 * k + 4]) * inv, __uint_as_float(o[8 * k + 5]) * inv);
                            wv.w = pack_bf16x2(__uint_as_float(o[8 * k + 6]) * inv, __uint_as_float(o[8 * k + 7]) * inv);
                            *reinterpret_cast<uint4*>(my_row + (((4 * (q & 1) + k) ^ x7) * 16)) = wv;
                        }
                        if (q & 1) {
                            ptx::fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                ptx::tma_store_2d(&p.tm_out, stage_u + tile_off, col0 + 64 * (q >> 1), row0);
                                ptx::bulk_commit_group();
                            }
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            *reinterpret_cast<float4*>(my_row + ((k ^ x7) * 16)) =
                                make_float4(__uint_as_float(o[4 * k]) * inv, __uint_as_float(o[4 * k + 1]) * inv,
                                            __uint_as_float(o[4 * k + 2]) * inv, __uint_as_float(o[4 * k + 3]) * inv);
                        ptx::fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            ptx::tma_store_2d(&p.tm_part, stage_u + tile_off, col0 + 32 * q, row0);
                            ptx::bulk_commit_group();
                        }
                    }
                }
                if (!final_tile) {
                    if (lane == 0) ptx::bulk_wait_read_all();   // the P buffer is written again by the next tile
                    __syncwarp();
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
    if (warp >= 4 && lane == 0) ptx::bulk_wait_all();   // the epilogue's stores have completed
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
    // The merge kernel may start only now: launched while this grid still
    // runs, its pending blocks slowed the decode down measurably.
    griddep_launch_dependents();
}

// ---------------------------------------------------------------------------
// Work schedule for very large unit counts (U > kInKernelUnits): the exclusive
// prefixes of pages, tiles and cut costs per unit, the units' key counts, the
// merge metadata and each cluster's page range, computed by one block of 1024
// threads with the same cut rule as the decode kernel's own scan.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
mla_sm100_schedule_kernel(const int32_t* __restrict__ seq_lens, int B, int T_q, int n_hb, int max_blocks,
                          int max_splits, int U, int32_t* __restrict__ prefix, int32_t* __restrict__ tprefix,
                          int32_t* __restrict__ wprefix, int32_t* __restrict__ kv_out, int4* __restrict__ unit_meta,
                          int4* __restrict__ cluster_info, int32_t* status) {
    __shared__ int warp_tot[3][32];
    __shared__ int carry[3];
    griddep_launch_dependents();
    griddep_wait();   // the workspace may still be read by an earlier decode call's kernels
    if (threadIdx.x == 0) carry[0] = carry[1] = carry[2] = 0;
    __syncthreads();
    int32_t* out[3] = {prefix, tprefix, wprefix};
    for (int base = 0; base < U; base += 1024) {
        const int u = base + threadIdx.x;
        int v[3] = {0, 0, 0};   // pages, tiles, cost
        if (u < U) {
            const int kv = unit_keys(seq_lens, u, n_hb, B, T_q, max_blocks);
            kv_out[u] = kv;
            v[0] = (kv + kPage - 1) / kPage;
            v[1] = (v[0] + kTilePages - 1) / kTilePages;
            v[2] = unit_cost(v[1]);
        }
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
        for (int q = 0; q < 3; ++q) {   // block inclusive scans
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, v[q], o);
                if (lane >= o) v[q] += y;
            }
            if (lane == 31) warp_tot[q][w] = v[q];
        }
        __syncthreads();
        if (w == 0) {
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                int t = warp_tot[q][lane];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, t, o);
                    if (lane >= o) t += y;
                }
                warp_tot[q][lane] = t;
            }
        }
        __syncthreads();
        int incl[3];
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            incl[q] = v[q] + (w > 0 ? warp_tot[q][w - 1] : 0) + carry[q];
            if (u < U) out[q][u + 1] = incl[q];
            if (u == 0) out[q][0] = 0;
        }
        __syncthreads();
        if (threadIdx.x == 1023)
            for (int q = 0; q < 3; ++q) carry[q] = incl[q];
        __syncthreads();
    }
    const int T = carry[0], Tt = carry[1];
    __shared__ int cuts[kClusters + 1], cut_tmp[kClusters + 1];
    compute_cuts(cuts, cut_tmp, prefix, tprefix, wprefix, U, T, Tt, max_splits);
    for (int u = threadIdx.x; u < U; u += 1024) {
        const int4 m = unit_meta_of(u, prefix, cuts, seq_lens, n_hb, B, T_q, max_blocks);
        unit_meta[u] = m;
        if (m.x == 0 && u < B * n_hb && u % n_hb == 0) raise_status(status, MLA_STATUS_BAD_SEQ_LEN);
    }
    for (int c = threadIdx.x; c < kClusters; c += 1024) {
        const int a = cuts[c], e = cuts[c + 1];
        cluster_info[c] = a < e ? make_int4(a, e, unit_of_page(prefix, U, a), unit_of_page(prefix, U, e - 1))
                                : make_int4(0, 0, 0, 0);
    }
}

// LSE merge of the partial slots of every unit covered by more than one
// cluster: one warp per (unit, head row), a lane per 16 latent columns.  The
// slots of unit u are meta.y + u .. meta.y + u + meta.z - 1.  Units of an
// invalid sequence (kv_len 0) get zeros and lse = -inf.
//
// The partial rows were written by the decode kernel just before and are read
// from L2 (ld.global.cg).  The first two slots' rows are fetched together with
// the log-sum-exps, so that a row split in two takes two dependent round trips
// (metadata, then everything else); further slots follow two at a time.
// Blocks of 8 warps, at most 64 registers a thread: 4 blocks per SM, one wave
// for the 4,096 rows of 32 split units.  (Blocks of 4 warps doubled the merge
// at prefill sizes, where most of the U x 128 rows belong to whole units and
// the time goes into scheduling blocks that exit at once.)
__global__ void __launch_bounds__(256, 4)
mla_sm100_merge_kernel(const int4* __restrict__ unit_meta, const float* __restrict__ part_o,
                       const float* __restrict__ part_lse, uint16_t* __restrict__ out_latent,
                       float* __restrict__ out_lse, int n_h, int n_hb, int B, int T_q, int U) {
    griddep_launch_dependents();
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int wg = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int u = wg >> 7, row = wg & 127;
    if (u >= U) return;
    const int4 meta = unit_meta[u];
    auto out_row = [&]() {   // this warp's output row
        const UnitIdx x = unit_index(u, n_hb, B);
        return static_cast<size_t>(x.b * T_q + x.t) * n_h + x.hb * 128 + row;
    };
    if (meta.x == 0) {
        const size_t grow = out_row();
        uint4* dst = reinterpret_cast<uint4*>(out_latent + grow * kDc + lane * 16);
        dst[0] = make_uint4(0, 0, 0, 0);
        dst[1] = make_uint4(0, 0, 0, 0);
        if (lane == 0) out_lse[grow] = -INFINITY;
        return;
    }
    const int parts = meta.z;   // <= kClusters
    if (parts <= 1) return;
    const size_t slot0 = static_cast<size_t>(meta.y) + u;
    const float* lse_row = part_lse + slot0 * 128 + row;                                       // slot i at + 128 i
    const float4* o_row = reinterpret_cast<const float4*>(part_o + (slot0 * 128 + row) * kDc) + lane * 4;
    constexpr size_t kSlot4 = static_cast<size_t>(128) * kDc / 4;                             // float4 per slot
    auto load_pair = [&](float4 (&v)[2][4], int i) {   // slots i, i + 1 (zeros past the last)
#pragma unroll
        for (int k = 0; k < 4; ++k) v[0][k] = __ldcg(o_row + i * kSlot4 + k);
#pragma unroll
        for (int k = 0; k < 4; ++k)
            v[1][k] = i + 1 < parts ? __ldcg(o_row + (i + 1) * kSlot4 + k) : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    float4 v[2][4];
    load_pair(v, 0);
    // log-sum-exp of slot lane + 32 k in ls[k] (parts <= 74 < 96)
    float ls[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) ls[k] = lane + 32 * k < parts ? __ldcg(lse_row + 128 * (lane + 32 * k)) : -INFINITY;
    const float mx = warp_max(fmaxf(fmaxf(ls[0], ls[1]), ls[2]));
    auto w_of = [&](float l) { return l == -INFINITY ? 0.f : ex2((l - mx) * kLog2e); };
    const float z = warp_sum(w_of(ls[0]) + w_of(ls[1]) + w_of(ls[2]));
    auto weight = [&](int i) {   // slot i's weight, from the lane that holds its log-sum-exp
        const float l = i < 32 ? ls[0] : (i < 64 ? ls[1] : ls[2]);
        return w_of(__shfl_sync(0xffffffffu, l, i & 31));
    };
    float acc[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = 0.f;
    for (int i = 0; i < parts; i += 2) {
        if (i > 0) load_pair(v, i);
        const float w0 = weight(i), w1 = i + 1 < parts ? weight(i + 1) : 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            acc[4 * k + 0] = fmaf(w1, v[1][k].x, fmaf(w0, v[0][k].x, acc[4 * k + 0]));
            acc[4 * k + 1] = fmaf(w1, v[1][k].y, fmaf(w0, v[0][k].y, acc[4 * k + 1]));
            acc[4 * k + 2] = fmaf(w1, v[1][k].z, fmaf(w0, v[0][k].z, acc[4 * k + 2]));
            acc[4 * k + 3] = fmaf(w1, v[1][k].w, fmaf(w0, v[0][k].w, acc[4 * k + 3]));
        }
    }
    const float inv = z > 0.f ? 1.f / z : 0.f;
    uint32_t pk[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) pk[k] = pack_bf16x2(acc[2 * k] * inv, acc[2 * k + 1] * inv);
    const size_t grow = out_row();
    uint4* dst = reinterpret_cast<uint4*>(out_latent + grow * kDc + lane * 16);
    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    if (lane == 0) out_lse[grow] = z > 0.f ? mx + logf(z) : -INFINITY;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

// The pool viewed as [chunk (9)][row][64 columns]: one box loads four 64-column
// chunks of the same 64 rows into consecutive 8 KB blocks.
bool make_map_chunks(CUtensorMap* m, const void* base, uint64_t rows) {
    const cuuint64_t dims[3] = {64, rows, kChunks};
    const cuuint64_t strides[2] = {kRow * 2, 128};
    const cuuint32_t box[3] = {64, 64, 4};
    return encode_tiled_cached(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B);
}

size_t r256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Sm100Ws {
    size_t prefix, tprefix, wprefix, kv, kv_cta, meta, cinfo, part_lse, part_o, total;
};

Sm100Ws sm100_ws(int U) {
    Sm100Ws w;
    w.prefix = 0;
    w.tprefix = w.prefix + r256(static_cast<size_t>(U + 1) * 4);
    w.wprefix = w.tprefix + r256(static_cast<size_t>(U + 1) * 4);
    w.kv = w.wprefix + r256(static_cast<size_t>(U + 1) * 4);
    w.kv_cta = w.kv + r256(static_cast<size_t>(U) * 4);
    w.meta = w.kv_cta + r256(static_cast<size_t>(2 * kClusters) * U * 4);
    w.cinfo = w.meta + r256(static_cast<size_t>(U) * 16);
    w.part_lse = w.cinfo + r256(static_cast<size_t>(kClusters) * 16);
    w.part_o = w.part_lse + r256(static_cast<size_t>(kClusters + U) * 128 * 4);
    w.total = w.part_o + r256(static_cast<size_t>(kClusters + U) * 128 * kDc * 4);
    return w;
}

// Test hook state: the next launch withholds one load and uses this wait bound.
std::atomic<uint64_t> g_test_wait_limit_ns{0};

}  // namespace

bool sm100_supports(int n_h, int d_c, int d_r) { return d_c == kDc && d_r == kDr && n_h % 128 == 0; }

size_t sm100_workspace_bytes(int n_h, int d_c, int B, int T_q) {
    if (n_h % 128 != 0 || d_c != kDc) return 0;
    return sm100_ws(B * T_q * (n_h / 128)).total;
}

int sm100_launches(int B, int T_q, int n_h) {
    const int U = B * T_q * (n_h / 128);
    return U <= kInKernelUnits ? 2 : 3;
}

size_t sm100_unit_meta_offset(int n_h, int B, int T_q) { return sm100_ws(B * T_q * (n_h / 128)).meta; }

void sm100_arm_timeout_test(uint64_t wait_limit_ns) { g_test_wait_limit_ns.store(wait_limit_ns); }

cudaError_t launch_decode_sm100(const DecodeParams& P, void* ws, int max_splits, cudaStream_t stream) {
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
        !make_map_2d(&k.tm_qr, P.q_r, kDr, q_rows, kDr * 2, 64, 64) ||
        !make_map_2d(&k.tm_out, P.out_latent, kDc, q_rows, kDc * 2, 64, 32) ||
        !make_map_2d_f32(&k.tm_part, base + w.part_o, kDc, static_cast<uint64_t>(kClusters + U) * 128, kDc * 4, 32,
                         32))
        return cudaErrorInvalidValue;
    k.block_table = P.block_table;
    k.seq_lens = P.seq_lens;
    k.prefix = reinterpret_cast<int32_t*>(base + w.prefix);
    k.unit_kv = reinterpret_cast<int32_t*>(base + w.kv);
    k.kv_cta = reinterpret_cast<int32_t*>(base + w.kv_cta);
    k.unit_meta = reinterpret_cast<int4*>(base + w.meta);
    k.cluster_info = reinterpret_cast<const int4*>(base + w.cinfo);
    k.out_latent = P.out_latent;
    k.out_lse = P.out_lse;
    k.part_o = reinterpret_cast<float*>(base + w.part_o);
    k.part_lse = reinterpret_cast<float*>(base + w.part_lse);
    k.status = P.status;
    k.n_h = P.n_h;
    k.n_hb = n_hb;
    k.B = P.B;
    k.T_q = P.T_q;
    k.U = U;
    k.num_blocks = P.num_blocks;
    k.max_blocks = P.max_blocks;
    k.max_splits = max_splits;
    k.in_kernel_schedule = U <= kInKernelUnits ? 1 : 0;
    const uint64_t test_limit = g_test_wait_limit_ns.exchange(0);
    k.withhold_load = test_limit != 0 ? 1 : 0;
    k.timeout_ns = test_limit != 0 ? test_limit : 2000000000ull;
    k.scale_log2 = P.scale_log2;

    cudaError_t e;
    if (!k.in_kernel_schedule) {
        e = launch_pdl(mla_sm100_schedule_kernel, dim3(1), dim3(1024), 0, stream, P.seq_lens, P.B, P.T_q, n_hb,
                       P.max_blocks, max_splits, U, k.prefix, reinterpret_cast<int32_t*>(base + w.tprefix),
                       reinterpret_cast<int32_t*>(base + w.wprefix),
                       k.unit_kv, k.unit_meta,
                       reinterpret_cast<int4*>(base + w.cinfo), P.status);
        if (e != cudaSuccess) return e;
    }
    static std::atomic<uint64_t> smem_set{0};
    e = allow_smem_once(mla_decode_sm100_kernel, static_cast<int>(kSmemBytes), smem_set);
    if (e != cudaSuccess) return e;
    e = launch_pdl(mla_decode_sm100_kernel, dim3(2 * kClusters), dim3(kThreads), kSmemBytes, stream, k);
    if (e != cudaSuccess) return e;
    const int rows = U * 128;
    return launch_pdl(mla_sm100_merge_kernel, dim3((rows + 7) / 8), dim3(256), 0, stream,
                      static_cast<const int4*>(k.unit_meta), static_cast<const float*>(k.part_o),
                      static_cast<const float*>(k.part_lse), P.out_latent, P.out_lse, P.n_h, n_hb, P.B, P.T_q, U);
}

}  // namespace mla
