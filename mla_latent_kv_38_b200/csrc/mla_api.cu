// Host side of the C ABI declared in include/mla.h: argument checks, workspace
// layout, kernel selection and launches.  No device memory is allocated here.

#include <math.h>
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "sm100_decode.h"
#include "sm100_proj.h"
#include "fold.h"

namespace {

using mla::DecodeParams;

constexpr int kMaxSplits = 256;
constexpr int kB200Sms = 148;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Portable kernels: key-range parts per query row -- the caller's bound, or
// enough (token, 32-head group) CTAs for about 8 per SM.
int choose_splits(const mla_config_t* c, int B, int T_q, int max_splits) {
    if (max_splits > 0) return max_splits < kMaxSplits ? max_splits : kMaxSplits;
    const long work = static_cast<long>(B) * T_q * ((c->n_h + 31) / 32);
    long s = (8L * kB200Sms + work - 1) / work;
    if (s < 1) s = 1;
    if (s > 64) s = 64;
    return static_cast<int>(s);
}

bool uses_sm100(const mla_config_t* c) {
    const bool shape = mla::sm100_supports(c->n_h, c->d_c, c->d_r);
    return c->impl == 2 || (c->impl == 0 && shape);
}

// Workspace: the status word (256 bytes), then the region of the kernel family
// that will run -- the portable kernel's split partials, or the tcgen05
// kernels' schedule arrays and partial slots.
struct WsLayout {
    size_t part_o, part_lse, sm100, total;
};

WsLayout ws_layout_simt(const mla_config_t* c, int B, int T_q, int max_splits) {
    WsLayout w;
    w.part_o = w.part_lse = w.sm100 = 256;
    const int splits = choose_splits(c, B, T_q, max_splits);
    const size_t rows = static_cast<size_t>(B) * T_q * c->n_h;
    const size_t simt_o = splits > 1 ? round256(static_cast<size_t>(splits) * rows * c->d_c * 4) : 0;
    const size_t simt_l = splits > 1 ? round256(static_cast<size_t>(splits) * rows * 4) : 0;
    w.part_lse = w.part_o + simt_o;
    w.total = w.part_lse + simt_l;
    return w;
}

WsLayout ws_layout(const mla_config_t* c, int B, int T_q, int max_splits) {
    if (!uses_sm100(c)) return ws_layout_simt(c, B, T_q, max_splits);
    WsLayout w;
    w.part_o = w.part_lse = w.sm100 = 256;
    w.total = w.sm100 + round256(mla::sm100_workspace_bytes(c->n_h, c->d_c, B, T_q));
    return w;
}

// Shapes of the e4m3 cache format: whole 64-column groups of the latent.
bool e4m3_shape(const mla_config_t* c) { return c->d_c % MLA_E4M3_GROUP == 0; }

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_LAUNCH; }

// Query rows of a decode call: B sequences x T_q tokens, T_q from 1 (decode)
// to a whole prefill chunk; at most 65,535 rows, and for the tcgen05 kernels
// at most 65,535 units of (query row, block of 128 heads).
bool rows_ok(const mla_config_t* c, int B, int T_q) {
    if (B < 1 || T_q < 1) return false;
    const long rows = static_cast<long>(B) * T_q;
    if (rows > 65535) return false;
    return !uses_sm100(c) || rows * (c->n_h / 128) <= 65535;
}

}  // namespace

namespace mla {

int check_config(const mla_config_t* c) {
    if (c == nullptr) return MLA_ERR_NULL;
    if (c->n_h < 1 || c->n_h > 1024) return MLA_ERR_CONFIG;
    if (c->d_c < 8 || c->d_c > 512 || c->d_c % 8) return MLA_ERR_CONFIG;
    if (c->d_r < 8 || c->d_r > 64 || c->d_r % 8) return MLA_ERR_CONFIG;
    if (c->d_h < 8 || c->d_h > 256 || c->d_h % 8) return MLA_ERR_CONFIG;
    if (c->block_size != 64) return MLA_ERR_CONFIG;
    if (c->impl < 0 || c->impl > 2) return MLA_ERR_CONFIG;
    if (!(c->scale == c->scale)) return MLA_ERR_CONFIG;  // NaN
    return MLA_OK;
}

float effective_scale(const mla_config_t* c) {
    return c->scale > 0.f ? c->scale : static_cast<float>(1.0 / sqrt(static_cast<double>(c->d_h + c->d_r)));
}

}  // namespace mla

using mla::check_config;
using mla::effective_scale;

extern "C" {

const char* mla_status_str(int code) {
    switch (code) {
        case MLA_OK: return "ok";
        case MLA_ERR_NULL: return "null pointer";
        case MLA_ERR_CONFIG: return "unsupported configuration";
        case MLA_ERR_SIZE: return "size out of range";
        case MLA_ERR_WORKSPACE: return "workspace too small or misaligned";
        case MLA_ERR_LAUNCH: return "CUDA launch or runtime error";
        case MLA_ERR_UNSUPPORTED: return "device or feature not supported";
        case MLA_ERR_ALIGN: return "pointer not 16-byte aligned";
        default: return "unknown status";
    }
}

int mla_check_device(void) {
    // answer cached per device: 0 unknown, 1 sm_100, 2 other
    static std::atomic<int> known[64];
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_UNSUPPORTED;
    const int k = dev >= 0 && dev < 64 ? known[dev].load(std::memory_order_relaxed) : 0;
    if (k != 0) return k == 1 ? MLA_OK : MLA_ERR_UNSUPPORTED;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MLA_ERR_UNSUPPORTED;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return MLA_ERR_UNSUPPORTED;
    const bool ok = major == 10 && minor == 0;
    if (dev >= 0 && dev < 64) known[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
    return ok ? MLA_OK : MLA_ERR_UNSUPPORTED;
}

int mla_rope_table(int d_r, double base, int max_pos, float* host_table) {
    if (host_table == nullptr) return MLA_ERR_NULL;
    if (d_r < 2 || d_r % 2 || max_pos < 1 || !(base > 0.0)) return MLA_ERR_SIZE;
    const int h = d_r / 2;
    for (int m = 0; m < h; ++m) {
        const double f = pow(base, -2.0 * m / d_r);
        for (int p = 0; p < max_pos; ++p) {
            const double th = static_cast<double>(p) * f;
            host_table[static_cast<size_t>(p) * d_r + m] = static_cast<float>(cos(th));
            host_table[static_cast<size_t>(p) * d_r + h + m] = static_cast<float>(sin(th));
        }
    }
    return MLA_OK;
}

int mla_rope_table_yarn(int d_r, double base, int max_pos, double s, double alpha, double beta, int orig_len,
                        float* host_table) {
    if (host_table == nullptr) return MLA_ERR_NULL;
    if (d_r < 2 || d_r % 2 || max_pos < 1 || !(base > 0.0)) return MLA_ERR_SIZE;
    if (!(s >= 1.0) || !(beta > alpha) || orig_len < 1) return MLA_ERR_SIZE;
    const int h = d_r / 2;
    const double two_pi = 6.283185307179586476925286766559;
    for (int m = 0; m < h; ++m) {
        const double f = pow(base, -2.0 * m / d_r);
        const double turns = orig_len * f / two_pi;   // turns of pair m over the training length
        double g = (turns - alpha) / (beta - alpha);
        g = g < 0.0 ? 0.0 : (g > 1.0 ? 1.0 : g);
        const double fy = f * ((1.0 - g) / s + g);
        for (int p = 0; p < max_pos; ++p) {
            const double th = static_cast<double>(p) * fy;
            host_table[static_cast<size_t>(p) * d_r + m] = static_cast<float>(cos(th));
            host_table[static_cast<size_t>(p) * d_r + h + m] = static_cast<float>(sin(th));
        }
    }
    return MLA_OK;
}

float mla_yarn_score_scale(int d_h, int d_r, double s, double coeff) {
    if (d_h < 1 || d_r < 0 || !(s >= 1.0) || !(coeff >= 0.0)) return 0.f;
    const double sqrt_t = coeff * log(s) + 1.0;
    return static_cast<float>(sqrt_t * sqrt_t / sqrt(static_cast<double>(d_h + d_r)));
}

int mla_absorb_q(const mla_config_t* cfg, const mla_bf16* q_c, const mla_bf16* w_uk,
                 mla_bf16* q_abs, int n_tok, int32_t* dev_status, void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!q_c || !w_uk || !q_abs) return MLA_ERR_NULL;
    if (!aligned16(q_c) || !aligned16(w_uk) || !aligned16(q_abs)) return MLA_ERR_ALIGN;
    if (dev_status && !aligned4(dev_status)) return MLA_ERR_ALIGN;
    if (n_tok < 1 || n_tok > 65536) return MLA_ERR_SIZE;
    const bool sm100_shape = mla::sm100_absorb_supports(cfg->d_h, cfg->d_c);
    if (cfg->impl == 2 && !sm100_shape) return MLA_ERR_CONFIG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cfg->impl == 2 || (cfg->impl == 0 && sm100_shape)) {
        if (mla_check_device() != MLA_OK) return MLA_ERR_UNSUPPORTED;
        return cuda_rc(
            mla::launch_absorb_q_sm100(q_c, w_uk, q_abs, n_tok, cfg->n_h, cfg->d_h, cfg->d_c, dev_status, st));
    }
    return cuda_rc(mla::launch_absorb_q_simt(q_c, w_uk, q_abs, n_tok, cfg->n_h, cfg->d_h, cfg->d_c, st));
}

int mla_rope_append(const mla_config_t* cfg, mla_bf16* q_r, const mla_bf16* k_r,
                    const mla_bf16* c_kv, const int32_t* positions, const float* rope_table,
                    int max_pos, const int32_t* block_table, int max_blocks_per_seq,
                    mla_bf16* pool, int num_blocks, int B, int T_q, int32_t* dev_status,
                    void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!k_r || !c_kv || !positions || !rope_table || !block_table || !pool) return MLA_ERR_NULL;
    if ((q_r && !aligned16(q_r)) || !aligned16(k_r) || !aligned16(c_kv) || !aligned16(pool))
        return MLA_ERR_ALIGN;
    if (!aligned4(positions) || !aligned4(rope_table) || !aligned4(block_table) ||
        (dev_status && !aligned4(dev_status)))
        return MLA_ERR_ALIGN;
    if (B < 1 || T_q < 1 || static_cast<long>(B) * T_q > (1L << 24)) return MLA_ERR_SIZE;
    if (max_pos < 1 || max_blocks_per_seq < 1 || num_blocks < 1) return MLA_ERR_SIZE;
    return cuda_rc(mla::launch_rope_append(q_r, k_r, c_kv, positions, rope_table, max_pos, block_table,
                                           max_blocks_per_seq, pool, false, num_blocks, B * T_q, T_q,
                                           cfg->n_h, cfg->d_c, cfg->d_r, cfg->block_size, dev_status,
                                           static_cast<cudaStream_t>(stream)));
}

size_t mla_decode_workspace_bytes(const mla_config_t* cfg, int B, int T_q, int max_splits) {
    if (check_config(cfg) || !rows_ok(cfg, B, T_q) || max_splits < 0) return 0;
    if (cfg->impl == 2 && !mla::sm100_supports(cfg->n_h, cfg->d_c, cfg->d_r)) return 0;
    return ws_layout(cfg, B, T_q, max_splits).total;
}

int mla_decode(const mla_config_t* cfg, const mla_bf16* q_abs, const mla_bf16* q_r,
               const mla_bf16* pool, int num_blocks, const int32_t* block_table,
               int max_blocks_per_seq, const int32_t* seq_lens, int B, int T_q, int max_splits,
               void* workspace, size_t ws_bytes, mla_bf16* out_latent, float* out_lse,
               void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!q_abs || !q_r || !pool || !block_table || !seq_lens || !workspace || !out_latent || !out_lse)
        return MLA_ERR_NULL;
    if (!aligned16(q_abs) || !aligned16(q_r) || !aligned16(pool) || !aligned16(out_latent) ||
        !aligned4(out_lse) || !aligned4(block_table) || !aligned4(seq_lens))
        return MLA_ERR_ALIGN;
    if (!rows_ok(cfg, B, T_q)) return MLA_ERR_SIZE;
    if (num_blocks < 1 || max_blocks_per_seq < 1 || max_splits < 0) return MLA_ERR_SIZE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLA_ERR_WORKSPACE;
    const bool sm100_shape = mla::sm100_supports(cfg->n_h, cfg->d_c, cfg->d_r);
    if (cfg->impl == 2 && !sm100_shape) return MLA_ERR_CONFIG;
    const bool use_sm100 = uses_sm100(cfg);
    const int splits = use_sm100 ? 0 : choose_splits(cfg, B, T_q, max_splits);
    const WsLayout w = ws_layout(cfg, B, T_q, max_splits);
    if (ws_bytes < w.total) return MLA_ERR_WORKSPACE;

    char* ws = static_cast<char*>(workspace);
    DecodeParams P;
    P.q_abs = q_abs;
    P.q_r = q_r;
    P.pool = pool;
    P.block_table = block_table;
    P.seq_lens = seq_lens;
    P.out_latent = out_latent;
    P.out_lse = out_lse;
    P.part_o = reinterpret_cast<float*>(ws + w.part_o);
    P.part_lse = reinterpret_cast<float*>(ws + w.part_lse);
    P.status = reinterpret_cast<int32_t*>(ws);
    P.n_h = cfg->n_h;
    P.d_c = cfg->d_c;
    P.d_r = cfg->d_r;
    P.block_size = cfg->block_size;
    P.num_blocks = num_blocks;
    P.max_blocks = max_blocks_per_seq;
    P.B = B;
    P.T_q = T_q;
    P.n_tok = B * T_q;
    P.splits = splits;
    P.scale_log2 = effective_scale(cfg) * mla::kLog2e;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    if (use_sm100) {
        if (mla_check_device() != MLA_OK) return MLA_ERR_UNSUPPORTED;
        return cuda_rc(mla::launch_decode_sm100(P, ws + w.sm100, max_splits, st));
    }
    return cuda_rc(mla::launch_decode_simt(P, st));
}

int mla_decode_launches(const mla_config_t* cfg, int B, int T_q, int max_splits) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!rows_ok(cfg, B, T_q) || max_splits < 0) return MLA_ERR_SIZE;
    const bool sm100_shape = mla::sm100_supports(cfg->n_h, cfg->d_c, cfg->d_r);
    if (cfg->impl == 2 && !sm100_shape) return MLA_ERR_CONFIG;
    if (cfg->impl == 2 || (cfg->impl == 0 && sm100_shape))
        return mla::sm100_launches(B, T_q, cfg->n_h);
    return choose_splits(cfg, B, T_q, max_splits) > 1 ? 2 : 1;
}

int mla_decode_split_counts(const mla_config_t* cfg, int B, int T_q, int max_splits, const void* workspace,
                            int32_t* host_counts, int n_counts, void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!workspace || !host_counts) return MLA_ERR_NULL;
    if (!rows_ok(cfg, B, T_q) || max_splits < 0) return MLA_ERR_SIZE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!uses_sm100(cfg)) {
        const int s = choose_splits(cfg, B, T_q, max_splits);
        for (int i = 0; i < n_counts; ++i) host_counts[i] = s;
        return cuda_rc(cudaStreamSynchronize(st));
    }
    if (!mla::sm100_supports(cfg->n_h, cfg->d_c, cfg->d_r)) return MLA_ERR_CONFIG;
    const int U = B * T_q * (cfg->n_h / 128);
    if (n_counts != U) return MLA_ERR_SIZE;
    const WsLayout w = ws_layout(cfg, B, T_q, max_splits);
    const char* meta = static_cast<const char*>(workspace) + w.sm100 + mla::sm100_unit_meta_offset(cfg->n_h, B, T_q);
    // the .z field (parts) of each int4 {kv_len, first cluster, parts, sequence}
    cudaError_t e = cudaMemcpy2DAsync(host_counts, sizeof(int32_t), meta + 2 * sizeof(int32_t), 4 * sizeof(int32_t),
                                      sizeof(int32_t), static_cast<size_t>(U), cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return MLA_ERR_LAUNCH;
    return cuda_rc(cudaStreamSynchronize(st));
}

int mla_test_arm_decode_timeout(uint64_t wait_limit_ns) {
    if (wait_limit_ns == 0 || wait_limit_ns > 2000000000ull) return MLA_ERR_SIZE;
    mla::sm100_arm_timeout_test(wait_limit_ns);
    return MLA_OK;
}

int mla_up_v(const mla_config_t* cfg, const mla_bf16* latent, const mla_bf16* w_uv, mla_bf16* out,
             int n_tok, int32_t* dev_status, void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!latent || !w_uv || !out) return MLA_ERR_NULL;
    if (!aligned16(latent) || !aligned16(w_uv) || !aligned16(out)) return MLA_ERR_ALIGN;
    if (dev_status && !aligned4(dev_status)) return MLA_ERR_ALIGN;
    if (n_tok < 1 || n_tok > 65536) return MLA_ERR_SIZE;
    const bool sm100_shape = mla::sm100_up_v_supports(cfg->d_h, cfg->d_c);
    if (cfg->impl == 2 && !sm100_shape) return MLA_ERR_CONFIG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cfg->impl == 2 || (cfg->impl == 0 && sm100_shape)) {
        if (mla_check_device() != MLA_OK) return MLA_ERR_UNSUPPORTED;
        return cuda_rc(
            mla::launch_up_v_sm100(latent, w_uv, out, n_tok, cfg->n_h, cfg->d_h, cfg->d_c, dev_status, st));
    }
    return cuda_rc(mla::launch_up_v_simt(latent, w_uv, out, n_tok, cfg->n_h, cfg->d_h, cfg->d_c, st));
}

int mla_fold_weights(const mla_config_t* cfg, int d_cq, int d_model, const mla_bf16* w_uq, const mla_bf16* w_uk,
                     const mla_bf16* w_uv, const mla_bf16* w_o, mla_bf16* w_fold_q, mla_bf16* w_fold_o,
                     void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!w_fold_q && !w_fold_o) return MLA_ERR_NULL;
    if (w_fold_q && (!w_uq || !w_uk)) return MLA_ERR_NULL;
    if (w_fold_o && (!w_uv || !w_o)) return MLA_ERR_NULL;
    if (d_cq < 1 || d_cq > 65536 || d_model < 1 || d_model > 65536) return MLA_ERR_SIZE;
    if (mla_check_device() != MLA_OK) return MLA_ERR_UNSUPPORTED;
    return cuda_rc(mla::launch_fold_weights(w_uq, w_uk, w_uv, w_o, w_fold_q, w_fold_o, cfg->n_h, cfg->d_h, cfg->d_c,
                                            d_cq, d_model, static_cast<cudaStream_t>(stream)));
}

int mla_absorb_q_folded(const mla_config_t* cfg, int d_cq, const mla_bf16* c_q, const mla_bf16* w_fold_q,
                        mla_bf16* q_abs, int n_tok, int32_t* dev_status, void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!c_q || !w_fold_q || !q_abs) return MLA_ERR_NULL;
    if (!aligned16(c_q) || !aligned16(w_fold_q) || !aligned16(q_abs)) return MLA_ERR_ALIGN;
    if (dev_status && !aligned4(dev_status)) return MLA_ERR_ALIGN;
    if (n_tok < 1 || n_tok > 65535 || d_cq < 64 || d_cq > 65536) return MLA_ERR_SIZE;
    if (!mla::fold_q_supports(cfg->d_c, d_cq)) return MLA_ERR_CONFIG;
    if (mla_check_device() != MLA_OK) return MLA_ERR_UNSUPPORTED;
    return cuda_rc(mla::launch_q_folded(c_q, w_fold_q, q_abs, n_tok, cfg->n_h, cfg->d_c, d_cq, dev_status,
                                        static_cast<cudaStream_t>(stream)));
}

size_t mla_up_o_folded_workspace_bytes(const mla_config_t* cfg, int d_model, int n_tok) {
    if (check_config(cfg) || n_tok < 1 || n_tok > 65535 || d_model < 1) return 0;
    if (!mla::fold_o_supports(cfg->n_h, cfg->d_c, d_model)) return 0;
    return round256(mla::o_folded_workspace_bytes(cfg->n_h, cfg->d_c, d_model, n_tok));
}

int mla_up_o_folded(const mla_config_t* cfg, int d_model, const mla_bf16* latent, const mla_bf16* w_fold_o,
                    mla_bf16* u, int n_tok, void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!latent || !w_fold_o || !u || !workspace) return MLA_ERR_NULL;
    if (!aligned16(latent) || !aligned16(w_fold_o) || !aligned16(u)) return MLA_ERR_ALIGN;
    if (dev_status && !aligned4(dev_status)) return MLA_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLA_ERR_WORKSPACE;
    if (n_tok < 1 || n_tok > 65535 || d_model < 1 || d_model > 65536) return MLA_ERR_SIZE;
    if (!mla::fold_o_supports(cfg->n_h, cfg->d_c, d_model)) return MLA_ERR_CONFIG;
    if (ws_bytes < mla::o_folded_workspace_bytes(cfg->n_h, cfg->d_c, d_model, n_tok)) return MLA_ERR_WORKSPACE;
    if (mla_check_device() != MLA_OK) return MLA_ERR_UNSUPPORTED;
    return cuda_rc(mla::launch_o_folded(latent, w_fold_o, u, n_tok, cfg->n_h, cfg->d_c, d_model, workspace,
                                        dev_status, static_cast<cudaStream_t>(stream)));
}

size_t mla_e4m3_row_bytes(int d_c, int d_r) {
    if (d_c < MLA_E4M3_GROUP || d_c > 512 || d_c % MLA_E4M3_GROUP) return 0;
    if (d_r < 8 || d_r > 64 || d_r % 8) return 0;
    return static_cast<size_t>(mla::e4m3_row(d_c, d_r).bytes);
}

int mla_rope_append_e4m3(const mla_config_t* cfg, mla_bf16* q_r, const mla_bf16* k_r,
                         const mla_bf16* c_kv, const int32_t* positions, const float* rope_table,
                         int max_pos, const int32_t* block_table, int max_blocks_per_seq,
                         uint8_t* pool, int num_blocks, int B, int T_q, int32_t* dev_status,
                         void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!e4m3_shape(cfg)) return MLA_ERR_CONFIG;
    if (!k_r || !c_kv || !positions || !rope_table || !block_table || !pool) return MLA_ERR_NULL;
    if ((q_r && !aligned16(q_r)) || !aligned16(k_r) || !aligned16(c_kv) || !aligned16(pool))
        return MLA_ERR_ALIGN;
    if (!aligned4(positions) || !aligned4(rope_table) || !aligned4(block_table) ||
        (dev_status && !aligned4(dev_status)))
        return MLA_ERR_ALIGN;
    if (B < 1 || T_q < 1 || static_cast<long>(B) * T_q > (1L << 24)) return MLA_ERR_SIZE;
    if (max_pos < 1 || max_blocks_per_seq < 1 || num_blocks < 1) return MLA_ERR_SIZE;
    return cuda_rc(mla::launch_rope_append(q_r, k_r, c_kv, positions, rope_table, max_pos, block_table,
                                           max_blocks_per_seq, pool, true, num_blocks, B * T_q, T_q,
                                           cfg->n_h, cfg->d_c, cfg->d_r, cfg->block_size, dev_status,
                                           static_cast<cudaStream_t>(stream)));
}

size_t mla_decode_e4m3_workspace_bytes(const mla_config_t* cfg, int B, int T_q, int max_splits) {
    if (check_config(cfg) || !e4m3_shape(cfg) || cfg->impl == 2 || max_splits < 0) return 0;
    if (B < 1 || T_q < 1 || static_cast<long>(B) * T_q > 65535) return 0;
    return ws_layout_simt(cfg, B, T_q, max_splits).total;
}

int mla_decode_e4m3(const mla_config_t* cfg, const mla_bf16* q_abs, const mla_bf16* q_r,
                    const uint8_t* pool, int num_blocks, const int32_t* block_table,
                    int max_blocks_per_seq, const int32_t* seq_lens, int B, int T_q, int max_splits,
                    void* workspace, size_t ws_bytes, mla_bf16* out_latent, float* out_lse,
                    void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!e4m3_shape(cfg) || cfg->impl == 2) return MLA_ERR_CONFIG;
    if (!q_abs || !q_r || !pool || !block_table || !seq_lens || !workspace || !out_latent || !out_lse)
        return MLA_ERR_NULL;
    if (!aligned16(q_abs) || !aligned16(q_r) || !aligned16(pool) || !aligned16(out_latent) ||
        !aligned4(out_lse) || !aligned4(block_table) || !aligned4(seq_lens))
        return MLA_ERR_ALIGN;
    if (B < 1 || T_q < 1 || static_cast<long>(B) * T_q > 65535) return MLA_ERR_SIZE;
    if (num_blocks < 1 || max_blocks_per_seq < 1 || max_splits < 0) return MLA_ERR_SIZE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLA_ERR_WORKSPACE;
    const WsLayout w = ws_layout_simt(cfg, B, T_q, max_splits);
    if (ws_bytes < w.total) return MLA_ERR_WORKSPACE;

    char* ws = static_cast<char*>(workspace);
    DecodeParams P;
    P.q_abs = q_abs;
    P.q_r = q_r;
    P.pool = nullptr;
    P.pool8 = pool;
    P.block_table = block_table;
    P.seq_lens = seq_lens;
    P.out_latent = out_latent;
    P.out_lse = out_lse;
    P.part_o = reinterpret_cast<float*>(ws + w.part_o);
    P.part_lse = reinterpret_cast<float*>(ws + w.part_lse);
    P.status = reinterpret_cast<int32_t*>(ws);
    P.n_h = cfg->n_h;
    P.d_c = cfg->d_c;
    P.d_r = cfg->d_r;
    P.block_size = cfg->block_size;
    P.num_blocks = num_blocks;
    P.max_blocks = max_blocks_per_seq;
    P.B = B;
    P.T_q = T_q;
    P.n_tok = B * T_q;
    P.splits = choose_splits(cfg, B, T_q, max_splits);
    P.scale_log2 = effective_scale(cfg) * mla::kLog2e;
    return cuda_rc(mla::launch_decode_simt(P, static_cast<cudaStream_t>(stream)));
}

int mla_clear_status(int32_t* dev_status, void* stream) {
    if (!dev_status) return MLA_ERR_NULL;
    return cuda_rc(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)));
}

int mla_read_status(const int32_t* dev_status, int32_t* host_status, void* stream) {
    if (!dev_status || !host_status) return MLA_ERR_NULL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(host_status, dev_status, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return MLA_ERR_LAUNCH;
    return cuda_rc(cudaStreamSynchronize(st));
}

}  // extern "C"
