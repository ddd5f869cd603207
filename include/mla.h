/*
 * mla.h -- C ABI of the B200 (sm_100a) MLA latent-KV decode library.
 *
 * One decode step of Multi-head Latent Attention over a paged latent cache:
 *
 *   mla_absorb_q     q_abs = W^UK^T q^C, per head
 *   mla_rope_append  RoPE on q^R and k^R, then c^KV || k^R appended to the cache
 *   mla_decode       causal softmax of the absorbed scores over the cached rows,
 *                    weighted sum of the latent rows (split-KV + LSE merge)
 *   mla_up_v         o = W^UV latent, per head
 *
 * and, around them: the folded projections (mla_fold_weights,
 * mla_absorb_q_folded, mla_up_o_folded), the YaRN-scaled RoPE table and score
 * scale, and a low-bit cache format with its own append and decode
 * (mla_rope_append_e4m3, mla_decode_e4m3).
 *
 * Sources (page title, section / equation):
 *   [notes]  "MLA(Multi-head Latent Attention): DeepSeek-V2 논문정리":
 *            eq. (9)-(11); "Key에 대한 수식 전개"; "Value에 대한 수식 전개";
 *            "Decoupled Rotary Position Embedding"; "MLA 코드 구현".
 *   [ru]     "Техотчёт DeepSeek-V2 (2024): MLA и экономика инференса":
 *            "Идея 1", "Идея 2: отделённый RoPE", "Сколько получилось".
 *   [v3]     DeepSeek-V3 report notes, "Multi-Head Attention 및 Output 계산
 *            (식 10, 11)", eq. (10).
 *   [review] "DeepSeek-V2 review", 2.1 (absorption, T = max(B/BW, F/P)),
 *            2.3 (Decoupled RoPE).
 *
 * Conventions for every call
 *   - Element type mla_bf16 is the raw 16-bit pattern of a bfloat16.
 *   - All tensor pointers are DEVICE pointers unless a parameter says "host".
 *     The caller allocates and owns every buffer; the library never allocates
 *     device memory.  mla_decode takes a caller-provided workspace whose size
 *     mla_decode_workspace_bytes() returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on that stream.
 *   - Return value: MLA_OK (0) or a negative MLA_ERR_* code.  Every argument
 *     check that needs no device data happens on the host before any launch;
 *     a rejected call launches nothing and writes nothing.
 *   - Checks that need device data (positions, block indices, sequence
 *     lengths) run in the kernels: an offending row is skipped (never read or
 *     written out of bounds) and a bit is OR-ed into a device status word
 *     (MLA_STATUS_* bits).  Read it with mla_read_status().
 *   - Layouts are row-major and densely packed in the order written.
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t mla_bf16;

/* Head shapes of one attention layer.  DeepSeek-V2: n_h = 128, d_c = 512,
 * d_h = 128, d_r = 64 ([ru] "Сколько получилось"; [v3]).  block_size is the
 * number of cache rows per page (64).  scale <= 0 selects 1/sqrt(d_h + d_r)
 * ([v3] eq. (10); [ru] "Идея 2").  impl selects among this library's own
 * decode kernels; all of them compute the same function. */
typedef struct {
    int n_h;
    int d_c;
    int d_h;
    int d_r;
    int block_size;
    float scale;
    int impl; /* kernel family: 0 = best for the shape, 1 = portable CUDA-core
                 kernels (any supported shape), 2 = tcgen05 tensor-core kernels,
                 MLA_ERR_CONFIG where they do not tile the shape:
                   mla_decode   d_c = 512, d_r = 64, n_h a multiple of 128
                   mla_absorb_q d_h a multiple of 64, d_c a multiple of 128
                   mla_up_v     d_h a multiple of 128
                 (mla_rope_append has one kernel for every shape) */
} mla_config_t;

enum {
    MLA_OK = 0,
    MLA_ERR_NULL = -1,        /* a required pointer is NULL                   */
    MLA_ERR_CONFIG = -2,      /* unsupported head shape / block size          */
    MLA_ERR_SIZE = -3,        /* a count is out of range (n_tok, B, T_q ...)  */
    MLA_ERR_WORKSPACE = -4,   /* workspace too small or misaligned            */
    MLA_ERR_LAUNCH = -5,      /* a CUDA launch or runtime call failed         */
    MLA_ERR_UNSUPPORTED = -6, /* device is not sm_100 or feature unavailable  */
    MLA_ERR_ALIGN = -7        /* a pointer breaks its alignment rule (below)  */
};

/* Device status word bits (see mla_read_status). */
enum {
    MLA_STATUS_BAD_POSITION = 1,  /* position < 0 or beyond the RoPE table    */
    MLA_STATUS_BAD_BLOCK = 2,     /* block-table entry outside [0, num_blocks) */
    MLA_STATUS_BAD_SEQ_LEN = 4,   /* seq_len < T_q or beyond the block table  */
    MLA_STATUS_TIMEOUT = 8        /* a bounded device wait ran out            */
};

/* Constraints shared by every call: d_c, d_r and d_h multiples of 8,
 * 8 <= d_c <= 512, 8 <= d_r <= 64, 8 <= d_h <= 256, block_size = 64,
 * 1 <= n_h <= 1024.  Pointers to bf16 tensors are 16-byte aligned; pointers
 * to int32 and float32 arrays (positions, tables, lengths, lse, status) are
 * 4-byte aligned; the mla_decode workspace is 256-byte aligned. */

/* Human-readable name of a return code. */
const char* mla_status_str(int code);

/* Compute capability check: returns MLA_OK when the current device is sm_100. */
int mla_check_device(void);

/* RoPE table on the HOST: host_table[p * d_r + m] = cos(p * f_m) and
 * host_table[p * d_r + d_r/2 + m] = sin(p * f_m) for p < max_pos and
 * f_m = base^(-2m/d_r), m < d_r/2, evaluated in double and rounded to float
 * ([notes] "MLA 코드 구현", build_rope_cache).  The caller copies it to the
 * device and passes it to mla_rope_append.  host_table holds max_pos * d_r
 * floats. */
int mla_rope_table(int d_r, double base, int max_pos, float* host_table);

/* YaRN RoPE table on the HOST, same layout as mla_rope_table, for a context
 * stretched s times past the training length orig_len ("Техотчёт DeepSeek-V2
 * (2024)", long context; "DeepSeek-V2 review", 4: YaRN on the decoupled
 * k^R, 4K -> 128K with s = 40, alpha = 1, beta = 32).  Pair m with frequency
 * f_m = base^(-2m/d_r) turns r_m = orig_len f_m / (2 pi) times over the
 * training length; with g_m = clamp((r_m - alpha) / (beta - alpha), 0, 1) it
 * rotates at f_m ((1 - g_m) / s + g_m): pairs turning fewer than alpha times
 * are interpolated by s, pairs turning more than beta times are kept.
 * Evaluated in double, rounded to float.  s >= 1, beta > alpha. */
int mla_rope_table_yarn(int d_r, double base, int max_pos, double s, double alpha, double beta,
                        int orig_len, float* host_table);

/* Score scale with the YaRN attention temperature: t / sqrt(d_h + d_r) with
 * sqrt(t) = coeff ln s + 1 (DeepSeek-V2 uses coeff = 0.0707; 0.1 in the
 * generic rule), i.e. both q and k multiplied by sqrt(t).  Pass it as
 * mla_config_t.scale.  Returns 0 for invalid arguments. */
float mla_yarn_score_scale(int d_h, int d_r, double s, double coeff);

/* q_abs[n, i, :] = W^UK_i^T q_c[n, i, :]  ([notes] "Key에 대한 수식 전개";
 * [ru] "Идея 1").
 *   q_c   (n_tok, n_h, d_h)  bf16
 *   w_uk  (n_h, d_h, d_c)    bf16; W^UK_i = w_uk[i] maps a latent to head i's key
 *   q_abs (n_tok, n_h, d_c)  bf16 out (float accumulation, RNE rounding)
 *   dev_status one int32 on the device (may be NULL): the tensor-core kernel
 *              ORs MLA_STATUS_TIMEOUT in when one of its bounded waits runs
 *              out; q_abs is then incomplete.
 * n_tok = B * T_q, token n = b * T_q + t.  1 <= n_tok <= 65536. */
int mla_absorb_q(const mla_config_t* cfg, const mla_bf16* q_c, const mla_bf16* w_uk,
                 mla_bf16* q_abs, int n_tok, int32_t* dev_status, void* stream);

/* Decoupled RoPE and paged append ([review] 2.3; [ru] "Идея 2"; [notes]
 * "Decoupled Rotary Position Embedding", "MLA 코드 구현" forward).
 * For token n = b * T_q + t with p = positions[n]:
 *   q_r[n, i, :] <- RoPE(q_r[n, i, :], p) for every head i (skipped if q_r NULL)
 *   pool[blk][p % block_size][0 : d_c]        <- c_kv[n, :]           (bit copy)
 *   pool[blk][p % block_size][d_c : d_c+d_r]  <- RoPE(k_r[n, :], p)
 * with blk = block_table[b * max_blocks_per_seq + p / block_size].
 * RoPE pairs element m with m + d_r/2 (half split) and uses float32 products
 * and sums without fused multiply-add on the float32 table, then rounds to
 * bf16 (round to nearest even).
 *   q_r        (n_tok, n_h, d_r) bf16, in place, may be NULL
 *   k_r        (n_tok, d_r) bf16;  c_kv (n_tok, d_c) bf16
 *   positions  (n_tok) int32
 *   rope_table (max_pos, d_r) float32 from mla_rope_table
 *   block_table (B, max_blocks_per_seq) int32
 *   pool       (num_blocks, block_size, d_c + d_r) bf16
 *   dev_status one int32 on the device (may be NULL): MLA_STATUS_* bits are
 *              OR-ed in for rows whose position or block index is invalid;
 *              those rows are not written. */
int mla_rope_append(const mla_config_t* cfg, mla_bf16* q_r, const mla_bf16* k_r,
                    const mla_bf16* c_kv, const int32_t* positions,
                    const float* rope_table, int max_pos,
                    const int32_t* block_table, int max_blocks_per_seq,
                    mla_bf16* pool, int num_blocks, int B, int T_q,
                    int32_t* dev_status, void* stream);

/* Bytes of workspace mla_decode needs for these sizes (256-byte aligned
 * pointer required).  max_splits as for mla_decode.  The size covers only the
 * kernel family that cfg selects for this shape; 0 for invalid arguments. */
size_t mla_decode_workspace_bytes(const mla_config_t* cfg, int B, int T_q, int max_splits);

/* Absorbed MLA decode over the paged cache ([v3] eq. (10) with [notes]
 * "Key에 대한 수식 전개" and "Value에 대한 수식 전개"):
 *   s[b,t,i,j] = scale * (q_abs[b,t,i,:] . pool_row(b,j)[0:d_c]
 *                         + q_r[b,t,i,:] . pool_row(b,j)[d_c:d_c+d_r])
 * for keys j <= seq_lens[b] - T_q + t (generalised causal mask, [notes]
 * "MLA 코드 구현" forward), softmax over j, and
 *   out_latent[b,t,i,:] = sum_j p[b,t,i,j] pool_row(b,j)[0:d_c]     (bf16)
 *   out_lse[b,t,i]      = log sum_j exp(s[b,t,i,j])                  (float32)
 *   q_abs (B*T_q, n_h, d_c) bf16;  q_r (B*T_q, n_h, d_r) bf16 (already RoPE'd)
 *   pool, block_table as for mla_rope_append; seq_lens (B) int32, the cache
 *   length AFTER the step's append, 1 <= T_q <= seq_lens[b].
 *   max_splits: upper bound on the parts the key range of one query row is
 *   split into (0 = the library chooses):
 *     tcgen05 kernels: the 256-key tiles of all (query row, block of 128
 *       heads) units are laid end to end and cut into 74 contiguous ranges,
 *       one per pair of SMs.  0 cuts them into equal ranges (a unit may span
 *       several); s > 0 moves every cut to the next of the points that divide
 *       each unit's P tiles into min(s, P) near-equal pieces, so no unit lies
 *       in more than s ranges (1 = no unit is split).
 *       mla_decode_split_counts reports the parts each unit got.
 *     portable kernels: exactly max_splits parts (0: a count from B, T_q, n_h).
 * Partial results (fp32 latent rows and log-sum-exp) of split rows go to the
 * workspace and are merged by a log-sum-exp reduction kernel.  The workspace
 * starts with the device status word (mla_read_status).
 * Sizes: B * T_q <= 65535 query rows (and B * T_q * n_h / 128 <= 65535 units
 * on the tcgen05 kernels).  T_q > 1 with the generalised mask is also chunked
 * prefill ([notes] "MLA 코드 구현", "학습 시와 디코딩 시의 흐름"): a chunk of
 * T_q new tokens, appended by mla_rope_append, attends to the cached prefix
 * and causally to itself; T_q = seq_lens[b] is prefill from an empty cache. */
int mla_decode(const mla_config_t* cfg, const mla_bf16* q_abs, const mla_bf16* q_r,
               const mla_bf16* pool, int num_blocks, const int32_t* block_table,
               int max_blocks_per_seq, const int32_t* seq_lens, int B, int T_q,
               int max_splits, void* workspace, size_t ws_bytes,
               mla_bf16* out_latent, float* out_lse, void* stream);

/* Number of kernel launches one mla_decode call with these arguments makes
 * (decode, optional scheduling and merge kernels); negative on bad arguments. */
int mla_decode_launches(const mla_config_t* cfg, int B, int T_q, int max_splits);

/* Diagnostic: after an mla_decode call with these arguments has completed on
 * `stream`, copies to host_counts the number of parts (key-range splits) of
 * each unit of work, read back from the workspace; synchronises `stream`.
 * tcgen05 kernels: one count per (query row, block of 128 heads), in the
 * kernels' token-major order u = (t * B + b) * (n_h / 128) + head block,
 * n_counts = B * T_q * n_h / 128 (0 for a row whose sequence length was
 * invalid).  Portable kernels: the
 * fixed split count, written to all n_counts entries. */
int mla_decode_split_counts(const mla_config_t* cfg, int B, int T_q, int max_splits,
                            const void* workspace, int32_t* host_counts, int n_counts,
                            void* stream);

/* Test hook for the bounded device waits (no page has a counterpart).  Arms the NEXT mla_decode call that runs the
 * tcgen05 kernels: that call never issues one of its cache loads, so a
 * barrier that nothing completes is waited on, and every wait of the call is
 * bounded by wait_limit_ns (1 ns .. 2 s) instead of 2 s.  The call returns
 * MLA_OK; the kernel unwinds, sets MLA_STATUS_TIMEOUT in the status word and
 * releases its tensor memory, and its outputs are undefined.  Later calls run
 * normally.  Not for production use. */
int mla_test_arm_decode_timeout(uint64_t wait_limit_ns);

/* mla_decode for callers that cannot allocate device memory: the pages have
 * no counterpart; this is a deployment variant of the same computation.
 * Callers inside frameworks that own every device allocation, plugins that
 * are handed only their input and output buffers, or hosts that must not grow
 * device memory after start-up cannot provide mla_decode's workspace.  This
 * call takes no workspace and allocates nothing: it runs the portable decode
 * kernel (the impl = 1 kernel, whatever cfg->impl says) and keeps its split-KV
 * partial results in a fixed 16 MiB device array inside this library, which
 * every GPU that loads the library holds until the process exits.
 *   Arguments as for mla_decode, except:
 *   splits      key-range splits per query row, 1..256 (no automatic choice);
 *               when splits > 1 the partials need
 *               splits * B * T_q * n_h * (4 * d_c + 4) bytes (plus 256-byte
 *               rounding) and a call needing more than 16 MiB returns
 *               MLA_ERR_SIZE without launching anything.
 *   dev_status  optional device int32 that device-side checks OR
 *               MLA_STATUS_* bits into (NULL: not reported).
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it; make that
 * first call before any stream capture.  A cudaDeviceReset invalidates the
 * cached address: do not call this entry point on a device again after
 * resetting it in the same process.  All calls share the one array, which
 * keeps the last call's contents (each call fully writes what it reads, so
 * nothing needs clearing); calls that overlap on the GPU, on different streams
 * or from different host threads, race on it and must be serialised by the
 * caller. */
int mla_decode_noalloc(const mla_config_t* cfg, const mla_bf16* q_abs, const mla_bf16* q_r,
                       const mla_bf16* pool, int num_blocks, const int32_t* block_table,
                       int max_blocks_per_seq, const int32_t* seq_lens, int B, int T_q,
                       int splits, mla_bf16* out_latent, float* out_lse,
                       int32_t* dev_status, void* stream);

/* o[n, i, :] = W^UV_i latent[n, i, :]  ([notes] "Value에 대한 수식 전개").
 *   latent (n_tok, n_h, d_c) bf16;  w_uv (n_h, d_h, d_c) bf16
 *   out    (n_tok, n_h, d_h) bf16 (float accumulation, RNE rounding)
 *   dev_status as for mla_absorb_q. */
int mla_up_v(const mla_config_t* cfg, const mla_bf16* latent, const mla_bf16* w_uv,
             mla_bf16* out, int n_tok, int32_t* dev_status, void* stream);

/* Folded projections ([notes] "Key에 대한 수식 전개": the key up-projection
 * folds into the query projection, W'^Q = (W^Q)^T W^UK; "Value에 대한 수식
 * 전개": the value up-projection folds into the output projection,
 * W'^O = W^O W^UV; [ru] "Идея 1").  With the query latent c^Q (d_cq columns,
 * 1536 at DeepSeek-V2) and the model width d_model (5120 at DeepSeek-V2):
 *   w_uq (n_h, d_h, d_cq): q^C[n, i, :] = w_uq[i] c_q[n]
 *   w_o  (d_model, n_h, d_h): u[n] = sum_i w_o[:, i, :] o[n, i, :]
 *   w_fold_q (n_h, d_c, d_cq): F_i = W^UK_i^T W^UQ_i
 *   w_fold_o (d_model, n_h, d_c): G_i = W^O_i W^UV_i
 * The fold multiplies the weight bytes a decode step reads (at DeepSeek-V2
 * 3.0 x on the query side, 3.6 x on the output side); it pays only where
 * the step is compute-bound.  All bf16, row-major, 16-byte aligned.
 *
 * mla_fold_weights: computes w_fold_q and/or w_fold_o (either may be null,
 * not both; fp32 sums rounded to bf16, CUDA cores; once per weight set). */
int mla_fold_weights(const mla_config_t* cfg, int d_cq, int d_model,
                     const mla_bf16* w_uq, const mla_bf16* w_uk, const mla_bf16* w_uv,
                     const mla_bf16* w_o, mla_bf16* w_fold_q, mla_bf16* w_fold_o, void* stream);

/* q_abs[n, i, :] = F_i c_q[n] (the folded mla_absorb_q, from the query
 * latent): c_q (n_tok, d_cq); q_abs (n_tok, n_h, d_c) as for mla_decode.
 * tcgen05 kernels only: d_c a multiple of 128, d_cq of 64 (MLA_ERR_CONFIG
 * otherwise).  dev_status as for mla_absorb_q. */
int mla_absorb_q_folded(const mla_config_t* cfg, int d_cq, const mla_bf16* c_q,
                        const mla_bf16* w_fold_q, mla_bf16* q_abs, int n_tok,
                        int32_t* dev_status, void* stream);

/* Bytes of workspace mla_up_o_folded needs (256-byte aligned pointer); 0 for
 * invalid arguments. */
size_t mla_up_o_folded_workspace_bytes(const mla_config_t* cfg, int d_model, int n_tok);

/* u[n] = sum_i G_i latent[n, i, :] (the folded mla_up_v followed by the output
 * projection): latent (n_tok, n_h, d_c) from mla_decode; u (n_tok, d_model).
 * One product with K = n_h d_c, split over K; the fp32 partial sums go to the
 * caller's workspace and are added by a second kernel.  tcgen05 kernels only:
 * d_model a multiple of 128, n_h d_c of 64. */
int mla_up_o_folded(const mla_config_t* cfg, int d_model, const mla_bf16* latent,
                    const mla_bf16* w_fold_o, mla_bf16* u, int n_tok, void* workspace,
                    size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---- Low-bit latent cache ------------------------------------------------
 * The pages quote a KV cache of about 6 bits per element for the served model
 * ("DeepSeek-V2 review", 4.2 Evaluation, "Inference efficiency"; [ru]
 * "Откуда берутся 93,3%") and give no format.  This library's format: the
 * latent c^KV as OCP FP8 E4M3 codes with one float32 scale per
 * MLA_E4M3_GROUP latent columns; the rotated RoPE key k^R stays bf16 (its
 * rotation carries the position, [ru] "Идея 2").  One cache row, bytes:
 *   [0, d_c)                          e4m3 codes of c^KV
 *   [S, S + 4 d_c / 64)               float32 scales,  S = d_c rounded up to 16
 *   [R, R + 2 d_r)                    bf16 RoPE key,   R = end of the scales
 *                                                        rounded up to 16
 *   padding to mla_e4m3_row_bytes(d_c, d_r) (a multiple of 16), zero.
 * At DeepSeek-V2 (d_c 512, d_r 64) a row is 672 bytes against 1,152 in bf16.
 * Quantisation of a group x (the bf16 latent values as float32): amax =
 * max |x|; inv = 448 / amax and scale = amax / 448 (float32 divisions,
 * round to nearest even); code = e4m3(x * inv) (float32 product, then round
 * to nearest even with saturation at +-448).  amax = 0 stores scale 0 and
 * zero codes.  A cached value reads back as e4m3(code) * scale.  Inputs must
 * be finite.  Pool: (num_blocks, block_size, mla_e4m3_row_bytes) bytes,
 * 16-byte aligned.  Shapes: d_c a multiple of 64 (MLA_ERR_CONFIG otherwise). */
#define MLA_E4M3_GROUP 64

/* Bytes of one cache row in the e4m3 format; 0 for an unsupported shape. */
size_t mla_e4m3_row_bytes(int d_c, int d_r);

/* mla_rope_append into an e4m3 pool: the same RoPE of q^R (in place) and
 * k^R, the same positions, block table and status bits; the appended row is
 * the quantised latent, its scales and the rotated bf16 key. */
int mla_rope_append_e4m3(const mla_config_t* cfg, mla_bf16* q_r, const mla_bf16* k_r,
                         const mla_bf16* c_kv, const int32_t* positions,
                         const float* rope_table, int max_pos,
                         const int32_t* block_table, int max_blocks_per_seq,
                         uint8_t* pool, int num_blocks, int B, int T_q,
                         int32_t* dev_status, void* stream);

/* Workspace bytes of mla_decode_e4m3 (256-byte aligned pointer required);
 * 0 for invalid arguments. */
size_t mla_decode_e4m3_workspace_bytes(const mla_config_t* cfg, int B, int T_q, int max_splits);

/* mla_decode over an e4m3 pool: the same scores, mask, softmax, outputs and
 * size limits, with every cached latent value read back as e4m3(code) *
 * scale (in float32) and the key's RoPE part as stored.  Runs the portable
 * CUDA-core decode kernel (cfg->impl 0 or 1; 2 returns MLA_ERR_CONFIG) with
 * exactly max_splits key-range parts per query row (0: a count from B, T_q,
 * n_h), merged by the log-sum-exp reduction.  The workspace starts with the
 * device status word. */
int mla_decode_e4m3(const mla_config_t* cfg, const mla_bf16* q_abs, const mla_bf16* q_r,
                    const uint8_t* pool, int num_blocks, const int32_t* block_table,
                    int max_blocks_per_seq, const int32_t* seq_lens, int B, int T_q,
                    int max_splits, void* workspace, size_t ws_bytes,
                    mla_bf16* out_latent, float* out_lse, void* stream);

/* Zero a device status word (async on stream). */
int mla_clear_status(int32_t* dev_status, void* stream);

/* Copy a device status word to *host_status; synchronises `stream`.  For
 * mla_decode the word is the first int32 of the workspace. */
int mla_read_status(const int32_t* dev_status, int32_t* host_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H */
