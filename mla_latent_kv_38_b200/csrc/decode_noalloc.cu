// mla_decode_noalloc: the portable decode kernel with its split-KV scratch held
// in a fixed device array of this library instead of a caller workspace.
//
// Some callers cannot allocate device memory at the point where they decode:
// code running inside a framework that owns every allocation through its own
// pool, plugins handed only input and output buffers, or hosts that must not
// grow device memory after start-up.  This entry point serves them.  The
// scratch is a file-scope __device__ array, so every GPU that loads the library
// holds kNoAllocScratchBytes of it until the process exits.
//
// The host cannot use the array's name as a device address: in host code it
// only names a host-side stand-in.  The device address is looked up once per
// device with cudaGetSymbolAddress, with that device current, the first time
// the entry point runs on it, and cached.  The cached address belongs to the
// device's context of that moment: after a cudaDeviceReset the module is
// loaded again and the array may sit elsewhere, so a process that resets a
// device must not call this entry point on that device again.

#include <math.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (set-up on first use).
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_LAUNCH;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
            return MLA_ERR_LAUNCH;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MLA_OK;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool al4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" int mla_decode_noalloc(const mla_config_t* cfg, const mla_bf16* q_abs, const mla_bf16* q_r,
                                  const mla_bf16* pool, int num_blocks, const int32_t* block_table,
                                  int max_blocks_per_seq, const int32_t* seq_lens, int B, int T_q,
                                  int splits, mla_bf16* out_latent, float* out_lse,
                                  int32_t* dev_status, void* stream) {
    const int rc_cfg = mla::check_config(cfg);   // the same checks as every other entry point
    if (rc_cfg != MLA_OK) return rc_cfg;
    if (!q_abs || !q_r || !pool || !block_table || !seq_lens || !out_latent || !out_lse)
        return MLA_ERR_NULL;
    if (!al16(q_abs) || !al16(q_r) || !al16(pool) || !al16(out_latent) || !al4(out_lse) ||
        !al4(block_table) || !al4(seq_lens) || (dev_status && !al4(dev_status)))
        return MLA_ERR_ALIGN;
    if (B < 1 || T_q < 1 || static_cast<long>(B) * T_q > 65535) return MLA_ERR_SIZE;
    if (num_blocks < 1 || max_blocks_per_seq < 1 || splits < 1 || splits > 256) return MLA_ERR_SIZE;

    // Scratch use: split partials, fp32 latent rows then fp32 lse, 256-aligned.
    // Nothing in it has to start at zero: every split writes its whole partial
    // (an empty key range writes lse = -inf) before the merge kernel reads it,
    // so the previous call's contents are never observed.
    const size_t rows = static_cast<size_t>(B) * T_q * cfg->n_h;
    const size_t o_bytes = splits > 1 ? ((static_cast<size_t>(splits) * rows * cfg->d_c * 4 + 255) & ~size_t(255)) : 0;
    const size_t l_bytes = splits > 1 ? static_cast<size_t>(splits) * rows * 4 : 0;
    if (o_bytes + l_bytes > kNoAllocScratchBytes) return MLA_ERR_SIZE;

    void* scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != MLA_OK) return rc;

    mla::DecodeParams P;
    P.q_abs = q_abs;
    P.q_r = q_r;
    P.pool = pool;
    P.block_table = block_table;
    P.seq_lens = seq_lens;
    P.out_latent = out_latent;
    P.out_lse = out_lse;
    P.part_o = static_cast<float*>(scratch);
    P.part_lse = reinterpret_cast<float*>(static_cast<char*>(scratch) + o_bytes);
    P.status = dev_status;
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
    P.scale_log2 = mla::effective_scale(cfg) * mla::kLog2e;
    return mla::launch_decode_simt(P, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MLA_OK
                                                                                          : MLA_ERR_LAUNCH;
}
