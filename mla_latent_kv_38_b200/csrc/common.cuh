// Shared device helpers of the MLA decode library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "mla.h"

namespace mla {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float bf2f(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// float -> bf16 bits, round to nearest even (hardware conversion)
__device__ __forceinline__ uint16_t f2bf(float f) {
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&h);
}

// two floats -> packed bf16x2 (lo in the low half), one paired conversion
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Two float32 values -> two OCP FP8 E4M3 codes (round to nearest even,
// saturating at +-448); lo in the low byte.
__device__ __forceinline__ uint16_t e4m3x2_from_f32(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two E4M3 codes (low byte first) -> their values as float32 (exact).
__device__ __forceinline__ float2 e4m3x2_to_f32(uint16_t codes) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(codes));
    float lo, hi;
    asm("{\n\t.reg .f16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
        : "=f"(lo), "=f"(hi) : "r"(h));
    return make_float2(lo, hi);
}

// Byte offsets of one e4m3 cache row (layout in include/mla.h): the group
// scales, the bf16 RoPE key, and the row's size.
struct E4m3Row {
    int scale_off, kr_off, bytes;
};

__host__ __device__ __forceinline__ E4m3Row e4m3_row(int d_c, int d_r) {
    E4m3Row r;
    r.scale_off = (d_c + 15) / 16 * 16;
    r.kr_off = (r.scale_off + 4 * (d_c / MLA_E4M3_GROUP) + 15) / 16 * 16;
    r.bytes = (r.kr_off + 2 * d_r + 15) / 16 * 16;
    return r;
}

// 2^x on the special-function unit (PTX ex2.approx; 2^-inf = +0)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void raise_status(int32_t* st, int bits) {
    if (st != nullptr) atomicOr(st, bits);
}

// ---- programmatic dependent launch --------------------------------------
// Kernels launched with launch_pdl() may be scheduled while the previous
// kernel of the stream is still running.  Each of them lets its own successor
// start early (griddep_launch_dependents) and executes griddep_wait() -- which
// returns once the previous kernel has completed and its writes are visible --
// before it reads or writes any buffer that an earlier kernel may touch, and
// always before it exits, so that completion stays ordered along the stream.

__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Raise a kernel's dynamic shared-memory limit to `bytes` once per device
// (the attribute is per device and function; later calls skip the runtime call).
template <typename... KArgs>
inline cudaError_t allow_smem_once(void (*kernel)(KArgs...), int bytes, std::atomic<uint64_t>& done_mask) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (done_mask.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done_mask.fetch_or(bit, std::memory_order_release);
    return e;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Parameters of one decode launch (shared by the SIMT and tcgen05 kernels).
struct DecodeParams {
    const uint16_t* q_abs;      // (n_tok, n_h, d_c)
    const uint16_t* q_r;        // (n_tok, n_h, d_r)
    const uint16_t* pool;       // (num_blocks, block_size, d_c + d_r)
    const uint8_t* pool8 = nullptr;   // e4m3 pool (portable kernel only), else null
    const int32_t* block_table; // (B, max_blocks)
    const int32_t* seq_lens;    // (B)
    uint16_t* out_latent;       // (n_tok, n_h, d_c)
    float* out_lse;             // (n_tok, n_h)
    float* part_o;              // (splits, n_tok, n_h, d_c) fp32
    float* part_lse;            // (splits, n_tok, n_h)
    int32_t* status;
    int n_h, d_c, d_r, block_size;
    int num_blocks, max_blocks, B, T_q, n_tok, splits;
    float scale_log2;           // scale * log2(e)
};

}  // namespace mla
