// Host-side encoding of TMA tensor maps (internal).  The driver entry point is
// looked up once through the runtime, so the library links only cudart.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

namespace mla {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
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

// Encoded tensor maps are cached by their arguments (the maps of a decode
// step's buffers do not change from step to step, and encoding one costs host
// time on every call): a small direct-mapped table under a mutex, so that
// repeated calls with the same buffers copy the map instead of re-encoding it.
struct TmapKey {
    uint64_t base;
    uint64_t dims[3], strides[2];
    uint32_t box[3], dtype, rank, swizzle;
};

inline bool encode_tiled_cached(CUtensorMap* m, CUtensorMapDataType dtype, uint32_t rank, const void* base,
                                const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                                CUtensorMapSwizzle swizzle) {
    constexpr int kSlots = 256;
    struct Slot {
        bool valid;
        TmapKey key;
        CUtensorMap map;
    };
    static Slot slots[kSlots];
    static std::mutex mu;
    TmapKey k;
    memset(&k, 0, sizeof(k));
    k.base = reinterpret_cast<uint64_t>(base);
    for (uint32_t i = 0; i < rank; ++i) {
        k.dims[i] = dims[i];
        k.box[i] = box[i];
        if (i + 1 < rank) k.strides[i] = strides[i];
    }
    k.dtype = static_cast<uint32_t>(dtype);
    k.rank = rank;
    k.swizzle = static_cast<uint32_t>(swizzle);
    uint64_t h = 1469598103934665603ull;   // FNV-1a over the key bytes
    const unsigned char* kb = reinterpret_cast<const unsigned char*>(&k);
    for (size_t i = 0; i < sizeof(k); ++i) h = (h ^ kb[i]) * 1099511628211ull;
    Slot& sl = slots[h % kSlots];
    {
        std::lock_guard<std::mutex> lock(mu);
        if (sl.valid && memcmp(&sl.key, &k, sizeof(k)) == 0) {
            *m = sl.map;
            return true;
        }
    }
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint32_t estr[3] = {1, 1, 1};
    if (fn(m, dtype, rank, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    std::lock_guard<std::mutex> lock(mu);
    sl.valid = true;
    sl.key = k;
    sl.map = *m;
    return true;
}

// A bf16 matrix of `rows` rows of `cols` elements, `row_bytes` apart, read in
// boxes of box_cols x box_rows with the 128-byte swizzle (box_cols = 64).
// Rows past the end read as zero.
inline bool make_map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                        uint32_t box_cols, uint32_t box_rows) {
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    return encode_tiled_cached(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B);
}

// The same for a float32 matrix (box_cols = 32: 128-byte rows).
inline bool make_map_2d_f32(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                            uint32_t box_cols, uint32_t box_rows) {
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    return encode_tiled_cached(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box,
                               CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace mla
