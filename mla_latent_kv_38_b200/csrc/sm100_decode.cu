// Placeholder until the tcgen05 kernel lands: no shape is routed here.
#include "common.cuh"
#include "sm100_decode.h"

namespace mla {

bool sm100_supports(int, int, int) { return false; }
size_t sm100_workspace_bytes(int, int, int, int) { return 0; }
int sm100_launches(int, int, int) { return MLA_ERR_UNSUPPORTED; }
cudaError_t launch_decode_sm100(const DecodeParams&, void*, int, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace mla
