// ba_attn_tc.cu -- tcgen05 tensor-core attention (placeholder until written).
#include "ba_common.cuh"

namespace ba {

bool attn_tc_supports(int, int, int, int, int) { return false; }

cudaError_t launch_attn_tc(const uint32_t*, const float*, const uint32_t*, const float*,
                           const int8_t*, const float*, int, const float*, int64_t, int, int,
                           int, int, int, int, void*, ba_dtype, int, unsigned*, cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace ba
