// ba_noalloc.cu -- the fused forward with library-owned scratch space.
//
// ba_attention_fwd_noalloc runs the same forward as ba_attention_fwd but
// takes no workspace: the key-side staging goes to a fixed-size device array
// of this library (one per device, address looked up once per device).
// Nothing is allocated at call time.  The array lives in this translation
// unit only, so with lazy module loading a process that never calls this
// entry point does not reserve it.
#include <mutex>

#include "ba_common.cuh"

namespace ba {

int64_t attn_tc_workspace_bytes(int B, int H, int N, int d, int bias_kind, int gh, int gw);
ba_status validate_fwd(const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                       const int8_t* vq, const float* sv, int bias_kind, const float* bias, int64_t bias_ld,
                       int grid_h, int grid_w, int B, int H, int N, int d, const void* out, ba_dtype out_dt);
ba_status check_stream(void* stream);

namespace {

constexpr int64_t kStaticScratchBytes = 80ll << 20;   // 80 MiB
__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};

void* static_scratch()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
        g_scratch[dev] = p;
    }
    return g_scratch[dev];
}

}  // namespace
}  // namespace ba

extern "C" ba_status ba_attention_fwd_noalloc(const uint32_t* bq, const float* muq,
                                              const uint32_t* bk, const float* muk,
                                              const int8_t* vq, const float* sv,
                                              int bias_kind, const float* bias, int64_t bias_ld,
                                              int grid_h, int grid_w,
                                              int B, int H, int N, int d,
                                              void* out, ba_dtype out_dt, void* stream)
{
    // The same argument checks as ba_attention_fwd, before the static array
    // is looked up (which loads this file's module on first use).
    const ba_status v = ba::validate_fwd(bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, grid_h, grid_w, B, H,
                                         N, d, out, out_dt);
    if (v != BA_OK) return v;
    const int64_t need = ba_attention_workspace_bytes(B, H, N, d, bias_kind, grid_h, grid_w);
    if (need < 0) return BA_ERR_INVALID_ARG;
    if (need > ba::kStaticScratchBytes) return BA_ERR_UNSUPPORTED;
    if (const ba_status e = ba::check_stream(stream)) return e;
    void* scratch = nullptr;
    if (need > 0) {
        scratch = ba::static_scratch();
        if (!scratch) return BA_ERR_CUDA;
    }
    return ba_attention_fwd(bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, grid_h, grid_w, B, H, N, d,
                            scratch, need > 0 ? ba::kStaticScratchBytes : 0, out, out_dt, stream);
}
