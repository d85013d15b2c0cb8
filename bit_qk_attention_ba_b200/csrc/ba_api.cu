// ba_api.cu -- the C ABI of libba: argument checks, dispatch, status word.
//
// Every entry point validates its arguments on the host before queueing any
// work, launches asynchronously on the caller's stream and returns a status
// code; nothing throws across the ABI and nothing is allocated (scratch space
// is the caller's workspace).
#include <mutex>

#include "ba_common.cuh"

namespace ba {

cudaError_t launch_pack(const void* x, ba_dtype dt, int64_t tokens, int d, uint32_t* bits,
                        float* mu, cudaStream_t st, int sm_count);
cudaError_t launch_quant_v(const void* v, ba_dtype dt, int B, int H, int N, int d, int8_t* vq,
                           float* sv, cudaStream_t st);
cudaError_t launch_prepass(const void* q, const void* k, const void* v, ba_dtype dt, int B, int H, int N,
                           int d, uint32_t* bq, float* muq, uint32_t* bk, float* muk, int8_t* vq, float* sv,
                           cudaStream_t st, int sm_count);
int prepass_launch_count(int N, int d, ba_dtype dt);
cudaError_t launch_scores(const uint32_t* bq, const uint32_t* bk, int B, int H, int N, int d,
                          int32_t* z, cudaStream_t st);
cudaError_t launch_attn_simt(const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                             const int8_t* vq, const float* sv, int bias_kind, const float* bias,
                             int64_t bias_ld, int gh, int gw, int B, int H, int N, int d,
                             void* out, ba_dtype out_dt, cudaStream_t st);
cudaError_t launch_attn_b1(const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                           const int8_t* vq, const float* sv, int bias_kind, const float* bias,
                           int64_t bias_ld, int gh, int gw, int B, int H, int N, int d,
                           void* out, ba_dtype out_dt, cudaStream_t st);
// Returns cudaErrorNotSupported when the tensor-core path cannot take the shape.
cudaError_t launch_attn_tc(const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                           const int8_t* vq, const float* sv, int bias_kind, const float* bias,
                           int64_t bias_ld, int gh, int gw, int B, int H, int N, int d,
                           void* workspace, int64_t workspace_bytes,
                           void* out, ba_dtype out_dt, int variant, unsigned* status, cudaStream_t st,
                           int starve_step = -1, uint64_t wait_ns = 2000000000ull);
bool attn_tc_supports(int bias_kind, int gh, int gw, int N, int d);
int64_t attn_decode_workspace_bytes(int B, int H, int Nk, int d, int sm_count);
cudaError_t launch_attn_decode(const uint32_t* bq, const float* muq, int Nq, const uint32_t* bk, const float* muk,
                               const int8_t* vq, const float* sv, int Nk, const float* bias, int64_t bias_ld,
                               int B, int H, int d, void* workspace, void* out, ba_dtype out_dt,
                               cudaStream_t st, int sm_count);
int64_t attn_tc_workspace_bytes(int B, int H, int N, int d, int bias_kind, int gh, int gw);
int64_t attn_bwd_workspace_bytes(int B, int H, int N);
cudaError_t launch_attn_bwd(const void* q, const void* k, ba_dtype dt, const uint32_t* bq, const float* muq,
                            const uint32_t* bk, const float* muk, const int8_t* vq, const float* sv, int bias_kind,
                            const float* bias, int64_t bias_ld, int gh, int gw, int B, int H, int N, int d,
                            const float* out, const float* dout, float clip, void* workspace, float* dq, float* dk,
                            float* dv, float* dbias, cudaStream_t st);

// One status word per device; kernels OR failure bits into it.
__device__ unsigned g_device_status;

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned* g_status_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

int current_device()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

// Per-device set-up, done once with the device current.
bool device_setup(int dev)
{
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_status_ptr[dev]) return true;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return false;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    g_sm_count[dev] = sms;
    g_status_ptr[dev] = static_cast<unsigned*>(p);
    return true;
}
}  // namespace

unsigned* device_status_ptr()
{
    const int dev = current_device();
    return device_setup(dev) ? g_status_ptr[dev] : nullptr;
}

static int sm_count()
{
    const int dev = current_device();
    return device_setup(dev) ? g_sm_count[dev] : 0;
}

static bool sizes_ok(int B, int H, int N, int d)
{
    return B >= 1 && H >= 1 && N >= 1 && d >= 1 && d <= 128 && (int64_t)B * H <= 65535 &&
           (int64_t)N <= (1 << 24);
}

// Non-null and aligned to `a` bytes.
static bool ptr_ok(const void* p, uintptr_t a) { return p != nullptr && aligned(p, a); }
static uintptr_t esize(ba_dtype dt) { return dt == BA_BF16 ? 2 : 4; }

static ba_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BA_OK : BA_ERR_CUDA; }

// The stream must belong to the current device: the status word, the SM
// count and any library scratch are looked up on the current device, so work
// queued on another device's stream would get the wrong ones.
// BA_ERR_CUDA when the runtime cannot say (no device), BA_ERR_INVALID_ARG
// when the stream belongs to another device.  Checked after every host-only
// argument check, just before work is queued.  A stream that is being
// captured into a CUDA graph cannot be asked for its device (the query would
// invalidate the capture), so it is taken to be the current device's.
ba_status check_stream(void* stream)
{
    int cur = 0, sdev = 0;
    if (cudaGetDevice(&cur) != cudaSuccess) return BA_ERR_CUDA;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) == cudaSuccess && cap != cudaStreamCaptureStatusNone) return BA_OK;
    cudaGetLastError();
    if (cudaStreamGetDevice(st, &sdev) != cudaSuccess) return BA_ERR_CUDA;
    return sdev == cur ? BA_OK : BA_ERR_INVALID_ARG;
}

static bool bias_ok(int kind, const float* bias, int64_t ld, int gh, int gw, int N)
{
    if (kind == BA_BIAS_NONE) return true;
    if (kind == BA_BIAS_DENSE) return ptr_ok(bias, 16) && ld >= N && ld % 4 == 0;
    if (kind == BA_BIAS_RELPOS2D)
        return ptr_ok(bias, 4) && gh >= 1 && gw >= 1 && (int64_t)gh * gw == N;
    if (kind == BA_BIAS_RELPOS2D_CLS)
        return ptr_ok(bias, 4) && gh >= 1 && gw >= 1 && (int64_t)gh * gw + 1 == N;
    return false;
}

// Every host-side check of the fused forward's arguments except the
// workspace size (which depends on the path taken).
ba_status validate_fwd(const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                       const int8_t* vq, const float* sv, int bias_kind, const float* bias, int64_t bias_ld,
                       int grid_h, int grid_w, int B, int H, int N, int d, const void* out, ba_dtype out_dt)
{
    if (!sizes_ok(B, H, N, d) || (out_dt != BA_F32 && out_dt != BA_BF16)) return BA_ERR_INVALID_ARG;
    if (!ptr_ok(bq, 4) || !ptr_ok(muq, 4) || !ptr_ok(bk, 4) || !ptr_ok(muk, 4) || !ptr_ok(vq, 16) ||
        !ptr_ok(sv, 4) || !ptr_ok(out, esize(out_dt)))
        return BA_ERR_INVALID_ARG;
    if (!bias_ok(bias_kind, bias, bias_ld, grid_h, grid_w, N)) return BA_ERR_INVALID_ARG;
    return BA_OK;
}

}  // namespace ba

using namespace ba;

extern "C" {

int ba_words(int d) { return words_for(d); }

int64_t ba_vq_ld(int N) { return round_up64(N, 16); }

const char* ba_status_string(ba_status s)
{
    switch (s) {
        case BA_OK: return "BA_OK";
        case BA_ERR_INVALID_ARG: return "BA_ERR_INVALID_ARG";
        case BA_ERR_UNSUPPORTED: return "BA_ERR_UNSUPPORTED";
        case BA_ERR_CUDA: return "BA_ERR_CUDA";
        case BA_ERR_DEVICE_STATUS: return "BA_ERR_DEVICE_STATUS";
    }
    return "BA_ERR_UNKNOWN";
}

ba_status ba_pack_qk(const void* x, ba_dtype dt, int B, int H, int N, int d,
                     uint32_t* bits, float* mu, void* stream)
{
    if (!sizes_ok(B, H, N, d) || (dt != BA_F32 && dt != BA_BF16)) return BA_ERR_INVALID_ARG;
    if (!ptr_ok(x, esize(dt)) || !ptr_ok(bits, 4) || !ptr_ok(mu, 4)) return BA_ERR_INVALID_ARG;
    if (const ba_status e = check_stream(stream)) return e;
    const int sms = sm_count();
    if (sms <= 0) return BA_ERR_CUDA;
    return from_cuda(launch_pack(x, dt, (int64_t)B * H * N, d, bits, mu,
                                 static_cast<cudaStream_t>(stream), sms));
}

ba_status ba_quant_v(const void* v, ba_dtype dt, int B, int H, int N, int d,
                     int8_t* vq, float* sv, void* stream)
{
    if (!sizes_ok(B, H, N, d) || (dt != BA_F32 && dt != BA_BF16)) return BA_ERR_INVALID_ARG;
    if (!ptr_ok(v, esize(dt)) || !ptr_ok(vq, 16) || !ptr_ok(sv, 4)) return BA_ERR_INVALID_ARG;
    if (const ba_status e = check_stream(stream)) return e;
    return from_cuda(launch_quant_v(v, dt, B, H, N, d, vq, sv, static_cast<cudaStream_t>(stream)));
}

ba_status ba_prepass_qkv(const void* q, const void* k, const void* v, ba_dtype dt, int B, int H, int N, int d,
                         uint32_t* bq, float* muq, uint32_t* bk, float* muk, int8_t* vq, float* sv, void* stream)
{
    if (!sizes_ok(B, H, N, d) || (dt != BA_F32 && dt != BA_BF16)) return BA_ERR_INVALID_ARG;
    if (!ptr_ok(q, esize(dt)) || !ptr_ok(k, esize(dt)) || !ptr_ok(v, esize(dt))) return BA_ERR_INVALID_ARG;
    if (!ptr_ok(bq, 4) || !ptr_ok(muq, 4) || !ptr_ok(bk, 4) || !ptr_ok(muk, 4) || !ptr_ok(vq, 16) ||
        !ptr_ok(sv, 4))
        return BA_ERR_INVALID_ARG;
    if (const ba_status e = check_stream(stream)) return e;
    const int sms = sm_count();
    if (sms <= 0) return BA_ERR_CUDA;
    return from_cuda(launch_prepass(q, k, v, dt, B, H, N, d, bq, muq, bk, muk, vq, sv,
                                    static_cast<cudaStream_t>(stream), sms));
}

int ba_prepass_launches(int N, int d, ba_dtype dt)
{
    if (!sizes_ok(1, 1, N, d) || (dt != BA_F32 && dt != BA_BF16)) return -1;
    return prepass_launch_count(N, d, dt);
}

ba_status ba_scores_debug(const uint32_t* bq, const uint32_t* bk, int B, int H, int N, int d,
                          int32_t* z, void* stream)
{
    if (!sizes_ok(B, H, N, d)) return BA_ERR_INVALID_ARG;
    if (!ptr_ok(bq, 4) || !ptr_ok(bk, 4) || !ptr_ok(z, 4)) return BA_ERR_INVALID_ARG;
    if (const ba_status e = check_stream(stream)) return e;
    if (ceil_div(N, 64) > 65535) return BA_ERR_UNSUPPORTED;
    return from_cuda(launch_scores(bq, bk, B, H, N, d, z, static_cast<cudaStream_t>(stream)));
}

int64_t ba_attention_workspace_bytes(int B, int H, int N, int d, int bias_kind, int grid_h, int grid_w)
{
    if (!sizes_ok(B, H, N, d)) return -1;
    if (bias_kind < BA_BIAS_NONE || bias_kind > BA_BIAS_RELPOS2D_CLS) return -1;
    if (bias_kind == BA_BIAS_RELPOS2D && (grid_h < 1 || grid_w < 1 || (int64_t)grid_h * grid_w != N)) return -1;
    if (bias_kind == BA_BIAS_RELPOS2D_CLS && (grid_h < 1 || grid_w < 1 || (int64_t)grid_h * grid_w + 1 != N))
        return -1;
    return attn_tc_workspace_bytes(B, H, N, d, bias_kind, grid_h, grid_w);
}

ba_status ba_attention_fwd_variant(const uint32_t* bq, const float* muq,
                                   const uint32_t* bk, const float* muk,
                                   const int8_t* vq, const float* sv,
                                   int bias_kind, const float* bias, int64_t bias_ld,
                                   int grid_h, int grid_w,
                                   int B, int H, int N, int d,
                                   void* workspace, int64_t workspace_bytes,
                                   void* out, ba_dtype out_dt, int variant, void* stream)
{
    const ba_status v = validate_fwd(bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, grid_h, grid_w, B, H, N, d,
                                     out, out_dt);
    if (v != BA_OK) return v;
    if (workspace_bytes < 0 || (workspace_bytes > 0 && !ptr_ok(workspace, 256))) return BA_ERR_INVALID_ARG;
    if (variant != BA_QK_AUTO && variant != BA_QK_POPC && variant != BA_QK_MMA_B1 && variant != BA_QK_TC_I8 &&
        variant != BA_QK_TC_F8)
        return BA_ERR_INVALID_ARG;
    const bool ws_needed = variant != BA_QK_MMA_B1 && variant != BA_QK_POPC &&
                           attn_tc_supports(bias_kind, grid_h, grid_w, N, d);
    if (ws_needed && workspace_bytes < attn_tc_workspace_bytes(B, H, N, d, bias_kind, grid_h, grid_w))
        return BA_ERR_INVALID_ARG;
    if (variant != BA_QK_AUTO && variant != BA_QK_POPC && variant != BA_QK_MMA_B1 && !ws_needed)
        return BA_ERR_UNSUPPORTED;
    if (const ba_status e = check_stream(stream)) return e;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (variant == BA_QK_MMA_B1)
        return from_cuda(launch_attn_b1(bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, grid_h,
                                        grid_w, B, H, N, d, out, out_dt, st));
    if (variant == BA_QK_POPC)
        return from_cuda(launch_attn_simt(bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, grid_h,
                                          grid_w, B, H, N, d, out, out_dt, st));
    const bool tc_ok = attn_tc_supports(bias_kind, grid_h, grid_w, N, d);
    if (!tc_ok) {
        if (variant != BA_QK_AUTO) return BA_ERR_UNSUPPORTED;
        return from_cuda(launch_attn_simt(bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, grid_h,
                                          grid_w, B, H, N, d, out, out_dt, st));
    }
    if (workspace_bytes < attn_tc_workspace_bytes(B, H, N, d, bias_kind, grid_h, grid_w)) return BA_ERR_INVALID_ARG;
    unsigned* status = device_status_ptr();
    if (!status) return BA_ERR_CUDA;
    const cudaError_t e = launch_attn_tc(bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, grid_h, grid_w,
                                         B, H, N, d, workspace, workspace_bytes, out, out_dt, variant, status, st);
    if (e == cudaErrorNotSupported) return BA_ERR_UNSUPPORTED;
    if (e == cudaErrorInvalidValue) return BA_ERR_INVALID_ARG;
    return from_cuda(e);
}

ba_status ba_attention_fwd(const uint32_t* bq, const float* muq,
                           const uint32_t* bk, const float* muk,
                           const int8_t* vq, const float* sv,
                           int bias_kind, const float* bias, int64_t bias_ld,
                           int grid_h, int grid_w,
                           int B, int H, int N, int d,
                           void* workspace, int64_t workspace_bytes,
                           void* out, ba_dtype out_dt, void* stream)
{
    return ba_attention_fwd_variant(bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, grid_h, grid_w,
                                    B, H, N, d, workspace, workspace_bytes, out, out_dt, BA_QK_AUTO, stream);
}

static bool decode_sizes_ok(int B, int H, int Nq, int Nk, int d)
{
    return Nq >= 1 && Nq <= 16 && sizes_ok(B, H, Nk, d);
}

int64_t ba_attention_decode_workspace_bytes(int B, int H, int Nq, int Nk, int d)
{
    if (!decode_sizes_ok(B, H, Nq, Nk, d)) return -1;
    const int sms = sm_count();
    if (sms <= 0) return -1;
    return attn_decode_workspace_bytes(B, H, Nk, d, sms);
}

ba_status ba_attention_decode(const uint32_t* bq, const float* muq, int Nq,
                              const uint32_t* bk, const float* muk, const int8_t* vq, const float* sv, int Nk,
                              const float* bias, int64_t bias_ld, int B, int H, int d,
                              void* workspace, int64_t workspace_bytes, void* out, ba_dtype out_dt, void* stream)
{
    if (!decode_sizes_ok(B, H, Nq, Nk, d) || (out_dt != BA_F32 && out_dt != BA_BF16)) return BA_ERR_INVALID_ARG;
    if (!ptr_ok(bq, 4) || !ptr_ok(muq, 4) || !ptr_ok(bk, 4) || !ptr_ok(muk, 4) || !ptr_ok(vq, 16) ||
        !ptr_ok(sv, 4) || !ptr_ok(out, esize(out_dt)) || !ptr_ok(workspace, 256))
        return BA_ERR_INVALID_ARG;
    if (bias != nullptr && (!ptr_ok(bias, 4) || bias_ld < Nk)) return BA_ERR_INVALID_ARG;
    if (const ba_status e = check_stream(stream)) return e;
    const int sms = sm_count();
    if (sms <= 0) return BA_ERR_CUDA;
    if (workspace_bytes < attn_decode_workspace_bytes(B, H, Nk, d, sms)) return BA_ERR_INVALID_ARG;
    return from_cuda(launch_attn_decode(bq, muq, Nq, bk, muk, vq, sv, Nk, bias, bias_ld, B, H, d, workspace, out,
                                        out_dt, static_cast<cudaStream_t>(stream), sms));
}

int64_t ba_attention_bwd_workspace_bytes(int B, int H, int N)
{
    if (!sizes_ok(B, H, N, 1)) return -1;
    return attn_bwd_workspace_bytes(B, H, N);
}

ba_status ba_attention_bwd(const void* q, const void* k, ba_dtype dt,
                           const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                           const int8_t* vq, const float* sv,
                           int bias_kind, const float* bias, int64_t bias_ld, int grid_h, int grid_w,
                           int B, int H, int N, int d,
                           const float* out, const float* dout, float ste_clip,
                           void* workspace, int64_t workspace_bytes,
                           float* dq, float* dk, float* dv, float* dbias, void* stream)
{
    if (!sizes_ok(B, H, N, d) || (dt != BA_F32 && dt != BA_BF16)) return BA_ERR_INVALID_ARG;
    if (!ptr_ok(q, esize(dt)) || !ptr_ok(k, esize(dt)) || !ptr_ok(bq, 4) || !ptr_ok(muq, 4) || !ptr_ok(bk, 4) ||
        !ptr_ok(muk, 4) || !ptr_ok(vq, 1) || !ptr_ok(sv, 4) || !ptr_ok(out, 4) || !ptr_ok(dout, 4) ||
        !ptr_ok(dq, 4) || !ptr_ok(dk, 4) || !ptr_ok(dv, 4) || (dbias != nullptr && !ptr_ok(dbias, 4)))
        return BA_ERR_INVALID_ARG;
    if (bias_kind == BA_BIAS_DENSE ? !(ptr_ok(bias, 4) && bias_ld >= N) : !bias_ok(bias_kind, bias, bias_ld, grid_h, grid_w, N))
        return BA_ERR_INVALID_ARG;
    if (!(ste_clip >= 0.f)) return BA_ERR_INVALID_ARG;            // NaN or negative
    if (!ptr_ok(workspace, 256) || workspace_bytes < attn_bwd_workspace_bytes(B, H, N)) return BA_ERR_INVALID_ARG;
    if (const ba_status e = check_stream(stream)) return e;
    return from_cuda(launch_attn_bwd(q, k, dt, bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, grid_h, grid_w,
                                     B, H, N, d, out, dout, ste_clip, workspace, dq, dk, dv, dbias,
                                     static_cast<cudaStream_t>(stream)));
}

ba_status ba_test_attention_fwd_starved(const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                                        const int8_t* vq, const float* sv, int B, int H, int N, int d,
                                        void* workspace, int64_t workspace_bytes, void* out, ba_dtype out_dt,
                                        int starve_step, int64_t wait_ns, void* stream)
{
    const ba_status v = validate_fwd(bq, muq, bk, muk, vq, sv, BA_BIAS_NONE, nullptr, 0, 0, 0, B, H, N, d, out,
                                     out_dt);
    if (v != BA_OK) return v;
    if (starve_step < 0 || wait_ns < 1000000 || wait_ns > 2000000000ll) return BA_ERR_INVALID_ARG;
    if (!attn_tc_supports(BA_BIAS_NONE, 0, 0, N, d)) return BA_ERR_UNSUPPORTED;
    if (!ptr_ok(workspace, 256) || workspace_bytes < attn_tc_workspace_bytes(B, H, N, d, BA_BIAS_NONE, 0, 0))
        return BA_ERR_INVALID_ARG;
    if (const ba_status e = check_stream(stream)) return e;
    unsigned* status = device_status_ptr();
    if (!status) return BA_ERR_CUDA;
    const cudaError_t e = launch_attn_tc(bq, muq, bk, muk, vq, sv, BA_BIAS_NONE, nullptr, 0, 0, 0, B, H, N, d,
                                         workspace, workspace_bytes, out, out_dt, BA_QK_AUTO, status,
                                         static_cast<cudaStream_t>(stream), starve_step, (uint64_t)wait_ns);
    if (e == cudaErrorNotSupported) return BA_ERR_UNSUPPORTED;
    return from_cuda(e);
}

ba_status ba_check_device_status(void* stream, int* code)
{
    unsigned* p = device_status_ptr();
    if (!p) return BA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned host = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess) return BA_ERR_CUDA;
    if (cudaMemcpy(&host, p, sizeof(host), cudaMemcpyDeviceToHost) != cudaSuccess) return BA_ERR_CUDA;
    if (host != 0 && cudaMemset(p, 0, sizeof(unsigned)) != cudaSuccess) return BA_ERR_CUDA;
    if (code) *code = (int)host;
    return host ? BA_ERR_DEVICE_STATUS : BA_OK;
}

}  // extern "C"
