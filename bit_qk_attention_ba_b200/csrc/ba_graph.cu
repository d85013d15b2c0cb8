// ba_graph.cu -- the forward hot path as one CUDA graph (ba_fwd_graph_*).
//
// The pre-pass (Key designs 1 and 3 of "BinaryAttention: One-Bit QK-Attention
// for Vision and Diffusion Transformers": sign bits, scales, V codes) and the
// fused forward (Key designs 1-3, Overall framework) are recorded by stream
// capture on a private stream, exactly as the two entry points queue them, so
// a step replays their kernels back to back from one graph launch instead of
// one host launch per kernel.  The capture runs in relaxed mode: the entry
// points set kernel attributes and encode tensor maps on the host while it
// records, which executes nothing on the device.
#include <new>

#include "ba_common.cuh"
#include "../../include/ba_graph.h"

struct ba_fwd_graph {
    cudaGraph_t graph;
    cudaGraphExec_t exec;
    int device;
    int kernels;
};

namespace ba {
ba_status check_stream(void* stream);
}

extern "C" {

ba_status ba_fwd_graph_create(const void* q, const void* k, const void* v, ba_dtype dt,
                              int B, int H, int N, int d,
                              uint32_t* bq, float* muq, uint32_t* bk, float* muk, int8_t* vq, float* sv,
                              int bias_kind, const float* bias, int64_t bias_ld, int grid_h, int grid_w,
                              void* workspace, int64_t workspace_bytes,
                              void* out, ba_dtype out_dt, int variant, ba_fwd_graph** graph)
{
    if (graph == nullptr) return BA_ERR_INVALID_ARG;
    *graph = nullptr;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BA_ERR_CUDA;
    // Per-device state (status word, SM count) is looked up once outside the capture.
    if (ba::device_status_ptr() == nullptr) return BA_ERR_CUDA;

    cudaStream_t cs = nullptr;
    if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return BA_ERR_CUDA;
    if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
        cudaStreamDestroy(cs);
        return BA_ERR_CUDA;
    }
    ba_status s = ba_prepass_qkv(q, k, v, dt, B, H, N, d, bq, muq, bk, muk, vq, sv, cs);
    if (s == BA_OK)
        s = ba_attention_fwd_variant(bq, muq, bk, muk, vq, sv, bias_kind, bias, bias_ld, grid_h, grid_w, B, H, N, d,
                                     workspace, workspace_bytes, out, out_dt, variant, cs);
    cudaGraph_t g = nullptr;
    const cudaError_t ec = cudaStreamEndCapture(cs, &g);   // ends the capture on every path
    cudaStreamDestroy(cs);
    if (s != BA_OK || ec != cudaSuccess || g == nullptr) {
        if (g != nullptr) cudaGraphDestroy(g);
        cudaGetLastError();
        return s != BA_OK ? s : BA_ERR_CUDA;
    }

    size_t n = 0;
    int kernels = 0;
    if (cudaGraphGetNodes(g, nullptr, &n) != cudaSuccess) {
        cudaGraphDestroy(g);
        return BA_ERR_CUDA;
    }
    if (n > 0) {
        cudaGraphNode_t* nodes = new (std::nothrow) cudaGraphNode_t[n];
        if (nodes == nullptr) {
            cudaGraphDestroy(g);
            return BA_ERR_CUDA;
        }
        bool ok = cudaGraphGetNodes(g, nodes, &n) == cudaSuccess;
        for (size_t i = 0; ok && i < n; ++i) {
            cudaGraphNodeType t;
            ok = cudaGraphNodeGetType(nodes[i], &t) == cudaSuccess;
            if (ok && t == cudaGraphNodeTypeKernel) ++kernels;
        }
        delete[] nodes;
        if (!ok) {
            cudaGraphDestroy(g);
            return BA_ERR_CUDA;
        }
    }

    cudaGraphExec_t exec = nullptr;
    if (cudaGraphInstantiate(&exec, g, 0) != cudaSuccess) {
        cudaGraphDestroy(g);
        cudaGetLastError();
        return BA_ERR_CUDA;
    }
    ba_fwd_graph* h = new (std::nothrow) ba_fwd_graph{g, exec, dev, kernels};
    if (h == nullptr) {
        cudaGraphExecDestroy(exec);
        cudaGraphDestroy(g);
        return BA_ERR_CUDA;
    }
    *graph = h;
    return BA_OK;
}

ba_status ba_fwd_graph_launch(const ba_fwd_graph* graph, void* stream)
{
    if (graph == nullptr) return BA_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BA_ERR_CUDA;
    if (dev != graph->device) return BA_ERR_INVALID_ARG;
    if (const ba_status e = ba::check_stream(stream)) return e;
    return cudaGraphLaunch(graph->exec, static_cast<cudaStream_t>(stream)) == cudaSuccess ? BA_OK : BA_ERR_CUDA;
}

int ba_fwd_graph_kernels(const ba_fwd_graph* graph)
{
    return graph == nullptr ? -1 : graph->kernels;
}

ba_status ba_fwd_graph_destroy(ba_fwd_graph* graph)
{
    if (graph == nullptr) return BA_OK;
    const bool ok = cudaGraphExecDestroy(graph->exec) == cudaSuccess && cudaGraphDestroy(graph->graph) == cudaSuccess;
    delete graph;
    return ok ? BA_OK : BA_ERR_CUDA;
}

}  // extern "C"
