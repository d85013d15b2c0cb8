/*
 * ba_graph.h -- the forward hot path of libba as one replayable CUDA graph.
 *
 * Same method sources and conventions as ba.h (which this header includes):
 * KD1-KD3 are Key designs 1-3 and FW the Overall framework of the paper-notes
 * page "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
 * Transformers".
 */
#ifndef BA_GRAPH_H_
#define BA_GRAPH_H_

#include "ba.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * KD1-KD3 + FW as one replayable step: the launches that
 *   ba_prepass_qkv(q, k, v, ...)            -> bq, muq, bk, muk, vq, sv
 *   ba_attention_fwd_variant(bq, ..., out)  -> out
 * make for these buffers, recorded once (stream capture on a stream the call
 * creates and destroys) into a CUDA graph.  ba_fwd_graph_launch then queues
 * the whole forward as ONE graph launch: its kernels run back to back with
 * no host launch per kernel.  Arguments, layouts and errors are those of the
 * two calls, whose checks run while the capture records (a capture executes
 * nothing); on any error *graph is left NULL and no work has been queued or
 * run.  BA_ERR_INVALID_ARG also for graph == NULL.  Device pointers are fixed
 * in the graph:
 * every buffer must keep its address until ba_fwd_graph_destroy, while its
 * contents may change between launches (new q, k, v every step).  The graph
 * belongs to the device current at creation and to nothing else; creation
 * queues no work on any caller stream.  Host memory for the handle and the
 * driver's graph objects are the only things allocated; no device memory.
 */
typedef struct ba_fwd_graph ba_fwd_graph;

ba_status ba_fwd_graph_create(const void* q, const void* k, const void* v, ba_dtype dt,
                              int B, int H, int N, int d,
                              uint32_t* bq, float* muq, uint32_t* bk, float* muk, int8_t* vq, float* sv,
                              int bias_kind, const float* bias, int64_t bias_ld, int grid_h, int grid_w,
                              void* workspace, int64_t workspace_bytes,
                              void* out, ba_dtype out_dt, int variant, ba_fwd_graph** graph);

/* Queue one forward step on `stream` (a stream of the graph's device, which
 * must be current).  BA_ERR_INVALID_ARG for a NULL graph or a stream of
 * another device. */
ba_status ba_fwd_graph_launch(const ba_fwd_graph* graph, void* stream);

/* Kernel launches one step of the graph makes (its kernel nodes); -1 for a
 * NULL graph. */
int ba_fwd_graph_kernels(const ba_fwd_graph* graph);

/* Release the graph and its handle (NULL is accepted).  Steps already queued
 * run to completion. */
ba_status ba_fwd_graph_destroy(ba_fwd_graph* graph);

#ifdef __cplusplus
}
#endif

#endif /* BA_GRAPH_H_ */
