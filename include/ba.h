/*
 * ba.h -- C ABI of libba, the B200 (sm_100a) BinaryAttention forward pass.
 *
 * Method source ("BA notes"): the paper-notes page "BinaryAttention: One-Bit
 * QK-Attention for Vision and Diffusion Transformers" (CVPR 2026, arXiv
 * 2603.09582).  Sections cited below:
 *   KD1  Key design 1, Scaled Binary Representations (sign Q/K + scale mu,
 *        XNOR/popcount dot product)
 *   KD2  Key design 2, Bias Enhancement (S = mu_q mu_k s.t / sqrt(d) + b)
 *   KD3  Key design 3, Hybrid Quantization (P as u8 with scale 1/255, V as
 *        channel-wise int8, integer PV product)
 *   FW   Overall framework (tiled attention in the FlashAttention2 style)
 *
 * ba_graph.h (same conventions) declares the pre-pass + fused forward as one
 * replayable CUDA graph.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, contiguous
 *     in the layout stated and aligned to their element size; the int8 V codes
 *     and a dense bias must be 16-byte aligned (they are read by the tensor
 *     memory accelerator).  The library allocates no device memory (the fused
 *     forward's scratch space is a caller workspace, see below) and never
 *     synchronises: work is queued on `stream` (a cudaStream_t passed as
 *     void*; NULL is the legacy default stream).
 *   - Arguments are validated before anything is queued; an invalid call
 *     returns BA_ERR_INVALID_ARG (or BA_ERR_UNSUPPORTED) and queues nothing.
 *   - Work runs on the CURRENT device: the library's per-device state (status
 *     word, SM count, the static scratch of ba_attention_fwd_noalloc) is that
 *     of the device current on the calling thread, and `stream` must belong
 *     to it (BA_ERR_INVALID_ARG otherwise; BA_ERR_CUDA when the runtime has
 *     no device).  The buffers must live on that device too.  A stream that
 *     is being captured into a CUDA graph is taken to belong to the current
 *     device (the runtime cannot be asked during a capture), so every entry
 *     point may be recorded into a caller's own graph.
 *   - A launch failure reported by the CUDA runtime returns BA_ERR_CUDA.
 *   - Kernels that wait on hardware barriers give up after a bounded number of
 *     polls, record a code in a device status word and exit cleanly;
 *     ba_check_device_status() reports it (BA_ERR_DEVICE_STATUS).
 *   - Sizes: B, H, N >= 1; 1 <= d <= 128.  Tokens are [B, H, N] in that order.
 *   - Nothing throws across the ABI.
 */
#ifndef BA_H_
#define BA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BA_OK = 0,
    BA_ERR_INVALID_ARG = 1,    /* bad size, null or misaligned pointer */
    BA_ERR_UNSUPPORTED = 2,    /* valid request the library cannot serve */
    BA_ERR_CUDA = 3,           /* the CUDA runtime reported an error */
    BA_ERR_DEVICE_STATUS = 4   /* a kernel recorded a failure (see below) */
} ba_status;

typedef enum { BA_F32 = 0, BA_BF16 = 1 } ba_dtype;

/* KD2: which additive bias b_ij enters the scores. */
typedef enum {
    BA_BIAS_NONE = 0,
    BA_BIAS_DENSE = 1,     /* fp32 [H, N, ld], b_ij = bias[h][i][j]; ld >= N, ld % 4 == 0 */
    BA_BIAS_RELPOS2D = 2,  /* fp32 [H, (2 gh - 1) * (2 gw - 1)], N == gh * gw, see below */
    BA_BIAS_RELPOS2D_CLS = 3  /* fp32 [H, (2 gh - 1) * (2 gw - 1) + 3], N == gh * gw + 1, see below */
} ba_bias_kind;

/* How the binary Q.K contraction runs inside ba_attention_fwd_variant. */
typedef enum {
    BA_QK_AUTO = 0,        /* the library's fastest path for the shape (tcgen05 kind::f8f6f4 or kind::i8) */
    BA_QK_POPC = 1,        /* CUDA cores: XOR + popcount on 32-bit words */
    BA_QK_MMA_B1 = 2,      /* warp mma.sync m16n8k128 .b1 XOR-popcount; PV by mma.sync u8 x s8 */
    BA_QK_TC_I8 = 3,       /* tcgen05 kind::i8, +-1 int8 operands, s32 in TMEM */
    BA_QK_TC_F8 = 4        /* tcgen05 kind::f8f6f4, +-1 e4m3 operands, f32 in TMEM */
} ba_qk_variant;

/* Number of 32-bit words per token in the packed sign layout: ceil(d / 32). */
int ba_words(int d);

/* Row stride (bytes = int8 elements) of the int8 V layout: N rounded up to 16. */
int64_t ba_vq_ld(int N);

/*
 * KD1 -- sign-binarise Q or K and take the per-token scale.
 *   x    : [B, H, N, d] values, dtype dt (BA_F32 or BA_BF16)
 *   bits : [B, H, N, W] uint32, W = ba_words(d).  Channel c is bit c % 32 of
 *          word c / 32 (least significant bit first); the bit is 1 when
 *          x >= 0 (so -0.0 gives 1, NaN gives 0).  Unused high bits are 0.
 *   mu   : [B, H, N] fp32, mu = (sum_c |x_c|) / d, the scale that minimises
 *          || x - mu sign(x) ||^2 (one scale per token; the page says only
 *          that mu keeps the token's magnitude).
 */
ba_status ba_pack_qk(const void* x, ba_dtype dt, int B, int H, int N, int d,
                     uint32_t* bits, float* mu, void* stream);

/*
 * KD3 -- channel-wise int8 quantisation of V.
 *   v  : [B, H, N, d] values, dtype dt
 *   vq : [B, H, d, ldv] int8 with ldv = ba_vq_ld(N): CHANNEL-major, keys
 *        contiguous, so a tile of keys is a K-major operand of the PV product.
 *        vq[b][h][c][j] = clamp(round_half_even(fl32(v_jc / sv_c)), -127, 127);
 *        the columns j in [N, ldv) are written as 0.
 *   sv : [B, H, d] fp32, sv_c = fl32(max_j |v_jc| / 127) (IEEE division); an
 *        all-zero channel has sv = 0 and codes 0.
 * Inputs must be finite.
 */
ba_status ba_quant_v(const void* v, ba_dtype dt, int B, int H, int N, int d,
                     int8_t* vq, float* sv, void* stream);

/*
 * KD1 + KD3 in one call: the same outputs, bit for bit, as
 *   ba_pack_qk(q) -> bq, muq;  ba_pack_qk(k) -> bk, muk;  ba_quant_v(v) -> vq, sv
 * (layouts as above; q, k, v all [B, H, N, d] in dtype dt), with q, k, v
 * 16-byte aligned:
 *   - 128-, 144- and 256-byte tokens (bf16 d = 64, 72 or 128, fp32 d = 32, 36
 *     or 64): one launch fed by tensor copies when ba_vq_ld(N) <= 1024; longer
 *     heads take three (V's channel absmax, then Q, K and the V codes, then V's
 *     scales);
 *   - otherwise ONE launch when the int8 codes of one (b, h) fit in 100 KB of
 *     shared memory (d (ba_vq_ld(N) + 4) bytes) and d size(dt) / 16 is in
 *     {2, 4, 8, 9, 12, 16}: a CTA per (b, h) packs the head's query and key
 *     tokens, then quantises its V;
 *   - otherwise the three passes as separate launches.
 * Errors as for the separate calls.
 */
ba_status ba_prepass_qkv(const void* q, const void* k, const void* v, ba_dtype dt, int B, int H, int N, int d,
                         uint32_t* bq, float* muq, uint32_t* bk, float* muk, int8_t* vq, float* sv,
                         void* stream);

/* Kernel launches ba_prepass_qkv makes for this shape with 16-byte aligned
 * inputs (1 when it runs fused); -1 for invalid arguments. */
int ba_prepass_launches(int N, int d, ba_dtype dt);

/*
 * Bytes of device workspace the fused forward needs for this problem (0 when
 * the shape runs on the CUDA-core path, which needs none); -1 for invalid
 * sizes or bias arguments.  The workspace holds the key side staged for the
 * tensor cores: +-1 operand tiles with their key scales, and for a 2-D
 * relative-position bias with grid_w a multiple of 128 the table rows
 * reversed in four shifted copies.  It is rewritten by every call.
 */
int64_t ba_attention_workspace_bytes(int B, int H, int N, int d, int bias_kind, int grid_h, int grid_w);

/*
 * KD1-KD3 + FW -- the fused forward.  For every (b, h, i):
 *   z_ij  = s_i . t_j = d - 2 popcount(bq_i XOR bk_j)                   (KD1)
 *   S_ij  = muq_i muk_j z_ij / sqrt(d) + b_ij                            (KD2)
 *   P~_ij = exp(S_ij - m_i) with m_i = max_j S_ij, the exact row maximum,
 *   pq_ij = round(255 P~_ij) in 0..255, l_i = sum_j P~_ij (unquantised)  (KD3)
 *   O_ic  = sv_c * sum_j pq_ij vq_jc / (255 l_i)                         (KD3)
 * Inputs: bq, bk [B, H, N, W] from ba_pack_qk; muq, muk [B, H, N];
 *   vq [B, H, d, ldv] and sv [B, H, d] from ba_quant_v.
 * Bias (shared over the batch): bias_kind selects none, dense or 2-D relative
 *   position.  DENSE: bias_ld is the row stride in floats (>= N, multiple of
 *   4).  RELPOS2D: token i sits at (i / grid_w, i % grid_w), N must equal
 *   grid_h * grid_w, and b_ij = table[h][(ri - rj + grid_h - 1) *
 *   (2 grid_w - 1) + (ci - cj + grid_w - 1)].  RELPOS2D_CLS (a token set with
 *   a class token; the page names no layout for it, this is the reading
 *   taken): N must equal grid_h * grid_w + 1, token 0 is the class token and
 *   token i >= 1 sits at ((i - 1) / grid_w, (i - 1) % grid_w); each head's
 *   table is the G = (2 grid_h - 1)(2 grid_w - 1) grid entries, indexed as
 *   for RELPOS2D between patch tokens, then table[h][G] for class query ->
 *   patch key, table[h][G + 1] for patch query -> class key and
 *   table[h][G + 2] for class -> class.
 * workspace: device scratch of at least ba_attention_workspace_bytes(...)
 *   bytes, 256-byte aligned (may be NULL when that size is 0); owned by the
 *   caller, used only by work queued on `stream` by this call.  Too small a
 *   workspace returns BA_ERR_INVALID_ARG.
 * out: [B, H, N, d] in out_dt (BA_F32 or BA_BF16).
 * The keys are swept twice inside the kernel (maximum first, then P and PV),
 * so pq is quantised against the exact maximum rather than a running one;
 * fp32 arithmetic can still move a code sitting on a rounding boundary by one.
 */
ba_status ba_attention_fwd(const uint32_t* bq, const float* muq,
                           const uint32_t* bk, const float* muk,
                           const int8_t* vq, const float* sv,
                           int bias_kind, const float* bias, int64_t bias_ld,
                           int grid_h, int grid_w,
                           int B, int H, int N, int d,
                           void* workspace, int64_t workspace_bytes,
                           void* out, ba_dtype out_dt, void* stream);

/* Same computation with an explicit QK contraction path (ba_qk_variant);
 * BA_ERR_UNSUPPORTED if that path cannot serve the shape.  BA_QK_POPC and
 * BA_QK_MMA_B1 take every valid shape and ignore the workspace (it may be
 * NULL with workspace_bytes 0); the tcgen05 paths need the workspace. */
ba_status ba_attention_fwd_variant(const uint32_t* bq, const float* muq,
                                   const uint32_t* bk, const float* muk,
                                   const int8_t* vq, const float* sv,
                                   int bias_kind, const float* bias, int64_t bias_ld,
                                   int grid_h, int grid_w,
                                   int B, int H, int N, int d,
                                   void* workspace, int64_t workspace_bytes,
                                   void* out, ba_dtype out_dt, int variant, void* stream);

/*
 * ba_attention_fwd without a caller workspace: the staging goes to scratch
 * space the library owns, a static device array of 80 MiB (83886080 bytes)
 * per device, reserved when this entry point is first used.  Returns
 * BA_ERR_UNSUPPORTED when ba_attention_workspace_bytes(...) exceeds that.
 * Calls share the array: at most one may be in flight per device at a time
 * (queue them on one stream, or synchronise between them).
 */
ba_status ba_attention_fwd_noalloc(const uint32_t* bq, const float* muq,
                                   const uint32_t* bk, const float* muk,
                                   const int8_t* vq, const float* sv,
                                   int bias_kind, const float* bias, int64_t bias_ld,
                                   int grid_h, int grid_w,
                                   int B, int H, int N, int d,
                                   void* out, ba_dtype out_dt, void* stream);

/*
 * KD1-KD3 in decode shape: Nq query tokens of each (b, h) attend to an
 * Nk-token cache of the same head (the compressed KV cache the page's
 * "Related work and inspiration" section points to for LLM inference).
 *   bq [B, H, Nq, W], muq [B, H, Nq]  : ba_pack_qk of the queries (N = Nq)
 *   bk [B, H, Nk, W], muk [B, H, Nk]  : ba_pack_qk of the cached keys (N = Nk)
 *   vq [B, H, d, ba_vq_ld(Nk)], sv [B, H, d] : ba_quant_v of the cached values
 *   bias : NULL, or dense fp32 [H, Nq, bias_ld] (bias_ld >= Nk), shared over B
 *   out  : [B, H, Nq, d] in out_dt
 * 1 <= Nq <= 16.  The same arithmetic as ba_attention_fwd (exact row maximum,
 * u8 codes of P~ against it, l the sum of the unquantised P~).  The keys are
 * split over CTAs; every split quantises against the exact maximum, so the
 * splits' int32 sums add exactly.  workspace: device scratch of at least
 * ba_attention_decode_workspace_bytes(B, H, Nq, Nk, d) bytes, 256-byte
 * aligned, owned by the caller, rewritten by every call.  Two kernel
 * launches on `stream`.
 */
ba_status ba_attention_decode(const uint32_t* bq, const float* muq, int Nq,
                              const uint32_t* bk, const float* muk, const int8_t* vq, const float* sv, int Nk,
                              const float* bias, int64_t bias_ld, int B, int H, int d,
                              void* workspace, int64_t workspace_bytes, void* out, ba_dtype out_dt, void* stream);

/* Workspace bytes ba_attention_decode needs on the current device; -1 for
 * invalid sizes or when no device is available. */
int64_t ba_attention_decode_workspace_bytes(int B, int H, int Nq, int Nk, int d);

/*
 * KD4 -- the training-side backward pass (quantisation-aware training with a
 * straight-through estimator for sign; the page's "QAT + Self-Distillation"
 * key design and its "Loss and training strategy" paragraph).  Readings: every
 * quantiser -- sign, the u8 rounding of P~, the int8 rounding of V -- passes
 * its gradient straight through, the sign's only where |x| <= ste_clip
 * (INFINITY for the plain identity estimator); the scale mu = mean |x|, the
 * bias and the softmax are differentiated exactly; the row maximum is a
 * constant.  With P = P~ / l, P^ = round(255 P~) / (255 l), V^ = sv vq:
 *   dv_j  = sum_i P^_ij dO_i
 *   dS_ij = P_ij (dO_i . V^_j - dO_i . O_i)
 *   dq_ic = [|q_ic| <= ste_clip] sum_j dS_ij mu_q,i mu_k,j t_jc / sqrt(d)
 *           + sign(q_ic) / d * sum_j dS_ij mu_k,j z_ij / sqrt(d)      (dk likewise)
 *   dbias = dS summed over the batch and over every (i, j) reading an entry.
 * Inputs: q, k [B, H, N, d] raw values (dtype dt; only their signs, already in
 *   bq / bk, and |x| <= ste_clip are used); bq, muq, bk, muk, vq, sv as for
 *   ba_attention_fwd; the bias arguments as there; out: the forward output O
 *   [B, H, N, d] fp32; dout: dO [B, H, N, d] fp32.
 * Outputs (fp32): dq, dk, dv [B, H, N, d]; dbias (NULL to skip) in the bias's
 *   own shape (dense [H, N, bias_ld], columns >= N set to 0; table [H, G] or
 *   [H, G + 3]), overwritten.  The bias gradient is summed with atomics, so
 *   its last bits depend on the order of the additions.
 * workspace: at least ba_attention_bwd_workspace_bytes(B, H, N) bytes of
 *   device scratch, 256-byte aligned, owned by the caller (row statistics).
 * Runs on CUDA cores (four launches: row statistics, dq with dbias, dk, dv).
 */
ba_status ba_attention_bwd(const void* q, const void* k, ba_dtype dt,
                           const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                           const int8_t* vq, const float* sv,
                           int bias_kind, const float* bias, int64_t bias_ld, int grid_h, int grid_w,
                           int B, int H, int N, int d,
                           const float* out, const float* dout, float ste_clip,
                           void* workspace, int64_t workspace_bytes,
                           float* dq, float* dk, float* dv, float* dbias, void* stream);

/* Workspace bytes ba_attention_bwd needs; -1 for invalid sizes. */
int64_t ba_attention_bwd_workspace_bytes(int B, int H, int N);

/*
 * KD1 -- the integer binary score matrix, for checking and debugging.
 *   z : [B, H, N, N] int32, z[b][h][i][j] = d - 2 popcount(bq_i XOR bk_j).
 */
ba_status ba_scores_debug(const uint32_t* bq, const uint32_t* bk,
                          int B, int H, int N, int d, int32_t* z, void* stream);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device.  BA_OK when no kernel recorded a failure, otherwise
 * BA_ERR_DEVICE_STATUS with the recorded bits in *code (may be NULL).
 */
ba_status ba_check_device_status(void* stream, int* code);

/*
 * TESTING ONLY -- exercises the bounded waits of the tensor-core forward.
 * Runs ba_attention_fwd (no bias, the 128-key tensor-core kernel) with its
 * loader stopping before key step `starve_step` (0-based over both sweeps)
 * and every barrier wait giving up after `wait_ns` nanoseconds (1 ms .. 2 s).
 * Every copy issued before that step has been consumed when the waits give
 * up, so nothing is left in flight: the roles record their bits in the
 * device status word, release tensor memory and return; out is undefined.
 * ba_check_device_status then reports BA_ERR_DEVICE_STATUS, and the next
 * normal call runs clean.  BA_ERR_UNSUPPORTED for shapes that do not run
 * the 128-key kernel.  Not part of the method: no production path calls it.
 */
ba_status ba_test_attention_fwd_starved(const uint32_t* bq, const float* muq, const uint32_t* bk, const float* muk,
                                        const int8_t* vq, const float* sv, int B, int H, int N, int d,
                                        void* workspace, int64_t workspace_bytes, void* out, ba_dtype out_dt,
                                        int starve_step, int64_t wait_ns, void* stream);

/* Static, human-readable name of a status code. */
const char* ba_status_string(ba_status s);

#ifdef __cplusplus
}
#endif

#endif /* BA_H_ */
