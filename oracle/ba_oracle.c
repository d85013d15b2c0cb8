/*
 * ba_oracle.c -- plain CPU oracle for the BinaryAttention forward pass and its
 * training-side backward pass (straight-through estimators).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library under bit_qk_attention_ba_b200/) never calls it, and this
 * file shares no code, header, table or helper with that path.
 *
 * Source cited throughout ("BA notes"): the paper-notes page
 *   "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
 *    Transformers" (CVPR 2026, arXiv 2603.09582),
 * sections "Key design 1: Scaled Binary Representations" (KD1),
 * "Key design 2: Bias Enhancement" (KD2), "Key design 3: Hybrid
 * Quantization" (KD3) and "Overall framework" (FA2 tiled attention).
 *
 * Everything is written for clarity, not speed: straight loops, double
 * precision, exact row maximum, int64 sums.  The only decisions taken in a
 * lower precision are the ones that produce integers the CUDA path must match
 * bit for bit (the int8 V codes): those are taken in IEEE fp32, the precision
 * of the kernel, as the parity rules require.
 *
 * Readings where the page is silent (each also listed in the design notes):
 *   - sign(x) is +1 when x >= 0 (so -0.0 -> +1) and -1 otherwise; NaN -> -1.
 *   - mu is one scale per token: mean |x| over the d channels.  This is the
 *     closed-form minimiser of || x - mu * sign(x) ||^2.
 *   - sqrt(d) uses the true head dimension d, never the padded width.
 *   - P~ = exp(S - m) with m the exact row maximum; pq = round-half-even(255 P~);
 *     the row denominator l is the sum of the UNQUANTISED P~.
 *   - V is quantised per (batch, head, channel) over the N tokens: symmetric
 *     absmax / 127, IEEE fp32 division, round-half-even, clamp to [-127, 127];
 *     an all-zero channel gets scale 0 and codes 0.
 *   - The bias is shared over the batch.  Dense: b[h][i][j] at row stride ld.
 *     2-D relative position: token i sits at (i / gw, i % gw); the table index
 *     is (ri - rj + gh - 1) * (2 gw - 1) + (ci - cj + gw - 1).
 *   - 2-D relative position with a class token (N = gh gw + 1): token 0 is the
 *     class token and token i >= 1 sits at ((i - 1) / gw, (i - 1) % gw).  The
 *     page names a relative-position bias but no class token; each head's
 *     table holds the G = (2 gh - 1)(2 gw - 1) grid entries, then three learned
 *     scalars: entry G for class query -> patch key, G + 1 for patch query ->
 *     class key, G + 2 for class -> class.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* Number of 32-bit words that hold d sign bits. */
int bao_words(int d) { return (d + 31) / 32; }

/* KD1: sign of one value, as the +-1 integer the dot product uses. */
static int sign_pm1(float x) { return (x >= 0.0f) ? +1 : -1; }

/*
 * KD1 (Scaled Binary Representations): sign-binarise each token and keep its
 * magnitude as a per-token scale.
 *   x    : [T, d] fp32 values (T = B*H*N tokens, channel fastest)
 *   bits : [T, W] words, W = ceil(d/32); channel c -> word c/32, bit c%32
 *          (least significant bit first); bit = 1 when sign is +1; unused
 *          high bits of the last word are 0.
 *   mu   : [T] mean |x| in double.
 */
void bao_pack(const float* x, int64_t T, int d, uint32_t* bits, double* mu)
{
    const int W = bao_words(d);
    for (int64_t t = 0; t < T; ++t) {
        const float* row = x + t * d;
        for (int w = 0; w < W; ++w) {
            uint32_t word = 0;
            for (int b = 0; b < 32; ++b) {
                int c = 32 * w + b;
                if (c < d && sign_pm1(row[c]) == +1) word |= (1u << b);
            }
            bits[t * W + w] = word;
        }
        double s = 0.0;
        for (int c = 0; c < d; ++c) s += fabs((double)row[c]);
        mu[t] = s / (double)d;
    }
}

/* KD1, definition form: s.t over +-1 vectors taken straight from the values. */
int32_t bao_dot_pm1(const float* q, const float* k, int d)
{
    int32_t z = 0;
    for (int c = 0; c < d; ++c) z += sign_pm1(q[c]) * sign_pm1(k[c]);
    return z;
}

/* Count set bits one at a time (no builtin, so it can be read by eye). */
static int count_bits(uint32_t v)
{
    int n = 0;
    for (int b = 0; b < 32; ++b) n += (int)((v >> b) & 1u);
    return n;
}

/*
 * KD1, XNOR/popcount form: s.t = d - 2 * hamming(bits_q, bits_k).  Padding
 * bits are zero in both operands, so they add nothing to the Hamming distance.
 */
int32_t bao_dot_bits(const uint32_t* a, const uint32_t* b, int d)
{
    const int W = bao_words(d);
    int ham = 0;
    for (int w = 0; w < W; ++w) ham += count_bits(a[w] ^ b[w]);
    return (int32_t)(d - 2 * ham);
}

/* Integer score matrix z[bh][i][j] = s_i . t_j for every (batch, head). */
void bao_scores(const uint32_t* bq, const uint32_t* bk, int64_t BH, int N, int d,
                int32_t* z)
{
    const int W = bao_words(d);
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int i = 0; i < N; ++i)
            for (int j = 0; j < N; ++j)
                z[(bh * N + i) * (int64_t)N + j] =
                    bao_dot_bits(bq + (bh * N + i) * W, bk + (bh * N + j) * W, d);
}

/* The same for a block of rows: z[r][j] = s_(rows[r]) . t_j for one head,
 * bq and bk pointing at that head's [N, W] bits. */
void bao_scores_rows(const uint32_t* bq, const uint32_t* bk, int N, int d,
                     const int32_t* rows, int n_rows, int32_t* z)
{
    const int W = bao_words(d);
    for (int r = 0; r < n_rows; ++r)
        for (int j = 0; j < N; ++j)
            z[(int64_t)r * N + j] = bao_dot_bits(bq + (int64_t)rows[r] * W, bk + (int64_t)j * W, d);
}

/* KD2 (Bias Enhancement): the additive bias b_ij of head h. */
double bao_bias_value(int kind, const float* bias, int64_t ld, int h, int N,
                      int gh, int gw, int i, int j)
{
    if (kind == 1) return (double)bias[((int64_t)h * N + i) * ld + j];
    if (kind == 2) {
        int ri = i / gw, ci = i % gw, rj = j / gw, cj = j % gw;
        int64_t per_head = (int64_t)(2 * gh - 1) * (2 * gw - 1);
        int64_t idx = (int64_t)(ri - rj + gh - 1) * (2 * gw - 1) + (ci - cj + gw - 1);
        return (double)bias[(int64_t)h * per_head + idx];
    }
    if (kind == 3) {
        int64_t grid = (int64_t)(2 * gh - 1) * (2 * gw - 1);
        const float* table = bias + (int64_t)h * (grid + 3);
        if (i == 0 && j == 0) return (double)table[grid + 2];   /* class -> class */
        if (i == 0) return (double)table[grid];                 /* class query -> patch key */
        if (j == 0) return (double)table[grid + 1];             /* patch query -> class key */
        int pi = i - 1, pj = j - 1;
        int ri = pi / gw, ci = pi % gw, rj = pj / gw, cj = pj % gw;
        int64_t idx = (int64_t)(ri - rj + gh - 1) * (2 * gw - 1) + (ci - cj + gw - 1);
        return (double)table[idx];
    }
    return 0.0;
}

/*
 * KD3 (Hybrid Quantization), V side: channel-wise symmetric int8.
 *   v  : [BH, N, d] fp32
 *   vq : [BH, N, d] int8 codes (natural layout; the CUDA path's own layout is
 *        its business, the tests rearrange)
 *   sv : [BH, d] fp32 scales, sv = fl32(absmax / 127)
 * The code of an element is round-half-even(fl32(v / sv)), clamped to +-127.
 */
void bao_quant_v(const float* v, int64_t BH, int N, int d, int8_t* vq, float* sv)
{
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int c = 0; c < d; ++c) {
            float a = 0.0f;
            for (int n = 0; n < N; ++n) {
                float m = fabsf(v[(bh * N + n) * d + c]);
                if (m > a) a = m;
            }
            volatile float s = a / 127.0f;   /* one IEEE fp32 division */
            sv[bh * d + c] = s;
            for (int n = 0; n < N; ++n) {
                int q = 0;
                if (s != 0.0f) {
                    volatile float r = v[(bh * N + n) * d + c] / s;
                    float rq = nearbyintf(r);  /* default mode: half to even */
                    if (rq > 127.0f) rq = 127.0f;
                    if (rq < -127.0f) rq = -127.0f;
                    q = (int)rq;
                }
                vq[(bh * N + n) * d + c] = (int8_t)q;
            }
        }
    }
}

/*
 * The whole forward for query rows [row_lo, row_hi) of one (batch, head) bh:
 *   S_ij  = muq_i * muk_j * (s_i . t_j) / sqrt(d) + b_ij          (KD2)
 *   m_i   = max_j S_ij                                             (exact)
 *   P~_ij = exp(S_ij - m_i),  l_i = sum_j P~_ij
 *   pq_ij = round-half-even(255 * P~_ij)  in 0..255                (KD3)
 *   O_ic  = sv_c * sum_j pq_ij * vq_jc / (255 * l_i)               (KD3)
 * Inputs use the layouts above (bits [BH,N,W], mu [BH,N], vq [BH,N,d],
 * sv [BH,d]).  out receives (row_hi - row_lo) rows of d doubles.  pq_out,
 * l_out and m_out are optional (NULL to skip) and receive the same rows.
 */
void bao_attention_rows(const uint32_t* bq, const double* muq,
                        const uint32_t* bk, const double* muk,
                        const int8_t* vq, const float* sv,
                        int bias_kind, const float* bias, int64_t ld, int gh, int gw,
                        int H, int N, int d, int64_t bh, int row_lo, int row_hi,
                        double* out, uint8_t* pq_out, double* l_out, double* m_out)
{
    const int W = bao_words(d);
    const int h = (int)(bh % H);
    const double rsd = sqrt((double)d);
    double* S = (double*)malloc(sizeof(double) * (size_t)N);
    int* pq = (int*)malloc(sizeof(int) * (size_t)N);

    for (int i = row_lo; i < row_hi; ++i) {
        const uint32_t* qi = bq + (bh * N + i) * W;
        for (int j = 0; j < N; ++j) {
            int32_t z = bao_dot_bits(qi, bk + (bh * N + j) * W, d);
            S[j] = muq[bh * N + i] * muk[bh * N + j] * (double)z / rsd
                 + bao_bias_value(bias_kind, bias, ld, h, N, gh, gw, i, j);
        }
        double m = S[0];
        for (int j = 1; j < N; ++j) if (S[j] > m) m = S[j];
        double l = 0.0;
        for (int j = 0; j < N; ++j) {
            double p = exp(S[j] - m);
            l += p;
            pq[j] = (int)nearbyint(255.0 * p);
        }
        int r = i - row_lo;
        for (int c = 0; c < d; ++c) {
            int64_t acc = 0;
            for (int j = 0; j < N; ++j) acc += (int64_t)pq[j] * vq[(bh * N + j) * d + c];
            out[(int64_t)r * d + c] = (double)sv[bh * d + c] * (double)acc / (255.0 * l);
        }
        if (pq_out) for (int j = 0; j < N; ++j) pq_out[(int64_t)r * N + j] = (uint8_t)pq[j];
        if (l_out) l_out[r] = l;
        if (m_out) m_out[r] = m;
    }
    free(S);
    free(pq);
}

/*
 * Decode-shaped forward: Nq query tokens of each (batch, head) attend to the
 * Nk cached key / value tokens of the same head (Nq and Nk independent).  The
 * steps are those of bao_attention_rows:
 *   S_ij  = muq_i * muk_j * (s_i . t_j) / sqrt(d) + b_ij          (KD2)
 *   m_i   = max_j S_ij,  P~_ij = exp(S_ij - m_i),  l_i = sum_j P~_ij
 *   pq_ij = round-half-even(255 * P~_ij)                           (KD3)
 *   O_ic  = sv_c * sum_j pq_ij * vq_jc / (255 * l_i)               (KD3)
 * bq [BH, Nq, W], muq [BH, Nq], bk [BH, Nk, W], muk [BH, Nk], vq [BH, Nk, d],
 * sv [BH, d]; bias kind 0 (none) or 1 (dense: b_ij = bias[h][i][j] at row
 * stride ld >= Nk, shared over the batch).  out [BH, Nq, d] doubles.
 */
void bao_attention_decode(const uint32_t* bq, const double* muq,
                          const uint32_t* bk, const double* muk,
                          const int8_t* vq, const float* sv,
                          int bias_kind, const float* bias, int64_t ld,
                          int64_t BH, int H, int Nq, int Nk, int d, double* out)
{
    const int W = bao_words(d);
    const double rsd = sqrt((double)d);
    double* S = (double*)malloc(sizeof(double) * (size_t)Nk);
    int* pq = (int*)malloc(sizeof(int) * (size_t)Nk);
    for (int64_t bh = 0; bh < BH; ++bh) {
        const int h = (int)(bh % H);
        for (int i = 0; i < Nq; ++i) {
            const uint32_t* qi = bq + (bh * Nq + i) * W;
            for (int j = 0; j < Nk; ++j) {
                int32_t z = bao_dot_bits(qi, bk + (bh * Nk + j) * W, d);
                double b = (bias_kind == 1) ? (double)bias[((int64_t)h * Nq + i) * ld + j] : 0.0;
                S[j] = muq[bh * Nq + i] * muk[bh * Nk + j] * (double)z / rsd + b;
            }
            double m = S[0];
            for (int j = 1; j < Nk; ++j) if (S[j] > m) m = S[j];
            double l = 0.0;
            for (int j = 0; j < Nk; ++j) {
                double p = exp(S[j] - m);
                l += p;
                pq[j] = (int)nearbyint(255.0 * p);
            }
            for (int c = 0; c < d; ++c) {
                int64_t acc = 0;
                for (int j = 0; j < Nk; ++j) acc += (int64_t)pq[j] * vq[(bh * Nk + j) * d + c];
                out[(bh * Nq + i) * d + c] = (double)sv[bh * d + c] * (double)acc / (255.0 * l);
            }
        }
    }
    free(S);
    free(pq);
}

/* ---- threaded driver over independent (batch, head, row-block) units ---- */

typedef struct {
    const uint32_t* bq; const double* muq; const uint32_t* bk; const double* muk;
    const int8_t* vq; const float* sv;
    int bias_kind; const float* bias; int64_t ld; int gh, gw;
    int H, N, d; int64_t BH;
    double* out;
    int row_lo, row_hi;           /* query rows computed in every head */
    int64_t n_units; int rows_per_unit;
    int64_t next;                 /* next unit to take, guarded by lock */
    pthread_mutex_t lock;
} fwd_job;

static void* fwd_worker(void* arg)
{
    fwd_job* J = (fwd_job*)arg;
    int span = J->row_hi - J->row_lo;
    int blocks = (span + J->rows_per_unit - 1) / J->rows_per_unit;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t u = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (u >= J->n_units) break;
        int64_t bh = u / blocks;
        int lo = J->row_lo + (int)(u % blocks) * J->rows_per_unit;
        int hi = lo + J->rows_per_unit < J->row_hi ? lo + J->rows_per_unit : J->row_hi;
        bao_attention_rows(J->bq, J->muq, J->bk, J->muk, J->vq, J->sv,
                           J->bias_kind, J->bias, J->ld, J->gh, J->gw,
                           J->H, J->N, J->d, bh, lo, hi,
                           J->out + (bh * span + (lo - J->row_lo)) * J->d, NULL, NULL, NULL);
    }
    return NULL;
}

/*
 * Threaded forward of query rows [row_lo, row_hi) in heads [0, n_heads):
 * out [n_heads, row_hi - row_lo, d] doubles.  nthreads <= 0 uses every online
 * core.  Returns the number of threads used.
 */
int bao_attention_fwd_rows(const uint32_t* bq, const double* muq,
                           const uint32_t* bk, const double* muk,
                           const int8_t* vq, const float* sv,
                           int bias_kind, const float* bias, int64_t ld, int gh, int gw,
                           int64_t n_heads, int H, int N, int d, int row_lo, int row_hi,
                           double* out, int nthreads)
{
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    fwd_job J;
    memset(&J, 0, sizeof(J));
    J.bq = bq; J.muq = muq; J.bk = bk; J.muk = muk; J.vq = vq; J.sv = sv;
    J.bias_kind = bias_kind; J.bias = bias; J.ld = ld; J.gh = gh; J.gw = gw;
    J.H = H; J.N = N; J.d = d; J.BH = n_heads; J.out = out;
    J.row_lo = row_lo; J.row_hi = row_hi;
    J.rows_per_unit = 16;
    J.n_units = J.BH * ((row_hi - row_lo + J.rows_per_unit - 1) / J.rows_per_unit);
    J.next = 0;
    pthread_mutex_init(&J.lock, NULL);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, fwd_worker, &J);
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return nthreads;
}

/* Full forward over all B*H heads, out [BH, N, d] doubles. */
int bao_attention_fwd(const uint32_t* bq, const double* muq,
                      const uint32_t* bk, const double* muk,
                      const int8_t* vq, const float* sv,
                      int bias_kind, const float* bias, int64_t ld, int gh, int gw,
                      int B, int H, int N, int d, double* out, int nthreads)
{
    return bao_attention_fwd_rows(bq, muq, bk, muk, vq, sv, bias_kind, bias, ld, gh, gw,
                                  (int64_t)B * H, H, N, d, 0, N, out, nthreads);
}

/* ---- training side: the backward pass with straight-through estimators ----
 *
 * Source: Key design 4 of the BA notes (QAT + self-distillation; "Loss and
 * training strategy"): training applies sign quantisation to Q and K in the
 * forward pass and approximates its gradient in the backward pass with a
 * straight-through estimator (STE).  The page says nothing more, so the
 * readings taken here (also listed in the design notes) are:
 *   - every quantiser passes its gradient straight through: sign(x) (optionally
 *     clipped, d sign(x)/dx := [|x| <= clip], clip = +inf for the plain
 *     identity), the u8 rounding of P~ and the int8 rounding of V;
 *   - everything else is differentiated exactly: the per-token scale
 *     mu = mean |x| (d mu / d x_c = sign(x_c) / d, with sign(0) = +1 as in the
 *     forward), the product with sqrt(d), the bias, the softmax;
 *   - the row maximum m is a constant of the backward (softmax is invariant
 *     to it), as in FlashAttention-style backward passes;
 *   - with pq the rounded codes, the forward is O = (pq / 255) V^ / l with
 *     l = sum_j P~ unquantised, so reverse-mode differentiation gives
 *       dV^_j = sum_i P^_ij dO_i                  (P^ = pq / (255 l))
 *       dS_ij = P_ij (dO_i . V^_j - dO_i . O_i)   (P = P~ / l, O the forward output)
 *     the quantised P^ where the product used it, the unquantised softmax
 *     Jacobian through the straight-through rounding.
 * Chain to the inputs (KD2: S = mu_q mu_k s.t / sqrt(d) + b):
 *   dz_ij   = dS_ij mu_q,i mu_k,j / sqrt(d)
 *   dmu_q,i = sum_j dS_ij mu_k,j z_ij / sqrt(d);  dmu_k,j likewise over i
 *   ds_i    = sum_j dz_ij t_j;   dt_j = sum_i dz_ij s_i
 *   dq_ic   = ds_ic [|q_ic| <= clip] + dmu_q,i sign(q_ic) / d;  dk likewise
 *   db_ij  += dS_ij (a bias shared over the batch sums over it)
 */

/*
 * The differentiable core for one (batch, head), on continuous inputs:
 *   S_ij = muq_i muk_j (s_i . t_j) / sqrt(d) + bias_ij,  P~ = exp(S - m),
 *   l_i = sum_j P~_ij,  O_i = sum_j W_ij vh_j  with W = P~ / l (quantise_p = 0)
 *   or W = round(255 P~) / (255 l) (quantise_p = 1).
 * s, t [N, d] and vh [N, d] are arbitrary reals here (for the method s, t are
 * the +-1 signs and vh the dequantised values); bias [N, N] (row stride N) is
 * the head's bias, or NULL.  Given dO [N, d] it returns O and the gradients
 * ds, dt, dvh [N, d], dmuq, dmuk [N] and dbias [N, N] (each may be NULL).
 */
void bao_bwd_core(const double* s, const double* t, const double* muq, const double* muk,
                  const double* vh, const double* bias, int N, int d, int quantise_p,
                  const double* dO, double* O, double* ds, double* dt, double* dvh,
                  double* dmuq, double* dmuk, double* dbias)
{
    const double rsd = sqrt((double)d);
    double* z = (double*)malloc(sizeof(double) * (size_t)N * N);
    double* P = (double*)malloc(sizeof(double) * (size_t)N * N);   /* P~ / l */
    double* W = (double*)malloc(sizeof(double) * (size_t)N * N);   /* what the product used */
    double* Oi = (double*)malloc(sizeof(double) * (size_t)N * d);
    double* dS = (double*)malloc(sizeof(double) * (size_t)N * N);

    for (int i = 0; i < N; ++i) {
        double m = -INFINITY;
        for (int j = 0; j < N; ++j) {
            double zz = 0.0;
            for (int c = 0; c < d; ++c) zz += s[(int64_t)i * d + c] * t[(int64_t)j * d + c];
            z[(int64_t)i * N + j] = zz;
            double S = muq[i] * muk[j] * zz / rsd + (bias ? bias[(int64_t)i * N + j] : 0.0);
            P[(int64_t)i * N + j] = S;
            if (S > m) m = S;
        }
        double l = 0.0;
        for (int j = 0; j < N; ++j) {
            double e = exp(P[(int64_t)i * N + j] - m);
            P[(int64_t)i * N + j] = e;
            l += e;
        }
        for (int j = 0; j < N; ++j) {
            double e = P[(int64_t)i * N + j];
            W[(int64_t)i * N + j] = quantise_p ? nearbyint(255.0 * e) / (255.0 * l) : e / l;
            P[(int64_t)i * N + j] = e / l;
        }
        for (int c = 0; c < d; ++c) {
            double o = 0.0;
            for (int j = 0; j < N; ++j) o += W[(int64_t)i * N + j] * vh[(int64_t)j * d + c];
            Oi[(int64_t)i * d + c] = o;
        }
    }
    /* dS_ij = P_ij (dO_i . vh_j - dO_i . O_i) */
    for (int i = 0; i < N; ++i) {
        double D = 0.0;
        for (int c = 0; c < d; ++c) D += dO[(int64_t)i * d + c] * Oi[(int64_t)i * d + c];
        for (int j = 0; j < N; ++j) {
            double dp = 0.0;
            for (int c = 0; c < d; ++c) dp += dO[(int64_t)i * d + c] * vh[(int64_t)j * d + c];
            dS[(int64_t)i * N + j] = P[(int64_t)i * N + j] * (dp - D);
        }
    }
    if (O) memcpy(O, Oi, sizeof(double) * (size_t)N * d);
    if (dvh)
        for (int j = 0; j < N; ++j)
            for (int c = 0; c < d; ++c) {
                double g = 0.0;
                for (int i = 0; i < N; ++i) g += W[(int64_t)i * N + j] * dO[(int64_t)i * d + c];
                dvh[(int64_t)j * d + c] = g;
            }
    if (dbias)
        for (int64_t e = 0; e < (int64_t)N * N; ++e) dbias[e] = dS[e];
    if (dmuq)
        for (int i = 0; i < N; ++i) {
            double g = 0.0;
            for (int j = 0; j < N; ++j) g += dS[(int64_t)i * N + j] * muk[j] * z[(int64_t)i * N + j] / rsd;
            dmuq[i] = g;
        }
    if (dmuk)
        for (int j = 0; j < N; ++j) {
            double g = 0.0;
            for (int i = 0; i < N; ++i) g += dS[(int64_t)i * N + j] * muq[i] * z[(int64_t)i * N + j] / rsd;
            dmuk[j] = g;
        }
    if (ds)
        for (int i = 0; i < N; ++i)
            for (int c = 0; c < d; ++c) {
                double g = 0.0;
                for (int j = 0; j < N; ++j)
                    g += dS[(int64_t)i * N + j] * muq[i] * muk[j] / rsd * t[(int64_t)j * d + c];
                ds[(int64_t)i * d + c] = g;
            }
    if (dt)
        for (int j = 0; j < N; ++j)
            for (int c = 0; c < d; ++c) {
                double g = 0.0;
                for (int i = 0; i < N; ++i)
                    g += dS[(int64_t)i * N + j] * muq[i] * muk[j] / rsd * s[(int64_t)i * d + c];
                dt[(int64_t)j * d + c] = g;
            }
    free(z); free(P); free(W); free(Oi); free(dS);
}

/*
 * The whole backward with straight-through estimators, from the raw inputs:
 *   q, k, v [BH, N, d] fp32 values; bias as for bao_bias_value (kind 0..3);
 *   dO [BH, N, d].  quantise = 1 runs the method (sign Q/K, u8 P, int8 V);
 *   quantise = 0 keeps the sign of Q/K but uses P unrounded and V itself.
 *   ste_clip: the sign's gradient passes where |x| <= ste_clip (+inf: always).
 * Outputs dq, dk, dv [BH, N, d]; O [BH, N, d] (the forward output, may be
 * NULL); dbias (may be NULL): dense [H, N, ld] (entries j >= N untouched), or
 * for the relative-position kinds the table's shape [H, G (+3)] -- summed
 * over the batch and over every (i, j) that reads an entry.  dbias is
 * overwritten.
 */
void bao_attention_bwd(const float* q, const float* k, const float* v,
                       int bias_kind, const float* bias, int64_t ld, int gh, int gw,
                       int B, int H, int N, int d, const double* dO,
                       double ste_clip, int quantise,
                       double* dq, double* dk, double* dv, double* O, double* dbias)
{
    const int64_t BH = (int64_t)B * H;
    const size_t Nd = (size_t)N * d;
    double* s = (double*)malloc(sizeof(double) * Nd);
    double* t = (double*)malloc(sizeof(double) * Nd);
    double* vh = (double*)malloc(sizeof(double) * Nd);
    double* muq = (double*)malloc(sizeof(double) * (size_t)N);
    double* muk = (double*)malloc(sizeof(double) * (size_t)N);
    double* b = bias_kind ? (double*)malloc(sizeof(double) * (size_t)N * N) : NULL;
    double* ds = (double*)malloc(sizeof(double) * Nd);
    double* dt = (double*)malloc(sizeof(double) * Nd);
    double* dmuq = (double*)malloc(sizeof(double) * (size_t)N);
    double* dmuk = (double*)malloc(sizeof(double) * (size_t)N);
    double* db = bias_kind ? (double*)malloc(sizeof(double) * (size_t)N * N) : NULL;
    int8_t* vq = (int8_t*)malloc(Nd);
    float* sv = (float*)malloc(sizeof(float) * (size_t)d);

    if (dbias && bias_kind) {
        int64_t per_head = 0;
        if (bias_kind == 1) per_head = (int64_t)N * ld;
        if (bias_kind == 2) per_head = (int64_t)(2 * gh - 1) * (2 * gw - 1);
        if (bias_kind == 3) per_head = (int64_t)(2 * gh - 1) * (2 * gw - 1) + 3;
        for (int64_t e = 0; e < (int64_t)H * per_head; ++e) dbias[e] = 0.0;
    }
    for (int64_t bh = 0; bh < BH; ++bh) {
        const int h = (int)(bh % H);
        const float* qh = q + bh * (int64_t)Nd;
        const float* kh = k + bh * (int64_t)Nd;
        const float* vhd = v + bh * (int64_t)Nd;
        for (int i = 0; i < N; ++i) {
            double aq = 0.0, ak = 0.0;
            for (int c = 0; c < d; ++c) {
                s[(int64_t)i * d + c] = sign_pm1(qh[(int64_t)i * d + c]);
                t[(int64_t)i * d + c] = sign_pm1(kh[(int64_t)i * d + c]);
                aq += fabs((double)qh[(int64_t)i * d + c]);
                ak += fabs((double)kh[(int64_t)i * d + c]);
            }
            muq[i] = aq / d;
            muk[i] = ak / d;
        }
        if (quantise) {
            bao_quant_v(vhd, 1, N, d, vq, sv);
            for (size_t e = 0; e < Nd; ++e) vh[e] = (double)sv[e % d] * (double)vq[e];
        } else {
            for (size_t e = 0; e < Nd; ++e) vh[e] = (double)vhd[e];
        }
        if (b)
            for (int i = 0; i < N; ++i)
                for (int j = 0; j < N; ++j)
                    b[(int64_t)i * N + j] = bao_bias_value(bias_kind, bias, ld, h, N, gh, gw, i, j);
        bao_bwd_core(s, t, muq, muk, vh, b, N, d, quantise, dO + bh * (int64_t)Nd,
                     O ? O + bh * (int64_t)Nd : NULL, ds, dt, dv + bh * (int64_t)Nd, dmuq, dmuk, db);
        for (int i = 0; i < N; ++i)
            for (int c = 0; c < d; ++c) {
                const int64_t e = (int64_t)i * d + c;
                const double xq = qh[e], xk = kh[e];
                dq[bh * (int64_t)Nd + e] = (fabs(xq) <= ste_clip ? ds[e] : 0.0) + dmuq[i] * s[e] / d;
                dk[bh * (int64_t)Nd + e] = (fabs(xk) <= ste_clip ? dt[e] : 0.0) + dmuk[i] * t[e] / d;
            }
        if (dbias && db) {
            for (int i = 0; i < N; ++i)
                for (int j = 0; j < N; ++j) {
                    const double g = db[(int64_t)i * N + j];
                    if (bias_kind == 1) {
                        dbias[((int64_t)h * N + i) * ld + j] += g;
                    } else if (bias_kind == 2) {
                        int ri = i / gw, ci = i % gw, rj = j / gw, cj = j % gw;
                        int64_t G = (int64_t)(2 * gh - 1) * (2 * gw - 1);
                        dbias[h * G + (int64_t)(ri - rj + gh - 1) * (2 * gw - 1) + (ci - cj + gw - 1)] += g;
                    } else if (bias_kind == 3) {
                        int64_t G = (int64_t)(2 * gh - 1) * (2 * gw - 1);
                        double* tb = dbias + h * (G + 3);
                        if (i == 0 && j == 0) tb[G + 2] += g;
                        else if (i == 0) tb[G] += g;
                        else if (j == 0) tb[G + 1] += g;
                        else {
                            int pi = i - 1, pj = j - 1;
                            int ri = pi / gw, ci = pi % gw, rj = pj / gw, cj = pj % gw;
                            tb[(int64_t)(ri - rj + gh - 1) * (2 * gw - 1) + (ci - cj + gw - 1)] += g;
                        }
                    }
                }
        }
    }
    free(s); free(t); free(vh); free(muq); free(muk); free(b); free(ds); free(dt);
    free(dmuq); free(dmuk); free(db); free(vq); free(sv);
}
