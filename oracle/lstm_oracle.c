/*
 * lstm_oracle.c -- plain, slow CPU reference of the multi-layer, optionally
 * bidirectional LSTM forward and its BPTT backward, in IEEE double.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the package's smoke check and the CPU
 * baseline leg of the benchmark call it; the CUDA library never does, and the
 * two share no code.  Nothing here is blocked, fused or reordered beyond what
 * the definitions below state: the batch loop is split over OpenMP threads
 * (rows are independent), and each weight-gradient element is summed in one
 * fixed order (b, then t), so results do not depend on the thread count.
 *
 * What it computes (sources are web pages; cited by title and section):
 *
 *  - Cell, "Long Short-Term Memory (LSTM)" (warp_nn API page), equation block:
 *        i = sig(W_ii x + b_ii + W_hi h + b_hi)     f = sig(W_if x + ... )
 *        g = tanh(W_ig x + b_ig + W_hg h + b_hg)    o = sig(W_io x + ... )
 *        c' = f*c + i*g                             h' = o*tanh(c')
 *    with the four gate blocks stacked in the order i, f, g, o along the 4H
 *    rows of weight_ih / weight_hh ("Learnable parameters" table; the same
 *    order in "Complete Trace: nn.LSTM", Native implementation, chunk(4), and
 *    in "LSTM Gate Equations > Comparing with PyTorch", the [i, f, c, o]
 *    stacking).  sig(z) = 1/(1+exp(-z)).
 *  - Layers: layer k > 0 reads the previous layer's output sequence; the
 *    lower layer's final (h, c) is not chained ("LSTM Forward Computation",
 *    Stack Multiple RNN Cells; warp_nn equation note on x_t).
 *  - Bidirectional: the reverse direction walks t = T-1 .. 0 with its own
 *    parameters and the output is [forward, reverse] along features (warp_nn
 *    page, paragraph after the equations).  The reverse output at position t
 *    is the reverse state after it has consumed x_{T-1} .. x_t, and its h_n is
 *    the state after t = 0 (plain reading of that paragraph).
 *  - Shapes: weight_ih_l{k} (4H, in_k), in_0 = I, in_k = D*H; weight_hh_l{k}
 *    (4H, H); biases 4H; x (B, T, I); h0, c0, h_n, c_n (L*D, B, H) indexed
 *    layer*D + direction; out (B, T, D*H) (warp_nn "Learnable parameters"
 *    table and __call__ parameters/returns).  Missing h0/c0 mean zeros.
 *  - Backward: back-propagation through time is reverse-mode differentiation
 *    of the unrolled loop ("LSTM Forward Computation", Loop Unroll); the
 *    weight and bias gradients are summed over every timestep (pulsatrix
 *    LSTMModule, backward()).  For one step, with dh the total gradient
 *    reaching h_t and dc the carry reaching c_t from step t+1:
 *        dc_t  = dc + dh*o*(1 - tanh(c_t)^2)
 *        da_o  = dh*tanh(c_t)*o*(1-o)      da_i = dc_t*g*i*(1-i)
 *        da_g  = dc_t*i*(1-g^2)            da_f = dc_t*c_{t-1}*f*(1-f)
 *        carry dc_{t-1} = dc_t*f,  dh_{t-1} = W_hh^T da,  dx_t = W_ih^T da
 *        dW_ih += da x_t^T,  dW_hh += da h_{t-1}^T,  db_ih = db_hh += da
 *    These are the chain rule applied to the cell equations above.
 *
 *  - Variable-length batches: "Complete Trace: nn.LSTM", Step 3, lists a
 *    second overload for packed sequences (per-step batch sizes), and
 *    "LSTM Forward Computation", Sequence Buckets, pads sequences to a fixed
 *    length.  Plain reading, with lengths[b] (0 <= lengths[b] <= T) valid
 *    steps in row b of the padded batch: row b is the ordinary problem on
 *    its first lengths[b] steps (the reverse direction starts at step
 *    lengths[b] - 1), its padded outputs are 0, h_n/c_n are its final states,
 *    the padding receives no gradient and contributes none.
 *  - Inter-layer dropout in training ("Complete Trace: nn.LSTM", the dropout
 *    argument of the LSTM op): with probability p each element of the output
 *    of layers 0..L-2 is zeroed before it enters the next layer, survivors
 *    are scaled by 1/(1-p); the last layer's output is not dropped.  The
 *    pages fix no random stream, so this build fixes one: for boundary l,
 *    element e = (t*B + b)*(D*H) + k of the time-major output sequence is kept
 *    iff (w >> 11) >= ceil(p * 2^53), where w is word e mod 4 of
 *    Philox4x64-10 (Salmon, Moraes, Dror, Shaw 2011, "Parallel random
 *    numbers: as easy as 1, 2, 3") with key (seed, l) and counter
 *    (floor(e/4), 0, 0, 0).  An integer decision, so every implementation
 *    takes the same one.
 *
 * Layout of every array is row-major and batch-first as listed; the Python
 * wrapper converts seq-first data before calling.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Single-precision build (gcc -DORACLE_SINGLE), used only for the precision
 * comparison of "LSTM Gate Equations > Comparing with PyTorch" (Out[20]: two
 * independent float32 renditions of the cell agree to a few 1e-8).  Every
 * array, state and sum below is then a float; exp/tanh, declared above, are
 * still evaluated in double and rounded when stored.  The library's tests and
 * the benchmark use the double build. */
#ifdef ORACLE_SINGLE
#define double float
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

static double sig(double z) { return 1.0 / (1.0 + exp(-z)); }

/* ---------------------------------------------------------------- Philox
 * Philox4x64-10 as defined by Salmon et al. (2011): ten rounds of
 *   (R0, R1, R2, R3) -> (hi(M1*R2) ^ R1 ^ K0, lo(M1*R2), hi(M0*R0) ^ R3 ^ K1, lo(M0*R0))
 * with the key bumped by the Weyl constants after every round. */
static void mul_hilo64(uint64_t a, uint64_t b, uint64_t* hi, uint64_t* lo) {
    const unsigned __int128 p = (unsigned __int128)a * b;
    *hi = (uint64_t)(p >> 64);
    *lo = (uint64_t)p;
}

void oracle_philox4x64_10(const uint64_t* ctr, const uint64_t* key, uint64_t* out) {
    const uint64_t M0 = 0xD2E7470EE14C6C93ULL, M1 = 0xCA5A826395121157ULL;
    const uint64_t W0 = 0x9E3779B97F4A7C15ULL, W1 = 0xBB67AE8584CAA73BULL;
    uint64_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3], k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        uint64_t hi0, lo0, hi1, lo1;
        mul_hilo64(M0, c0, &hi0, &lo0);
        mul_hilo64(M1, c2, &hi1, &lo1);
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
        k0 += W0;
        k1 += W1;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Dropout decision for element e of boundary l (see the header comment). */
static int dropout_keep(uint64_t seed, int l, uint64_t e, uint64_t thresh) {
    const uint64_t ctr[4] = {e >> 2, 0, 0, 0};
    const uint64_t key[2] = {seed, (uint64_t)l};
    uint64_t w[4];
    oracle_philox4x64_10(ctr, key, w);
    return (w[e & 3] >> 11) >= thresh;
}

/* Problem description shared by the entry points. */
typedef struct {
    int L, D, I, H, B, T, bias;
    const int* lengths;   /* [B] valid steps per row, or NULL (all T) */
    double dropout;       /* inter-layer dropout probability (training), 0 = none */
    uint64_t seed;
} prob;

static uint64_t dropout_thresh(double p) { return (uint64_t)ceil(p * 9007199254740992.0); /* p * 2^53 */ }

/* Row b's output sequence of layer l ([T][D*H]) as the next layer's input:
 * multiplied by the dropout mask over 1-p (training, l < L-1, p > 0). */
static void apply_dropout(const prob* p, int l, int b, double* seq) {
    if (!(p->dropout > 0.0) || l >= p->L - 1) return;
    const int DH = p->D * p->H;
    const uint64_t th = dropout_thresh(p->dropout);
    const double scale = 1.0 / (1.0 - p->dropout);
    for (int t = 0; t < p->T; ++t)
        for (int k = 0; k < DH; ++k) {
            const uint64_t e = ((uint64_t)t * p->B + b) * DH + k;
            seq[(size_t)t * DH + k] *= dropout_keep(p->seed, l, e, th) ? scale : 0.0;
        }
}

/* Valid steps of row b. */
static int row_len(const prob* p, int b) { return p->lengths ? p->lengths[b] : p->T; }

static int in_size(const prob* p, int layer) { return layer == 0 ? p->I : p->D * p->H; }

/* Per-row forward record kept for the backward.
 *   seq[l]  : layer l's input sequence, [T][in_l]  (seq[0] = the x row)
 *   act[l*D+d] : [T][5H] = i, f, g, o, c_t after step t (gates post-activation)
 *   hs[l*D+d]  : [T][H]  = h_t
 * The layer output is [T][D*H]; it is seq[l+1] (or the final output).
 */
typedef struct {
    double** seq;   /* L+1 entries; seq[L] is the final output [T][D*H] */
    double** act;   /* L*D */
    double** hs;    /* L*D */
} row_record;

/* One (layer, direction) pass of the cell over time for one batch row.
 * seq_in [T][in], h and c hold the initial state on entry and h_n, c_n on exit,
 * y receives h_t at y[t*ystride + u]. */
static void cell_pass(int T, int in, int H, int reverse, int bias,
                      const double* seq_in, const double* W_ih, const double* W_hh,
                      const double* b_ih, const double* b_hh,
                      double* h, double* c, double* y, int ystride,
                      double* act, double* hs, double* a, double* hprev)
{
    const int G = 4 * H;
    for (int s = 0; s < T; ++s) {
        const int t = reverse ? T - 1 - s : s;
        memcpy(hprev, h, sizeof(double) * (size_t)H);
        /* pre-activations: a = W_ih x_t + b_ih + W_hh h_{t-1} + b_hh */
        for (int r = 0; r < G; ++r) {
            double acc = 0.0;
            const double* wi = W_ih + (size_t)r * in;
            const double* xt = seq_in + (size_t)t * in;
            for (int k = 0; k < in; ++k) acc += wi[k] * xt[k];
            const double* wh = W_hh + (size_t)r * H;
            for (int j = 0; j < H; ++j) acc += wh[j] * hprev[j];
            if (bias) acc += b_ih[r] + b_hh[r];
            a[r] = acc;
        }
        for (int u = 0; u < H; ++u) {
            const double ig = sig(a[u]);
            const double fg = sig(a[H + u]);
            const double gg = tanh(a[2 * H + u]);
            const double og = sig(a[3 * H + u]);
            c[u] = fg * c[u] + ig * gg;
            h[u] = og * tanh(c[u]);
            y[(size_t)t * ystride + u] = h[u];
            if (act) {
                double* at = act + (size_t)t * 5 * H;
                at[u] = ig; at[H + u] = fg; at[2 * H + u] = gg; at[3 * H + u] = og; at[4 * H + u] = c[u];
            }
            if (hs) hs[(size_t)t * H + u] = h[u];
        }
    }
}

/* Forward for one batch row b.  When rec != NULL the activations are kept. */
static int forward_row(const prob* p, int b,
                       const double* x, const double* h0, const double* c0,
                       const double* const* w_ih, const double* const* w_hh,
                       const double* const* b_ih, const double* const* b_hh,
                       double* out, double* h_n, double* c_n, row_record* rec)
{
    const int L = p->L, D = p->D, H = p->H, T = p->T, B = p->B, G = 4 * H;
    int maxin = p->I > D * H ? p->I : D * H;
    double* a = (double*)malloc(sizeof(double) * (size_t)G);
    double* hprev = (double*)malloc(sizeof(double) * (size_t)H);
    double* h = (double*)malloc(sizeof(double) * (size_t)H);
    double* c = (double*)malloc(sizeof(double) * (size_t)H);
    double* bufA = (double*)malloc(sizeof(double) * ((size_t)T * maxin + 1));
    double* bufB = (double*)malloc(sizeof(double) * ((size_t)T * maxin + 1));
    if (!a || !hprev || !h || !c || !bufA || !bufB) {
        free(a); free(hprev); free(h); free(c); free(bufA); free(bufB);
        return ORACLE_ERR_NOMEM;
    }
    const int n = row_len(p, b);   /* this row's steps; positions n..T-1 are padding */
    /* layer-0 input: the x row */
    double* cur = rec ? rec->seq[0] : bufA;
    memcpy(cur, x + (size_t)b * T * p->I, sizeof(double) * (size_t)T * p->I);
    for (int l = 0; l < L; ++l) {
        const int in = in_size(p, l);
        double* nxt = rec ? rec->seq[l + 1] : (cur == bufA ? bufB : bufA);
        memset(nxt, 0, sizeof(double) * (size_t)T * D * H);   /* padded outputs stay 0 */
        for (int d = 0; d < D; ++d) {
            const int ld = l * D + d;
            for (int u = 0; u < H; ++u) {
                h[u] = h0 ? h0[((size_t)ld * B + b) * H + u] : 0.0;
                c[u] = c0 ? c0[((size_t)ld * B + b) * H + u] : 0.0;
            }
            cell_pass(n, in, H, d == 1, p->bias, cur, w_ih[ld], w_hh[ld],
                      p->bias ? b_ih[ld] : NULL, p->bias ? b_hh[ld] : NULL,
                      h, c, nxt + d * H, D * H,
                      rec ? rec->act[ld] : NULL, rec ? rec->hs[ld] : NULL, a, hprev);
            for (int u = 0; u < H; ++u) {
                if (h_n) h_n[((size_t)ld * B + b) * H + u] = h[u];
                if (c_n) c_n[((size_t)ld * B + b) * H + u] = c[u];
            }
        }
        apply_dropout(p, l, b, nxt);   /* what the next layer reads */
        cur = nxt;
    }
    if (out) memcpy(out + (size_t)b * T * D * H, cur, sizeof(double) * (size_t)T * D * H);
    free(a); free(hprev); free(h); free(c); free(bufA); free(bufB);
    return ORACLE_OK;
}

static int check_prob(const prob* p) {
    if (p->L < 1 || (p->D != 1 && p->D != 2) || p->I < 1 || p->H < 1 || p->B < 0 || p->T < 0)
        return ORACLE_ERR_ARG;
    if (p->lengths)
        for (int b = 0; b < p->B; ++b)
            if (p->lengths[b] < 0 || p->lengths[b] > p->T) return ORACLE_ERR_ARG;
    return ORACLE_OK;
}

/*
 * Forward.  x [B][T][I]; h0, c0 [L*D][B][H] or NULL (zeros); w_ih[l*D+d]
 * [4H][in_l]; w_hh [4H][H]; b_ih, b_hh [4H] (ignored when bias == 0);
 * lengths [B] or NULL; out [B][T][D*H]; h_n, c_n [L*D][B][H].  Returns 0 on
 * success.
 */
int oracle_lstm_forward(int L, int D, int I, int H, int B, int T, int bias, const int* lengths,
                        const double* x, const double* h0, const double* c0,
                        const double* const* w_ih, const double* const* w_hh,
                        const double* const* b_ih, const double* const* b_hh,
                        double* out, double* h_n, double* c_n)
{
    prob p = {L, D, I, H, B, T, bias, lengths, 0.0, 0};
    if (check_prob(&p)) return ORACLE_ERR_ARG;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(|:err)
    for (int b = 0; b < B; ++b)
        err |= forward_row(&p, b, x, h0, c0, w_ih, w_hh, b_ih, b_hh, out, h_n, c_n, NULL);
    return err;
}

static void free_record(const prob* p, row_record* r) {
    if (r->seq) for (int l = 0; l <= p->L; ++l) free(r->seq[l]);
    if (r->act) for (int i = 0; i < p->L * p->D; ++i) free(r->act[i]);
    if (r->hs) for (int i = 0; i < p->L * p->D; ++i) free(r->hs[i]);
    free(r->seq); free(r->act); free(r->hs);
    r->seq = r->act = r->hs = NULL;
}

static int alloc_record(const prob* p, row_record* r) {
    const int L = p->L, D = p->D, H = p->H, T = p->T;
    r->seq = (double**)calloc((size_t)L + 1, sizeof(double*));
    r->act = (double**)calloc((size_t)L * D, sizeof(double*));
    r->hs = (double**)calloc((size_t)L * D, sizeof(double*));
    if (!r->seq || !r->act || !r->hs) { free_record(p, r); return ORACLE_ERR_NOMEM; }
    for (int l = 0; l <= L; ++l) {
        const int w = l == 0 ? p->I : D * H;
        r->seq[l] = (double*)malloc(sizeof(double) * ((size_t)T * w + 1));
        if (!r->seq[l]) { free_record(p, r); return ORACLE_ERR_NOMEM; }
    }
    for (int i = 0; i < L * D; ++i) {
        r->act[i] = (double*)malloc(sizeof(double) * ((size_t)T * 5 * H + 1));
        r->hs[i] = (double*)malloc(sizeof(double) * ((size_t)T * H + 1));
        if (!r->act[i] || !r->hs[i]) { free_record(p, r); return ORACLE_ERR_NOMEM; }
    }
    return ORACLE_OK;
}

/*
 * BPTT for one row.  Fills da[l*D+d] ([T][4H], pre-activation gradients),
 * dx row, dh0/dc0 row.  grad_out row [T][D*H] is the gradient reaching the
 * top layer's output.
 */
static int backward_row(const prob* p, int b, const row_record* rec,
                        const double* c0,
                        const double* const* w_ih, const double* const* w_hh,
                        const double* grad_out, const double* grad_hn, const double* grad_cn,
                        double** da, double* dx, double* dh0, double* dc0)
{
    const int L = p->L, D = p->D, H = p->H, T = p->T, B = p->B, G = 4 * H;
    int maxin = p->I > D * H ? p->I : D * H;
    double* dy = (double*)malloc(sizeof(double) * ((size_t)T * D * H + 1));     /* grad reaching layer output */
    double* din = (double*)malloc(sizeof(double) * ((size_t)T * maxin + 1));    /* grad reaching layer input */
    double* dh = (double*)malloc(sizeof(double) * (size_t)H);
    double* dc = (double*)malloc(sizeof(double) * (size_t)H);
    double* dhn = (double*)malloc(sizeof(double) * (size_t)H);
    if (!dy || !din || !dh || !dc || !dhn) {
        free(dy); free(din); free(dh); free(dc); free(dhn);
        return ORACLE_ERR_NOMEM;
    }
    const int n = row_len(p, b);   /* steps n..T-1 are padding: no gradient in or out */
    memcpy(dy, grad_out + (size_t)b * T * D * H, sizeof(double) * (size_t)T * D * H);
    for (int l = L - 1; l >= 0; --l) {
        const int in = in_size(p, l);
        const double* seq_in = rec->seq[l];
        memset(din, 0, sizeof(double) * (size_t)T * in);
        for (int d = 0; d < D; ++d) {
            const int ld = l * D + d;
            const double* act = rec->act[ld];
            const double* hs = rec->hs[ld];
            double* dal = da[ld];
            for (int u = 0; u < H; ++u) {
                dh[u] = grad_hn ? grad_hn[((size_t)ld * B + b) * H + u] : 0.0;
                dc[u] = grad_cn ? grad_cn[((size_t)ld * B + b) * H + u] : 0.0;
            }
            /* walk time opposite to the forward order of this direction */
            for (int s = n - 1; s >= 0; --s) {
                const int t = d == 1 ? n - 1 - s : s;
                const int tp = d == 1 ? t + 1 : t - 1;   /* forward-order predecessor */
                const int has_prev = d == 1 ? (t + 1 < n) : (t >= 1);
                const double* at = act + (size_t)t * 5 * H;
                double* dat = dal + (size_t)t * G;
                for (int u = 0; u < H; ++u) {
                    const double ig = at[u], fg = at[H + u], gg = at[2 * H + u], og = at[3 * H + u];
                    const double ct = at[4 * H + u];
                    const double cp = has_prev ? act[(size_t)tp * 5 * H + 4 * H + u]
                                               : (c0 ? c0[((size_t)ld * B + b) * H + u] : 0.0);
                    const double th = tanh(ct);
                    const double dht = dy[(size_t)t * D * H + d * H + u] + dh[u];
                    const double dct = dc[u] + dht * og * (1.0 - th * th);
                    dat[u] = dct * gg * ig * (1.0 - ig);              /* i */
                    dat[H + u] = dct * cp * fg * (1.0 - fg);          /* f */
                    dat[2 * H + u] = dct * ig * (1.0 - gg * gg);      /* g */
                    dat[3 * H + u] = dht * th * og * (1.0 - og);      /* o */
                    dc[u] = dct * fg;
                }
                /* dh_{t-1} = W_hh^T da_t ; d(input_t) += W_ih^T da_t */
                for (int j = 0; j < H; ++j) dhn[j] = 0.0;
                const double* Wh = w_hh[ld];
                for (int r = 0; r < G; ++r) {
                    const double g = dat[r];
                    const double* wr = Wh + (size_t)r * H;
                    for (int j = 0; j < H; ++j) dhn[j] += wr[j] * g;
                }
                memcpy(dh, dhn, sizeof(double) * (size_t)H);
                const double* Wi = w_ih[ld];
                double* dint = din + (size_t)t * in;
                for (int r = 0; r < G; ++r) {
                    const double g = dat[r];
                    const double* wr = Wi + (size_t)r * in;
                    for (int k = 0; k < in; ++k) dint[k] += wr[k] * g;
                }
                (void)hs; (void)seq_in;
            }
            for (int u = 0; u < H; ++u) {
                dh0[((size_t)ld * B + b) * H + u] = dh[u];
                dc0[((size_t)ld * B + b) * H + u] = dc[u];
            }
        }
        if (l > 0) {
            memcpy(dy, din, sizeof(double) * (size_t)T * in);
            apply_dropout(p, l - 1, b, dy);   /* the same mask carries the gradient back */
        }
        else memcpy(dx + (size_t)b * T * p->I, din, sizeof(double) * (size_t)T * p->I);
    }
    free(dy); free(din); free(dh); free(dc); free(dhn);
    return ORACLE_OK;
}

/*
 * Forward + BPTT.  Same inputs as oracle_lstm_forward plus grad_out
 * [B][T][D*H] and grad_hn, grad_cn [L*D][B][H] (NULL = zeros).  Outputs:
 * out, h_n, c_n (may be NULL), dx [B][T][I], dh0, dc0 [L*D][B][H],
 * dw_ih[l*D+d] [4H][in_l], dw_hh [4H][H], db_ih, db_hh [4H] (bias only).
 * The weight gradients are overwritten, not accumulated.  dropout in [0, 1)
 * and seed select the inter-layer dropout of the training forward.
 */
int oracle_lstm_backward(int L, int D, int I, int H, int B, int T, int bias, const int* lengths,
                         double dropout, uint64_t seed, const double* x, const double* h0, const double* c0,
                         const double* const* w_ih, const double* const* w_hh,
                         const double* const* b_ih, const double* const* b_hh,
                         const double* grad_out, const double* grad_hn, const double* grad_cn,
                         double* out, double* h_n, double* c_n,
                         double* dx, double* dh0, double* dc0,
                         double* const* dw_ih, double* const* dw_hh,
                         double* const* db_ih, double* const* db_hh)
{
    prob p = {L, D, I, H, B, T, bias, lengths, dropout, seed};
    if (check_prob(&p)) return ORACLE_ERR_ARG;
    if (!(dropout >= 0.0 && dropout < 1.0)) return ORACLE_ERR_ARG;
    const int G = 4 * H, LD = L * D;
    row_record* recs = (row_record*)calloc((size_t)B + 1, sizeof(row_record));
    double*** da = (double***)calloc((size_t)B + 1, sizeof(double**));
    if (!recs || !da) { free(recs); free(da); return ORACLE_ERR_NOMEM; }
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(|:err)
    for (int b = 0; b < B; ++b) {
        int e = alloc_record(&p, &recs[b]);
        da[b] = (double**)calloc((size_t)LD, sizeof(double*));
        if (!e && !da[b]) e = ORACLE_ERR_NOMEM;
        for (int i = 0; !e && i < LD; ++i) {
            da[b][i] = (double*)malloc(sizeof(double) * ((size_t)T * G + 1));
            if (!da[b][i]) e = ORACLE_ERR_NOMEM;
        }
        if (!e) e = forward_row(&p, b, x, h0, c0, w_ih, w_hh, b_ih, b_hh, out, h_n, c_n, &recs[b]);
        if (!e) e = backward_row(&p, b, &recs[b], c0, w_ih, w_hh, grad_out, grad_hn, grad_cn,
                                 da[b], dx, dh0, dc0);
        err |= e;
    }
    if (!err) {
        /* weight and bias gradients: sum over b, then t, per output element */
        for (int ld = 0; ld < LD; ++ld) {
            const int l = ld / D, d = ld % D;
            const int in = in_size(&p, l);
#pragma omp parallel for schedule(static)
            for (int r = 0; r < G; ++r) {
                double* wi = dw_ih[ld] + (size_t)r * in;
                double* wh = dw_hh[ld] + (size_t)r * H;
                double sb = 0.0;
                for (int k = 0; k < in; ++k) wi[k] = 0.0;
                for (int j = 0; j < H; ++j) wh[j] = 0.0;
                for (int b = 0; b < B; ++b) {
                    const double* dal = da[b][ld];
                    const double* seq_in = recs[b].seq[l];
                    const double* hs = recs[b].hs[ld];
                    const int n = row_len(&p, b);
                    for (int t = 0; t < n; ++t) {
                        const double g = dal[(size_t)t * G + r];
                        sb += g;
                        const double* xt = seq_in + (size_t)t * in;
                        for (int k = 0; k < in; ++k) wi[k] += g * xt[k];
                        /* h_{t-1} in this direction's order; h0 (or 0) at the start */
                        const int has_prev = d == 1 ? (t + 1 < n) : (t >= 1);
                        if (has_prev) {
                            const double* hp = hs + (size_t)(d == 1 ? t + 1 : t - 1) * H;
                            for (int j = 0; j < H; ++j) wh[j] += g * hp[j];
                        } else if (h0) {
                            const double* hp = h0 + ((size_t)ld * B + b) * H;
                            for (int j = 0; j < H; ++j) wh[j] += g * hp[j];
                        }
                    }
                }
                if (bias) {
                    db_ih[ld][r] = sb;
                    db_hh[ld][r] = sb;
                }
            }
        }
    }
    for (int b = 0; b < B; ++b) {
        free_record(&p, &recs[b]);
        if (da[b]) for (int i = 0; i < LD; ++i) free(da[b][i]);
        free(da[b]);
    }
    free(recs); free(da);
    return err;
}
