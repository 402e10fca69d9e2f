/*
 * lc_oracle.c -- fp64 CPU oracle for block-sparse 3D-RoPE video self-attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously-correct
 * statement of what the GPU library computes.  Only the test-suite, the smoke
 * check and the CPU-baseline leg of the benchmark may load it.  It shares no
 * code, header, table or constant with the CUDA library, and the library never
 * loads it.
 *
 * Sources (the web pages this method is described on):
 *   [RS]  "longcat-video-rs" (code.brandonhubbard.com): the header card
 *         "PARTITIONED 3D-ROPE 16T + 24H + 24W", section 03-01 "Partitioned
 *         3D-RoPE (16T+24H+24W)", section 03-03 "Block-Sparse & Multi-Audio",
 *         and the section 02 benchmark-table row "Block-Sparse Self-Attention
 *         (block=64, local=2, stride=4)".
 *   [QB]  "美团视频生成模型来了！一出手就是开源 SOTA" (myzaker / QbitAI), section
 *         "背后技术原理": tasks differ only by the number of condition frames,
 *         condition frames are concatenated before the noisy frames on the time
 *         axis, and a block attention with KV cache keeps condition tokens
 *         unaffected by noise tokens.
 *   [ZC]  "美团开源 LongCat-Video" (zhichai.net), section "Block Sparse
 *         Attention": dense inside blocks, sparse across blocks.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *   - RoPE: channels [0,16) rotate by the frame index t, [16,40) by the row h,
 *     [40,64) by the column w; adjacent channel pairs (c, c+1) form one complex
 *     number; pair k of an axis of width d turns by pos * theta^(-2k/d);
 *     theta = 10000; integer positions from 0.
 *   - token n of the full sequence sits at t = n / (H*W), h = (n / W) % H,
 *     w = n % W (t-major, then h, then w).
 *   - a block is 64 consecutive tokens of one segment (condition segment or
 *     noisy segment); the last block of a segment may be short.
 *   - noisy block i attends noisy block j iff |i-j| <= local, or stride > 0
 *     and j % stride == 0 ("local sliding window plus strided global blocks").
 *   - condition queries attend all condition keys and nothing else; noisy
 *     queries attend all condition keys plus the block-sparse noisy keys.
 *   - softmax scale 1/sqrt(head_dim).
 *
 * Parity pins: every function here is checked by tests against closed forms,
 * invariants, library routines and the figures the pages print (see the
 * tests directory); none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------------------
 * Position of a token in the latent video grid.
 * [RS] 03-01 passes (t, h, w) to apply_rope; the flattening order is t-major.
 * ------------------------------------------------------------------------- */
static void orc_decode_position(long n, int H, int W, long *t, long *h, long *w)
{
    long hw = (long)H * (long)W;
    *t = n / hw;
    *h = (n / W) % H;
    *w = n % W;
}

/* ---------------------------------------------------------------------------
 * Rotate one head vector x[0..hd) of the token at (t, h, w) in place.
 * [RS] header card and 03-01: the 64-D head is split into 16 temporal,
 * 24 vertical and 24 horizontal channels, each rotated as complex pairs
 * (norm preserving).  dt + dh + dw must equal hd; each must be even.
 * ------------------------------------------------------------------------- */
void orc_rope3d_rotate_vec(double *x, int hd, long t, long h, long w,
                           double theta, int dt, int dh, int dw)
{
    const int widths[3] = {dt, dh, dw};
    const long pos[3] = {t, h, w};
    int off = 0;
    (void)hd;
    for (int axis = 0; axis < 3; ++axis) {
        int d = widths[axis];
        for (int k = 0; k < d / 2; ++k) {
            double omega = pow(theta, -2.0 * (double)k / (double)d);
            double phi = (double)pos[axis] * omega;
            double c = cos(phi), s = sin(phi);
            int i0 = off + 2 * k, i1 = off + 2 * k + 1;
            double a = x[i0], b = x[i1];
            x[i0] = a * c - b * s;
            x[i1] = a * s + b * c;
        }
        off += d;
    }
}

/* x: [B, ntok, heads, hd] fp64, rotated in place.  Token index n of x is
 * token n + tok_offset of the full (condition + noisy) sequence. */
void orc_rope3d_apply(double *x, int B, long ntok, int heads, int hd,
                      long tok_offset, int H, int W, double theta,
                      int dt, int dh, int dw)
{
    for (int b = 0; b < B; ++b)
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
        for (long n = 0; n < ntok; ++n) {
            long t, h, w;
            orc_decode_position(n + tok_offset, H, W, &t, &h, &w);
            for (int hh = 0; hh < heads; ++hh) {
                double *v = x + (((long)b * ntok + n) * heads + hh) * hd;
                orc_rope3d_rotate_vec(v, hd, t, h, w, theta, dt, dh, dw);
            }
        }
}

/* ---------------------------------------------------------------------------
 * Block rule between noisy blocks.  [RS] 03-03: local sliding-window blocks
 * combined with strided global key/value blocks; parameters of the table row
 * in section 02 are block=64, local=2, stride=4.
 * ------------------------------------------------------------------------- */
int orc_noisy_block_rule(long i, long j, int local, int stride)
{
    long d = i - j;
    if (d < 0) d = -d;
    if (d <= local) return 1;
    if (stride > 0 && (j % stride) == 0) return 1;
    return 0;
}

/* Token-level mask, written from the definition (not from any block list).
 * n = query token, m = key token, both indices of the full sequence whose
 * first Nc tokens are condition tokens.  [QB]: condition tokens are not
 * affected by noise tokens; noisy tokens see every condition token. */
int orc_token_allowed(long n, long m, long Nc, int block, int local, int stride)
{
    if (n < Nc) return m < Nc;
    if (m < Nc) return 1;
    return orc_noisy_block_rule((n - Nc) / block, (m - Nc) / block, local, stride);
}

/* ---------------------------------------------------------------------------
 * Block CSR by brute force over every (query block, key block) pair.
 * Blocks 0..Cb-1 are condition blocks, Cb..Cb+Nb-1 noisy blocks.
 * Returns nnz; fills row_ptr[Cb+Nb+1] and col_idx[nnz] when not NULL.
 * ------------------------------------------------------------------------- */
long orc_block_csr(int T, int H, int W, int block, int local, int stride,
                   int n_cond, int *row_ptr, int *col_idx)
{
    long Nc = (long)n_cond * H * W;
    long Nn = (long)(T - n_cond) * H * W;
    long Cb = (Nc + block - 1) / block;
    long Nb = (Nn + block - 1) / block;
    long nnz = 0;
    if (row_ptr) row_ptr[0] = 0;
    for (long r = 0; r < Cb + Nb; ++r) {
        for (long c = 0; c < Cb + Nb; ++c) {
            int attend;
            if (r < Cb) attend = (c < Cb);
            else if (c < Cb) attend = 1;
            else attend = orc_noisy_block_rule(r - Cb, c - Cb, local, stride);
            if (attend) {
                if (col_idx) col_idx[nnz] = (int)c;
                ++nnz;
            }
        }
        if (row_ptr) row_ptr[r + 1] = (int)nnz;
    }
    return nnz;
}

/* Number of attended (query token, key token) pairs of the whole sequence,
 * counted token by token from orc_token_allowed.  O(N^2): small cases only. */
long long orc_count_token_pairs(long N, long Nc, int block, int local, int stride)
{
    long long cnt = 0;
    for (long n = 0; n < N; ++n)
        for (long m = 0; m < N; ++m)
            cnt += orc_token_allowed(n, m, Nc, block, local, stride);
    return cnt;
}

/* ---------------------------------------------------------------------------
 * Masked softmax attention for selected query rows.
 *
 *   qrot : [B, Nq, heads, hd]   rotated queries; query token r of qrot is
 *                               token r + q_offset of the full sequence
 *   krot : [B, N,  heads, hd]   rotated keys of the full sequence
 *   v    : [B, N,  heads, hd]
 *   rows : R triples (b, head, r) with r an index into qrot
 *   out  : [R, hd],  lse : [R] (natural log), both fp64
 *
 * Per row: s_m = scale * <q_n, k_m> over the allowed keys m, mx = max s,
 * p_m = exp(s_m - mx), l = sum p, o = sum p_m v_m / l, lse = mx + ln l.
 * ------------------------------------------------------------------------- */
void orc_attention_rows(const double *qrot, const double *krot, const double *v,
                        int B, long Nq, long q_offset, long N, int heads, int hd,
                        long Nc, int block, int local, int stride, double scale,
                        const long *rows, long R, double *out, double *lse,
                        int nthreads)
{
    (void)B;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        unsigned char *ok = (unsigned char *)malloc((size_t)N);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (long ri = 0; ri < R; ++ri) {
            long b = rows[3 * ri + 0], hh = rows[3 * ri + 1], r = rows[3 * ri + 2];
            long n = r + q_offset;
            const double *qv = qrot + ((b * Nq + r) * heads + hh) * hd;
            double mx = -INFINITY;
            for (long m = 0; m < N; ++m) {
                ok[m] = (unsigned char)orc_token_allowed(n, m, Nc, block, local, stride);
                if (!ok[m]) continue;
                const double *kv = krot + ((b * N + m) * heads + hh) * hd;
                double dot = 0.0;
                for (int d = 0; d < hd; ++d) dot += qv[d] * kv[d];
                s[m] = scale * dot;
                if (s[m] > mx) mx = s[m];
            }
            double l = 0.0;
            double *o = out + ri * hd;
            for (int d = 0; d < hd; ++d) o[d] = 0.0;
            for (long m = 0; m < N; ++m) {
                if (!ok[m]) continue;
                double p = exp(s[m] - mx);
                l += p;
                const double *vv = v + ((b * N + m) * heads + hh) * hd;
                for (int d = 0; d < hd; ++d) o[d] += p * vv[d];
            }
            for (int d = 0; d < hd; ++d) o[d] /= l;
            lse[ri] = mx + log(l);
        }
        free(s);
        free(ok);
    }
}

/* Softmax probabilities of one query row over the full key sequence (zero on
 * masked keys), for the row-sum and mask-support checks. */
void orc_attention_row_probs(const double *qrot, const double *krot,
                             long Nq, long q_offset, long N, int heads, int hd,
                             long Nc, int block, int local, int stride,
                             double scale, long b, long hh, long r, double *probs)
{
    long n = r + q_offset;
    const double *qv = qrot + ((b * Nq + r) * heads + hh) * hd;
    double mx = -INFINITY;
    for (long m = 0; m < N; ++m) {
        probs[m] = -INFINITY;
        if (!orc_token_allowed(n, m, Nc, block, local, stride)) continue;
        const double *kv = krot + ((b * N + m) * heads + hh) * hd;
        double dot = 0.0;
        for (int d = 0; d < hd; ++d) dot += qv[d] * kv[d];
        probs[m] = scale * dot;
        if (probs[m] > mx) mx = probs[m];
    }
    double l = 0.0;
    for (long m = 0; m < N; ++m) {
        probs[m] = (probs[m] == -INFINITY) ? 0.0 : exp(probs[m] - mx);
        l += probs[m];
    }
    for (long m = 0; m < N; ++m) probs[m] /= l;
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
