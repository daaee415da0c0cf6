/*
 * wf_oracle.c -- CPU fp64 oracle for the Wave Forcing wave-round hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the test suite, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * library; the two meet only through seeded input arrays.
 *
 * What it computes (all arithmetic in IEEE double, plain loops, no blocking):
 *
 *   wfo_bf16_to_f64 / wfo_f64_to_bf16
 *       exact widening of bf16 bit patterns, and round-to-nearest-even
 *       narrowing straight from double (IEEE 754 definition of RNE).
 *
 *   wfo_positions
 *       (t,h,w) of every wave token: wave chunk c of round r is absolute chunk
 *       g = r + c; token n = c*L + f*gh*gw + y*gw + x has t = g*F + f, h = y,
 *       w = x.  (The pages fix 3-latent-frame chunks and a 480x832 grid, see
 *       "Wave Forcing", airadar.tv summary, usage notes on --num-frames; the
 *       absolute-time reading is ours, parity for it is pinned by closed form.)
 *
 *   wfo_append
 *       per (token, head): per-head RMSNorm of q and k with gain gamma[h,:],
 *       then 3D RoPE on (t,h,w), then one rounding to bf16; v is copied.
 *       The pages name no norm or RoPE formula (they are fixed by the problem
 *       statement of the hot path); the readings are:
 *         y_d = x_d * gamma_d / sqrt(mean_d x_d^2 + eps)
 *         channels [0,dt) rotate with t, [dt,dt+dh) with h, [dt+dh,D) with w;
 *         pair (2i, 2i+1) of an axis block of width da turns by pos*theta^(-2i/da).
 *
 *   wfo_qk_norm_rope_f64
 *       the same per-head RMSNorm and 3D RoPE on rows given in double (the
 *       exact product of a projection, before any rounding); used by the
 *       oracle of the QKV projection with the append fused into it.
 *
 *   wfo_chunk_causal_attn_rows
 *       softmax attention of selected (query row, head) pairs over an explicit
 *       concatenation of key chunks, each tagged with its absolute chunk id.
 *       Key j is visible to query n exactly when chunk_id(j) <= chunk_id(n):
 *       later chunks see earlier (cleaner) chunks and all of their own chunk,
 *       never a later chunk ("Wave Forcing" abstract: under chunk-wise causal
 *       attention a chunk uses the less noisy chunks ahead of it while they
 *       are still being denoised).  s_j = q.k_j / sqrt(D); p = softmax over
 *       visible j;
 *       O = sum_j p_j v_j; lse = m + log(sum_j exp(s_j - m)).
 *
 *   wfo_e4m3_encode / wfo_e4m3_decode
 *       the 8-bit E4M3 floating-point format (1 sign, 4 exponent bits with bias
 *       7, 3 mantissa bits; exponent field 0 holds subnormals m * 2^-9; no
 *       infinities; S.1111.111 is NaN; largest finite 1.75 * 2^8 = 448).
 *       Encoding rounds to nearest, ties to even, and saturates finite values
 *       beyond 448 to +-448.
 *
 *   wfo_chunk_causal_attn_rows_fp8qk
 *       the same attention with q and k given as E4M3 codes and fp32 scales:
 *       q~[n,h,:] = e4m3(q8[n,h,:]) * q_scale[h,n] (one scale per row and
 *       head), k~[j,h,:] = e4m3(k8[j,h,:]) * k_scale[chunk, tile, h] (one scale
 *       per 128-row key tile of a chunk and head); v stays bf16.  (The codes
 *       and scales come from the quantization rule in oracle/__init__.py.)
 *
 * Parity pins live in tests/test_oracle_pins.py and tests/test_fp8_pins.py
 * (brute-force dense mask, library softmax attention on the unmasked special
 * case, the format's published values, a library float8 cast, closed forms and
 * invariants).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- bf16 <-> double ---------------------------------------------------- */

static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round-to-nearest, ties-to-even, from double to bf16 (8 significand bits,
 * 8 exponent bits).  Works on the real value: find the bf16 quantum q of the
 * binade holding |x|, take rint(x / q) (the C default rounding mode is
 * nearest-even), multiply back.  The result is a float-representable value,
 * whose top 16 bits are the bf16 pattern. */
static uint16_t double_to_bf16_bits(double x)
{
    if (isnan(x)) return 0x7FC0u;
    if (isinf(x)) return x > 0 ? 0x7F80u : 0xFF80u;
    if (x == 0.0) return signbit(x) ? 0x8000u : 0x0000u;
    int e2;
    (void)frexp(fabs(x), &e2);          /* |x| = m * 2^e2, m in [0.5, 1) */
    int e = e2 - 1;                     /* |x| in [2^e, 2^(e+1)) */
    if (e < -126) e = -126;             /* subnormal range: fixed quantum */
    double quantum = ldexp(1.0, e - 7);
    double y = rint(x / quantum) * quantum;
    if (fabs(y) >= ldexp(1.0, 128))     /* rounded past the largest finite */
        return y > 0 ? 0x7F80u : 0xFF80u;
    float f = (float)y;                 /* exact: y has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

void wfo_bf16_to_f64(const uint16_t *in, double *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = bf16_bits_to_double(in[i]);
}

void wfo_f64_to_bf16(const double *in, uint16_t *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = double_to_bf16_bits(in[i]);
}

/* ---- positions ------------------------------------------------------------ */

void wfo_positions(long round, int n_wave, int F, int gh, int gw, int32_t *pos)
{
    const int L = F * gh * gw;
    for (int c = 0; c < n_wave; ++c) {
        long g = round + c;
        for (int f = 0; f < F; ++f)
            for (int y = 0; y < gh; ++y)
                for (int x = 0; x < gw; ++x) {
                    long n = (long)c * L + (long)f * gh * gw + (long)y * gw + x;
                    pos[3 * n + 0] = (int32_t)(g * F + f);
                    pos[3 * n + 1] = y;
                    pos[3 * n + 2] = x;
                }
    }
}

/* ---- RMSNorm and RoPE on one head vector -------------------------------- */

void wfo_rms_norm(const double *x, const double *gamma, int D, double eps, double *y)
{
    double ss = 0.0;
    for (int d = 0; d < D; ++d) ss += x[d] * x[d];
    double inv = 1.0 / sqrt(ss / D + eps);
    for (int d = 0; d < D; ++d) y[d] = x[d] * inv * gamma[d];
}

void wfo_rope_3d(const double *x, int D, int dt, int dh, int dw, double theta,
                 const int32_t *pos_thw, double *y)
{
    const int width[3] = {dt, dh, dw};
    int off = 0;
    for (int a = 0; a < 3; ++a) {
        const int da = width[a];
        for (int i = 0; i < da / 2; ++i) {
            double omega = pow(theta, -2.0 * i / (double)da);
            double phi = (double)pos_thw[a] * omega;
            double cs = cos(phi), sn = sin(phi);
            double x0 = x[off + 2 * i], x1 = x[off + 2 * i + 1];
            y[off + 2 * i]     = x0 * cs - x1 * sn;
            y[off + 2 * i + 1] = x0 * sn + x1 * cs;
        }
        off += da;
    }
    (void)D;
}

/* ---- fused append (norm + rope + bf16 rounding) ------------------------- */

int wfo_append(int T, int H, int D,
               const uint16_t *q, const uint16_t *k, const uint16_t *v,
               const int32_t *pos,                 /* [T,3] */
               const float *gamma_q, const float *gamma_k,   /* [H,D] */
               double eps, int dt, int dh, int dw, double theta,
               uint16_t *q_out, uint16_t *k_out, uint16_t *v_out,  /* [T,H,D] */
               double *q_f64, double *k_f64)       /* [T,H,D] or NULL */
{
    if (dt + dh + dw != D || (dt | dh | dw) & 1) return -1;
    const long rows = (long)T * H;
#pragma omp parallel
    {
        double *xin = (double *)malloc(sizeof(double) * D);
        double *gam = (double *)malloc(sizeof(double) * D);
        double *nrm = (double *)malloc(sizeof(double) * D);
        double *rot = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(static)
        for (long row = 0; row < rows; ++row) {
            const long n = row / H, h = row % H;
            const long base = row * D;
            for (int which = 0; which < 2; ++which) {
                const uint16_t *src = which ? k : q;
                const float *g = which ? gamma_k : gamma_q;
                uint16_t *dst = which ? k_out : q_out;
                double *dst64 = which ? k_f64 : q_f64;
                for (int d = 0; d < D; ++d) {
                    xin[d] = bf16_bits_to_double(src[base + d]);
                    gam[d] = (double)g[h * D + d];
                }
                wfo_rms_norm(xin, gam, D, eps, nrm);
                wfo_rope_3d(nrm, D, dt, dh, dw, theta, pos + 3 * n, rot);
                for (int d = 0; d < D; ++d) {
                    dst[base + d] = double_to_bf16_bits(rot[d]);
                    if (dst64) dst64[base + d] = rot[d];
                }
            }
            for (int d = 0; d < D; ++d) v_out[base + d] = v[base + d];
        }
        free(xin); free(gam); free(nrm); free(rot);
    }
    return 0;
}

/* ---- norm + rope on double rows (projection output, not rounded) ------- */

int wfo_qk_norm_rope_f64(int T, int H, int D, const double *x, const int32_t *pos,
                         const float *gamma, double eps, int dt, int dh, int dw,
                         double theta, double *y)
{
    if (dt + dh + dw != D || (dt | dh | dw) & 1) return -1;
    const long rows = (long)T * H;
#pragma omp parallel
    {
        double *gam = (double *)malloc(sizeof(double) * D);
        double *nrm = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(static)
        for (long row = 0; row < rows; ++row) {
            const long n = row / H, h = row % H;
            for (int d = 0; d < D; ++d) gam[d] = (double)gamma[h * D + d];
            wfo_rms_norm(x + row * D, gam, D, eps, nrm);
            wfo_rope_3d(nrm, D, dt, dh, dw, theta, pos + 3 * n, y + row * D);
        }
        free(gam); free(nrm);
    }
    return 0;
}

/* ---- chunk-causal attention on selected rows ----------------------------- */

/*
 * q       : [Tq, H, D] bf16 bits, the queries (wave tokens, already normed/roped)
 * q_chunk : absolute chunk id of every query chunk; query n lies in chunk n / L
 * kv      : k, v as [n_kchunks * L, H, D] bf16 bits, chunk b holds rows [b*L, (b+1)*L)
 * k_chunk : absolute chunk id of every key chunk
 * rows, heads : the n_sel (query row, head) pairs to compute
 * o       : [n_sel, D] doubles; lse : [n_sel] natural-log sum-exp (may be NULL)
 */
int wfo_chunk_causal_attn_rows(int H, int D, int L,
                               const uint16_t *q, const int64_t *q_chunk,
                               const uint16_t *k, const uint16_t *v,
                               const int64_t *k_chunk, int n_kchunks,
                               int n_sel, const int32_t *rows, const int32_t *heads,
                               double *o, double *lse)
{
    const long nk = (long)n_kchunks * L;
    const double scale = 1.0 / sqrt((double)D);
    int bad = 0;
#pragma omp parallel
    {
        double *qd = (double *)malloc(sizeof(double) * D);
        double *s = (double *)malloc(sizeof(double) * (nk > 0 ? nk : 1));
        unsigned char *vis = (unsigned char *)malloc(nk > 0 ? nk : 1);
        double *acc = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < n_sel; ++i) {
            const long n = rows[i];
            const int h = heads[i];
            const int64_t qid = q_chunk[n / L];
            for (int d = 0; d < D; ++d)
                qd[d] = bf16_bits_to_double(q[(n * H + h) * D + d]);
            double m = -INFINITY;
            long nvis = 0;
            for (long j = 0; j < nk; ++j) {
                vis[j] = k_chunk[j / L] <= qid;
                if (!vis[j]) continue;
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += qd[d] * bf16_bits_to_double(k[(j * H + h) * D + d]);
                s[j] = dot * scale;
                if (s[j] > m) m = s[j];
                ++nvis;
            }
            if (nvis == 0) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            double z = 0.0;
            for (int d = 0; d < D; ++d) acc[d] = 0.0;
            for (long j = 0; j < nk; ++j) {
                if (!vis[j]) continue;
                double w = exp(s[j] - m);
                z += w;
                for (int d = 0; d < D; ++d)
                    acc[d] += w * bf16_bits_to_double(v[(j * H + h) * D + d]);
            }
            for (int d = 0; d < D; ++d) o[(long)i * D + d] = acc[d] / z;
            if (lse) lse[i] = m + log(z);
        }
        free(qd); free(s); free(vis); free(acc);
    }
    return bad ? -2 : 0;
}

/* ---- E4M3 ---------------------------------------------------------------- */

static double e4m3_value(uint8_t c)
{
    const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    const double v = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

static uint8_t e4m3_from_double(double x)
{
    if (isnan(x)) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    const double a = fabs(x);
    if (a >= 448.0) return sign | 0x7E;
    int e;
    frexp(a, &e);                          /* a = f * 2^e, f in [0.5, 1) */
    int E = e - 1;                         /* floor(log2 a) */
    if (a == 0.0 || E < -6) E = -6;        /* subnormal range: quantum 2^-9 */
    const double quantum = ldexp(1.0, E - 3);
    const double r = nearbyint(a / quantum);   /* exact quotient, ties to even */
    const double v = r * quantum;
    if (v == 0.0) return sign;
    int e2;
    frexp(v, &e2);
    const int E2 = e2 - 1;
    if (E2 < -6) return sign | (uint8_t)(v / ldexp(1.0, -9));
    const int mant = (int)(v / ldexp(1.0, E2) * 8.0) - 8;
    return sign | (uint8_t)((E2 + 7) << 3) | (uint8_t)mant;
}

void wfo_e4m3_decode(const uint8_t *in, double *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = e4m3_value(in[i]);
}

void wfo_e4m3_encode(const double *in, uint8_t *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = e4m3_from_double(in[i]);
}

/*
 * wfo_chunk_causal_attn_rows_fp8qk: as wfo_chunk_causal_attn_rows, with
 * q8      : [Tq, H, D] E4M3 codes, q_scale : [H, Tq] fp32
 * k8      : [n_kchunks*L, H, D] E4M3 codes, k_scale : [n_kchunks, ceil(L/128), H] fp32
 * v       : [n_kchunks*L, H, D] bf16 bits
 */
int wfo_chunk_causal_attn_rows_fp8qk(int H, int D, int L, int Tq,
                                     const uint8_t *q8, const float *q_scale,
                                     const int64_t *q_chunk,
                                     const uint8_t *k8, const float *k_scale,
                                     const uint16_t *v, const int64_t *k_chunk, int n_kchunks,
                                     int n_sel, const int32_t *rows, const int32_t *heads,
                                     double *o, double *lse)
{
    const long nk = (long)n_kchunks * L;
    const int nt = (L + 127) / 128;
    const double scale = 1.0 / sqrt((double)D);
    double table[256];
    for (int c = 0; c < 256; ++c) table[c] = e4m3_value((uint8_t)c);
    int bad = 0;
#pragma omp parallel
    {
        double *qd = (double *)malloc(sizeof(double) * D);
        double *s = (double *)malloc(sizeof(double) * (nk > 0 ? nk : 1));
        unsigned char *vis = (unsigned char *)malloc(nk > 0 ? nk : 1);
        double *acc = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < n_sel; ++i) {
            const long n = rows[i];
            const int h = heads[i];
            const int64_t qid = q_chunk[n / L];
            const double sq = (double)q_scale[(long)h * Tq + n];
            for (int d = 0; d < D; ++d) qd[d] = table[q8[(n * H + h) * D + d]] * sq;
            double m = -INFINITY;
            long nvis = 0;
            for (long j = 0; j < nk; ++j) {
                vis[j] = k_chunk[j / L] <= qid;
                if (!vis[j]) continue;
                const long b = j / L, t = (j % L) / 128;
                const double sk = (double)k_scale[(b * nt + t) * H + h];
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += qd[d] * (table[k8[(j * H + h) * D + d]] * sk);
                s[j] = dot * scale;
                if (s[j] > m) m = s[j];
                ++nvis;
            }
            if (nvis == 0) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            double z = 0.0;
            for (int d = 0; d < D; ++d) acc[d] = 0.0;
            for (long j = 0; j < nk; ++j) {
                if (!vis[j]) continue;
                double w = exp(s[j] - m);
                z += w;
                for (int d = 0; d < D; ++d)
                    acc[d] += w * bf16_bits_to_double(v[(j * H + h) * D + d]);
            }
            for (int d = 0; d < D; ++d) o[(long)i * D + d] = acc[d] / z;
            if (lse) lse[i] = m + log(z);
        }
        free(qd); free(s); free(vis); free(acc);
    }
    return bad ? -2 : 0;
}

int wfo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
