/*
 * Gated DeltaNet token mixer -- fp64 sequential CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg do. It shares no code with the CUDA library.
 *
 * What it computes (the plain definition, token by token, no chunking):
 *
 *   The Herbert pages name the Gated DeltaNet mixer and its recurrence as one
 *   of the engine's computation families ("On descend d'un cran", section
 *   "Ce que fait le moteur"; "On descend d'un cran : #001 un compilateur pour
 *   moteur de LLM", section "Un compilateur, pas une bibliothèque de
 *   kernels") and fuse its whole decode step into one launch ("One level
 *   down: #004 the same compiler on Apple's chips", section "Decode"), but
 *   they never print its equation. This oracle takes the gated delta rule
 *   of the Gated DeltaNet layer as the definition, per sequence n and value
 *   head h, with state S of shape d_v x d_k:
 *
 *       q^_t = q_t / sqrt(|q_t|^2 + eps) * scale      (scale = d_k^-1/2 by default)
 *       k^_t = k_t / sqrt(|k_t|^2 + eps)
 *       alpha_t = exp(g_t)                             (g is the log-decay, <= 0)
 *       S_t = alpha_t S_{t-1} (I - beta_t k^_t k^_t^T) + beta_t v_t k^_t^T
 *       o_t = S_t q^_t                                 (read after the update)
 *
 *   S_{t-1}(I - beta k k^T) is evaluated as S - beta (S k) k^T, which is the
 *   same product written without forming the d_k x d_k matrix.
 *
 *   Value head h reads query/key head floor(h / (Hv/Hqk)) (contiguous groups).
 *   Varlen sequences are packed token-major; sequence n owns the tokens
 *   [cu_seqlens[n], cu_seqlens[n+1]) and starts from state_in[n] (or zero).
 *
 * Precision: every value is an fp64 widening of the exact inputs the GPU is
 * given; arithmetic is IEEE fp64 (build without fast-math), so the only
 * differences from exact arithmetic are fp64 rounding.
 *
 * Layouts (row-major, innermost last):
 *   q, k      [T_total, Hqk, d_k]
 *   v         [T_total, Hv, d_v]
 *   g, beta   [T_total, Hv]
 *   state     [N, Hv, d_v, d_k]
 *   o         [T_total, Hv, d_v]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* out = x / sqrt(sum x^2 + eps) * scale */
static void l2_normalise(const double *x, int d, double eps, double scale, double *out)
{
    double ss = 0.0;
    for (int i = 0; i < d; ++i) ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss + eps);
    for (int i = 0; i < d; ++i) out[i] = x[i] * inv * scale;
}

/*
 * One token of the recurrence on one (sequence, value head) state.
 * S [dv][dk] is updated in place; o [dv] receives S_t q^_t.
 * q, k are the raw (unnormalised) vectors; work must hold 3*dk + dv doubles.
 */
static void delta_rule_step(double *S, int dk, int dv,
                            const double *q, const double *k, const double *v,
                            double g, double beta, double scale, double eps,
                            double *o, double *work)
{
    double *qh = work;           /* [dk] */
    double *kh = work + dk;      /* [dk] */
    double *sk = work + 2 * dk;  /* [dv] : S_{t-1} k^ */
    l2_normalise(q, dk, eps, scale, qh);
    l2_normalise(k, dk, eps, 1.0, kh);
    double alpha = exp(g);

    for (int i = 0; i < dv; ++i) {
        const double *row = S + (size_t)i * dk;
        double acc = 0.0;
        for (int j = 0; j < dk; ++j) acc += row[j] * kh[j];
        sk[i] = acc;
    }
    /* S <- alpha * (S - beta (S k^) k^T) + beta v k^T */
    for (int i = 0; i < dv; ++i) {
        double *row = S + (size_t)i * dk;
        double a = beta * sk[i];
        double b = beta * v[i];
        for (int j = 0; j < dk; ++j)
            row[j] = alpha * (row[j] - a * kh[j]) + b * kh[j];
    }
    /* o = S_t q^ */
    for (int i = 0; i < dv; ++i) {
        const double *row = S + (size_t)i * dk;
        double acc = 0.0;
        for (int j = 0; j < dk; ++j) acc += row[j] * qh[j];
        o[i] = acc;
    }
}

/*
 * Prefill over packed sequences. Only value heads in [h_lo, h_hi) are
 * computed; o and state_out entries of other heads are left untouched, so a
 * caller can check a sample of heads of a large problem.
 * state_in may be NULL (zero initial state). Returns 0, or -1 on bad sizes.
 */
int gdn_oracle_prefill(const double *q, const double *k, const double *v,
                       const double *g, const double *beta,
                       const double *state_in, const int64_t *cu_seqlens,
                       int n_seqs, int Hqk, int Hv, int dk, int dv,
                       double scale, double eps, int h_lo, int h_hi,
                       double *o, double *state_out, int n_threads)
{
    if (n_seqs < 0 || Hqk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0) return -1;
    if (Hv % Hqk != 0) return -1;
    if (h_lo < 0 || h_hi > Hv || h_lo > h_hi) return -1;
    for (int n = 0; n < n_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    const int group = Hv / Hqk;
    const int nh = h_hi - h_lo;
    const long pairs = (long)n_seqs * nh;
    if (n_threads <= 0) n_threads = 1;

#pragma omp parallel num_threads(n_threads)
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)dv * dk);
        double *work = (double *)malloc(sizeof(double) * (size_t)(3 * dk + dv));
#pragma omp for schedule(dynamic, 1)
        for (long p = 0; p < pairs; ++p) {
            int n = (int)(p / nh);
            int h = h_lo + (int)(p % nh);
            int hq = h / group;
            size_t sbase = ((size_t)n * Hv + h) * (size_t)dv * dk;
            if (state_in)
                memcpy(S, state_in + sbase, sizeof(double) * (size_t)dv * dk);
            else
                memset(S, 0, sizeof(double) * (size_t)dv * dk);
            for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
                delta_rule_step(S, dk, dv,
                                q + ((size_t)t * Hqk + hq) * dk,
                                k + ((size_t)t * Hqk + hq) * dk,
                                v + ((size_t)t * Hv + h) * dv,
                                g[(size_t)t * Hv + h], beta[(size_t)t * Hv + h],
                                scale, eps,
                                o + ((size_t)t * Hv + h) * dv, work);
            }
            memcpy(state_out + sbase, S, sizeof(double) * (size_t)dv * dk);
        }
        free(work);
        free(S);
    }
    return 0;
}

/*
 * One decode step for B independent sequences (one token each). state
 * [B, Hv, dv, dk] is updated in place for value heads in [h_lo, h_hi);
 * o [B, Hv, dv] receives S_t q^_t for those heads.
 */
/*
 * x rounded to the nearest bfloat16, ties to even, by way of the nearest
 * float (the value a computation carried in float would round): the 16 low
 * bits of the float are dropped after adding half an ulp of the kept part
 * plus its lowest bit. Infinities and NaN pass through.
 */
static double round_to_bf16(double x)
{
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u) return (double)f;
    u += 0x7fffu + ((u >> 16) & 1u);
    u &= 0xffff0000u;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* The rounding above over n values (exported so that tests can pin it). */
void gdn_oracle_round_bf16(const double *x, double *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = round_to_bf16(x[i]);
}

/*
 * One decode step (see gdn_oracle_decode). With round_state_bf16 the updated
 * state is stored rounded to bfloat16 -- the storage contract of the Metal
 * article ("One level down: #004 the same compiler on Apple's chips", section
 * "In short": states kept in bf16, arithmetic in f32) -- after o has been
 * read from the unrounded state.
 */
int gdn_oracle_decode_ex(const double *q, const double *k, const double *v,
                         const double *g, const double *beta, double *state,
                         int B, int Hqk, int Hv, int dk, int dv,
                         double scale, double eps, int h_lo, int h_hi,
                         double *o, int n_threads, int round_state_bf16)
{
    if (B < 0 || Hqk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0) return -1;
    if (Hv % Hqk != 0) return -1;
    if (h_lo < 0 || h_hi > Hv || h_lo > h_hi) return -1;
    const int group = Hv / Hqk;
    const int nh = h_hi - h_lo;
    const long pairs = (long)B * nh;
    if (n_threads <= 0) n_threads = 1;

#pragma omp parallel num_threads(n_threads)
    {
        double *work = (double *)malloc(sizeof(double) * (size_t)(3 * dk + dv));
#pragma omp for schedule(static)
        for (long p = 0; p < pairs; ++p) {
            int b = (int)(p / nh);
            int h = h_lo + (int)(p % nh);
            int hq = h / group;
            delta_rule_step(state + ((size_t)b * Hv + h) * (size_t)dv * dk, dk, dv,
                            q + ((size_t)b * Hqk + hq) * dk,
                            k + ((size_t)b * Hqk + hq) * dk,
                            v + ((size_t)b * Hv + h) * dv,
                            g[(size_t)b * Hv + h], beta[(size_t)b * Hv + h],
                            scale, eps, o + ((size_t)b * Hv + h) * dv, work);
            if (round_state_bf16) {
                double *S = state + ((size_t)b * Hv + h) * (size_t)dv * dk;
                for (size_t e = 0; e < (size_t)dv * dk; ++e) S[e] = round_to_bf16(S[e]);
            }
        }
        free(work);
    }
    return 0;
}

int gdn_oracle_decode(const double *q, const double *k, const double *v,
                      const double *g, const double *beta, double *state,
                      int B, int Hqk, int Hv, int dk, int dv,
                      double scale, double eps, int h_lo, int h_hi,
                      double *o, int n_threads)
{
    return gdn_oracle_decode_ex(q, k, v, g, beta, state, B, Hqk, Hv, dk, dv, scale, eps, h_lo, h_hi, o,
                                n_threads, 0);
}

/* Number of threads OpenMP would use by default (for reporting). */
int gdn_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
