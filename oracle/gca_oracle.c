/*
 * CPU oracle core: plain fp64 softmax attention over an explicit key set.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference arm may load this library.  It shares no code,
 * header or constant with the CUDA library.
 *
 * What it computes (LingBot-Map paper digest, §2.5 "attention mask" table and
 * §2.2 frame types; the key set is chosen by the Python side of the oracle
 * from those visibility rules):
 *
 *     s_u   = scale * <q_r,h , k_u,h>                 for every key u
 *     O_r,h = sum_u exp(s_u - max s) v_u,h / sum_u exp(s_u - max s)
 *     lse   = max s + ln(sum_u exp(s_u - max s))       (natural log)
 *
 * Inputs are float32 arrays holding exact copies of the bf16 or fp32 stream
 * values; every product and sum is formed in double.  Two passes over the
 * keys (scores, then weighted sum) — no blocking, no online rescaling.
 *
 * Layouts: q [nq][H][D] (token-major, as streamed), k and v [H][nk][D]
 * (head-major, so one (row, head) pair scans contiguous memory),
 * out [nq][H][D] double, lse [nq][H] double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int gca_oracle_attention(const float* q, int64_t nq, const float* k, const float* v,
                         int64_t nk, int32_t H, int32_t D, double scale,
                         double* out, double* lse)
{
    if (nq < 0 || nk <= 0 || H <= 0 || D <= 0) return 1;
    int failed = 0;
#pragma omp parallel reduction(| : failed)
    {
        double* s = (double*)malloc((size_t)nk * sizeof(double));
        double* acc = (double*)malloc((size_t)D * sizeof(double));
        if (!s || !acc) {
            failed = 1;
        } else {
#pragma omp for collapse(2) schedule(dynamic, 1)
            for (int64_t r = 0; r < nq; ++r) {
                for (int32_t h = 0; h < H; ++h) {
                    const float* qr = q + ((size_t)r * H + h) * D;
                    const float* kh = k + (size_t)h * nk * D;
                    const float* vh = v + (size_t)h * nk * D;
                    double mx = -INFINITY;
                    for (int64_t u = 0; u < nk; ++u) {
                        const float* ku = kh + (size_t)u * D;
                        double dot = 0.0;
                        for (int32_t d = 0; d < D; ++d) dot += (double)qr[d] * (double)ku[d];
                        s[u] = scale * dot;
                        if (s[u] > mx) mx = s[u];
                    }
                    double sum = 0.0;
                    for (int64_t u = 0; u < nk; ++u) {
                        s[u] = exp(s[u] - mx);
                        sum += s[u];
                    }
                    for (int32_t d = 0; d < D; ++d) acc[d] = 0.0;
                    for (int64_t u = 0; u < nk; ++u) {
                        const float* vu = vh + (size_t)u * D;
                        const double p = s[u];
                        for (int32_t d = 0; d < D; ++d) acc[d] += p * (double)vu[d];
                    }
                    double* o = out + ((size_t)r * H + h) * D;
                    for (int32_t d = 0; d < D; ++d) o[d] = acc[d] / sum;
                    if (lse) lse[(size_t)r * H + h] = mx + log(sum);
                }
            }
        }
        free(s);
        free(acc);
    }
    return failed;
}

/* Threads the OpenMP runtime will use (for reporting the CPU baseline). */
int gca_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
