/*
 * Test infrastructure only: the fp64 CPU oracle for the SSD layer forward.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * call it; the product path never links or loads this file.
 *
 * What it computes is the plain definition of the layer, the scalar-identity
 * selective SSM in its linear (recurrent) form ("Transformers are SSMs:
 * Generalized Models and Efficient Algorithms Through Structured State Space
 * Duality", Knowl 1, linear form), with the per-token step size dt and the
 * skip term D of the Mamba-2 layer:
 *
 *     a_t   = exp(dt_t * A_h)                          (a_t in [0,1] for A_h <= 0)
 *     h_t   = a_t * h_{t-1} + dt_t * x_t (outer) B_t   h_{-1} = initial state or 0
 *     y_t   = C_t . h_t + D_h * x_t
 *
 * per batch row b and head h, with group g = h / (H/G) supplying B and C
 * (Knowl 7, grouped-input pattern). The state is kept as [P][N] (head dim by
 * state dim), the layout of the library's state tensors; the pages write it
 * N x P, which is the same numbers transposed.
 *
 * All arithmetic is fp64 on inputs given as fp64 (the caller upcasts the stored
 * bf16/fp32 values exactly). One loop over time, no blocking, no reordering.
 * OpenMP runs independent (b, h) sequences in parallel; each sequence is still
 * one sequential loop, so the result does not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int ssd_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * x      [b, T, H, P]     dt [b, T, H]     A [H]
 * B, C   [b, T, G, N]     D  [H] or NULL (treated as 0)
 * init   [b, H, P, N] or NULL (h_{-1} = 0)
 * y      [b, T, H, P]     final [b, H, P, N] or NULL
 * chunk, entry [b, nc, H, P, N] or NULL: when given, entry[b, c, h] receives the
 *        state h_{cQ-1} entering chunk c (the state before token c*chunk), for
 *        c = 0 .. nc-1, nc = ceil(T / chunk).
 * bh_list [n_bh][2] or NULL: when given, only these (b, h) sequences are run and
 *        only their outputs are written.
 * Returns 0, or -1 on a bad argument or allocation failure.
 */
int ssd_oracle_recurrence(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                          int64_t ngroups, int64_t dstate,
                          const double* x, const double* dt, const double* A,
                          const double* B, const double* C, const double* D,
                          const double* init, double* y, double* final_states,
                          int64_t chunk, double* entry,
                          const int64_t* bh_list, int64_t n_bh)
{
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || ngroups <= 0 ||
        dstate <= 0 || nheads % ngroups != 0)
        return -1;
    if (entry && chunk <= 0) return -1;
    const int64_t T = seqlen, H = nheads, P = headdim, G = ngroups, N = dstate;
    const int64_t heads_per_group = H / G;
    const int64_t nc = entry ? (T + chunk - 1) / chunk : 0;
    const int64_t total = bh_list ? n_bh : batch * H;
    int failed = 0;

    #pragma omp parallel for schedule(dynamic, 1) reduction(|:failed)
    for (int64_t idx = 0; idx < total; ++idx) {
        const int64_t b = bh_list ? bh_list[2 * idx] : idx / H;
        const int64_t h = bh_list ? bh_list[2 * idx + 1] : idx % H;
        if (b < 0 || b >= batch || h < 0 || h >= H) { failed = 1; continue; }
        const int64_t g = h / heads_per_group;
        double* S = (double*)malloc(sizeof(double) * (size_t)(P * N));
        if (!S) { failed = 1; continue; }
        if (init) memcpy(S, init + (b * H + h) * P * N, sizeof(double) * (size_t)(P * N));
        else memset(S, 0, sizeof(double) * (size_t)(P * N));
        const double Dh = D ? D[h] : 0.0;

        for (int64_t t = 0; t < T; ++t) {
            if (entry && t % chunk == 0)
                memcpy(entry + ((b * nc + t / chunk) * H + h) * P * N, S,
                       sizeof(double) * (size_t)(P * N));
            const double dtv = dt[(b * T + t) * H + h];
            const double a = exp(dtv * A[h]);
            const double* xt = x + ((b * T + t) * H + h) * P;
            const double* Bt = B + ((b * T + t) * G + g) * N;
            const double* Ct = C + ((b * T + t) * G + g) * N;
            double* yt = y + ((b * T + t) * H + h) * P;
            for (int64_t p = 0; p < P; ++p) {
                const double u = dtv * xt[p];
                double* Sp = S + p * N;
                for (int64_t n = 0; n < N; ++n) Sp[n] = a * Sp[n] + u * Bt[n];
            }
            for (int64_t p = 0; p < P; ++p) {
                const double* Sp = S + p * N;
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) acc += Ct[n] * Sp[n];
                yt[p] = acc + Dh * xt[p];
            }
        }
        if (final_states)
            memcpy(final_states + (b * H + h) * P * N, S, sizeof(double) * (size_t)(P * N));
        free(S);
    }
    return failed ? -1 : 0;
}
