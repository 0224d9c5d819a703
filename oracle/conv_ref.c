/*
 * Oracle for the equivariant message-passing convolution: plain loops, fp64
 * accumulation.  TEST INFRASTRUCTURE ONLY: compiled by oracle/build.py and
 * called from the tests, smoke() and the CPU-baseline leg of bench.py.  It
 * shares no code with the CUDA library.
 *
 * Definition (e3j, abstract and Table 1: message-passing convolution of
 * MACE-style potentials; FlashCart App. B: sender features combined with the
 * direction tensors along admissible paths, radially weighted; §4 / App. D:
 * summed into the receiver, channel-diagonal):
 *
 *   y[i, o3+m3, c] = sum_{e: recv(e)=i} sum_p w[e,p,c]
 *                    sum_{m1,m2} C_p[m1,m2,m3] x[send(e), o1+m1, c] Y[e, o2+m2]
 *
 * and its gradients given gy:
 *   dx[j, o1+m1, c] = sum_{e: send(e)=j} sum_p w[e,p,c]
 *                     sum_{m2,m3} C_p[m1,m2,m3] Y[e,o2+m2] gy[recv(e), o3+m3, c]
 *   dw[e, p, c]     = sum_{m1,m2,m3} C_p x[send(e),o1+m1,c] Y[e,o2+m2] gy[recv(e),o3+m3,c]
 *   gY[e, o2+m2]    = sum_c sum_{p with this l2} w[e,p,c]
 *                     sum_{m1,m3} C_p x[send(e),o1+m1,c] gy[recv(e),o3+m3,c]
 *
 * Path descriptor pd[6p..6p+5] = (o1, d1, o2, d2, o3, d3) with d = 2l+1; the
 * coupling of path p is cg[cgo[p] + (m1*d2 + m2)*d3 + m3].  Y is given per
 * edge in fp64 (computed by oracle/sh.py).  Rows listed in `rows` are
 * computed; every output row is overwritten.
 */
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* y rows for the receivers in rows[0..n_rows): y_out[n][D_out][C] */
void oracle_forward(int C, int D_in, int D_sh, int D_out, int P, const int* pd,
                    const int64_t* cgo, const double* cg,
                    int n_rows, const int* rows, const int* recv_ptr, const int* recv_perm,
                    const int* senders, const float* x, const double* Y, const float* w,
                    double* y_out, int nthreads) {
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 16)
    for (int n = 0; n < n_rows; ++n) {
        const int i = rows[n];
        double* yi = y_out + (int64_t)n * D_out * C;
        memset(yi, 0, sizeof(double) * (size_t)D_out * C);
        for (int k = recv_ptr[i]; k < recv_ptr[i + 1]; ++k) {
            const int e = recv_perm[k];
            const int s = senders[e];
            const float* xs = x + (int64_t)s * D_in * C;
            const double* Ye = Y + (int64_t)e * D_sh;
            for (int p = 0; p < P; ++p) {
                const int o1 = pd[6 * p], d1 = pd[6 * p + 1], o2 = pd[6 * p + 2];
                const int d2 = pd[6 * p + 3], o3 = pd[6 * p + 4], d3 = pd[6 * p + 5];
                const double* Cp = cg + cgo[p];
                const float* wep = w + ((int64_t)e * P + p) * C;
                for (int m3 = 0; m3 < d3; ++m3)
                    for (int c = 0; c < C; ++c) {
                        double acc = 0.0;
                        for (int m1 = 0; m1 < d1; ++m1)
                            for (int m2 = 0; m2 < d2; ++m2)
                                acc += Cp[(m1 * d2 + m2) * d3 + m3] *
                                       (double)xs[(o1 + m1) * C + c] * Ye[o2 + m2];
                        yi[(o3 + m3) * C + c] += (double)wep[c] * acc;
                    }
            }
        }
    }
}

/* dx rows for the senders in rows[0..n_rows): dx_out[n][D_in][C] */
void oracle_backward_dx(int C, int D_in, int D_sh, int D_out, int P, const int* pd,
                        const int64_t* cgo, const double* cg,
                        int n_rows, const int* rows, const int* send_ptr, const int* send_perm,
                        const int* receivers, const float* gy, const double* Y, const float* w,
                        double* dx_out, int nthreads) {
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 16)
    for (int n = 0; n < n_rows; ++n) {
        const int j = rows[n];
        double* dxj = dx_out + (int64_t)n * D_in * C;
        memset(dxj, 0, sizeof(double) * (size_t)D_in * C);
        for (int k = send_ptr[j]; k < send_ptr[j + 1]; ++k) {
            const int e = send_perm[k];
            const int i = receivers[e];
            const float* gyi = gy + (int64_t)i * D_out * C;
            const double* Ye = Y + (int64_t)e * D_sh;
            for (int p = 0; p < P; ++p) {
                const int o1 = pd[6 * p], d1 = pd[6 * p + 1], o2 = pd[6 * p + 2];
                const int d2 = pd[6 * p + 3], o3 = pd[6 * p + 4], d3 = pd[6 * p + 5];
                const double* Cp = cg + cgo[p];
                const float* wep = w + ((int64_t)e * P + p) * C;
                for (int m1 = 0; m1 < d1; ++m1)
                    for (int c = 0; c < C; ++c) {
                        double acc = 0.0;
                        for (int m2 = 0; m2 < d2; ++m2)
                            for (int m3 = 0; m3 < d3; ++m3)
                                acc += Cp[(m1 * d2 + m2) * d3 + m3] * Ye[o2 + m2] *
                                       (double)gyi[(o3 + m3) * C + c];
                        dxj[(o1 + m1) * C + c] += (double)wep[c] * acc;
                    }
            }
        }
    }
}

/* dw and gY for the edges in edges[0..n): dw_out[n][P][C], gY_out[n][D_sh] */
void oracle_backward_edges(int C, int D_in, int D_sh, int D_out, int P, const int* pd,
                           const int64_t* cgo, const double* cg,
                           int n_edges, const int* edges, const int* senders, const int* receivers,
                           const float* x, const float* gy, const double* Y, const float* w,
                           double* dw_out, double* gY_out, int nthreads) {
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 64)
    for (int n = 0; n < n_edges; ++n) {
        const int e = edges[n];
        const int s = senders[e], i = receivers[e];
        const float* xs = x + (int64_t)s * D_in * C;
        const float* gyi = gy + (int64_t)i * D_out * C;
        const double* Ye = Y + (int64_t)e * D_sh;
        double* dwe = dw_out + (int64_t)n * P * C;
        double* gYe = gY_out + (int64_t)n * D_sh;
        memset(gYe, 0, sizeof(double) * (size_t)D_sh);
        for (int p = 0; p < P; ++p) {
            const int o1 = pd[6 * p], d1 = pd[6 * p + 1], o2 = pd[6 * p + 2];
            const int d2 = pd[6 * p + 3], o3 = pd[6 * p + 4], d3 = pd[6 * p + 5];
            const double* Cp = cg + cgo[p];
            const float* wep = w + ((int64_t)e * P + p) * C;
            for (int c = 0; c < C; ++c) {
                double dwv = 0.0;
                for (int m2 = 0; m2 < d2; ++m2) {
                    double g = 0.0;
                    for (int m1 = 0; m1 < d1; ++m1)
                        for (int m3 = 0; m3 < d3; ++m3)
                            g += Cp[(m1 * d2 + m2) * d3 + m3] * (double)xs[(o1 + m1) * C + c] *
                                 (double)gyi[(o3 + m3) * C + c];
                    dwv += g * Ye[o2 + m2];
                    gYe[o2 + m2] += (double)wep[c] * g;
                }
                dwe[p * C + c] = dwv;
            }
        }
    }
}
