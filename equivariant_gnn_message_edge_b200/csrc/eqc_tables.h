// Compile-time coupling tables of the equivariant convolution.
//
// FlashCart (arXiv 2610.06409), App. B: an admissible path (l1, l2, l3)
// satisfies the triangle inequalities and its equivariant bilinear coupling is
// unique up to normalisation; the convolution uses natural-parity outputs.
// The coefficients are fixed here as:
//   * complex CG <l1 m1 l2 m2 | l3 m3> by the Racah formula (Condon-Shortley);
//   * real basis U^l (rows real m, columns complex mu):
//       m > 0: ((-1)^m |m> + |-m>)/sqrt2,  m = 0: |0>,  m < 0: i(|m> - (-1)^m |-m>)/sqrt2,
//     C[m1,m2,m3] = sum U3[m3,mu3] conj(U1[m1,mu1]) conj(U2[m2,mu2]) <..|..>
//     (real for natural-parity paths);
//   * sign: the first entry with |c| > 1e-9 in (m1, m2, m3) order is positive;
//   * orthonormal: sum_{m1,m2} C[m1,m2,m3] C[m1,m2,m3'] = delta.
// Everything is constexpr, so kernels read the coefficients as immediates and
// entries that are zero vanish at compile time; the host planner calls the
// same functions at run time.
#pragma once

#if defined(__CUDACC__)
#define EQC_HD __host__ __device__
#else
#define EQC_HD
#endif

namespace eqc {

constexpr int kMaxL = 3;
constexpr int kMaxPaths = 64;

struct cplx {
    double re, im;
};
constexpr cplx cmul(cplx a, cplx b) { return {a.re * b.re - a.im * b.im, a.re * b.im + a.im * b.re}; }
constexpr cplx cconj(cplx a) { return {a.re, -a.im}; }

constexpr double cfact(int n) {
    double r = 1.0;
    for (int i = 2; i <= n; ++i) r *= (double)i;
    return r;
}

// Newton iteration from above; stops when it no longer decreases.
constexpr double csqrt(double x) {
    if (x <= 0.0) return 0.0;
    double r = x >= 1.0 ? x : 1.0;
    for (int i = 0; i < 400; ++i) {
        double n = 0.5 * (r + x / r);
        if (!(n < r)) break;
        r = n;
    }
    return r;
}

constexpr int iabs(int a) { return a < 0 ? -a : a; }

// <j1 m1 j2 m2 | J M> by the Racah formula.
constexpr double cg_complex(int j1, int m1, int j2, int m2, int J, int M) {
    if (m1 + m2 != M) return 0.0;
    if (J < iabs(j1 - j2) || J > j1 + j2) return 0.0;
    if (iabs(m1) > j1 || iabs(m2) > j2 || iabs(M) > J) return 0.0;
    double pref2 = (2.0 * J + 1.0) * cfact(J + j1 - j2) * cfact(J - j1 + j2) * cfact(j1 + j2 - J) /
                   cfact(j1 + j2 + J + 1);
    pref2 *= cfact(J + M) * cfact(J - M) * cfact(j1 - m1) * cfact(j1 + m1) * cfact(j2 - m2) *
             cfact(j2 + m2);
    double s = 0.0;
    for (int k = 0; k <= j1 + j2 + J; ++k) {
        const int a0 = k, a1 = j1 + j2 - J - k, a2 = j1 - m1 - k, a3 = j2 + m2 - k;
        const int a4 = J - j2 + m1 + k, a5 = J - j1 - m2 + k;
        if (a0 < 0 || a1 < 0 || a2 < 0 || a3 < 0 || a4 < 0 || a5 < 0) continue;
        const double den = cfact(a0) * cfact(a1) * cfact(a2) * cfact(a3) * cfact(a4) * cfact(a5);
        s += ((k & 1) ? -1.0 : 1.0) / den;
    }
    return csqrt(pref2) * s;
}

// Element U^l[m][mu] of the complex -> real change of basis.
constexpr cplx umat(int m, int mu) {
    const double r2 = 0.70710678118654752440;
    if (m > 0) {
        if (mu == m) return {(m & 1) ? -r2 : r2, 0.0};
        if (mu == -m) return {r2, 0.0};
        return {0.0, 0.0};
    }
    if (m == 0) return {mu == 0 ? 1.0 : 0.0, 0.0};
    if (mu == m) return {0.0, r2};
    if (mu == -m) return {0.0, (m & 1) ? r2 : -r2};
    return {0.0, 0.0};
}

struct CG3 {
    double v[2 * kMaxL + 1][2 * kMaxL + 1][2 * kMaxL + 1];  // [m1+l1][m2+l2][m3+l3]
    double max_imag;
};

constexpr CG3 make_real_cg(int l1, int l2, int l3) {
    CG3 t{};
    t.max_imag = 0.0;
    for (int m1 = -l1; m1 <= l1; ++m1)
        for (int m2 = -l2; m2 <= l2; ++m2)
            for (int m3 = -l3; m3 <= l3; ++m3) {
                cplx acc{0.0, 0.0};
                // U rows have nonzeros only at mu = +-m
                for (int s1 = 0; s1 < 2; ++s1)
                    for (int s2 = 0; s2 < 2; ++s2)
                        for (int s3 = 0; s3 < 2; ++s3) {
                            const int mu1 = s1 ? -m1 : m1, mu2 = s2 ? -m2 : m2, mu3 = s3 ? -m3 : m3;
                            if ((s1 && m1 == 0) || (s2 && m2 == 0) || (s3 && m3 == 0)) continue;
                            if (mu1 + mu2 != mu3) continue;
                            const double c = cg_complex(l1, mu1, l2, mu2, l3, mu3);
                            if (c == 0.0) continue;
                            cplx u = cmul(cmul(umat(m3, mu3), cconj(umat(m1, mu1))), cconj(umat(m2, mu2)));
                            acc.re += u.re * c;
                            acc.im += u.im * c;
                        }
                const double ai = acc.im < 0 ? -acc.im : acc.im;
                if (ai > t.max_imag) t.max_imag = ai;
                t.v[m1 + l1][m2 + l2][m3 + l3] = acc.re;
            }
    // clean rounding residue so that zero entries are exactly zero
    for (int a = 0; a < 2 * l1 + 1; ++a)
        for (int b = 0; b < 2 * l2 + 1; ++b)
            for (int c = 0; c < 2 * l3 + 1; ++c) {
                const double v = t.v[a][b][c];
                if (v < 1e-12 && v > -1e-12) t.v[a][b][c] = 0.0;
            }
    // canonical sign
    double first = 0.0;
    for (int a = 0; a < 2 * l1 + 1 && first == 0.0; ++a)
        for (int b = 0; b < 2 * l2 + 1 && first == 0.0; ++b)
            for (int c = 0; c < 2 * l3 + 1 && first == 0.0; ++c) {
                const double v = t.v[a][b][c];
                if (v > 1e-9 || v < -1e-9) first = v;
            }
    if (first < 0.0)
        for (int a = 0; a < 2 * l1 + 1; ++a)
            for (int b = 0; b < 2 * l2 + 1; ++b)
                for (int c = 0; c < 2 * l3 + 1; ++c) t.v[a][b][c] = -t.v[a][b][c];
    return t;
}

template <int L1, int L2, int L3>
struct RealCG {
    static constexpr CG3 t = make_real_cg(L1, L2, L3);
    static_assert(t.max_imag < 1e-12, "natural-parity coupling must be real");
};

// Natural-parity paths for irreps 0..LIN (in), SH degrees 0..LSH, 0..LOUT (out),
// ordered by (l1, l2, l3).
struct PathList {
    int n;
    int l1[kMaxPaths], l2[kMaxPaths], l3[kMaxPaths];
};

constexpr PathList make_paths(int LIN, int LSH, int LOUT) {
    PathList P{};
    P.n = 0;
    for (int a = 0; a <= LIN; ++a)
        for (int b = 0; b <= LSH; ++b)
            for (int c = 0; c <= LOUT; ++c)
                if (c >= iabs(a - b) && c <= a + b && ((a + b + c) & 1) == 0) {
                    P.l1[P.n] = a;
                    P.l2[P.n] = b;
                    P.l3[P.n] = c;
                    ++P.n;
                }
    return P;
}

// Offsets of each path's per-edge coupling matrix A_p[m3][m1] (paths with
// l2 > 0 only), each padded to a multiple of 4 floats.
struct AOffsets {
    int off[kMaxPaths];
    int total;
};

constexpr AOffsets make_aoffsets(const PathList& P) {
    AOffsets A{};
    int o = 0;
    for (int p = 0; p < P.n; ++p) {
        A.off[p] = o;
        if (P.l2[p] > 0) {
            const int sz = (2 * P.l1[p] + 1) * (2 * P.l3[p] + 1);
            o += (sz + 3) & ~3;
        }
    }
    A.total = o;
    return A;
}

}  // namespace eqc
