// Compile-time coupling tables of the equivariant convolution.
//
// FlashCart (arXiv 2610.06409), App. B: an admissible path (l1, l2, l3)
// satisfies the triangle inequalities and its equivariant bilinear coupling is
// unique up to normalisation.  Natural-parity outputs take the paths with an
// even l1 + l2 + l3; both-parity outputs also take the odd ones (the
// antisymmetric couplings, e.g. 1 x 1 -> 1 is the cross product).
// The coefficients are fixed here as:
//   * complex CG <l1 m1 l2 m2 | l3 m3> by the Racah formula (Condon-Shortley);
//   * real basis U^l (rows real m, columns complex mu):
//       m > 0: ((-1)^m |m> + |-m>)/sqrt2,  m = 0: |0>,  m < 0: i(|m> - (-1)^m |-m>)/sqrt2,
//     C[m1,m2,m3] = sum U3[m3,mu3] conj(U1[m1,mu1]) conj(U2[m2,mu2]) <..|..>
//     (real when l1 + l2 + l3 is even, imaginary when it is odd: the
//     coupling is its real or its imaginary part);
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
    double max_dropped;   // largest |part| that must vanish (imag if even, real if odd)
};

constexpr CG3 make_real_cg(int l1, int l2, int l3) {
    CG3 t{};
    t.max_dropped = 0.0;
    const bool odd = ((l1 + l2 + l3) & 1) != 0;
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
                const double drop = odd ? acc.re : acc.im;
                const double ad = drop < 0 ? -drop : drop;
                if (ad > t.max_dropped) t.max_dropped = ad;
                t.v[m1 + l1][m2 + l2][m3 + l3] = odd ? acc.im : acc.re;
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
    static_assert(t.max_dropped < 1e-12, "coupling must be purely real or purely imaginary");
};

// Output variants (bits of the plan's mode):
//   kModeAllParity - outputs of both parities for every l3 >= 1, laid out
//                    0e, 1o, 1e, 2e, 2o, 3o, 3e (natural parity first; 0o has
//                    no path from natural-parity inputs), and the paths with
//                    odd l1 + l2 + l3 that reach the second block of each l3;
//   kModePerPath   - every path writes its own output block, in path order
//                    (no summation over paths that share an output irrep).
constexpr int kModeAllParity = 1;
constexpr int kModePerPath = 2;

// Row offset of output irrep (l, natural or not) in the summed layouts.
constexpr int out_row(int l, bool natural, int mode) {
    if (!(mode & kModeAllParity)) return l * l;
    if (l == 0) return 0;
    return natural ? 2 * l * l - 1 : 2 * l * l + 2 * l;
}

// Paths for natural-parity inputs 0..LIN, SH degrees 0..LSH and outputs of
// degree 0..LOUT, ordered by (l1, l2, l3); o3 is the path's output row and
// dout the row count of the output layout.
struct PathList {
    int n, dout;
    int l1[kMaxPaths], l2[kMaxPaths], l3[kMaxPaths], o3[kMaxPaths];
};

constexpr PathList make_paths(int LIN, int LSH, int LOUT, int MODE = 0) {
    PathList P{};
    P.n = 0;
    int row = 0;
    for (int a = 0; a <= LIN; ++a)
        for (int b = 0; b <= LSH; ++b)
            for (int c = 0; c <= LOUT; ++c) {
                const bool natural = ((a + b + c) & 1) == 0;
                if (c < iabs(a - b) || c > a + b) continue;
                if (!natural && !(MODE & kModeAllParity)) continue;
                P.l1[P.n] = a;
                P.l2[P.n] = b;
                P.l3[P.n] = c;
                P.o3[P.n] = (MODE & kModePerPath) ? row : out_row(c, natural, MODE);
                row += 2 * c + 1;
                ++P.n;
            }
    if (MODE & kModePerPath)
        P.dout = row;
    else
        P.dout = (MODE & kModeAllParity) ? (LOUT == 0 ? 1 : 2 * (LOUT + 1) * (LOUT + 1) - 1)
                                         : (LOUT + 1) * (LOUT + 1);
    return P;
}

// Paths of the symmetric product of one natural-parity feature with itself
// (correlation order 2): unordered pairs l1 <= l2 <= LA, outputs L <= LOUT,
// triangle rule, l1 + l2 + L even (the odd couplings of equal inputs vanish
// and (l2, l1, L) equals (l1, l2, L) on the symmetric product), ordered by
// (l1, l2, L); o3 = L^2 (outputs summed by irrep).
constexpr PathList make_sym_paths(int LA, int LOUT) {
    PathList P{};
    P.n = 0;
    for (int a = 0; a <= LA; ++a)
        for (int b = a; b <= LA; ++b)
            for (int c = 0; c <= LOUT; ++c) {
                if (c < iabs(a - b) || c > a + b || ((a + b + c) & 1)) continue;
                P.l1[P.n] = a;
                P.l2[P.n] = b;
                P.l3[P.n] = c;
                P.o3[P.n] = c * c;
                ++P.n;
            }
    P.dout = (LOUT + 1) * (LOUT + 1);
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
