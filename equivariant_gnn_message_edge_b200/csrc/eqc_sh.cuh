// Real spherical harmonics of the edge direction, l <= 3, and the gradient
// contraction for dr (device code).
//
// FlashCart (arXiv 2610.06409) §2 and App. B: degree-l direction tensors are
// the degree-l real spherical tensors of the unit edge direction; forces are
// energy gradients.  Convention: component normalisation
// (sum_m Y_lm^2 = 2l+1), z polar, m > 0 ~ cos(m phi), m < 0 ~ sin(|m| phi),
// positive leading coefficients.  Y_lm(u) = P_lm(u) with P_lm the homogeneous
// Cartesian polynomials below, so for r = |r| u:
//     dY_lm/dr = (grad P_lm(u) - u (u . grad P_lm(u))) / |r|.
// Zero-length edges (|r|^2 < 1e-24): Y_0 = 1, Y_{l>0} = 0, dr = 0.
#pragma once

namespace eqc {

constexpr float kS3 = 1.7320508075688772f;     // sqrt(3)
constexpr float kS5 = 2.2360679774997897f;     // sqrt(5)
constexpr float kS15 = 3.8729833462074170f;    // sqrt(15)
constexpr float kH15 = 1.9364916731037085f;    // sqrt(15)/2
constexpr float kH5 = 1.1180339887498949f;     // sqrt(5)/2
constexpr float kA3 = 2.0916500663351889f;     // sqrt(35/2)/2
constexpr float kB3 = 10.246950765959598f;     // sqrt(105)
constexpr float kA1 = 1.6201851746019651f;     // sqrt(21/2)/2
constexpr float kC0 = 1.3228756555322954f;     // sqrt(7)/2
constexpr float kH105 = 5.1234753829797990f;   // sqrt(105)/2
constexpr float kZeroLen2 = 1e-24f;

// Unit direction and 1/|r|; returns false for a zero-length edge.
__device__ __forceinline__ bool unit_dir(float rx, float ry, float rz, float& x, float& y, float& z,
                                         float& inv_len) {
    const float r2 = fmaf(rx, rx, fmaf(ry, ry, rz * rz));
    if (r2 < kZeroLen2) {
        x = y = z = 0.f;
        inv_len = 0.f;
        return false;
    }
    inv_len = rsqrtf(r2);
    x = rx * inv_len;
    y = ry * inv_len;
    z = rz * inv_len;
    return true;
}

// Y[0 .. (L+1)^2) of the unit vector (x, y, z); ok = false gives Y_0 = 1 only.
template <int L>
__device__ __forceinline__ void sh_eval(bool ok, float x, float y, float z, float* Y) {
    Y[0] = 1.f;
    if constexpr (L >= 1) {
        Y[1] = kS3 * y;
        Y[2] = kS3 * z;
        Y[3] = kS3 * x;
    }
    if constexpr (L >= 2) {
        const float xx = x * x, yy = y * y, zz = z * z;
        Y[4] = kS15 * x * y;
        Y[5] = kS15 * y * z;
        Y[6] = kH5 * (2.f * zz - xx - yy);
        Y[7] = kS15 * x * z;
        Y[8] = kH15 * (xx - yy);
    }
    if constexpr (L >= 3) {
        const float xx = x * x, yy = y * y, zz = z * z;
        Y[9] = kA3 * y * (3.f * xx - yy);
        Y[10] = kB3 * x * y * z;
        Y[11] = kA1 * y * (4.f * zz - xx - yy);
        Y[12] = kC0 * z * (2.f * zz - 3.f * xx - 3.f * yy);
        Y[13] = kA1 * x * (4.f * zz - xx - yy);
        Y[14] = kH105 * z * (xx - yy);
        Y[15] = kA3 * x * (xx - 3.f * yy);
    }
    if (!ok) {
#pragma unroll
        for (int k = 1; k < (L + 1) * (L + 1); ++k) Y[k] = 0.f;
    }
}

// dr = (dY/dr)^T gY, with gY[k-1] the gradient w.r.t. Y[k], k = 1 .. (L+1)^2-1.
template <int L>
__device__ __forceinline__ void sh_grad_contract(bool ok, float x, float y, float z, float inv_len,
                                                 const float* gY, float& dx, float& dy, float& dz) {
    float gx = 0.f, gy = 0.f, gz = 0.f;
    if constexpr (L >= 1) {
        gy = fmaf(kS3, gY[0], gy);
        gz = fmaf(kS3, gY[1], gz);
        gx = fmaf(kS3, gY[2], gx);
    }
    if constexpr (L >= 2) {
        const float a = gY[3], b = gY[4], c = gY[5], d = gY[6], e = gY[7];
        // xy, yz, (sqrt5/2)(2z^2-x^2-y^2), xz, (x^2-y^2)
        gx += kS15 * (a * y + d * z + e * x) - kS5 * c * x;
        gy += kS15 * (a * x + b * z - e * y) - kS5 * c * y;
        gz += kS15 * (b * y + d * x) + 2.f * kS5 * c * z;
    }
    if constexpr (L >= 3) {
        const float xx = x * x, yy = y * y, zz = z * z;
        const float a = gY[8], b = gY[9], c = gY[10], d = gY[11], e = gY[12], f = gY[13], g = gY[14];
        // -3: a3 (3x^2 y - y^3)        grad a3 (6xy, 3x^2-3y^2, 0)
        // -2: b3 xyz                   grad b3 (yz, xz, xy)
        // -1: a1 (4yz^2 - x^2 y - y^3) grad a1 (-2xy, 4z^2-x^2-3y^2, 8yz)
        //  0: c0 (2z^3 - 3x^2 z - 3y^2 z) grad c0 (-6xz, -6yz, 6z^2-3x^2-3y^2)
        //  1: a1 (4xz^2 - x^3 - xy^2) grad a1 (4z^2-3x^2-y^2, -2xy, 8xz)
        //  2: h105 (x^2 z - y^2 z)      grad h105 (2xz, -2yz, x^2-y^2)
        //  3: a3 (x^3 - 3xy^2)         grad a3 (3x^2-3y^2, -6xy, 0)
        gx += kA3 * (6.f * x * y * a + (3.f * xx - 3.f * yy) * g) + kB3 * y * z * b +
              kA1 * (-2.f * x * y * c + (4.f * zz - 3.f * xx - yy) * e) + kC0 * (-6.f * x * z) * d +
              kH105 * (2.f * x * z) * f;
        gy += kA3 * ((3.f * xx - 3.f * yy) * a - 6.f * x * y * g) + kB3 * x * z * b +
              kA1 * ((4.f * zz - xx - 3.f * yy) * c - 2.f * x * y * e) + kC0 * (-6.f * y * z) * d +
              kH105 * (-2.f * y * z) * f;
        gz += kB3 * x * y * b + kA1 * (8.f * y * z * c + 8.f * x * z * e) +
              kC0 * (6.f * zz - 3.f * xx - 3.f * yy) * d + kH105 * (xx - yy) * f;
    }
    if (!ok) {
        dx = dy = dz = 0.f;
        return;
    }
    const float ug = fmaf(x, gx, fmaf(y, gy, z * gz));
    dx = (gx - ug * x) * inv_len;
    dy = (gy - ug * y) * inv_len;
    dz = (gz - ug * z) * inv_len;
}

}  // namespace eqc

// ------------------------------------------------ directional derivatives
//
// The double backward needs rho = (dY/dr) q (a Jacobian-vector product) and
// H q = d/dr [(dY/dr)^T g] q (a Hessian-vector product).  Both are the
// derivative part of the first-order formulas evaluated at r + eps q in dual
// numbers (a + b eps, eps^2 = 0), so the polynomials are written once, for a
// generic scalar type.

namespace eqc {

struct Dual {
    float v, d;
};
__host__ __device__ __forceinline__ Dual operator+(Dual a, Dual b) { return {a.v + b.v, a.d + b.d}; }
__host__ __device__ __forceinline__ Dual operator-(Dual a, Dual b) { return {a.v - b.v, a.d - b.d}; }
__host__ __device__ __forceinline__ Dual operator*(Dual a, Dual b) { return {a.v * b.v, a.v * b.d + a.d * b.v}; }
__host__ __device__ __forceinline__ Dual operator*(float s, Dual a) { return {s * a.v, s * a.d}; }
__host__ __device__ __forceinline__ Dual operator*(Dual a, float s) { return {s * a.v, s * a.d}; }
__host__ __device__ __forceinline__ Dual operator-(float s, Dual a) { return {s - a.v, -a.d}; }
__host__ __device__ __forceinline__ Dual operator+(Dual a, float s) { return {a.v + s, a.d}; }

__device__ __forceinline__ float rsqrt_any(float a) { return rsqrtf(a); }
__device__ __forceinline__ Dual rsqrt_any(Dual a) {
    const float s = rsqrtf(a.v);
    return {s, -0.5f * a.d * s * s * s};
}

// Y[1 .. (L+1)^2) of a unit vector (x, y, z) in scalar type T (the same
// polynomials as sh_eval).
template <int L, class T>
__device__ __forceinline__ void sh_poly(T x, T y, T z, T* Y) {
    if constexpr (L >= 1) {
        Y[1] = kS3 * y;
        Y[2] = kS3 * z;
        Y[3] = kS3 * x;
    }
    if constexpr (L >= 2) {
        const T xx = x * x, yy = y * y, zz = z * z;
        Y[4] = kS15 * (x * y);
        Y[5] = kS15 * (y * z);
        Y[6] = kH5 * (2.f * zz - xx - yy);
        Y[7] = kS15 * (x * z);
        Y[8] = kH15 * (xx - yy);
    }
    if constexpr (L >= 3) {
        const T xx = x * x, yy = y * y, zz = z * z;
        Y[9] = kA3 * (y * (3.f * xx - yy));
        Y[10] = kB3 * (x * (y * z));
        Y[11] = kA1 * (y * (4.f * zz - xx - yy));
        Y[12] = kC0 * (z * (2.f * zz - 3.f * xx - 3.f * yy));
        Y[13] = kA1 * (x * (4.f * zz - xx - yy));
        Y[14] = kH105 * (z * (xx - yy));
        Y[15] = kA3 * (x * (xx - 3.f * yy));
    }
}

// grad_u sum_k g[k-1] P_k(u), k = 1 .. (L+1)^2-1, in scalar type T (the same
// gradient as sh_grad_contract before the tangential projection).
template <int L, class T>
__device__ __forceinline__ void sh_poly_grad(T x, T y, T z, const float* g, T& gx, T& gy, T& gz) {
    gx = T{0.f};
    gy = T{0.f};
    gz = T{0.f};
    if constexpr (L >= 1) {
        gy = gy + kS3 * g[0];
        gz = gz + kS3 * g[1];
        gx = gx + kS3 * g[2];
    }
    if constexpr (L >= 2) {
        const float a = g[3], b = g[4], c = g[5], d = g[6], e = g[7];
        gx = gx + kS15 * (a * y + d * z + e * x) - (kS5 * c) * x;
        gy = gy + kS15 * (a * x + b * z - e * y) - (kS5 * c) * y;
        gz = gz + kS15 * (b * y + d * x) + (2.f * kS5 * c) * z;
    }
    if constexpr (L >= 3) {
        const T xx = x * x, yy = y * y, zz = z * z;
        const float a = g[8], b = g[9], c = g[10], d = g[11], e = g[12], f = g[13], h = g[14];
        gx = gx + kA3 * ((6.f * a) * (x * y) + h * (3.f * xx - 3.f * yy)) + (kB3 * b) * (y * z) +
             kA1 * ((-2.f * c) * (x * y) + e * (4.f * zz - 3.f * xx - yy)) + (-6.f * kC0 * d) * (x * z) +
             (2.f * kH105 * f) * (x * z);
        gy = gy + kA3 * (a * (3.f * xx - 3.f * yy) - (6.f * h) * (x * y)) + (kB3 * b) * (x * z) +
             kA1 * (c * (4.f * zz - xx - 3.f * yy) - (2.f * e) * (x * y)) + (-6.f * kC0 * d) * (y * z) +
             (-2.f * kH105 * f) * (y * z);
        gz = gz + (kB3 * b) * (x * y) + kA1 * ((8.f * c) * (y * z) + (8.f * e) * (x * z)) +
             (kC0 * d) * (6.f * zz - 3.f * xx - 3.f * yy) + (kH105 * f) * (xx - yy);
    }
}

// rho[k] = dY_k/dr . q for k = 0 .. (L+1)^2-1 (rho[0] = 0; all zero for a
// zero-length edge).
template <int L>
__device__ __forceinline__ void sh_jvp(float rx, float ry, float rz, float qx, float qy, float qz, float* rho) {
    constexpr int D = (L + 1) * (L + 1);
    rho[0] = 0.f;
    const Dual X{rx, qx}, Yv{ry, qy}, Z{rz, qz};
    const Dual r2 = X * X + Yv * Yv + Z * Z;
    if (r2.v < kZeroLen2) {
#pragma unroll
        for (int k = 1; k < D; ++k) rho[k] = 0.f;
        return;
    }
    const Dual il = rsqrt_any(r2);
    Dual P[D > 1 ? D : 2];
    sh_poly<L, Dual>(X * il, Yv * il, Z * il, P);
#pragma unroll
    for (int k = 1; k < D; ++k) rho[k] = P[k].d;
}

// (dY/dr)^T g and H(r; g) q = d/dr[(dY/dr)^T g] q, with g[k-1] the weight of
// Y_k (k >= 1); both zero for a zero-length edge.
template <int L>
__device__ __forceinline__ void sh_grad_and_hvp(float rx, float ry, float rz, float qx, float qy, float qz,
                                                const float* g, float* grad, float* hq) {
    const Dual X{rx, qx}, Yv{ry, qy}, Z{rz, qz};
    const Dual r2 = X * X + Yv * Yv + Z * Z;
    if (L == 0 || r2.v < kZeroLen2) {
        grad[0] = grad[1] = grad[2] = hq[0] = hq[1] = hq[2] = 0.f;
        return;
    }
    const Dual il = rsqrt_any(r2);
    const Dual ux = X * il, uy = Yv * il, uz = Z * il;
    Dual gx, gy, gz;
    sh_poly_grad<L, Dual>(ux, uy, uz, g, gx, gy, gz);
    const Dual ug = ux * gx + uy * gy + uz * gz;
    const Dual dx = (gx - ug * ux) * il, dy = (gy - ug * uy) * il, dz = (gz - ug * uz) * il;
    grad[0] = dx.v;
    grad[1] = dy.v;
    grad[2] = dz.v;
    hq[0] = dx.d;
    hq[1] = dy.d;
    hq[2] = dz.d;
}

}  // namespace eqc
