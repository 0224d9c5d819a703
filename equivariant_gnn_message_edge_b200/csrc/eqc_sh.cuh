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
