// Host-side NVFP4 encoding of a weight matrix: 4-bit E2M1 codes, one E4M3
// scale byte per 16 elements along K and an fp32 scale for the tensor
// ("Compression", section "NVFP4: 3.18x smaller weights": packed 4-bit weights
// plus one float8_e4m3fn block scale per 16 elements, 0.5625 bytes per
// element, quantised at load time).
//
// Rounding is to nearest, ties to even, on the exact fp64 quotients: the
// significand of a quotient scaled into [1, 2) is multiplied by 8 (E4M3) or 2
// (E2M1), which is exact, and rounded with nearbyint in the default rounding
// mode.  A carry out of the mantissa moves to the next binade; results
// saturate at the format's largest finite value.
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "../../include/wl.h"

namespace {

constexpr int kBlock = 16;
constexpr double kE2m1Max = 6.0;
constexpr double kE4m3Max = 448.0;

// Non-negative x -> E4M3 byte (bias 7, 3 mantissa bits; subnormal step 2^-9).
uint8_t e4m3_rne(double x) {
    if (!(x < kE4m3Max)) return 0x7E;  // 448, also for x = 448 exactly
    if (x < 0x1p-6) {
        // subnormals, and the carry into the smallest normal (code 8 = 2^-6)
        return (uint8_t)std::nearbyint(x * 0x1p9);
    }
    int ex = 0;
    const double f = std::frexp(x, &ex);  // x = f 2^ex, f in [0.5, 1)
    int e = ex - 1;                        // x = (2f) 2^e, 2f in [1, 2)
    int m = (int)std::nearbyint((2.0 * f - 1.0) * 8.0);
    if (m == 8) {
        m = 0;
        ++e;
    }
    const int code = ((e + 7) << 3) | m;
    return (uint8_t)(code > 0x7E ? 0x7E : code);
}

double e4m3_value(uint8_t b) {
    const int e = (b >> 3) & 15, m = b & 7;
    const double mag = e == 0 ? std::ldexp((double)m, -9) : std::ldexp(8.0 + m, e - 10);
    return (b & 0x80) ? -mag : mag;
}

// v -> E2M1 code (bit 3 the sign; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6).
uint8_t e2m1_rne(double v) {
    const uint8_t sign = std::signbit(v) ? 8 : 0;
    double a = std::fabs(v);
    if (a > kE2m1Max) a = kE2m1Max;
    uint8_t code;
    if (a < 1.0) {
        code = (uint8_t)std::nearbyint(a * 2.0);  // 0, 0.5, and the carry to 1.0 (code 2)
    } else {
        int ex = 0;
        const double f = std::frexp(a, &ex);
        int e = ex - 1;  // 0, 1 or 2
        int m = (int)std::nearbyint((2.0 * f - 1.0) * 2.0);
        if (m == 2) {
            m = 0;
            ++e;
        }
        const int c = ((e + 1) << 1) | m;
        code = (uint8_t)(c > 7 ? 7 : c);
    }
    return sign | code;
}

}  // namespace

extern "C" wl_status wl_quantize_nvfp4(const float *W, int N, int K, float tensor_scale, uint8_t *codes,
                                       uint8_t *scales, float *tensor_scale_out) {
    if (N < 0 || K < 0) return WL_ERR_INVALID_ARG;
    if (K % kBlock != 0) return WL_ERR_ALIGNMENT;
    if (!(tensor_scale >= 0.0f) || std::isinf(tensor_scale)) return WL_ERR_INVALID_ARG;
    if (!tensor_scale_out) return WL_ERR_INVALID_ARG;
    const size_t n = (size_t)N * K;
    if (n > 0 && (!W || !codes || !scales)) return WL_ERR_INVALID_ARG;
    for (size_t i = 0; i < n; ++i)
        if (!std::isfinite(W[i])) return WL_ERR_INVALID_ARG;
    if (std::fegetround() != FE_TONEAREST) return WL_ERR_UNSUPPORTED;

    double ts = tensor_scale;
    if (ts == 0.0) {
        double amax = 0.0;
        for (size_t i = 0; i < n; ++i) amax = std::fmax(amax, std::fabs((double)W[i]));
        const float ts32 = (float)(amax / (kE2m1Max * kE4m3Max));
        ts = ts32 > 0.0f ? (double)ts32 : 1.0;
    }
    *tensor_scale_out = (float)ts;

    const int nb = K / kBlock;
    for (int r = 0; r < N; ++r) {
        const float *w = W + (size_t)r * K;
        uint8_t *c = codes + (size_t)r * (K / 2);
        for (int b = 0; b < nb; ++b) {
            double bmax = 0.0;
            for (int i = 0; i < kBlock; ++i) bmax = std::fmax(bmax, std::fabs((double)w[b * kBlock + i]));
            const uint8_t sb = e4m3_rne(bmax / (kE2m1Max * ts));
            scales[(size_t)r * nb + b] = sb;
            const double denom = e4m3_value(sb) * ts;
            for (int i = 0; i < kBlock; i += 2) {
                const double v0 = w[b * kBlock + i], v1 = w[b * kBlock + i + 1];
                const uint8_t c0 = denom > 0.0 ? e2m1_rne(v0 / denom) : 0;
                const uint8_t c1 = denom > 0.0 ? e2m1_rne(v1 / denom) : 0;
                c[(b * kBlock + i) / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    }
    return WL_OK;
}
