// Host-side FP32 -> FP8 E4M3 encoding (the OCP 8-bit floating-point format that
// the tensor cores' kind::f8f6f4 MMAs read): 1 sign bit, 4 exponent bits with
// bias 7, 3 mantissa bits; exponent field 0 holds the subnormals m * 2^-9; no
// infinities, S.1111.111 is NaN, so the largest finite magnitude is
// 1.75 * 2^8 = 448.  Rounding is to nearest, ties to even; magnitudes beyond
// 448 saturate to 448 (the device conversion, cvt.rn.satfinite, does the same).
#pragma once

#include <cmath>
#include <cstdint>

namespace jd {

inline uint8_t e4m3_encode(float f) {
    const uint8_t sign = std::signbit(f) ? 0x80 : 0x00;
    const float a = std::fabs(f);
    if (std::isnan(f)) return 0x7f;
    if (a >= 448.0f) return sign | 0x7e;
    int e = 0;
    std::frexp(a, &e);  // a = m * 2^e, m in [0.5, 1): a = 1.f * 2^(e - 1)
    int E = e - 1;
    if (a == 0.0f || E < -6) {  // subnormal range: multiples of 2^-9
        const float q = std::nearbyint(std::ldexp(a, 9));  // 0 .. 8, ties to even
        return sign | (uint8_t)q;                          // q = 8 is the smallest normal, code 0x08
    }
    float q = std::nearbyint(std::ldexp(a, 3 - E));  // 8 .. 16: the leading one and three mantissa bits
    if (q >= 16.0f) {
        q = 8.0f;
        ++E;
    }
    if (E > 8) return sign | 0x7e;
    const int code = ((E + 7) << 3) | ((int)q - 8);
    return sign | (uint8_t)(code > 0x7e ? 0x7e : code);
}

}  // namespace jd
