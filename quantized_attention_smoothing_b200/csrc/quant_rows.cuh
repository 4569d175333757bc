// quant_rows.cuh -- the per-row arithmetic of the INT8 quantisation of
// Q and K: bf16 -> fp32, f32x2 operations, the Sylvester butterfly on fp32
// pairs of a row held by one thread, and the codes rne(x_hat * (127 / a))
// ("Sage v2 in AITER" / "qr_hadamard_quant": rotate, block absmax, scale,
// INT8). The attention kernel's in-CTA Q path uses the row helpers; the
// quantisation kernels (a row spread over four threads) use the same
// primitives in the same order, so both produce the same bits. Internal to
// libsage.
#pragma once

#include <cstdint>

namespace sage {
namespace qrow {

constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}

__device__ __forceinline__ uint32_t pack_clamp4(float y0, float y1, float y2, float y3) {
    const float y[4] = {y0, y1, y2, y3};
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int code = __float2int_rn(y[i]);
        code = max(-127, min(127, code));
        word |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * i);
    }
    return word;
}

// fp32 pairs (sm_100 f32x2 arithmetic): each lane is one IEEE RN operation,
// so results equal the scalar ones bit for bit. A product feeding an add must
// not be written as mul.rn.f32x2 + add.rn.f32x2: ptxas contracts that pair
// into one FMA (a single rounding) despite the explicit rounding modifiers.
__device__ __forceinline__ uint64_t p2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float p2lo(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return lo;
}
__device__ __forceinline__ float p2hi(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return hi;
}
__device__ __forceinline__ uint64_t p2add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t p2sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t p2fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t p2mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// The butterfly of `butterfly` on a row held as D/2 pairs x2[i] = (x[2i],
// x[2i+1]): stage h = 1 inside each pair, stages h = 2 .. D/2 as pair
// operations between pairs i and i + h/2. Same operations, same order per
// element, so the same bits.
template <int D>
__device__ __forceinline__ void butterfly_pairs(uint64_t (&x2)[D / 2]) {
#pragma unroll
    for (int i = 0; i < D / 2; ++i) {
        const float a = p2lo(x2[i]), c = p2hi(x2[i]);
        x2[i] = p2(__fadd_rn(a, c), __fsub_rn(a, c));
    }
#pragma unroll
    for (int lg = 0; (2 << lg) < D; ++lg) {
        const int hp = 1 << lg;                  // pair distance = h / 2
#pragma unroll
        for (int k = 0; k < D / 4; ++k) {
            const int i = ((k >> lg) << (lg + 1)) + (k & (hp - 1));
            const uint64_t a = x2[i], c = x2[i + hp];
            x2[i] = p2add(a, c);
            x2[i + hp] = p2sub(a, c);
        }
    }
}

// Codes 16c .. 16c + 15 of one row: rne(x_hat * rr) for the values held as
// pairs, four codes per word (element 16c + 4i + e in byte e of word i).
// |x_hat * r| <= a * fl(127 / a) rounds to at most 127 whenever rr is finite,
// so the magic-number rounding needs no clamp; a block whose amax is so small
// that 127 / a overflows takes the clamped conversion.
template <int D>
__device__ __forceinline__ uint4 row_codes16(const uint64_t (&x2)[D / 2], float rr, int c) {
    uint32_t w4[4];
    if (isfinite(rr)) {
        const uint64_t rr2 = p2(rr, rr), mg2 = p2(kRoundMagic, kRoundMagic);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // the product is rounded on its own (an FMA with +0), so the
            // magic add that follows cannot be contracted into it
            const uint64_t t01 = p2add(p2fma(x2[8 * c + 2 * i], rr2, 0ull), mg2);
            const uint64_t t23 = p2add(p2fma(x2[8 * c + 2 * i + 1], rr2, 0ull), mg2);
            w4[i] = __byte_perm(__byte_perm(__float_as_uint(p2lo(t01)), __float_as_uint(p2hi(t01)), 0x0040),
                                __byte_perm(__float_as_uint(p2lo(t23)), __float_as_uint(p2hi(t23)), 0x0040),
                                0x5410);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint64_t* pv = x2 + 8 * c + 2 * i;
            w4[i] = pack_clamp4(__fmul_rn(p2lo(pv[0]), rr), __fmul_rn(p2hi(pv[0]), rr),
                                __fmul_rn(p2lo(pv[1]), rr), __fmul_rn(p2hi(pv[1]), rr));
        }
    }
    return make_uint4(w4[0], w4[1], w4[2], w4[3]);
}

}  // namespace qrow
}  // namespace sage
