// packed_f32.cuh — fp32 arithmetic on sm_100a that takes a pair of floats
// per instruction (fma/add/sub .f32x2), the three-input maximum, the
// hardware 2^x approximation and a 2^x on a pair from FMA-pipe arithmetic
// alone.
#pragma once

namespace pkv {

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// max of three (NaN inputs are ignored, as in fmaxf)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// max of N values as a tree of three-input maxima (depth log3 N)
template <int N>
__device__ __forceinline__ float max_tree(const float* v) {
    if constexpr (N == 1) {
        return v[0];
    } else if constexpr (N == 2) {
        return fmaxf(v[0], v[1]);
    } else {
        constexpr int M = (N + 2) / 3;
        float w[M];
#pragma unroll
        for (int i = 0; i < N / 3; ++i) w[i] = fmax3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
        if constexpr (N % 3 == 1) w[M - 1] = v[N - 1];
        if constexpr (N % 3 == 2) w[M - 1] = fmaxf(v[N - 2], v[N - 1]);
        return max_tree<M>(w);
    }
}

// 2^x by the hardware approximation (relative error near 2^-22; -inf -> 0;
// subnormal results flush to zero)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// a + b on a pair, rounded toward minus infinity
__device__ __forceinline__ float2 fadd2_rm(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rm.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// 2^x on a pair without the exponential unit: FMA-pipe arithmetic only, so
// that a softmax can split its exponentials between the two pipes (as
// FlashAttention-4 does on Blackwell).  For x <= 2^22:
//   - x is clamped to -127 below (-inf and NaN included);
//   - adding 1.5 * 2^23 rounded down leaves floor(x) = j as an integer in
//     the low mantissa bits of the sum t, and f = x - j in [0, 1) is exact;
//   - 2^f comes from a degree-4 polynomial with constant term 1, its other
//     coefficients fitted here by linear programming to the least maximum
//     relative error over [0, 1] (3.0e-6, evaluated in fp32);
//   - 2^j is added into the exponent field: t's bits shifted left by 23
//     are j << 23 modulo 2^32.
// So x = -127 gives exactly +0 (the polynomial's 1.0 carries exponent 127)
// and x in (-127, -126) a subnormal below 2^-126; from -126 up the result
// is 2^x within the fit's error.
__device__ __forceinline__ float2 ex2_poly2(float2 x) {
    x.x = fmaxf(x.x, -127.f);
    x.y = fmaxf(x.y, -127.f);
    const float2 magic = make_float2(12582912.f, 12582912.f);  // 1.5 * 2^23
    const float2 t = fadd2_rm(x, magic);
    const float2 f = fsub2(x, fsub2(t, magic));
    float2 q = ffma2(make_float2(0x1.b7ea5cp-7f, 0x1.b7ea5cp-7f), f,
                     make_float2(0x1.abfe7ep-5f, 0x1.abfe7ep-5f));
    q = ffma2(q, f, make_float2(0x1.ee2374p-3f, 0x1.ee2374p-3f));
    q = ffma2(q, f, make_float2(0x1.62d6d0p-1f, 0x1.62d6d0p-1f));
    q = ffma2(q, f, make_float2(1.f, 1.f));
    return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

}  // namespace pkv
