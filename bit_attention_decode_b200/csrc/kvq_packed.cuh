// kvq_packed.cuh -- packed fp32 pair arithmetic (sm_100a).
//
// sm_100a executes two fp32 operations per lane in one instruction; each half
// is an ordinary IEEE operation rounded to nearest even, as its scalar form.
#pragma once

#include <cuda_runtime.h>

namespace kvq {

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{ .reg .b64 ra, rb, rc, rd; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5}; mov.b64 rc, {%6, %7};\n"
        "  fma.rn.f32x2 rd, ra, rb, rc; mov.b64 {%0, %1}, rd; }"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{ .reg .b64 ra, rb, rd; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5};\n"
        "  add.rn.f32x2 rd, ra, rb; mov.b64 {%0, %1}, rd; }"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
    float2 d;
    asm("{ .reg .b64 ra, rb, rd; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5};\n"
        "  sub.rn.f32x2 rd, ra, rb; mov.b64 {%0, %1}, rd; }"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("{ .reg .b64 ra, rb, rd; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5};\n"
        "  mul.rn.f32x2 rd, ra, rb; mov.b64 {%0, %1}, rd; }"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
// max of three (exact, like any max)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
// absmax of a 16-block held as 8 pairs
__device__ __forceinline__ float absmax16(const float2* y) {
    const float m0 = fmax3(fabsf(y[0].x), fabsf(y[0].y), fabsf(y[1].x));
    const float m1 = fmax3(fabsf(y[1].y), fabsf(y[2].x), fabsf(y[2].y));
    const float m2 = fmax3(fabsf(y[3].x), fabsf(y[3].y), fabsf(y[4].x));
    const float m3 = fmax3(fabsf(y[4].y), fabsf(y[5].x), fabsf(y[5].y));
    const float m4 = fmax3(fabsf(y[6].x), fabsf(y[6].y), fabsf(y[7].x));
    return fmaxf(fmax3(m0, m1, m2), fmax3(m3, m4, fabsf(y[7].y)));
}

}  // namespace kvq
