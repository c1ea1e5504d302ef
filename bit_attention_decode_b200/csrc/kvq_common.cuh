// kvq_common.cuh -- device helpers shared by the kvq kernels (sm_100a).
//
// Format conversions use the sm_100a PTX conversions to and from the packed
// FP4 (E2M1) and FP8 (E4M3) formats; the rounding they implement is checked
// elementwise against an independent reference by the test suite.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kD = 128;          // head_dim
constexpr int kBlk = 16;         // NVFP4 block length along head_dim
constexpr int kPage = 16;        // tokens per page
constexpr int kTile = 2304;      // bytes of one kv head of one page
constexpr int kKCodes = 0;       // 16 rows x 64 B
constexpr int kKScales = 1024;   // 16 rows x 8 B, token-major
constexpr int kVCodes = 1152;    // 16 rows x 64 B
constexpr int kVScales = 2176;   // 8 blocks x 16 B, block-major

// fp32 nearest to 1/sqrt(128): the normalisation of the Hadamard-128 rotation
constexpr float kInvSqrt128 = 0.08838834764831845f;
// 6 * 448: the absmax of a tensor maps to the largest E2M1 value times the
// largest E4M3 value under the FP32 tensor scale
constexpr float kTensorRange = 2688.0f;

// ---------------------------------------------------------------- formats
// Two fp32 values -> one byte of two E2M1 codes (hi -> high nibble).
__device__ __forceinline__ uint32_t e2m1x2_rn(float hi, float lo) {
    uint16_t r;
    asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u16.u8 %0, t; }"
        : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// One fp32 value -> E4M3 code (round-to-nearest-even, saturating).
__device__ __forceinline__ uint32_t e4m3_rn(float x) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
    return r & 0xFFu;
}

// Two E4M3 codes (low byte -> low half) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
    uint32_t r;
    uint16_t in = (uint16_t)two_codes;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(in));
    return r;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    uint32_t h2 = e4m3x2_to_f16x2(code & 0xFFu);
    return __half2float(__ushort_as_half((uint16_t)(h2 & 0xFFFFu)));
}

// One byte of two E2M1 codes -> f16x2 (low nibble -> low half), exact.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    uint32_t r;
    uint16_t in = (uint16_t)(byte & 0xFFu);
    asm("{ .reg .b8 t; cvt.u8.u16 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(r) : "h"(in));
    return r;
}

// ---------------------------------------------------------------- inputs
__device__ __forceinline__ float load_elem(const float* p) { return *p; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// 16 consecutive elements starting at p (16-byte aligned for fp32, 32 B for bf16)
__device__ __forceinline__ void load16(const float* p, float* x) {
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float4 t = __ldg(q + i);
        x[4 * i] = t.x; x[4 * i + 1] = t.y; x[4 * i + 2] = t.z; x[4 * i + 3] = t.w;
    }
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float* x) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        uint4 t = __ldg(q + i);
        uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            x[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            x[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

// ---------------------------------------------------------------- key transform
// Normalised Hadamard-128 of a key row held as 8 blocks of 16 in 8
// consecutive lanes (lane & 7 == blk): butterflies h = 1, 2, 4, 8 inside the
// thread, h = 16, 32, 64 across lanes, then one multiply by fp32(1/sqrt(128)).
// Every operation is a single fp32 rounding, in the order listed; every lane
// of the warp must call it.
__device__ __forceinline__ void hadamard_block(float* y, int blk) {
#pragma unroll
    for (int h = 1; h < kBlk; h <<= 1) {
#pragma unroll
        for (int j = 0; j < kBlk; ++j) {
            if ((j & h) == 0) {
                float a = y[j], b = y[j + h];
                y[j] = __fadd_rn(a, b);
                y[j + h] = __fsub_rn(a, b);
            }
        }
    }
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) {
        const bool upper = (blk & m) != 0;
#pragma unroll
        for (int j = 0; j < kBlk; ++j) {
            float other = __shfl_xor_sync(0xFFFFFFFFu, y[j], m);
            y[j] = upper ? __fsub_rn(other, y[j]) : __fadd_rn(y[j], other);
        }
    }
#pragma unroll
    for (int i = 0; i < kBlk; ++i) y[i] = __fmul_rn(y[i], kInvSqrt128);
}

// Key pre-transform of one block: smoothing multiply y = k * inv_s, then the
// optional rotation (see hadamard_block).
__device__ __forceinline__ void transform_key_block(float* y, const float* __restrict__ inv_s_row,
                                                    int blk, bool hadamard) {
#pragma unroll
    for (int i = 0; i < kBlk; ++i) y[i] = __fmul_rn(y[i], __ldg(inv_s_row + blk * kBlk + i));
    if (hadamard) hadamard_block(y, blk);
}

__device__ __forceinline__ void set_status(int32_t* status, int32_t bits) {
    if (status) atomicOr(status, bits);
}

}  // namespace kvq
