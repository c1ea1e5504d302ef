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
// mixed cache (BF16 keys, NVFP4 values): 5248-byte tiles
constexpr int kTileBf16K = 5248;
constexpr int kBf16VCodes = 4096;    // after 16 rows x 256 B of bf16 keys
constexpr int kBf16VScales = 5120;
__host__ __device__ constexpr int tile_bytes(int k_format) { return k_format == KVQ_K_BF16 ? kTileBf16K : kTile; }

// fp32 nearest to 1/sqrt(128): the normalisation of the Hadamard-128 rotation
constexpr float kInvSqrt128 = 0.08838834764831845f;
// 6 * 448: the absmax of a tensor maps to the largest E2M1 value times the
// largest E4M3 value under the FP32 tensor scale
constexpr float kTensorRange = 2688.0f;

// ---------------------------------------------------------------- formats
// Eight fp32 values as four pairs -> four bytes of E2M1 codes, round to
// nearest even, saturating at 6, sign kept: pair i -> byte i, its .x in the
// low nibble.  Every quantiser of the library (the append, the KLT key
// append, the FP4 query of the prefill) converts through this routine, and
// kvq_round_e2m1 exposes it for an exhaustive check.
__device__ __forceinline__ uint32_t e2m1x8_rn(float2 a, float2 b, float2 c, float2 d) {
    uint32_t w;
    asm("{ .reg .b8 b0, b1, b2, b3;\n"
        "  cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1; cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
        "  cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5; cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
        "  mov.b32 %0, {b0, b1, b2, b3}; }"
        : "=r"(w)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y), "f"(d.x), "f"(d.y));
    return w;
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

__device__ __forceinline__ void set_status(int32_t* status, int32_t bits) {
    if (status) atomicOr(status, bits);
}

}  // namespace kvq
