// kvq_transform.cuh -- input loads and the key pre-transform shared by the
// calibration and quantise-append kernels (sm_100a).
//
// Method: "NVFP4 attention cache on W4A4 Qwen3-8B" (rstation.ai) -- results
// table rows on static per-channel sqrt(absmax) smoothing and on Hadamard-128;
// the rotation is the Sylvester-ordered Walsh-Hadamard transform normalised
// by 1/sqrt(128).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "kvq_common.cuh"
#include "kvq_packed.cuh"

namespace kvq {

// Two bf16 (low half first) -> (lo, hi) as fp32, exact.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// 16 consecutive elements starting at p as 8 pairs (16-byte aligned for
// fp32, 32 B for bf16); plain loads, so p may be global or shared.
__device__ __forceinline__ void load16(const float* p, float2* x) {
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 t = q[i];
        x[2 * i] = make_float2(t.x, t.y);
        x[2 * i + 1] = make_float2(t.z, t.w);
    }
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float2* x) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint4 t = q[i];
        x[4 * i] = bf16x2_to_f2(t.x);
        x[4 * i + 1] = bf16x2_to_f2(t.y);
        x[4 * i + 2] = bf16x2_to_f2(t.z);
        x[4 * i + 3] = bf16x2_to_f2(t.w);
    }
}

// ---------------------------------------------------------------- key transform
// Normalised Hadamard-128 of a key row held as 8 blocks of 16 in 8
// consecutive lanes (lane & 7 == blk), element 2i + e of the block in y[i]
// (.x for e = 0): butterflies h = 1 inside each pair, h = 2, 4, 8 between
// pairs of the thread, h = 16, 32, 64 across lanes, then one multiply by
// fp32(1/sqrt(128)).  Every result is a single fp32 rounding of the stage's
// sum or difference, in stage order (the packed forms round each half like
// the scalar ones; across lanes, fma(y, -1, a) rounds a - y exactly once).
// Every lane of the warp must call it.
__device__ __forceinline__ void hadamard_block(float2* y, int blk) {
#pragma unroll
    for (int i = 0; i < kBlk / 2; ++i) {
        const float a = y[i].x, b = y[i].y;
        y[i] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int hp = 1; hp < kBlk / 2; hp <<= 1) {
#pragma unroll
        for (int i = 0; i < kBlk / 2; ++i) {
            if ((i & hp) == 0) {
                const float2 a = y[i], b = y[i + hp];
                y[i] = fadd2(a, b);
                y[i + hp] = fsub2(a, b);
            }
        }
    }
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) {
        // the lane holding the upper index keeps (partner - own), the other (own + partner)
        const float sg = (blk & m) ? -1.0f : 1.0f;
        const float2 s2 = make_float2(sg, sg);
#pragma unroll
        for (int i = 0; i < kBlk / 2; ++i) {
            const float2 o = make_float2(__shfl_xor_sync(0xFFFFFFFFu, y[i].x, m),
                                         __shfl_xor_sync(0xFFFFFFFFu, y[i].y, m));
            y[i] = ffma2(y[i], s2, o);
        }
    }
    const float2 c2 = make_float2(kInvSqrt128, kInvSqrt128);
#pragma unroll
    for (int i = 0; i < kBlk / 2; ++i) y[i] = fmul2(y[i], c2);
}

// Smoothing multiply y = k * inv_s of one block (inv_row: the block's 16
// factors, 16-byte aligned).
__device__ __forceinline__ void smooth_block(float2* y, const float* __restrict__ inv_row) {
    const float4* ip = reinterpret_cast<const float4*>(inv_row);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 f = __ldg(ip + i);
        y[2 * i] = fmul2(y[2 * i], make_float2(f.x, f.y));
        y[2 * i + 1] = fmul2(y[2 * i + 1], make_float2(f.z, f.w));
    }
}

}  // namespace kvq
