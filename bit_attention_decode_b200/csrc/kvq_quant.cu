// kvq_quant.cu -- calibration of the smoothing factors and tensor scales, and
// the quantise-and-append of tokens into the packed NVFP4 cache.
//
// Method: "NVFP4 attention cache on W4A4 Qwen3-8B" (rstation.ai) -- setup
// paragraph (NVFP4 on post-RoPE keys and values, 16-blocks along head_dim),
// results table rows on static per-channel sqrt(absmax) smoothing with
// position 0 excluded and on Hadamard-128; "OSFP4" (paperlayer.ai summary)
// Problem bullet / sec. 1 (absmax mapped to 6), sec. 3 (global
// calibration-based scale for online quantisation), sec. D.1 (E2M1 values,
// E4M3 scale per 16, FP32 tensor scale).
#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

// ------------------------------------------------------------------ calibrate
// Per-channel key absmax over the calibration tokens (t >= t0), as fp32 bits
// combined with atomicMax (order-independent, so the result is exact).
template <typename T>
__global__ void __launch_bounds__(256)
calib_absmax_kernel(const T* __restrict__ k, int W, int Tlen, int Hkv, int t0, int tok_per_cta,
                    uint32_t* __restrict__ absmax_bits /* [L][Hkv][D] */) {
    const int l = blockIdx.z, w = blockIdx.y;
    const int tb = blockIdx.x * tok_per_cta;
    const int te = min(Tlen, tb + tok_per_cta);
    const int row = Hkv * kD;
    const T* base = k + ((size_t)l * W + w) * (size_t)Tlen * row;
    for (int i = threadIdx.x; i < row; i += blockDim.x) {
        float m = 0.0f;
        for (int t = max(tb, t0); t < te; ++t) m = fmaxf(m, fabsf(load_elem(base + (size_t)t * row + i)));
        atomicMax(absmax_bits + (size_t)l * row + i, __float_as_uint(m));
    }
}

__global__ void calib_finalize_smooth_kernel(float* __restrict__ s, float* __restrict__ inv_s, int n) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float A = s[i];  // holds the absmax until here
    float sc = (A > 0.0f) ? __fsqrt_rn(A) : 1.0f;
    s[i] = sc;
    inv_s[i] = __frcp_rn(sc);
}

// Tensor absmax of the transformed keys and of the values over every
// calibration token (position 0 included).  8 lanes per (token, head) row.
template <typename T>
__global__ void __launch_bounds__(256)
calib_tensor_amax_kernel(const T* __restrict__ k, const T* __restrict__ v, int W, int Tlen, int Hkv,
                         const float* __restrict__ inv_s /* [L][Hkv][D] */, int hadamard,
                         uint32_t* __restrict__ gk_bits, uint32_t* __restrict__ gv_bits) {
    const int l = blockIdx.y;
    const int rows = W * Tlen * Hkv;  // rows of one layer
    const int lane_row = (blockIdx.x * blockDim.x + threadIdx.x) >> 3;
    const int blk = threadIdx.x & 7;
    const bool live = lane_row < rows;
    const int r = live ? lane_row : rows - 1;   // dead lanes still join the shuffles
    const int h = r % Hkv;
    const size_t off = ((size_t)l * rows + r) * kD + blk * kBlk;
    float y[kBlk], x[kBlk];
    load16(k + off, y);
    load16(v + off, x);
    transform_key_block(y, inv_s + ((size_t)l * Hkv + h) * kD, blk, hadamard != 0);
    float ak = 0.0f, av = 0.0f;
#pragma unroll
    for (int i = 0; i < kBlk; ++i) { ak = fmaxf(ak, fabsf(y[i])); av = fmaxf(av, fabsf(x[i])); }
    if (!live) { ak = 0.0f; av = 0.0f; }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        ak = fmaxf(ak, __shfl_xor_sync(0xFFFFFFFFu, ak, m));
        av = fmaxf(av, __shfl_xor_sync(0xFFFFFFFFu, av, m));
    }
    if ((threadIdx.x & 31) == 0) {
        atomicMax(gk_bits + l, __float_as_uint(ak));
        atomicMax(gv_bits + l, __float_as_uint(av));
    }
}

__global__ void calib_finalize_gscale_kernel(float* __restrict__ gk, float* __restrict__ gv, int L) {
    int l = blockIdx.x * blockDim.x + threadIdx.x;
    if (l >= L) return;
    float a = gk[l], b = gv[l];
    gk[l] = (a > 0.0f) ? __fdiv_rn(a, kTensorRange) : 1.0f;
    gv[l] = (b > 0.0f) ? __fdiv_rn(b, kTensorRange) : 1.0f;
}

// ------------------------------------------------------------------ quantise
// One 16-element block: E4M3 block scale from the absmax, then E2M1 codes.
// enc = 1/(6 g) is computed once per tensor by the caller.
__device__ __forceinline__ void quantize_block(const float* y, float g, float enc, uint2& codes,
                                               uint32_t& sf) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < kBlk; ++i) a = fmaxf(a, fabsf(y[i]));
    sf = e4m3_rn(__fmul_rn(a, enc));
    const float d = __fmul_rn(e4m3_to_f32(sf), g);
    const float r = (d == 0.0f) ? 0.0f : __frcp_rn(d);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < kBlk / 2; ++j) {
        uint32_t byte = e2m1x2_rn(__fmul_rn(y[2 * j + 1], r), __fmul_rn(y[2 * j], r));
        w[j >> 2] |= byte << (8 * (j & 3));
    }
    codes = make_uint2(w[0], w[1]);
}

// grid (num_tokens, nlayers); block Hkv * 16 threads: threads [0, 8 Hkv) own
// the 8 key blocks of each head, the rest the value blocks.
template <typename T>
__global__ void __launch_bounds__(256)
append_kernel(const T* __restrict__ k, const T* __restrict__ v, const int64_t* __restrict__ slots,
              int num_tokens, int Hkv, const float* __restrict__ inv_s, const float* __restrict__ gk,
              const float* __restrict__ gv, uint8_t* __restrict__ cache, int64_t layer_stride,
              int num_pages, int hadamard, int32_t* __restrict__ status) {
    const int tok = blockIdx.x, li = blockIdx.y;
    const int64_t slot = __ldg(slots + tok);
    if (slot < 0) return;  // padding token
    if (slot >= (int64_t)num_pages * kPage) {
        if (threadIdx.x == 0) set_status(status, KVQ_DEV_BAD_SLOT);
        return;
    }
    const int t = threadIdx.x;
    const bool is_v = t >= Hkv * 8;
    const int h = (t >> 3) % Hkv;
    const int blk = t & 7;
    const size_t src = (((size_t)li * num_tokens + tok) * Hkv + h) * kD + blk * kBlk;
    float y[kBlk];
    load16(is_v ? v + src : k + src, y);
    const float* inv_row = inv_s + ((size_t)li * Hkv + h) * kD;
    if (hadamard) {
        // every lane joins the cross-lane butterflies (groups of 8 lanes never
        // mix keys and values); value lanes discard the result
        float z[kBlk];
#pragma unroll
        for (int i = 0; i < kBlk; ++i) z[i] = y[i];
        transform_key_block(z, inv_row, blk, true);
        if (!is_v) {
#pragma unroll
            for (int i = 0; i < kBlk; ++i) y[i] = z[i];
        }
    } else if (!is_v) {
        transform_key_block(y, inv_row, blk, false);
    }
    const float g = is_v ? __ldg(gv + li) : __ldg(gk + li);
    const float enc = __frcp_rn(__fmul_rn(6.0f, g));
    uint2 codes;
    uint32_t sf;
    quantize_block(y, g, enc, codes, sf);
    const int64_t page = slot >> 4;
    const int off = (int)(slot & 15);
    uint8_t* tile = cache + (size_t)li * layer_stride + ((size_t)page * Hkv + h) * kTile;
    if (!is_v) {
        *reinterpret_cast<uint2*>(tile + kKCodes + off * 64 + blk * 8) = codes;
        tile[kKScales + off * 8 + blk] = (uint8_t)sf;
    } else {
        *reinterpret_cast<uint2*>(tile + kVCodes + off * 64 + blk * 8) = codes;
        tile[kVScales + blk * 16 + off] = (uint8_t)sf;
    }
}

// ------------------------------------------------------------------ utilities
__global__ void round_e2m1_kernel(const float* __restrict__ x, uint8_t* __restrict__ out, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = (uint8_t)(e2m1x2_rn(0.0f, x[i]) & 0xFu);
}

__global__ void round_e4m3_kernel(const float* __restrict__ x, uint8_t* __restrict__ out, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = (uint8_t)e4m3_rn(x[i]);
}

// ------------------------------------------------------------------ launchers
template <typename T>
static kvq_status launch_calibrate(const kvq_shape& s, const T* k, const T* v, int W, int Tlen,
                                   int exclude_pos0, const kvq_calib& out, cudaStream_t st) {
    const int L = s.num_layers, H = s.num_kv_heads;
    const size_t n = (size_t)L * H * kD;
    if (cudaMemsetAsync(out.k_smooth, 0, n * sizeof(float), st) != cudaSuccess ||
        cudaMemsetAsync(out.k_gscale, 0, L * sizeof(float), st) != cudaSuccess ||
        cudaMemsetAsync(out.v_gscale, 0, L * sizeof(float), st) != cudaSuccess)
        return KVQ_ECUDA;
    const int tpc = 64;
    dim3 g1((Tlen + tpc - 1) / tpc, W, L);
    calib_absmax_kernel<T><<<g1, 256, 0, st>>>(k, W, Tlen, H, exclude_pos0 ? 1 : 0, tpc,
                                              reinterpret_cast<uint32_t*>(out.k_smooth));
    calib_finalize_smooth_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(out.k_smooth, out.k_inv_smooth, (int)n);
    const long rows = (long)W * Tlen * H;
    dim3 g3((unsigned)((rows * 8 + 255) / 256), L);
    calib_tensor_amax_kernel<T><<<g3, 256, 0, st>>>(k, v, W, Tlen, H, out.k_inv_smooth, s.use_hadamard,
                                                   reinterpret_cast<uint32_t*>(out.k_gscale),
                                                   reinterpret_cast<uint32_t*>(out.v_gscale));
    calib_finalize_gscale_kernel<<<(L + 63) / 64, 64, 0, st>>>(out.k_gscale, out.v_gscale, L);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

kvq_status calibrate(const kvq_shape& s, const void* k, const void* v, int dtype, int W, int Tlen,
                     int exclude_pos0, const kvq_calib& out, cudaStream_t st) {
    if (dtype == KVQ_F32)
        return launch_calibrate(s, (const float*)k, (const float*)v, W, Tlen, exclude_pos0, out, st);
    return launch_calibrate(s, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, W, Tlen, exclude_pos0, out, st);
}

kvq_status quantize_append(const kvq_shape& s, const kvq_calib& c, const kvq_cache& cache, int layer0,
                           int nlayers, const void* k, const void* v, int dtype, const int64_t* slots,
                           int num_tokens, int32_t* status, cudaStream_t st) {
    const int H = s.num_kv_heads;
    const float* inv_s = c.k_inv_smooth + (size_t)layer0 * H * kD;
    const float* gk = c.k_gscale + layer0;
    const float* gv = c.v_gscale + layer0;
    uint8_t* base = cache.data + (size_t)layer0 * cache.layer_stride_bytes;
    dim3 grid(num_tokens, nlayers);
    if (dtype == KVQ_F32)
        append_kernel<float><<<grid, H * 16, 0, st>>>((const float*)k, (const float*)v, slots, num_tokens, H,
                                                     inv_s, gk, gv, base, cache.layer_stride_bytes,
                                                     cache.num_pages, s.use_hadamard, status);
    else
        append_kernel<__nv_bfloat16><<<grid, H * 16, 0, st>>>(
            (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, slots, num_tokens, H, inv_s, gk, gv, base,
            cache.layer_stride_bytes, cache.num_pages, s.use_hadamard, status);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

kvq_status round_e2m1(const float* x, uint8_t* out, int64_t n, cudaStream_t st) {
    round_e2m1_kernel<<<1184, 256, 0, st>>>(x, out, n);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

kvq_status round_e4m3(const float* x, uint8_t* out, int64_t n, cudaStream_t st) {
    round_e4m3_kernel<<<1184, 256, 0, st>>>(x, out, n);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

}  // namespace kvq
