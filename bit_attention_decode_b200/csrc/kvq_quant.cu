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
#include "kvq_sync.cuh"

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

// Bulk-copy staging of the inputs.  A work item is a chunk of `tc`
// consecutive tokens of one layer: its key rows and value rows are two
// contiguous ranges (tc x Hkv x 128 elements each), streamed into a ring of
// kAppendStages shared-memory stages with cp.async.bulk and an mbarrier
// transaction count.  Thread 0 keeps kAppendStages - 1 chunks in flight.
// Quantisation then reads the stage: a token takes Hkv * 16 threads, threads
// [0, 8 Hkv) owning the 8 key blocks of each head and the rest the value
// blocks; a CTA of 256 threads works on 256 / (16 Hkv) tokens at a time.
// With the rotation Hkv is even, so every warp lies inside one token and the
// cross-lane butterflies stay uniform.
constexpr int kAppendStages = 3;
constexpr int kAppendStageBytes = 32768;   // key + value rows of one chunk

template <typename T>
__device__ __forceinline__ void load16_smem(const T* p, float* x);
template <>
__device__ __forceinline__ void load16_smem<float>(const float* p, float* x) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float4 t = reinterpret_cast<const float4*>(p)[i];
        x[4 * i] = t.x; x[4 * i + 1] = t.y; x[4 * i + 2] = t.z; x[4 * i + 3] = t.w;
    }
}
template <>
__device__ __forceinline__ void load16_smem<__nv_bfloat16>(const __nv_bfloat16* p, float* x) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        uint4 t = reinterpret_cast<const uint4*>(p)[i];
        uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            x[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            x[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(288, 2)
append_kernel(const T* __restrict__ k, const T* __restrict__ v, const int64_t* __restrict__ slots,
              int num_tokens, int nlayers, int Hkv, int tc, const float* __restrict__ inv_s,
              const float* __restrict__ gk, const float* __restrict__ gv, uint8_t* __restrict__ cache,
              int64_t layer_stride, int num_pages, int hadamard, int32_t* __restrict__ status) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t full[kAppendStages], empty[kAppendStages];
    __shared__ int s_timeout, s_issued;
    const int row = Hkv * kD;                                  // elements per token row
    const uint32_t half_stage = kAppendStageBytes / 2;         // key rows, then value rows
    const int chunks = (num_tokens + tc - 1) / tc;
    const long items = (long)chunks * nlayers;
    const int mine = items > blockIdx.x ? (int)((items - 1 - blockIdx.x) / gridDim.x + 1) : 0;
    const int workers = 8;                                     // warps 0..7; warp 8 streams the inputs
    const int warp = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
        s_timeout = 0;
        s_issued = 0;
        for (int i = 0; i < kAppendStages; ++i) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&full[i])));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(&empty[i])), "r"(workers));
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == workers) {
        // ---------------------------------------------------------- producer
        if ((threadIdx.x & 31) == 0) {
            int j = 0;
            for (; j < mine; ++j) {
                const int st = j % kAppendStages;
                if (j >= kAppendStages && !mbar_wait(&empty[st], ((j / kAppendStages) - 1) & 1)) {
                    atomicOr(&s_timeout, 1);
                    break;
                }
                const long it = blockIdx.x + (long)j * gridDim.x;
                const int li = (int)(it / chunks), t0 = (int)(it % chunks) * tc;
                const int n = min(tc, num_tokens - t0);
                const uint32_t bytes = (uint32_t)n * row * sizeof(T);
                uint8_t* dst = smem + st * kAppendStageBytes;
                const size_t off = ((size_t)li * num_tokens + t0) * row;
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(&full[st])),
                             "r"(2 * bytes) : "memory");
                asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                             ::"r"(smem_u32(dst)), "l"(k + off), "r"(bytes), "r"(smem_u32(&full[st])) : "memory");
                asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                             ::"r"(smem_u32(dst + half_stage)), "l"(v + off), "r"(bytes), "r"(smem_u32(&full[st]))
                             : "memory");
            }
            s_issued = j;
        }
    } else {
        // ---------------------------------------------------------- workers
        // a token takes 8 Hkv threads, thread (h, blk) owning block blk of
        // head h for both the key and the value row
        const int per_tok = Hkv * 8;                           // a multiple of 8: lane & 7 == blk
        const int tpc = (workers * 32) / per_tok;              // tokens side by side
        const int t = threadIdx.x % per_tok, sub = threadIdx.x / per_tok;
        const int h = t >> 3, blk = t & 7;
        const bool active = sub < tpc;
        for (int j = 0; j < mine; ++j) {
            const long it = blockIdx.x + (long)j * gridDim.x;
            const int li = (int)(it / chunks), t0 = (int)(it % chunks) * tc;
            const int n = min(tc, num_tokens - t0);
            // per-chunk constants, loaded before waiting for the inputs
            float inv[kBlk];
            const float4* ip = reinterpret_cast<const float4*>(inv_s + ((size_t)li * Hkv + h) * kD + blk * kBlk);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 q4 = __ldg(ip + i);
                inv[4 * i] = q4.x; inv[4 * i + 1] = q4.y; inv[4 * i + 2] = q4.z; inv[4 * i + 3] = q4.w;
            }
            const float g_k = __ldg(gk + li), g_v = __ldg(gv + li);
            const float enc_k = __frcp_rn(__fmul_rn(6.0f, g_k)), enc_v = __frcp_rn(__fmul_rn(6.0f, g_v));
            uint8_t* layer_cache = cache + (size_t)li * layer_stride;
            const int st = j % kAppendStages;
            // warp-uniform outcome: a warp never splits before its shuffles
            if (!mbar_wait_warp(&full[st], (j / kAppendStages) & 1)) {
                atomicOr(&s_timeout, 1);
                break;
            }
            const T* stage = reinterpret_cast<const T*>(smem + st * kAppendStageBytes);
            // Every lane runs the same number of iterations (the rotation's
            // butterflies are full-warp shuffles, and a warp may hold the
            // lanes of two tokens or idle lanes when 8 Hkv does not divide
            // 256): lanes without a token compute on zeros and store nothing.
            for (int base = 0; base < n; base += tpc) {
                const int tt = base + sub;
                const bool live = active && tt < n;
                const int64_t slot = live ? __ldg(slots + t0 + tt) : -1;
                const bool ok = slot >= 0 && slot < (int64_t)num_pages * kPage;
                if (live && slot >= (int64_t)num_pages * kPage && t == 0) set_status(status, KVQ_DEV_BAD_SLOT);
                float y[kBlk];
                const size_t e = (size_t)(live ? tt : 0) * row + h * kD + blk * kBlk;
                if (live) {
                    load16_smem<T>(stage + e, y);
                } else {
#pragma unroll
                    for (int i = 0; i < kBlk; ++i) y[i] = 0.0f;
                }
                // key: smoothing multiply, then the optional rotation
#pragma unroll
                for (int i = 0; i < kBlk; ++i) y[i] = __fmul_rn(y[i], inv[i]);
                if (hadamard) hadamard_block(y, blk);
                uint2 codes;
                uint32_t sf;
                quantize_block(y, g_k, enc_k, codes, sf);
                const int64_t page = slot >> 4;
                const int off = (int)(slot & 15);
                uint8_t* tile = layer_cache + ((size_t)page * Hkv + h) * kTile;
                if (ok) {
                    *reinterpret_cast<uint2*>(tile + kKCodes + off * 64 + blk * 8) = codes;
                    tile[kKScales + off * 8 + blk] = (uint8_t)sf;
                }
                if (live) {
                    load16_smem<T>(stage + half_stage / sizeof(T) + e, y);
                } else {
#pragma unroll
                    for (int i = 0; i < kBlk; ++i) y[i] = 0.0f;
                }
                quantize_block(y, g_v, enc_v, codes, sf);
                if (ok) {
                    *reinterpret_cast<uint2*>(tile + kVCodes + off * 64 + blk * 8) = codes;
                    tile[kVScales + blk * 16 + off] = (uint8_t)sf;
                }
            }
            __syncwarp();
            if ((threadIdx.x & 31) == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(
                                                          smem_u32(&empty[st])) : "memory");
        }
    }
    __syncthreads();
    if (s_timeout && threadIdx.x == 32 * workers) {
        // wait (bounded) for the copies still in flight before leaving
        const int issued = s_issued;
        for (int j = max(0, issued - kAppendStages); j < issued; ++j)
            (void)mbar_wait(&full[j % kAppendStages], (j / kAppendStages) & 1);
        set_status(status, KVQ_DEV_TIMEOUT);
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
    // tokens per chunk: key rows of one chunk fill half a stage
    const int row_bytes = H * kD * (dtype == KVQ_F32 ? 4 : 2);
    const int tc = max(1, (kAppendStageBytes / 2) / row_bytes);
    const long items = (long)((num_tokens + tc - 1) / tc) * nlayers;
    const int threads = 288;
    const size_t smem = (size_t)kAppendStages * kAppendStageBytes;
    int dev = 0, sms = 148, per_sm = 2;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e;
    if (dtype == KVQ_F32) {
        e = cudaFuncSetAttribute(append_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, append_kernel<float>, threads, smem);
    } else {
        e = cudaFuncSetAttribute(append_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, append_kernel<__nv_bfloat16>, threads, smem);
    }
    if (e != cudaSuccess) return KVQ_ECUDA;
    const long wave = (long)sms * max(per_sm, 1);
    const int grid = (int)(items < wave ? items : wave);
    if (dtype == KVQ_F32)
        append_kernel<float><<<grid, threads, smem, st>>>((const float*)k, (const float*)v, slots, num_tokens,
                                                        nlayers, H, tc, inv_s, gk, gv, base, cache.layer_stride_bytes,
                                                        cache.num_pages, s.use_hadamard, status);
    else
        append_kernel<__nv_bfloat16><<<grid, threads, smem, st>>>(
            (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, slots, num_tokens, nlayers, H, tc, inv_s, gk, gv, base,
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
