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
#include "kvq_transform.cuh"

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
    float2 y[kBlk / 2], x[kBlk / 2];
    load16(k + off, y);
    load16(v + off, x);
    smooth_block(y, inv_s + ((size_t)l * Hkv + h) * kD + blk * kBlk);
    if (hadamard) hadamard_block(y, blk);
    float ak = absmax16(y), av = absmax16(x);
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
// enc = 1/(6 g); rtab[c] = 1/(val(c) g) for every scale code c (0 where the
// product is zero), both computed once per tensor.
__device__ __forceinline__ void quantize_block(const float2* y, float enc, const float* rtab, uint2& codes,
                                               uint32_t& sf) {
    sf = e4m3_rn(__fmul_rn(absmax16(y), enc));
    const float r = rtab[sf & 0x7Fu];
    const float2 r2 = make_float2(r, r);
    float2 z[kBlk / 2];
#pragma unroll
    for (int i = 0; i < kBlk / 2; ++i) z[i] = fmul2(y[i], r2);
    codes = make_uint2(e2m1x8_rn(z[0], z[1], z[2], z[3]), e2m1x8_rn(z[4], z[5], z[6], z[7]));
}

// Bulk-copy staging of the inputs.  A work item is a chunk of `tc`
// consecutive tokens of one layer: its key rows and value rows are two
// contiguous ranges (tc x Hkv x 128 elements each), streamed into a ring of
// kAppendStages shared-memory stages with cp.async.bulk and an mbarrier
// transaction count.  The producer warp also copies the chunk's slots into
// the stage's slot array, so that no worker waits on a global load per
// token, and (when the stage last held another layer) writes the layer's
// quantiser constants: enc = 1/(6 g) and the reciprocal 1/(val(c) g) of
// every E4M3 scale code c, for the keys and for the values.  A block then
// looks its reciprocal up instead of dividing.  A stage is full once the
// copies have landed and the producer has arrived twice (before the copies,
// and after its shared-memory stores).
// Quantisation then reads the stage: a token takes Hkv * 8 threads, thread
// (h, blk) owning block blk of head h for both the key and the value row; a
// CTA of 256 worker threads works on 256 / (8 Hkv) tokens at a time.  With
// the rotation Hkv is even, so every warp lies inside one token and the
// cross-lane butterflies stay uniform.
constexpr int kAppendStages = 3;
constexpr int kAppendStageBytes = 32768;   // key + value rows of one chunk
constexpr int kAppendMaxChunk = 64;        // tokens: bf16 rows of one kv head fill half a stage

template <typename T>
__global__ void __launch_bounds__(288, 2)
append_kernel(const T* __restrict__ k, const T* __restrict__ v, const int64_t* __restrict__ slots,
              int num_tokens, int nlayers, int Hkv, int tc, const float* __restrict__ inv_s,
              const float* __restrict__ gk, const float* __restrict__ gv, uint8_t* __restrict__ cache,
              int64_t layer_stride, int num_pages, int hadamard, int k_bf16, int32_t* __restrict__ status) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t full[kAppendStages], empty[kAppendStages];
    __shared__ int64_t s_slot[kAppendStages][kAppendMaxChunk];
    __shared__ float s_rtab[kAppendStages][2][128];           // [stage][key, value][scale code]
    __shared__ float s_enc[kAppendStages][2];
    __shared__ int s_layer[kAppendStages];                    // layer of the stage's constants
    __shared__ int s_timeout, s_issued;
    const int row = Hkv * kD;                                  // elements per token row
    const uint32_t half_stage = kAppendStageBytes / 2;         // key rows, then value rows
    const int chunks = (num_tokens + tc - 1) / tc;
    const long items = (long)chunks * nlayers;
    // a contiguous run of items per CTA: its layer (and so the stage's
    // constants) changes at most a few times
    const long per = items / gridDim.x, extra = items % gridDim.x;
    const long first = blockIdx.x * per + min((long)blockIdx.x, extra);
    const int mine = (int)(per + ((long)blockIdx.x < extra ? 1 : 0));
    const int workers = 8;                                     // warps 0..7; warp 8 streams the inputs
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t num_slots = (int64_t)num_pages * kPage;
    // tile geometry: NVFP4 keys, or bf16 keys (mixed cache)
    // k_bf16: 0 packed keys, 1 bf16 keys (mixed cache), 2 keys written by the
    // KLT kernel (packed layout, this kernel does the values only)
    const int tile_b = k_bf16 == 1 ? kTileBf16K : kTile;
    const int v_codes = k_bf16 == 1 ? kBf16VCodes : kVCodes, v_scales = k_bf16 == 1 ? kBf16VScales : kVScales;

    if (threadIdx.x == 0) {
        s_timeout = 0;
        s_issued = 0;
        for (int i = 0; i < kAppendStages; ++i) {
            mbar_init(&full[i], 2);
            mbar_init(&empty[i], workers);
            s_layer[i] = -1;
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == workers) {
        // ---------------------------------------------------------- producer
        int j = 0;
        for (; j < mine; ++j) {
            const int st = j % kAppendStages;
            if (j >= kAppendStages && !mbar_wait_warp(&empty[st], ((j / kAppendStages) - 1) & 1)) {
                if (lane == 0) atomicOr(&s_timeout, 1);
                break;
            }
            const long it = first + j;
            const int li = (int)(it / chunks), t0 = (int)(it % chunks) * tc;
            const int n = min(tc, num_tokens - t0);
            if (lane == 0) {
                const uint32_t bytes = (uint32_t)n * row * sizeof(T);
                uint8_t* dst = smem + st * kAppendStageBytes;
                const size_t off = ((size_t)li * num_tokens + t0) * row;
                mbar_arrive_expect_tx(&full[st], 2 * bytes);
                bulk_g2s(dst, k + off, bytes, &full[st]);
                bulk_g2s(dst + half_stage, v + off, bytes, &full[st]);
            }
            for (int x = lane; x < n; x += 32) s_slot[st][x] = __ldg(slots + t0 + x);
            if (s_layer[st] != li) {
                // the same operations, in the same fp32 order, as a per-block
                // d = val(sf) * g, r = (d == 0) ? 0 : 1/d
                const float g_k = __ldg(gk + li), g_v = __ldg(gv + li);
                for (int x = lane; x < 256; x += 32) {
                    const float d = __fmul_rn(e4m3_to_f32(x & 127), (x < 128) ? g_k : g_v);
                    s_rtab[st][x >> 7][x & 127] = (d == 0.0f) ? 0.0f : __frcp_rn(d);
                }
                if (lane < 2) s_enc[st][lane] = __frcp_rn(__fmul_rn(6.0f, lane ? g_v : g_k));
                __syncwarp();
                if (lane == 0) s_layer[st] = li;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[st]);
        }
        if (lane == 0) s_issued = j;
    } else {
        // ---------------------------------------------------------- workers
        const int per_tok = Hkv * 8;                           // a multiple of 8: lane & 7 == blk
        const int tpc = (workers * 32) / per_tok;              // tokens side by side
        const int t = threadIdx.x % per_tok, sub = threadIdx.x / per_tok;
        const int h = t >> 3, blk = t & 7;
        const bool active = sub < tpc;
        float2 inv[kBlk / 2];                                  // smoothing factors of layer inv_layer
        int inv_layer = -1;
        for (int j = 0; j < mine; ++j) {
            const long it = first + j;
            const int li = (int)(it / chunks), t0 = (int)(it % chunks) * tc;
            const int n = min(tc, num_tokens - t0);
            if (li != inv_layer) {
                // loaded before waiting for the inputs
                const float4* ip = reinterpret_cast<const float4*>(inv_s + ((size_t)li * Hkv + h) * kD + blk * kBlk);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 f = __ldg(ip + i);
                    inv[2 * i] = make_float2(f.x, f.y);
                    inv[2 * i + 1] = make_float2(f.z, f.w);
                }
                inv_layer = li;
            }
            uint8_t* layer_cache = cache + (size_t)li * layer_stride;
            const int st = j % kAppendStages;
            // warp-uniform outcome: a warp never splits before its shuffles
            if (!mbar_wait_warp(&full[st], (j / kAppendStages) & 1)) {
                if (lane == 0) atomicOr(&s_timeout, 1);
                break;
            }
            const T* stage = reinterpret_cast<const T*>(smem + st * kAppendStageBytes);
            const float enc_k = s_enc[st][0], enc_v = s_enc[st][1];
            const float* rtab_k = s_rtab[st][0];
            const float* rtab_v = s_rtab[st][1];
            // Every lane runs the same number of iterations (the rotation's
            // butterflies are full-warp shuffles, and a warp may hold the
            // lanes of two tokens or idle lanes when 8 Hkv does not divide
            // 256): lanes without a token compute on the chunk's first row
            // and store nothing.  A token's 8 Hkv lanes are consecutive and
            // share its liveness, so no live lane ever exchanges with them.
            for (int base = 0; base < n; base += tpc) {
                const int tt = base + sub;
                const bool live = active && tt < n;
                const int64_t slot = live ? s_slot[st][tt] : -1;
                const bool ok = slot >= 0 && slot < num_slots;
                if (live && slot >= num_slots && t == 0) set_status(status, KVQ_DEV_BAD_SLOT);
                const size_t e = (size_t)(live ? tt : 0) * row + h * kD + blk * kBlk;
                float2 y[kBlk / 2];
                load16(stage + e, y);
                const int64_t page = slot >> 4;
                const int off = (int)(slot & 15);
                uint8_t* tile = layer_cache + ((size_t)page * Hkv + h) * tile_b;
                uint2 codes;
                uint32_t sf;
                if (k_bf16 == 2) {
                    // KLT cache: the keys are transformed and written by their own kernel
                } else if (k_bf16) {
                    // mixed cache: the key block is kept as bf16, untransformed
                    if (ok) {
                        uint32_t wb[8];
#pragma unroll
                        for (int i = 0; i < kBlk / 2; ++i) {
                            const __nv_bfloat162 t2 = __floats2bfloat162_rn(y[i].x, y[i].y);
                            wb[i] = *reinterpret_cast<const uint32_t*>(&t2);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(tile + off * 256 + blk * 32);
                        dst[0] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
                        dst[1] = make_uint4(wb[4], wb[5], wb[6], wb[7]);
                    }
                } else {
                    // key: smoothing multiply, then the optional rotation
#pragma unroll
                    for (int i = 0; i < kBlk / 2; ++i) y[i] = fmul2(y[i], inv[i]);
                    if (hadamard) hadamard_block(y, blk);
                    quantize_block(y, enc_k, rtab_k, codes, sf);
                    if (ok) {
                        *reinterpret_cast<uint2*>(tile + kKCodes + off * 64 + blk * 8) = codes;
                        tile[kKScales + off * 8 + blk] = (uint8_t)sf;
                    }
                }
                load16(stage + half_stage / sizeof(T) + e, y);
                quantize_block(y, enc_v, rtab_v, codes, sf);
                if (ok) {
                    *reinterpret_cast<uint2*>(tile + v_codes + off * 64 + blk * 8) = codes;
                    tile[v_scales + blk * 16 + off] = (uint8_t)sf;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
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
// Each thread converts 8 consecutive inputs with the quantisers' own
// e2m1x8_rn: even inputs go through the low-nibble operand, odd ones through
// the high-nibble operand (a caller checks both by converting x and x + 1).
__global__ void round_e2m1_kernel(const float* __restrict__ x, uint8_t* __restrict__ out, int64_t n) {
    const int64_t groups = (n + 7) / 8;
    for (int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gi < groups;
         gi += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i0 = 8 * gi;
        float v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = (i0 + k < n) ? x[i0 + k] : 0.0f;
        const uint32_t w = e2m1x8_rn(make_float2(v[0], v[1]), make_float2(v[2], v[3]), make_float2(v[4], v[5]),
                                     make_float2(v[6], v[7]));
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (i0 + k < n) out[i0 + k] = (uint8_t)((w >> (4 * k)) & 0xFu);
    }
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

__global__ void fill_kernel(float* __restrict__ x, float value, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) x[i] = value;
}

// Native basis: s = inv = 1, then the tensor scales of the unsmoothed keys
// (the tensor-absmax kernel multiplies by inv = 1, which is exact).
template <typename T>
static kvq_status launch_calibrate_native(const kvq_shape& s, const T* k, const T* v, int W, int Tlen,
                                          const kvq_calib& out, cudaStream_t st) {
    const int L = s.num_layers, H = s.num_kv_heads;
    const int n = L * H * kD;
    if (cudaMemsetAsync(out.k_gscale, 0, L * sizeof(float), st) != cudaSuccess ||
        cudaMemsetAsync(out.v_gscale, 0, L * sizeof(float), st) != cudaSuccess)
        return KVQ_ECUDA;
    fill_kernel<<<(n + 255) / 256, 256, 0, st>>>(out.k_smooth, 1.0f, n);
    fill_kernel<<<(n + 255) / 256, 256, 0, st>>>(out.k_inv_smooth, 1.0f, n);
    const long rows = (long)W * Tlen * H;
    dim3 g3((unsigned)((rows * 8 + 255) / 256), L);
    calib_tensor_amax_kernel<T><<<g3, 256, 0, st>>>(k, v, W, Tlen, H, out.k_inv_smooth, s.use_hadamard,
                                                   reinterpret_cast<uint32_t*>(out.k_gscale),
                                                   reinterpret_cast<uint32_t*>(out.v_gscale));
    calib_finalize_gscale_kernel<<<(L + 63) / 64, 64, 0, st>>>(out.k_gscale, out.v_gscale, L);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

kvq_status calibrate_native(const kvq_shape& s, const void* k, const void* v, int dtype, int W, int Tlen,
                            const kvq_calib& out, cudaStream_t st) {
    if (dtype == KVQ_F32)
        return launch_calibrate_native(s, (const float*)k, (const float*)v, W, Tlen, out, st);
    return launch_calibrate_native(s, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, W, Tlen, out, st);
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
    const int kbf = s.use_klt ? 2 : (s.k_format == KVQ_K_BF16 ? 1 : 0);
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
                                                        cache.num_pages, s.use_hadamard, kbf, status);
    else
        append_kernel<__nv_bfloat16><<<grid, threads, smem, st>>>(
            (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, slots, num_tokens, nlayers, H, tc, inv_s, gk, gv, base,
            cache.layer_stride_bytes, cache.num_pages, s.use_hadamard, kbf, status);
    if (cudaGetLastError() != cudaSuccess) return KVQ_ECUDA;
    if (s.use_klt) return append_klt_keys(s, c, cache, layer0, nlayers, k, dtype, slots, num_tokens, status, st);
    return KVQ_OK;
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
