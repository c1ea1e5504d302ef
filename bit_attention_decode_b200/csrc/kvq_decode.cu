// kvq_decode.cu -- attention over the packed NVFP4 cache: split-K decode, the
// log-sum-exp combine of the splits, and a causal prefill chunk.
//
// The query carries the key smoothing: q~ = q * s (then H q~ / sqrt(128)
// when keys are rotated), so q~ . T(k) = q . k -- "NVFP4 attention cache on
// W4A4 Qwen3-8B" (rstation.ai), observation 2 (SmoothAttention); "QServe
// SmoothAttention" record, Activation scheme field.  The attention reads the
// packed cache directly and is memory-bound on it, as the QServe record's
// Kernels field describes for its 4-bit cache.
#include <math.h>

#include "kvq_common.cuh"
#include "kvq_internal.h"
#include "kvq_attn.cuh"

namespace kvq {

__device__ __forceinline__ void load4(const float* p, float* x) {
    float4 t = *reinterpret_cast<const float4*>(p);
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float* x) {
    uint2 t = *reinterpret_cast<const uint2*>(p);
    x[0] = __uint_as_float(t.x << 16); x[1] = __uint_as_float(t.x & 0xFFFF0000u);
    x[2] = __uint_as_float(t.y << 16); x[3] = __uint_as_float(t.y & 0xFFFF0000u);
}
__device__ __forceinline__ void store4(float* p, const float* x) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float* x) {
    __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
    uint2 t = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
    *reinterpret_cast<uint2*>(p) = t;
}

// Query transform of one head, lane holding dims 4 lane .. 4 lane + 3:
// q~ = q * s, optional normalised Hadamard-128, then the softmax scale
// 1/sqrt(128), log2(e) (scores in the exp2 domain) and the key tensor scale.
__device__ __forceinline__ void query_transform(float* q, const float* srow, int lane, bool hadamard,
                                                float scale) {
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] *= __ldg(srow + 4 * lane + i);
    if (hadamard) {
        float a = q[0], b = q[1], c = q[2], d = q[3];
        q[0] = a + b; q[1] = a - b; q[2] = c + d; q[3] = c - d;
        a = q[0]; b = q[1]; c = q[2]; d = q[3];
        q[0] = a + c; q[1] = b + d; q[2] = a - c; q[3] = b - d;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const bool upper = (lane & m) != 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float o = __shfl_xor_sync(0xFFFFFFFFu, q[i], m);
                q[i] = upper ? o - q[i] : q[i] + o;
            }
        }
        scale *= kInvSqrt128;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] *= scale;
}

// Online-softmax attention of one query head (one warp) over cached tokens
// [tok0, tok1) of one sequence.  Returns the running max m (exp2 domain), the
// sum l and the unnormalised o (value tensor scale not applied).  Sets `bad`
// when a page id is outside the pool.
__device__ __forceinline__ void attend_tokens(const AttnArgs& a, const uint8_t* layer_base, int b, int h,
                                              const float* q, int tok0, int tok1, int lane, float& m,
                                              float& l, float* o, bool& bad) {
    for (int t0 = tok0 & ~15; t0 < tok1; t0 += 16) {
        const int page = __ldg(a.page_table + (size_t)b * a.max_pages + (t0 >> 4));
        if (page < 0 || page >= a.num_pages) { bad = true; return; }
        const uint8_t* tile = layer_base + ((size_t)page * a.Hkv + h) * kTile;
        const int tb = max(tok0, t0) - t0, te = min(tok1 - t0, 16);
        for (int t = tb; t < te; ++t) {
            const uint32_t kc = *reinterpret_cast<const uint16_t*>(tile + kKCodes + t * 64 + 2 * lane);
            const float ksf = e4m3_to_f32(tile[kKScales + t * 8 + (lane >> 2)]);
            const uint32_t k01 = e2m1x2_to_f16x2(kc & 0xFFu), k23 = e2m1x2_to_f16x2(kc >> 8);
            const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&k01));
            const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&k23));
            // the block scale belongs to this lane's 4 dims (block lane / 4)
            float s = (q[0] * f01.x + q[1] * f01.y + q[2] * f23.x + q[3] * f23.y) * ksf;
#pragma unroll
            for (int w = 16; w >= 1; w >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, w);
            const uint32_t vc = *reinterpret_cast<const uint16_t*>(tile + kVCodes + t * 64 + 2 * lane);
            const float vsf = e4m3_to_f32(tile[kVScales + (lane >> 2) * 16 + t]);
            const uint32_t v01 = e2m1x2_to_f16x2(vc & 0xFFu), v23 = e2m1x2_to_f16x2(vc >> 8);
            const float2 g01 = __half22float2(*reinterpret_cast<const __half2*>(&v01));
            const float2 g23 = __half22float2(*reinterpret_cast<const __half2*>(&v23));
            const float v[4] = {g01.x * vsf, g01.y * vsf, g23.x * vsf, g23.y * vsf};
            if (s > m) {
                const float alpha = exp2f(m - s);
                l = l * alpha + 1.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) o[i] = o[i] * alpha + v[i];
                m = s;
            } else {
                const float p = exp2f(s - m);
                l += p;
#pragma unroll
                for (int i = 0; i < 4; ++i) o[i] += p * v[i];
            }
        }
    }
}

// Log-sum-exp merge of the split partials in split order.  A poisoned split
// (bad page or length) zeroes the row.  grid (batch * Hq, nlayers), block 128.
template <typename TO>
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ partials, int splits,
                                                      const float* __restrict__ gv, TO* __restrict__ out,
                                                      int rows) {
    const int row = blockIdx.x, li = blockIdx.y, d = threadIdx.x;
    const float* base = partials + ((size_t)li * rows + row) * splits * kPartialStride;
    float M = -INFINITY;
    bool poison = false;
    for (int s = 0; s < splits; ++s) {
        const float ms = base[(size_t)s * kPartialStride];
        poison |= (ms == INFINITY);
        M = fmaxf(M, ms);
    }
    float L = 0.0f, acc = 0.0f;
    if (!poison && M != -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const float* p = base + (size_t)s * kPartialStride;
            const float w = (p[0] == -INFINITY) ? 0.0f : exp2f(p[0] - M);
            L += w * p[1];
            acc += w * p[4 + d];
        }
    }
    const float r = (poison || L == 0.0f) ? 0.0f : acc / L * __ldg(gv + li);
    TO* dst = out + ((size_t)li * rows + row) * kD + d;
    if constexpr (sizeof(TO) == 4) *dst = r; else *dst = __float2bfloat16_rn(r);
}

// Causal prefill chunk: grid (q_len, batch * Hkv, nlayers); block 32 * G.
// Query i of sequence b attends cached tokens j <= min(q_start + i, len - 1).
template <typename TQ, typename TO>
__global__ void __launch_bounds__(256) prefill_kernel(AttnArgs a) {
    const int i = blockIdx.x, b = blockIdx.y / a.Hkv, h = blockIdx.y % a.Hkv, li = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hq = h * a.G + warp;
    const int len = __ldg(a.seq_lens + b);
    bool bad = false;
    if (len < 0 || len > a.max_pages * kPage) {
        bad = true;
        if (threadIdx.x == 0 && i == 0 && h == 0) set_status(a.status, KVQ_DEV_BAD_LEN);
    }
    const size_t row = ((((size_t)li * a.batch + b) * a.q_len + i) * a.Hq + hq) * kD + 4 * lane;
    float q[4];
    load4(reinterpret_cast<const TQ*>(a.q) + row, q);
    query_transform(q, a.smooth + ((size_t)li * a.Hkv + h) * kD, lane, a.hadamard != 0,
                    __ldg(a.gk + li) * kLog2e * kInvSqrt128);
    float m = -INFINITY, l = 0.0f, o[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (!bad) {
        const int n = min(len, __ldg(a.q_start + b) + i + 1);
        attend_tokens(a, a.cache + (size_t)li * a.layer_stride, b, h, q, 0, n, lane, m, l, o, bad);
        if (bad && lane == 0) set_status(a.status, KVQ_DEV_BAD_PAGE);
    }
    const float sc = (bad || l == 0.0f) ? 0.0f : __ldg(a.gv + li) / l;
    float r[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) r[k] = o[k] * sc;
    store4(reinterpret_cast<TO*>(a.out) + row, r);
}

// ------------------------------------------------------------------ host side
DecodePlan decode_plan(const kvq_shape& s, int nlayers, int batch, int max_pages) {
    // one CTA per (layer, sequence, split) covering all kv heads; aim for two
    // waves at two resident CTAs per SM, splitting sequences only when the
    // (layer, sequence) units alone cannot fill the GPU
    (void)s;
    const long units = (long)nlayers * batch;
    const long target = 148L * 2 * 2;
    int splits = 1;
    if (units < target && max_pages > 8) {
        splits = (int)((target + units - 1) / units);
        splits = min(splits, (max_pages + 7) / 8);   // at least 8 pages per split
    }
    int pps = (max_pages + splits - 1) / splits;
    if (pps < 1) pps = 1;
    splits = (max_pages + pps - 1) / pps;
    if (splits < 1) splits = 1;
    return {pps, splits};
}

size_t decode_workspace(const kvq_shape& s, int nlayers, int batch, int max_pages) {
    DecodePlan p = decode_plan(s, nlayers, batch, max_pages);
    if (p.splits == 1) return 0;
    return (size_t)nlayers * batch * s.num_q_heads * p.splits * kPartialStride * sizeof(float);
}

static AttnArgs make_args(const kvq_shape& s, const kvq_calib& c, const kvq_cache& cache, int layer0,
                          const void* q, const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                          int batch, void* out, int32_t* status) {
    AttnArgs a{};
    a.cache = cache.data + (size_t)layer0 * cache.layer_stride_bytes;
    a.layer_stride = cache.layer_stride_bytes;
    a.num_pages = cache.num_pages;
    a.Hkv = s.num_kv_heads;
    a.Hq = s.num_q_heads;
    a.G = s.num_q_heads / s.num_kv_heads;
    a.hadamard = s.use_hadamard;
    a.smooth = c.k_smooth + (size_t)layer0 * s.num_kv_heads * kD;
    a.gk = c.k_gscale + layer0;
    a.gv = c.v_gscale + layer0;
    a.q = q;
    a.page_table = page_table;
    a.max_pages = max_pages;
    a.seq_lens = seq_lens;
    a.batch = batch;
    a.out = out;
    a.status = status;
    return a;
}

kvq_status decode(const kvq_shape& s, const kvq_calib& c, const kvq_cache& cache, int layer0, int nlayers,
                  const void* q, int q_dtype, const int32_t* page_table, int max_pages,
                  const int32_t* seq_lens, int batch, void* out, int out_dtype, void* ws, size_t ws_bytes,
                  int32_t* status, cudaStream_t st) {
    AttnArgs a = make_args(s, c, cache, layer0, q, page_table, max_pages, seq_lens, batch, out, status);
    DecodePlan p = decode_plan(s, nlayers, batch, max_pages);
    a.splits = p.splits;
    a.pps = p.pages_per_split;
    a.q_len = 1;
    a.partials = reinterpret_cast<float*>(ws);
    const bool qb = q_dtype == KVQ_BF16, ob = out_dtype == KVQ_BF16;
    if (launch_decode_tc(a, nlayers, qb, ob, st) != cudaSuccess) return KVQ_ECUDA;
    if (p.splits > 1) {
        dim3 g2(batch * s.num_q_heads, nlayers);
        if (ob) combine_kernel<__nv_bfloat16><<<g2, kD, 0, st>>>(a.partials, p.splits, a.gv, (__nv_bfloat16*)out, batch * s.num_q_heads);
        else combine_kernel<float><<<g2, kD, 0, st>>>(a.partials, p.splits, a.gv, (float*)out, batch * s.num_q_heads);
    }
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

size_t prefill_workspace(const kvq_shape&, int, int, int) { return 0; }

kvq_status prefill(const kvq_shape& s, const kvq_calib& c, const kvq_cache& cache, int layer0, int nlayers,
                   const void* q, int q_dtype, int q_len, const int32_t* q_start, const int32_t* page_table,
                   int max_pages, const int32_t* seq_lens, int batch, void* out, int out_dtype, void*, size_t,
                   int32_t* status, cudaStream_t st) {
    AttnArgs a = make_args(s, c, cache, layer0, q, page_table, max_pages, seq_lens, batch, out, status);
    a.q_len = q_len;
    a.q_start = q_start;
    dim3 grid(q_len, batch * s.num_kv_heads, nlayers);
    const int threads = 32 * a.G;
    const bool qb = q_dtype == KVQ_BF16, ob = out_dtype == KVQ_BF16;
    if (qb && ob) prefill_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, threads, 0, st>>>(a);
    else if (qb) prefill_kernel<__nv_bfloat16, float><<<grid, threads, 0, st>>>(a);
    else if (ob) prefill_kernel<float, __nv_bfloat16><<<grid, threads, 0, st>>>(a);
    else prefill_kernel<float, float><<<grid, threads, 0, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

}  // namespace kvq
