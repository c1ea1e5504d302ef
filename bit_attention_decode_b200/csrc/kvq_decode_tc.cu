// kvq_decode_tc.cu -- split-K decode over the packed NVFP4 cache, with the
// per-page contractions on the tensor cores (mma.sync m16n8k16, fp16 in,
// fp32 accumulate) and the dequantisation in registers.
//
// Why tensor cores in a bandwidth-bound kernel: one 16-token page of one kv
// head is 2304 bytes but carries 16 x 128 x 4 multiply-adds for Q.K and as
// many for P.V (GQA group of 4).  At the HBM roof that is ~125 FP32 FMAs per
// clock per SM -- the whole FP32 pipe -- before any dequantisation; the
// tensor cores take the contractions and leave the ALUs the dequantisation
// and the online softmax.  Every dequantised E2M1 x E4M3 product is exact in
// fp16; the query is split into fp16 hi + lo columns (its rounding would
// otherwise reach the scores at ~1e-2), the probabilities are rounded once to
// fp16 (relative error <= 2^-11 per weight), and everything accumulates in
// fp32.
//
// Work unit (one CTA): one layer, one sequence, one split of its pages, all
// kv heads.  Warp Hkv is the producer: it streams whole pages (Hkv x 2304
// contiguous bytes per layer) into a ring of shared-memory stages with
// cp.async.bulk and mbarrier transaction counts.  Warps 0..Hkv-1 consume:
// warp h owns kv head h and its G <= 4 query heads.
//
// Method: "NVFP4 attention cache on W4A4 Qwen3-8B" (rstation.ai), setup and
// observation 2 (the smoothing folded into the query); "QServe
// SmoothAttention" record, Kernels field (fused attention made memory-bound
// on the 4-bit cache).
#include "kvq_attn.cuh"
#include "kvq_common.cuh"
#include "kvq_internal.h"
#include "kvq_sync.cuh"

namespace kvq {

constexpr int kStages = 6;
constexpr unsigned kFull = 0xFFFFFFFFu;

// ------------------------------------------------------------------ primitives
__device__ __forceinline__ void mma16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// the same with bf16 operands (keys of the mixed cache)
__device__ __forceinline__ void mma16816_bf16(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ float2 unpack_bf2(uint32_t a) {
    return make_float2(__uint_as_float(a << 16), __uint_as_float(a & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    __half2 r = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ float2 unpack_h2(uint32_t a) {
    return __half22float2(*reinterpret_cast<__half2*>(&a));
}
__device__ __forceinline__ uint32_t bcast_lo(uint32_t h2) { return (h2 & 0xFFFFu) | (h2 << 16); }
__device__ __forceinline__ uint32_t bcast_hi(uint32_t h2) { return (h2 & 0xFFFF0000u) | (h2 >> 16); }
// barrier of the consumer warps alone (the producer warp has exited)
__device__ __forceinline__ void consumers_sync(int threads) {
    asm volatile("bar.sync 1, %0;" ::"r"(threads) : "memory");
}
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// four bytes of E2M1 code pairs -> four f16x2 (byte j -> r[j])
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t* r) {
    asm("{ .reg .b8 b0, b1, b2, b3; mov.b32 {b0, b1, b2, b3}, %4;\n"
        "  cvt.rn.f16x2.e2m1x2 %0, b0; cvt.rn.f16x2.e2m1x2 %1, b1;\n"
        "  cvt.rn.f16x2.e2m1x2 %2, b2; cvt.rn.f16x2.e2m1x2 %3, b3; }"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
        : "r"(w));
}

template <typename T>
__device__ __forceinline__ void load32(const T* p, float* x);
template <>
__device__ __forceinline__ void load32<float>(const float* p, float* x) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float4 t = __ldg(reinterpret_cast<const float4*>(p) + i);
        x[4 * i] = t.x; x[4 * i + 1] = t.y; x[4 * i + 2] = t.z; x[4 * i + 3] = t.w;
    }
}
template <>
__device__ __forceinline__ void load32<__nv_bfloat16>(const __nv_bfloat16* p, float* x) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint4 t = __ldg(reinterpret_cast<const uint4*>(p) + i);
        uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            x[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            x[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

__device__ __forceinline__ void store16(float* p, const float* x) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
        reinterpret_cast<float4*>(p)[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
}
__device__ __forceinline__ void store16(__nv_bfloat16* p, const float* x) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        __nv_bfloat162 t = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&t);
    }
    reinterpret_cast<uint4*>(p)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(p)[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// ------------------------------------------------------------------ split merge
// Log-sum-exp merge of one query head's split partials (m: reference in log2
// units, INFINITY for a poisoned split, -INFINITY for an empty one; l: sum of
// weights; o: weighted values) in split order, scaled by g_V / l; a lane
// handles 4 dims.  A poisoned or empty row is written as zeros.
__device__ __forceinline__ void store4(float* p, const float* r) {
    *reinterpret_cast<float4*>(p) = make_float4(r[0], r[1], r[2], r[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float* r) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf2(r[0], r[1]), pack_bf2(r[2], r[3]));
}
template <typename TO>
__device__ __forceinline__ void merge_store(const float* m, const float* l, const float4* o, int n, float gv,
                                            TO* dst) {
    float M = -INFINITY;
    bool poison = false;
    for (int sp = 0; sp < n; ++sp) {
        poison |= (m[sp] == INFINITY);
        M = fmaxf(M, m[sp]);
    }
    float L = 0.0f, acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (!poison && M != -INFINITY) {
        for (int sp = 0; sp < n; ++sp) {
            const float w = (m[sp] == -INFINITY) ? 0.0f : exp2f(m[sp] - M);
            L += w * l[sp];
            acc[0] += w * o[sp].x;
            acc[1] += w * o[sp].y;
            acc[2] += w * o[sp].z;
            acc[3] += w * o[sp].w;
        }
    }
    float r[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) r[k] = (poison || L == 0.0f) ? 0.0f : acc[k] / L * gv;
    store4(dst, r);
}
// the same for any number of splits, read from the partials in two passes
template <typename TO>
__device__ __forceinline__ void merge_store_n(const float* base, int n, int lane, float gv, TO* dst) {
    float M = -INFINITY;
    bool poison = false;
    for (int sp = 0; sp < n; ++sp) {
        const float ms = __ldcg(base + (size_t)sp * kPartialStride);
        poison |= (ms == INFINITY);
        M = fmaxf(M, ms);
    }
    float L = 0.0f, acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (!poison && M != -INFINITY) {
        for (int sp = 0; sp < n; ++sp) {
            const float* ps = base + (size_t)sp * kPartialStride;
            const float ms = __ldcg(ps);
            const float w = (ms == -INFINITY) ? 0.0f : exp2f(ms - M);
            L += w * __ldcg(ps + 1);
            const float4 ov = __ldcg(reinterpret_cast<const float4*>(ps + 4) + lane);
            acc[0] += w * ov.x;
            acc[1] += w * ov.y;
            acc[2] += w * ov.z;
            acc[3] += w * ov.w;
        }
    }
    float r[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) r[k] = (poison || L == 0.0f) ? 0.0f : acc[k] / L * gv;
    store4(dst, r);
}

// ------------------------------------------------------------------ kernel
// grid (splits, nlayers, batch); block 32 * (Hkv + 1); dynamic smem
// kStages * Hkv * 2304 + barriers.
template <typename TQ, typename TO, bool KB>
__global__ void __launch_bounds__(288, 2) decode_tc_kernel(AttnArgs a) {
    // KB: keys stored as bf16 (mixed cache, 5248-byte tiles, 2 stages)
    constexpr int kST = KB ? 2 : kStages;
    constexpr int kTB = KB ? kTileBf16K : kTile;
    constexpr int kVC = KB ? kBf16VCodes : kVCodes;
    constexpr int kVS = KB ? kBf16VScales : kVScales;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_flags;    // 1: a bounded wait gave up
    __shared__ int s_issued;   // pages the producer issued
    __shared__ int s_last;     // split merge: this CTA is the unit's last split to finish
    __shared__ int s_badp;     // the producer met a page id outside the pool

    const int Hkv = a.Hkv;
    const uint32_t page_bytes = (uint32_t)Hkv * kTB;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kST * page_bytes);
    uint64_t* empty = full + kST;

    __shared__ int s_seq;      // sequence of this CTA (longest-first order)
    const int split = blockIdx.x, li = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Longest sequences first: blockIdx.z is a rank in decreasing length
    // (ties by index), so the CTAs left at the end of the grid are the short
    // ones.  Ranking costs O(batch^2 / threads) per CTA; past 256 sequences
    // the natural order is used (many small units balance statistically).
    if (a.batch <= 256) {
        const int r = blockIdx.z;
        for (int cand = threadIdx.x; cand < a.batch; cand += blockDim.x) {
            const int lc = __ldg(a.seq_lens + cand);
            int rank = 0;
            for (int j = 0; j < a.batch; ++j) {
                const int lj = __ldg(a.seq_lens + j);
                rank += (lj > lc) || (lj == lc && j < cand);
            }
            if (rank == r) s_seq = cand;
        }
        __syncthreads();
    } else if (threadIdx.x == 0) {
        s_seq = blockIdx.z;
    }
    __syncthreads();
    const int b = s_seq;
    const int len = __ldg(a.seq_lens + b);
    const bool bad_len = len < 0 || len > a.max_pages * kPage;
    const int npages = bad_len ? 0 : (len + kPage - 1) / kPage;
    const int p0 = split * a.pps;
    const int n = max(0, min(npages, p0 + a.pps) - p0);
    const int32_t* pt = a.page_table + (size_t)b * a.max_pages + p0;

    if (threadIdx.x == 0) {
        s_flags = 0;
        s_issued = 0;
        s_badp = 0;
        for (int s = 0; s < kST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], Hkv);
        }
        mbar_fence_init();
        if (bad_len && split == 0) set_status(a.status, KVQ_DEV_BAD_LEN);
    }
    __syncthreads();
    // page ids are checked by the producer as it issues the copies (no
    // up-front pass over the page table delays the first copy); a unit with a
    // bad page is poisoned and its output discarded at the end
    const bool poison = bad_len;
    const uint8_t* layer_base = a.cache + (size_t)li * a.layer_stride;

    // consumer state (kept in registers across the final barrier)
    const int g = lane >> 2, c = lane & 3;
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m_h = -INFINITY, l_h = 0.0f;       // running reference and sum of head c

    if (warp == Hkv) {
        // ---------------------------------------------------------- producer
        if (lane == 0 && !poison) {
            int i = 0;
            int st = 0;
            uint32_t ph = 0;          // parity of round i / kST
            bool bad = false;
            for (; i < n; ++i) {
                if (i >= kST && !mbar_wait(&empty[st], ph ^ 1u)) {
                    atomicOr(&s_flags, 1);
                    break;
                }
                const int pg = __ldg(pt + i);
                bad |= (pg < 0 || pg >= a.num_pages);
                if (bad) {
                    // a page outside the pool, here or earlier: nothing is
                    // copied; the stage completes empty so the consumers
                    // move on, and the unit's result is discarded
                    mbar_arrive(&full[st]);
                } else {
                    mbar_arrive_expect_tx(&full[st], page_bytes);
                    bulk_g2s(smem + st * page_bytes, layer_base + (size_t)pg * page_bytes, page_bytes, &full[st]);
                }
                if (++st == kST) {
                    st = 0;
                    ph ^= 1u;
                }
            }
            s_issued = i;
            if (bad) {
                s_badp = 1;
                set_status(a.status, KVQ_DEV_BAD_PAGE);
            }
        }
    } else if (!poison) {
        // ---------------------------------------------------------- consumer
        const int h = warp;
        const int G = a.G;
        // B-fragment column g of Q.K: head g >> 1, its hi part for even g and
        // its lo part for odd g, so score columns 2c and 2c + 1 are the two
        // parts of head c and a lane adds them without a shuffle
        const int jq = g >> 1;
        const bool head_ok = jq < G;
        // query prologue: lane (g, c) holds dims 32c..32c+31 of head jq
        float qv[32];
        {
            const TQ* qs = reinterpret_cast<const TQ*>(a.q) +
                           (((size_t)li * a.batch + b) * a.Hq + h * G + (head_ok ? jq : 0)) * kD + 32 * c;
            load32<TQ>(qs, qv);
            float scale;
            if constexpr (KB) {
                // bf16 keys are stored as given: the query is used unchanged
#pragma unroll
                for (int i = 0; i < 32; ++i) qv[i] = head_ok ? qv[i] : 0.0f;
                scale = kLog2e * kInvSqrt128;
            } else {
                if (a.qpre) {
                    // the KLT cache: q already carries the smoothing and the rotation
#pragma unroll
                    for (int i = 0; i < 32; ++i) qv[i] = head_ok ? qv[i] : 0.0f;
                } else {
                    const float* srow = a.smooth + ((size_t)li * Hkv + h) * kD + 32 * c;
#pragma unroll
                    for (int i = 0; i < 32; ++i) qv[i] = head_ok ? qv[i] * __ldg(srow + i) : 0.0f;
                }
                scale = __ldg(a.gk + li) * kLog2e * kInvSqrt128;
            }
            if (!KB && a.hadamard) {
#pragma unroll
                for (int hh = 1; hh < 32; hh <<= 1)
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if ((j & hh) == 0) {
                            const float x = qv[j], y = qv[j + hh];
                            qv[j] = x + y;
                            qv[j + hh] = x - y;
                        }
#pragma unroll
                for (int m = 1; m <= 2; m <<= 1) {
                    const bool upper = (c & m) != 0;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float y = __shfl_xor_sync(kFull, qv[j], m);
                        qv[j] = upper ? y - qv[j] : qv[j] + y;
                    }
                }
                scale *= kInvSqrt128;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) qv[i] *= scale;
        }
        // power-of-two normalisation of each head into the fp16 range
        float mx = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) mx = fmaxf(mx, fabsf(qv[i]));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        int ex = 0;
        if (mx > 0.0f) {
            frexpf(mx, &ex);
            ex = max(ex - 1, -100);
        }
        const float sig = ldexpf(1.0f, 14 - ex), isig = ldexpf(1.0f, ex - 14);
        uint32_t qb[16];
#pragma unroll
        for (int s = 0; s < 8; ++s)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const float x0 = qv[4 * s + 2 * r] * sig, x1 = qv[4 * s + 2 * r + 1] * sig;
                if constexpr (KB) {
                    // bf16 hi + lo: 16 significant bits of the query
                    const uint32_t hv = pack_bf2(x0, x1);
                    const float2 f = unpack_bf2(hv);
                    qb[2 * s + r] = (g & 1) ? pack_bf2(x0 - f.x, x1 - f.y) : hv;
                } else {
                    const uint32_t hv = pack_h2(x0, x1);
                    const float2 f = unpack_h2(hv);
                    qb[2 * s + r] = (g & 1) ? pack_h2(x0 - f.x, x1 - f.y) : hv;
                }
            }
        const float isg = __shfl_sync(kFull, isig, 8 * c);   // head c's normalisation (lane g = 2c)
        float thr = -INFINITY;   // raw-score threshold (m + 8) / isg past which m moves

        const uint8_t* my_tile = smem + h * kTB;
        int st = 0;
        uint32_t ph = 0;              // parity of round i / kST
        for (int i = 0; i < n; ++i) {
            if (!mbar_wait(&full[st], ph)) {
                atomicOr(&s_flags, 1);
                break;
            }
            const uint8_t* T = my_tile + st * page_bytes;
            const int nvalid = min(kPage, len - (p0 + i) * kPage);
            uint2 v0, v1, v2, v3;
            uint32_t vs01, vs89;
            // ---- S = K q~ : tokens (rows) x [hi, lo of head 0, ..., hi, lo of head 3] (cols);
            // two accumulators (even / odd words) halve the dependent MMA chain
            float sacc[4] = {0.0f, 0.0f, 0.0f, 0.0f}, sacc2[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            if constexpr (KB) {
                v0 = *reinterpret_cast<const uint2*>(T + kVC + (2 * c) * 64 + 8 * g);
                v1 = *reinterpret_cast<const uint2*>(T + kVC + (2 * c + 1) * 64 + 8 * g);
                v2 = *reinterpret_cast<const uint2*>(T + kVC + (2 * c + 8) * 64 + 8 * g);
                v3 = *reinterpret_cast<const uint2*>(T + kVC + (2 * c + 9) * 64 + 8 * g);
                vs01 = *reinterpret_cast<const uint16_t*>(T + kVS + 16 * g + 2 * c);
                vs89 = *reinterpret_cast<const uint16_t*>(T + kVS + 16 * g + 2 * c + 8);
                // bf16 key rows g and g + 8, dims 32c..32c+31: 16 bytes give
                // the A operands of two k-steps, in the order of the query's
                // B operands (the same contraction order as the packed keys)
                const uint8_t* ra = T + g * 256 + 64 * c;
                const uint8_t* rb = ra + 8 * 256;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint4 x = *reinterpret_cast<const uint4*>(ra + 16 * u);
                    const uint4 y = *reinterpret_cast<const uint4*>(rb + 16 * u);
                    float* acc = (u & 1) ? sacc2 : sacc;
                    mma16816_bf16(acc, x.x, y.x, x.y, y.y, qb[4 * u], qb[4 * u + 1]);
                    mma16816_bf16(acc, x.z, y.z, x.w, y.w, qb[4 * u + 2], qb[4 * u + 3]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            } else {
                // everything this warp needs from the stage, then release it
                const uint4 kA = *reinterpret_cast<const uint4*>(T + kKCodes + g * 64 + 16 * c);
                const uint4 kB = *reinterpret_cast<const uint4*>(T + kKCodes + (g + 8) * 64 + 16 * c);
                const uint32_t ksA = *reinterpret_cast<const uint16_t*>(T + kKScales + g * 8 + 2 * c);
                const uint32_t ksB = *reinterpret_cast<const uint16_t*>(T + kKScales + (g + 8) * 8 + 2 * c);
                v0 = *reinterpret_cast<const uint2*>(T + kVC + (2 * c) * 64 + 8 * g);
                v1 = *reinterpret_cast<const uint2*>(T + kVC + (2 * c + 1) * 64 + 8 * g);
                v2 = *reinterpret_cast<const uint2*>(T + kVC + (2 * c + 8) * 64 + 8 * g);
                v3 = *reinterpret_cast<const uint2*>(T + kVC + (2 * c + 9) * 64 + 8 * g);
                vs01 = *reinterpret_cast<const uint16_t*>(T + kVS + 16 * g + 2 * c);
                vs89 = *reinterpret_cast<const uint16_t*>(T + kVS + 16 * g + 2 * c + 8);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);

                const uint32_t sfA = e4m3x2_to_f16x2(ksA), sfB = e4m3x2_to_f16x2(ksB);
                const uint32_t sc[4] = {bcast_lo(sfA), bcast_hi(sfA), bcast_lo(sfB), bcast_hi(sfB)};
                const uint32_t wa[4] = {kA.x, kA.y, kA.z, kA.w}, wb[4] = {kB.x, kB.y, kB.z, kB.w};
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t ra[4], rb[4];
                    e2m1x8_to_f16x2(wa[w], ra);
                    e2m1x8_to_f16x2(wb[w], rb);
                    const uint32_t sa = sc[w >> 1], sb = sc[2 + (w >> 1)];
                    float* acc = (w & 1) ? sacc2 : sacc;
                    // word w holds k-steps 2w (bytes 0, 1) and 2w + 1 (bytes 2, 3)
                    mma16816(acc, hmul2(ra[0], sa), hmul2(rb[0], sb), hmul2(ra[1], sa), hmul2(rb[1], sb),
                             qb[4 * w], qb[4 * w + 1]);
                    mma16816(acc, hmul2(ra[2], sa), hmul2(rb[2], sb), hmul2(ra[3], sa), hmul2(rb[3], sb),
                             qb[4 * w + 2], qb[4 * w + 3]);
                }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) sacc[k] += sacc2[k];
            // hi + lo columns -> scores of head c for tokens g, g + 8
            float s0 = sacc[0] + sacc[1];
            float s1 = sacc[2] + sacc[3];
            if (nvalid < kPage) {
                if (g >= nvalid) s0 = -INFINITY;
                if (g + 8 >= nvalid) s1 = -INFINITY;
                // stale slots past the end may hold anything: zero their value scales
                const uint32_t m01 = ((2 * c < nvalid) ? 0xFFFFu : 0u) | ((2 * c + 1 < nvalid) ? 0xFFFF0000u : 0u);
                const uint32_t m89 = ((2 * c + 8 < nvalid) ? 0xFFFFu : 0u) | ((2 * c + 9 < nvalid) ? 0xFFFF0000u : 0u);
                vs01 = e4m3x2_to_f16x2(vs01) & m01;
                vs89 = e4m3x2_to_f16x2(vs89) & m89;
            } else {
                vs01 = e4m3x2_to_f16x2(vs01);
                vs89 = e4m3x2_to_f16x2(vs89);
            }
            // ---- online softmax (exp2 domain) with a lazy reference: m moves
            // only when a score of this page exceeds it by more than 8 (a
            // weight above 2^8), so most pages skip the cross-lane max and the
            // rescale.  Any common reference gives the same o / l; bounding the
            // weights by 2^8 keeps them, scaled by 2^7, inside fp16.
            const float lm = fmaxf(s0, s1);
            if (__any_sync(kFull, lm > thr)) {
                float pm = lm;
#pragma unroll
                for (int x = 4; x < 32; x <<= 1) pm = fmaxf(pm, __shfl_xor_sync(kFull, pm, x));
                const float mn = fmaxf(m_h, pm * isg);
                const float al = fast_exp2(m_h - mn);
                l_h *= al;
                // output columns 2c, 2c + 1 are heads (2c) & 3, (2c + 1) & 3
                const float al_a = __shfl_sync(kFull, al, (lane & ~3) | ((2 * c) & 3));
                const float al_b = __shfl_sync(kFull, al, (lane & ~3) | ((2 * c + 1) & 3));
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    o[t][0] *= al_a; o[t][2] *= al_a;
                    o[t][1] *= al_b; o[t][3] *= al_b;
                }
                m_h = mn;
                thr = (mn + 8.0f) * __frcp_rn(isg);   // exact: isg is a power of two
            }
            // weights (<= 2^8 against the reference) scaled by 2^7 for the fp16 operand
            const float ca = 7.0f - m_h;
            const float p0 = fast_exp2(fmaf(s0, isg, ca)), p1 = fast_exp2(fmaf(s1, isg, ca));
            l_h += p0 + p1;
            // P (fp16, relative rounding <= 2^-11) as the B operand [tokens] x
            // [4 heads | the same 4 heads again]: lane (g, c) needs tokens 2c,
            // 2c + 1 (b0) and 2c + 8, 2c + 9 (b1) of head g & 3, held by lanes
            // (2c, g & 3) and (2c + 1, g & 3) as their (token, token + 8) pairs
            const uint32_t pp = pack_h2(p0, p1);
            const uint32_t x = __shfl_sync(kFull, pp, (c << 3) | (g & 3));
            const uint32_t y = __shfl_sync(kFull, pp, (c << 3) | 4 | (g & 3));
            const uint32_t pb0 = __byte_perm(x, y, 0x5410), pb1 = __byte_perm(x, y, 0x7632);
            // ---- O^T += V^T P : rows = dims 16g + 2t (+1), k = tokens
            const uint32_t w0[2] = {v0.x, v0.y}, w1[2] = {v1.x, v1.y};
            const uint32_t w2[2] = {v2.x, v2.y}, w3[2] = {v3.x, v3.y};
#pragma unroll
            for (int wi = 0; wi < 2; ++wi) {
                // pair tokens (2c, 2c+1) and (2c+8, 2c+9) nibble by nibble
                const uint32_t L01 = (w0[wi] & 0x0F0F0F0Fu) | ((w1[wi] << 4) & 0xF0F0F0F0u);
                const uint32_t H01 = ((w0[wi] >> 4) & 0x0F0F0F0Fu) | (w1[wi] & 0xF0F0F0F0u);
                const uint32_t L89 = (w2[wi] & 0x0F0F0F0Fu) | ((w3[wi] << 4) & 0xF0F0F0F0u);
                const uint32_t H89 = ((w2[wi] >> 4) & 0x0F0F0F0Fu) | (w3[wi] & 0xF0F0F0F0u);
                uint32_t rl01[4], rh01[4], rl89[4], rh89[4];
                e2m1x8_to_f16x2(L01, rl01);
                e2m1x8_to_f16x2(H01, rh01);
                e2m1x8_to_f16x2(L89, rl89);
                e2m1x8_to_f16x2(H89, rh89);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma16816(o[4 * wi + j], hmul2(rl01[j], vs01), hmul2(rh01[j], vs01), hmul2(rl89[j], vs89),
                             hmul2(rh89[j], vs89), pb0, pb1);
            }
            if (++st == kST) {
                st = 0;
                ph ^= 1u;
            }
        }
    }

    __syncthreads();
    const bool timed_out = s_flags != 0;
    if (timed_out && threadIdx.x == 32 * Hkv) {
        // drain: wait (bounded) for every copy still in flight before exiting
        const int issued = s_issued;
        for (int st = 0; st < kST && st < issued; ++st) {
            const int last = st + ((issued - 1 - st) / kST) * kST;
            (void)mbar_wait(&full[st], (last / kST) & 1);
        }
        set_status(a.status, KVQ_DEV_TIMEOUT);
    }
    if (warp >= Hkv) return;

    // ------------------------------------------------------------------ epilogue
    const bool dead = poison || timed_out || s_badp != 0;
#pragma unroll
    for (int x = 4; x < 32; x <<= 1) {
        l_h += __shfl_xor_sync(kFull, l_h, x);
    }
    // lane (g, c) writes dims 16g..16g+15 of one head: c < 2 -> head 2c (its
    // column 2c), else head 2(c-2)+1 (its column 2c + 1, which repeats it)
    const int h = warp;
    const bool first = c < 2;
    const int head = first ? 2 * c : 2 * (c - 2) + 1;
    // head's sum and reference live in lanes (g, head)
    const float l = __shfl_sync(kFull, l_h, (lane & ~3) | head);
    const float m = __shfl_sync(kFull, m_h, (lane & ~3) | head);
    if (head < a.G) {
        float r[16];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            r[2 * t] = first ? o[t][0] : o[t][1];
            r[2 * t + 1] = first ? o[t][2] : o[t][3];
        }
        const int hq = h * a.G + head;
        if (a.splits == 1) {
            // (a poisoned unit may have computed on stale stages: select, not scale)
            const bool zero = dead || l == 0.0f;
            const float sc = zero ? 0.0f : __ldg(a.gv + li) / l;
#pragma unroll
            for (int k = 0; k < 16; ++k) r[k] = zero ? 0.0f : r[k] * sc;
            store16(reinterpret_cast<TO*>(a.out) + (((size_t)li * a.batch + b) * a.Hq + hq) * kD + 16 * g, r);
        } else {
            float* part = a.partials + ((((size_t)li * a.batch + b) * a.Hq + hq) * a.splits + split) * kPartialStride;
            if (g == 0) {
                part[0] = dead ? INFINITY : m;
                part[1] = l;
            }
            store16(part + 4 + 16 * g, r);
        }
    }
    if (a.splits == 1) return;

    // ---- split merge, fused: the last split of a (layer, sequence) unit to
    // arrive merges the partials of all its splits, in split order (so the
    // result does not depend on which split came last), and resets the
    // unit's arrival counter for the next call.
    consumers_sync(32 * Hkv);                          // every partial of this CTA is written
    if (threadIdx.x == 0) {
        __threadfence();                               // ... and visible, before the arrival
        unsigned* ctr = a.counters + (size_t)li * a.batch + b;
        const unsigned old = atomicAdd(ctr, 1u);
        const bool last = old + 1u == (unsigned)a.splits;
        if (last) atomicExch(ctr, 0u);
        // a counter that did not start at zero: the workspace header was not zero-filled
        if (old >= (unsigned)a.splits) set_status(a.status, KVQ_DEV_BAD_WORKSPACE);
        s_last = last;
    }
    consumers_sync(32 * Hkv);
    if (!s_last) return;
    __threadfence();
    // warp h merges the G query heads of kv head h; lane covers dims 4 lane .. 4 lane + 3
    const float gvl = __ldg(a.gv + li);
    const size_t row0 = ((size_t)li * a.batch + b) * a.Hq + (size_t)h * a.G;   // first query head of the warp
    TO* dst0 = reinterpret_cast<TO*>(a.out) + row0 * kD + 4 * lane;
    if (a.splits == 2) {
        // every load of the merge issued at once: one round trip to L2
        float mv[4][2], lv[4][2];
        float4 ov[4][2];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int sp = 0; sp < 2; ++sp) {
                mv[j][sp] = -INFINITY;
                lv[j][sp] = 0.0f;
                ov[j][sp] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (j < a.G) {
                    const float* ps = a.partials + ((row0 + j) * 2 + sp) * kPartialStride;
                    mv[j][sp] = __ldcg(ps);
                    lv[j][sp] = __ldcg(ps + 1);
                    ov[j][sp] = __ldcg(reinterpret_cast<const float4*>(ps + 4) + lane);
                }
            }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (j >= a.G) break;
            merge_store<TO>(mv[j], lv[j], ov[j], 2, gvl, dst0 + (size_t)j * kD);
        }
    } else {
        for (int j = 0; j < a.G; ++j) {
            const float* base = a.partials + (row0 + j) * a.splits * kPartialStride;
            merge_store_n<TO>(base, a.splits, lane, gvl, dst0 + (size_t)j * kD);
        }
    }
}

// ------------------------------------------------------------------ launcher
size_t decode_tc_smem(int Hkv, bool kbf16) {
    const int stages = kbf16 ? 2 : kStages;
    return (size_t)stages * Hkv * (kbf16 ? kTileBf16K : kTile) + 2 * stages * sizeof(uint64_t);
}

template <typename TQ, typename TO, bool KB>
static cudaError_t launch_one(const AttnArgs& a, dim3 grid, cudaStream_t st) {
    const size_t smem = decode_tc_smem(a.Hkv, KB);
    cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<TQ, TO, KB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    decode_tc_kernel<TQ, TO, KB><<<grid, 32 * (a.Hkv + 1), smem, st>>>(a);
    return cudaGetLastError();
}

template <bool KB>
static cudaError_t launch_kf(const AttnArgs& a, dim3 grid, bool q_bf16, bool out_bf16, cudaStream_t st) {
    if (q_bf16 && out_bf16) return launch_one<__nv_bfloat16, __nv_bfloat16, KB>(a, grid, st);
    if (q_bf16) return launch_one<__nv_bfloat16, float, KB>(a, grid, st);
    if (out_bf16) return launch_one<float, __nv_bfloat16, KB>(a, grid, st);
    return launch_one<float, float, KB>(a, grid, st);
}

cudaError_t launch_decode_tc(const AttnArgs& a, int nlayers, bool q_bf16, bool out_bf16, cudaStream_t st) {
    dim3 grid(a.splits, nlayers, a.batch);
    if (a.kbf16) return launch_kf<true>(a, grid, q_bf16, out_bf16, st);
    return launch_kf<false>(a, grid, q_bf16, out_bf16, st);
}

}  // namespace kvq
