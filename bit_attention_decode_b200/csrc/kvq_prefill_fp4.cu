// kvq_prefill_fp4.cu -- chunked causal prefill with Q.K on the block-scaled
// FP4 tensor cores (tcgen05.mma kind::mxf4nvf4: E2M1 operands, one E4M3
// scale per 16 elements of K on each side, fp32 accumulate in TMEM).
//
// The key cache already is NVFP4 ("NVFP4 attention cache on W4A4 Qwen3-8B"
// (rstation.ai), setup: KV cache in NVFP4), so the keys go to the tensor
// cores as stored: their codes are only re-laid out in shared memory and
// their block scales copied to TMEM; no key is dequantised.  The query --
// smoothed (observation 2), rotated when the cache is -- is quantised to
// NVFP4 on the fly ("OSFP4" (paperlayer.ai summary), Problem bullet, sec. 1
// and sec. D.1: absmax of a 16-block to 6, E4M3 block scale), under an FP32
// scale per row, g_q = amax(row) / 2688, taken the way the cache's static
// tensor scales are.  Every step of that quantiser is one IEEE fp32 rounding
// in the cache quantiser's order, so the query codes are those of the
// reference quantiser bit for bit.  Score (log2 units) =
// (Q.K on codes and block scales) * g_q * g_K * log2(e) / sqrt(128).
// P.V stays on fp16 operands (kind::f16), the values dequantised as in the
// fp16 prefill.
//
// One CTA: one layer, one sequence, one kv head, two tiles of 32 query
// tokens x G heads (128 MMA rows each).  Per 64-token key block:
//   copy warp: bulk-copies the 4 packed page tiles into a staging ring.
//   dequant warps (2): key codes are copied into the unswizzled K-major FP4
//     layout the MMA reads (8-row x 16-byte core matrices) and key scales
//     into the 128-row scale layout (row r's 4 scales of a 64-element K step
//     at byte (r % 32) * 16 + (r / 32) * 4); values are dequantised to fp16.
//   MMA warp: tcgen05.cp of the key scales into TMEM, then per tile two
//     block-scaled MMAs (M=128, N=64, K=64) into the tile's score columns;
//     O += P V (M=128, N=128, K=16 steps) with P read from TMEM.
//   softmax warpgroups: as in the fp16 prefill; the score buffer is single
//     (freed as soon as the scores are in registers), P has its own columns.
// TMEM: O_A, O_B [0, 256); S_A, S_B [256, 384); P_A, P_B [384, 448);
// query scales [448, 464); key scales (two buffers) [464, 480).
// Every hand-off is an mbarrier with a bounded wait; a wait that runs out
// sets KVQ_DEV_TIMEOUT, the CTA writes zeros and frees its TMEM.
#include "kvq_attn.cuh"
#include "kvq_common.cuh"
#include "kvq_internal.h"
#include "kvq_packed.cuh"
#include "kvq_sync.cuh"
#include "kvq_tcgen05.cuh"

namespace kvq {
namespace {

constexpr int kRows = 128;          // MMA M of one tile: 4 heads x 32 query tokens
constexpr int kQTok = 32;           // query tokens per tile
constexpr int kTiles = 2;           // query tiles per CTA
constexpr int kBlkTok = 64;         // key tokens per block (4 pages)
constexpr int kStageN = 6;          // packed-page staging stages
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 256, kColP = 384, kColSFA = 448, kColSFB = 464;
// The softmax reference moves only when a block's max passes it by more than
// kRescaleThreshold (log2 units); the probabilities are scaled by
// 2^kPScaleLog2, so they stay below 2^(12 + 3) = 2^15, inside fp16, and a
// weight 2^-17 of the row's largest is still a normal fp16 number.
constexpr float kRescaleThreshold = 12.0f;
constexpr float kPScaleLog2 = 3.0f;
constexpr int kPidCap = 1024;       // page ids held in shared memory (keys up to 16384 tokens)

// shared memory map (offsets from a 1024-aligned base)
constexpr int kVBytes = kBlkTok * kD * 2;         // 16 KB fp16 value tile (128B-swizzled)
constexpr int kQBytes = kRows * kD / 2;           // 8 KB FP4 query tile
constexpr int kKBytes = kBlkTok * kD / 2;         // 4 KB FP4 key tile
constexpr int kSFBytes = 512;                     // scales of 128 rows x one K step (4 blocks)
constexpr int kStageBytes = 4 * kTile;
constexpr int kOffV = 0;                                  // 2 buffers
constexpr int kOffQ = kOffV + 2 * kVBytes;                // [tile]
constexpr int kOffK = kOffQ + kTiles * kQBytes;           // 2 buffers
constexpr int kOffSFA = kOffK + 2 * kKBytes;              // [tile][K step]
constexpr int kOffSFB = kOffSFA + kTiles * 2 * kSFBytes;  // [buffer][K step]
constexpr int kOffStage = kOffSFB + 2 * 2 * kSFBytes;     // kStageN stages
constexpr int kSmemBytes = kOffStage + kStageN * kStageBytes;
// two CTAs (with the 1 KB each reserves) would not fit in the SM's 228 KB:
// one CTA, which holds all 512 TMEM columns, runs per SM
constexpr int kSmemAlloc = kSmemBytes + 1024;
static_assert(2 * (kSmemAlloc + 1024) > 228 * 1024 && kSmemAlloc <= 227 * 1024, "one CTA per SM");

// warps 8, 9 re-lay the keys and dequantise the values; warp 10 issues the
// bulk copies (a copy takes the issuing thread hundreds of cycles, which a
// warp that also dequantises would put on the critical path every block)
enum { kWarpsSoftmax = 4 * kTiles, kWarpsDequant = 2 };
constexpr int kDequantWarp0 = kWarpsSoftmax;                   // warps 8, 9
constexpr int kCopyWarp = kDequantWarp0 + kWarpsDequant;       // warp 10
constexpr int kMmaWarp = kCopyWarp + 1;                        // warp 11
constexpr int kThreads = 32 * (kMmaWarp + 1);

// byte offset of 16-byte chunk c (32 FP4 elements along K) of row `row` in an
// unswizzled K-major FP4 tile of 64-byte rows: core matrices of 8 rows along
// K 128 bytes apart, 8-row groups 512 bytes apart
__device__ __forceinline__ uint32_t fp4_off(int row, int c) {
    return (uint32_t)((row >> 3) * 512 + c * 128 + (row & 7) * 16);
}
// byte offset of row `row`'s 4 scales in a 128-row scale block
__device__ __forceinline__ uint32_t sf_off(int row) { return (uint32_t)((row & 31) * 16 + (row >> 5) * 4); }

struct Fp4Bars {
    uint64_t q_ready;                 // query tiles and scales written (count 8)
    uint64_t stage_full[kStageN];     // packed pages landed (tx bytes)
    uint64_t stage_empty[kStageN];    // dequant warps read the stage (count 2)
    uint64_t k_full[2];               // K tile + scales of block j written (count 2)
    uint64_t v_full[2];               // V tile j written (count 2)
    uint64_t k_free[2];               // Q.K(j) of both tiles done (commit)
    uint64_t s_full[kTiles];          // Q.K(tile, j) done (commit)
    uint64_t s_free[kTiles];          // scores of (tile, j) loaded (count 4)
    uint64_t p_full[kTiles];          // P(tile, j) stored, O rescaled (count 4)
    uint64_t pv_done[kTiles][2];      // P.V(tile, j) done (commit), by j & 1
    uint64_t drain;
    uint32_t tmem_base;
    int flags;                        // 1: a bounded wait ran out
    int issued;
};

// grid (query-tile pairs, batch * Hkv, nlayers), block 384
template <typename TQ, typename TO>
__global__ void __launch_bounds__(kThreads, 1) prefill_fp4_kernel(AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ Fp4Bars bars;
    __shared__ int32_t s_pid[kPidCap];   // the sequence's page ids, read once for every copy

    const int pair = blockIdx.x, b = blockIdx.y / a.Hkv, h = blockIdx.y % a.Hkv, li = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int len = __ldg(a.seq_lens + b);
    const int qs = __ldg(a.q_start + b);
    const int q0 = pair * (kTiles * kQTok);
    const int qn = min(kTiles * kQTok, a.q_len - q0);
    const bool bad_len = len < 0 || len > a.max_pages * kPage;
    int kv_end = bad_len ? 0 : min(len, qs + q0 + qn);
    if (kv_end < 0) kv_end = 0;
    const int nb = (kv_end + kBlkTok - 1) / kBlkTok;
    const int npg = (kv_end + kPage - 1) / kPage;
    const int32_t* pt = a.page_table + (size_t)b * a.max_pages;
    const uint8_t* layer_base = a.cache + (size_t)li * a.layer_stride;

    if (threadIdx.x == 0) {
        bars.flags = 0;
        bars.issued = 0;
        mbar_init(&bars.q_ready, kWarpsSoftmax);
        for (int i = 0; i < kStageN; ++i) {
            mbar_init(&bars.stage_full[i], 1);
            mbar_init(&bars.stage_empty[i], kWarpsDequant);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.k_full[i], kWarpsDequant);
            mbar_init(&bars.v_full[i], kWarpsDequant);
            mbar_init(&bars.k_free[i], 1);
            for (int t = 0; t < kTiles; ++t) mbar_init(&bars.pv_done[t][i], 1);
        }
        for (int t = 0; t < kTiles; ++t) {
            mbar_init(&bars.s_full[t], 1);
            mbar_init(&bars.s_free[t], 4);
            mbar_init(&bars.p_full[t], 4);
        }
        mbar_init(&bars.drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // the key-scale blocks: rows 64..127 are never written (N = 64); zero them
    for (int i = threadIdx.x; i < 2 * 2 * kSFBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(smem + kOffSFB)[i] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    int badp = 0;
    for (int i = threadIdx.x; i < npg; i += blockDim.x) {
        const int pg = __ldg(pt + i);
        badp |= (pg < 0 || pg >= a.num_pages);
        if (i < kPidCap) s_pid[i] = pg;
    }
    badp = __syncthreads_or(badp);
    if (threadIdx.x == 0) {
        if (bad_len && pair == 0 && h == 0) set_status(a.status, KVQ_DEV_BAD_LEN);
        if (badp) set_status(a.status, KVQ_DEV_BAD_PAGE);
    }
    const bool poison = bad_len || badp;

    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&bars.tmem_base)),
                     "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    auto tO = [&](int t) { return tmem + 128u * t; };
    auto tS = [&](int t) { return tmem + kColS + 64u * t; };
    auto tP = [&](int t) { return tmem + kColP + 32u * t; };

    float m_run = -INFINITY, l_run = 0.0f, isig = 1.0f;

    if (!poison && nb > 0) {
        if (warp < kWarpsSoftmax) {
            // ------------------------------------------------------ softmax warpgroups
            const int t = warp >> 2;
            const int r = threadIdx.x & 127;           // TMEM lane = MMA row
            const int head = r >> 5, tok = r & 31;     // row = head * 32 + token
            const int qi = q0 + t * kQTok + tok;
            const bool row_ok = head < a.G && (t * kQTok + tok) < qn;
            const int qpos = qs + qi;
            // query prologue: y = q * s (then H y / sqrt(128)), NVFP4 with an
            // FP32 scale per row; every step one IEEE fp32 rounding
            {
                float x[kD];
                if (row_ok) {
                    const TQ* src = reinterpret_cast<const TQ*>(a.q) +
                                    ((((size_t)li * a.batch + b) * a.q_len + qi) * a.Hq + h * a.G + head) * kD;
                    load_row128<TQ>(src, x);
                    if (!a.qpre) {   // (the KLT cache's queries arrive smoothed and rotated)
                        const float* srow = a.smooth + ((size_t)li * a.Hkv + h) * kD;
#pragma unroll
                        for (int i = 0; i < kD; ++i) x[i] = __fmul_rn(x[i], __ldg(srow + i));
                        if (a.hadamard) {
#pragma unroll
                            for (int hh = 1; hh < kD; hh <<= 1)
#pragma unroll
                                for (int j = 0; j < kD; ++j)
                                    if ((j & hh) == 0) {
                                        const float u = x[j], v = x[j + hh];
                                        x[j] = __fadd_rn(u, v);
                                        x[j + hh] = __fsub_rn(u, v);
                                    }
#pragma unroll
                            for (int i = 0; i < kD; ++i) x[i] = __fmul_rn(x[i], kInvSqrt128);
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < kD; ++i) x[i] = 0.0f;
                }
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < kD; ++i) amax = fmaxf(amax, fabsf(x[i]));
                const float g = amax > 0.0f ? __fdiv_rn(amax, kTensorRange) : 1.0f;
                const float enc = __frcp_rn(__fmul_rn(6.0f, g));
                isig = g * (__ldg(a.gk + li) * kLog2e * kInvSqrt128);
                uint8_t* qt = smem + kOffQ + t * kQBytes;
                uint32_t sfw[2] = {0u, 0u};
#pragma unroll
                for (int blk = 0; blk < kD / kBlk; ++blk) {
                    const float* y = x + blk * kBlk;
                    float am = 0.0f;
#pragma unroll
                    for (int i = 0; i < kBlk; ++i) am = fmaxf(am, fabsf(y[i]));
                    const uint32_t sc = e4m3_rn(__fmul_rn(am, enc));
                    const float d = __fmul_rn(e4m3_to_f32(sc), g);
                    const float rr = d == 0.0f ? 0.0f : __frcp_rn(d);
                    float2 z[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) z[k] = make_float2(__fmul_rn(y[2 * k], rr), __fmul_rn(y[2 * k + 1], rr));
                    const uint32_t w[2] = {e2m1x8_rn(z[0], z[1], z[2], z[3]), e2m1x8_rn(z[4], z[5], z[6], z[7])};
                    // 16 codes = 8 bytes at byte 8 * blk of the row
                    *reinterpret_cast<uint2*>(qt + fp4_off(r, blk >> 1) + (blk & 1) * 8) = make_uint2(w[0], w[1]);
                    sfw[blk >> 2] |= sc << (8 * (blk & 3));
                }
#pragma unroll
                for (int s = 0; s < 2; ++s)
                    *reinterpret_cast<uint32_t*>(smem + kOffSFA + (2 * t + s) * kSFBytes + sf_off(r)) = sfw[s];
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.q_ready);
            }
            const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
            for (int j = 0; j < nb; ++j) {
                if (!mbar_wait_warp(&bars.s_full[t], j & 1)) { atomicOr(&bars.flags, 1); break; }
                tc_fence_after();
                float s[kBlkTok];
                tmem_ld32(tS(t) + lane_addr, s);
                tmem_ld32(tS(t) + 32 + lane_addr, s + 32);
                // the score columns are free for Q.K(j + 1) once every lane has them
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.s_free[t]);
                const int kp0 = j * kBlkTok;
                if (kp0 + kBlkTok - 1 > qpos || kp0 + kBlkTok > kv_end) {
#pragma unroll
                    for (int c = 0; c < kBlkTok; ++c) {
                        const int kp = kp0 + c;
                        s[c] = (kp <= qpos && kp < kv_end) ? s[c] : -INFINITY;
                    }
                }
                float m21[22];
#pragma unroll
                for (int c = 0; c < 21; ++c) m21[c] = fmax3(s[3 * c], s[3 * c + 1], s[3 * c + 2]);
                m21[21] = s[63];
                float m8[8];
#pragma unroll
                for (int c = 0; c < 7; ++c) m8[c] = fmax3(m21[3 * c], m21[3 * c + 1], m21[3 * c + 2]);
                m8[7] = m21[21];
                float bm = fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], fmax3(m8[5], m8[6], m8[7])));
                bm *= isig;
                // P.V(j - 1) must be done before O is rescaled (rare) or P(j) is
                // stored over P(j - 1): waited for as late as possible
                bool pv_ok = j == 0;
                auto wait_pv = [&]() {
                    if (!pv_ok) {
                        pv_ok = mbar_wait_warp(&bars.pv_done[t][(j - 1) & 1], ((j - 1) >> 1) & 1);
                        tc_fence_after();
                    }
                    return pv_ok;
                };
                const bool grow = bm > m_run + kRescaleThreshold || (m_run == -INFINITY && bm > -INFINITY);
                const bool any_grow = __any_sync(0xFFFFFFFFu, grow);
                float al = 1.0f;
                if (any_grow) {
                    const float mn = grow ? bm : m_run;
                    al = (m_run == -INFINITY) ? 0.0f : ex2(m_run - mn);
                    l_run *= al;
                    m_run = mn;
                }
                const float2 sc2 = make_float2(isig, isig);
                const float2 nm2 = make_float2(kPScaleLog2 - m_run, kPScaleLog2 - m_run);
                float2 lsum[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                                  make_float2(0.0f, 0.0f)};
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float2 x = ffma2(make_float2(s[2 * c], s[2 * c + 1]), sc2, nm2);
                    float2 pp;
                    pp.x = ex2(x.x);
                    pp.y = ex2(x.y);
                    lsum[c & 3] = fadd2(lsum[c & 3], pp);
                    pk[c] = h2(pp.x, pp.y);
                }
                if (!wait_pv()) { atomicOr(&bars.flags, 1); break; }
                tmem_st16u(tP(t) + lane_addr, pk);
                tmem_st16u(tP(t) + 16 + lane_addr, pk + 16);
                const float2 l2 = fadd2(fadd2(lsum[0], lsum[1]), fadd2(lsum[2], lsum[3]));
                l_run += l2.x + l2.y;
                if (any_grow && j > 0) {
                    // P.V(j - 1) is done (waited above): bring O to the new
                    // reference before P.V(j) adds to it, in one TMEM round trip
                    float o[kD];
                    tmem_ld128(tO(t) + lane_addr, o);
#pragma unroll
                    for (int i = 0; i < kD; i += 2) {
                        const float2 v = fmul2(make_float2(o[i], o[i + 1]), make_float2(al, al));
                        o[i] = v.x;
                        o[i + 1] = v.y;
                    }
                    tmem_st128(tO(t) + lane_addr, o);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.p_full[t]);
            }
        } else if (warp == kCopyWarp) {
            // ------------------------------------------------------ copy warp
            // block j's 4 page tiles into stage j % kStageN, once the dequant
            // warps have read block j - kStageN out of it
            if (lane == 0) {
                int issued = 0;
                for (; issued < nb; ++issued) {
                    const int st = issued % kStageN;
                    if (issued >= kStageN &&
                        !mbar_wait(&bars.stage_empty[st], ((issued - kStageN) / kStageN) & 1)) {
                        atomicOr(&bars.flags, 1);
                        break;
                    }
                    const int p_lo = issued * 4, n_p = min(npg, p_lo + 4) - p_lo;
                    mbar_arrive_expect_tx(&bars.stage_full[st], (uint32_t)n_p * kTile);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (k < n_p) {
                            const int p = p_lo + k;
                            const int pg = p < kPidCap ? s_pid[p] : __ldg(pt + p);
                            bulk_g2s(smem + kOffStage + st * kStageBytes + k * kTile,
                                     layer_base + ((size_t)pg * a.Hkv + h) * kTile, kTile, &bars.stage_full[st]);
                        }
                }
                bars.issued = issued;
            }
        } else if (warp < kMmaWarp) {
            // ------------------------------------------------------ dequant warps
            const int dt = threadIdx.x - 32 * kDequantWarp0;   // 0..63
            // items (token, half of head_dim): 128 per block over 64 threads
            constexpr int kItems = 2 * kBlkTok, kDqThreads = 32 * kWarpsDequant;
            constexpr int kPer = (kItems + kDqThreads - 1) / kDqThreads;
            struct Staged {
                uint4 kc[kPer][2], vc[kPer][2];
                uint32_t ks[kPer], vs[kPer][4];
            };
            auto load_block = [&](int j, Staged& S) -> bool {
                const int st = j % kStageN;
                if (!mbar_wait_warp(&bars.stage_full[st], (j / kStageN) & 1)) return false;
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    const int it = dt + e * kDqThreads;
                    const int tkn = it >> 1, half = it & 1;
                    S.kc[e][0] = S.kc[e][1] = S.vc[e][0] = S.vc[e][1] = make_uint4(0, 0, 0, 0);
                    S.ks[e] = 0;
                    S.vs[e][0] = S.vs[e][1] = S.vs[e][2] = S.vs[e][3] = 0;
                    if (it < kItems && j * kBlkTok + tkn < kv_end) {
                        const int trow = tkn & 15;
                        const uint8_t* T = smem + kOffStage + st * kStageBytes + (tkn >> 4) * kTile;
                        S.kc[e][0] = *reinterpret_cast<const uint4*>(T + kKCodes + trow * 64 + half * 32);
                        S.kc[e][1] = *reinterpret_cast<const uint4*>(T + kKCodes + trow * 64 + half * 32 + 16);
                        S.ks[e] = *reinterpret_cast<const uint32_t*>(T + kKScales + trow * 8 + half * 4);
                        S.vc[e][0] = *reinterpret_cast<const uint4*>(T + kVCodes + trow * 64 + half * 32);
                        S.vc[e][1] = *reinterpret_cast<const uint4*>(T + kVCodes + trow * 64 + half * 32 + 16);
#pragma unroll
                        for (int q = 0; q < 4; ++q) S.vs[e][q] = T[kVScales + (half * 4 + q) * 16 + trow];
                    }
                }
                __syncwarp();
                if ((dt & 31) == 0) mbar_arrive(&bars.stage_empty[st]);
                return true;
            };
            // key codes and scales of block j into buffer j & 1, free once
            // both tiles' Q.K(j - 2) are done; tokens past the sequence are
            // zero codes with zero scales
            auto store_k = [&](int j, const Staged& S) -> bool {
                const int buf = j & 1;
                if (j >= 2 && !mbar_wait_warp(&bars.k_free[buf], ((j - 2) >> 1) & 1)) return false;
                uint8_t* Kt = smem + kOffK + buf * kKBytes;
                uint8_t* SFt = smem + kOffSFB + buf * 2 * kSFBytes;
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    const int it = dt + e * kDqThreads;
                    if (it >= kItems) break;
                    const int tkn = it >> 1, half = it & 1;   // half = K step (dims 64 half .. +63)
                    *reinterpret_cast<uint4*>(Kt + fp4_off(tkn, 2 * half)) = S.kc[e][0];
                    *reinterpret_cast<uint4*>(Kt + fp4_off(tkn, 2 * half + 1)) = S.kc[e][1];
                    *reinterpret_cast<uint32_t*>(SFt + half * kSFBytes + sf_off(tkn)) = S.ks[e];
                }
                fence_async_smem();
                __syncwarp();
                if ((dt & 31) == 0) mbar_arrive(&bars.k_full[buf]);
                return true;
            };
            // values of block j into V buffer j & 1 (fp16, MN-major, 128-byte
            // swizzle), free once both tiles' P.V(j - 2) are done
            auto store_v = [&](int j, const Staged& S) -> bool {
                const int buf = j & 1;
                if (j >= 2 && !mbar_wait_warp(&bars.pv_done[kTiles - 1][buf], ((j - 2) >> 1) & 1)) return false;
                uint8_t* Vt = smem + kOffV + buf * kVBytes;
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    const int it = dt + e * kDqThreads;
                    if (it >= kItems) break;
                    const int tkn = it >> 1, half = it & 1;
                    const bool valid = j * kBlkTok + tkn < kv_end;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4& c1 = S.vc[e][q >> 1];
                        const uint32_t vw0 = (q & 1) ? c1.z : c1.x, vw1 = (q & 1) ? c1.w : c1.y;
                        uint32_t va[4], vb[4];
                        e2m1x8(vw0, va);
                        e2m1x8(vw1, vb);
                        const uint32_t vsh = e4m3x2_to_f16x2(S.vs[e][q]) & 0xFFFFu;
                        const uint32_t sc = valid ? (vsh | (vsh << 16)) : 0u;
                        const int dim_chunk = half * 8 + 2 * q;
                        const int plane = dim_chunk >> 3, ch = dim_chunk & 7;
                        sts128(Vt + plane * (kBlkTok * 128) + sw128(tkn, ch), hmul2u(va[0], sc), hmul2u(va[1], sc),
                               hmul2u(va[2], sc), hmul2u(va[3], sc));
                        sts128(Vt + plane * (kBlkTok * 128) + sw128(tkn, ch + 1), hmul2u(vb[0], sc),
                               hmul2u(vb[1], sc), hmul2u(vb[2], sc), hmul2u(vb[3], sc));
                    }
                }
                fence_async_smem();
                __syncwarp();
                if ((dt & 31) == 0) mbar_arrive(&bars.v_full[buf]);
                return true;
            };
            // the keys of block j + 1 go out before the values of block j
            // (Q.K(j + 1) is issued before P.V(j))
            Staged cur, nxt;
            bool dq_ok = nb == 0 || (load_block(0, cur) && store_k(0, cur));
            for (int j = 0; dq_ok && j < nb; ++j) {
                if (j + 1 < nb) dq_ok = load_block(j + 1, nxt) && store_k(j + 1, nxt);
                dq_ok = dq_ok && store_v(j, cur);
                cur = nxt;
            }
            if (!dq_ok) atomicOr(&bars.flags, 1);
        } else if (lane == 0) {
            // ------------------------------------------------------ MMA issuer
            constexpr uint32_t qk = fp4_idesc(kRows, kBlkTok);
            const uint32_t pv = f16_idesc(kRows, kD, true);
            // Descriptors are built once per operand tile; a tile, buffer or K
            // step only moves the 14-bit start-address field (16-byte units)
            // by a constant, which never carries out of the field for
            // shared-memory addresses.
            const uint64_t qd0 = nosw_desc(smem_u32(smem + kOffQ), 128, 512);
            const uint64_t kd0 = nosw_desc(smem_u32(smem + kOffK), 128, 512);
            const uint64_t sfa0 = nosw_desc(smem_u32(smem + kOffSFA), 128, 128);
            const uint64_t sfb0 = nosw_desc(smem_u32(smem + kOffSFB), 128, 128);
            const uint64_t vd0 = sw128_desc(smem_u32(smem + kOffV), kBlkTok * 128, 1024);
            auto qd = [&](int t, int s) { return qd0 + (uint64_t)((t * kQBytes + 256 * s) >> 4); };
            auto kd = [&](int u, int s) { return kd0 + (uint64_t)((u * kKBytes + 256 * s) >> 4); };
            auto sfa = [&](int t, int s) { return sfa0 + (uint64_t)(((2 * t + s) * kSFBytes) >> 4); };
            auto sfb = [&](int u, int s) { return sfb0 + (uint64_t)(((2 * u + s) * kSFBytes) >> 4); };
            auto vd = [&](int u) { return vd0 + (uint64_t)((u * kVBytes) >> 4); };
            // O(t) += P(t, jp) V(jp); V buffer jp & 1 is waited for by tile 0
            auto issue_pv = [&](int t, int jp) -> bool {
                const int pb = jp & 1;
                if (t == 0 && !mbar_wait(&bars.v_full[pb], (jp >> 1) & 1)) return false;
                if (!mbar_wait(&bars.p_full[t], jp & 1)) return false;
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16_ta(tO(t), tP(t) + 8 * s, vd(pb) + (uint64_t)((s * 2048) >> 4), pv, (jp | s) ? 1u : 0u);
                mma_commit(&bars.pv_done[t][pb]);
                return true;
            };
            bool ok = mbar_wait(&bars.q_ready, 0);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int t = 0; t < kTiles; ++t)
#pragma unroll
                    for (int s = 0; s < 2; ++s) tmem_cp_scales(tmem + kColSFA + 8 * t + 4 * s, sfa(t, s));
            }
            for (int j = 0; ok && j <= nb; ++j) {
                if (j < nb) {
                    const int buf = j & 1;
                    if (!mbar_wait(&bars.k_full[buf], (j >> 1) & 1)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 2; ++s) tmem_cp_scales(tmem + kColSFB + 8 * buf + 4 * s, sfb(buf, s));
                    // tile by tile: Q.K(j) then P.V(j - 1) of tile A, then of tile
                    // B, so that one tile's P.V is not held behind the other
                    // tile's scores
                    for (int t = 0; t < kTiles; ++t) {
                        // the tile's scores of block j - 1 must be in registers
                        if (j >= 1 && !mbar_wait(&bars.s_free[t], (j - 1) & 1)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int s = 0; s < 2; ++s)
                            mma_fp4(tS(t), qd(t, s), kd(buf, s), qk, tmem + kColSFA + 8 * t + 4 * s,
                                    tmem + kColSFB + 8 * buf + 4 * s, (uint32_t)s);
                        mma_commit(&bars.s_full[t]);
                        if (t == kTiles - 1) mma_commit(&bars.k_free[buf]);
                        if (j >= 1 && !issue_pv(t, j - 1)) { ok = false; break; }
                    }
                    if (!ok) break;
                } else {
                    // after the last block: its P.V
                    for (int t = 0; t < kTiles; ++t)
                        if (!issue_pv(t, j - 1)) { ok = false; break; }
                }
            }
            if (!ok) atomicOr(&bars.flags, 1);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool timed_out = bars.flags != 0;
    if (timed_out && threadIdx.x == 32 * kDequantWarp0) {
        const int issued = bars.issued;
        for (int j = max(0, issued - kStageN); j < issued; ++j)
            (void)mbar_wait(&bars.stage_full[j % kStageN], (j / kStageN) & 1);
        set_status(a.status, KVQ_DEV_TIMEOUT);
    }
    if (timed_out && threadIdx.x == 32 * kMmaWarp) {
        mma_commit(&bars.drain);
        (void)mbar_wait(&bars.drain, 0);
    }

    // ---------------------------------------------------------------- epilogue
    const bool dead = poison || timed_out || nb == 0;
    if (warp < kWarpsSoftmax) {
        const int t = warp >> 2;
        const int r = threadIdx.x & 127;
        const int head = r >> 5, tok = r & 31;
        const int qi = q0 + t * kQTok + tok;
        float res[kD];
        if (!dead) {
            const int jl = nb - 1;
            const bool ok = mbar_wait_warp(&bars.pv_done[t][jl & 1], (jl >> 1) & 1);
            tc_fence_after();
            const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
            const float sc = (ok && l_run > 0.0f) ? __ldg(a.gv + li) / l_run : 0.0f;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float o[32];
                tmem_ld32(tO(t) + cc * 32 + lane_addr, o);
#pragma unroll
                for (int i = 0; i < 32; ++i) res[cc * 32 + i] = ok ? o[i] * sc : 0.0f;
            }
            if (!ok && lane == 0) set_status(a.status, KVQ_DEV_TIMEOUT);
        } else {
#pragma unroll
            for (int i = 0; i < kD; ++i) res[i] = 0.0f;
        }
        if (head < a.G && (t * kQTok + tok) < qn) {
            TO* dst = reinterpret_cast<TO*>(a.out) +
                      ((((size_t)li * a.batch + b) * a.q_len + qi) * a.Hq + h * a.G + head) * kD;
            if constexpr (sizeof(TO) == 4) {
#pragma unroll
                for (int i = 0; i < kD / 4; ++i)
                    reinterpret_cast<float4*>(dst)[i] = make_float4(res[4 * i], res[4 * i + 1], res[4 * i + 2],
                                                                    res[4 * i + 3]);
            } else {
#pragma unroll
                for (int i = 0; i < kD / 8; ++i) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 t2 = __floats2bfloat162_rn(res[8 * i + 2 * e], res[8 * i + 2 * e + 1]);
                        w[e] = *reinterpret_cast<uint32_t*>(&t2);
                    }
                    reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

}  // namespace

cudaError_t launch_prefill_fp4(const AttnArgs& a, int nlayers, bool q_bf16, bool out_bf16, cudaStream_t st) {
    const dim3 grid((a.q_len + kTiles * kQTok - 1) / (kTiles * kQTok), a.batch * a.Hkv, nlayers);
    cudaError_t e;
#define KVQ_LAUNCH(TQ, TO)                                                                                  \
    e = cudaFuncSetAttribute(prefill_fp4_kernel<TQ, TO>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc); \
    if (e != cudaSuccess) return e;                                                                         \
    prefill_fp4_kernel<TQ, TO><<<grid, kThreads, kSmemAlloc, st>>>(a);
    if (q_bf16 && out_bf16) { KVQ_LAUNCH(__nv_bfloat16, __nv_bfloat16) }
    else if (q_bf16) { KVQ_LAUNCH(__nv_bfloat16, float) }
    else if (out_bf16) { KVQ_LAUNCH(float, __nv_bfloat16) }
    else { KVQ_LAUNCH(float, float) }
#undef KVQ_LAUNCH
    return cudaGetLastError();
}

}  // namespace kvq
