// kvq_prefill_tc.cu -- chunked causal prefill over the packed NVFP4 cache on
// the 5th-generation tensor cores (tcgen05.mma, accumulators in TMEM).
//
// The chunk's own keys and values are appended to the cache first; query i
// of sequence b (absolute position q_start + i) then attends cached
// positions j <= q_start + i ("chunked causal prefill", with the smoothing
// and rotation folded into the query as in "NVFP4 attention cache on W4A4
// Qwen3-8B" (rstation.ai), observation 2).
//
// One CTA: one layer, one sequence, one kv head, and two tiles (A, B) of 32
// query tokens each.  A tile's 128 MMA rows are the G <= 4 query heads of
// the kv head times its 32 tokens (row = head * 32 + token), so each
// dequantised key/value block feeds 8 query heads x 32 tokens.  Keys are
// taken in blocks of 128 tokens (8 pages), so every MMA has N = 128: at that
// shape an MMA's shared-memory operand reads (A and B, 4 KB each per 16-deep
// step) keep pace with its math, where N = 64 would leave the tensor pipe
// waiting on shared memory.  Per block:
//   dequant warps (3): read the block's packed page tiles straight from
//     global memory (one block ahead, in registers), dequantise to fp16
//     (E2M1 x E4M3 is exact in fp16) into a K tile (K-major, two buffers)
//     and a V tile (MN-major, one buffer), both in the 128-byte-swizzled
//     canonical layouts the MMA reads; rows past the sequence are zeros.
//   MMA warp (1 elected thread): per tile, S = Q_hi K^T + Q_lo K^T (M = 128,
//     N = 128, K = 16 steps; the query is split into fp16 hi + lo parts so
//     its rounding does not reach the scores) into the tile's score columns;
//     then O += P V (M = 128, N = 128) with P read from TMEM.  Order per
//     block: QK_A, QK_B, PV_A, PV_B; a tile's next QK is issued only after
//     its previous PV has completed (P lives in the score columns).
//   softmax warpgroups (one per tile; a thread owns one TMEM lane = row):
//     causal mask on diagonal blocks only, a lazy softmax reference (it
//     moves, and the output in TMEM is rescaled in one round trip, only when
//     a block's max passes it by more than 2^12), probabilities rounded once
//     to fp16 and stored back over the first 64 columns of the tile's score
//     buffer as the A operand of P V.
// TMEM: O_A, O_B (128 columns each), S_A, S_B (128 each) = 512 columns.
// Shared memory: the query tiles (hi, lo per tile) 128 KB, two K tiles 64 KB,
// one V tile 32 KB.
// All hand-offs are mbarriers with bounded waits; a wait that runs out sets
// KVQ_DEV_TIMEOUT, the CTA writes zeros and frees its TMEM.
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
constexpr int kTiles = 2;           // query tiles per CTA (A, B)
constexpr int kBlkTok = 128;        // key tokens per block (8 pages)
constexpr int kBlkPages = kBlkTok / kPage;
constexpr uint32_t kTmemCols = 512; // O_A, O_B [0,256), S_A [256,384), S_B [384,512)
// The softmax reference moves only when a block's max passes it by more than
// kRescaleThreshold (log2 units); the probabilities are scaled by
// 2^kPScaleLog2, so they stay below 2^(12 + 3) = 2^15, inside fp16, and a
// weight 2^-17 of the row's largest is still a normal fp16 number.
constexpr float kRescaleThreshold = 12.0f;
constexpr float kPScaleLog2 = 3.0f;
constexpr int kPidCap = 256;        // page ids held in shared memory (keys up to 4096 tokens)

// shared memory map (offsets from a 1024-aligned base)
constexpr int kQBytes = kRows * kD * 2;           // 32 KB per fp16 query tile part (hi or lo)
constexpr int kKBytes = kBlkTok * kD * 2;         // 32 KB per fp16 key tile
constexpr int kVBytes = kBlkTok * kD * 2;         // 32 KB fp16 value tile
constexpr int kPlane = kBlkTok * 128;             // one 64-dim plane of a K or V tile (128-byte rows)
constexpr int kOffQ = 0;                          // [tile][hi, lo]
constexpr int kOffK = kOffQ + kTiles * 2 * kQBytes;   // 2 buffers
constexpr int kOffV = kOffK + 2 * kKBytes;        // 1 buffer
constexpr int kSmemBytes = kOffV + kVBytes;
constexpr int kSmemAlloc = kSmemBytes + 1024;     // room to align the base

// warps 0-7 softmax (two warpgroups), 8-10 dequantise, 11 issues the MMAs
enum { kWarpsSoftmax = 4 * kTiles, kWarpsDequant = 3 };
constexpr int kDequantWarp0 = kWarpsSoftmax;
constexpr int kMmaWarp = kDequantWarp0 + kWarpsDequant;
constexpr int kThreads = 32 * (kMmaWarp + 1);
constexpr int kDqThreads = 32 * kWarpsDequant;
// dequant work items of a block: (token, half of head_dim)
constexpr int kItems = 2 * kBlkTok;
constexpr int kPer = (kItems + kDqThreads - 1) / kDqThreads;

struct PrefillBars {
    uint64_t q_ready;                 // both softmax warpgroups wrote their query tiles (count 8)
    uint64_t k_full[2];               // K tile j % 2 written (count 3)
    uint64_t k_free[2];               // QK of both tiles read K tile j % 2 (commit)
    uint64_t v_full;                  // V tile written (count 3)
    uint64_t v_free;                  // PV of both tiles read the V tile (commit)
    uint64_t s_full[kTiles];          // QK(tile, j) done (commit)
    uint64_t p_full[kTiles];          // P(tile, j) stored in TMEM, O rescaled (count 4)
    uint64_t pv_done[kTiles];         // PV(tile, j) done (commit)
    uint64_t drain;                   // last commit before TMEM is freed after a timeout
    uint32_t tmem_base;
    int flags;                        // 1: a bounded wait ran out
};

// ------------------------------------------------------------------ kernel
// grid (query-tile pairs, batch * Hkv, nlayers), block 384.
// KB: mixed cache (bf16 keys, untransformed: the key rows are copied into
// the key tile as they are, and Q.K runs on bf16 operands).
template <typename TQ, typename TO, bool KB>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ PrefillBars bars;
    __shared__ int32_t s_pid[kPidCap];   // the sequence's first page ids, read once

    constexpr int tile = KB ? kTileBf16K : kTile;           // bytes of one kv head of one page
    constexpr int vcodes = KB ? kBf16VCodes : kVCodes;
    constexpr int vscales = KB ? kBf16VScales : kVScales;

    const int pair = blockIdx.x, b = blockIdx.y / a.Hkv, h = blockIdx.y % a.Hkv, li = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int len = __ldg(a.seq_lens + b);
    const int qs = __ldg(a.q_start + b);
    const int q0 = pair * (kTiles * kQTok);
    const int qn = min(kTiles * kQTok, a.q_len - q0);        // query tokens of the pair
    const bool bad_len = len < 0 || len > a.max_pages * kPage;
    // keys needed by the pair: positions < min(len, q_start + q0 + qn)
    int kv_end = bad_len ? 0 : min(len, qs + q0 + qn);
    if (kv_end < 0) kv_end = 0;
    const int nb = (kv_end + kBlkTok - 1) / kBlkTok;          // 128-token blocks
    const int npg = (kv_end + kPage - 1) / kPage;             // pages touched
    const int32_t* pt = a.page_table + (size_t)b * a.max_pages;
    const uint8_t* layer_base = a.cache + (size_t)li * a.layer_stride;

    if (threadIdx.x == 0) {
        bars.flags = 0;
        mbar_init(&bars.q_ready, kWarpsSoftmax);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.k_full[i], kWarpsDequant);
            mbar_init(&bars.k_free[i], 1);
        }
        mbar_init(&bars.v_full, kWarpsDequant);
        mbar_init(&bars.v_free, 1);
        for (int t = 0; t < kTiles; ++t) {
            mbar_init(&bars.s_full[t], 1);
            mbar_init(&bars.p_full[t], 4);
            mbar_init(&bars.pv_done[t], 1);
        }
        mbar_init(&bars.drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
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

    // TMEM: one warp allocates all 512 columns for the CTA (one CTA per SM)
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&bars.tmem_base)),
                     "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    // per tile t: O at tmem + 128 t; S (and P over its first 64 columns) at tmem + 256 + 128 t
    auto tO = [&](int t) { return tmem + 128u * t; };
    auto tS = [&](int t) { return tmem + 256u + 128u * t; };

    // per-row state of the softmax warps, kept to the epilogue
    float m_run = -INFINITY, l_run = 0.0f, isig = 1.0f;

    if (!poison && nb > 0) {
        if (warp < kWarpsSoftmax) {
            // ------------------------------------------------------ softmax warpgroups
            const int t = warp >> 2;                   // tile of this warpgroup
            const int r = threadIdx.x & 127;           // TMEM lane = MMA row
            const int head = r >> 5, tok = r & 31;     // row = head * 32 + token
            const int qi = q0 + t * kQTok + tok;
            const bool row_ok = head < a.G && (t * kQTok + tok) < qn;
            const int qpos = qs + qi;                  // absolute position of this query
            // query prologue: q~ = q * s (+ rotation) * g_K log2(e) / sqrt(128),
            // per-row power-of-two normalisation, fp16 hi + lo tiles
            {
                float x[kD];
                if (row_ok) {
                    const TQ* src = reinterpret_cast<const TQ*>(a.q) +
                                    ((((size_t)li * a.batch + b) * a.q_len + qi) * a.Hq + h * a.G + head) * kD;
                    load_row128<TQ>(src, x);
                    float scale;
                    if constexpr (KB) {
                        scale = kLog2e * kInvSqrt128;     // bf16 keys: the query as given
                    } else {
                        if (!a.qpre) {   // (the KLT cache's queries arrive smoothed and rotated)
                            const float* srow = a.smooth + ((size_t)li * a.Hkv + h) * kD;
#pragma unroll
                            for (int i = 0; i < kD; ++i) x[i] *= __ldg(srow + i);
                        }
                        scale = __ldg(a.gk + li) * kLog2e * kInvSqrt128;
                    }
                    if (!KB && a.hadamard) {
#pragma unroll
                        for (int hh = 1; hh < kD; hh <<= 1)
#pragma unroll
                            for (int j = 0; j < kD; ++j)
                                if ((j & hh) == 0) {
                                    const float u = x[j], v = x[j + hh];
                                    x[j] = u + v;
                                    x[j + hh] = u - v;
                                }
                        scale *= kInvSqrt128;
                    }
#pragma unroll
                    for (int i = 0; i < kD; ++i) x[i] *= scale;
                } else {
#pragma unroll
                    for (int i = 0; i < kD; ++i) x[i] = 0.0f;
                }
                float mx = 0.0f;
#pragma unroll
                for (int i = 0; i < kD; ++i) mx = fmaxf(mx, fabsf(x[i]));
                int ex = 0;
                if (mx > 0.0f) {
                    frexpf(mx, &ex);
                    ex = max(ex - 1, -100);
                }
                const float sig = ldexpf(1.0f, 14 - ex);
                isig = ldexpf(1.0f, ex - 14);
                uint8_t* qhi = smem + kOffQ + (2 * t) * kQBytes;
                uint8_t* qlo = qhi + kQBytes;
                // K-major 128B-swizzled tiles: dims 0..63 in atom plane 0, 64..127 in plane 1
#pragma unroll
                for (int ch = 0; ch < 16; ++ch) {
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float u = x[8 * ch + 2 * e] * sig, v = x[8 * ch + 2 * e + 1] * sig;
                        if constexpr (KB) {
                            hi[e] = bf2(u, v);
                            const float2 f = make_float2(__uint_as_float(hi[e] << 16),
                                                         __uint_as_float(hi[e] & 0xFFFF0000u));
                            lo[e] = bf2(u - f.x, v - f.y);
                        } else {
                            hi[e] = h2(u, v);
                            const float2 f = __half22float2(*reinterpret_cast<__half2*>(&hi[e]));
                            lo[e] = h2(u - f.x, v - f.y);
                        }
                    }
                    const uint32_t off = (ch >> 3) * (kRows * 128) + sw128(r, ch & 7);
                    sts128(qhi + off, hi[0], hi[1], hi[2], hi[3]);
                    sts128(qlo + off, lo[0], lo[1], lo[2], lo[3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.q_ready);
            }
            const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
            for (int j = 0; j < nb; ++j) {
                if (!mbar_wait_warp(&bars.s_full[t], j & 1)) { atomicOr(&bars.flags, 1); break; }
                tc_fence_after();
                float s[kBlkTok];
                tmem_ld128(tS(t) + lane_addr, s);
                const int kp0 = j * kBlkTok;
                // interior blocks (every key visible to this row) skip the mask
                if (kp0 + kBlkTok - 1 > qpos || kp0 + kBlkTok > kv_end) {
#pragma unroll
                    for (int c = 0; c < kBlkTok; ++c) {
                        const int kp = kp0 + c;
                        s[c] = (kp <= qpos && kp < kv_end) ? s[c] : -INFINITY;
                    }
                }
                // block max as a tree of three-input maxima
                float m43[43];
#pragma unroll
                for (int c = 0; c < 42; ++c) m43[c] = fmax3(s[3 * c], s[3 * c + 1], s[3 * c + 2]);
                m43[42] = fmaxf(s[126], s[127]);
                float m15[15];
#pragma unroll
                for (int c = 0; c < 14; ++c) m15[c] = fmax3(m43[3 * c], m43[3 * c + 1], m43[3 * c + 2]);
                m15[14] = m43[42];
                float m5[5];
#pragma unroll
                for (int c = 0; c < 5; ++c) m5[c] = fmax3(m15[3 * c], m15[3 * c + 1], m15[3 * c + 2]);
                float bm = fmaxf(fmax3(m5[0], m5[1], m5[2]), fmaxf(m5[3], m5[4]));
                bm *= isig;
                // lazy reference: it moves only when the block max passes it by
                // more than kRescaleThreshold (log2 units), so most blocks leave
                // O alone; the weights, at most 2^(threshold + kPScaleLog2) = 2^15,
                // stay inside fp16
                const bool grow = bm > m_run + kRescaleThreshold || (m_run == -INFINITY && bm > -INFINITY);
                const bool any_grow = __any_sync(0xFFFFFFFFu, grow);
                float al = 1.0f;
                if (any_grow) {
                    const float mn = grow ? bm : m_run;
                    al = (m_run == -INFINITY) ? 0.0f : ex2(m_run - mn);
                    l_run *= al;
                    m_run = mn;
                }
                // probabilities, fp16, stored over the first 64 columns of the score
                // buffer (every exponential on the MUFU unit: this loop is bound by
                // instruction issue, which a polynomial share would only add to)
                const float2 sc2 = make_float2(isig, isig);
                const float2 nm2 = make_float2(kPScaleLog2 - m_run, kPScaleLog2 - m_run);
                // four independent partial sums (the row sum is a long chain otherwise)
                float2 lsum[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                                  make_float2(0.0f, 0.0f)};
                uint32_t pk[kBlkTok / 2];
#pragma unroll
                for (int c = 0; c < kBlkTok / 2; ++c) {
                    const float2 x = ffma2(make_float2(s[2 * c], s[2 * c + 1]), sc2, nm2);
                    float2 pp;
                    pp.x = ex2(x.x);
                    pp.y = ex2(x.y);
                    lsum[c & 3] = fadd2(lsum[c & 3], pp);
                    pk[c] = h2(pp.x, pp.y);
                }
                tmem_st64u(tS(t) + lane_addr, pk);
                const float2 l2 = fadd2(fadd2(lsum[0], lsum[1]), fadd2(lsum[2], lsum[3]));
                l_run += l2.x + l2.y;
                if (any_grow && j > 0) {
                    // O holds P.V of the blocks before j, complete (QK(j) was issued
                    // only after PV(j - 1) finished): bring it to the new reference
                    // before PV(j) adds to it, in one TMEM round trip
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
        } else if (warp < kMmaWarp) {
            // ------------------------------------------------------ dequant warps
            // Each block's packed tiles are read straight from global memory
            // into registers one block ahead of their dequantisation.
            const int dt = threadIdx.x - 32 * kDequantWarp0;   // 0..95
            struct Staged {
                uint4 kc[kPer][2], vc[kPer][2];
                uint32_t ks[kPer], vs[kPer];
            };
            auto page_of = [&](int p) { return p < kPidCap ? s_pid[p] : __ldg(pt + p); };
            // global address of item `it`'s page tile for block j, or null past the keys
            auto tile_of = [&](int j, int it) -> const uint8_t* {
                const int tkn = it >> 1;
                if (it >= kItems || j * kBlkTok + tkn >= kv_end) return nullptr;
                const int pg = page_of(j * kBlkPages + (tkn >> 4));
                return layer_base + ((size_t)pg * a.Hkv + h) * tile;
            };
            auto load_k = [&](int j, Staged& S) {
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    const int it = dt + e * kDqThreads;
                    S.kc[e][0] = S.kc[e][1] = make_uint4(0, 0, 0, 0);
                    S.ks[e] = 0;
                    if constexpr (!KB) {
                        const uint8_t* T = tile_of(j, it);
                        if (T) {
                            const int trow = (it >> 1) & 15, half = it & 1;
                            S.kc[e][0] = __ldg(reinterpret_cast<const uint4*>(T + kKCodes + trow * 64 + half * 32));
                            S.kc[e][1] = __ldg(reinterpret_cast<const uint4*>(T + kKCodes + trow * 64 + half * 32 + 16));
                            S.ks[e] = __ldg(reinterpret_cast<const uint32_t*>(T + kKScales + trow * 8 + half * 4));
                        }
                    }
                }
            };
            auto load_v = [&](int j, Staged& S) {
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    const int it = dt + e * kDqThreads;
                    S.vc[e][0] = S.vc[e][1] = make_uint4(0, 0, 0, 0);
                    S.vs[e] = 0;
                    const uint8_t* T = tile_of(j, it);
                    if (T) {
                        const int trow = (it >> 1) & 15, half = it & 1;
                        S.vc[e][0] = __ldg(reinterpret_cast<const uint4*>(T + vcodes + trow * 64 + half * 32));
                        S.vc[e][1] = __ldg(reinterpret_cast<const uint4*>(T + vcodes + trow * 64 + half * 32 + 16));
                        uint32_t w = 0;
#pragma unroll
                        for (int q = 0; q < 4; ++q) w |= (uint32_t)__ldg(T + vscales + (half * 4 + q) * 16 + trow) << (8 * q);
                        S.vs[e] = w;
                    }
                }
            };
            // fp16 rows of one item into a 128B-swizzled tile: 4 blocks of 16 dims,
            // each 8 code bytes and one scale; a zero scale (past the keys) zeroes the row
            auto write_rows = [&](uint8_t* tl, int it, const uint4* c, uint32_t scales) {
                const int tkn = it >> 1, half = it & 1;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4& c0 = c[q >> 1];
                    const uint32_t w0 = (q & 1) ? c0.z : c0.x, w1 = (q & 1) ? c0.w : c0.y;
                    uint32_t ra[4], rb[4];
                    e2m1x8(w0, ra);
                    e2m1x8(w1, rb);
                    const uint32_t sh = e4m3x2_to_f16x2((scales >> (8 * q)) & 0xFFu) & 0xFFFFu;
                    const uint32_t sc = sh | (sh << 16);
                    // chunk index along head_dim: 2 chunks (8 dims each) per block
                    const int dim_chunk = half * 8 + 2 * q;          // 0..15
                    const int plane = dim_chunk >> 3, ch = dim_chunk & 7;
                    sts128(tl + plane * kPlane + sw128(tkn, ch), hmul2u(ra[0], sc), hmul2u(ra[1], sc),
                           hmul2u(ra[2], sc), hmul2u(ra[3], sc));
                    sts128(tl + plane * kPlane + sw128(tkn, ch + 1), hmul2u(rb[0], sc), hmul2u(rb[1], sc),
                           hmul2u(rb[2], sc), hmul2u(rb[3], sc));
                }
            };
            // keys of block j into K buffer j & 1, once both tiles' QK(j - 2) read it
            auto store_k = [&](int j, const Staged& S) -> bool {
                const int buf = j & 1;
                if (j >= 2 && !mbar_wait_warp(&bars.k_free[buf], ((j - 2) >> 1) & 1)) return false;
                uint8_t* Kt = smem + kOffK + buf * kKBytes;
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    const int it = dt + e * kDqThreads;
                    if (it < kItems) write_rows(Kt, it, S.kc[e], S.ks[e]);
                }
                fence_async_smem();
                __syncwarp();
                if ((dt & 31) == 0) mbar_arrive(&bars.k_full[buf]);
                return true;
            };
            // bf16 keys of block j: 16-byte asynchronous copies of each row straight
            // into its swizzled place (zeros past the keys); finish_k waits for them
            auto issue_k = [&](int j) -> bool {
                const int buf = j & 1;
                if (j >= 2 && !mbar_wait_warp(&bars.k_free[buf], ((j - 2) >> 1) & 1)) return false;
                uint8_t* Kt = smem + kOffK + buf * kKBytes;
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    const int it = dt + e * kDqThreads;
                    if (it >= kItems) break;
                    const int tkn = it >> 1, half = it & 1;
                    uint8_t* dst = Kt + half * kPlane;
                    const uint8_t* T = tile_of(j, it);
                    if (T) {
                        const uint8_t* src = T + (tkn & 15) * 256 + half * 128;
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) cp_async16(dst + sw128(tkn, ch), src + ch * 16);
                    } else {
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) sts128(dst + sw128(tkn, ch), 0u, 0u, 0u, 0u);
                    }
                }
                cp_async_commit();
                return true;
            };
            auto finish_k = [&](int j) {
                cp_async_wait_all();
                fence_async_smem();
                __syncwarp();
                if ((dt & 31) == 0) mbar_arrive(&bars.k_full[j & 1]);
            };
            // values of block j into the V tile, once both tiles' PV(j - 1) read it
            auto store_v = [&](int j, const Staged& S) -> bool {
                if (j >= 1 && !mbar_wait_warp(&bars.v_free, (j - 1) & 1)) return false;
                uint8_t* Vt = smem + kOffV;
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    const int it = dt + e * kDqThreads;
                    if (it < kItems) write_rows(Vt, it, S.vc[e], S.vs[e]);
                }
                fence_async_smem();
                __syncwarp();
                if ((dt & 31) == 0) mbar_arrive(&bars.v_full);
                return true;
            };
            // The keys of block j + 1 are wanted before the values of block j + 1
            // but after the values of block j (QK(j + 1) follows PV(j)).
            Staged S;
            bool dq_ok = true;
            load_k(0, S);
            load_v(0, S);
            if constexpr (KB) {
                dq_ok = issue_k(0);
                if (dq_ok) finish_k(0);
                for (int j = 0; dq_ok && j < nb; ++j) {
                    const bool more = j + 1 < nb;
                    if (more) dq_ok = issue_k(j + 1);
                    dq_ok = dq_ok && store_v(j, S);
                    if (more && dq_ok) {
                        load_v(j + 1, S);
                        finish_k(j + 1);
                    }
                }
                cp_async_wait_all();   // nothing in flight past this point
            } else {
                for (int j = 0; dq_ok && j < nb; ++j) {
                    dq_ok = store_k(j, S);
                    if (dq_ok && j + 1 < nb) load_k(j + 1, S);
                    dq_ok = dq_ok && store_v(j, S);
                    if (dq_ok && j + 1 < nb) load_v(j + 1, S);
                }
            }
            if (!dq_ok) atomicOr(&bars.flags, 1);
        } else if (lane == 0) {
            // ------------------------------------------------------ MMA issuer
            // Descriptors are built once; a k-step only advances the 14-bit
            // start-address field (16-byte units) by a constant, which never
            // carries out of the field for shared-memory addresses.
            // bf16 keys: both Q.K operands bf16 (A and B formats 1)
            const uint32_t qk = f16_idesc(kRows, kBlkTok, false) | (KB ? ((1u << 7) | (1u << 10)) : 0u);
            const uint32_t pv = f16_idesc(kRows, kD, true);
            uint64_t qd[kTiles][2], kd[2];
#pragma unroll
            for (int t = 0; t < kTiles; ++t)
#pragma unroll
                for (int part = 0; part < 2; ++part)
                    qd[t][part] = sw128_desc(smem_u32(smem + kOffQ + (2 * t + part) * kQBytes), 16, 1024);
#pragma unroll
            for (int u = 0; u < 2; ++u) kd[u] = sw128_desc(smem_u32(smem + kOffK + u * kKBytes), 16, 1024);
            const uint64_t vd = sw128_desc(smem_u32(smem + kOffV), kPlane, 1024);
            bool ok = mbar_wait(&bars.q_ready, 0);
            for (int j = 0; ok && j < nb; ++j) {
                const int buf = j & 1;
                if (!mbar_wait(&bars.k_full[buf], (j >> 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint64_t kb = kd[buf];
#pragma unroll
                for (int t = 0; t < kTiles; ++t) {
                    // the tile's P(j - 1) sits in its score columns until PV(j - 1) is done
                    if (j > 0 && !mbar_wait(&bars.pv_done[t], (j - 1) & 1)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sd = tS(t);
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int s = 0; s < 8; ++s)
                            mma_f16(sd, qd[t][part] + (uint64_t)(((s >> 2) * (kRows * 128) + (s & 3) * 32) >> 4),
                                    kb + (uint64_t)(((s >> 2) * kPlane + (s & 3) * 32) >> 4), qk,
                                    (part | s) ? 1u : 0u);
                    mma_commit(&bars.s_full[t]);
                }
                if (!ok) break;
                mma_commit(&bars.k_free[buf]);
                if (!mbar_wait(&bars.v_full, j & 1)) { ok = false; break; }
#pragma unroll
                for (int t = 0; t < kTiles; ++t) {
                    if (!mbar_wait(&bars.p_full[t], j & 1)) { ok = false; break; }
                    tc_fence_after();
                    // P: 16 tokens = 8 packed columns of the score buffer;
                    // V: 16 tokens = two 8-row atoms (2048 bytes)
#pragma unroll
                    for (int s = 0; s < kBlkTok / 16; ++s)
                        mma_f16_ta(tO(t), tS(t) + 8 * s, vd + (uint64_t)((s * 2048) >> 4), pv, (j | s) ? 1u : 0u);
                    mma_commit(&bars.pv_done[t]);
                }
                if (!ok) break;
                mma_commit(&bars.v_free);
            }
            if (!ok) atomicOr(&bars.flags, 1);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool timed_out = bars.flags != 0;
    if (timed_out && threadIdx.x == 32 * kDequantWarp0) set_status(a.status, KVQ_DEV_TIMEOUT);
    if (timed_out && threadIdx.x == 32 * kMmaWarp) {
        // drain: every MMA issued by this thread completes before the commit
        // arrives; TMEM is freed only after that
        mma_commit(&bars.drain);
        (void)mbar_wait(&bars.drain, 0);
    }

    // ---------------------------------------------------------------- epilogue
    // (dead is uniform across the CTA, so the warp-collective TMEM loads below
    // run on every lane of a softmax warp or on none)
    const bool dead = poison || timed_out || nb == 0;
    if (warp < kWarpsSoftmax) {
        const int t = warp >> 2;
        const int r = threadIdx.x & 127;
        const int head = r >> 5, tok = r & 31;
        const int qi = q0 + t * kQTok + tok;
        float res[kD];
        if (!dead) {
            // the last P.V of this tile has landed once its pv_done completes
            const bool ok = mbar_wait_warp(&bars.pv_done[t], (nb - 1) & 1);
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

// ------------------------------------------------------------------ launcher
template <bool KB>
static cudaError_t launch_prefill(const AttnArgs& a, dim3 grid, bool qb, bool ob, cudaStream_t st) {
    cudaError_t e;
#define KVQ_LAUNCH(TQ, TO)                                                                                     \
    e = cudaFuncSetAttribute(prefill_tc_kernel<TQ, TO, KB>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc); \
    if (e != cudaSuccess) return e;                                                                            \
    prefill_tc_kernel<TQ, TO, KB><<<grid, kThreads, kSmemAlloc, st>>>(a);
    if (qb && ob) { KVQ_LAUNCH(__nv_bfloat16, __nv_bfloat16) }
    else if (qb) { KVQ_LAUNCH(__nv_bfloat16, float) }
    else if (ob) { KVQ_LAUNCH(float, __nv_bfloat16) }
    else { KVQ_LAUNCH(float, float) }
#undef KVQ_LAUNCH
    return cudaGetLastError();
}

cudaError_t launch_prefill_tc(const AttnArgs& a, int nlayers, bool q_bf16, bool out_bf16, cudaStream_t st) {
    dim3 grid((a.q_len + kTiles * kQTok - 1) / (kTiles * kQTok), a.batch * a.Hkv, nlayers);
    if (a.kbf16) return launch_prefill<true>(a, grid, q_bf16, out_bf16, st);
    return launch_prefill<false>(a, grid, q_bf16, out_bf16, st);
}

}  // namespace kvq
