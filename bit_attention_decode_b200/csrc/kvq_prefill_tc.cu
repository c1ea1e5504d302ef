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
// dequantised key/value block feeds 8 query heads x 32 tokens.  Per 64-token
// key block (4 pages):
//   copy warp: bulk-copies the 4 packed page tiles into a staging ring.
//   dequant warps (2): dequantise to fp16 (E2M1 x E4M3 is exact in fp16)
//     into a K tile (K-major) and a V tile (MN-major), both in the
//     128-byte-swizzled canonical layouts the MMA reads; rows past the
//     sequence are zeros.
//   MMA warp (1 elected thread): for each tile, S = Q_hi K^T + Q_lo K^T
//     (M=128, N=64, K=16 steps; the query is split into fp16 hi + lo parts
//     so its rounding does not reach the scores) into one of the tile's two
//     TMEM score buffers, then O += P V (M=128, N=128) with P read from TMEM.
//   softmax warpgroups (one per tile; a thread owns one TMEM lane = row):
//     causal mask on diagonal blocks only, running max with lazy rescaling
//     (the output in TMEM is rescaled only when the max grows by more than
//     2^8), probabilities rounded once to fp16 and stored back over the
//     first 32 columns of their own score buffer as the A operand of P V.
// The two tiles ping-pong: while one warpgroup works on its scores, the
// tensor pipe runs the other tile's MMAs.  TMEM: O_A, O_B (128 columns each),
// S_A[2], S_B[2] (64 each) = 512 columns.
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
constexpr int kBlkTok = 64;         // key tokens per block (4 pages)
constexpr int kStageN = 3;          // packed-page staging stages
constexpr uint32_t kTmemCols = 512; // O_A, O_B [0,256), S_A[2] [256,384), S_B[2] [384,512)
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr int kPidCap = 1024;       // page ids held in shared memory (keys up to 16384 tokens)

// shared memory map (offsets from a 1024-aligned base)
constexpr int kQBytes = kRows * kD * 2;           // 32 KB per fp16 query tile part (hi or lo)
constexpr int kKBytes = kBlkTok * kD * 2;         // 16 KB per fp16 key tile
constexpr int kVBytes = kBlkTok * kD * 2;         // 16 KB per fp16 value tile
constexpr int kStageBytes = 4 * kTile;            // 4 packed page tiles of one head
constexpr int kVPart = kTileBf16K - kBf16VCodes;  // 1152: values of a bf16-key tile (staged alone)
constexpr int kOffQ = 0;                          // [tile][hi, lo]
constexpr int kOffK = kOffQ + kTiles * 2 * kQBytes;   // 2 buffers
constexpr int kOffV = kOffK + 2 * kKBytes;        // 2 buffers
constexpr int kOffStage = kOffV + 2 * kVBytes;    // kStageN stages
constexpr int kSmemBytes = kOffStage + kStageN * kStageBytes;
constexpr int kSmemAlloc = kSmemBytes + 1024;     // room to align the base

// warps 8, 9 dequantise; warp 10 only issues the bulk copies (a copy costs
// the issuing thread hundreds of cycles, which would otherwise sit on a
// dequant warp's path every block)
enum { kWarpsSoftmax = 4 * kTiles, kWarpsDequant = 2 };
constexpr int kDequantWarp0 = kWarpsSoftmax;                   // warps 8, 9
constexpr int kCopyWarp = kDequantWarp0 + kWarpsDequant;       // warp 10
constexpr int kMmaWarp = kCopyWarp + 1;                        // warp 11
constexpr int kThreads = 32 * (kMmaWarp + 1);

struct PrefillBars {
    uint64_t q_ready;                 // both softmax warpgroups wrote their query tiles (count 8)
    uint64_t stage_full[kStageN];     // packed pages landed (tx bytes)
    uint64_t stage_empty[kStageN];    // dequant warps read the stage (count 2)
    uint64_t k_full[2];               // K tile j%2 written (count 2)
    uint64_t v_full[2];               // V tile j%2 written (count 2)
    uint64_t s_full[kTiles][2];       // QK(tile, j) done (commit)
    uint64_t p_full[kTiles][2];       // P(tile, j) stored in TMEM, O rescaled (count 4)
    uint64_t pv_done[kTiles][2];      // PV(tile, j) done (commit)
    uint64_t drain;                   // last commit before TMEM is freed after a timeout
    uint32_t tmem_base;
    int flags;                        // 1: a bounded wait ran out
    int issued;                       // packed-page stages issued
};

// ------------------------------------------------------------------ kernel
// grid (query-tile pairs, batch * Hkv, nlayers), block 384.
// KB: mixed cache (bf16 keys, untransformed; only the value parts of the
// tiles are staged, the key rows are copied into the key tile directly, and
// Q.K runs on bf16 operands).
template <typename TQ, typename TO, bool KB>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ PrefillBars bars;
    __shared__ int32_t s_pid[kPidCap];   // the sequence's page ids, read once for every copy

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
    const int nb = (kv_end + kBlkTok - 1) / kBlkTok;          // 64-token blocks
    const int npg = (kv_end + kPage - 1) / kPage;             // pages touched
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
            for (int t = 0; t < kTiles; ++t) {
                mbar_init(&bars.s_full[t][i], 1);
                mbar_init(&bars.p_full[t][i], 4);
                mbar_init(&bars.pv_done[t][i], 1);
            }
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
    // per tile t: O at tmem + 128 t; S buffer u at tmem + 256 + 128 t + 64 u
    auto tO = [&](int t) { return tmem + 128u * t; };
    auto tS = [&](int t, int u) { return tmem + 256u + 128u * t + 64u * u; };

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
                const int u = j & 1;
                if (!mbar_wait_warp(&bars.s_full[t][u], (j >> 1) & 1)) { atomicOr(&bars.flags, 1); break; }
                tc_fence_after();
                float s[kBlkTok];
                tmem_ld32(tS(t, u) + lane_addr, s);
                tmem_ld32(tS(t, u) + 32 + lane_addr, s + 32);
                const int kp0 = j * kBlkTok;
                // interior blocks (every key visible to this row) skip the mask
                if (kp0 + kBlkTok - 1 > qpos || kp0 + kBlkTok > kv_end) {
#pragma unroll
                    for (int c = 0; c < kBlkTok; ++c) {
                        const int kp = kp0 + c;
                        s[c] = (kp <= qpos && kp < kv_end) ? s[c] : -INFINITY;
                    }
                }
                // block max as a tree of three-input maxima (depth 4, not 64)
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
                // lazy rescale: move the reference max only when it grows by > 2^8
                const bool grow = bm > m_run + kRescaleThreshold || (m_run == -INFINITY && bm > -INFINITY);
                bool stop = false;
                if (__any_sync(0xFFFFFFFFu, grow)) {
                    const float mn = grow ? bm : m_run;
                    const float al = (m_run == -INFINITY) ? 0.0f : ex2(m_run - mn);
                    if (j > 0) {
                        // the previous P.V must have landed before O is rescaled
                        if (!mbar_wait_warp(&bars.pv_done[t][u ^ 1], ((j - 1) >> 1) & 1)) {
                            atomicOr(&bars.flags, 1);
                            stop = true;
                        }
                        if (!stop) {
                            tc_fence_after();
#pragma unroll 1
                            for (int cc = 0; cc < 4; ++cc) {
                                float o[32];
                                tmem_ld32(tO(t) + cc * 32 + lane_addr, o);
#pragma unroll
                                for (int i = 0; i < 32; ++i) o[i] *= al;
                                tmem_st32(tO(t) + cc * 32 + lane_addr, o);
                            }
                        }
                    }
                    l_run *= al;
                    m_run = mn;
                }
                if (stop) break;
                // probabilities, fp16, stored over the first 32 columns of the score
                // buffer; one pair in four is exponentiated on the FMA pipe
                const float2 sc2 = make_float2(isig, isig), nm2 = make_float2(-m_run, -m_run);
                // four independent partial sums (the row sum is a 32-deep chain otherwise)
                float2 lsum[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                                  make_float2(0.0f, 0.0f)};
#pragma unroll
                for (int hv = 0; hv < 2; ++hv) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float2 x = ffma2(make_float2(s[32 * hv + 2 * c], s[32 * hv + 2 * c + 1]), sc2, nm2);
                        float2 pp;
                        if ((c & 3) == 3) {
                            pp.x = poly_exp2(x.x);
                            pp.y = poly_exp2(x.y);
                        } else {
                            pp.x = ex2(x.x);
                            pp.y = ex2(x.y);
                        }
                        lsum[c & 3] = fadd2(lsum[c & 3], pp);
                        pk[c] = h2(pp.x, pp.y);
                    }
                    tmem_st16u(tS(t, u) + 16 * hv + lane_addr, pk);
                }
                const float2 l2 = fadd2(fadd2(lsum[0], lsum[1]), fadd2(lsum[2], lsum[3]));
                l_run += l2.x + l2.y;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.p_full[t][u]);
            }
        } else if (warp == kCopyWarp) {
            // ------------------------------------------------------ copy warp
            // block j's page tiles (the value parts only for bf16 keys) into
            // stage j % kStageN, once the dequant warps have read block
            // j - kStageN out of it; page ids come from shared memory
            if (lane == 0) {
                constexpr int part = KB ? kVPart : kTile;          // bytes staged per page
                constexpr int part0 = KB ? kBf16VCodes : 0;       // offset of that part in the tile
                constexpr int tile = KB ? kTileBf16K : kTile;
                int issued = 0;
                for (; issued < nb; ++issued) {
                    const int st = issued % kStageN;
                    if (issued >= kStageN &&
                        !mbar_wait(&bars.stage_empty[st], ((issued - kStageN) / kStageN) & 1)) {
                        atomicOr(&bars.flags, 1);
                        break;
                    }
                    const int p_lo = issued * 4, n_p = min(npg, p_lo + 4) - p_lo;
                    mbar_arrive_expect_tx(&bars.stage_full[st], (uint32_t)n_p * part);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (k < n_p) {
                            const int p = p_lo + k;
                            const int pg = p < kPidCap ? s_pid[p] : __ldg(pt + p);
                            bulk_g2s(smem + kOffStage + st * kStageBytes + k * part,
                                     layer_base + ((size_t)pg * a.Hkv + h) * tile + part0, part, &bars.stage_full[st]);
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
            // read block j's codes and scales out of its stage and release it
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
                        if constexpr (KB) {
                            // the stage holds the value parts only
                            const uint8_t* T = smem + kOffStage + st * kStageBytes + (tkn >> 4) * kVPart;
                            S.vc[e][0] = *reinterpret_cast<const uint4*>(T + trow * 64 + half * 32);
                            S.vc[e][1] = *reinterpret_cast<const uint4*>(T + trow * 64 + half * 32 + 16);
#pragma unroll
                            for (int q = 0; q < 4; ++q) S.vs[e][q] = T[1024 + (half * 4 + q) * 16 + trow];
                        } else {
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
                }
                __syncwarp();
                if ((dt & 31) == 0) mbar_arrive(&bars.stage_empty[st]);
                return true;
            };
            // keys of block j into K buffer j & 1, free once both tiles'
            // Q.K(j - 2) are done (the commit after the last MMA covers all)
            auto store_k = [&](int j, const Staged& S) -> bool {
                const int buf = j & 1;
                if (j >= 2 && !mbar_wait_warp(&bars.s_full[kTiles - 1][buf], ((j - 2) >> 1) & 1)) return false;
                uint8_t* Kt = smem + kOffK + buf * kKBytes;
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    const int it = dt + e * kDqThreads;
                    if (it >= kItems) break;
                    const int tkn = it >> 1, half = it & 1;
                    const bool valid = j * kBlkTok + tkn < kv_end;
                    // 4 blocks of 16 dims: 8 code bytes and one scale each
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4& c0 = S.kc[e][q >> 1];
                        const uint32_t kw0 = (q & 1) ? c0.z : c0.x, kw1 = (q & 1) ? c0.w : c0.y;
                        uint32_t ka[4], kb[4];
                        e2m1x8(kw0, ka);
                        e2m1x8(kw1, kb);
                        const uint32_t ksh = e4m3x2_to_f16x2((S.ks[e] >> (8 * q)) & 0xFFu) & 0xFFFFu;
                        const uint32_t ksc = valid ? (ksh | (ksh << 16)) : 0u;
                        // chunk index along head_dim: 2 chunks (8 dims each) per block
                        const int dim_chunk = half * 8 + 2 * q;          // 0..15
                        const int plane = dim_chunk >> 3, ch = dim_chunk & 7;
                        // keys: K-major, row = token, dims 0..63 / 64..127 in planes of 64 rows x 128 B
                        sts128(Kt + plane * (kBlkTok * 128) + sw128(tkn, ch), hmul2u(ka[0], ksc),
                               hmul2u(ka[1], ksc), hmul2u(ka[2], ksc), hmul2u(ka[3], ksc));
                        sts128(Kt + plane * (kBlkTok * 128) + sw128(tkn, ch + 1), hmul2u(kb[0], ksc),
                               hmul2u(kb[1], ksc), hmul2u(kb[2], ksc), hmul2u(kb[3], ksc));
                    }
                }
                fence_async_smem();
                __syncwarp();
                if ((dt & 31) == 0) mbar_arrive(&bars.k_full[buf]);
                return true;
            };
            // bf16 keys of block j: once K buffer j & 1 is free, 16-byte async
            // copies of each row straight into its swizzled place (zeros past
            // the sequence); finish_k waits for them and hands the tile over
            auto issue_k = [&](int j) -> bool {
                const int buf = j & 1;
                if (j >= 2 && !mbar_wait_warp(&bars.s_full[kTiles - 1][buf], ((j - 2) >> 1) & 1)) return false;
                uint8_t* Kt = smem + kOffK + buf * kKBytes;
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    const int it = dt + e * kDqThreads;
                    if (it >= kItems) break;
                    const int tkn = it >> 1, half = it & 1;
                    uint8_t* dst = Kt + half * (kBlkTok * 128);
                    if (j * kBlkTok + tkn < kv_end) {
                        const int p = j * 4 + (tkn >> 4);
                        const int pg = p < kPidCap ? s_pid[p] : __ldg(pt + p);
                        const uint8_t* src = layer_base + ((size_t)pg * a.Hkv + h) * kTileBf16K + (tkn & 15) * 256 +
                                             half * 128;
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
            // values of block j into V buffer j & 1, free once both tiles'
            // P.V(j - 2) are done
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
                        // values: MN-major, row = token (the K of P.V), 128-byte rows of 64 dims
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
            // Software-pipelined: the keys of block j + 1 are written before
            // the values of block j, because the MMA warp needs them first
            // (Q.K(j + 1) is issued before P.V(j)).
            Staged cur, nxt;
            bool dq_ok = true;
            if constexpr (KB) {
                // the copies of block j + 1's keys overlap the values of block j
                if (nb > 0) {
                    dq_ok = load_block(0, cur) && issue_k(0);
                    if (dq_ok) finish_k(0);
                }
                for (int j = 0; dq_ok && j < nb; ++j) {
                    const bool more = j + 1 < nb;
                    if (more) dq_ok = load_block(j + 1, nxt) && issue_k(j + 1);
                    dq_ok = dq_ok && store_v(j, cur);
                    if (more && dq_ok) finish_k(j + 1);
                    cur = nxt;
                }
                cp_async_wait_all();   // nothing in flight past this point
            } else {
                dq_ok = nb == 0 || (load_block(0, cur) && store_k(0, cur));
                for (int j = 0; dq_ok && j < nb; ++j) {
                    if (j + 1 < nb) dq_ok = load_block(j + 1, nxt) && store_k(j + 1, nxt);
                    dq_ok = dq_ok && store_v(j, cur);
                    cur = nxt;
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
            uint64_t qd[kTiles][2], kd[2], vd[2];
#pragma unroll
            for (int t = 0; t < kTiles; ++t)
#pragma unroll
                for (int part = 0; part < 2; ++part)
                    qd[t][part] = sw128_desc(smem_u32(smem + kOffQ + (2 * t + part) * kQBytes), 16, 1024);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                kd[u] = sw128_desc(smem_u32(smem + kOffK + u * kKBytes), 16, 1024);
                vd[u] = sw128_desc(smem_u32(smem + kOffV + u * kVBytes), kBlkTok * 128, 1024);
            }
            bool ok = mbar_wait(&bars.q_ready, 0);
            for (int j = 0; ok && j <= nb; ++j) {
                if (j < nb) {
                    const int buf = j & 1;
                    if (!mbar_wait(&bars.k_full[buf], (j >> 1) & 1)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t kb = kd[buf];
                    // tile by tile, so that tile A's softmax starts while the
                    // tensor pipe works on tile B
#pragma unroll
                    for (int t = 0; t < kTiles; ++t) {
                        const uint32_t sd = tS(t, buf);
#pragma unroll
                        for (int part = 0; part < 2; ++part)
#pragma unroll
                            for (int s = 0; s < 8; ++s)
                                mma_f16(sd, qd[t][part] + (uint64_t)(((s >> 2) * (kRows * 128) + (s & 3) * 32) >> 4),
                                        kb + (uint64_t)(((s >> 2) * (kBlkTok * 128) + (s & 3) * 32) >> 4), qk,
                                        (part | s) ? 1u : 0u);
                        mma_commit(&bars.s_full[t][buf]);
                    }
                }
                if (j >= 1) {
                    const int jp = j - 1, buf = jp & 1;
                    const uint64_t vb = vd[buf];
                    if (!mbar_wait(&bars.v_full[buf], (jp >> 1) & 1)) { ok = false; break; }
#pragma unroll
                    for (int t = 0; t < kTiles; ++t) {
                        if (!mbar_wait(&bars.p_full[t][buf], (jp >> 1) & 1)) { ok = false; break; }
                        tc_fence_after();
                        // P: 16 tokens = 8 packed columns of the score buffer;
                        // V: 16 tokens = two 8-row atoms (2048 bytes)
#pragma unroll
                        for (int s = 0; s < 4; ++s)
                            mma_f16_ta(tO(t), tS(t, buf) + 8 * s, vb + (uint64_t)((s * 2048) >> 4), pv,
                                       (jp | s) ? 1u : 0u);
                        mma_commit(&bars.pv_done[t][buf]);
                    }
                    if (!ok) break;
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
        // drain: the packed-page copies still in flight
        const int issued = bars.issued;
        for (int j = max(0, issued - kStageN); j < issued; ++j)
            (void)mbar_wait(&bars.stage_full[j % kStageN], (j / kStageN) & 1);
        set_status(a.status, KVQ_DEV_TIMEOUT);
    }
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
