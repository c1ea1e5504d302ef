// kvq_klt.cu -- static per-head KLT of the keys: calibration (second moment,
// eigenbasis, tensor scale), the key transform of the append, and the query
// transform of the attention calls.
//
// Method: "NVFP4 attention cache on W4A4 Qwen3-8B" (rstation.ai), results
// table rows "K: static per-head KLT" and "K: static KLT + smoothing": after
// the static smoothing, each (layer, kv head) rotates its keys by a fixed
// orthogonal 128 x 128 basis fitted on the calibration windows, and the query
// is rotated to match (q~ = U^T (q * s), so q~ . U^T y = q . k).
//
// The basis is the eigenbasis of the second-moment matrix C = sum y y^T of
// the smoothed calibration keys (position 0 of each window left out, as for
// the smoothing absmax), ordered by decreasing eigenvalue, each vector signed
// so that its largest-magnitude component is positive.  The key transform is
// y'_i = sum_c U[c][i] y_c, each output one fp32 fused multiply-add chain
// over c = 0..127 starting from 0 -- a fixed order, so the codes that follow
// are reproducible bit for bit.
#include <cuda_bf16.h>

#include <type_traits>

#include "kvq_common.cuh"
#include "kvq_internal.h"
#include "kvq_sync.cuh"
#include "kvq_transform.cuh"

namespace kvq {

constexpr int kKltRows = 32;          // calibration tokens staged per step

// ------------------------------------------------------------------ covariance
// C[l][h] = sum over calibration tokens t >= t0 of y y^T, y = k * inv_s
// (fp32).  One CTA per (layer, head), tokens in order: deterministic.
// Thread (i, j) of a 16 x 16 grid owns the 8 x 8 block C[8i.., 8j..].
template <typename T>
__global__ void __launch_bounds__(256)
klt_covariance_kernel(const T* __restrict__ k, int W, int Tlen, int Hkv, int t0,
                      const float* __restrict__ inv_s, float* __restrict__ C) {
    __shared__ __align__(16) float ys[kKltRows][kD];
    const int h = blockIdx.x, l = blockIdx.y;
    const int bi = threadIdx.x >> 4, bj = threadIdx.x & 15;
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;
    const float* inv = inv_s + ((size_t)l * Hkv + h) * kD;
    const int per_win = Tlen - t0;
    const int total = W * per_win;
    for (int base = 0; base < total; base += kKltRows) {
        const int nrow = min(kKltRows, total - base);
        __syncthreads();
        for (int e = threadIdx.x; e < nrow * kD; e += blockDim.x) {
            const int r = e / kD, c = e % kD;
            const int idx = base + r, w = idx / per_win, t = t0 + idx % per_win;
            const size_t off = ((((size_t)l * W + w) * Tlen + t) * Hkv + h) * kD + c;
            ys[r][c] = __fmul_rn(load_elem(k + off), __ldg(inv + c));
        }
        __syncthreads();
        for (int r = 0; r < nrow; ++r) {
            float yi[8], yj[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                yi[a] = ys[r][8 * bi + a];
                yj[a] = ys[r][8 * bj + a];
            }
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(yi[a], yj[b], acc[a][b]);
        }
    }
    float* out = C + ((size_t)l * Hkv + h) * kD * kD;
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) out[(8 * bi + a) * kD + 8 * bj + b] = acc[a][b];
}

// ------------------------------------------------------------------ eigenbasis
// Cyclic parallel Jacobi on one symmetric 128 x 128 matrix (one CTA): each
// round rotates 64 disjoint (p, q) planes chosen by the circle method (127
// rounds cover every pair once per sweep); a rotation zeroes A[p][q]:
//   theta = (A_qq - A_pp) / (2 A_pq),  t = sgn(theta) / (|theta| + sqrt(theta^2 + 1)),
//   c = 1 / sqrt(t^2 + 1),  s = t c,
// applied as A <- J^T A J and V <- V J.  The matrix is read from and the
// basis written to the same array (U[c][i] = component c of vector i).
constexpr int kJacobiSweeps = 12;
constexpr size_t kJacobiSmem = 2 * kD * kD * sizeof(float) + 2 * 64 * sizeof(float) + 2 * 64 * sizeof(int) +
                               kD * sizeof(float) + kD * sizeof(int);

__global__ void __launch_bounds__(256) klt_jacobi_kernel(float* __restrict__ CU, int Hkv) {
    extern __shared__ __align__(16) float sm[];
    float* A = sm;                       // [128][128]
    float* V = A + kD * kD;              // [128][128]
    float* cs = V + kD * kD;             // c[64], s[64]
    int* pq = reinterpret_cast<int*>(cs + 128);   // p[64], q[64]
    float* ev = reinterpret_cast<float*>(pq + 128);
    int* rank = reinterpret_cast<int*>(ev + kD);
    const int h = blockIdx.x, l = blockIdx.y;
    float* M = CU + ((size_t)l * Hkv + h) * kD * kD;
    for (int e = threadIdx.x; e < kD * kD; e += blockDim.x) {
        A[e] = M[e];
        V[e] = (e / kD == e % kD) ? 1.0f : 0.0f;
    }
    __syncthreads();
    for (int sweep = 0; sweep < kJacobiSweeps; ++sweep) {
        for (int round = 0; round < kD - 1; ++round) {
            if (threadIdx.x < 64) {
                // circle method: 127 rotates around the fixed player 127
                const int k = threadIdx.x;
                int p, q;
                if (k == 0) {
                    p = round;
                    q = kD - 1;
                } else {
                    p = (round + k) % (kD - 1);
                    q = (round - k + (kD - 1)) % (kD - 1);
                }
                if (p > q) { const int x = p; p = q; q = x; }
                const float apq = A[p * kD + q], app = A[p * kD + p], aqq = A[q * kD + q];
                float c = 1.0f, s = 0.0f;
                if (apq != 0.0f && fabsf(apq) > 1e-30f * (fabsf(app) + fabsf(aqq))) {
                    const float theta = (aqq - app) / (2.0f * apq);
                    const float t = copysignf(1.0f, theta) / (fabsf(theta) + sqrtf(theta * theta + 1.0f));
                    c = 1.0f / sqrtf(t * t + 1.0f);
                    s = t * c;
                }
                pq[k] = p;
                pq[64 + k] = q;
                cs[k] = c;
                cs[64 + k] = s;
            }
            __syncthreads();
            // rows: A <- J^T A   (pair k owns rows p_k and q_k)
            for (int e = threadIdx.x; e < 64 * kD; e += blockDim.x) {
                const int k = e / kD, col = e % kD;
                const int p = pq[k], q = pq[64 + k];
                const float c = cs[k], s = cs[64 + k];
                const float ap = A[p * kD + col], aq = A[q * kD + col];
                A[p * kD + col] = c * ap - s * aq;
                A[q * kD + col] = s * ap + c * aq;
            }
            __syncthreads();
            // columns: A <- A J, V <- V J
            for (int e = threadIdx.x; e < 64 * kD; e += blockDim.x) {
                const int k = e % 64, row = e / 64;
                const int p = pq[k], q = pq[64 + k];
                const float c = cs[k], s = cs[64 + k];
                const float ap = A[row * kD + p], aq = A[row * kD + q];
                A[row * kD + p] = c * ap - s * aq;
                A[row * kD + q] = s * ap + c * aq;
                const float vp = V[row * kD + p], vq = V[row * kD + q];
                V[row * kD + p] = c * vp - s * vq;
                V[row * kD + q] = s * vp + c * vq;
            }
            __syncthreads();
        }
    }
    // unit length (the rotations' roundings drift the norms by ~1e-5), then
    // order by decreasing eigenvalue (ties by index) and sign each vector
    if (threadIdx.x < kD) {
        const int i = threadIdx.x;
        float n2 = 0.0f;
        for (int c = 0; c < kD; ++c) n2 = fmaf(V[c * kD + i], V[c * kD + i], n2);
        const float inv = 1.0f / sqrtf(n2);
        for (int c = 0; c < kD; ++c) V[c * kD + i] *= inv;
        ev[i] = A[i * kD + i];
    }
    __syncthreads();
    if (threadIdx.x < kD) {
        const int i = threadIdx.x;
        int r = 0;
        for (int j = 0; j < kD; ++j) r += (ev[j] > ev[i]) || (ev[j] == ev[i] && j < i);
        rank[i] = r;
    }
    __syncthreads();
    if (threadIdx.x < kD) {
        const int i = threadIdx.x;          // source column
        int big = 0;
        float bv = -1.0f;
        for (int c = 0; c < kD; ++c) {
            const float a = fabsf(V[c * kD + i]);
            if (a > bv) { bv = a; big = c; }
        }
        const float sg = V[big * kD + i] < 0.0f ? -1.0f : 1.0f;
        const int dst = rank[i];
        for (int c = 0; c < kD; ++c) M[c * kD + dst] = sg * V[c * kD + i];
    }
}

// ------------------------------------------------------------------ transform
// out_i = sum_c U[c][i] y_c for the rows of a tile, one fp32 FMA chain per
// output over c in order.  The tile is 64 rows (tokens) x 128; thread
// (tg, dg) of a 16 x 16 grid owns rows 4tg..4tg+3 and outputs 8dg..8dg+7.
// Yt: [128][64] (transposed), U: [128][128], both in shared memory.
__device__ __forceinline__ void klt_tile(const float* __restrict__ Yt, const float* __restrict__ U, int tg, int dg,
                                         float (&acc)[4][8]) {
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;
#pragma unroll 4
    for (int c = 0; c < kD; ++c) {
        const float4 y4 = *reinterpret_cast<const float4*>(Yt + c * 64 + 4 * tg);
        const float4 u0 = *reinterpret_cast<const float4*>(U + c * kD + 8 * dg);
        const float4 u1 = *reinterpret_cast<const float4*>(U + c * kD + 8 * dg + 4);
        const float y[4] = {y4.x, y4.y, y4.z, y4.w};
        const float u[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(u[b], y[a], acc[a][b]);
    }
}

constexpr size_t kKltTileSmem = (size_t)kD * kD * sizeof(float) + (size_t)kD * 64 * sizeof(float);

// Eight consecutive key elements of one token, as loaded from global memory
// (kept raw in registers until they are smoothed and transposed).
template <typename T>
struct Raw8;
template <>
struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = __ldg(reinterpret_cast<const float4*>(p));
        b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.0f, 0.0f, 0.0f, 0.0f); }
    __device__ __forceinline__ void unpack(float* x) const {
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
};
template <>
struct Raw8<__nv_bfloat16> {
    uint4 v;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { v = __ldg(reinterpret_cast<const uint4*>(p)); }
    __device__ __forceinline__ void zero() { v = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void unpack(float* x) const {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            x[2 * j] = __uint_as_float(w[j] << 16);
            x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
};

// Load U of (l, h) into shared memory.
__device__ __forceinline__ void klt_load_basis(float* Us, const float* __restrict__ U) {
    for (int e = threadIdx.x; e < kD * kD / 4; e += blockDim.x)
        reinterpret_cast<float4*>(Us)[e] = __ldg(reinterpret_cast<const float4*>(U) + e);
}

// Tensor absmax of the transformed calibration keys (every token, position 0
// included): grid (token tiles, Hkv, L).
template <typename T>
__global__ void __launch_bounds__(256)
klt_tensor_amax_kernel(const T* __restrict__ k, int rows, int Hkv, const float* __restrict__ inv_s,
                       const float* __restrict__ U, uint32_t* __restrict__ gk_bits) {
    extern __shared__ __align__(16) float sm[];
    float* Us = sm;
    float* Yt = sm + kD * kD;
    const int h = blockIdx.y, l = blockIdx.z, r0 = blockIdx.x * 64;
    klt_load_basis(Us, U + ((size_t)l * Hkv + h) * kD * kD);
    const float* inv = inv_s + ((size_t)l * Hkv + h) * kD;
    for (int e = threadIdx.x; e < 64 * kD; e += blockDim.x) {
        const int r = e / kD, c = e % kD;
        float y = 0.0f;
        if (r0 + r < rows)
            y = __fmul_rn(load_elem(k + (((size_t)l * rows + r0 + r) * Hkv + h) * kD + c), __ldg(inv + c));
        Yt[c * 64 + r] = y;
    }
    __syncthreads();
    const int tg = threadIdx.x >> 4, dg = threadIdx.x & 15;
    float acc[4][8];
    klt_tile(Yt, Us, tg, dg, acc);
    float m = 0.0f;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) m = fmaxf(m, fabsf(acc[a][b]));   // padded rows are 0
#pragma unroll
    for (int x = 16; x >= 1; x >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, x));
    if ((threadIdx.x & 31) == 0) atomicMax(gk_bits + l, __float_as_uint(m));
}

// Value absmax (every token) for g_V.
template <typename T>
__global__ void klt_value_amax_kernel(const T* __restrict__ v, size_t per_layer, uint32_t* __restrict__ gv_bits) {
    const int l = blockIdx.y;
    float m = 0.0f;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < per_layer; i += (size_t)gridDim.x * blockDim.x)
        m = fmaxf(m, fabsf(load_elem(v + (size_t)l * per_layer + i)));
#pragma unroll
    for (int x = 16; x >= 1; x >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, x));
    if ((threadIdx.x & 31) == 0) atomicMax(gv_bits + l, __float_as_uint(m));
}

__global__ void klt_finalize_kernel(float* __restrict__ gk, float* __restrict__ gv, int L) {
    const int l = blockIdx.x * blockDim.x + threadIdx.x;
    if (l >= L) return;
    const float a = gk[l], b = gv[l];
    gk[l] = (a > 0.0f) ? __fdiv_rn(a, kTensorRange) : 1.0f;
    gv[l] = (b > 0.0f) ? __fdiv_rn(b, kTensorRange) : 1.0f;
}

// ------------------------------------------------------------------ append
// Keys of the KLT cache: one CTA per SM, each taking an equal run of the
// 128-token tiles of all (layer, head) units in (layer, head)-major order.  A
// CTA is two tile groups (128 threads each) that share the unit's basis and
// take every other tile of the run; one group's tile load overlaps the
// other's transform.  Smoothing y = k * inv_s, the transform y' = U^T y
// (one fp32 FMA chain per output over c = 0..127), then the NVFP4 quantiser
// of the append (absmax -> E4M3 scale -> reciprocal -> E2M1, each step one
// fp32 rounding) and the scatter to the token's slot.
//
// Thread (warp w, lane l) of a group holds 8 tokens (8 (4w + l / 8) .. + 7)
// x one 16-block of dims (16 (l % 8) .. + 15): 128 accumulators, and the
// block's absmax without a shuffle.  Per step c it reads the 8 token values
// (two 16-byte loads, shared by 8 lanes) and the block's 16 basis values
// (four 16-byte loads).  The basis rows are stored with their 16-byte chunks
// permuted, so the 8 blocks' i-th chunks sit in 8 distinct bank groups: 6
// shared-memory wavefronts per warp and step for 128 FMAs.  The FMAs run in
// packed pairs of dims (fma.rn.f32x2, each half rounded as fmaf), 64
// instructions per step, ordered by dim pair and then token so that
// consecutive ones share their basis operand; the chains and their order
// are unchanged.
constexpr int kKltTok = 128;  // tokens per append tile
constexpr int kKltGroups = 2; // tile groups per CTA
constexpr int kKltThreads = 128 * kKltGroups;
constexpr size_t kKltAppendSmem = (size_t)kD * kD * sizeof(float) +
                                  (size_t)kKltGroups * kD * kKltTok * sizeof(float) + 128 * sizeof(float) +
                                  (size_t)kKltGroups * kKltTok * sizeof(int64_t) + 16;

// Physical 16-byte chunk, within a basis row, of dims 16 blk + 4 i .. + 3:
// chunk i of the 8 blocks lands in 8 distinct bank groups.
__device__ __forceinline__ int klt_chunk(int blk, int i) { return 8 * i + ((blk + i) & 7); }

// barrier of one 128-thread tile group (named barriers 1..kKltGroups)
__device__ __forceinline__ void group_sync(int grp) {
    asm volatile("bar.sync %0, 128;" ::"r"(grp + 1) : "memory");
}

template <typename T>
__global__ void __launch_bounds__(kKltThreads, 1)
klt_append_keys_kernel(const T* __restrict__ k, const int64_t* __restrict__ slots, int num_tokens, int Hkv,
                       int nlayers, const float* __restrict__ inv_s, const float* __restrict__ U,
                       const float* __restrict__ gk, uint8_t* __restrict__ cache, int64_t layer_stride, int num_pages,
                       int32_t* __restrict__ status) {
    extern __shared__ __align__(16) float sm[];
    const int grp = threadIdx.x >> 7, tid = threadIdx.x & 127;
    float* Us = sm;                                            // [c][permuted chunks of i]
    float* Yt = Us + kD * kD + grp * kD * kKltTok;             // this group's [c][token]
    float* rtab = Us + kD * kD + kKltGroups * kD * kKltTok;
    int64_t* sslot = reinterpret_cast<int64_t*>(rtab + 128) + grp * kKltTok;
    const int64_t num_slots = (int64_t)num_pages * kPage;
    const int lane = threadIdx.x & 31;
    const int tg = 4 * (tid >> 5) + (lane >> 3);               // tokens 8 tg .. + 7
    const int blk = lane & 7;                                  // dims 16 blk .. + 15
    const int ntiles = (num_tokens + kKltTok - 1) / kKltTok;
    // This CTA's share of the tiles of all (layer, head) units, taken in
    // (layer, head)-major order: a run that crosses a unit boundary loads the
    // next unit's basis (and, past a layer, its table) between the two parts,
    // so every SM gets an equal share whatever the number of units.
    const long total = (long)nlayers * Hkv * ntiles;
    const long r0 = total * blockIdx.x / gridDim.x, r1 = total * (blockIdx.x + 1) / gridDim.x;
    // Thread tid loads token tid's key row, 16 runs of 8 elements, and its
    // slot.  The first kAhead runs (bf16: a quarter of the row) and the slot are
    // loaded one tile ahead, into registers, so their global-memory latency
    // overlaps this tile's transform; the rest when the tile starts.
    constexpr int kAhead = sizeof(T) == 2 ? 4 : 0;
    Raw8<T> raw[16];
    int64_t nslot = -1;
    int cur_li = -1;
    float enc = 0.0f;
    for (long s0 = r0; s0 < r1;) {
        // segment: tiles [tb, te) of unit u
        const int u = (int)(s0 / ntiles);
        const int tb = (int)(s0 - (long)u * ntiles);
        const int te = (int)(min(r1, (long)(u + 1) * ntiles) - (long)u * ntiles);
        s0 = (long)u * ntiles + te;
        const int li = u / Hkv, h = u - li * Hkv;
        const float* inv = inv_s + ((size_t)li * Hkv + h) * kD;
        uint8_t* layer_cache = cache + (size_t)li * layer_stride;
        auto fetch = [&](int tile_i, int e0, int e1) {
            const int t0 = tile_i * kKltTok;
            const bool live = tile_i < te && t0 + tid < num_tokens;
            const T* row = k + (((size_t)li * num_tokens + t0 + tid) * Hkv + h) * kD;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                if (e < e0 || e >= e1) continue;
                if (live) raw[e].load(row + 8 * e);
                else raw[e].zero();
            }
            if (e0 == 0) nslot = live ? __ldg(slots + t0 + tid) : -1;
        };
        const int first = tb + grp;
        if (kAhead > 0) fetch(first, 0, kAhead);
        __syncthreads();     // both groups are done with the previous unit's basis and table
        {
            const float4* src = reinterpret_cast<const float4*>(U + ((size_t)li * Hkv + h) * kD * kD);
            for (int e = threadIdx.x; e < kD * kD / 4; e += kKltThreads) {
                const int c = e >> 5, q = e & 31;              // row, logical chunk (block q / 4, i = q % 4)
                reinterpret_cast<float4*>(Us)[c * 32 + klt_chunk(q >> 2, q & 3)] = __ldg(src + e);
            }
        }
        if (li != cur_li) {
            const float g = __ldg(gk + li);
            enc = __frcp_rn(__fmul_rn(6.0f, g));
            if (threadIdx.x < 128) {
                // the append's reciprocal of every E4M3 scale code: 1/(val(c) g)
                const float d = __fmul_rn(e4m3_to_f32(threadIdx.x), g);
                rtab[threadIdx.x] = (d == 0.0f) ? 0.0f : __frcp_rn(d);
            }
            cur_li = li;
        }
        __syncthreads();     // the basis and the table are in place
        // each group walks every other tile of the segment
        for (int tile_i = first; tile_i < te; tile_i += kKltGroups) {
            group_sync(grp);     // the previous tile's Yt and slots are consumed
            fetch(tile_i, kAhead, 16);
            sslot[tid] = nslot;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                float x[8];
                raw[e].unpack(x);
#pragma unroll
                for (int j = 0; j < 8; ++j) Yt[(8 * e + j) * kKltTok + tid] = __fmul_rn(x[j], __ldg(inv + 8 * e + j));
            }
            group_sync(grp);
            if (kAhead > 0) fetch(tile_i + kKltGroups, 0, kAhead);
            float2 acc[8][8];    // token a, dims 16 blk + 2 p, + 1
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int p = 0; p < 8; ++p) acc[a][p] = make_float2(0.0f, 0.0f);
            const float* yrow = Yt + 8 * tg;
            const float4* urow = reinterpret_cast<const float4*>(Us);
#pragma unroll 4
            for (int c = 0; c < kD; ++c) {
                const float4 y0 = *reinterpret_cast<const float4*>(yrow + c * kKltTok);
                const float4 y1 = *reinterpret_cast<const float4*>(yrow + c * kKltTok + 4);
                float2 u[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 t = urow[c * 32 + klt_chunk(blk, i)];
                    u[2 * i] = make_float2(t.x, t.y);
                    u[2 * i + 1] = make_float2(t.z, t.w);
                }
                const float y[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
                // packed pairs of dims: each half is fma(u, y, acc), rounded once
                float2 yy[8];
#pragma unroll
                for (int a = 0; a < 8; ++a) yy[a] = make_float2(y[a], y[a]);
#pragma unroll
                for (int p = 0; p < 8; ++p)
#pragma unroll
                    for (int a = 0; a < 8; ++a) acc[a][p] = ffma2(u[p], yy[a], acc[a][p]);
            }
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const int64_t slot = sslot[8 * tg + a];
                float2 v[8];
#pragma unroll
                for (int p = 0; p < 8; ++p) v[p] = acc[a][p];
                const uint32_t sf = e4m3_rn(__fmul_rn(absmax16(v), enc));
                const float r = rtab[sf & 0x7Fu];
#pragma unroll
                for (int p = 0; p < 8; ++p) v[p] = make_float2(__fmul_rn(v[p].x, r), __fmul_rn(v[p].y, r));
                const uint2 w = make_uint2(e2m1x8_rn(v[0], v[1], v[2], v[3]), e2m1x8_rn(v[4], v[5], v[6], v[7]));
                if (slot >= num_slots) {
                    if (blk == 0) set_status(status, KVQ_DEV_BAD_SLOT);
                } else if (slot >= 0) {
                    uint8_t* tile = layer_cache + ((size_t)(slot >> 4) * Hkv + h) * kTile;
                    const int off = (int)(slot & 15);
                    // dims 16 blk .. + 15: code bytes 8 blk .. + 7, scale byte blk
                    *reinterpret_cast<uint2*>(tile + kKCodes + off * 64 + 8 * blk) = w;
                    tile[kKScales + off * 8 + blk] = (uint8_t)sf;
                }
            }
        }
    }
}

kvq_status append_klt_keys(const kvq_shape& s, const kvq_calib& c, const kvq_cache& cache, int layer0, int nlayers,
                           const void* k, int dtype, const int64_t* slots, int num_tokens, int32_t* status,
                           cudaStream_t st) {
    const int H = s.num_kv_heads;
    const float* inv = c.k_inv_smooth + (size_t)layer0 * H * kD;
    const float* U = c.k_klt + (size_t)layer0 * H * kD * kD;
    const float* gk = c.k_gscale + layer0;
    uint8_t* base = cache.data + (size_t)layer0 * cache.layer_stride_bytes;
    // one CTA per SM (no partial second wave), each with an equal share of
    // all units' tiles
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long total = (long)(num_tokens + kKltTok - 1) / kKltTok * H * nlayers;
    if (total == 0) return KVQ_OK;
    const long pairs = (total + kKltGroups - 1) / kKltGroups;
    const dim3 grid((unsigned)(pairs < sms ? pairs : sms));
    cudaError_t e;
    if (dtype == KVQ_F32) {
        e = cudaFuncSetAttribute(klt_append_keys_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kKltAppendSmem);
        if (e != cudaSuccess) return KVQ_ECUDA;
        klt_append_keys_kernel<float><<<grid, kKltThreads, kKltAppendSmem, st>>>(
            (const float*)k, slots, num_tokens, H, nlayers, inv, U, gk, base, cache.layer_stride_bytes, cache.num_pages,
            status);
    } else {
        e = cudaFuncSetAttribute(klt_append_keys_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kKltAppendSmem);
        if (e != cudaSuccess) return KVQ_ECUDA;
        klt_append_keys_kernel<__nv_bfloat16><<<grid, kKltThreads, kKltAppendSmem, st>>>(
            (const __nv_bfloat16*)k, slots, num_tokens, H, nlayers, inv, U, gk, base, cache.layer_stride_bytes,
            cache.num_pages, status);
    }
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

// ------------------------------------------------------------------ queries
// q~ = U^T (q * s) for every query vector of a KLT cache (decode and
// prefill), written as fp32: grid (tiles of 64 vectors, Hkv, nlayers); the
// vectors of kv head h are (row r, group member j) -> q[(l, r)][h G + j].
template <typename TQ>
__global__ void __launch_bounds__(256)
klt_query_kernel(const TQ* __restrict__ q, int rows, int Hq, int Hkv, const float* __restrict__ smooth,
                 const float* __restrict__ U, float* __restrict__ out) {
    extern __shared__ __align__(16) float sm[];
    float* Us = sm;
    float* Yt = Us + kD * kD;
    const int h = blockIdx.y, l = blockIdx.z, v0 = blockIdx.x * 64;
    const int G = Hq / Hkv, nvec = rows * G;
    klt_load_basis(Us, U + ((size_t)l * Hkv + h) * kD * kD);
    const float* sr = smooth + ((size_t)l * Hkv + h) * kD;
    for (int e = threadIdx.x; e < 64 * kD; e += blockDim.x) {
        const int vv = e / kD, c = e % kD, vec = v0 + vv;
        float y = 0.0f;
        if (vec < nvec) {
            const int r = vec / G, j = vec % G;
            y = load_elem(q + (((size_t)l * rows + r) * Hq + h * G + j) * kD + c) * __ldg(sr + c);
        }
        Yt[c * 64 + vv] = y;
    }
    __syncthreads();
    const int tg = threadIdx.x >> 4, dg = threadIdx.x & 15;
    float acc[4][8];
    klt_tile(Yt, Us, tg, dg, acc);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int vec = v0 + 4 * tg + a;
        if (vec >= nvec) continue;
        const int r = vec / G, j = vec % G;
        float4* o = reinterpret_cast<float4*>(out + (((size_t)l * rows + r) * Hq + h * G + j) * kD + 8 * dg);
        o[0] = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
        o[1] = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
    }
}

kvq_status klt_queries(const kvq_shape& s, const kvq_calib& c, int layer0, int nlayers, const void* q, int q_dtype,
                       int rows, float* out, cudaStream_t st) {
    const int H = s.num_kv_heads, G = s.num_q_heads / H;
    const float* sm = c.k_smooth + (size_t)layer0 * H * kD;
    const float* U = c.k_klt + (size_t)layer0 * H * kD * kD;
    const dim3 grid((unsigned)(((long)rows * G + 63) / 64), H, nlayers);
    cudaError_t e;
    if (q_dtype == KVQ_F32) {
        e = cudaFuncSetAttribute(klt_query_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kKltTileSmem);
        if (e != cudaSuccess) return KVQ_ECUDA;
        klt_query_kernel<float><<<grid, 256, kKltTileSmem, st>>>((const float*)q, rows, s.num_q_heads, H, sm, U, out);
    } else {
        e = cudaFuncSetAttribute(klt_query_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kKltTileSmem);
        if (e != cudaSuccess) return KVQ_ECUDA;
        klt_query_kernel<__nv_bfloat16><<<grid, 256, kKltTileSmem, st>>>((const __nv_bfloat16*)q, rows,
                                                                         s.num_q_heads, H, sm, U, out);
    }
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

template <typename T>
static kvq_status launch_calibrate_klt(const kvq_shape& s, const T* k, const T* v, int W, int Tlen, int exclude_pos0,
                                       const kvq_calib& out, cudaStream_t st) {
    // smoothing factors as kvq_calibrate_smoothing (its tensor scales are
    // recomputed below for the rotated keys)
    kvq_status r = calibrate(s, k, v, std::is_same<T, float>::value ? KVQ_F32 : KVQ_BF16, W, Tlen, exclude_pos0, out,
                             st);
    if (r != KVQ_OK) return r;
    const int L = s.num_layers, H = s.num_kv_heads;
    klt_covariance_kernel<T><<<dim3(H, L), 256, 0, st>>>(k, W, Tlen, H, exclude_pos0 ? 1 : 0, out.k_inv_smooth,
                                                         out.k_klt);
    if (cudaFuncSetAttribute(klt_jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kJacobiSmem) !=
        cudaSuccess)
        return KVQ_ECUDA;
    klt_jacobi_kernel<<<dim3(H, L), 256, kJacobiSmem, st>>>(out.k_klt, H);
    if (cudaMemsetAsync(out.k_gscale, 0, L * sizeof(float), st) != cudaSuccess ||
        cudaMemsetAsync(out.v_gscale, 0, L * sizeof(float), st) != cudaSuccess)
        return KVQ_ECUDA;
    const int rows = W * Tlen;
    if (cudaFuncSetAttribute(klt_tensor_amax_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kKltTileSmem) != cudaSuccess)
        return KVQ_ECUDA;
    klt_tensor_amax_kernel<T><<<dim3((rows + 63) / 64, H, L), 256, kKltTileSmem, st>>>(
        k, rows, H, out.k_inv_smooth, out.k_klt, reinterpret_cast<uint32_t*>(out.k_gscale));
    const size_t per_layer = (size_t)rows * H * kD;
    klt_value_amax_kernel<T><<<dim3(64, L), 256, 0, st>>>(v, per_layer, reinterpret_cast<uint32_t*>(out.v_gscale));
    klt_finalize_kernel<<<(L + 63) / 64, 64, 0, st>>>(out.k_gscale, out.v_gscale, L);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

kvq_status calibrate_klt(const kvq_shape& s, const void* k, const void* v, int dtype, int W, int Tlen,
                         int exclude_pos0, const kvq_calib& out, cudaStream_t st) {
    if (dtype == KVQ_F32)
        return launch_calibrate_klt(s, (const float*)k, (const float*)v, W, Tlen, exclude_pos0, out, st);
    return launch_calibrate_klt(s, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, W, Tlen, exclude_pos0, out, st);
}

}  // namespace kvq
