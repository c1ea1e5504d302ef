// kvq_decode.cu -- host side of the attention calls: split plan, workspace
// layout, argument block, launches.  (The log-sum-exp merge of the decode
// splits runs inside the decode kernel, in the last split of each unit.)
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

// ------------------------------------------------------------------ host side
DecodePlan decode_plan(const kvq_shape& s, int nlayers, int batch, int max_pages) {
    // One CTA per (layer, sequence, split) covers all kv heads; two CTAs are
    // resident per SM.  When the (layer, sequence) units fill at least one
    // wave they are not split: the longest-first order balances the waves
    // and no partials have to be merged.  Otherwise take the split count that
    // minimises  waves(units * splits) * (pages_per_split + 4)  for sequences
    // of max_pages (the + 4 stands for a CTA's fixed work: prologue and
    // partial), the largest among equal costs: the lengths are not known on
    // the host, and shorter pieces balance ragged lengths better.  Splits of
    // under 8 pages are not considered; the partials stay below one wave of
    // units x 64 splits.
    (void)s;
    const long units = (long)nlayers * batch;
    const long slots = 148L * 2;
    int best_s = 1;
    if (units < slots) {
        long best = -1;
        const int max_s = max(1, min(64, max_pages / 8));
        for (int sp = 1; sp <= max_s; ++sp) {
            const long pps = (max_pages + sp - 1) / sp;
            const long waves = (units * sp + slots - 1) / slots;
            const long cost = waves * (pps + 4);
            if (best < 0 || cost <= best) {
                best = cost;
                best_s = sp;
            }
        }
    }
    int pps = (max_pages + best_s - 1) / best_s;
    if (pps < 1) pps = 1;
    int splits = (max_pages + pps - 1) / pps;
    if (splits < 1) splits = 1;
    return {pps, splits};
}

// Workspace of a decode: the counter header (kWsHeader bytes, zero between
// calls), the split partials, then (KLT cache) the transformed queries.  No
// workspace at all when neither partials nor queries are needed.
static size_t partial_bytes(const kvq_shape& s, int nlayers, int batch, int max_pages) {
    DecodePlan p = decode_plan(s, nlayers, batch, max_pages);
    if (p.splits == 1) return 0;
    return (size_t)nlayers * batch * s.num_q_heads * p.splits * kPartialStride * sizeof(float);
}
static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t decode_workspace(const kvq_shape& s, int nlayers, int batch, int max_pages) {
    const size_t part = partial_bytes(s, nlayers, batch, max_pages);
    if (part == 0 && !s.use_klt) return 0;
    size_t n = kWsHeader + align256(part);
    if (s.use_klt) n += (size_t)nlayers * batch * s.num_q_heads * kD * sizeof(float);
    return n;
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
    a.kbf16 = s.k_format == KVQ_K_BF16;
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
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    a.counters = reinterpret_cast<unsigned*>(wsb);
    a.partials = wsb ? reinterpret_cast<float*>(wsb + kWsHeader) : nullptr;
    bool qb = q_dtype == KVQ_BF16;
    const bool ob = out_dtype == KVQ_BF16;
    if (p.splits > 1 && (long)nlayers * batch > kWsCounters) return KVQ_EINVAL;   // not reached by the plan
    if (s.use_klt) {
        // the queries, rotated by the KLT (and smoothed), go through the workspace
        float* qt = reinterpret_cast<float*>(wsb + kWsHeader + align256(partial_bytes(s, nlayers, batch, max_pages)));
        const kvq_status r = klt_queries(s, c, layer0, nlayers, q, q_dtype, batch, qt, st);
        if (r != KVQ_OK) return r;
        a.q = qt;
        a.qpre = 1;
        qb = false;
    }
    if (launch_decode_tc(a, nlayers, qb, ob, st) != cudaSuccess) return KVQ_ECUDA;
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

size_t prefill_workspace(const kvq_shape& s, int nlayers, int batch, int q_len) {
    // KLT cache: the rotated queries, after the header a decode's counters
    // use (untouched here, so one workspace can serve both calls)
    if (!s.use_klt) return 0;
    return kWsHeader + (size_t)nlayers * batch * q_len * s.num_q_heads * kD * sizeof(float);
}

kvq_status prefill(const kvq_shape& s, const kvq_calib& c, const kvq_cache& cache, int layer0, int nlayers,
                   const void* q, int q_dtype, int q_len, const int32_t* q_start, const int32_t* page_table,
                   int max_pages, const int32_t* seq_lens, int batch, void* out, int out_dtype, void* ws, size_t,
                   int32_t* status, cudaStream_t st, bool qk_fp4) {
    AttnArgs a = make_args(s, c, cache, layer0, q, page_table, max_pages, seq_lens, batch, out, status);
    a.q_len = q_len;
    a.q_start = q_start;
    bool qb = q_dtype == KVQ_BF16;
    const bool ob = out_dtype == KVQ_BF16;
    if (s.use_klt) {
        float* qt = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kWsHeader);
        const kvq_status r = klt_queries(s, c, layer0, nlayers, q, q_dtype, batch * q_len, qt, st);
        if (r != KVQ_OK) return r;
        a.q = qt;
        a.qpre = 1;
        qb = false;
    }
    const cudaError_t e = qk_fp4 ? launch_prefill_fp4(a, nlayers, qb, ob, st) : launch_prefill_tc(a, nlayers, qb, ob, st);
    if (e != cudaSuccess) return KVQ_ECUDA;
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

}  // namespace kvq
