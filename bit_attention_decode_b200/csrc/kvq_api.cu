// kvq_api.cu -- the C ABI: argument validation, then the launches.
//
// Every check here runs on the host before anything is launched; a failed
// check returns an error code and leaves device memory untouched.
#include <stdint.h>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

#define KVQ_TRY_LOCAL(x)                 \
    do {                                 \
        kvq_status _st = (x);            \
        if (_st != KVQ_OK) return _st;   \
    } while (0)

kvq_status check_shape(const kvq_shape* s) {
    if (!s) return KVQ_EINVAL;
    if (s->head_dim != kvq::kD || s->page_size != kvq::kPage) return KVQ_EUNSUPPORTED;
    if (s->num_layers < 1 || s->num_kv_heads < 1 || s->num_q_heads < 1) return KVQ_EINVAL;
    if (s->num_q_heads % s->num_kv_heads != 0) return KVQ_EINVAL;
    // one decode CTA holds a warp per kv head; a warp serves up to 4 query heads
    if (s->num_kv_heads > 8 || s->num_q_heads / s->num_kv_heads > 4) return KVQ_EUNSUPPORTED;
    if (s->use_hadamard != 0 && s->use_hadamard != 1) return KVQ_EINVAL;
    // the rotation's cross-lane butterflies need whole warps of key lanes
    if (s->use_hadamard && (s->num_kv_heads & 1)) return KVQ_EUNSUPPORTED;
    if (s->k_format != KVQ_K_NVFP4 && s->k_format != KVQ_K_BF16) return KVQ_EINVAL;
    // bf16 keys are stored untransformed
    if (s->k_format == KVQ_K_BF16 && s->use_hadamard) return KVQ_EINVAL;
    // the KLT replaces the rotation and rotates packed keys only
    if (s->use_klt != 0 && s->use_klt != 1) return KVQ_EINVAL;
    if (s->use_klt && (s->use_hadamard || s->k_format != KVQ_K_NVFP4)) return KVQ_EINVAL;
    return KVQ_OK;
}

kvq_status check_device() {
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ECUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return KVQ_ECUDA;
    return major == 10 ? KVQ_OK : KVQ_EUNSUPPORTED;
}

bool good_dtype(int32_t d) { return d == KVQ_F32 || d == KVQ_BF16; }

kvq_status check_calib(const kvq_calib* c) {
    if (!c || !c->k_smooth || !c->k_inv_smooth || !c->k_gscale || !c->v_gscale) return KVQ_EINVAL;
    return KVQ_OK;
}

// a KLT shape also needs the bases
kvq_status check_calib(const kvq_shape* s, const kvq_calib* c) {
    KVQ_TRY_LOCAL(check_calib(c));
    if (s->use_klt && (!c->k_klt || !aligned(c->k_klt, 16))) return KVQ_EINVAL;
    return KVQ_OK;
}

kvq_status check_cache(const kvq_shape* s, const kvq_cache* c) {
    if (!c || !c->data || c->num_pages < 1) return KVQ_EINVAL;
    if (!aligned(c->data, 16) || (c->layer_stride_bytes & 15) != 0) return KVQ_EINVAL;
    if (c->layer_stride_bytes < (int64_t)c->num_pages * s->num_kv_heads * kvq::tile_bytes(s->k_format))
        return KVQ_EINVAL;
    return KVQ_OK;
}

kvq_status check_layers(const kvq_shape* s, int32_t layer0, int32_t nlayers) {
    if (layer0 < 0 || nlayers < 1 || layer0 + nlayers > s->num_layers || nlayers > 65535) return KVQ_EINVAL;
    return KVQ_OK;
}

#define KVQ_TRY(x)                       \
    do {                                 \
        kvq_status _st = (x);            \
        if (_st != KVQ_OK) return _st;   \
    } while (0)

}  // namespace

extern "C" {

size_t kvq_page_bytes(const kvq_shape* shape) {
    if (check_shape(shape) != KVQ_OK) return 0;
    return (size_t)shape->num_kv_heads * kvq::tile_bytes(shape->k_format);
}

const char* kvq_status_string(kvq_status st) {
    switch (st) {
        case KVQ_OK: return "ok";
        case KVQ_EINVAL: return "invalid argument";
        case KVQ_ECUDA: return "CUDA error";
        case KVQ_EUNSUPPORTED: return "unsupported shape or device";
        case KVQ_EWORKSPACE: return "workspace too small";
        default: return "unknown status";
    }
}

const char* kvq_version(void) { return "kvq 0.1 sm_100a"; }

kvq_status kvq_calibrate_smoothing(const kvq_shape* shape, const void* k_calib, const void* v_calib,
                                   int32_t dtype, int32_t num_windows, int32_t window_len,
                                   int32_t exclude_pos0, const kvq_calib* out, void* stream) {
    KVQ_TRY(check_shape(shape));
    KVQ_TRY(check_calib(out));
    if (!k_calib || !v_calib || !good_dtype(dtype) || num_windows < 1 || window_len < 1) return KVQ_EINVAL;
    if (exclude_pos0 != 0 && exclude_pos0 != 1) return KVQ_EINVAL;
    if (!aligned(k_calib, 16) || !aligned(v_calib, 16)) return KVQ_EINVAL;
    if (num_windows > 65535 || (long)num_windows * window_len * shape->num_kv_heads > (1L << 28)) return KVQ_EINVAL;
    KVQ_TRY(check_device());
    return kvq::calibrate(*shape, k_calib, v_calib, dtype, num_windows, window_len, exclude_pos0, *out,
                          (cudaStream_t)stream);
}

kvq_status kvq_calibrate_native(const kvq_shape* shape, const void* k_calib, const void* v_calib, int32_t dtype,
                                int32_t num_windows, int32_t window_len, const kvq_calib* out, void* stream) {
    KVQ_TRY(check_shape(shape));
    KVQ_TRY(check_calib(out));
    if (!k_calib || !v_calib || !good_dtype(dtype) || num_windows < 1 || window_len < 1) return KVQ_EINVAL;
    if (!aligned(k_calib, 16) || !aligned(v_calib, 16)) return KVQ_EINVAL;
    if (num_windows > 65535 || (long)num_windows * window_len * shape->num_kv_heads > (1L << 28)) return KVQ_EINVAL;
    KVQ_TRY(check_device());
    return kvq::calibrate_native(*shape, k_calib, v_calib, dtype, num_windows, window_len, *out,
                                 (cudaStream_t)stream);
}

kvq_status kvq_calibrate_klt(const kvq_shape* shape, const void* k_calib, const void* v_calib, int32_t dtype,
                             int32_t num_windows, int32_t window_len, int32_t exclude_pos0, const kvq_calib* out,
                             void* stream) {
    KVQ_TRY(check_shape(shape));
    if (!shape->use_klt) return KVQ_EINVAL;
    KVQ_TRY(check_calib(shape, out));
    if (!k_calib || !v_calib || !good_dtype(dtype) || num_windows < 1 || window_len < 1) return KVQ_EINVAL;
    if (exclude_pos0 != 0 && exclude_pos0 != 1) return KVQ_EINVAL;
    if (window_len <= exclude_pos0) return KVQ_EINVAL;
    if (!aligned(k_calib, 16) || !aligned(v_calib, 16)) return KVQ_EINVAL;
    if (num_windows > 65535 || (long)num_windows * window_len * shape->num_kv_heads > (1L << 28)) return KVQ_EINVAL;
    KVQ_TRY(check_device());
    return kvq::calibrate_klt(*shape, k_calib, v_calib, dtype, num_windows, window_len, exclude_pos0, *out,
                              (cudaStream_t)stream);
}

kvq_status kvq_quantize_append(const kvq_shape* shape, const kvq_calib* calib, const kvq_cache* cache,
                               int32_t layer0, int32_t nlayers, const void* k, const void* v, int32_t dtype,
                               const int64_t* slot_mapping, int32_t num_tokens, int32_t* dev_status,
                               void* stream) {
    KVQ_TRY(check_shape(shape));
    KVQ_TRY(check_calib(shape, calib));
    KVQ_TRY(check_cache(shape, cache));
    KVQ_TRY(check_layers(shape, layer0, nlayers));
    if (num_tokens < 0 || !good_dtype(dtype)) return KVQ_EINVAL;
    if (num_tokens == 0) return KVQ_OK;
    if (!k || !v || !slot_mapping || !aligned(k, 16) || !aligned(v, 16) || !aligned(slot_mapping, 8))
        return KVQ_EINVAL;
    KVQ_TRY(check_device());
    return kvq::quantize_append(*shape, *calib, *cache, layer0, nlayers, k, v, dtype, slot_mapping, num_tokens,
                                dev_status, (cudaStream_t)stream);
}

size_t kvq_decode_workspace_bytes(const kvq_shape* shape, int32_t nlayers, int32_t batch,
                                  int32_t max_pages_per_seq) {
    if (check_shape(shape) != KVQ_OK || nlayers < 1 || batch < 1 || max_pages_per_seq < 1) return 0;
    return kvq::decode_workspace(*shape, nlayers, batch, max_pages_per_seq);
}

kvq_status kvq_decode_attention(const kvq_shape* shape, const kvq_calib* calib, const kvq_cache* cache,
                                int32_t layer0, int32_t nlayers, const void* q, int32_t q_dtype,
                                const int32_t* page_table, int32_t max_pages_per_seq, const int32_t* seq_lens,
                                int32_t batch, void* out, int32_t out_dtype, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, void* stream) {
    KVQ_TRY(check_shape(shape));
    KVQ_TRY(check_calib(shape, calib));
    KVQ_TRY(check_cache(shape, cache));
    KVQ_TRY(check_layers(shape, layer0, nlayers));
    if (batch < 1 || max_pages_per_seq < 1 || (long)batch * shape->num_kv_heads > 65535) return KVQ_EINVAL;
    if (!good_dtype(q_dtype) || !good_dtype(out_dtype)) return KVQ_EINVAL;
    if (!q || !out || !page_table || !seq_lens || !aligned(q, 16) || !aligned(out, 16)) return KVQ_EINVAL;
    const size_t need = kvq::decode_workspace(*shape, nlayers, batch, max_pages_per_seq);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16))) return KVQ_EWORKSPACE;
    KVQ_TRY(check_device());
    return kvq::decode(*shape, *calib, *cache, layer0, nlayers, q, q_dtype, page_table, max_pages_per_seq,
                       seq_lens, batch, out, out_dtype, workspace, workspace_bytes, dev_status,
                       (cudaStream_t)stream);
}

size_t kvq_prefill_workspace_bytes(const kvq_shape* shape, int32_t nlayers, int32_t batch, int32_t q_len) {
    if (check_shape(shape) != KVQ_OK || nlayers < 1 || batch < 1 || q_len < 1) return 0;
    return kvq::prefill_workspace(*shape, nlayers, batch, q_len);
}

static kvq_status prefill_common(const kvq_shape* shape, const kvq_calib* calib, const kvq_cache* cache,
                                 int32_t layer0, int32_t nlayers, const void* q, int32_t q_dtype, int32_t q_len,
                                 const int32_t* q_start, const int32_t* page_table, int32_t max_pages_per_seq,
                                 const int32_t* seq_lens, int32_t batch, void* out, int32_t out_dtype,
                                 void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream, bool qk_fp4) {
    KVQ_TRY(check_shape(shape));
    KVQ_TRY(check_calib(shape, calib));
    KVQ_TRY(check_cache(shape, cache));
    KVQ_TRY(check_layers(shape, layer0, nlayers));
    // FP4 Q.K needs packed keys
    if (qk_fp4 && shape->k_format != KVQ_K_NVFP4) return KVQ_EINVAL;
    if (batch < 1 || q_len < 1 || max_pages_per_seq < 1 || (long)batch * shape->num_kv_heads > 65535)
        return KVQ_EINVAL;
    if (!good_dtype(q_dtype) || !good_dtype(out_dtype)) return KVQ_EINVAL;
    if (!q || !out || !q_start || !page_table || !seq_lens || !aligned(q, 16) || !aligned(out, 16))
        return KVQ_EINVAL;
    const size_t need = kvq::prefill_workspace(*shape, nlayers, batch, q_len);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16))) return KVQ_EWORKSPACE;
    KVQ_TRY(check_device());
    return kvq::prefill(*shape, *calib, *cache, layer0, nlayers, q, q_dtype, q_len, q_start, page_table,
                        max_pages_per_seq, seq_lens, batch, out, out_dtype, workspace, workspace_bytes,
                        dev_status, (cudaStream_t)stream, qk_fp4);
}


kvq_status kvq_prefill_attention(const kvq_shape* shape, const kvq_calib* calib, const kvq_cache* cache,
                                 int32_t layer0, int32_t nlayers, const void* q, int32_t q_dtype, int32_t q_len,
                                 const int32_t* q_start, const int32_t* page_table, int32_t max_pages_per_seq,
                                 const int32_t* seq_lens, int32_t batch, void* out, int32_t out_dtype,
                                 void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
    return prefill_common(shape, calib, cache, layer0, nlayers, q, q_dtype, q_len, q_start, page_table,
                          max_pages_per_seq, seq_lens, batch, out, out_dtype, workspace, workspace_bytes, dev_status,
                          stream, false);
}

kvq_status kvq_prefill_attention_fp4(const kvq_shape* shape, const kvq_calib* calib, const kvq_cache* cache,
                                     int32_t layer0, int32_t nlayers, const void* q, int32_t q_dtype, int32_t q_len,
                                     const int32_t* q_start, const int32_t* page_table, int32_t max_pages_per_seq,
                                     const int32_t* seq_lens, int32_t batch, void* out, int32_t out_dtype,
                                     void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
    return prefill_common(shape, calib, cache, layer0, nlayers, q, q_dtype, q_len, q_start, page_table,
                          max_pages_per_seq, seq_lens, batch, out, out_dtype, workspace, workspace_bytes, dev_status,
                          stream, true);
}

kvq_status kvq_selftest_wait_timeout(int32_t* dev_status, int64_t limit_ns, void* stream) {
    if (!dev_status || limit_ns < 1000 || limit_ns > 10000000000LL) return KVQ_EINVAL;
    KVQ_TRY(check_device());
    return kvq::selftest_wait_timeout(dev_status, (long long)limit_ns, (cudaStream_t)stream);
}

kvq_status kvq_round_e2m1(const float* x, uint8_t* codes, int64_t n, void* stream) {
    if (n < 0 || (n > 0 && (!x || !codes))) return KVQ_EINVAL;
    if (n == 0) return KVQ_OK;
    KVQ_TRY(check_device());
    return kvq::round_e2m1(x, codes, n, (cudaStream_t)stream);
}

kvq_status kvq_round_e4m3(const float* x, uint8_t* codes, int64_t n, void* stream) {
    if (n < 0 || (n > 0 && (!x || !codes))) return KVQ_EINVAL;
    if (n == 0) return KVQ_OK;
    KVQ_TRY(check_device());
    return kvq::round_e4m3(x, codes, n, (cudaStream_t)stream);
}

}  // extern "C"
