// kvq_internal.h -- entry points between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>

#include "kvq.h"

namespace kvq {

// Split plan of a decode launch: pages of a sequence per CTA and the number of
// splits.  Depends only on host-known sizes, so the workspace query and the
// launch agree.
struct DecodePlan {
    int pages_per_split;
    int splits;
};
DecodePlan decode_plan(const kvq_shape& s, int nlayers, int batch, int max_pages_per_seq);
size_t decode_workspace(const kvq_shape& s, int nlayers, int batch, int max_pages_per_seq);

kvq_status calibrate(const kvq_shape& s, const void* k, const void* v, int dtype, int W, int Tlen,
                     int exclude_pos0, const kvq_calib& out, cudaStream_t st);
kvq_status calibrate_native(const kvq_shape& s, const void* k, const void* v, int dtype, int W, int Tlen,
                            const kvq_calib& out, cudaStream_t st);
kvq_status calibrate_klt(const kvq_shape& s, const void* k, const void* v, int dtype, int W, int Tlen,
                         int exclude_pos0, const kvq_calib& out, cudaStream_t st);
kvq_status append_klt_keys(const kvq_shape& s, const kvq_calib& c, const kvq_cache& cache, int layer0, int nlayers,
                           const void* k, int dtype, const int64_t* slots, int num_tokens, int32_t* status,
                           cudaStream_t st);
kvq_status klt_queries(const kvq_shape& s, const kvq_calib& c, int layer0, int nlayers, const void* q, int q_dtype,
                       int rows, float* out, cudaStream_t st);
kvq_status quantize_append(const kvq_shape& s, const kvq_calib& c, const kvq_cache& cache, int layer0,
                           int nlayers, const void* k, const void* v, int dtype, const int64_t* slots,
                           int num_tokens, int32_t* status, cudaStream_t st);
kvq_status decode(const kvq_shape& s, const kvq_calib& c, const kvq_cache& cache, int layer0, int nlayers,
                  const void* q, int q_dtype, const int32_t* page_table, int max_pages,
                  const int32_t* seq_lens, int batch, void* out, int out_dtype, void* ws, size_t ws_bytes,
                  int32_t* status, cudaStream_t st);
size_t prefill_workspace(const kvq_shape& s, int nlayers, int batch, int q_len);
kvq_status prefill(const kvq_shape& s, const kvq_calib& c, const kvq_cache& cache, int layer0, int nlayers,
                   const void* q, int q_dtype, int q_len, const int32_t* q_start, const int32_t* page_table,
                   int max_pages, const int32_t* seq_lens, int batch, void* out, int out_dtype, void* ws,
                   size_t ws_bytes, int32_t* status, cudaStream_t st, bool qk_fp4 = false);
kvq_status round_e2m1(const float* x, uint8_t* out, int64_t n, cudaStream_t st);
kvq_status selftest_wait_timeout(int32_t* status, long long limit_ns, cudaStream_t st);
kvq_status round_e4m3(const float* x, uint8_t* out, int64_t n, cudaStream_t st);

}  // namespace kvq
