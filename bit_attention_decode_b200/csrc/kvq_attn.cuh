// kvq_attn.cuh -- argument block and constants shared by the attention kernels.
#pragma once

#include "kvq_common.cuh"

namespace kvq {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kPartialStride = 132;  // floats per split partial: m, l, pad, pad, o[128]
// The first bytes of every attention workspace: one arrival counter per
// (layer, sequence) unit of a split decode.  They must hold zeros before the
// first call and every decode leaves them zero (the last split of a unit
// resets its counter), so a workspace is zero-filled once, when allocated.
// Splits are used only below one wave of (layer, sequence) units (fewer than
// 296), so 1024 counters always suffice.
constexpr size_t kWsHeader = 4096;
constexpr int kWsCounters = (int)(kWsHeader / sizeof(unsigned));

struct AttnArgs {
    const uint8_t* cache;      // layer layer0
    int64_t layer_stride;
    int num_pages, Hkv, Hq, G, hadamard;
    int kbf16;                 // keys stored as bf16 (mixed cache)
    int qpre;                  // q already carries the smoothing and the KLT (fp32)
    const float* smooth;       // [nl][Hkv][D] at layer0
    const float* gk;           // [nl] at layer0
    const float* gv;
    const void* q;             // decode [nl][B][Hq][D]; prefill [nl][B][q_len][Hq][D]
    const int32_t* page_table;
    int max_pages;
    const int32_t* seq_lens;
    const int32_t* q_start;    // prefill only
    int batch, q_len;
    void* out;
    float* partials;           // decode with splits > 1
    unsigned* counters;        // decode with splits > 1: [nl][B] arrivals (workspace header)
    int splits, pps;
    int32_t* status;
};

// tensor-core split-K decode (kvq_decode_tc.cu)
cudaError_t launch_decode_tc(const AttnArgs& a, int nlayers, bool q_bf16, bool out_bf16, cudaStream_t st);
size_t decode_tc_smem(int Hkv, bool kbf16);
// tensor-core (tcgen05) chunked causal prefill (kvq_prefill_tc.cu)
cudaError_t launch_prefill_tc(const AttnArgs& a, int nlayers, bool q_bf16, bool out_bf16, cudaStream_t st);
// the same with Q.K on block-scaled FP4 operands (kvq_prefill_fp4.cu)
cudaError_t launch_prefill_fp4(const AttnArgs& a, int nlayers, bool q_bf16, bool out_bf16, cudaStream_t st);

}  // namespace kvq
