// kvq_noalloc.cu -- kvq_decode_attention_noalloc: the decode entry point for
// callers that cannot allocate device memory.
//
// Some callers have no way to obtain a workspace: code that runs inside a
// host runtime which owns the whole device-memory budget (a serving engine's
// pool, a plugin slot) and forbids stray allocations, or latency-critical
// paths where cudaMalloc's implicit device-wide synchronisation is not
// acceptable.  For them the split-K partials live in one file-scope device
// array, reserved when the library is loaded and held until process exit on
// every GPU that loads it.
//
// The array is shared by every call on a device and keeps whatever the last
// call left there.  The decode kernel writes every partial it later reads
// (each split of each row writes its own slot before the combine reads it),
// so nothing has to be cleared between calls.  Two calls whose GPU work
// overlaps -- on different streams, or from different host threads -- race
// on the array and corrupt each other's results; serialise them.
#include <mutex>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace {

// 16 MiB: enough for the split-K partials of a 36-layer Qwen3-8B-shaped decode
// at batch 4 x 2304 tokens (about 12 MB); larger problems get KVQ_EWORKSPACE.
constexpr size_t kScratchBytes = (size_t)KVQ_NOALLOC_SCRATCH_BYTES;

__device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the array on the current device.  The name
// g_decode_scratch in host code is only a host-side stand-in, so the address
// is looked up once per device (with that device current) and kept.
kvq_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return KVQ_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KVQ_ECUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return KVQ_OK;
}

}  // namespace

extern "C" kvq_status kvq_decode_attention_noalloc(const kvq_shape* shape, const kvq_calib* calib,
                                                   const kvq_cache* cache, int32_t layer0, int32_t nlayers,
                                                   const void* q, int32_t q_dtype, const int32_t* page_table,
                                                   int32_t max_pages_per_seq, const int32_t* seq_lens,
                                                   int32_t batch, void* out, int32_t out_dtype,
                                                   int32_t* dev_status, void* stream) {
    // same host checks as kvq_decode_attention, then the scratch-size check
    size_t need = kvq_decode_workspace_bytes(shape, nlayers, batch, max_pages_per_seq);
    if (need > kScratchBytes) return KVQ_EWORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        kvq_status st = scratch_address(&scratch);
        if (st != KVQ_OK) return st;
    }
    return kvq_decode_attention(shape, calib, cache, layer0, nlayers, q, q_dtype, page_table, max_pages_per_seq,
                                seq_lens, batch, out, out_dtype, need > 0 ? scratch : nullptr,
                                need > 0 ? kScratchBytes : 0, dev_status, stream);
}
