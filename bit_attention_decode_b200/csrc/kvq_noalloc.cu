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
#include <cuda.h>

#include <mutex>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace {

// 16 MiB: the split-K partials of a 36-layer decode of 4 sequences of 2304
// tokens (2 splits: about 4.9 MB) fit with room to spare; larger problems
// get KVQ_EWORKSPACE.
constexpr size_t kScratchBytes = (size_t)KVQ_NOALLOC_SCRATCH_BYTES;

__device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct ScratchEntry {
    unsigned long long ctx_id;   // context the address belongs to (0: none yet)
    void* addr;
};
ScratchEntry g_scratch[kMaxDevices] = {};

// Unique id of the calling thread's current context, or 0 when there is none
// (or the driver cannot say).  The driver calls are reached through the
// runtime's entry-point query, so the library links no driver library.
unsigned long long current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        looked_up = true;
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(f);
    }
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the array on the current device.  The name
// g_decode_scratch in host code is only a host-side stand-in, so the address
// is looked up with the device current and kept per device, together with
// the id of the context it was looked up in: after a cudaDeviceReset (a new
// primary context, the module loaded again) the address is looked up anew.
kvq_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return KVQ_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    const unsigned long long id = current_context_id();
    if (id == 0 || g_scratch[dev].ctx_id != id || !g_scratch[dev].addr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KVQ_ECUDA;
        g_scratch[dev] = {current_context_id(), p};
    }
    *out = g_scratch[dev].addr;
    return KVQ_OK;
}

}  // namespace

extern "C" kvq_status kvq_decode_attention_noalloc(const kvq_shape* shape, const kvq_calib* calib,
                                                   const kvq_cache* cache, int32_t layer0, int32_t nlayers,
                                                   const void* q, int32_t q_dtype, const int32_t* page_table,
                                                   int32_t max_pages_per_seq, const int32_t* seq_lens,
                                                   int32_t batch, void* out, int32_t out_dtype,
                                                   int32_t* dev_status, void* stream) {
    // kvq_decode_attention runs every host check, the scratch size last: a
    // problem whose split-K partials need more than the array gets
    // KVQ_EWORKSPACE after the argument checks, and nothing is launched
    void* scratch = nullptr;
    kvq_status st = scratch_address(&scratch);
    if (st != KVQ_OK) return st;
    return kvq_decode_attention(shape, calib, cache, layer0, nlayers, q, q_dtype, page_table, max_pages_per_seq,
                                seq_lens, batch, out, out_dtype, scratch, kScratchBytes, dev_status, stream);
}
