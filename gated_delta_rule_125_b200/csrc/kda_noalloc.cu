// kda_noalloc.cu -- kda_prefill_noalloc: the chunkwise prefill for callers
// that cannot hand the library a device workspace.
//
// Some callers have no way to allocate device memory at the point where they
// run the prefill: a runtime that owns every byte of device memory through its
// own fixed pool and forbids libraries from calling cudaMalloc, a plugin
// hosted by a framework that does not expose its allocator, or a
// latency-critical serving loop where cudaMalloc (which can synchronise the
// whole device) is not acceptable. For them this entry point runs the same
// kernels as kda_prefill, with the workspace taken from one fixed array that
// is part of the library's device image.
//
// The array is file-scope, 256-byte aligned and kNoAllocScratchBytes large;
// every GPU that loads the library holds it until the process exits. Every
// call shares it and it keeps the last call's contents. The prefill needs no
// part of it to start at zero except its counters and ring flags, which the
// prefill's own planning kernel clears at the start of every call. Calls that overlap
// on the GPU (different streams, or several host threads) race on the array
// and give wrong results; the caller must order them.
#include "kda_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(KDA_NOALLOC_SCRATCH_BYTES);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

kda::SymbolCache g_noalloc_cache;

// Device address of the scratch array on the current device: resolved with
// cudaGetSymbolAddress, with that device current, on the first call made in
// the device's context, then cached (resolved again for a new context).
void *noalloc_scratch() {
    return kda::symbol_address(reinterpret_cast<const void *>(&g_noalloc_scratch), g_noalloc_cache);
}

}  // namespace

extern "C" kda_status kda_prefill_noalloc(const void *q, const void *k, const void *v,
                                          const float *log_alpha, const float *beta,
                                          const float *S0, const int32_t *cu_seqlens,
                                          int32_t num_seqs, int64_t total_tokens,
                                          int32_t max_seqlen, int32_t H, int32_t dk, int32_t dv,
                                          kda_dtype dtype, int32_t chunk, uint32_t flags, void *o,
                                          float *S_T, kda_stream_t stream) {
    // Problems whose smallest workspace does not fit the array are refused
    // before anything is enqueued; invalid arguments are left to kda_prefill,
    // which reports them the same way for both entry points.
    const size_t need = kda_prefill_workspace_min(num_seqs, total_tokens, max_seqlen, H, dk, dv,
                                                  dtype, chunk, flags);
    if (need > kNoAllocScratchBytes) return KDA_ERR_WORKSPACE;
    void *scratch = noalloc_scratch();
    if (!scratch) return KDA_ERR_CUDA;
    return kda_prefill(q, k, v, log_alpha, beta, S0, cu_seqlens, num_seqs, total_tokens,
                       max_seqlen, H, dk, dv, dtype, chunk, flags, o, S_T, scratch,
                       kNoAllocScratchBytes, stream);
}
