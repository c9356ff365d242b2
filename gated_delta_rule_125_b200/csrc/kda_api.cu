// kda_api.cu -- the extern "C" boundary of libkda.so: argument validation on
// the host, workspace planning and dispatch to the kernels. Nothing here
// allocates device memory or synchronises.
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "kda_internal.cuh"

namespace {

constexpr float kEps = 1e-6f;  // eps in q / max(||q||, eps)
constexpr uint32_t kKnownFlags = KDA_FLAG_NO_L2NORM | KDA_FLAG_EXACT | KDA_FLAG_SCALAR_GATE;

bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// log_alpha: 16 bytes (tensor-map rows), or 4 with one gate per (token, head).
bool gate_aligned(const void *p, uint32_t flags) {
    return (flags & KDA_FLAG_SCALAR_GATE) ? (reinterpret_cast<uintptr_t>(p) & 3u) == 0 : aligned16(p);
}

// The fused output step's arguments (nullptr: none).
kda_status check_output_gate(const kda_output_gate *g, bool any_tokens) {
    if (!g) return KDA_OK;
    if (!(g->eps > 0.f) || (any_tokens && (!g->gate || !g->weight))) return KDA_ERR_INVALID_ARG;
    if (!aligned16(g->gate) || (reinterpret_cast<uintptr_t>(g->weight) & 3u)) return KDA_ERR_MISALIGNED;
    return KDA_OK;
}

bool dims_supported(int32_t dk, int32_t dv) {
    return (dk == 64 || dk == 128) && (dv == 64 || dv == 128);
}

// Shape checks shared by the workspace queries and the prefill itself.
kda_status check_prefill_shape(int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t dk,
                               int32_t dv, kda_dtype dtype, int32_t chunk, uint32_t flags) {
    if (num_seqs < 1 || num_seqs > 65535 || total_tokens < 0 || H < 1 || H > 65535 || dk < 1 ||
        dv < 1 || chunk < 1)
        return KDA_ERR_INVALID_ARG;
    if (flags & ~kKnownFlags) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
    if (!dims_supported(dk, dv) || chunk != kda::kChunk) return KDA_ERR_UNSUPPORTED;
    if (total_tokens > (int64_t)INT32_MAX * kda::kChunk) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

// How the prefill uses its workspace.
// CUDA-core path: it runs in waves of chunks; workspace = [state carry: N*H*dk*dv
// fp32 (several waves only)][slots of one wave].
// Tensor-core path: one persistent kernel; workspace = the schedule tables and
// a ring of R slots for each of `streams` streams (more slots: the chunk
// preparation runs further ahead of the scan).
struct Plan {
    bool tc;             // tensor-core path
    int64_t max_chunks;  // chunks of the longest sequence
    size_t slot_bytes;   // per (chunk, sequence, head), CUDA-core path
    size_t units;        // N * H
    size_t state_bytes;  // running-state carry between waves, CUDA-core path
    int streams;         // tensor-core path: scan streams
    int64_t max_len;     // tensor-core path: bound on a stream's chunk count
};

bool use_tc(kda_dtype dtype, int32_t dk, int32_t dv, uint32_t flags) {
    return dtype == KDA_DTYPE_BF16 && dk == 128 && dv == 128 && !(flags & KDA_FLAG_EXACT);
}

Plan make_plan(int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen, int32_t H, int32_t dk,
               int32_t dv, kda_dtype dtype, uint32_t flags) {
    Plan p;
    p.tc = use_tc(dtype, dk, dv, flags);
    int64_t L = (max_seqlen > 0) ? std::min<int64_t>(max_seqlen, total_tokens) : total_tokens;
    p.max_chunks = (L + kda::kChunk - 1) / kda::kChunk;
    p.slot_bytes = kda::simt_slot_bytes(dk);
    p.units = (size_t)num_seqs * H;
    p.state_bytes = (size_t)num_seqs * H * dk * dv * sizeof(float);
    p.streams = (int)std::min<size_t>(p.units, (size_t)kda::kTcMaxStreams);
    p.max_len = (int64_t)((p.units + p.streams - 1) / p.streams) * std::max<int64_t>(p.max_chunks, 1);
    return p;
}

// Tensor-core path: recommended and smallest ring (slots per stream).
constexpr int64_t kRingMin = 4;
int tc_ring(const Plan &p, int64_t want) {
    return (int)std::max<int64_t>(1, std::min<int64_t>({want, (int64_t)kda::tc_max_ring(), p.max_len}));
}
size_t tc_bytes(const Plan &p, int R) { return kda::tc_workspace_bytes((long long)p.units, p.streams, R); }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// CUDA-core path: bytes needed for waves of nw chunks (several waves also
// need the state carry).
size_t bytes_for(const Plan &p, int64_t nw, bool multi) {
    return round_up((size_t)nw * p.units * p.slot_bytes, 1024) + (multi ? round_up(p.state_bytes, 1024) : 0);
}

// CUDA-core path: the smaller of one wave holding every chunk and the smallest
// multi-wave plan. Tensor-core path: the smallest ring.
size_t min_bytes(const Plan &p) {
    if (p.tc) return tc_bytes(p, tc_ring(p, kRingMin));
    const size_t single = bytes_for(p, std::max<int64_t>(p.max_chunks, 1), false);
    if (p.max_chunks <= 1) return single;
    return std::min(single, bytes_for(p, 1, true));
}

constexpr size_t kRecommendedCap = size_t(512) << 20;

// Chunks per wave for a workspace of `bytes` (>= min_bytes(p)).
int64_t waves_chunks(const Plan &p, size_t bytes) {
    const int64_t all = std::max<int64_t>(p.max_chunks, 1);
    if (p.max_chunks <= 1 || bytes_for(p, all, false) <= bytes) return all;
    int64_t lo = 1, hi = all - 1;  // largest nw with bytes_for(nw, multi) <= bytes
    while (lo < hi) {
        const int64_t mid = (lo + hi + 1) / 2;
        if (bytes_for(p, mid, true) <= bytes) lo = mid;
        else hi = mid - 1;
    }
    return std::min<int64_t>(lo, INT32_MAX);
}

}  // namespace

namespace kda {

__device__ int g_device_error;  // set by kernels whose bounded waits ran out

namespace {
// cuCtxGetCurrent / cuCtxGetId through the runtime's driver entry points (no
// libcuda link): the identity of the current context, unique for the life of
// the process, so a cached device address is re-resolved after the device's
// context was destroyed and recreated (cudaDeviceReset).
typedef int (*PfnCtxGetCurrent)(void **);
typedef int (*PfnCtxGetId)(void *, unsigned long long *);
bool context_id(unsigned long long *id) {
    static PfnCtxGetCurrent get_current = nullptr;
    static PfnCtxGetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PfnCtxGetCurrent>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PfnCtxGetId>(p);
    });
    void *ctx = nullptr;
    return get_current && get_id && get_current(&ctx) == 0 && ctx && get_id(ctx, id) == 0;
}
}  // namespace

void *symbol_address(const void *symbol, SymbolCache &cache) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= SymbolCache::kMaxDevices) return nullptr;
    unsigned long long ctx = 0;
    std::lock_guard<std::mutex> lock(cache.mu);
    if (context_id(&ctx) && cache.addr[dev] && cache.ctx[dev] == ctx) return cache.addr[dev];
    // (the runtime makes the device's primary context current here if it is not yet)
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess || !p) return nullptr;
    cache.addr[dev] = p;
    cache.ctx[dev] = context_id(&ctx) ? ctx : 0;  // 0: never matches, resolved on every call
    return p;
}

int *device_error_word() {
    static SymbolCache cache;
    return static_cast<int *>(symbol_address(reinterpret_cast<const void *>(&g_device_error), cache));
}

}  // namespace kda

extern "C" {

const char *kda_status_string(kda_status s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: null pointer or invalid size";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: shape, chunk or dtype not implemented";
        case KDA_ERR_MISALIGNED: return "KDA_ERR_MISALIGNED: pointer not 16-byte aligned";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing or too small";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA error while enqueueing";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: bounded device wait gave up";
    }
    return "KDA_ERR_UNKNOWN";
}

int32_t kda_version(void) { return 100; }

size_t kda_prefill_workspace_min(int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen,
                                 int32_t H, int32_t dk, int32_t dv, kda_dtype dtype,
                                 int32_t chunk, uint32_t flags) {
    if (check_prefill_shape(num_seqs, total_tokens, H, dk, dv, dtype, chunk, flags) != KDA_OK) return 0;
    return min_bytes(make_plan(num_seqs, total_tokens, max_seqlen, H, dk, dv, dtype, flags));
}

size_t kda_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen,
                                  int32_t H, int32_t dk, int32_t dv, kda_dtype dtype,
                                  int32_t chunk, uint32_t flags) {
    if (check_prefill_shape(num_seqs, total_tokens, H, dk, dv, dtype, chunk, flags) != KDA_OK) return 0;
    Plan p = make_plan(num_seqs, total_tokens, max_seqlen, H, dk, dv, dtype, flags);
    const int64_t all = std::max<int64_t>(p.max_chunks, 1);
    if (p.tc) return tc_bytes(p, tc_ring(p, kda::tc_max_ring()));
    const size_t single = bytes_for(p, all, false);
    if (single <= kRecommendedCap) return single;
    const int64_t nw = std::max<int64_t>(1, (int64_t)(kRecommendedCap / (p.units * p.slot_bytes)));
    return std::max(min_bytes(p), bytes_for(p, std::min(nw, all), true));
}

int64_t kda_prefill_launches(int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen,
                             int32_t H, int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk,
                             uint32_t flags, size_t workspace_bytes) {
    if (check_prefill_shape(num_seqs, total_tokens, H, dk, dv, dtype, chunk, flags) != KDA_OK) return -1;
    Plan p = make_plan(num_seqs, total_tokens, max_seqlen, H, dk, dv, dtype, flags);
    if (workspace_bytes < min_bytes(p)) return -1;
    if (p.tc) return 2;  // planning kernel + persistent prefill kernel
    const int64_t nw = waves_chunks(p, workspace_bytes);
    if (p.max_chunks == 0) return 1;
    const int64_t waves = (p.max_chunks + nw - 1) / nw;
    return 2 * waves;  // prep, scan per wave
}

kda_status kda_prefill(const void *q, const void *k, const void *v, const float *log_alpha,
                       const float *beta, const float *S0, const int32_t *cu_seqlens,
                       int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen, int32_t H,
                       int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk, uint32_t flags,
                       void *o, float *S_T, void *workspace, size_t workspace_bytes,
                       kda_stream_t stream) {
    return kda_prefill_ex(q, k, v, log_alpha, beta, S0, cu_seqlens, num_seqs, total_tokens,
                          max_seqlen, H, dk, dv, dtype, chunk, flags, nullptr, o, S_T, workspace,
                          workspace_bytes, stream);
}

}  // extern "C"

namespace {
// kda_prefill_ex and kda_prefill_conv: `conv` holds the three inputs' short
// convolutions (nullptr entries, or a nullptr array: none).
kda_status prefill_impl(const void *q, const void *k, const void *v, const float *log_alpha,
                        const float *beta, const float *S0, const int32_t *cu_seqlens, int32_t num_seqs,
                        int64_t total_tokens, int32_t max_seqlen, int32_t H, int32_t dk, int32_t dv,
                        kda_dtype dtype, int32_t chunk, uint32_t flags, const kda_short_conv *const *conv,
                        const kda_output_gate *out_gate, void *o, float *S_T, void *workspace,
                        size_t workspace_bytes, kda_stream_t stream) {
    kda_status rc = check_prefill_shape(num_seqs, total_tokens, H, dk, dv, dtype, chunk, flags);
    if (rc != KDA_OK) return rc;
    if ((rc = check_output_gate(out_gate, total_tokens > 0)) != KDA_OK) return rc;
    if (cu_seqlens == nullptr && num_seqs != 1) return KDA_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !o)) return KDA_ERR_INVALID_ARG;
    if (!workspace) return KDA_ERR_WORKSPACE;
    const void *ptrs[] = {q, k, v, S0, cu_seqlens, o, S_T, workspace};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(beta) & 3u) return KDA_ERR_MISALIGNED;
    if (!gate_aligned(log_alpha, flags)) return KDA_ERR_MISALIGNED;

    Plan p = make_plan(num_seqs, total_tokens, max_seqlen, H, dk, dv, dtype, flags);
    bool any_conv = false;
    for (int i = 0; conv && i < 3; ++i) {
        const kda_short_conv *c = conv[i];
        if (!c) continue;
        if (!p.tc || c->width < 1 || c->width > kda::kPrefillMaxConvWidth) return KDA_ERR_UNSUPPORTED;
        if (!c->weight) return KDA_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(c->weight) & 3u) return KDA_ERR_MISALIGNED;
        if (!aligned16(c->state_in) || !aligned16(c->state_out)) return KDA_ERR_MISALIGNED;
        any_conv = true;
    }
    if (workspace_bytes < min_bytes(p)) return KDA_ERR_WORKSPACE;

    kda::PrefillArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0;
    a.cu = cu_seqlens; a.total = total_tokens;
    a.N = num_seqs; a.H = H; a.dk = dk; a.dv = dv;
    a.l2norm = (flags & KDA_FLAG_NO_L2NORM) ? 0 : 1;
    a.la_scalar = (flags & KDA_FLAG_SCALAR_GATE) ? 1 : 0;
    a.eps = kEps;
    a.og_gate = out_gate ? out_gate->gate : nullptr;
    a.og_w = out_gate ? out_gate->weight : nullptr;
    a.og_eps = out_gate ? out_gate->eps : 0.f;
    a.o = o; a.S_T = S_T;
    a.slot_bytes = p.slot_bytes;
    for (int i = 0; i < 3; ++i) {
        const kda_short_conv *c = conv ? conv[i] : nullptr;
        a.conv_W[i] = c ? c->width : 0;
        a.conv_w[i] = c ? c->weight : nullptr;
        a.conv_state[i] = c ? c->state_in : nullptr;
    }

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);

    if (p.tc) {
        int *err = kda::device_error_word();
        if (!err) return KDA_ERR_CUDA;
        a.state = nullptr;
        a.slots = nullptr;
        if (kda::tc_prefill(a, ws, workspace_bytes, p.streams, err, st) != cudaSuccess) return KDA_ERR_CUDA;
        // each sequence's last W-1 raw inputs, after the prefill has read the initial states
        for (int i = 0; any_conv && i < 3; ++i) {
            const kda_short_conv *c = conv[i];
            if (!c || !c->state_out || c->width < 2) continue;
            kda::ShortConvArgs sa;
            sa.x = i == 0 ? q : i == 1 ? k : v;
            sa.y = nullptr;
            sa.w = c->weight;
            sa.state_in = c->state_in;
            sa.state_out = c->state_out;
            sa.cu = cu_seqlens;
            sa.N = num_seqs;
            sa.total = total_tokens;
            sa.C = H * (i == 2 ? dv : dk);
            sa.W = c->width;
            if (kda::short_conv_state(sa, true, st) != cudaSuccess) return KDA_ERR_CUDA;
        }
        return KDA_OK;
    }
    const int64_t nw = waves_chunks(p, workspace_bytes);
    const bool multi = nw < p.max_chunks;
    a.state = multi ? reinterpret_cast<float *>(ws) : nullptr;
    a.slots = ws + (multi ? round_up(p.state_bytes, 1024) : 0);
    const bool bf16 = dtype == KDA_DTYPE_BF16;
    if (p.max_chunks == 0)  // only empty sequences: S_T = S0
        return kda::simt_prefill_wave(a, 0, 0, bf16, st) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    for (int64_t j0 = 0; j0 < p.max_chunks; j0 += nw) {
        const int n = (int)std::min<int64_t>(nw, p.max_chunks - j0);
        if (kda::simt_prefill_wave(a, (int)j0, n, bf16, st) != cudaSuccess) return KDA_ERR_CUDA;
    }
    if (a.og_gate && total_tokens > 0 && kda::simt_output_gate(a, bf16, st) != cudaSuccess) return KDA_ERR_CUDA;
    return KDA_OK;
}
}  // namespace

extern "C" {

kda_status kda_prefill_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, const float *S0, const int32_t *cu_seqlens,
                          int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen, int32_t H,
                          int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk, uint32_t flags,
                          const kda_output_gate *out_gate, void *o, float *S_T, void *workspace,
                          size_t workspace_bytes, kda_stream_t stream) {
    return prefill_impl(q, k, v, log_alpha, beta, S0, cu_seqlens, num_seqs, total_tokens, max_seqlen, H, dk, dv,
                        dtype, chunk, flags, nullptr, out_gate, o, S_T, workspace, workspace_bytes, stream);
}

kda_status kda_prefill_conv(const void *q, const void *k, const void *v, const float *log_alpha,
                            const float *beta, const float *S0, const int32_t *cu_seqlens,
                            int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen, int32_t H,
                            int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk, uint32_t flags,
                            const kda_short_conv *conv_q, const kda_short_conv *conv_k,
                            const kda_short_conv *conv_v, const kda_output_gate *out_gate, void *o,
                            float *S_T, void *workspace, size_t workspace_bytes, kda_stream_t stream) {
    const kda_short_conv *conv[3] = {conv_q, conv_k, conv_v};
    return prefill_impl(q, k, v, log_alpha, beta, S0, cu_seqlens, num_seqs, total_tokens, max_seqlen, H, dk, dv,
                        dtype, chunk, flags, conv, out_gate, o, S_T, workspace, workspace_bytes, stream);
}

kda_status kda_device_error(int32_t *code, int32_t reset) {
    if (!code) return KDA_ERR_INVALID_ARG;
    int *w = kda::device_error_word();
    if (!w) return KDA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
    if (reset && v != 0) {
        const int zero = 0;
        if (cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return KDA_ERR_CUDA;
    }
    *code = v;
    return v == 0 ? KDA_OK : KDA_ERR_TIMEOUT;
}

uint64_t kda_set_wait_limit_ns(uint64_t ns) { return kda::tc_set_wait_limit(ns); }

kda_status kda_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, float *S, int32_t N, int32_t H, int32_t dk,
                           int32_t dv, kda_dtype dtype, uint32_t flags, void *o,
                           kda_stream_t stream) {
    return kda_decode_step_ex(q, k, v, log_alpha, beta, S, N, H, dk, dv, dtype, flags, nullptr, o,
                              stream);
}

kda_status kda_decode_step_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, float *S, int32_t N, int32_t H, int32_t dk,
                              int32_t dv, kda_dtype dtype, uint32_t flags,
                              const kda_output_gate *out_gate, void *o, kda_stream_t stream) {
    if (N < 1 || H < 1 || dk < 1 || dv < 1 || (int64_t)N * H > INT32_MAX) return KDA_ERR_INVALID_ARG;
    if (flags & ~kKnownFlags) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
    if (!dims_supported(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !log_alpha || !beta || !S || !o) return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, S, o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(beta) & 3u) return KDA_ERR_MISALIGNED;
    if (!gate_aligned(log_alpha, flags)) return KDA_ERR_MISALIGNED;
    const kda_status rc = check_output_gate(out_gate, true);
    if (rc != KDA_OK) return rc;
    cudaError_t e = kda::decode_step(q, k, v, log_alpha, beta, S, N, H, dk, dv,
                                     dtype == KDA_DTYPE_BF16, (flags & KDA_FLAG_NO_L2NORM) ? 0 : 1,
                                     (flags & KDA_FLAG_SCALAR_GATE) ? 1 : 0, kEps,
                                     out_gate ? out_gate->gate : nullptr,
                                     out_gate ? out_gate->weight : nullptr, out_gate ? out_gate->eps : 0.f,
                                     nullptr, o, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

namespace {
// Chunk slots of the backward: H per chunk of every sequence (bounded by total / 64 + N), kept
// within one launch grid.
bool backward_fits(int32_t num_seqs, int64_t total_tokens, int32_t H) {
    return kda::backward_slots_per_head(num_seqs, total_tokens) * H <= INT32_MAX;
}
}  // namespace

size_t kda_backward_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t max_seqlen, int32_t H,
                                   int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk, uint32_t flags) {
    if (check_prefill_shape(num_seqs, total_tokens, H, dk, dv, dtype, chunk, flags) != KDA_OK) return 0;
    (void)max_seqlen;  // the slots follow the sequences' own chunk counts
    if (!backward_fits(num_seqs, total_tokens, H)) return 0;
    return kda::backward_workspace_bytes(num_seqs, H, total_tokens, dk, dv);
}

kda_status kda_backward(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                        const float *S0, const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                        int32_t max_seqlen, int32_t H, int32_t dk, int32_t dv, kda_dtype dtype, int32_t chunk,
                        uint32_t flags, const void *dout, const float *dS_T, float *dq, float *dk_out,
                        float *dv_out, float *dlog_alpha, float *dbeta, float *dS0, void *workspace,
                        size_t workspace_bytes, kda_stream_t stream) {
    kda_status rc = check_prefill_shape(num_seqs, total_tokens, H, dk, dv, dtype, chunk, flags);
    if (rc != KDA_OK) return rc;
    if (cu_seqlens == nullptr && num_seqs != 1) return KDA_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !dout || !dq || !dk_out || !dv_out ||
                             !dlog_alpha || !dbeta))
        return KDA_ERR_INVALID_ARG;
    if (!backward_fits(num_seqs, total_tokens, H)) return KDA_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < kda::backward_workspace_bytes(num_seqs, H, total_tokens, dk, dv))
        return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 15u)) return KDA_ERR_MISALIGNED;
    kda::BackwardArgs a;
    a.q = q; a.k = k; a.v = v; a.dout = dout;
    a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0; a.dS_T = dS_T; a.cu = cu_seqlens;
    a.total = total_tokens; a.N = num_seqs; a.H = H; a.dk = dk; a.dv = dv;
    a.l2norm = (flags & KDA_FLAG_NO_L2NORM) ? 0 : 1;
    a.la_scalar = (flags & KDA_FLAG_SCALAR_GATE) ? 1 : 0;
    a.eps = kEps;
    a.dq = dq; a.dk_out = dk_out; a.dv_out = dv_out; a.dlog_alpha = dlog_alpha; a.dbeta = dbeta; a.dS0 = dS0;
    a.ws = workspace;
    a.err = kda::device_error_word();
    const cudaError_t e = kda::backward(a, dtype == KDA_DTYPE_BF16, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_short_conv_swish(const void *x, void *y, const kda_short_conv *conv, const int32_t *cu_seqlens,
                                int32_t num_seqs, int64_t total_tokens, int32_t channels, kda_dtype dtype,
                                kda_stream_t stream) {
    if (!conv || num_seqs < 1 || total_tokens < 0 || channels < 8 || channels % 8) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
    if (conv->width < 1 || conv->width > KDA_MAX_CONV_WIDTH) return KDA_ERR_UNSUPPORTED;
    if (cu_seqlens == nullptr && num_seqs != 1) return KDA_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!x || !y || !conv->weight)) return KDA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(conv->state_in) || !aligned16(conv->state_out))
        return KDA_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(conv->weight) & 3u) return KDA_ERR_MISALIGNED;
    const size_t es = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    const uintptr_t xb = reinterpret_cast<uintptr_t>(x), yb = reinterpret_cast<uintptr_t>(y);
    const uintptr_t bytes = (uintptr_t)total_tokens * (uintptr_t)channels * es;
    if (total_tokens > 0 && xb < yb + bytes && yb < xb + bytes) return KDA_ERR_INVALID_ARG;  // y overlaps x
    kda::ShortConvArgs a;
    a.x = x;
    a.y = y;
    a.w = conv->weight;
    a.state_in = conv->state_in;
    a.state_out = conv->state_out;
    a.cu = cu_seqlens;
    a.N = num_seqs;
    a.total = total_tokens;
    a.C = channels;
    a.W = conv->width;
    const cudaError_t e = kda::short_conv_swish(a, dtype == KDA_DTYPE_BF16, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int64_t kda_short_conv_launches(int32_t width, int32_t writes_state, int64_t total_tokens) {
    if (width < 1 || width > KDA_MAX_CONV_WIDTH || total_tokens < 0) return -1;
    return kda::short_conv_launches(width, writes_state != 0, total_tokens);
}

kda_status kda_decode_step_conv(const void *q, const void *k, const void *v, const float *log_alpha,
                                const float *beta, float *S, int32_t N, int32_t H, int32_t dk, int32_t dv,
                                kda_dtype dtype, uint32_t flags, const kda_short_conv *conv_q,
                                const kda_short_conv *conv_k, const kda_short_conv *conv_v,
                                const kda_output_gate *out_gate, void *o, kda_stream_t stream) {
    if (N < 1 || H < 1 || dk < 1 || dv < 1 || (int64_t)N * H > INT32_MAX) return KDA_ERR_INVALID_ARG;
    if (flags & ~kKnownFlags) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
    if (!dims_supported(dk, dv)) return KDA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !log_alpha || !beta || !S || !o) return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, S, o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(beta) & 3u) return KDA_ERR_MISALIGNED;
    if (!gate_aligned(log_alpha, flags)) return KDA_ERR_MISALIGNED;
    kda_status rc = check_output_gate(out_gate, true);
    if (rc != KDA_OK) return rc;
    kda::DecodeConv cv{};
    const kda_short_conv *cs[3] = {conv_q, conv_k, conv_v};
    for (int i = 0; i < 3; ++i) {
        if (!cs[i]) continue;
        if (cs[i]->width < 1 || cs[i]->width > kda::kDecodeMaxConvWidth) return KDA_ERR_UNSUPPORTED;
        if (!cs[i]->weight) return KDA_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(cs[i]->weight) & 3u) return KDA_ERR_MISALIGNED;
        if (!aligned16(cs[i]->state_in) || !aligned16(cs[i]->state_out)) return KDA_ERR_MISALIGNED;
        cv.W[i] = cs[i]->width;
        cv.w[i] = cs[i]->weight;
        cv.state_in[i] = cs[i]->state_in;
        cv.state_out[i] = cs[i]->state_out;
    }
    cudaError_t e = kda::decode_step(q, k, v, log_alpha, beta, S, N, H, dk, dv,
                                     dtype == KDA_DTYPE_BF16, (flags & KDA_FLAG_NO_L2NORM) ? 0 : 1,
                                     (flags & KDA_FLAG_SCALAR_GATE) ? 1 : 0, kEps,
                                     out_gate ? out_gate->gate : nullptr,
                                     out_gate ? out_gate->weight : nullptr, out_gate ? out_gate->eps : 0.f,
                                     &cv, o, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
