// kda_internal.cuh -- declarations shared by the libkda translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "kda.h"

namespace kda {

constexpr int kChunk = 64;  // chunk length C of the chunkwise prefill

// Swish of the short convolution ("[Kimi-2] Kimi Linear" §6.1): z sigmoid(z) =
// z / (1 + 2^(-z log2 e)) with the hardware's approximate 2^x and reciprocal (PTX
// ex2.approx / rcp.approx, relative errors about 2^-22 and 2^-23) and every other
// operation an explicit round-to-nearest one, so that each convolution kernel (and the
// pair form in kda_tc.cuh) gets the same bits. A large negative z gives e = inf and -0.
constexpr float kSwishNegLog2e = -1.4426950408889634f;
__device__ __forceinline__ float swish(float z) {
    float e, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(__fmul_rn(z, kSwishNegLog2e)));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(__fadd_rn(1.f, e)));
    return __fmul_rn(z, r);
}

// Element I/O for the two input/output dtypes; arithmetic is always fp32.
template <typename T> struct IO;
template <> struct IO<float> {
    static __device__ __forceinline__ float ld(const float *p) { return *p; }
    static __device__ __forceinline__ void st(float *p, float x) { *p = x; }
};
template <> struct IO<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

// Bounds of sequence s in the packed token axis (cu == nullptr: one sequence).
__device__ __forceinline__ void seq_bounds(const int32_t *cu, int s, int64_t total, int64_t &bos,
                                           int64_t &eos) {
    if (cu) {
        bos = cu[s];
        eos = cu[s + 1];
    } else {
        bos = 0;
        eos = total;
    }
}

// Parameters of a prefill call (the CUDA-core path runs it in waves: chunk
// indices [j0, j0 + nw) of every sequence per wave).
struct PrefillArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    const int32_t *cu;
    int64_t total;
    int N, H, dk, dv;
    int l2norm;
    int la_scalar;  // log_alpha is [T][H] (one gate per token and head)
    float eps;
    // fused output step (og_gate == nullptr: none): o <- RMSNorm(o) * og_w * sigmoid(og_gate)
    const void *og_gate;
    const float *og_w;
    float og_eps;
    void *o;
    float *S_T;
    // causal short convolution + Swish fused into the loads of q, k, v (index 0, 1, 2;
    // tensor-core path): window (0: the input is used as it is), taps [H * d][W] fp32,
    // initial states [N][W - 1][H * d] in the io dtype (nullptr: zeros)
    int conv_W[3];
    const float *conv_w[3];
    const void *conv_state[3];
    // workspace
    float *state;      // running state between waves ([N][H][dk][dv]) or nullptr
    char *slots;       // per-chunk slots of this wave
    size_t slot_bytes; // bytes per (chunk, seq, head) slot
};

// fp32 CUDA-core path (exact arithmetic; any supported shape).
size_t simt_slot_bytes(int dk);
cudaError_t simt_prefill_wave(const PrefillArgs &a, int j0, int nw, bool bf16, cudaStream_t st);

// tensor-core path (bf16, d_k = d_v = 128): one planning kernel and one
// persistent cooperative kernel. The (sequence, head) units are dealt to
// `ns` <= kTcMaxStreams streams, each scanned by two CTAs and fed through a
// ring of R slots in the workspace; R follows from the workspace size.
constexpr int kTcMaxStreams = 32;
size_t tc_workspace_bytes(long long NH, int ns, int R);   // NH = N * H units
int tc_ring_slots(long long NH, int ns, size_t bytes);   // R for a workspace (capped)
int tc_max_ring();
cudaError_t tc_prefill(const PrefillArgs &a, char *ws, size_t ws_bytes, int ns, int *err, cudaStream_t st);
// Bound of the tensor-core prefill's waits between CTAs (ns), for calls enqueued from now on.
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
uint64_t tc_set_wait_limit(uint64_t ns);

// Device address of a __device__ variable in the current device's context,
// resolved with cudaGetSymbolAddress on the first use in that context (with the
// device current) and cached per device; a new context on the device (after
// cudaDeviceReset) resolves it again. nullptr if it cannot be resolved.
struct SymbolCache {
    static constexpr int kMaxDevices = 64;
    std::mutex mu;
    unsigned long long ctx[kMaxDevices] = {};
    void *addr[kMaxDevices] = {};
};
void *symbol_address(const void *symbol, SymbolCache &cache);

// Address of this device's error word (set by kernels whose bounded waits ran
// out), or nullptr if it cannot be resolved.
int *device_error_word();

// Causal short convolution + Swish of one projection x [T][C] (C % 8 == 0).
struct ShortConvArgs {
    const void *x;
    void *y;
    const float *w;        // [C][W]
    const void *state_in;  // [N][W-1][C] or nullptr (zeros)
    void *state_out;       // [N][W-1][C] or nullptr
    const int32_t *cu;     // [N+1] or nullptr (one sequence)
    int N;
    int64_t total;
    int C, W;
};
cudaError_t short_conv_swish(const ShortConvArgs &a, bool bf16, cudaStream_t st);
// Only the final states (state_out from x and state_in; a.y unused).
cudaError_t short_conv_state(const ShortConvArgs &a, bool bf16, cudaStream_t st);
constexpr int kPrefillMaxConvWidth = 4;  // KDA_PREFILL_MAX_CONV_WIDTH
int short_conv_launches(int W, bool state_out, int64_t total);

constexpr int kDecodeMaxConvWidth = 4;  // widest window the decode step fuses
// The same convolution fused into a decode step's loads of q, k, v (index 0, 1, 2):
// W[i] == 0 leaves that input as it is. States are [N][W-1][H * d].
struct DecodeConv {
    int W[3];
    const float *w[3];
    const void *state_in[3];
    void *state_out[3];
};

// Backward of the chunkwise prefill (fp32 CUDA cores; gradients fp32).
struct BackwardArgs {
    const void *q, *k, *v, *dout;  // io dtype
    const float *log_alpha, *beta, *S0, *dS_T;
    const int32_t *cu;
    int64_t total;
    int N, H, dk, dv;
    int l2norm;
    int la_scalar;  // log_alpha and dlog_alpha are [T][H]: one gate per (token, head)
    float eps;
    float *dq, *dk_out, *dv_out, *dlog_alpha, *dbeta, *dS0;
    void *ws;
    int *err;
};
int64_t backward_slots_per_head(int N, int64_t total);  // chunk slots per head (>= the chunks)
size_t backward_workspace_bytes(int N, int H, int64_t total, int dk, int dv);
cudaError_t backward(const BackwardArgs &b, bool bf16, cudaStream_t st);

// decode step
cudaError_t decode_step(const void *q, const void *k, const void *v, const float *la,
                        const float *beta, float *S, int N, int H, int dk, int dv, bool bf16,
                        int l2norm, int la_scalar, float eps, const void *og_gate, const float *og_w,
                        float og_eps, const DecodeConv *conv, void *o, cudaStream_t st);
// fp32 CUDA-core path: the output step applied to o in place after the prefill.
cudaError_t simt_output_gate(const PrefillArgs &a, bool bf16, cudaStream_t st);

}  // namespace kda
