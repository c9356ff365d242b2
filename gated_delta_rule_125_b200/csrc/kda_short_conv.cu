// kda_short_conv.cu -- causal short convolution + Swish over packed sequences.
//
// "[Kimi-2] Kimi Linear：用 KDA 重写长上下文注意力" §6 and §6.1 (and "Kimi Delta
// Attention：把遗忘门做到每个通道", the pre-processing of q and k): each channel c
// of a projection x [T][C] is convolved over the tokens of its own sequence,
//     z_t[c] = sum_{j<W} w[c][j] x_{t-W+1+j}[c],   y_t[c] = z_t[c] sigmoid(z_t[c]),
// positions before a sequence's first token reading its initial state (W-1 raw
// inputs, oldest first) or zero.
//
// HBM-bound streaming: a thread owns 8 consecutive channels (one 16-byte bf16
// vector) of kTile consecutive tokens. A tile inside one sequence issues all
// its kTile + W - 1 row loads before the first use (kept as loaded, unpacked
// into a sliding W-deep window as they are used); each input is read from HBM
// once (the W-1 halo rows are the previous tile's last rows, L2 hits). A tile
// that meets a sequence boundary takes the token-by-token path. Consecutive
// threads take consecutive channel vectors of the same tokens: every warp
// access is a coalesced sweep.
// A second launch writes each sequence's last W-1 inputs (the state a decode
// step continues from); one thread per (sequence, channel vector) reads all it
// needs before it writes, so the output state may alias the input state.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kConvThreads = 256;
constexpr int kTile = 8;  // tokens per thread

template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
    using Raw = uint4;  // 8 channels as loaded
    static __device__ __forceinline__ Raw ldraw(const __nv_bfloat16 *p) { return *reinterpret_cast<const uint4 *>(p); }
    static __device__ __forceinline__ void unpack(const Raw &u, float (&x)[8]) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    static __device__ __forceinline__ void ld(const __nv_bfloat16 *p, float (&x)[8]) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, const float (&x)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};
template <> struct Vec8<float> {
    struct Raw {
        float4 a, b;
    };
    static __device__ __forceinline__ Raw ldraw(const float *p) {
        return Raw{reinterpret_cast<const float4 *>(p)[0], reinterpret_cast<const float4 *>(p)[1]};
    }
    static __device__ __forceinline__ void unpack(const Raw &r, float (&x)[8]) {
        x[0] = r.a.x; x[1] = r.a.y; x[2] = r.a.z; x[3] = r.a.w;
        x[4] = r.b.x; x[5] = r.b.y; x[6] = r.b.z; x[7] = r.b.w;
    }
    static __device__ __forceinline__ void ld(const float *p, float (&x)[8]) {
        const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
    static __device__ __forceinline__ void st(float *p, const float (&x)[8]) {
        reinterpret_cast<float4 *>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
        reinterpret_cast<float4 *>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
    }
};

// Index of the sequence holding token t: the last s with cu[s] <= t.
__device__ __forceinline__ int seq_of(const int32_t *cu, int N, int64_t t) {
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Raw input of position `pos` of sequence s (pos < 0: from the initial state).
template <int W, typename T>
__device__ __forceinline__ void ld_hist(const T *x, const T *state_in, int64_t bos, int64_t pos, int s,
                                        int C, int c0, float (&v)[8]) {
    if (pos >= 0) {
        Vec8<T>::ld(x + (size_t)(bos + pos) * C + c0, v);
    } else if (state_in) {
        Vec8<T>::ld(state_in + ((size_t)s * (W - 1) + (W - 1 + pos)) * C + c0, v);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
}

template <int W, typename T>
__global__ void __launch_bounds__(kConvThreads)
conv_kernel(const T *__restrict__ x, T *__restrict__ y, const float *__restrict__ w, const T *state_in,
            const int32_t *__restrict__ cu, int N, int64_t total, int C) {
    const int nv = C / 8;
    const int64_t g = (int64_t)blockIdx.x * kConvThreads + threadIdx.x;
    const int64_t tile = g / nv;
    const int c0 = (int)(g % nv) * 8;
    const int64_t t0 = tile * kTile;
    if (t0 >= total) return;
    const int64_t t1 = t0 + kTile < total ? t0 + kTile : total;

    float wt[8][W];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < W; ++j) wt[i][j] = w[(size_t)(c0 + i) * W + j];

    int s = cu ? seq_of(cu, N, t0) : 0;
    int64_t bos = cu ? cu[s] : 0, eos = cu ? cu[s + 1] : total;
    if (t0 - bos >= W - 1 && t0 + kTile <= eos) {
        // the whole window of the tile lies in one sequence: every row load first
        typename Vec8<T>::Raw raw[kTile + W - 1];
#pragma unroll
        for (int r = 0; r < kTile + W - 1; ++r) raw[r] = Vec8<T>::ldraw(x + (size_t)(t0 - (W - 1) + r) * C + c0);
        float win[W][8];
#pragma unroll
        for (int j = 0; j < W - 1; ++j) Vec8<T>::unpack(raw[j], win[j]);
#pragma unroll
        for (int r = 0; r < kTile; ++r) {
            Vec8<T>::unpack(raw[r + W - 1], win[W - 1]);
            float out[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float z = 0.f;
#pragma unroll
                for (int j = 0; j < W; ++j) z = fmaf(wt[i][j], win[j][i], z);
                out[i] = swish(z);
            }
            Vec8<T>::st(y + (size_t)(t0 + r) * C + c0, out);
#pragma unroll
            for (int j = 0; j < W - 1; ++j)
#pragma unroll
                for (int i = 0; i < 8; ++i) win[j][i] = win[j + 1][i];
        }
        return;
    }
    float win[W][8];  // win[W-1] is the current token, win[0] the oldest
    auto fill = [&](int64_t t) {  // window positions t-W+1 .. t-1 of t's sequence
#pragma unroll
        for (int j = 0; j < W - 1; ++j) ld_hist<W, T>(x, state_in, bos, t - bos - (W - 1) + j, s, C, c0, win[j]);
    };
    fill(t0);
    for (int64_t t = t0; t < t1; ++t) {
        if (t == eos) {  // the tile runs into the next sequence (skipping empty ones)
            do {
                ++s;
                bos = cu[s];
                eos = cu[s + 1];
            } while (eos == bos);
            fill(t);
        }
        Vec8<T>::ld(x + (size_t)t * C + c0, win[W - 1]);
        float out[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float z = 0.f;
#pragma unroll
            for (int j = 0; j < W; ++j) z = fmaf(wt[i][j], win[j][i], z);
            out[i] = swish(z);
        }
        Vec8<T>::st(y + (size_t)t * C + c0, out);
#pragma unroll
        for (int j = 0; j < W - 1; ++j)
#pragma unroll
            for (int i = 0; i < 8; ++i) win[j][i] = win[j + 1][i];
    }
}

// state_out[s][j] = raw input of position len_s - (W-1) + j of sequence s.
template <int W, typename T>
__global__ void __launch_bounds__(kConvThreads)
conv_state_kernel(const T *__restrict__ x, const T *state_in, T *state_out, const int32_t *__restrict__ cu,
                  int N, int64_t total, int C) {
    if constexpr (W > 1) {
        const int nv = C / 8;
        const int64_t g = (int64_t)blockIdx.x * kConvThreads + threadIdx.x;
        if (g >= (int64_t)N * nv) return;
        const int s = (int)(g / nv), c0 = (int)(g % nv) * 8;
        const int64_t bos = cu ? cu[s] : 0, eos = cu ? cu[s + 1] : total, len = eos - bos;
        float v[W - 1][8];
#pragma unroll
        for (int j = 0; j < W - 1; ++j) ld_hist<W, T>(x, state_in, bos, len - (W - 1) + j, s, C, c0, v[j]);
#pragma unroll
        for (int j = 0; j < W - 1; ++j) Vec8<T>::st(state_out + ((size_t)s * (W - 1) + j) * C + c0, v[j]);
    }
}

template <int W, typename T>
cudaError_t launch_state(const ShortConvArgs &a, cudaStream_t st) {
    if (W > 1 && a.state_out) {
        const int64_t threads = (int64_t)a.N * (a.C / 8);
        conv_state_kernel<W, T><<<(unsigned)((threads + kConvThreads - 1) / kConvThreads), kConvThreads, 0, st>>>(
            static_cast<const T *>(a.x), static_cast<const T *>(a.state_in), static_cast<T *>(a.state_out), a.cu,
            a.N, a.total, a.C);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

template <int W, typename T>
cudaError_t launch_w(const ShortConvArgs &a, cudaStream_t st) {
    const T *x = static_cast<const T *>(a.x);
    const T *sin = static_cast<const T *>(a.state_in);
    const int nv = a.C / 8;
    if (a.total > 0) {
        const int64_t threads = (a.total + kTile - 1) / kTile * nv;
        conv_kernel<W, T><<<(unsigned)((threads + kConvThreads - 1) / kConvThreads), kConvThreads, 0, st>>>(
            x, static_cast<T *>(a.y), a.w, sin, a.cu, a.N, a.total, a.C);
        if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return e;
    }
    if (W > 1 && a.state_out) {
        const int64_t threads = (int64_t)a.N * nv;
        conv_state_kernel<W, T><<<(unsigned)((threads + kConvThreads - 1) / kConvThreads), kConvThreads, 0, st>>>(
            x, sin, static_cast<T *>(a.state_out), a.cu, a.N, a.total, a.C);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t launch_t(const ShortConvArgs &a, cudaStream_t st) {
    switch (a.W) {
    case 1: return launch_w<1, T>(a, st);
    case 2: return launch_w<2, T>(a, st);
    case 3: return launch_w<3, T>(a, st);
    case 4: return launch_w<4, T>(a, st);
    case 5: return launch_w<5, T>(a, st);
    case 6: return launch_w<6, T>(a, st);
    case 7: return launch_w<7, T>(a, st);
    case 8: return launch_w<8, T>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_state_t(const ShortConvArgs &a, cudaStream_t st) {
    switch (a.W) {
    case 1: return launch_state<1, T>(a, st);
    case 2: return launch_state<2, T>(a, st);
    case 3: return launch_state<3, T>(a, st);
    case 4: return launch_state<4, T>(a, st);
    case 5: return launch_state<5, T>(a, st);
    case 6: return launch_state<6, T>(a, st);
    case 7: return launch_state<7, T>(a, st);
    case 8: return launch_state<8, T>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t short_conv_swish(const ShortConvArgs &a, bool bf16, cudaStream_t st) {
    return bf16 ? launch_t<__nv_bfloat16>(a, st) : launch_t<float>(a, st);
}

cudaError_t short_conv_state(const ShortConvArgs &a, bool bf16, cudaStream_t st) {
    return bf16 ? launch_state_t<__nv_bfloat16>(a, st) : launch_state_t<float>(a, st);
}

int short_conv_launches(int W, bool state_out, int64_t total) {
    return (total > 0 ? 1 : 0) + ((W > 1 && state_out) ? 1 : 0);
}

}  // namespace kda
