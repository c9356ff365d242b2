// kda_decode.cu -- single-token KDA decode step, state updated in place.
//
// "[Kimi-2] Kimi Linear：用 KDA 重写长上下文注意力" §5 (recurrent decode:
// S_(t-1) + current token -> S_t + output) applied to the §3 update
//     S~ = Diag(alpha) S,  u = beta (v - S~^T k),  S_t = S~ + k u^T,
//     o  = S_t^T q = S~^T q + (k . q) u
// with q, k L2-normalised (§6.2).
//
// The step is HBM-bound: per (sequence, head) it reads and writes the fp32
// d_k x d_v state (64 KiB each way at d = 128) and touches < 1.5 KiB of
// token inputs. CTAs of 256 threads own the state columns of one (sequence,
// head): all d_v of them, or (the plain step at d_v = 128) half of them, since
// the columns are independent (each needs its own column sums and k . q,
// which every CTA forms). Two CTAs per state halve the registers a thread
// needs, so twice as many CTAs (and bytes in flight) fit on an SM. Thread (row
// group, column group) keeps R rows x 4 contiguous columns of S in registers,
// so every warp access is a coalesced 16-byte-per-lane sweep (read once,
// evict-first; written once, streaming). The two column sums over d_k (S~^T k
// and S~^T q) are per-thread partial sums finished through shared memory;
// nothing else touches HBM.
//
// Optionally the layer's causal short convolution + Swish (§6.1) is applied to
// q, k, v as they are loaded: the step's raw projection and the channel's last
// W-1 raw inputs (the convolution state, read and then shifted in place by the
// same thread) give z = sum_j w[c][j] x_{t-W+1+j}, and the input becomes
// z sigmoid(z) (then q, k are L2-normalised as before).
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kDecodeThreads = 256;
constexpr int kMaxConvW = kDecodeMaxConvWidth;

// Short convolution + Swish of a lane's NM channels cbase + lane + 32 m of
// sequence s (C channels per state row): every load is issued first (the
// step's input, the W-1 state entries, the W taps), then z and Swish, then the
// state is written back shifted by one (the same thread read it: in place is safe).
template <typename T, int NM>
__device__ __forceinline__ void conv_swish_lane(const T *__restrict__ xrow, int W, const float *__restrict__ w,
                                                const void *sin_, void *sout_, int s, int C, int cbase,
                                                int lane, float (&out)[NM]) {
    const T *sin = static_cast<const T *>(sin_);
    T *sout = static_cast<T *>(sout_);
    float xv[NM], h[NM][kMaxConvW - 1], wv[NM][kMaxConvW];
#pragma unroll
    for (int m = 0; m < NM; ++m) {
        const int c = cbase + lane + 32 * m;
        xv[m] = IO<T>::ld(xrow + lane + 32 * m);
#pragma unroll
        for (int j = 0; j < kMaxConvW - 1; ++j)
            h[m][j] = (j < W - 1 && sin) ? IO<T>::ld(sin + ((size_t)s * (W - 1) + j) * C + c) : 0.f;
#pragma unroll
        for (int j = 0; j < kMaxConvW; ++j) wv[m][j] = j < W ? w[(size_t)c * W + j] : 0.f;
    }
#pragma unroll
    for (int m = 0; m < NM; ++m) {
        float z = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxConvW; ++j) {
            if (j < W - 1) z = fmaf(wv[m][j], h[m][j < kMaxConvW - 1 ? j : 0], z);
            else if (j == W - 1) z = fmaf(wv[m][j], xv[m], z);
        }
        out[m] = swish(z);
    }
    if (sout) {
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            const int c = cbase + lane + 32 * m;
#pragma unroll
            for (int j = 0; j < kMaxConvW - 1; ++j) {
                if (j < W - 1) {
                    const float nv = (j + 1 < W - 1) ? h[m][j + 1 < kMaxConvW - 1 ? j + 1 : 0] : xv[m];
                    IO<T>::st(sout + ((size_t)s * (W - 1) + j) * C + c, nv);
                }
            }
        }
    }
}

template <int DK, int DV, typename T, bool CONV, int SPLIT = 1>
__global__ void __launch_bounds__(kDecodeThreads, 2 * SPLIT)
decode_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
              const float *__restrict__ log_alpha, const float *__restrict__ beta,
              float *__restrict__ S, T *__restrict__ o, int l2norm, int la_scalar, float eps,
              const T *__restrict__ og_gate, const float *__restrict__ og_w, float og_eps, DecodeConv cv,
              int H) {
    // SPLIT > 1: the unit's state columns are divided among SPLIT CTAs (columns are
    // independent: each needs only its own column sums, and k . q, which every CTA forms).
    constexpr int DVC = DV / SPLIT;           // state columns of this CTA
    constexpr int CG = DVC / 4;               // 16-byte column groups per state row
    constexpr int RPP = kDecodeThreads / CG;  // state rows covered per pass
    constexpr int R = DK / RPP;               // rows held per thread
    static_assert(R * RPP == DK && CG * 4 == DVC, "shape");
    static_assert(SPLIT == 1 || !CONV, "the fused convolution runs unsplit");

    __shared__ float s_q[DK], s_k[DK], s_a[DK], s_v[DV], s_u[DV];
    __shared__ float s_red[RPP][CG][8];
    __shared__ float s_misc[2];  // beta, k.q
    __shared__ float s_o[DV], s_gss[DV / 32];  // fused output step: o, per-warp sums of o^2

    const int unit = blockIdx.x / SPLIT;  // sequence * H + head
    const int c0 = (blockIdx.x % SPLIT) * DVC;  // first state column of this CTA
    const int tid = threadIdx.x;
    const int cg = tid % CG, r0 = tid / CG;
    float *Su = S + (size_t)unit * DK * DV + c0;

    // 1. Issue the whole state tile load first (R independent 16-byte loads).
    float4 s[R];
#pragma unroll
    for (int m = 0; m < R; ++m)
        s[m] = __ldcs(reinterpret_cast<const float4 *>(Su + (size_t)(r0 + m * RPP) * DV) + cg);

    // 2. Token inputs while the state is in flight: warp 0 normalises q, k and
    //    forms k.q; warp 1 exponentiates the gate; warp 2 stages v and beta.
    const int warp = tid >> 5, lane = tid & 31;
    const int seq = unit / H, hc = unit % H;  // for the convolution state
    if constexpr (CONV) {
        // 2'. With the short convolution: warp 0 q, warp 3 k, warp 2 v and beta (each
        //     convolved or as is), warp 1 the gate; then warp 0 normalises q, k.
        if (warp == 0 || warp == 3) {
            const bool isq = warp == 0;
            const T *x = isq ? q : k;
            const int Wc = isq ? cv.W[0] : cv.W[1];
            float xs[DK / 32];
            if (Wc) {
                conv_swish_lane<T, DK / 32>(x + (size_t)unit * DK, Wc, isq ? cv.w[0] : cv.w[1],
                                            isq ? cv.state_in[0] : cv.state_in[1],
                                            isq ? cv.state_out[0] : cv.state_out[1], seq, H * DK, hc * DK, lane, xs);
            } else {
#pragma unroll
                for (int m = 0; m < DK / 32; ++m) xs[m] = IO<T>::ld(x + (size_t)unit * DK + lane + 32 * m);
            }
            float *dst = warp == 0 ? s_q : s_k;
#pragma unroll
            for (int m = 0; m < DK / 32; ++m) dst[lane + 32 * m] = xs[m];
        } else if (warp == 1) {
            for (int i = lane; i < DK; i += 32)
                s_a[i] = expf(la_scalar ? log_alpha[unit] : log_alpha[(size_t)unit * DK + i]);
        } else if (warp == 2) {
            float vs[DV / 32];
            if (cv.W[2]) {
                conv_swish_lane<T, DV / 32>(v + (size_t)unit * DV, cv.W[2], cv.w[2], cv.state_in[2], cv.state_out[2],
                                            seq, H * DV, hc * DV, lane, vs);
            } else {
#pragma unroll
                for (int m = 0; m < DV / 32; ++m) vs[m] = IO<T>::ld(v + (size_t)unit * DV + lane + 32 * m);
            }
#pragma unroll
            for (int m = 0; m < DV / 32; ++m) s_v[lane + 32 * m] = vs[m];
            if (lane == 0) s_misc[0] = beta[unit];
        }
        __syncthreads();
        if (warp == 0) {
            float qq = 0.f, kk = 0.f, qk = 0.f;
#pragma unroll
            for (int m = 0; m < DK / 32; ++m) {
                const float a = s_q[lane + 32 * m], b = s_k[lane + 32 * m];
                qq += a * a;
                kk += b * b;
                qk += a * b;
            }
#pragma unroll
            for (int off = 16; off; off >>= 1) {
                qq += __shfl_xor_sync(0xffffffffu, qq, off);
                kk += __shfl_xor_sync(0xffffffffu, kk, off);
                qk += __shfl_xor_sync(0xffffffffu, qk, off);
            }
            float iq = 1.f, ik = 1.f;
            if (l2norm) {
                iq = 1.f / fmaxf(sqrtf(qq), eps);
                ik = 1.f / fmaxf(sqrtf(kk), eps);
            }
#pragma unroll
            for (int m = 0; m < DK / 32; ++m) {
                s_q[lane + 32 * m] *= iq;
                s_k[lane + 32 * m] *= ik;
            }
            if (lane == 0) s_misc[1] = qk * iq * ik;
        }
    } else {
      if (warp == 0) {
        float qq = 0.f, kk = 0.f, qk = 0.f;
        float qv[DK / 32], kv[DK / 32];
#pragma unroll
        for (int m = 0; m < DK / 32; ++m) {
            qv[m] = IO<T>::ld(q + (size_t)unit * DK + lane + 32 * m);
            kv[m] = IO<T>::ld(k + (size_t)unit * DK + lane + 32 * m);
            qq += qv[m] * qv[m];
            kk += kv[m] * kv[m];
            qk += qv[m] * kv[m];
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            qq += __shfl_xor_sync(0xffffffffu, qq, off);
            kk += __shfl_xor_sync(0xffffffffu, kk, off);
            qk += __shfl_xor_sync(0xffffffffu, qk, off);
        }
        float iq = 1.f, ik = 1.f;
        if (l2norm) {
            iq = 1.f / fmaxf(sqrtf(qq), eps);
            ik = 1.f / fmaxf(sqrtf(kk), eps);
        }
#pragma unroll
        for (int m = 0; m < DK / 32; ++m) {
            s_q[lane + 32 * m] = qv[m] * iq;
            s_k[lane + 32 * m] = kv[m] * ik;
        }
        if (lane == 0) s_misc[1] = qk * iq * ik;
      } else if (warp == 1) {
        for (int i = lane; i < DK; i += 32)
            s_a[i] = expf(la_scalar ? log_alpha[unit] : log_alpha[(size_t)unit * DK + i]);
      } else if (warp == 2) {
        for (int j = lane; j < DVC; j += 32) s_v[j] = IO<T>::ld(v + (size_t)unit * DV + c0 + j);
        if (lane == 0) s_misc[0] = beta[unit];
      }
    }
    __syncthreads();

    // 3. Partial column sums of S~^T k and S~^T q over this thread's rows.
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f), z = y;
#pragma unroll
    for (int m = 0; m < R; ++m) {
        const int i = r0 + m * RPP;
        const float a = s_a[i], ka = a * s_k[i], qa = a * s_q[i];
        y.x += ka * s[m].x; y.y += ka * s[m].y; y.z += ka * s[m].z; y.w += ka * s[m].w;
        z.x += qa * s[m].x; z.y += qa * s[m].y; z.z += qa * s[m].z; z.w += qa * s[m].w;
    }
    *reinterpret_cast<float4 *>(&s_red[r0][cg][0]) = y;
    *reinterpret_cast<float4 *>(&s_red[r0][cg][4]) = z;
    __syncthreads();

    // 4. Finish the sums per column: u = beta (v - S~^T k), o = S~^T q + (k.q) u.
    if (tid < DVC) {
        const int j = tid, g = j >> 2, c = j & 3;
        float yy = 0.f, zz = 0.f;
#pragma unroll
        for (int r = 0; r < RPP; ++r) {
            yy += s_red[r][g][c];
            zz += s_red[r][g][4 + c];
        }
        const float u = s_misc[0] * (s_v[j] - yy);
        s_u[j] = u;
        const float oj = zz + s_misc[1] * u;
        if (og_gate) {
            // fused output step: keep o_j for the head's RMSNorm (sum of squares per warp)
            s_o[j] = oj;
            float ss = oj * oj;
#pragma unroll
            for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            if ((j & 31) == 0) s_gss[j >> 5] = ss;
        } else {
            IO<T>::st(o + (size_t)unit * DV + c0 + j, oj);
        }
    }
    __syncthreads();
    // 4b. Fused output step: o <- o / sqrt(mean(o^2) + eps) * w * sigmoid(gate).
    if (og_gate && tid < DV) {
        const int j = tid;
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < DV / 32; ++w) tot += s_gss[w];
        const float gv = IO<T>::ld(og_gate + (size_t)unit * DV + j);
        const float y = s_o[j] * rsqrtf(tot / DV + og_eps) * og_w[j] / (1.f + __expf(-gv));
        IO<T>::st(o + (size_t)unit * DV + j, y);
    }

    // 5. S_t = Diag(alpha) S + k u^T, written back once.
    const float4 u4 = *reinterpret_cast<const float4 *>(&s_u[4 * cg]);
#pragma unroll
    for (int m = 0; m < R; ++m) {
        const int i = r0 + m * RPP;
        const float a = s_a[i], kk = s_k[i];
        float4 w;
        w.x = a * s[m].x + kk * u4.x;
        w.y = a * s[m].y + kk * u4.y;
        w.z = a * s[m].z + kk * u4.z;
        w.w = a * s[m].w + kk * u4.w;
        __stcs(reinterpret_cast<float4 *>(Su + (size_t)i * DV) + cg, w);
    }
}

template <int DK, int DV, typename T>
cudaError_t launch(const void *q, const void *k, const void *v, const float *la, const float *beta,
                   float *S, int N, int H, int l2norm, int la_scalar, float eps, const void *og_gate,
                   const float *og_w, float og_eps, const DecodeConv &cv, void *o, cudaStream_t st) {
    const unsigned units = (unsigned)N * (unsigned)H;
    if (cv.W[0] | cv.W[1] | cv.W[2])
        decode_kernel<DK, DV, T, true><<<units, kDecodeThreads, 0, st>>>(
            (const T *)q, (const T *)k, (const T *)v, la, beta, S, (T *)o, l2norm, la_scalar, eps,
            (const T *)og_gate, og_w, og_eps, cv, H);
    else if (og_gate == nullptr && DV == 128)
        decode_kernel<DK, DV, T, false, 2><<<2 * units, kDecodeThreads, 0, st>>>(
            (const T *)q, (const T *)k, (const T *)v, la, beta, S, (T *)o, l2norm, la_scalar, eps,
            (const T *)og_gate, og_w, og_eps, cv, H);
    else
        decode_kernel<DK, DV, T, false><<<units, kDecodeThreads, 0, st>>>(
            (const T *)q, (const T *)k, (const T *)v, la, beta, S, (T *)o, l2norm, la_scalar, eps,
            (const T *)og_gate, og_w, og_eps, cv, H);
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch(const void *q, const void *k, const void *v, const float *la,
                     const float *beta, float *S, int N, int H, int dk, int dv, int l2norm,
                     int la_scalar, float eps, const void *og, const float *ow, float oe, const DecodeConv &cv,
                     void *o, cudaStream_t st) {
    if (dk == 128 && dv == 128) return launch<128, 128, T>(q, k, v, la, beta, S, N, H, l2norm, la_scalar, eps, og, ow, oe, cv, o, st);
    if (dk == 128 && dv == 64) return launch<128, 64, T>(q, k, v, la, beta, S, N, H, l2norm, la_scalar, eps, og, ow, oe, cv, o, st);
    if (dk == 64 && dv == 128) return launch<64, 128, T>(q, k, v, la, beta, S, N, H, l2norm, la_scalar, eps, og, ow, oe, cv, o, st);
    if (dk == 64 && dv == 64) return launch<64, 64, T>(q, k, v, la, beta, S, N, H, l2norm, la_scalar, eps, og, ow, oe, cv, o, st);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t decode_step(const void *q, const void *k, const void *v, const float *la,
                        const float *beta, float *S, int N, int H, int dk, int dv, bool bf16,
                        int l2norm, int la_scalar, float eps, const void *og_gate, const float *og_w,
                        float og_eps, const DecodeConv *conv, void *o, cudaStream_t st) {
    DecodeConv cv{};
    if (conv) cv = *conv;
    if (bf16)
        return dispatch<__nv_bfloat16>(q, k, v, la, beta, S, N, H, dk, dv, l2norm, la_scalar, eps, og_gate, og_w,
                                       og_eps, cv, o, st);
    return dispatch<float>(q, k, v, la, beta, S, N, H, dk, dv, l2norm, la_scalar, eps, og_gate, og_w, og_eps, cv,
                           o, st);
}

}  // namespace kda
