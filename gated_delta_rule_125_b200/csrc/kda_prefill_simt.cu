// kda_prefill_simt.cu -- chunkwise KDA prefill in fp32 on the CUDA cores.
//
// The exact path: it serves fp32 inputs (whose tolerance rules out bf16/tf32
// tensor-core operands) and KDA_FLAG_EXACT, for d_k, d_v in {64, 128}.
//
// Chunkwise form ("[Kimi-2] Kimi Linear：用 KDA 重写长上下文注意力" §5: the UT
// transform turns a chunk's rank-1 transitions into dense products; the output
// adds an inter-chunk read of the entry state and an intra-chunk read of
// earlier tokens' pseudo-values). Per chunk of C = 64 rows with entry state S
// and G = cumulative sum of log_alpha over the chunk's rows:
//   A[r][i] = sum_c k_rc k_ic e^{G_rc - G_ic}  (i < r),   P[r][i] same with q_r (i <= r)
//   T  = (I + Diag(beta) A)^{-1} Diag(beta),   W = T (K*e^G)
//   U  = T V - W S
//   O  = (Q*e^G) S + P U
//   S' = Diag(e^{G_last}) S + (K*e^{G_last - G})^T U
//
// Two kernels per wave of chunks:
//  * prep (one CTA per chunk x head, all chunks of the wave in parallel):
//    L2 norm, G, A and P with element-wise exponents (never exp(+G), so any
//    decay strength is safe), the triangular solve for T, and W, Q*e^G,
//    K*e^{G_last-G}, P, T, e^{G_last} written to a workspace slot;
//  * scan (one CTA per sequence x head x 32-column tile of d_v, chunks in
//    order): U, O and S' from the slot, V and the running state.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int C = kChunk;
constexpr int kThreads = 256;
constexpr int kDvTile = 32;

// Workspace slot (fp32), one per (chunk, sequence, head):
//   Wt  [DK][C]  W transposed          Qgt [DK][C]  (Q*e^G) transposed
//   Kd  [C][DK]  K*e^{G_last - G}      Tt  [C][C]   T transposed
//   Pt  [C][C]   P transposed          D   [DK]     e^{G_last}
template <int DK> struct Slot {
    static constexpr int WT = 0;
    static constexpr int QGT = WT + DK * C;
    static constexpr int KD = QGT + DK * C;
    static constexpr int TT = KD + C * DK;
    static constexpr int PT = TT + C * C;
    static constexpr int D = PT + C * C;
    static constexpr int FLOATS = D + DK;
    static constexpr size_t BYTES = ((size_t)FLOATS * 4 + 255) / 256 * 256;
};

template <int DK, typename T>
__global__ void __launch_bounds__(kThreads)
prep_kernel(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ la,
            const float *__restrict__ beta, const int32_t *__restrict__ cu, int64_t total, int H,
            int N, int j0, int l2norm, int la_scalar, float eps, char *__restrict__ slots, size_t slot_bytes) {
    constexpr int LD = DK + 1;  // padded row stride: rows i, i+1 fall in different banks
    const int jl = blockIdx.x, s = blockIdx.y, h = blockIdx.z;
    int64_t bos, eos;
    seq_bounds(cu, s, total, bos, eos);
    const int64_t j = (int64_t)j0 + jl;
    if (j * C >= eos - bos) return;
    const int n = (int)(eos - bos - j * C < C ? eos - bos - j * C : C);
    const int64_t t0 = bos + j * C;
    float *slot = reinterpret_cast<float *>(slots + ((size_t)jl * N + s) * H * slot_bytes + (size_t)h * slot_bytes);

    extern __shared__ float sm[];
    float *sK = sm;             // [C][LD]  k (normalised), later K*e^G
    float *sQ = sK + C * LD;    // [C][LD]  q (normalised)
    float *sG = sQ + C * LD;    // [C][LD]  log_alpha, then G
    float *sA = sG + C * LD;    // [C][C+1]
    float *sP = sA + C * (C + 1);
    float *sT = sP + C * (C + 1);
    float *sB = sT + C * (C + 1);  // [C] beta
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // 1. Load the chunk; rows past the sequence end are zero (k = q = 0,
    //    log_alpha = 0, beta = 0), which makes them inert in every product.
    for (int idx = tid; idx < C * DK; idx += kThreads) {
        const int r = idx / DK, c = idx % DK;
        float kv = 0.f, qv = 0.f, lv = 0.f;
        if (r < n) {
            const size_t off = ((size_t)(t0 + r) * H + h) * DK + c;
            kv = IO<T>::ld(k + off);
            qv = IO<T>::ld(q + off);
            lv = la_scalar ? la[(size_t)(t0 + r) * H + h] : la[off];
        }
        sK[r * LD + c] = kv;
        sQ[r * LD + c] = qv;
        sG[r * LD + c] = lv;
    }
    if (tid < C) sB[tid] = tid < n ? beta[(size_t)(t0 + tid) * H + h] : 0.f;
    __syncthreads();

    // 2. L2 norm of q and k rows (warp per row); 3. G = cumsum of log_alpha.
    if (l2norm) {
        for (int r = warp; r < C; r += kThreads / 32) {
            float sk = 0.f, sq = 0.f;
            for (int c = lane; c < DK; c += 32) {
                sk += sK[r * LD + c] * sK[r * LD + c];
                sq += sQ[r * LD + c] * sQ[r * LD + c];
            }
#pragma unroll
            for (int off = 16; off; off >>= 1) {
                sk += __shfl_xor_sync(0xffffffffu, sk, off);
                sq += __shfl_xor_sync(0xffffffffu, sq, off);
            }
            const float ik = 1.f / fmaxf(sqrtf(sk), eps), iq = 1.f / fmaxf(sqrtf(sq), eps);
            for (int c = lane; c < DK; c += 32) {
                sK[r * LD + c] *= ik;
                sQ[r * LD + c] *= iq;
            }
        }
    }
    if (tid < DK) {
        float run = 0.f;
        for (int r = 0; r < C; ++r) {
            run += sG[r * LD + tid];
            sG[r * LD + tid] = run;
        }
    }
    __syncthreads();

    // 4. A (strictly lower) and P (lower incl. diagonal), exponents element-wise.
    for (int p = tid; p < C * C; p += kThreads) {
        const int r = p / C, i = p % C;
        float a = 0.f, pp = 0.f;
        if (i <= r) {
            for (int c = 0; c < DK; ++c) {
                const float e = expf(sG[r * LD + c] - sG[i * LD + c]);
                const float ki = sK[i * LD + c] * e;
                a += sK[r * LD + c] * ki;
                pp += sQ[r * LD + c] * ki;
            }
        }
        sA[r * (C + 1) + i] = (i < r) ? a : 0.f;
        sP[r * (C + 1) + i] = pp;
    }
    __syncthreads();

    if (tid < C) {
        // 5. T column by column (forward substitution, one thread per column c):
        //    T[r][c] = beta_r (delta_rc - sum_{c <= i < r} A[r][i] T[i][c]).
        const int c = tid;
        for (int r = 0; r < C; ++r) {
            float val = 0.f;
            if (r == c) {
                val = sB[c];
            } else if (r > c) {
                float acc = 0.f;
                for (int i = c; i < r; ++i) acc += sA[r * (C + 1) + i] * sT[i * (C + 1) + c];
                val = -sB[r] * acc;
            }
            sT[r * (C + 1) + c] = val;
        }
    } else {
        // 6. Meanwhile: Q*e^G and K*e^{G_last-G} to the slot, K*e^G kept in smem.
        for (int idx = tid - C; idx < C * DK; idx += kThreads - C) {
            const int c = idx / C, r = idx % C;  // transposed walk: r fastest
            const float g = sG[r * LD + c], gl = sG[(C - 1) * LD + c];
            const float e = expf(g);
            slot[Slot<DK>::QGT + c * C + r] = sQ[r * LD + c] * e;
            slot[Slot<DK>::KD + r * DK + c] = sK[r * LD + c] * expf(gl - g);
        }
        for (int c = tid - C; c < DK; c += kThreads - C) slot[Slot<DK>::D + c] = expf(sG[(C - 1) * LD + c]);
    }
    __syncthreads();
    for (int idx = tid; idx < C * DK; idx += kThreads) {
        const int r = idx / DK, c = idx % DK;
        sK[r * LD + c] *= expf(sG[r * LD + c]);
    }
    __syncthreads();

    // 7. W = T (K*e^G), stored transposed; P and T stored transposed.
    for (int idx = tid; idx < C * DK; idx += kThreads) {
        const int c = idx / C, r = idx % C;
        float acc = 0.f;
        for (int i = 0; i <= r; ++i) acc += sT[r * (C + 1) + i] * sK[i * LD + c];
        slot[Slot<DK>::WT + c * C + r] = acc;
    }
    for (int idx = tid; idx < C * C; idx += kThreads) {
        const int i = idx / C, r = idx % C;
        slot[Slot<DK>::TT + i * C + r] = sT[r * (C + 1) + i];
        slot[Slot<DK>::PT + i * C + r] = sP[r * (C + 1) + i];
    }
}

template <int DK, typename T>
__global__ void __launch_bounds__(kThreads)
scan_kernel(const T *__restrict__ v, const int32_t *__restrict__ cu, int64_t total, int H, int N,
            int DV, int j0, int nw, const char *__restrict__ slots, size_t slot_bytes,
            const float *__restrict__ S0, float *__restrict__ state, float *__restrict__ S_T,
            T *__restrict__ o) {
    const int jv = blockIdx.x, s = blockIdx.y, h = blockIdx.z;
    int64_t bos, eos;
    seq_bounds(cu, s, total, bos, eos);
    const int64_t len = eos - bos;
    const int nch = (int)((len + C - 1) / C);
    if (j0 >= nch && !(nch == 0 && j0 == 0)) return;
    const int jend = min(j0 + nw, nch);

    extern __shared__ float sm[];
    float *sWt = sm;                 // [DK][C]
    float *sQgt = sWt + DK * C;      // [DK][C]
    float *sKd = sQgt + DK * C;      // [C][DK]
    float *sTt = sKd + C * DK;       // [C][C]
    float *sPt = sTt + C * C;        // [C][C]
    float *sD = sPt + C * C;         // [DK]
    float *sV = sD + DK;             // [C][32]
    float *sU = sV + C * kDvTile;    // [C][32]
    float *sS = sU + C * kDvTile;    // [DK][32]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t sofs = ((size_t)s * H + h) * DK * DV + (size_t)jv * kDvTile;

    // Entry state of this wave: S0 (or zeros) on the first wave, else the carry.
    const float *Sin = (j0 == 0) ? S0 : state;
    for (int idx = tid; idx < DK * kDvTile; idx += kThreads) {
        const int c = idx / kDvTile, jj = idx % kDvTile;
        sS[idx] = Sin ? Sin[sofs + (size_t)c * DV + jj] : 0.f;
    }

    constexpr int RT = C / (kThreads / 32);   // rows per thread in the row-parallel phases (8)
    constexpr int CT = DK / (kThreads / 32);  // state rows per thread in the update (16 or 8)
    const int r0 = warp * RT, c0 = warp * CT;

    for (int j = j0; j < jend; ++j) {
        const int n = (int)(len - (int64_t)j * C < C ? len - (int64_t)j * C : C);
        const int64_t t0 = bos + (int64_t)j * C;
        const float4 *src = reinterpret_cast<const float4 *>(
            slots + ((size_t)(j - j0) * N + s) * H * slot_bytes + (size_t)h * slot_bytes);
        float4 *dst = reinterpret_cast<float4 *>(sWt);
        for (int idx = tid; idx < Slot<DK>::FLOATS / 4; idx += kThreads) dst[idx] = src[idx];
        for (int idx = tid; idx < C * kDvTile; idx += kThreads) {
            const int r = idx / kDvTile, jj = idx % kDvTile;
            sV[idx] = r < n ? IO<T>::ld(v + ((size_t)(t0 + r) * H + h) * DV + jv * kDvTile + jj) : 0.f;
        }
        __syncthreads();

        // U = T V - W S  (rows r0..r0+7, column lane)
        float acc[RT];
#pragma unroll
        for (int m = 0; m < RT; ++m) acc[m] = 0.f;
        for (int i = 0; i < C; ++i) {
            const float x = sV[i * kDvTile + lane];
#pragma unroll
            for (int m = 0; m < RT; ++m) acc[m] += sTt[i * C + r0 + m] * x;
        }
        for (int c = 0; c < DK; ++c) {
            const float x = sS[c * kDvTile + lane];
#pragma unroll
            for (int m = 0; m < RT; ++m) acc[m] -= sWt[c * C + r0 + m] * x;
        }
#pragma unroll
        for (int m = 0; m < RT; ++m) sU[(r0 + m) * kDvTile + lane] = acc[m];
        __syncthreads();

        // O = (Q e^G) S + P U
#pragma unroll
        for (int m = 0; m < RT; ++m) acc[m] = 0.f;
        for (int c = 0; c < DK; ++c) {
            const float x = sS[c * kDvTile + lane];
#pragma unroll
            for (int m = 0; m < RT; ++m) acc[m] += sQgt[c * C + r0 + m] * x;
        }
        for (int i = 0; i < C; ++i) {
            const float x = sU[i * kDvTile + lane];
#pragma unroll
            for (int m = 0; m < RT; ++m) acc[m] += sPt[i * C + r0 + m] * x;
        }
#pragma unroll
        for (int m = 0; m < RT; ++m)
            if (r0 + m < n) IO<T>::st(o + ((size_t)(t0 + r0 + m) * H + h) * DV + jv * kDvTile + lane, acc[m]);

        // S' = Diag(e^{G_last}) S + Kd^T U
        float sn[CT];
#pragma unroll
        for (int m = 0; m < CT; ++m) sn[m] = sD[c0 + m] * sS[(c0 + m) * kDvTile + lane];
        for (int r = 0; r < C; ++r) {
            const float x = sU[r * kDvTile + lane];
#pragma unroll
            for (int m = 0; m < CT; ++m) sn[m] += sKd[r * DK + c0 + m] * x;
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < CT; ++m) sS[(c0 + m) * kDvTile + lane] = sn[m];
        __syncthreads();
    }
    __syncthreads();

    // Exit: the final state when the sequence ended in this wave, else the carry.
    float *Sout = (jend == nch) ? S_T : state;
    if (Sout)
        for (int idx = tid; idx < DK * kDvTile; idx += kThreads) {
            const int c = idx / kDvTile, jj = idx % kDvTile;
            Sout[sofs + (size_t)c * DV + jj] = sS[idx];
        }
}

template <int DK> constexpr size_t prep_smem() { return (3 * C * (DK + 1) + 3 * C * (C + 1) + C) * 4; }
template <int DK> constexpr size_t scan_smem() {
    return (size_t)(Slot<DK>::FLOATS + 2 * C * kDvTile + DK * kDvTile) * 4;
}

template <int DK, typename T>
cudaError_t wave(const PrefillArgs &a, int j0, int nw, cudaStream_t st) {
    // Per-call attribute set (cheap, host-only, and correct on every device).
    cudaError_t e = cudaFuncSetAttribute(prep_kernel<DK, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)prep_smem<DK>());
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(scan_kernel<DK, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)scan_smem<DK>());
    if (e != cudaSuccess) return e;
    if (nw > 0) {
        dim3 gp(nw, a.N, a.H);
        prep_kernel<DK, T><<<gp, kThreads, prep_smem<DK>(), st>>>(
            (const T *)a.q, (const T *)a.k, a.log_alpha, a.beta, a.cu, a.total, a.H, a.N, j0,
            a.l2norm, a.la_scalar, a.eps, a.slots, a.slot_bytes);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    dim3 gs(a.dv / kDvTile, a.N, a.H);
    scan_kernel<DK, T><<<gs, kThreads, scan_smem<DK>(), st>>>(
        (const T *)a.v, a.cu, a.total, a.H, a.N, a.dv, j0, nw, a.slots, a.slot_bytes, a.S0,
        a.state, a.S_T, (T *)a.o);
    return cudaGetLastError();
}

}  // namespace

size_t simt_slot_bytes(int dk) { return dk == 64 ? Slot<64>::BYTES : Slot<128>::BYTES; }

// Output step after the fp32 prefill, in place on o: one warp per (token, head)
// row, o <- o / sqrt(mean(o^2) + eps) * w * sigmoid(gate) over the DV channels.
template <int DV, typename T>
__global__ void __launch_bounds__(256)
output_gate_kernel(T *__restrict__ o, const T *__restrict__ gate, const float *__restrict__ w, float eps,
                   int64_t rows) {
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float x[DV / 32], ss = 0.f;
#pragma unroll
    for (int i = 0; i < DV / 32; ++i) {
        x[i] = IO<T>::ld(o + row * DV + lane + 32 * i);
        ss += x[i] * x[i];
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float r = rsqrtf(ss / DV + eps);
#pragma unroll
    for (int i = 0; i < DV / 32; ++i) {
        const int c = lane + 32 * i;
        const float g = IO<T>::ld(gate + row * DV + c);
        IO<T>::st(o + row * DV + c, x[i] * r * w[c] / (1.f + __expf(-g)));
    }
}

template <int DV, typename T>
cudaError_t output_gate(const PrefillArgs &a, cudaStream_t st) {
    const int64_t rows = a.total * a.H;
    output_gate_kernel<DV, T><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
        (T *)a.o, (const T *)a.og_gate, a.og_w, a.og_eps, rows);
    return cudaGetLastError();
}

cudaError_t simt_output_gate(const PrefillArgs &a, bool bf16, cudaStream_t st) {
    if (a.dv == 128) return bf16 ? output_gate<128, __nv_bfloat16>(a, st) : output_gate<128, float>(a, st);
    if (a.dv == 64) return bf16 ? output_gate<64, __nv_bfloat16>(a, st) : output_gate<64, float>(a, st);
    return cudaErrorInvalidValue;
}

cudaError_t simt_prefill_wave(const PrefillArgs &a, int j0, int nw, bool bf16, cudaStream_t st) {
    if (a.dk == 128) return bf16 ? wave<128, __nv_bfloat16>(a, j0, nw, st) : wave<128, float>(a, j0, nw, st);
    if (a.dk == 64) return bf16 ? wave<64, __nv_bfloat16>(a, j0, nw, st) : wave<64, float>(a, j0, nw, st);
    return cudaErrorInvalidValue;
}

}  // namespace kda
