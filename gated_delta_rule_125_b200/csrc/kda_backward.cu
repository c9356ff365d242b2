// kda_backward.cu -- gradients of the chunkwise prefill (training backward).
//
// The pages mention training ("[Kimi-2] Kimi Linear：用 KDA 重写长上下文注意力"
// §5) but give no backward; this follows the chunked reverse-mode algebra
// derived for the fp64 oracle's chunkwise backward. Per chunk (rows r, entry
// state S, G the inclusive cumsum of log_alpha, g its last row; Qg = Q e^G,
// Kg = K e^G, Kn = K e^-G, Kd = K e^(g-G); A = strict_lower(Kg Kn^T),
// P = lower(Qg Kn^T); X = (I + Diag(beta) A)^-1, T = X Diag(beta), W = T Kg,
// U = T V - W S; O = Qg S + P U, S' = Diag(e^g) S + Kd^T U) and given dO, dS':
//
//   dS  = Diag(e^g) dS' + Qg^T dO - W^T dU,   dU = Kd dS' + P^T dO
//   dKd = U dS'^T,  dP = lower(dO U^T),  dQg = dO S^T,  dW = -dU S^T
//   dT  = lower(dU V^T + dW Kg^T),  dV = T^T dU,  dKg = T^T dW
//   dX  = dT Diag(beta),  dM = -X^T dX X^T,  dA = strict_lower(Diag(beta) dM)
//   dbeta_i = sum_r dT_ri X_ri + sum_m dM_im A_im
//   dKg += dA Kn,  dKn = dA^T Kg + dP^T Qg,  dQg += dP Kn
//   dG  = dQg Qg + dKg Kg - dKn Kn - dKd Kd,  dg = colsum(dKd Kd) + e^g rowsum(dS' S)
//   dlog_alpha_r = sum_{r' >= r} dG_r' + dg
//
// then through q/max(|q|, eps), k/max(|k|, eps).
//
// A CUDA-core implementation in fp32, seven launches (bw_offsets: the first chunk of each
// sequence, so that the chunk slots are packed; then):
//   1. bw_prep   (one CTA per chunk): normalised q, k; G, Qg, Kg, Kn, Kd, A, P,
//                the unit-lower-triangular inverse X by column forward
//                substitution, T, W, T V;
//   2. bw_fwd    (one CTA per 16 state columns of a (sequence, head)): the
//                chunks' entry states and U, W and Kd staged in shared memory;
//   3. bw_bwd    (likewise): dU and the state gradient entering each chunk, in
//                reverse chunk order; dS0;
//   4. bw_rowstate (one CTA per chunk): dKd, dQg, dW, dP and dT, the
//                contractions over the value (and key) dimension, by shared-memory tiles;
//      bw_grads  (one CTA per chunk): every other per-chunk gradient above;
//   5. bw_norm   (one warp per (token, head)): through the L2 normalisation.
// Everything lives in the caller's workspace (fp32); each product is a plain
// loop over its output elements. The factorised exponents need e^-G finite:
// a chunk whose decay range exceeds 60 nats sets device error code 2.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int C = kChunk;  // 64
constexpr int kBwThreads = 256;
constexpr float kBwRange = 60.f;
constexpr int kVb = 32;        // columns per shared-memory tile of the tiled contractions
constexpr int kLdA = kVb + 1;  // tile row length (floats): rows apart by one bank

// Per-chunk scratch (floats), in this order.
struct Slot {
    int dk, dv;
    __host__ __device__ size_t cd() const { return (size_t)C * dk; }
    __host__ __device__ size_t cv() const { return (size_t)C * dv; }
    __host__ __device__ size_t kv() const { return (size_t)dk * dv; }
    __host__ __device__ size_t floats() const { return 11 * cd() + 9 * (size_t)C * C + 3 * cv() + 2 * kv(); }
};
struct SlotPtr {
    float *G, *Qg, *Kg, *Kn, *Kd, *W;          // C x dk
    float *dKd, *dQg, *dW, *dKg, *dKn;         // C x dk
    float *A, *P, *X, *T, *dP, *dT, *dM, *Y, *dA;  // C x C
    float *TV, *U, *dU;                        // C x dv
    float *S, *dSn;                            // dk x dv
    __device__ SlotPtr(float *base, const Slot &s) {
        float *p = base;
        G = p; p += s.cd(); Qg = p; p += s.cd(); Kg = p; p += s.cd(); Kn = p; p += s.cd();
        Kd = p; p += s.cd(); W = p; p += s.cd();
        dKd = p; p += s.cd(); dQg = p; p += s.cd(); dW = p; p += s.cd(); dKg = p; p += s.cd();
        dKn = p; p += s.cd();
        A = p; p += C * C; P = p; p += C * C; X = p; p += C * C; T = p; p += C * C;
        dP = p; p += C * C; dT = p; p += C * C; dM = p; p += C * C; Y = p; p += C * C; dA = p; p += C * C;
        TV = p; p += s.cv(); U = p; p += s.cv(); dU = p; p += s.cv();
        S = p; p += s.kv(); dSn = p;
    }
};

struct BwArgs {
    const void *q, *k, *v, *dout;
    const float *la, *beta, *S0, *dST;
    const int32_t *cu;
    int64_t total;
    int N, H, dk, dv, NC;  // NC: chunk slots per head, at least the chunks of all sequences
    int l2norm, la_scalar;
    float eps;
    float *dq, *dkk, *dvv, *dla, *dbeta, *dS0;
    float *slots;          // NC * H slots: chunk ci of head h in slot ci * H + h
    int *coff;             // [N + 1]: first chunk of each sequence (prefix sums of ceil(len / 64))
    float *qh, *kh, *dqh, *dkh, *nq, *nk;  // per (token, head)
    int *err;
};

// Slot of block b of the per-chunk kernels (grid H * NC): chunk ci = b / H of head h = b % H,
// sequence s the last one whose first chunk is at or before ci, j its chunk; false past the chunks.
__device__ __forceinline__ bool slot_chunk(const BwArgs &a, int b, int &s, int &h, int &j) {
    const int ci = b / a.H;
    h = b % a.H;
    if (ci >= a.coff[a.N]) return false;
    int lo = 0, hi = a.N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.coff[mid] <= ci) lo = mid;
        else hi = mid - 1;
    }
    s = lo;
    j = ci - a.coff[lo];
    return true;
}
__device__ __forceinline__ size_t slot_of(const BwArgs &a, int s, int h, int j) {
    return (size_t)(a.coff[s] + j) * a.H + h;
}

// First chunk of each sequence: one CTA, each thread a run of sequences, then a scan of the runs.
__global__ void __launch_bounds__(1024) bw_offsets(BwArgs a) {
    __shared__ int part[1024];
    const int tid = threadIdx.x, per = (a.N + 1023) / 1024, s0 = tid * per, s1 = min(a.N, s0 + per);
    auto nch = [&](int s) {
        int64_t bos, eos;
        seq_bounds(a.cu, s, a.total, bos, eos);
        return (int)((eos - bos + C - 1) / C);
    };
    int sum = 0;
    for (int s = s0; s < s1; ++s) sum += nch(s);
    part[tid] = sum;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {  // inclusive scan of the runs
        const int v = tid >= off ? part[tid - off] : 0;
        __syncthreads();
        part[tid] += v;
        __syncthreads();
    }
    int run = part[tid] - sum;
    for (int s = s0; s < s1; ++s) {
        a.coff[s] = run;
        run += nch(s);
    }
    if (tid == 1023) a.coff[a.N] = part[1023];
}

__device__ __forceinline__ void chunk_rows(const BwArgs &a, int s, int j, int64_t &t0, int &n) {
    int64_t bos, eos;
    seq_bounds(a.cu, s, a.total, bos, eos);
    t0 = bos + (int64_t)j * C;
    const int64_t rem = eos - t0;
    n = rem <= 0 ? 0 : (rem < C ? (int)rem : C);
}

// 1. Per chunk: normalised q, k; G, Qg, Kg, Kn, Kd; A, P; X, T; W = T Kg; T V.
template <typename T>
__global__ void __launch_bounds__(kBwThreads) bw_prep(BwArgs a) {
    const int slot = blockIdx.x;
    int s, h, j;
    if (!slot_chunk(a, slot, s, h, j)) return;
    int64_t t0;
    int n;
    chunk_rows(a, s, j, t0, n);
    if (n == 0) return;
    const int dk = a.dk, dv = a.dv, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const Slot sl{dk, dv};
    SlotPtr m(a.slots + (size_t)slot * sl.floats(), sl);
    const T *q = static_cast<const T *>(a.q), *k = static_cast<const T *>(a.k), *v = static_cast<const T *>(a.v);
    // normalised rows (a warp per row)
    for (int r = warp; r < n; r += kBwThreads / 32) {
        const size_t row = (size_t)(t0 + r) * a.H + h;
        float sq = 0.f, sk = 0.f;
        for (int c = lane; c < dk; c += 32) {
            const float x = IO<T>::ld(q + row * dk + c), y = IO<T>::ld(k + row * dk + c);
            sq += x * x;
            sk += y * y;
        }
        for (int off = 16; off; off >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
        }
        const float nq = a.l2norm ? fmaxf(sqrtf(sq), a.eps) : 1.f, nk = a.l2norm ? fmaxf(sqrtf(sk), a.eps) : 1.f;
        for (int c = lane; c < dk; c += 32) {
            a.qh[row * dk + c] = IO<T>::ld(q + row * dk + c) / nq;
            a.kh[row * dk + c] = IO<T>::ld(k + row * dk + c) / nk;
        }
        if (lane == 0) {
            a.nq[row] = a.l2norm ? sqrtf(sq) : 1.f;
            a.nk[row] = a.l2norm ? sqrtf(sk) : 1.f;
        }
    }
    __syncthreads();
    // G (cumsum over the rows), exponent factors
    for (int c = tid; c < dk; c += kBwThreads) {
        float run = 0.f;
        for (int r = 0; r < n; ++r) {
            run += a.la_scalar ? a.la[(size_t)(t0 + r) * a.H + h] : a.la[(size_t)(t0 + r) * a.H * dk + (size_t)h * dk + c];
            m.G[r * dk + c] = run;
        }
        if (-run > kBwRange && a.err) atomicCAS(a.err, 0, 2);
    }
    __syncthreads();
    for (int e = tid; e < n * dk; e += kBwThreads) {
        const int r = e / dk, c = e % dk;
        const size_t row = (size_t)(t0 + r) * a.H + h;
        const float G = m.G[e], g = m.G[(n - 1) * dk + c];
        const float qv = a.qh[row * dk + c], kv = a.kh[row * dk + c];
        m.Qg[e] = qv * expf(G);
        m.Kg[e] = kv * expf(G);
        m.Kn[e] = kv * expf(-G);
        m.Kd[e] = kv * expf(g - G);
    }
    __syncthreads();
    // A = strict_lower(Kg Kn^T), P = lower(Qg Kn^T): 32-column tiles of Kg, Qg and Kn
    // in shared memory, a 4 x 4 block of each per thread
    extern __shared__ float4 smem4[];
    float *sm = reinterpret_cast<float *>(smem4);
    {
        float *tKg = sm, *tQg = tKg + C * kLdA, *tKn = tQg + C * kLdA;
        const int r0 = 4 * (tid >> 4), i0 = 4 * (tid & 15);
        float aa[4][4] = {}, pp[4][4] = {};
        for (int cb = 0; cb < dk; cb += kVb) {
            __syncthreads();  // the exponent factors are written; the previous tile is consumed
            for (int e = tid; e < C * kVb; e += kBwThreads) {
                const int r = e / kVb, c = e % kVb;
                const bool in = r < n;
                tKg[r * kLdA + c] = in ? m.Kg[(size_t)r * dk + cb + c] : 0.f;
                tQg[r * kLdA + c] = in ? m.Qg[(size_t)r * dk + cb + c] : 0.f;
                tKn[r * kLdA + c] = in ? m.Kn[(size_t)r * dk + cb + c] : 0.f;
            }
            __syncthreads();
            for (int c = 0; c < kVb; ++c) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float kg = tKg[(r0 + q) * kLdA + c], qg = tQg[(r0 + q) * kLdA + c];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const float kn = tKn[(i0 + x) * kLdA + c];
                        aa[q][x] += kg * kn;
                        pp[q][x] += qg * kn;
                    }
                }
            }
        }
        __syncthreads();  // the tiles are consumed: A takes the shared memory (rows of C + 1)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = r0 + q;
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int i = i0 + x;
                const float av = (r < n && i < r) ? aa[q][x] : 0.f;
                m.A[r * C + i] = av;
                sm[r * (C + 1) + i] = av;
                m.P[r * C + i] = (r < n && i <= r) ? pp[q][x] : 0.f;
            }
        }
    }
    __syncthreads();
    // X = (I + Diag(beta) A)^-1: column i by forward substitution (rows >= i), A and X in
    // shared memory (rows of C + 1 floats)
    const float *bt = a.beta;
    {
        const float *sA = sm;
        float *sXs = sm + C * (C + 1);
        for (int i = tid; i < C; i += kBwThreads) {
            for (int r = 0; r < C; ++r) {
                float x = 0.f;
                if (r < n && i < n && r >= i) {
                    if (r == i) {
                        x = 1.f;
                    } else {
                        float acc = 0.f;
                        for (int mm = i; mm < r; ++mm) acc += sA[r * (C + 1) + mm] * sXs[mm * (C + 1) + i];
                        x = -bt[(size_t)(t0 + r) * a.H + h] * acc;
                    }
                }
                sXs[r * (C + 1) + i] = x;
            }
        }
        __syncthreads();
        for (int e = tid; e < C * C; e += kBwThreads) m.X[e] = sXs[(e / C) * (C + 1) + e % C];
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += kBwThreads) {
        const int i = e % C;
        m.T[e] = i < n ? m.X[e] * bt[(size_t)(t0 + i) * a.H + h] : 0.f;
    }
    __syncthreads();
    // W = T Kg, TV = T V
    for (int e = tid; e < n * dk; e += kBwThreads) {
        const int r = e / dk, c = e % dk;
        float acc = 0.f;
        for (int i = 0; i <= r; ++i) acc += m.T[r * C + i] * m.Kg[i * dk + c];
        m.W[e] = acc;
    }
    for (int e = tid; e < n * dv; e += kBwThreads) {
        const int r = e / dv, c = e % dv;
        float acc = 0.f;
        for (int i = 0; i <= r; ++i) acc += m.T[r * C + i] * IO<T>::ld(v + ((size_t)(t0 + i) * a.H + h) * dv + c);
        m.TV[e] = acc;
    }
}

// 2. Entry states and U, chunk by chunk. The recurrence acts on each state column
//    on its own (S' = Diag(e^g) S + Kd^T (TV - W S), column by column), so a CTA takes
//    kCols columns of one (sequence, head): the columns in shared memory, and per chunk
//    W and Kd staged there from the slot.
constexpr int kCols = 16;
__host__ __device__ inline size_t fwd_smem_floats(int dk) { return (size_t)dk * kCols + 2 * (size_t)C * dk + C * kCols; }
__global__ void __launch_bounds__(kBwThreads, 2) bw_fwd(BwArgs a) {
    extern __shared__ float4 smem4[];
    const int groups = a.dv / kCols;
    const int unit = blockIdx.x / groups, c0 = (blockIdx.x % groups) * kCols, s = unit / a.H, tid = threadIdx.x;
    const int dk = a.dk, dv = a.dv;
    const Slot sl{dk, dv};
    float *sS = reinterpret_cast<float *>(smem4), *sW = sS + dk * kCols, *sKd = sW + C * dk, *sU = sKd + C * dk;
    for (int e = tid; e < dk * kCols; e += kBwThreads)
        sS[e] = a.S0 ? a.S0[(size_t)unit * dk * dv + (size_t)(e / kCols) * dv + c0 + e % kCols] : 0.f;
    const int nchunks = a.coff[s + 1] - a.coff[s];
    for (int j = 0; j < nchunks; ++j) {
        int64_t t0;
        int n;
        chunk_rows(a, s, j, t0, n);
        if (n == 0) break;
        SlotPtr m(a.slots + slot_of(a, s, unit % a.H, j) * sl.floats(), sl);
        for (int e = tid; e < n * dk / 4; e += kBwThreads) {
            reinterpret_cast<float4 *>(sW)[e] = reinterpret_cast<const float4 *>(m.W)[e];
            reinterpret_cast<float4 *>(sKd)[e] = reinterpret_cast<const float4 *>(m.Kd)[e];
        }
        __syncthreads();  // the staged rows; the state columns of the previous chunk
        for (int e = tid; e < dk * kCols; e += kBwThreads) m.S[(size_t)(e / kCols) * dv + c0 + e % kCols] = sS[e];
        // U = TV - W S: thread (row r, four columns)
        if (tid < n * 4) {
            const int r = tid >> 2, cq = (tid & 3) * 4;
            float4 acc = *reinterpret_cast<const float4 *>(m.TV + (size_t)r * dv + c0 + cq);
            for (int i = 0; i < dk; ++i) {
                const float w = sW[r * dk + i];
                const float4 x = *reinterpret_cast<const float4 *>(sS + i * kCols + cq);
                acc.x -= w * x.x;
                acc.y -= w * x.y;
                acc.z -= w * x.z;
                acc.w -= w * x.w;
            }
            *reinterpret_cast<float4 *>(sU + r * kCols + cq) = acc;
            *reinterpret_cast<float4 *>(m.U + (size_t)r * dv + c0 + cq) = acc;
        }
        __syncthreads();
        // S' = Diag(e^g) S + Kd^T U: thread (state row i, eight columns), in place
        if (tid < 2 * dk) {
            const int i = tid >> 1, ch = (tid & 1) * 8;
            const float eg = expf(m.G[(n - 1) * dk + i]);
            float acc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = eg * sS[i * kCols + ch + q];
            for (int r = 0; r < n; ++r) {
                const float kd = sKd[r * dk + i];
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] += kd * sU[r * kCols + ch + q];
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) sS[i * kCols + ch + q] = acc[q];
        }
        __syncthreads();
    }
}

// 3. State gradient entering each chunk (reverse order), dU; dS0. Column by column like
//    bw_fwd: dU = Kd dS' + P^T dO and dS = Diag(e^g) dS' + Qg^T dO - W^T dU act on each
//    column of dS' and dO on its own.
__host__ __device__ inline size_t bwd_smem_floats(int dk) {
    return (size_t)dk * kCols + 2 * (size_t)C * dk + (size_t)C * C + 2 * C * kCols;
}
template <typename T>
__global__ void __launch_bounds__(kBwThreads, 2) bw_bwd(BwArgs a) {
    extern __shared__ float4 smem4[];
    const int groups = a.dv / kCols;
    const int unit = blockIdx.x / groups, c0 = (blockIdx.x % groups) * kCols, s = unit / a.H, h = unit % a.H;
    const int tid = threadIdx.x, dk = a.dk, dv = a.dv;
    const Slot sl{dk, dv};
    const T *dout = static_cast<const T *>(a.dout);
    float *sG = reinterpret_cast<float *>(smem4), *sA = sG + dk * kCols, *sB = sA + C * dk, *sP = sB + C * dk,
          *sdO = sP + C * C, *sdU = sdO + C * kCols;
    for (int e = tid; e < dk * kCols; e += kBwThreads)
        sG[e] = a.dST ? a.dST[(size_t)unit * dk * dv + (size_t)(e / kCols) * dv + c0 + e % kCols] : 0.f;
    for (int j = a.coff[s + 1] - a.coff[s] - 1; j >= 0; --j) {
        int64_t t0;
        int n;
        chunk_rows(a, s, j, t0, n);
        if (n == 0) continue;
        SlotPtr m(a.slots + slot_of(a, s, h, j) * sl.floats(), sl);
        for (int e = tid; e < n * dk / 4; e += kBwThreads) {
            reinterpret_cast<float4 *>(sA)[e] = reinterpret_cast<const float4 *>(m.Kd)[e];
            reinterpret_cast<float4 *>(sB)[e] = reinterpret_cast<const float4 *>(m.W)[e];
        }
        for (int e = tid; e < C * C / 4; e += kBwThreads)
            reinterpret_cast<float4 *>(sP)[e] = reinterpret_cast<const float4 *>(m.P)[e];
        for (int e = tid; e < n * kCols; e += kBwThreads)
            sdO[e] = IO<T>::ld(dout + ((size_t)(t0 + e / kCols) * a.H + h) * dv + c0 + e % kCols);
        __syncthreads();
        for (int e = tid; e < dk * kCols; e += kBwThreads) m.dSn[(size_t)(e / kCols) * dv + c0 + e % kCols] = sG[e];
        // dU = Kd dS' + P^T dO: thread (row r, four columns)
        if (tid < n * 4) {
            const int r = tid >> 2, cq = (tid & 3) * 4;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int i = 0; i < dk; ++i) {
                const float w = sA[r * dk + i];
                const float4 x = *reinterpret_cast<const float4 *>(sG + i * kCols + cq);
                acc.x += w * x.x;
                acc.y += w * x.y;
                acc.z += w * x.z;
                acc.w += w * x.w;
            }
            for (int rr = r; rr < n; ++rr) {
                const float pv = sP[rr * C + r];
                const float4 x = *reinterpret_cast<const float4 *>(sdO + rr * kCols + cq);
                acc.x += pv * x.x;
                acc.y += pv * x.y;
                acc.z += pv * x.z;
                acc.w += pv * x.w;
            }
            *reinterpret_cast<float4 *>(sdU + r * kCols + cq) = acc;
            *reinterpret_cast<float4 *>(m.dU + (size_t)r * dv + c0 + cq) = acc;
        }
        __syncthreads();  // Kd is no longer read: Qg takes its place
        for (int e = tid; e < n * dk / 4; e += kBwThreads)
            reinterpret_cast<float4 *>(sA)[e] = reinterpret_cast<const float4 *>(m.Qg)[e];
        __syncthreads();
        // dS = Diag(e^g) dS' + Qg^T dO - W^T dU: thread (state row i, eight columns), in place
        if (tid < 2 * dk) {
            const int i = tid >> 1, ch = (tid & 1) * 8;
            const float eg = expf(m.G[(n - 1) * dk + i]);
            float acc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = eg * sG[i * kCols + ch + q];
            for (int r = 0; r < n; ++r) {
                const float qg = sA[r * dk + i], w = sB[r * dk + i];
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] += qg * sdO[r * kCols + ch + q] - w * sdU[r * kCols + ch + q];
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) sG[i * kCols + ch + q] = acc[q];
        }
        __syncthreads();
    }
    if (a.dS0)
        for (int e = tid; e < dk * kCols; e += kBwThreads)
            a.dS0[(size_t)unit * dk * dv + (size_t)(e / kCols) * dv + c0 + e % kCols] = sG[e];
}

// 4a. Per chunk, the contractions over the value dimension: dKd = U dS'^T,
//     dQg = dO S^T, dW = -dU S^T (n x dk) and dP = lower(dO U^T) (C x C). Shared-memory
//     tiles over 32 value columns at a time: the row operands (U, dO, dU) as they are,
//     S and dS' transposed; a thread accumulates a 4 x 4 block of each output.
__host__ __device__ inline size_t rs_smem_floats(int dk) { return 3 * (size_t)C * kLdA + 2 * (size_t)kVb * (dk + 4); }
template <typename T>
__global__ void __launch_bounds__(kBwThreads) bw_rowstate(BwArgs a) {
    extern __shared__ float4 smem4[];
    const int slot = blockIdx.x;
    int s, h, j;
    if (!slot_chunk(a, slot, s, h, j)) return;
    int64_t t0;
    int n;
    chunk_rows(a, s, j, t0, n);
    if (n == 0) return;
    const int dk = a.dk, dv = a.dv, tid = threadIdx.x, ldb = dk + 4;
    const Slot sl{dk, dv};
    SlotPtr m(a.slots + (size_t)slot * sl.floats(), sl);
    const T *dout = static_cast<const T *>(a.dout);
    float *sU = reinterpret_cast<float *>(smem4), *sdO = sU + C * kLdA, *sdU = sdO + C * kLdA;
    float *sS = sdU + C * kLdA, *sSn = sS + kVb * ldb;  // [value column][state row]
    const int ngi = dk / 4, rows_per_round = 4 * (kBwThreads / ngi), rounds = C / rows_per_round;
    for (int round = 0; round < rounds; ++round) {
        const int r0 = round * rows_per_round + 4 * (tid / ngi), i0 = 4 * (tid % ngi);
        const int pr0 = 4 * (tid >> 4), pi0 = 4 * (tid & 15);  // the dP block (round 0)
        float kd[4][4] = {}, qg[4][4] = {}, w[4][4] = {}, dp[4][4] = {};
        for (int cb = 0; cb < dv; cb += kVb) {
            __syncthreads();  // the previous tile is consumed
            for (int e = tid; e < C * kVb; e += kBwThreads) {
                const int r = e / kVb, c = e % kVb;
                const bool in = r < n;
                sU[r * kLdA + c] = in ? m.U[(size_t)r * dv + cb + c] : 0.f;
                sdU[r * kLdA + c] = in ? m.dU[(size_t)r * dv + cb + c] : 0.f;
                sdO[r * kLdA + c] = in ? IO<T>::ld(dout + ((size_t)(t0 + r) * a.H + h) * dv + cb + c) : 0.f;
            }
            for (int e = tid; e < dk * kVb; e += kBwThreads) {
                const int i = e / kVb, c = e % kVb;
                sS[c * ldb + i] = m.S[(size_t)i * dv + cb + c];
                sSn[c * ldb + i] = m.dSn[(size_t)i * dv + cb + c];
            }
            __syncthreads();
            for (int c = 0; c < kVb; ++c) {
                const float4 bs = *reinterpret_cast<const float4 *>(sS + c * ldb + i0);
                const float4 bn = *reinterpret_cast<const float4 *>(sSn + c * ldb + i0);
                const float vs[4] = {bs.x, bs.y, bs.z, bs.w}, vn[4] = {bn.x, bn.y, bn.z, bn.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float u = sU[(r0 + q) * kLdA + c], o = sdO[(r0 + q) * kLdA + c], du = sdU[(r0 + q) * kLdA + c];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        kd[q][x] += u * vn[x];
                        qg[q][x] += o * vs[x];
                        w[q][x] -= du * vs[x];
                    }
                }
                if (round == 0) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float o = sdO[(pr0 + q) * kLdA + c];
#pragma unroll
                        for (int x = 0; x < 4; ++x) dp[q][x] += o * sU[(pi0 + x) * kLdA + c];
                    }
                }
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = r0 + q;
            if (r < n) {
                *reinterpret_cast<float4 *>(m.dKd + (size_t)r * dk + i0) = make_float4(kd[q][0], kd[q][1], kd[q][2], kd[q][3]);
                *reinterpret_cast<float4 *>(m.dQg + (size_t)r * dk + i0) = make_float4(qg[q][0], qg[q][1], qg[q][2], qg[q][3]);
                *reinterpret_cast<float4 *>(m.dW + (size_t)r * dk + i0) = make_float4(w[q][0], w[q][1], w[q][2], w[q][3]);
            }
        }
        if (round == 0) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = pr0 + q;
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int i = pi0 + x;
                    m.dP[r * C + i] = (r < n && i <= r) ? dp[q][x] : 0.f;
                }
            }
        }
    }
    // dT = lower(dU V^T + dW Kg^T): tiles over the value columns (dU, V), then the key
    // columns (dW, written above, and Kg); the same 4 x 4 blocks as dP.
    __syncthreads();  // dW of every row is in the slot
    {
        const T *v = static_cast<const T *>(a.v);
        const int pr0 = 4 * (tid >> 4), pi0 = 4 * (tid & 15);
        float dt[4][4] = {};
        float *sR = sU, *sI = sdO;  // [row][32 + 1]: the r rows and the i rows of a tile
        for (int cb = 0; cb < dv + dk; cb += kVb) {
            __syncthreads();
            const bool val = cb < dv;
            for (int e = tid; e < C * kVb; e += kBwThreads) {
                const int r = e / kVb, c = e % kVb;
                const bool in = r < n;
                sR[r * kLdA + c] = !in ? 0.f : val ? m.dU[(size_t)r * dv + cb + c] : m.dW[(size_t)r * dk + cb - dv + c];
                sI[r * kLdA + c] = !in ? 0.f
                                       : val ? IO<T>::ld(v + ((size_t)(t0 + r) * a.H + h) * dv + cb + c)
                                             : m.Kg[(size_t)r * dk + cb - dv + c];
            }
            __syncthreads();
            for (int c = 0; c < kVb; ++c) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float x0 = sR[(pr0 + q) * kLdA + c];
#pragma unroll
                    for (int x = 0; x < 4; ++x) dt[q][x] += x0 * sI[(pi0 + x) * kLdA + c];
                }
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = pr0 + q;
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int i = pi0 + x;
                m.dT[r * C + i] = (r < n && i <= r) ? dt[q][x] : 0.f;
            }
        }
    }
}

// 4. Every per-chunk gradient.
template <typename T>
__global__ void __launch_bounds__(kBwThreads) bw_grads(BwArgs a) {
    const int slot = blockIdx.x;
    int s, h, j;
    if (!slot_chunk(a, slot, s, h, j)) return;
    int64_t t0;
    int n;
    chunk_rows(a, s, j, t0, n);
    if (n == 0) return;
    const int dk = a.dk, dv = a.dv, tid = threadIdx.x;
    const Slot sl{dk, dv};
    SlotPtr m(a.slots + (size_t)slot * sl.floats(), sl);
    extern __shared__ float4 smem4[];
    float *sX = reinterpret_cast<float *>(smem4), *sdT = sX + C * (C + 1), *sY = sdT + C * (C + 1);
    auto beta = [&](int r) { return a.beta[(size_t)(t0 + r) * a.H + h]; };
    // (1) dKd, dQg, dW and dP: bw_rowstate
    // (2) dT: bw_rowstate; dV = T^T dU
    for (int e = tid; e < n * dv; e += kBwThreads) {
        const int r = e / dv, c = e % dv;
        float acc = 0.f;
        for (int rr = r; rr < n; ++rr) acc += m.T[rr * C + r] * m.dU[rr * dv + c];
        a.dvv[((size_t)(t0 + r) * a.H + h) * dv + c] = acc;
    }
    __syncthreads();
    // (3) dKg = T^T dW; Y = X^T dX with dX = dT Diag(beta)
    for (int e = tid; e < n * dk; e += kBwThreads) {
        const int r = e / dk, c = e % dk;
        float acc = 0.f;
        for (int rr = r; rr < n; ++rr) acc += m.T[rr * C + r] * m.dW[rr * dk + c];
        m.dKg[e] = acc;
    }
    // X, dT and Y in shared memory, rows padded to C + 1 floats (conflict-free by row and by column)
    constexpr int LD = C + 1;
    for (int e = tid; e < C * C; e += kBwThreads) {
        sX[(e / C) * LD + e % C] = m.X[e];
        sdT[(e / C) * LD + e % C] = m.dT[e];
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += kBwThreads) {
        const int r = e / C, i = e % C;
        float acc = 0.f;
        if (r < n && i < n)
            for (int mm = 0; mm < n; ++mm) acc += sX[mm * LD + r] * sdT[mm * LD + i] * beta(i);
        m.Y[e] = acc;
        sY[r * LD + i] = acc;
    }
    __syncthreads();
    // (4) dM = -Y X^T
    for (int e = tid; e < C * C; e += kBwThreads) {
        const int r = e / C, i = e % C;
        float acc = 0.f;
        if (r < n && i < n)
            for (int mm = 0; mm < n; ++mm) acc -= sY[r * LD + mm] * sX[i * LD + mm];
        m.dM[e] = acc;
        sdT[r * LD + i] = acc;  // dT is no longer read: dM takes its place
    }
    __syncthreads();
    // (5) dA = strict_lower(Diag(beta) dM); dbeta
    for (int e = tid; e < C * C; e += kBwThreads) {
        const int r = e / C, i = e % C;
        m.dA[e] = (r < n && i < r) ? beta(r) * m.dM[e] : 0.f;
    }
    for (int i = tid; i < n; i += kBwThreads) {
        float acc = 0.f;
        for (int r = 0; r < n; ++r) acc += m.dT[r * C + i] * m.X[r * C + i];
        for (int mm = 0; mm < i; ++mm) acc += sdT[i * LD + mm] * m.A[i * C + mm];
        a.dbeta[(size_t)(t0 + i) * a.H + h] = acc;
    }
    __syncthreads();
    // (6) dKg += dA Kn; dKn = dA^T Kg + dP^T Qg; dQg += dP Kn
    for (int e = tid; e < n * dk; e += kBwThreads) {
        const int r = e / dk, c = e % dk;
        float kg = 0.f, kn = 0.f, qg = 0.f;
        for (int i = 0; i < n; ++i) {
            kg += m.dA[r * C + i] * m.Kn[i * dk + c];
            kn += m.dA[i * C + r] * m.Kg[i * dk + c] + m.dP[i * C + r] * m.Qg[i * dk + c];
            qg += m.dP[r * C + i] * m.Kn[i * dk + c];
        }
        m.dKg[e] += kg;
        m.dKn[e] = kn;
        m.dQg[e] += qg;
    }
    __syncthreads();
    // (7)(8) dG, dg, dlog_alpha (reverse cumsum); d q^, d k^ through the exponents.
    // The row sums of dS' * S first, a warp per state row (coalesced), into shared memory.
    float *sss = sX;  // X is no longer read
    for (int c = tid >> 5; c < dk; c += kBwThreads / 32) {
        float acc = 0.f;
        for (int cc = tid & 31; cc < dv; cc += 32) acc += m.dSn[c * dv + cc] * m.S[c * dv + cc];
        for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if ((tid & 31) == 0) sss[c] = acc;
    }
    float *srow = sY;  // one gate per (token, head): the per-channel gradients summed per row
    for (int r = tid; r < C; r += kBwThreads) srow[r] = 0.f;
    __syncthreads();
    for (int c = tid; c < dk; c += kBwThreads) {
        const float g = m.G[(n - 1) * dk + c];
        float dg = 0.f;
        for (int r = 0; r < n; ++r) dg += m.dKd[r * dk + c] * m.Kd[r * dk + c];
        dg += expf(g) * sss[c];
        float run = 0.f;
        for (int r = n - 1; r >= 0; --r) {
            const int e = r * dk + c;
            run += m.dQg[e] * m.Qg[e] + m.dKg[e] * m.Kg[e] - m.dKn[e] * m.Kn[e] - m.dKd[e] * m.Kd[e];
            const size_t row = (size_t)(t0 + r) * a.H + h;
            if (a.la_scalar) atomicAdd(&srow[r], run + dg);
            else a.dla[row * dk + c] = run + dg;
            const float G = m.G[e];
            a.dqh[row * dk + c] = m.dQg[e] * expf(G);
            a.dkh[row * dk + c] = m.dKg[e] * expf(G) + m.dKn[e] * expf(-G) + m.dKd[e] * expf(g - G);
        }
    }
    if (a.la_scalar) {
        __syncthreads();
        for (int r = tid; r < n; r += kBwThreads) a.dla[(size_t)(t0 + r) * a.H + h] = srow[r];
    }
}

// 5. Through x / max(|x|, eps): a warp per (token, head).
__global__ void __launch_bounds__(kBwThreads) bw_norm(BwArgs a) {
    const int64_t w = ((int64_t)blockIdx.x * kBwThreads + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31, dk = a.dk;
    if (w >= a.total * a.H) return;
    for (int which = 0; which < 2; ++which) {
        const float *xh = which ? a.kh : a.qh, *dxh = which ? a.dkh : a.dqh;
        const float nrm = (which ? a.nk : a.nq)[w];
        float *dx = which ? a.dkk : a.dq;
        float dot = 0.f;
        for (int c = lane; c < dk; c += 32) dot += xh[w * dk + c] * dxh[w * dk + c];
        for (int off = 16; off; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        for (int c = lane; c < dk; c += 32) {
            const float g = dxh[w * dk + c];
            float out = g;
            if (a.l2norm) out = nrm > a.eps ? (g - xh[w * dk + c] * dot) / nrm : g / a.eps;
            dx[w * dk + c] = out;
        }
    }
}

template <typename T>
cudaError_t run(const BwArgs &a, cudaStream_t st) {
    const unsigned units = (unsigned)a.N * (unsigned)a.H, groups = (unsigned)(a.dv / kCols);
    const size_t fwd_smem = fwd_smem_floats(a.dk) * sizeof(float), bwd_smem = bwd_smem_floats(a.dk) * sizeof(float);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(bw_fwd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fwd_smem)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(bw_bwd<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bwd_smem)) !=
        cudaSuccess)
        return e;
    const size_t prep_smem = 2 * (size_t)C * (C + 1) * sizeof(float);  // >= the three 64 x 33 tiles
    if ((e = cudaFuncSetAttribute(bw_prep<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_smem)) !=
        cudaSuccess)
        return e;
    bw_offsets<<<1, 1024, 0, st>>>(a);
    const unsigned slots = (unsigned)a.H * (unsigned)a.NC;
    bw_prep<T><<<slots, kBwThreads, prep_smem, st>>>(a);
    bw_fwd<<<units * groups, kBwThreads, fwd_smem, st>>>(a);
    bw_bwd<T><<<units * groups, kBwThreads, bwd_smem, st>>>(a);
    const size_t rs_smem = rs_smem_floats(a.dk) * sizeof(float);
    if ((e = cudaFuncSetAttribute(bw_rowstate<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rs_smem)) !=
        cudaSuccess)
        return e;
    bw_rowstate<T><<<slots, kBwThreads, rs_smem, st>>>(a);
    const size_t gr_smem = 3 * (size_t)C * (C + 1) * sizeof(float);
    if ((e = cudaFuncSetAttribute(bw_grads<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gr_smem)) !=
        cudaSuccess)
        return e;
    bw_grads<T><<<slots, kBwThreads, gr_smem, st>>>(a);
    const int64_t warps = a.total * a.H;
    if (warps > 0) bw_norm<<<(unsigned)((warps * 32 + kBwThreads - 1) / kBwThreads), kBwThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

int64_t backward_slots_per_head(int N, int64_t total) { return total / C + N; }  // >= sum of ceil(len / 64)

size_t backward_workspace_bytes(int N, int H, int64_t total, int dk, int dv) {
    const Slot sl{dk, dv};
    return ((size_t)backward_slots_per_head(N, total) * H * sl.floats() + (size_t)total * H * (4 * (size_t)dk + 2) +
            ((size_t)N + 4) / 4 * 4) * sizeof(float);
}

cudaError_t backward(const BackwardArgs &b, bool bf16, cudaStream_t st) {
    BwArgs a;
    a.q = b.q; a.k = b.k; a.v = b.v; a.dout = b.dout;
    a.la = b.log_alpha; a.beta = b.beta; a.S0 = b.S0; a.dST = b.dS_T; a.cu = b.cu;
    a.total = b.total; a.N = b.N; a.H = b.H; a.dk = b.dk; a.dv = b.dv;
    a.NC = (int)backward_slots_per_head(b.N, b.total);
    a.l2norm = b.l2norm; a.la_scalar = b.la_scalar; a.eps = b.eps;
    a.dq = b.dq; a.dkk = b.dk_out; a.dvv = b.dv_out; a.dla = b.dlog_alpha; a.dbeta = b.dbeta; a.dS0 = b.dS0;
    const Slot sl{b.dk, b.dv};
    float *p = static_cast<float *>(b.ws);
    a.slots = p;
    p += (size_t)a.NC * b.H * sl.floats();
    const size_t th = (size_t)b.total * b.H;
    a.qh = p; p += th * b.dk;
    a.kh = p; p += th * b.dk;
    a.dqh = p; p += th * b.dk;
    a.dkh = p; p += th * b.dk;
    a.nq = p; p += th;
    a.nk = p; p += th;
    a.coff = reinterpret_cast<int *>(p);
    a.err = b.err;
    return bf16 ? run<__nv_bfloat16>(a, st) : run<float>(a, st);
}

}  // namespace kda
