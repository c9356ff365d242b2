// kda_prefill_tc.cu -- chunkwise KDA prefill on the sm_100a tensor cores
// (bf16 q/k/v, d_k = d_v = 128, chunk C = 64, fp32 state).
//
// Math ("[Kimi-2] Kimi Linear：用 KDA 重写长上下文注意力" §5, the UT transform and the
// inter-/intra-chunk split; §3 for the per-token update it rearranges). Per chunk
// with entry state S, G = cumulative sum of log_alpha over the chunk's rows:
//   Gram:  [A ; P] = [K e^G ; Q e^G] (K e^-G)^T      (masked: A strictly lower, P lower)
//   solve: T = (I + Diag(beta) A)^{-1} Diag(beta),   W = T (K e^G)
//   scan:  U = T V - W S,  O = (Q e^G) S + P U,  S' = Diag(e^{G_last}) S + (K e^{G_last-G})^T U
//
// Two kernels per wave of chunks, plus an exact fallback:
//  * prep_kernel (one CTA per chunk x head, all chunks of the wave in parallel):
//    L2 norm, G, the exponentiated operands, the Gram on the tensor cores
//    (one M=128 tcgen05.mma stacking K e^G over Q e^G), the 64x64 triangular
//    solve on the CUDA cores (16x16 blocks), W^T = (K e^G)^T T^T on the tensor
//    cores, and the whole workspace slot assembled in shared memory in the
//    scan's operand layout and written with one TMA bulk store.
//    The factorisation e^{G_r - G_i} = e^{G_r} e^{-G_i} needs e^{-G} to stay
//    finite; chunks whose decay range exceeds kTau are queued instead.
//  * fix_kernel: recomputes queued chunks in fp32 with element-wise exponents.
//  * scan_kernel (one CTA per sequence x head x 64-column tile of d_v): the
//    slot of chunk j+1 arrives by TMA bulk copy while chunk j computes; all
//    products are M=128 tcgen05.mma with fp32 accumulators in TMEM; the fp32
//    state lives in registers (thread = state row = TMEM lane) and a bf16 copy
//    in shared memory feeds the next chunk's products.
#include "kda_internal.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace {

using namespace tc;
using bf16 = __nv_bfloat16;

constexpr int C = kChunk;  // 64
constexpr int DK = 128;
constexpr int DV = 128;
constexpr int DVT = 64;                    // state columns per scan CTA
constexpr float kTau = 60.f;               // largest per-chunk decay range for the factorised Gram
constexpr uint64_t kWaitNs = 2000000000ull;  // bound of every device-side wait (2 s)

// ---------------------------------------------------------------- slot ----
// One slot per (chunk, sequence, head), bytes (every tile 1024-byte aligned):
//   WQ [W ; Q e^G]   128 x 128 bf16, K-major SW128      (A operand of [W;Qg] S)
//   KD K e^{Gl-G}    64 (r) x 128 (c) bf16, MN-major     (A operand of Kd^T U)
//   T                64 x 64 bf16, K-major               (A operand of T V)
//   P                64 x 64 bf16, K-major               (A operand of P U)
//   D  e^{G_last}    128 fp32
constexpr uint32_t SL_WQ = 0, SL_KD = 32768, SL_T = 49152, SL_P = 57344, SL_D = 65536;
constexpr uint32_t SL_USED = 66048, SL_BYTES = 66560;

__device__ __forceinline__ void load8_bf16(const bf16 *p, float (&x)[8]) {
    unpack8(__ldg(reinterpret_cast<const uint4 *>(p)), x);
}

// Records a device-side failure (first one wins) for kda_device_error().
__device__ __forceinline__ void flag_error(int *err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// ---------------------------------------------------------------- prep ----
constexpr int PT = 256;
constexpr uint32_t PS_SL = 0;                    // slot staging (66560); WQ first holds [Kg ; Qg]
constexpr uint32_t PS_GB = 66560;                // K e^-G, K-major 64 x 128 (B of the Gram)
constexpr uint32_t PS_KGT = PS_GB + 16384;       // K e^G,  MN-major 64 x 128 (A of W^T)
constexpr uint32_t PS_GF = PS_KGT + 16384;       // fp32 G [64][128]; later X [64][65]
constexpr uint32_t PS_AF = PS_GF + 33280;        // fp32 A [64][65] (strictly lower, upper blocks scratch)
constexpr uint32_t PS_SMALL = PS_AF + 16640;     // invq[64] invk[64] beta[64] gl[128]
constexpr uint32_t PS_BAR = PS_SMALL + 1280;     // 2 mbarriers, tmem base, flags
constexpr uint32_t PS_BYTES = PS_BAR + 64;
constexpr uint32_t PS_ALLOC = PS_BYTES + 1024;   // + alignment slack

__global__ void __launch_bounds__(PT, 1)
prep_kernel(const bf16 *__restrict__ q, const bf16 *__restrict__ k, const float *__restrict__ la,
            const float *__restrict__ beta, const int32_t *__restrict__ cu, int64_t total, int H,
            int N, int j0, int l2norm, float eps, char *__restrict__ slots, int *__restrict__ fix,
            int fix_cap, int *__restrict__ err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int jl = blockIdx.x, s = blockIdx.y, h = blockIdx.z;
    int64_t bos, eos;
    seq_bounds(cu, s, total, bos, eos);
    const int64_t j = (int64_t)j0 + jl;
    if (j * C >= eos - bos) return;
    const int n = (int)((eos - bos - j * C) < C ? (eos - bos - j * C) : C);
    const int64_t t0 = bos + j * C;
    const int slot_id = (jl * N + s) * H + h;
    char *gslot = slots + (size_t)slot_id * SL_BYTES;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t *GA = sm + PS_SL + SL_WQ;
    uint8_t *GB = sm + PS_GB;
    uint8_t *KGT = sm + PS_KGT;
    float *GF = reinterpret_cast<float *>(sm + PS_GF);
    float *AF = reinterpret_cast<float *>(sm + PS_AF);
    float *invq = reinterpret_cast<float *>(sm + PS_SMALL);
    float *invk = invq + 64, *sbeta = invk + 64, *sgl = sbeta + 64;
    float *Dv = reinterpret_cast<float *>(sm + PS_SL + SL_D);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + PS_BAR);
    uint32_t *tbase = reinterpret_cast<uint32_t *>(bars + 2);
    int *sflag = reinterpret_cast<int *>(tbase + 1);  // [0] unsafe range, [1] wait failed

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        sflag[0] = 0;
        sflag[1] = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tbase, 128);
        tmem_relinquish();
    }
    __syncthreads();  // flags and barriers initialised before anyone sets them

    // 1. G (threads = key channels) | row norms and beta (warps 4..7).
    if (tid < DK) {
        const int c = tid;
        const float *src = la + ((size_t)t0 * H + h) * DK + c;
        const size_t stride = (size_t)H * DK;
        float run = 0.f;
#pragma unroll 8
        for (int r = 0; r < C; ++r) {
            run += (r < n) ? __ldg(src + (size_t)r * stride) : 0.f;
            GF[r * DK + c] = run;
        }
        sgl[c] = run;
        Dv[c] = expf(run);
        if (-run > kTau) sflag[0] = 1;
    } else {
        const int w = warp - 4;
        for (int rr = 0; rr < 16; ++rr) {
            const int r = w * 16 + rr;
            float sq = 0.f, sk = 0.f;
            if (r < n) {
                const size_t off = ((size_t)(t0 + r) * H + h) * DK + lane * 4;
                const uint2 qv = __ldg(reinterpret_cast<const uint2 *>(q + off));
                const uint2 kv = __ldg(reinterpret_cast<const uint2 *>(k + off));
                const uint32_t qw[2] = {qv.x, qv.y}, kw[2] = {kv.x, kv.y};
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float a = __uint_as_float(qw[i] << 16), b = __uint_as_float(qw[i] & 0xFFFF0000u);
                    const float c2 = __uint_as_float(kw[i] << 16), d = __uint_as_float(kw[i] & 0xFFFF0000u);
                    sq += a * a + b * b;
                    sk += c2 * c2 + d * d;
                }
            }
#pragma unroll
            for (int off = 16; off; off >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, off);
                sk += __shfl_xor_sync(0xffffffffu, sk, off);
            }
            if (lane == 0) {
                const bool live = r < n;
                invq[r] = !live ? 0.f : (l2norm ? 1.f / fmaxf(sqrtf(sq), eps) : 1.f);
                invk[r] = !live ? 0.f : (l2norm ? 1.f / fmaxf(sqrtf(sk), eps) : 1.f);
            }
        }
        const int r = tid - DK;
        if (r < C) sbeta[r] = r < n ? beta[(size_t)(t0 + r) * H + h] : 0.f;
    }
    __syncthreads();
    const bool safe = sflag[0] == 0;

    // 2. Operands, one (row, 8-channel chunk) item at a time.
    for (int it = tid; it < C * (DK / 8); it += PT) {
        const int r = it >> 4, c8 = it & 15;
        float kf[8], qf[8];
        if (r < n) {
            const size_t off = ((size_t)(t0 + r) * H + h) * DK + c8 * 8;
            load8_bf16(k + off, kf);
            load8_bf16(q + off, qf);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) kf[e] = qf[e] = 0.f;
        }
        const float ik = invk[r], iq = invq[r];
        float kg[8], qg[8], kn[8], kd[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float g = GF[r * DK + c8 * 8 + e];
            const float ep = __expf(g), en = __expf(-g);
            const float kk = kf[e] * ik;
            kg[e] = kk * ep;
            qg[e] = qf[e] * iq * ep;
            kn[e] = kk * en;
            kd[e] = kn[e] * Dv[c8 * 8 + e];
        }
        const uint4 ukg = pack8(kg);
        *reinterpret_cast<uint4 *>(GA + kmaj_chunk(r, c8, 128)) = ukg;
        *reinterpret_cast<uint4 *>(GA + kmaj_chunk(64 + r, c8, 128)) = pack8(qg);
        *reinterpret_cast<uint4 *>(GB + kmaj_chunk(r, c8, 64)) = pack8(kn);
        *reinterpret_cast<uint4 *>(KGT + mnmaj_chunk(r, c8, 64)) = ukg;
        *reinterpret_cast<uint4 *>(sm + PS_SL + SL_KD + mnmaj_chunk(r, c8, 64)) = pack8(kd);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tbase;

    if (!safe) {
        // Decay range too large for e^{-G}: leave the slot to the exact fallback.
        if (tid == 0) {
            const int pos = atomicAdd(fix, 1);
            if (pos < fix_cap) fix[1 + pos] = slot_id;
            else flag_error(err, 2);
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) tmem_dealloc(tm, 128);
        return;
    }

    // 3. Gram on the tensor cores: TMEM cols [0,64) = [Kg ; Qg] (K e^-G)^T.
    if (tid == 0) {
        const uint32_t a = smem_u32(GA), b = smem_u32(GB);
        const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int st = 0; st < DK / 16; ++st) mma_bf16(tm, kmaj_desc(a, st, 128), kmaj_desc(b, st, 64), id, st > 0);
        mma_commit(&bars[0]);
    }
    if (!mbar_wait(&bars[0], 0, kWaitNs)) sflag[1] = 1;
    tc_fence_after();

    // 4. A (fp32, strictly lower) to smem; P (bf16, lower incl. diagonal) to the slot.
    if (warp < 4) {
        const int row = warp * 32 + lane;
        for (int c0 = 0; c0 < C; c0 += 16) {
            float v[16];
            tmem_ld16(tm + ((uint32_t)(warp * 32) << 16) + c0, v);
            tmem_wait_ld();
            if (row < C) {
#pragma unroll
                for (int i = 0; i < 16; ++i) AF[row * 65 + c0 + i] = (c0 + i < row) ? v[i] : 0.f;
            } else {
                const int r = row - C;
                float lo[8], hi[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    lo[i] = (c0 + i <= r) ? v[i] : 0.f;
                    hi[i] = (c0 + 8 + i <= r) ? v[8 + i] : 0.f;
                }
                *reinterpret_cast<uint4 *>(sm + PS_SL + SL_P + kmaj_chunk(r, c0 / 8, 64)) = pack8(lo);
                *reinterpret_cast<uint4 *>(sm + PS_SL + SL_P + kmaj_chunk(r, c0 / 8 + 1, 64)) = pack8(hi);
            }
        }
    }
    __syncthreads();

    // 5. X = (I + Diag(beta) A)^{-1} by 16x16 blocks; T = X Diag(beta).
    float *X = GF;  // [64][65]
    if (tid < C) {
        // diagonal blocks: column cc of block b by forward substitution
        const int b = tid >> 4, cc = tid & 15;
        float x[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            const int r = 16 * b + rr;
            float acc = 0.f;
#pragma unroll
            for (int ii = 0; ii < rr; ++ii) acc += AF[r * 65 + 16 * b + ii] * x[ii];
            x[rr] = (rr == cc) ? 1.f : (rr > cc ? -sbeta[r] * acc : 0.f);
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) X[(16 * b + rr) * 65 + 16 * b + cc] = x[rr];
    }
    __syncthreads();
    for (int d = 1; d < 4; ++d) {
        // R_ij = Diag(beta_i) sum_{k=j}^{i-1} A_ik X_kj  (kept in the unused upper block (j, i) of AF)
        for (int e = tid; e < (4 - d) * 256; e += PT) {
            const int jb = e >> 8, ib = jb + d, rr = (e >> 4) & 15, cc = e & 15;
            const int r = 16 * ib + rr;
            float acc = 0.f;
            for (int kb = jb; kb < ib; ++kb)
#pragma unroll
                for (int t = 0; t < 16; ++t) acc += AF[r * 65 + 16 * kb + t] * X[(16 * kb + t) * 65 + 16 * jb + cc];
            AF[(16 * jb + rr) * 65 + 16 * ib + cc] = sbeta[r] * acc;
        }
        __syncthreads();
        // X_ij = -X_ii R_ij
        for (int e = tid; e < (4 - d) * 256; e += PT) {
            const int jb = e >> 8, ib = jb + d, rr = (e >> 4) & 15, cc = e & 15;
            float acc = 0.f;
#pragma unroll
            for (int t = 0; t < 16; ++t)
                acc += X[(16 * ib + rr) * 65 + 16 * ib + t] * AF[(16 * jb + t) * 65 + 16 * ib + cc];
            X[(16 * ib + rr) * 65 + 16 * jb + cc] = -acc;
        }
        __syncthreads();
    }
    for (int it = tid; it < C * 8; it += PT) {
        const int r = it >> 3, c8 = it & 7;
        float t8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int c = c8 * 8 + e;
            t8[e] = (c <= r) ? X[r * 65 + c] * sbeta[c] : 0.f;
        }
        *reinterpret_cast<uint4 *>(sm + PS_SL + SL_T + kmaj_chunk(r, c8, 64)) = pack8(t8);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // 6. W^T = (K e^G)^T T^T on the tensor cores: TMEM cols [64,128), lane = key channel.
    if (tid == 0) {
        const uint32_t a = smem_u32(KGT), b = smem_u32(sm + PS_SL + SL_T);
        const uint32_t id = idesc_bf16(128, 64, true, false);
#pragma unroll
        for (int st = 0; st < C / 16; ++st) mma_bf16(tm + 64, mnmaj_desc(a, st, 64), kmaj_desc(b, st, 64), id, st > 0);
        mma_commit(&bars[1]);
    }
    if (!mbar_wait(&bars[1], 0, kWaitNs)) sflag[1] = 1;
    tc_fence_after();

    // 7. W rows into the top half of WQ (its Kg rows are no longer needed).
    if (warp < 4) {
        const int c = warp * 32 + lane;
        for (int c0 = 0; c0 < C; c0 += 16) {
            float v[16];
            tmem_ld16(tm + ((uint32_t)(warp * 32) << 16) + 64 + c0, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i)
                *reinterpret_cast<bf16 *>(GA + kmaj_off(c0 + i, c, 128)) = __float2bfloat16_rn(v[i]);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // 8. The assembled slot goes out in one bulk store.
    if (tid == 0) {
        if (sflag[1]) flag_error(err, 1);
        bulk_s2g(gslot, sm + PS_SL, SL_USED);
        bulk_commit();
        bulk_wait_read();
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 128);
}

// ----------------------------------------------------------------- fix ----
// Exact fallback for queued chunks: element-wise exponents e^{G_r - G_i} <= 1.
constexpr int FT = 256;
constexpr int FLD = DK + 1;
constexpr size_t FS_BYTES = (size_t)(3 * C * FLD + 3 * C * (C + 1) + C) * 4;

__global__ void __launch_bounds__(FT)
fix_kernel(const bf16 *__restrict__ q, const bf16 *__restrict__ k, const float *__restrict__ la,
           const float *__restrict__ beta, const int32_t *__restrict__ cu, int64_t total, int H, int N,
           int j0, int l2norm, float eps, char *__restrict__ slots, const int *__restrict__ fix,
           int fix_cap) {
    extern __shared__ float fsm[];
    float *sK = fsm, *sQ = sK + C * FLD, *sG = sQ + C * FLD;
    float *sA = sG + C * FLD, *sP = sA + C * (C + 1), *sT = sP + C * (C + 1), *sB = sT + C * (C + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int count = min(fix[0], fix_cap);
    for (int e = blockIdx.x; e < count; e += gridDim.x) {
        const int slot_id = fix[1 + e];
        const int h = slot_id % H, s = (slot_id / H) % N, jl = slot_id / (H * N);
        int64_t bos, eos;
        seq_bounds(cu, s, total, bos, eos);
        const int64_t j = (int64_t)j0 + jl;
        const int n = (int)((eos - bos - j * C) < C ? (eos - bos - j * C) : C);
        const int64_t t0 = bos + j * C;
        uint8_t *g = reinterpret_cast<uint8_t *>(slots + (size_t)slot_id * SL_BYTES);
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += FT) {
            const int r = idx / DK, c = idx % DK;
            float kv = 0.f, qv = 0.f, lv = 0.f;
            if (r < n) {
                const size_t off = ((size_t)(t0 + r) * H + h) * DK + c;
                kv = __bfloat162float(k[off]);
                qv = __bfloat162float(q[off]);
                lv = la[off];
            }
            sK[r * FLD + c] = kv;
            sQ[r * FLD + c] = qv;
            sG[r * FLD + c] = lv;
        }
        if (tid < C) sB[tid] = tid < n ? beta[(size_t)(t0 + tid) * H + h] : 0.f;
        __syncthreads();
        if (l2norm) {
            for (int r = warp; r < C; r += FT / 32) {
                float a = 0.f, b = 0.f;
                for (int c = lane; c < DK; c += 32) {
                    a += sK[r * FLD + c] * sK[r * FLD + c];
                    b += sQ[r * FLD + c] * sQ[r * FLD + c];
                }
#pragma unroll
                for (int off = 16; off; off >>= 1) {
                    a += __shfl_xor_sync(0xffffffffu, a, off);
                    b += __shfl_xor_sync(0xffffffffu, b, off);
                }
                const float ia = 1.f / fmaxf(sqrtf(a), eps), ib = 1.f / fmaxf(sqrtf(b), eps);
                for (int c = lane; c < DK; c += 32) {
                    sK[r * FLD + c] *= ia;
                    sQ[r * FLD + c] *= ib;
                }
            }
        }
        if (tid < DK) {
            float run = 0.f;
            for (int r = 0; r < C; ++r) {
                run += sG[r * FLD + tid];
                sG[r * FLD + tid] = run;
            }
        }
        __syncthreads();
        for (int p = tid; p < C * C; p += FT) {
            const int r = p / C, i = p % C;
            float a = 0.f, pp = 0.f;
            if (i <= r)
                for (int c = 0; c < DK; ++c) {
                    const float ex = expf(sG[r * FLD + c] - sG[i * FLD + c]);
                    const float ki = sK[i * FLD + c] * ex;
                    a += sK[r * FLD + c] * ki;
                    pp += sQ[r * FLD + c] * ki;
                }
            sA[r * (C + 1) + i] = (i < r) ? a : 0.f;
            sP[r * (C + 1) + i] = pp;
        }
        __syncthreads();
        if (tid < C) {
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
        }
        __syncthreads();
        // Q e^G -> WQ rows 64..127; K e^{Gl-G} -> KD; D; K e^G kept in sK
        for (int idx = tid; idx < C * DK; idx += FT) {
            const int r = idx / DK, c = idx % DK;
            const float gg = sG[r * FLD + c], gl = sG[(C - 1) * FLD + c];
            const float ex = expf(gg);
            *reinterpret_cast<bf16 *>(g + SL_WQ + kmaj_off(64 + r, c, 128)) = __float2bfloat16_rn(sQ[r * FLD + c] * ex);
            *reinterpret_cast<bf16 *>(g + SL_KD + mnmaj_off(r, c, 64)) = __float2bfloat16_rn(sK[r * FLD + c] * expf(gl - gg));
        }
        for (int c = tid; c < DK; c += FT) reinterpret_cast<float *>(g + SL_D)[c] = expf(sG[(C - 1) * FLD + c]);
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += FT) {
            const int r = idx / DK, c = idx % DK;
            sK[r * FLD + c] *= expf(sG[r * FLD + c]);
        }
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += FT) {
            const int r = idx / DK, c = idx % DK;
            float acc = 0.f;
            for (int i = 0; i <= r; ++i) acc += sT[r * (C + 1) + i] * sK[i * FLD + c];
            *reinterpret_cast<bf16 *>(g + SL_WQ + kmaj_off(r, c, 128)) = __float2bfloat16_rn(acc);
        }
        for (int idx = tid; idx < C * C; idx += FT) {
            const int r = idx / C, c = idx % C;
            *reinterpret_cast<bf16 *>(g + SL_T + kmaj_off(r, c, 64)) = __float2bfloat16_rn(sT[r * (C + 1) + c]);
            *reinterpret_cast<bf16 *>(g + SL_P + kmaj_off(r, c, 64)) = __float2bfloat16_rn(sP[r * (C + 1) + c]);
        }
    }
}

// ---------------------------------------------------------------- scan ----
constexpr int ST = 128;
// shared memory (bytes): two slot buffers, then V, S (bf16), U (bf16), barriers
constexpr uint32_t SB_WQ = 0, SB_KD = 32768, SB_TT = 49152, SB_PP = 65536, SB_D = 81920, SB_BYTES = 82944;
constexpr uint32_t SS_V = 2 * SB_BYTES;          // [64 (i)][64 (j)] MN-major
constexpr uint32_t SS_S = SS_V + 8192;           // [128 (c)][64 (j)] MN-major
constexpr uint32_t SS_U = SS_S + 16384;          // [64 (r)][64 (j)] MN-major
constexpr uint32_t SS_BAR = SS_U + 8192;         // full[2], bU, bS, tmem base, flag
constexpr uint32_t SS_BYTES = SS_BAR + 64;
constexpr uint32_t SS_ALLOC = SS_BYTES + 1024;
constexpr uint32_t SLOT_COPY_BYTES = 32768 + 16384 + 2 * 8192 + 8192 + 512;
// TMEM columns: X (two buffers), Y, Z
constexpr uint32_t TM_X0 = 0, TM_X1 = 64, TM_Y = 128, TM_Z = 192;

__device__ __forceinline__ void issue_slot_copy(uint8_t *buf, const char *g, uint64_t *bar) {
    mbar_arrive_expect_tx(bar, SLOT_COPY_BYTES);
    bulk_g2s(buf + SB_WQ, g + SL_WQ, 32768, bar);
    bulk_g2s(buf + SB_KD, g + SL_KD, 16384, bar);
    bulk_g2s(buf + SB_TT, g + SL_T, 8192, bar);
    bulk_g2s(buf + SB_TT + 8192, g + SL_T, 8192, bar);
    bulk_g2s(buf + SB_PP + 8192, g + SL_P, 8192, bar);
    bulk_g2s(buf + SB_D, g + SL_D, 512, bar);
}

__global__ void __launch_bounds__(ST, 1)
scan_kernel(const bf16 *__restrict__ v, const int32_t *__restrict__ cu, int64_t total, int H, int N,
            int j0, int nw, const char *__restrict__ slots, const float *__restrict__ S0,
            float *__restrict__ state, float *__restrict__ S_T, bf16 *__restrict__ o,
            int *__restrict__ err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int jv = blockIdx.x, s = blockIdx.y, h = blockIdx.z;
    int64_t bos, eos;
    seq_bounds(cu, s, total, bos, eos);
    const int64_t len = eos - bos;
    const int nch = (int)((len + C - 1) / C);
    if (j0 >= nch && !(nch == 0 && j0 == 0)) return;
    const int jend = min(j0 + nw, nch);
    const int nj = jend - j0 > 0 ? jend - j0 : 0;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t *sV = sm + SS_V, *sS = sm + SS_S, *sU = sm + SS_U;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SS_BAR);  // full0, full1, bU, bS
    uint32_t *tbase = reinterpret_cast<uint32_t *>(bars + 4);
    int *sfail = reinterpret_cast<int *>(tbase + 1);
    const size_t sofs = ((size_t)s * H + h) * DK * DV + (size_t)jv * DVT;
    const int c = tid;  // state row owned by this thread (= TMEM lane)

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        *sfail = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tbase, 256);
        tmem_relinquish();
    }
    // Rows 0..63 of both [0 ; P] operand buffers stay zero.
    for (int i = tid; i < 2 * 512; i += ST) {
        uint8_t *b = sm + (i >> 9) * SB_BYTES + SB_PP;
        reinterpret_cast<uint4 *>(b)[i & 511] = make_uint4(0, 0, 0, 0);
    }
    // Entry state: S0 (or zeros) on the first wave, else the carry.
    float Sr[DVT];
    {
        const float *Sin = (j0 == 0) ? S0 : state;
#pragma unroll
        for (int q4 = 0; q4 < DVT / 4; ++q4) {
            float4 x = Sin ? *reinterpret_cast<const float4 *>(Sin + sofs + (size_t)c * DV + 4 * q4)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            Sr[4 * q4] = x.x; Sr[4 * q4 + 1] = x.y; Sr[4 * q4 + 2] = x.z; Sr[4 * q4 + 3] = x.w;
        }
    }
    auto store_state_bf16 = [&]() {
#pragma unroll
        for (int c8 = 0; c8 < DVT / 8; ++c8) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = Sr[c8 * 8 + e];
            *reinterpret_cast<uint4 *>(sS + mnmaj_chunk(c, c8, DK)) = pack8(x);
        }
    };
    store_state_bf16();
    // V rows of chunk jj (zeros past the sequence end): 4 x 16 bytes per thread.
    uint4 vreg[4];
    auto load_v = [&](int jj) {
        const int nn = (int)((len - (int64_t)jj * C) < C ? (len - (int64_t)jj * C) : C);
        const int64_t tt = bos + (int64_t)jj * C;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int qi = tid + ST * m, i = qi >> 3, c8 = qi & 7;
            vreg[m] = (i < nn) ? __ldg(reinterpret_cast<const uint4 *>(v + ((size_t)(tt + i) * H + h) * DV + jv * DVT + c8 * 8))
                               : make_uint4(0, 0, 0, 0);
        }
    };
    auto store_v = [&]() {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int qi = tid + ST * m, i = qi >> 3, c8 = qi & 7;
            *reinterpret_cast<uint4 *>(sV + mnmaj_chunk(i, c8, C)) = vreg[m];
        }
    };
    auto slot_ptr = [&](int jj) {
        return slots + ((size_t)((jj - j0) * N + s) * H + h) * SL_BYTES;
    };
    if (nj > 0) {
        if (tid == 0) issue_slot_copy(sm, slot_ptr(j0), &bars[0]);
        load_v(j0);
        store_v();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tbase;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t id128 = idesc_bf16(128, DVT, false, true);    // K-major A, MN-major B
    const uint32_t idKd = idesc_bf16(128, DVT, true, true);      // MN-major A (Kd^T)
    bool ok = true;

    if (nj > 0 && tid == 0) {
        // X(j0) = [T ; T] V
        if (!mbar_wait(&bars[0], 0, kWaitNs)) *sfail = 1;
        const uint32_t a = smem_u32(sm + SB_TT), b = smem_u32(sV);
#pragma unroll
        for (int st = 0; st < C / 16; ++st) mma_bf16(tm + TM_X0, kmaj_desc(a, st, 128), mnmaj_desc(b, st, C), id128, st > 0);
    }

    for (int it = 0; it < nj && ok; ++it) {
        const int jj = j0 + it, b = it & 1;
        uint8_t *buf = sm + b * SB_BYTES;
        const int nn = (int)((len - (int64_t)jj * C) < C ? (len - (int64_t)jj * C) : C);
        const int64_t tt = bos + (int64_t)jj * C;
        const uint32_t tmX = tm + ((it & 1) ? TM_X1 : TM_X0);
        // Y = [W ; Q e^G] S ; prefetch the next slot
        if (tid == 0) {
            if (!mbar_wait(&bars[b], (it >> 1) & 1, kWaitNs)) *sfail = 1;
            if (it + 1 < nj) issue_slot_copy(sm + (b ^ 1) * SB_BYTES, slot_ptr(jj + 1), &bars[b ^ 1]);
            const uint32_t a = smem_u32(buf + SB_WQ), bs = smem_u32(sS);
#pragma unroll
            for (int st = 0; st < DK / 16; ++st) mma_bf16(tm + TM_Y, kmaj_desc(a, st, 128), mnmaj_desc(bs, st, DK), id128, st > 0);
            mma_commit(&bars[2]);
        }
        if (it + 1 < nj) load_v(jj + 1);
        if (!mbar_wait(&bars[2], it & 1, kWaitNs)) *sfail = 1;
        tc_fence_after();
        // U = X - Y (rows 0..63 live in lanes 0..63: warps 0 and 1)
        if (warp < 2) {
            const int r = c;
#pragma unroll
            for (int c0 = 0; c0 < DVT; c0 += 16) {
                float xv[16], yv[16];
                tmem_ld16(tmX + lane_base + c0, xv);
                tmem_ld16(tm + TM_Y + lane_base + c0, yv);
                tmem_wait_ld();
                float lo[8], hi[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    lo[e] = xv[e] - yv[e];
                    hi[e] = xv[8 + e] - yv[8 + e];
                }
                *reinterpret_cast<uint4 *>(sU + mnmaj_chunk(r, c0 / 8, C)) = pack8(lo);
                *reinterpret_cast<uint4 *>(sU + mnmaj_chunk(r, c0 / 8 + 1, C)) = pack8(hi);
            }
        }
        if (it + 1 < nj) store_v();
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // O: Y += [0 ; P] U ; Z = Kd^T U ; then X(j+1) = [T ; T] V(j+1)
        if (tid == 0) {
            const uint32_t bu = smem_u32(sU);
            const uint32_t ap = smem_u32(buf + SB_PP), ak = smem_u32(buf + SB_KD);
#pragma unroll
            for (int st = 0; st < C / 16; ++st) mma_bf16(tm + TM_Y, kmaj_desc(ap, st, 128), mnmaj_desc(bu, st, C), id128, 1);
#pragma unroll
            for (int st = 0; st < C / 16; ++st) mma_bf16(tm + TM_Z, mnmaj_desc(ak, st, C), mnmaj_desc(bu, st, C), idKd, st > 0);
            mma_commit(&bars[3]);
            if (it + 1 < nj) {
                uint8_t *nbuf = sm + (b ^ 1) * SB_BYTES;
                if (!mbar_wait(&bars[b ^ 1], ((it + 1) >> 1) & 1, kWaitNs)) *sfail = 1;
                const uint32_t a = smem_u32(nbuf + SB_TT), bv = smem_u32(sV);
                const uint32_t tmXn = tm + ((it & 1) ? TM_X0 : TM_X1);
#pragma unroll
                for (int st = 0; st < C / 16; ++st) mma_bf16(tmXn, kmaj_desc(a, st, 128), mnmaj_desc(bv, st, C), id128, st > 0);
            }
        }
        if (!mbar_wait(&bars[3], it & 1, kWaitNs)) *sfail = 1;
        if (!mbar_wait(&bars[b], (it >> 1) & 1, kWaitNs)) *sfail = 1;  // D of this chunk
        tc_fence_after();
        // S' = Diag(e^{G_last}) S + Z   (row c)
        {
            const float dc = reinterpret_cast<const float *>(buf + SB_D)[c];
#pragma unroll
            for (int c0 = 0; c0 < DVT; c0 += 16) {
                float zv[16];
                tmem_ld16(tm + TM_Z + lane_base + c0, zv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) Sr[c0 + e] = dc * Sr[c0 + e] + zv[e];
            }
            store_state_bf16();
        }
        // O rows live in lanes 64..127 (warps 2, 3)
        if (warp >= 2) {
            const int r = c - 64;
#pragma unroll
            for (int c0 = 0; c0 < DVT; c0 += 16) {
                float yv[16];
                tmem_ld16(tm + TM_Y + lane_base + c0, yv);
                tmem_wait_ld();
                if (r < nn) {
                    bf16 *dst = o + ((size_t)(tt + r) * H + h) * DV + jv * DVT + c0;
                    float lo[8], hi[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        lo[e] = yv[e];
                        hi[e] = yv[8 + e];
                    }
                    reinterpret_cast<uint4 *>(dst)[0] = pack8(lo);
                    reinterpret_cast<uint4 *>(dst)[1] = pack8(hi);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        ok = (*sfail == 0);
    }
    if (!ok) {
        if (tid == 0) flag_error(err, 1);
    }

    // Exit: final state when the sequence ended in this wave, else the carry.
    float *Sout = (jend == nch) ? S_T : state;
    if (Sout && ok) {
#pragma unroll
        for (int q4 = 0; q4 < DVT / 4; ++q4)
            *reinterpret_cast<float4 *>(Sout + sofs + (size_t)c * DV + 4 * q4) =
                make_float4(Sr[4 * q4], Sr[4 * q4 + 1], Sr[4 * q4 + 2], Sr[4 * q4 + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 256);
}

}  // namespace

size_t tc_slot_bytes() { return SL_BYTES; }

cudaError_t tc_prefill_wave(const PrefillArgs &a, int j0, int nw, int *fix, int fix_cap, int *err,
                            cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PS_ALLOC);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FS_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SS_ALLOC);
    if (e != cudaSuccess) return e;
    if (nw > 0) {
        e = cudaMemsetAsync(fix, 0, sizeof(int), st);
        if (e != cudaSuccess) return e;
        prep_kernel<<<dim3(nw, a.N, a.H), PT, PS_ALLOC, st>>>(
            (const bf16 *)a.q, (const bf16 *)a.k, a.log_alpha, a.beta, a.cu, a.total, a.H, a.N, j0,
            a.l2norm, a.eps, a.slots, fix, fix_cap, err);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        fix_kernel<<<148, FT, FS_BYTES, st>>>((const bf16 *)a.q, (const bf16 *)a.k, a.log_alpha, a.beta,
                                              a.cu, a.total, a.H, a.N, j0, a.l2norm, a.eps, a.slots,
                                              fix, fix_cap);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    scan_kernel<<<dim3(DV / DVT, a.N, a.H), ST, SS_ALLOC, st>>>(
        (const bf16 *)a.v, a.cu, a.total, a.H, a.N, j0, nw, a.slots, a.S0, a.state, a.S_T, (bf16 *)a.o, err);
    return cudaGetLastError();
}

}  // namespace kda
