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
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include <mutex>

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
//   WQ [Q e^G ; W]   128 x 128 bf16, K-major SW128      (A operand of [Qg;W] S)
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
// Persistent, two CTAs per SM (~84 KB shared memory each), each walking the
// wave's (chunk, sequence, head) items. q and k stay in registers (coalesced
// 16-byte loads); log_alpha arrives by one tensor-map TMA box and is turned
// into G in place; that buffer is then reused for A, X and the solve's
// scratch. The slot's WQ and T tiles leave by TMA bulk stores; KD, P and D
// are stored straight from registers.
constexpr int PT = 256;
constexpr uint32_t PS_LA = 0;                     // log_alpha -> G [64][128] fp32; later A, X
constexpr uint32_t PS_GA = 34816;                 // [Qg ; Kg] K-major 128 x 128 -> WQ   (34 * 1024)
constexpr uint32_t PS_GB = PS_GA + 32768;         // K e^-G K-major 64 x 128; later T (8 KB) + R2
constexpr uint32_t PS_SMALL = PS_GB + 16384;      // invq[64] invk[64] beta[64] eGl[128]
constexpr uint32_t PS_BAR = PS_SMALL + 1280;      // la, mma barriers; tmem base; flags
constexpr uint32_t PS_BYTES = PS_BAR + 64;
constexpr uint32_t PS_ALLOC = PS_BYTES + 1024;    // + alignment slack
constexpr int ALD = 68, XLD = 64;                 // row strides of A and X (floats)
constexpr uint32_t PS_AF = PS_LA, PS_X = PS_LA + 17408;
constexpr uint32_t PS_T = PS_GB, PS_R2 = PS_GB + 8192;

struct Item {
    int64_t t0;
    int n, h, slot;
};

// Item `id` of the wave; false if that chunk lies past its sequence's end.
__device__ __forceinline__ bool decode_item(int id, const int32_t *cu, int64_t total, int H, int N,
                                            int j0, Item &it) {
    const int h = id % H, s = (id / H) % N, jl = id / (H * N);
    int64_t bos, eos;
    seq_bounds(cu, s, total, bos, eos);
    const int64_t j = (int64_t)j0 + jl;
    if (j * C >= eos - bos) return false;
    it.n = (int)((eos - bos - j * C) < C ? (eos - bos - j * C) : C);
    it.t0 = bos + j * C;
    it.h = h;
    it.slot = id;
    return true;
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// D (16x8) += A (16x8, row-major) x B (8x8) with tf32 operands, fp32 accumulation.
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// One warp: C[16 x 8] = A[16 x K] B[K x 8] for A(r, k), B(k, n) given as functors;
// the result is handed back through `out(r, n, value)`.
template <int K, typename FA, typename FB, typename FO>
__device__ __forceinline__ void warp_gemm_16x8(int lane, FA A, FB B, FO out) {
    const int g = lane >> 2, t = lane & 3;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < K / 8; ++ks) {
        const uint32_t a[4] = {to_tf32(A(g, 8 * ks + t)), to_tf32(A(g + 8, 8 * ks + t)),
                               to_tf32(A(g, 8 * ks + t + 4)), to_tf32(A(g + 8, 8 * ks + t + 4))};
        const uint32_t b[2] = {to_tf32(B(8 * ks + t, g)), to_tf32(B(8 * ks + t + 4, g))};
        mma_tf32(acc, a, b);
    }
    out(g, 2 * t, acc[0]);
    out(g, 2 * t + 1, acc[1]);
    out(g + 8, 2 * t, acc[2]);
    out(g + 8, 2 * t + 1, acc[3]);
}

__global__ void __launch_bounds__(PT, 2)
prep_kernel(const bf16 *__restrict__ q, const bf16 *__restrict__ k,
            const __grid_constant__ CUtensorMap tmap_la, const float *__restrict__ beta,
            const int32_t *__restrict__ cu, int64_t total, int H, int N, int j0, int nw, int l2norm,
            float eps, char *__restrict__ slots, int *__restrict__ fix, int fix_cap,
            int *__restrict__ err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int items = nw * N * H;
    float *G = reinterpret_cast<float *>(sm + PS_LA);
    float *AF = reinterpret_cast<float *>(sm + PS_AF);
    float *X = reinterpret_cast<float *>(sm + PS_X);
    float *R2 = reinterpret_cast<float *>(sm + PS_R2);
    uint8_t *GA = sm + PS_GA;
    uint8_t *GB = sm + PS_GB;
    uint8_t *TT = sm + PS_T;
    float *invq = reinterpret_cast<float *>(sm + PS_SMALL);
    float *invk = invq + 64, *sbeta = invk + 64, *eGl = sbeta + 64;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + PS_BAR);  // [0] log_alpha box, [1] MMA
    uint32_t *tbase = reinterpret_cast<uint32_t *>(bars + 2);
    int *sflag = reinterpret_cast<int *>(tbase + 1);  // [0] unsafe range, [1] wait failed, [2] next item

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        sflag[0] = 0;
        sflag[1] = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tbase, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tbase;
    uint32_t la_phase = 0, mma_phase = 0;
    const int c8 = tid & 15, rb = tid >> 4;  // thread's 16-byte channel chunk and first row

    // Items are claimed from a counter (fix[1]) so that CTAs that start late, e.g.
    // while another kernel holds SMs, simply find no work left. Thread 0 claims.
    auto claim = [&]() {
        Item tmp;
        int i = atomicAdd(&fix[1], 1);
        while (i < items && !decode_item(i, cu, total, H, N, j0, tmp)) i = atomicAdd(&fix[1], 1);
        return i;
    };
    // Inputs of an item: log_alpha by one TMA box (thread 0), q and k rows into
    // registers (rows rb + 16 m, chunk c8), beta into a register (threads < 64).
    uint4 qraw[4], kraw[4];
    float bnext = 0.f;
    auto fetch = [&](const Item &it) {
        if (tid == 0) {
            mbar_arrive_expect_tx(&bars[0], 32768u);
            tma_load_3d(G, &tmap_la, 0, it.h, (int)it.t0, &bars[0]);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int r = rb + 16 * m;
            const size_t off = ((size_t)(it.t0 + r) * H + it.h) * DK + c8 * 8;
            qraw[m] = (r < it.n) ? __ldg(reinterpret_cast<const uint4 *>(q + off)) : make_uint4(0, 0, 0, 0);
            kraw[m] = (r < it.n) ? __ldg(reinterpret_cast<const uint4 *>(k + off)) : make_uint4(0, 0, 0, 0);
        }
        bnext = (tid < it.n) ? __ldg(beta + (size_t)(it.t0 + tid) * H + it.h) : 0.f;
    };

    if (tid == 0) sflag[2] = claim();
    __syncthreads();
    Item cur;
    int id = sflag[2];
    if (id < items) {
        decode_item(id, cu, total, H, N, j0, cur);
        fetch(cur);
    }
    while (id < items) {
        const int n = cur.n;
        char *gslot = slots + (size_t)cur.slot * SL_BYTES;
        if (tid < C) sbeta[tid] = bnext;

        // 1a. Row norms: 16 lanes share a row; shuffle-reduce over them.
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            float qf[8], kf[8], sq = 0.f, sk = 0.f;
            unpack8(qraw[m], qf);
            unpack8(kraw[m], kf);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                sq += qf[e] * qf[e];
                sk += kf[e] * kf[e];
            }
#pragma unroll
            for (int off = 1; off < 16; off <<= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, off);
                sk += __shfl_xor_sync(0xffffffffu, sk, off);
            }
            const int r = rb + 16 * m;
            if (c8 == 0) {
                const bool live = r < n;
                invq[r] = !live ? 0.f : (l2norm ? 1.f / fmaxf(sqrtf(sq), eps) : 1.f);
                invk[r] = !live ? 0.f : (l2norm ? 1.f / fmaxf(sqrtf(sk), eps) : 1.f);
            }
        }
        // 1b. G = cumulative sum of log_alpha over rows, in place: thread (channel,
        //     half) scans 32 rows in registers; the upper half adds the lower total.
        if (!mbar_wait(&bars[0], la_phase, kWaitNs)) sflag[1] = 1;
        la_phase ^= 1;
        {
            const int c = tid & (DK - 1), half = tid >> 7, r0 = half * 32;
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = (r0 + i < n) ? G[(r0 + i) * DK + c] : 0.f;
#pragma unroll
            for (int i = 1; i < 32; ++i) v[i] += v[i - 1];
            if (half == 0) eGl[c] = v[31];
            __syncthreads();
            const float base = half ? eGl[c] : 0.f;
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 32; ++i) G[(r0 + i) * DK + c] = v[i] + base;
            if (half == 1) {
                const float gl = v[31] + base;
                eGl[c] = expf(gl);
                reinterpret_cast<float *>(gslot + SL_D)[c] = eGl[c];
                if (-gl > kTau) sflag[0] = 1;
            }
        }
        // GA / GB are rewritten next: the previous slot's bulk stores must have read them.
        if (tid == 0) bulk_wait_read();
        __syncthreads();
        const bool safe = sflag[0] == 0;

        if (tid == 0) sflag[2] = claim();  // next item, read by all after the sync below
        // 2. Operands for (row, 8-channel chunk): [Qg ; Kg] and K e^-G to smem, Kd to the slot.
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int r = rb + 16 * m;
            float kf[8], qf[8];
            unpack8(kraw[m], kf);
            unpack8(qraw[m], qf);
            const float ik = invk[r], iq = invq[r];
            const float4 g0 = *reinterpret_cast<const float4 *>(G + r * DK + c8 * 8);
            const float4 g1 = *reinterpret_cast<const float4 *>(G + r * DK + c8 * 8 + 4);
            const float4 d0 = *reinterpret_cast<const float4 *>(eGl + c8 * 8);
            const float4 d1 = *reinterpret_cast<const float4 *>(eGl + c8 * 8 + 4);
            const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
            float kg[8], qg[8], kn[8], kd[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float ep = __expf(gg[e]), en = __expf(-gg[e]);
                const float kk = kf[e] * ik;
                kg[e] = kk * ep;
                qg[e] = qf[e] * iq * ep;
                kn[e] = kk * en;
                kd[e] = kn[e] * dd[e];
            }
            *reinterpret_cast<uint4 *>(GA + kmaj_chunk(r, c8, 128)) = pack8(qg);
            *reinterpret_cast<uint4 *>(GA + kmaj_chunk(64 + r, c8, 128)) = pack8(kg);
            *reinterpret_cast<uint4 *>(GB + kmaj_chunk(r, c8, 64)) = pack8(kn);
            if (safe) *reinterpret_cast<uint4 *>(gslot + SL_KD + mnmaj_chunk(r, c8, 64)) = pack8(kd);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        Item nxt;
        const int nid = sflag[2];
        if (nid < items) decode_item(nid, cu, total, H, N, j0, nxt);
        if (!safe) {
            // Decay range too large for e^{-G}: the exact fallback takes this slot.
            if (tid == 0) {
                const int pos = atomicAdd(fix, 1);
                if (pos < fix_cap) fix[2 + pos] = cur.slot;
                else flag_error(err, 2);
                sflag[0] = 0;
            }
            __syncthreads();
            if (nid < items) fetch(nxt);
            id = nid;
            cur = nxt;
            continue;
        }

        // 3. Gram: TMEM cols [0,64) = [Qg ; Kg] (K e^-G)^T = [P ; A] before masking.
        if (tid == 0) {
            const uint32_t a = smem_u32(GA), b = smem_u32(GB);
            const uint32_t idg = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int st = 0; st < DK / 16; ++st) mma_bf16(tm, kmaj_desc(a, st, 128), kmaj_desc(b, st, 64), idg, st > 0);
            mma_commit(&bars[1]);
        }
        if (!mbar_wait(&bars[1], mma_phase, kWaitNs)) sflag[1] = 1;
        mma_phase ^= 1;
        tc_fence_after();

        // 4. P (bf16, lower incl. diagonal; TMEM lanes 0..63) to the slot; A (fp32,
        //    strictly lower; lanes 64..127) over the consumed G.
        if (warp < 4) {
            const int row = warp * 32 + lane;
            for (int c0 = 0; c0 < C; c0 += 16) {
                float v[16];
                tmem_ld16(tm + ((uint32_t)(warp * 32) << 16) + c0, v);
                tmem_wait_ld();
                if (row >= C) {
                    const int r = row - C;
#pragma unroll
                    for (int i4 = 0; i4 < 4; ++i4)
                        *reinterpret_cast<float4 *>(AF + r * ALD + c0 + 4 * i4) =
                            make_float4((c0 + 4 * i4 + 0 < r) ? v[4 * i4 + 0] : 0.f, (c0 + 4 * i4 + 1 < r) ? v[4 * i4 + 1] : 0.f,
                                        (c0 + 4 * i4 + 2 < r) ? v[4 * i4 + 2] : 0.f, (c0 + 4 * i4 + 3 < r) ? v[4 * i4 + 3] : 0.f);
                } else {
                    const int r = row;
                    float lo[8], hi[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        lo[i] = (c0 + i <= r) ? v[i] : 0.f;
                        hi[i] = (c0 + 8 + i <= r) ? v[8 + i] : 0.f;
                    }
                    *reinterpret_cast<uint4 *>(gslot + SL_P + kmaj_chunk(r, c0 / 8, 64)) = pack8(lo);
                    *reinterpret_cast<uint4 *>(gslot + SL_P + kmaj_chunk(r, c0 / 8 + 1, 64)) = pack8(hi);
                }
            }
        } else {
            for (int i = tid - 128; i < C * XLD / 4; i += 128)
                reinterpret_cast<float4 *>(X)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        tc_fence_before();
        __syncthreads();

        // 5. X = (I + Diag(beta) A)^{-1}: diagonal 16x16 blocks by forward substitution,
        //    then the 2x2 block recursion with tf32 tensor-core products:
        //    [X11 0; X21 X22] with X21 = -X22 (Diag(beta_2) A21) X11.
        if (tid < C) {
            const int b = tid >> 4, cc = tid & 15;
            float x[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                const int r = 16 * b + rr;
                float acc = 0.f;
#pragma unroll
                for (int ii = 0; ii < rr; ++ii) acc += AF[r * ALD + 16 * b + ii] * x[ii];
                x[rr] = (rr == cc) ? 1.f : (rr > cc ? -sbeta[r] * acc : 0.f);
            }
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) X[(16 * b + rr) * XLD + 16 * b + cc] = x[rr];
        }
        __syncthreads();
        // 16-row level: warps 0, 1 build X[16..31][0..15], warps 2, 3 X[48..63][32..47] (8-column halves).
        if (warp < 4) {
            const int o = (warp >> 1) * 32, nh = (warp & 1) * 8;  // block offset, column half
            float *Rw = R2 + warp * 128;                          // 16 x 8 scratch per warp
            warp_gemm_16x8<16>(
                lane, [&](int r, int kk) { return sbeta[o + 16 + r] * AF[(o + 16 + r) * ALD + o + kk]; },
                [&](int kk, int nn) { return X[(o + kk) * XLD + o + nh + nn]; },
                [&](int r, int nn, float v) { Rw[r * 8 + nn] = v; });
            __syncwarp();
            warp_gemm_16x8<16>(
                lane, [&](int r, int kk) { return X[(o + 16 + r) * XLD + o + 16 + kk]; },
                [&](int kk, int nn) { return Rw[kk * 8 + nn]; },
                [&](int r, int nn, float v) { X[(o + 16 + r) * XLD + o + nh + nn] = -v; });
        }
        __syncthreads();
        // 32-row level: R2 = (Diag(beta) A)[32..63][0..31] X[0..31][0..31], then X[32..63][0..31] = -X22 R2.
        {
            const int mt = warp >> 2, nt = warp & 3;  // 16-row tile, 8-column tile
            warp_gemm_16x8<32>(
                lane, [&](int r, int kk) { return sbeta[32 + 16 * mt + r] * AF[(32 + 16 * mt + r) * ALD + kk]; },
                [&](int kk, int nn) { return X[kk * XLD + 8 * nt + nn]; },
                [&](int r, int nn, float v) { R2[(16 * mt + r) * 32 + 8 * nt + nn] = v; });
            __syncthreads();
            warp_gemm_16x8<32>(
                lane, [&](int r, int kk) { return X[(32 + 16 * mt + r) * XLD + 32 + kk]; },
                [&](int kk, int nn) { return R2[kk * 32 + 8 * nt + nn]; },
                [&](int r, int nn, float v) { X[(32 + 16 * mt + r) * XLD + 8 * nt + nn] = -v; });
        }
        __syncthreads();
        // T = X Diag(beta), lower triangle, bf16: A operand of W (smem) and the slot's T tile.
        for (int e2 = tid; e2 < C * 8; e2 += PT) {
            const int r = e2 >> 3, cc8 = e2 & 7;
            float t8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int c = cc8 * 8 + e;
                t8[e] = (c <= r) ? X[r * XLD + c] * sbeta[c] : 0.f;
            }
            *reinterpret_cast<uint4 *>(TT + kmaj_chunk(r, cc8, 64)) = pack8(t8);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // 6. W = T (K e^G): M = 64 MMA, A = T (K-major), B = rows 64..127 of [Qg ; Kg] read as
        //    an MN-major tile (64-column blocks 128 rows apart); TMEM cols [64,192), M=64 layout:
        //    row r in lane (r % 16) + 32 (r / 16).
        if (tid == 0) {
            bulk_s2g(gslot + SL_T, TT, 8192);
            const uint32_t a = smem_u32(TT), b = smem_u32(GA);
            const uint32_t idw = idesc_bf16(64, 128, false, true);
#pragma unroll
            for (int st = 0; st < C / 16; ++st)
                mma_bf16(tm + 64, kmaj_desc(a, st, 64), sdesc(b + 64 * 128 + st * 16 * 128, 128 * 128, 1024), idw,
                         st > 0);
            mma_commit(&bars[1]);
        }
        // The log_alpha buffer (A, X) is consumed: fetch the next item's inputs now.
        if (nid < items) fetch(nxt);
        if (!mbar_wait(&bars[1], mma_phase, kWaitNs)) sflag[1] = 1;
        mma_phase ^= 1;
        tc_fence_after();

        // 7. W rows (16-byte chunks) into the lower half of WQ = [Qg ; W] (its Kg rows are consumed).
        if (warp < 4) {
            const int r = 16 * warp + (lane & 15);
            for (int c0 = 0; c0 < DK; c0 += 32) {
                float v[32];
                tmem_ld32(tm + 64 + ((uint32_t)(warp * 32) << 16) + c0, v);
                tmem_wait_ld();
                if (lane < 16) {
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        float w8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) w8[e] = v[q8 * 8 + e];
                        *reinterpret_cast<uint4 *>(GA + kmaj_chunk(64 + r, c0 / 8 + q8, 128)) = pack8(w8);
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // 8. WQ leaves in one bulk store; waited for before GA is rewritten.
        if (tid == 0) {
            bulk_s2g(gslot + SL_WQ, GA, 32768);
            bulk_commit();
        }
        id = nid;
        cur = nxt;
    }
    if (tid == 0) {
        bulk_wait_all();
        if (sflag[1]) flag_error(err, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 256);
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
        const int slot_id = fix[2 + e];
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
        // Q e^G -> WQ rows 0..63; K e^{Gl-G} -> KD; D; K e^G kept in sK
        for (int idx = tid; idx < C * DK; idx += FT) {
            const int r = idx / DK, c = idx % DK;
            const float gg = sG[r * FLD + c], gl = sG[(C - 1) * FLD + c];
            const float ex = expf(gg);
            *reinterpret_cast<bf16 *>(g + SL_WQ + kmaj_off(r, c, 128)) = __float2bfloat16_rn(sQ[r * FLD + c] * ex);
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
            *reinterpret_cast<bf16 *>(g + SL_WQ + kmaj_off(64 + r, c, 128)) = __float2bfloat16_rn(acc);
        }
        for (int idx = tid; idx < C * C; idx += FT) {
            const int r = idx / C, c = idx % C;
            *reinterpret_cast<bf16 *>(g + SL_T + kmaj_off(r, c, 64)) = __float2bfloat16_rn(sT[r * (C + 1) + c]);
            *reinterpret_cast<bf16 *>(g + SL_P + kmaj_off(r, c, 64)) = __float2bfloat16_rn(sP[r * (C + 1) + c]);
        }
    }
}

// ---------------------------------------------------------------- scan ----
// The big tiles of a chunk (WQ = [Q e^G ; W], K e^{Gl-G}) are triple-buffered
// and fetched two chunks ahead; the small ones (T, P, the V tile, e^{Gl}) are
// double-buffered, one chunk ahead. Every product is an M = 128 tcgen05.mma;
// the 128-row A operands of T V and P U take the 64 rows next to T (before)
// and P (after) as filler whose output rows are never read, so no zero
// padding is stored. TMEM lanes: 0..63 hold O = Q e^G S + P U, 64..127 hold
// W S and T V (their difference is U); Z = Kd^T U fills all 128 lanes.
constexpr int ST = 160;  // warps 0..3: TMEM-lane epilogues; warp 4: copy and MMA issue
constexpr uint32_t SA_WQ = 0, SA_KD = 32768, SA_BYTES = 49152;                 // x3
constexpr uint32_t SB_T = 0, SB_P = 8192, SB_V = 16384, SB_D = 24576, SB_BYTES = 25600;  // x2
constexpr uint32_t SS_A = 0;
constexpr uint32_t SS_B = 3 * SA_BYTES;          // T of B0 is preceded by the last A buffer
constexpr uint32_t SS_S = SS_B + 2 * SB_BYTES;   // [128 (c)][64 (j)] MN-major bf16 state
constexpr uint32_t SS_U = SS_S + 16384;          // [64 (r)][64 (j)] MN-major bf16 pseudo-values
constexpr uint32_t SS_BAR = SS_U + 8192;         // fullA[3] fullB[2] bU bS uready sready, tmem base, flag
constexpr uint32_t SS_BYTES = SS_BAR + 96;
constexpr uint32_t SS_ALLOC = SS_BYTES + 1024;
constexpr uint32_t COPY_A = 32768 + 16384, COPY_B = 8192 + 8192 + 8192 + 512;
// TMEM columns: X and Y double-buffered, Z
constexpr uint32_t TM_X = 0, TM_Y = 128, TM_Z = 256;

__global__ void __launch_bounds__(ST, 1)
scan_kernel(const __grid_constant__ CUtensorMap tmap_v, const int32_t *__restrict__ cu, int64_t total,
            int H, int N, int j0, int nw, const char *__restrict__ slots, const float *__restrict__ S0,
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
    uint8_t *sS = sm + SS_S, *sU = sm + SS_U;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SS_BAR);
    uint64_t *fullA = bars, *fullB = bars + 3, *bU = bars + 5, *bS = bars + 6, *uready = bars + 7,
             *sready = bars + 8;
    uint32_t *tbase = reinterpret_cast<uint32_t *>(bars + 9);
    int *sfail = reinterpret_cast<int *>(tbase + 1);
    const size_t sofs = ((size_t)s * H + h) * DK * DV + (size_t)jv * DVT;
    const int c = tid;  // epilogue threads: state row owned (= TMEM lane)

    if (tid == 0) {
        for (int i = 0; i < 7; ++i) mbar_init(&bars[i], 1);
        mbar_init(uready, 64);   // the 64 threads of warps 2, 3
        mbar_init(sready, 128);  // the 128 epilogue threads
        *sfail = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tbase, 512);
        tmem_relinquish();
    }
    float Sr[DVT];
    auto store_state_bf16 = [&]() {
#pragma unroll
        for (int c8 = 0; c8 < DVT / 8; ++c8) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = Sr[c8 * 8 + e];
            *reinterpret_cast<uint4 *>(sS + mnmaj_chunk(c, c8, DK)) = pack8(x);
        }
    };
    if (tid < 128) {
        // Entry state: S0 (or zeros) on the first wave, else the carry.
        const float *Sin = (j0 == 0) ? S0 : state;
#pragma unroll
        for (int q4 = 0; q4 < DVT / 4; ++q4) {
            float4 x = Sin ? *reinterpret_cast<const float4 *>(Sin + sofs + (size_t)c * DV + 4 * q4)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            Sr[4 * q4] = x.x; Sr[4 * q4 + 1] = x.y; Sr[4 * q4 + 2] = x.z; Sr[4 * q4 + 3] = x.w;
        }
        store_state_bf16();
    }
    auto slot_of = [&](int jj) { return slots + ((size_t)((jj - j0) * N + s) * H + h) * SL_BYTES; };
    auto copy_a = [&](int jj) {  // big tiles of chunk jj -> A buffer (jj - j0) % 3
        const int ab = (jj - j0) % 3;
        uint8_t *buf = sm + SS_A + ab * SA_BYTES;
        const char *g = slot_of(jj);
        mbar_arrive_expect_tx(&fullA[ab], COPY_A);
        bulk_g2s(buf + SA_WQ, g + SL_WQ, 32768, &fullA[ab]);
        bulk_g2s(buf + SA_KD, g + SL_KD, 16384, &fullA[ab]);
    };
    auto copy_b = [&](int jj) {  // small tiles and the V box of chunk jj -> B buffer (jj - j0) % 2
        const int bb = (jj - j0) & 1;
        uint8_t *buf = sm + SS_B + bb * SB_BYTES;
        const char *g = slot_of(jj);
        mbar_arrive_expect_tx(&fullB[bb], COPY_B);
        bulk_g2s(buf + SB_T, g + SL_T, 8192, &fullB[bb]);
        bulk_g2s(buf + SB_P, g + SL_P, 8192, &fullB[bb]);
        bulk_g2s(buf + SB_D, g + SL_D, 512, &fullB[bb]);
        tma_load_3d(buf + SB_V, &tmap_v, jv * DVT, h, (int)(bos + (int64_t)jj * C), &fullB[bb]);
    };
    if (nj > 0 && tid == 128) {
        copy_a(j0);
        if (nj > 1) copy_a(j0 + 1);
        copy_b(j0);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tbase;

    if (warp == 4) {
        // ---------------- copy and MMA issue (one thread) ----------------
        if (lane == 0 && nj > 0) {
            const uint32_t id128 = idesc_bf16(128, DVT, false, true);  // K-major A, MN-major B
            const uint32_t idKd = idesc_bf16(128, DVT, true, true);    // MN-major A (Kd^T)
            // Descriptors of buffer 0; buffer i is i strides further (16-byte units).
            const uint64_t dWQ = sdesc(smem_u32(sm + SS_A + SA_WQ), 16, 1024);
            const uint64_t dKD = sdesc(smem_u32(sm + SS_A + SA_KD), C * 128, 1024);
            // "T then filler": 128 rows starting 64 rows before T (output rows 0..63 unused)
            const uint64_t dTf = sdesc(smem_u32(sm + SS_B + SB_T) - 8192, 16, 1024);
            // "P then filler": rows 64..127 read the V tile after P (output rows unused)
            const uint64_t dP = sdesc(smem_u32(sm + SS_B + SB_P), 16, 1024);
            const uint64_t dV = sdesc(smem_u32(sm + SS_B + SB_V), C * 128, 1024);
            const uint64_t dS = sdesc(smem_u32(sS), DK * 128, 1024), dU = sdesc(smem_u32(sU), C * 128, 1024);
            constexpr uint64_t kA = SA_BYTES >> 4, kB = SB_BYTES >> 4;
            auto issue_x = [&](int bb, uint32_t xb) {
#pragma unroll
                for (int st = 0; st < C / 16; ++st)
                    mma_bf16(tm + TM_X + xb, dTf + bb * kB + kmaj_step(st, 128), dV + bb * kB + mnmaj_step(st), id128,
                             st > 0);
            };
            if (!mbar_wait(&fullB[0], 0, kWaitNs)) *sfail = 1;
            issue_x(0, 0);
            for (int it = 0; it < nj; ++it) {
                const int jj = j0 + it, ab = it % 3, bb = it & 1;
                const uint32_t yb = (uint32_t)bb * 64;
                bool good = mbar_wait(&fullA[ab], (it / 3) & 1, kWaitNs);
                if (it > 0) good = good && mbar_wait(sready, (it - 1) & 1, kWaitNs);  // S(jj) in smem
                tc_fence_after();
                if (it + 2 < nj) copy_a(jj + 2);
                if (it + 1 < nj) copy_b(jj + 1);
                // Y = [Q e^G ; W] S
                const uint64_t dWQa = dWQ + ab * kA, dKDa = dKD + ab * kA, dPb = dP + bb * kB;
#pragma unroll
                for (int st = 0; st < DK / 16; ++st)
                    mma_bf16(tm + TM_Y + yb, dWQa + kmaj_step(st, 128), dS + mnmaj_step(st), id128, st > 0);
                mma_commit(bU);
                good = good && mbar_wait(uready, it & 1, kWaitNs);  // U(jj) in smem
                tc_fence_after();
                // O: Y += [P ; filler] U ;  Z = Kd^T U
#pragma unroll
                for (int st = 0; st < C / 16; ++st)
                    mma_bf16(tm + TM_Y + yb, dPb + kmaj_step(st, 128), dU + mnmaj_step(st), id128, 1);
#pragma unroll
                for (int st = 0; st < C / 16; ++st)
                    mma_bf16(tm + TM_Z, dKDa + mnmaj_step(st), dU + mnmaj_step(st), idKd, st > 0);
                mma_commit(bS);
                if (it + 1 < nj) {
                    good = good && mbar_wait(&fullB[bb ^ 1], ((it + 1) >> 1) & 1, kWaitNs);
                    issue_x(bb ^ 1, yb ^ 64);
                }
                if (!good) {
                    *sfail = 1;
                    break;
                }
            }
        }
    } else {
        // ---------------- epilogues (TMEM lane = thread) ----------------
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        for (int it = 0; it < nj; ++it) {
            const int jj = j0 + it, bb = it & 1;
            const uint32_t xb = (uint32_t)bb * 64, yb = (uint32_t)bb * 64;
            const uint8_t *bbuf = sm + SS_B + bb * SB_BYTES;
            bool good = true;
            if (warp >= 2) {
                // U = T V - W S for rows r = lane - 64 (TMEM lanes 64..127)
                good = mbar_wait(bU, it & 1, kWaitNs);
                tc_fence_after();
                const int r = c - 64;
#pragma unroll
                for (int c0 = 0; c0 < DVT; c0 += 32) {
                    float xv[32], yv[32];
                    tmem_ld32(tm + TM_X + xb + lane_base + c0, xv);
                    tmem_ld32(tm + TM_Y + yb + lane_base + c0, yv);
                    tmem_wait_ld();
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        float u8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) u8[e] = xv[q8 * 8 + e] - yv[q8 * 8 + e];
                        *reinterpret_cast<uint4 *>(sU + mnmaj_chunk(r, c0 / 8 + q8, C)) = pack8(u8);
                    }
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(uready);
            }
            // S' = Diag(e^{G_last}) S + Z  (row c); needs Z(jj) and e^{Gl} of the chunk
            good = mbar_wait(bS, it & 1, kWaitNs) && good;
            good = mbar_wait(&fullB[bb], (it >> 1) & 1, kWaitNs) && good;
            tc_fence_after();
            const float dc = reinterpret_cast<const float *>(bbuf + SB_D)[c];
#pragma unroll
            for (int c0 = 0; c0 < DVT; c0 += 32) {
                float zv[32];
                tmem_ld32(tm + TM_Z + lane_base + c0, zv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) Sr[c0 + e] = dc * Sr[c0 + e] + zv[e];
            }
            store_state_bf16();
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(sready);
            // O(jj) = rows 0..63 of Y, complete with Z: warps 0, 1 store it
            if (warp < 2) {
                const int nn = (int)((len - (int64_t)jj * C) < C ? (len - (int64_t)jj * C) : C);
                const int64_t tt = bos + (int64_t)jj * C;
#pragma unroll
                for (int c0 = 0; c0 < DVT; c0 += 32) {
                    float yv[32];
                    tmem_ld32(tm + TM_Y + yb + lane_base + c0, yv);
                    tmem_wait_ld();
                    if (c < nn) {
                        bf16 *dst = o + ((size_t)(tt + c) * H + h) * DV + jv * DVT + c0;
#pragma unroll
                        for (int q8 = 0; q8 < 4; ++q8) {
                            float o8[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) o8[e] = yv[q8 * 8 + e];
                            reinterpret_cast<uint4 *>(dst)[q8] = pack8(o8);
                        }
                    }
                }
            }
            if (!good) {
                *sfail = 1;
                break;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    const bool ok = (*sfail == 0);
    if (!ok && tid == 0) flag_error(err, 1);

    // Exit: final state when the sequence ended in this wave, else the carry.
    float *Sout = (jend == nch) ? S_T : state;
    if (Sout && ok && tid < 128) {
#pragma unroll
        for (int q4 = 0; q4 < DVT / 4; ++q4)
            *reinterpret_cast<float4 *>(Sout + sofs + (size_t)c * DV + 4 * q4) =
                make_float4(Sr[4 * q4], Sr[4 * q4 + 1], Sr[4 * q4 + 2], Sr[4 * q4 + 3]);
    }
    if (warp == 0) tmem_dealloc(tm, 512);
}

// cuTensorMapEncodeTiled, resolved once through the runtime (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// v viewed as [T][H][DV] bf16; a box is 64 columns x 1 head x 64 tokens, SW128.
bool make_v_map(CUtensorMap *m, const void *v, int64_t total, int H) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)DV, (cuuint64_t)H, (cuuint64_t)total};
    const cuuint64_t strides[2] = {(cuuint64_t)DV * 2, (cuuint64_t)H * DV * 2};
    const cuuint32_t box[3] = {64, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(v), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q, k or log_alpha viewed as [T][H][128]; a box is 128 channels x 1 head x 64 tokens.
bool make_row_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, int64_t total, int H) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)DK, (cuuint64_t)H, (cuuint64_t)total};
    const cuuint64_t strides[2] = {(cuuint64_t)DK * esize, (cuuint64_t)H * DK * esize};
    const cuuint32_t box[3] = {(cuuint32_t)DK, 1, (cuuint32_t)C};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

cudaError_t set_attributes() {
    cudaError_t e = cudaFuncSetAttribute(prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PS_ALLOC);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FS_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SS_ALLOC);
    return e;
}

// Prep (+ exact fallback) of chunks [j0, j0 + nw) into `slots`; `queue` = [fallback count,
// item counter, fallback entries...].
cudaError_t tc_prep(const PrefillArgs &a, int j0, int nw, char *slots, int *queue, int cap, int *err,
                    cudaStream_t st) {
    CUtensorMap lamap;
    if (!make_row_map(&lamap, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.total, a.H))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(queue, 0, 2 * sizeof(int), st);
    if (e != cudaSuccess) return e;
    const int sms = sm_count();
    const int items = nw * a.N * a.H;
    const int grid = items < 2 * sms ? items : 2 * sms;
    prep_kernel<<<grid, PT, PS_ALLOC, st>>>((const bf16 *)a.q, (const bf16 *)a.k, lamap, a.beta, a.cu, a.total,
                                            a.H, a.N, j0, nw, a.l2norm, a.eps, slots, queue, cap, err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    fix_kernel<<<sms, FT, FS_BYTES, st>>>((const bf16 *)a.q, (const bf16 *)a.k, a.log_alpha, a.beta, a.cu,
                                          a.total, a.H, a.N, j0, a.l2norm, a.eps, slots, queue, cap);
    return cudaGetLastError();
}

cudaError_t tc_scan(const PrefillArgs &a, int j0, int nw, const char *slots, int *err, cudaStream_t st) {
    CUtensorMap vmap;
    memset(&vmap, 0, sizeof(vmap));
    if (a.total > 0 && !make_v_map(&vmap, a.v, a.total, a.H)) return cudaErrorInvalidValue;
    scan_kernel<<<dim3(DV / DVT, a.N, a.H), ST, SS_ALLOC, st>>>(vmap, a.cu, a.total, a.H, a.N, j0, nw, slots,
                                                                a.S0, a.state, a.S_T, (bf16 *)a.o, err);
    return cudaGetLastError();
}

// Per-device side stream and events for overlapping the prep of wave w+1 with
// the scan of wave w. Created on first use and kept for the process lifetime;
// the enqueue sequence of a call holds the mutex so that calls from several
// host threads do not interleave their use of the shared events.
struct Overlap {
    cudaStream_t side = nullptr;
    cudaEvent_t start = nullptr, prep[2] = {nullptr, nullptr}, scan[2] = {nullptr, nullptr};
    bool ok = false;
};
std::mutex g_overlap_mu;
Overlap g_overlap[64];

Overlap *overlap_for_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    Overlap &o = g_overlap[dev];
    if (!o.ok) {
        const unsigned f = cudaEventDisableTiming;
        if (cudaStreamCreateWithFlags(&o.side, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&o.start, f) != cudaSuccess ||
            cudaEventCreateWithFlags(&o.prep[0], f) != cudaSuccess ||
            cudaEventCreateWithFlags(&o.prep[1], f) != cudaSuccess ||
            cudaEventCreateWithFlags(&o.scan[0], f) != cudaSuccess ||
            cudaEventCreateWithFlags(&o.scan[1], f) != cudaSuccess)
            return nullptr;
        o.ok = true;
    }
    return &o;
}

}  // namespace

size_t tc_slot_bytes() { return SL_BYTES; }

cudaError_t tc_prefill(const PrefillArgs &a, int64_t max_chunks, int nw, char *const buf_slots[2],
                       int *const buf_queue[2], int cap, int *err, cudaStream_t st) {
    cudaError_t e = set_attributes();
    if (e != cudaSuccess) return e;
    if (max_chunks == 0) return tc_scan(a, 0, 0, buf_slots[0], err, st);  // only empty sequences
    if (nw >= max_chunks) {  // one wave: everything on the caller's stream
        if ((e = tc_prep(a, 0, (int)max_chunks, buf_slots[0], buf_queue[0], cap, err, st)) != cudaSuccess) return e;
        return tc_scan(a, 0, (int)max_chunks, buf_slots[0], err, st);
    }
    std::lock_guard<std::mutex> lock(g_overlap_mu);
    Overlap *ov = overlap_for_device();
    if (!ov) return cudaErrorInitializationError;
    if ((e = cudaEventRecord(ov->start, st)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(ov->side, ov->start, 0)) != cudaSuccess) return e;
    int w = 0;
    for (int64_t j0 = 0; j0 < max_chunks; j0 += nw, ++w) {
        const int n = (int)((max_chunks - j0) < nw ? (max_chunks - j0) : nw);
        const int b = w & 1;
        if (w >= 2 && (e = cudaStreamWaitEvent(ov->side, ov->scan[b], 0)) != cudaSuccess) return e;
        if ((e = tc_prep(a, (int)j0, n, buf_slots[b], buf_queue[b], cap, err, ov->side)) != cudaSuccess) return e;
        if ((e = cudaEventRecord(ov->prep[b], ov->side)) != cudaSuccess) return e;
        if ((e = cudaStreamWaitEvent(st, ov->prep[b], 0)) != cudaSuccess) return e;
        if ((e = tc_scan(a, (int)j0, n, buf_slots[b], err, st)) != cudaSuccess) return e;
        if ((e = cudaEventRecord(ov->scan[b], st)) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace kda
