// kda_prefill_tc.cu -- chunkwise KDA prefill on the sm_100a tensor cores
// (bf16 q/k/v, d_k = d_v = 128, chunk C = 64, fp32 state).
//
// Math ("[Kimi-2] Kimi Linear：用 KDA 重写长上下文注意力" §5, the UT transform and the
// inter-/intra-chunk split; §3 for the per-token update it rearranges). Per chunk
// with entry state S, G = cumulative sum of log_alpha over the chunk's rows:
//   Gram:  [P ; A] = [Q e^G ; K e^G] (K e^-G)^T      (masked: P lower, A strictly lower)
//   solve: T = (I + Diag(beta) A)^{-1} Diag(beta),   W = T (K e^G)
//   scan:  U = T V - W S,  O = (Q e^G) S + P U,  S' = Diag(e^{G_last}) S + (K e^{G_last-G})^T U
//
// One persistent kernel per call, after a one-CTA planning kernel:
//  * The (sequence, head) units are dealt round-robin to NS streams. Scan
//    CTAs 2 st and 2 st + 1 walk stream st's units chunk by chunk, each for 64
//    of the 128 state columns; the fp32 state stays on chip for a whole unit.
//    All products are M = 128 tcgen05.mma with fp32 accumulators in TMEM.
//  * Every other CTA runs two prep engines of 256 threads. An engine claims
//    the next (stream, position) item in a global order, computes that
//    chunk's operands (L2 norm, G, the Gram on the tensor cores, the 64 x 64
//    triangular solve, W on the tensor cores) and publishes them in the
//    stream's ring of R slots in the workspace (L2-resident).
//  * Ring handshake: a slot carries a ready generation (set by the engine
//    with a gpu-scope release after its stores completed) and a release count
//    (two per generation, one from each scan CTA of the stream once the
//    slot's bytes are in its shared memory). The kernel is launched
//    cooperatively, so scan and prep CTAs are co-resident and these waits
//    always end; each is bounded all the same (2 s), and one that runs out
//    sets the device error word and an abort flag that ends the others.
//  * The factorisation e^{G_r - G_i} = e^{G_r} e^{-G_i} needs e^{-G} finite:
//    for a chunk whose decay range exceeds kTau the engine builds P and A with
//    element-wise exponents (all <= 1) instead of the Gram MMA.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include <atomic>
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
constexpr int DVT = 64;                      // state columns per scan CTA
constexpr float kTau = 60.f;                 // largest per-chunk decay range for the factorised Gram
constexpr float kLog2e = 1.4426950408889634f;  // G is kept in base 2: e^{+-G} = 2^{+-G log2 e}
constexpr uint64_t kWaitNs = kDefaultWaitNs;  // bound of a CTA's waits for its own copies and products (2 s)
constexpr int kThreads = 512;                // per CTA: two prep engines, or one scan CTA
constexpr int kMaxRing = 16;                 // ring slots per stream, upper bound (~34 MB at 32 streams)

// ---------------------------------------------------------------- slot ----
// One ring slot per item, bytes (every tile 1024-byte aligned):
//   WQ [Q e^G ; W]   128 x 128 bf16, K-major SW128      (A operand of [Qg;W] S)
//   KD K e^-G        64 (r) x 128 (c) bf16, MN-major     (A operand of Kd^T U)
//   T                64 x 64 bf16, K-major               (A operand of T V)
//   P                64 x 64 bf16, K-major               (A operand of P U)
//   D  e^{G_last}, DZ  2 x 128 fp32: the scan forms S' = Diag(D) S + Diag(DZ) Kd^T U,
//                    so DZ = e^{G_last} with KD = K e^-G; a chunk past kTau ships
//                    KD = K e^{G_last - G} (element-wise exponents) with DZ = 1
constexpr uint32_t SL_WQ = 0, SL_KD = 32768, SL_T = 49152, SL_P = 57344, SL_D = 65536;
constexpr uint32_t SL_BYTES = 66560;

// ----------------------------------------------------------- workspace ----
// [header 256 B][L: int64 per stream][order: int32 per stream] (1 KiB)
// [ustart: int64 per unit][nch: int32 per unit] (1 KiB aligned)
// [ready: int32 x kMaxStreams*kMaxRing][freed: same]
// [ring: NS*R slots]
// [output-step exchange: per scan CTA, 4 x 64 words (row sum of squares, position tag)]
struct Hdr {
    unsigned long long claim;  // next item to claim
    long long total;           // items over all streams
    long long maxlen;          // positions of the longest stream
    int uniform;               // every stream has the same length
    int abort_flag;            // a bounded wait of this call gave up
};
constexpr size_t WS_L = 256, WS_ORDER = 768, WS_USTART = 1024;
constexpr size_t kFlagInts = (size_t)kTcMaxStreams * kMaxRing;

__host__ __device__ inline size_t ru1024(size_t x) { return (x + 1023) & ~size_t(1023); }
__host__ __device__ inline size_t ws_nch(long long NH) { return WS_USTART + 8 * (size_t)NH; }
__host__ __device__ inline size_t ws_flags(long long NH) { return ru1024(ws_nch(NH) + 4 * (size_t)NH); }
__host__ __device__ inline size_t ws_ring(long long NH) { return ru1024(ws_flags(NH) + 2 * kFlagInts * sizeof(int)); }
constexpr size_t kXchWords = (size_t)kTcMaxStreams * 2 * 4 * 64;
__host__ __device__ inline size_t ws_xch(long long NH, int ns, int R) { return ws_ring(NH) + (size_t)ns * R * SL_BYTES; }

struct FusedParams {
    CUtensorMap tmap_la;  // log_alpha [T][H][128] fp32, box 128 x 1 x 64
    CUtensorMap tmap_v;   // v [T][H][128] bf16, box 64 x 1 x 64, SW128
    CUtensorMap tmap_q;   // q, k: as v
    CUtensorMap tmap_k;
    const bf16 *q, *k, *v;
    // causal short convolution + Swish fused into the loads of q, k, v (index 0, 1, 2)
    int cw[3];           // window (0: the input as it is), at most 4
    const float *cwt[3];  // taps [H * 128][W]
    const bf16 *cst[3];   // initial states [N][W - 1][H * 128] (nullptr: zeros)
    const float *beta, *S0;
    const float *la;  // log_alpha, read directly when it is one gate per (token, head)
    const int32_t *cu;
    float *S_T;
    bf16 *o;
    const bf16 *og_gate;  // fused output step (nullptr: none)
    const float *og_w;
    float og_eps;
    char *ws;
    int *err;
    long long total;  // tokens
    unsigned long long xwait_ns;  // bound of the waits between CTAs (ring flags, row-sum exchange)
    int N, H, ns, R, l2norm, la_scalar;
    float eps;
};

__device__ __forceinline__ void flag_error(int *err, int code) {
    if (err) atomicCAS(err, 0, code);
}
// A bounded wait gave up: record it and make every other wait of the call end.
__device__ __forceinline__ void fail_call(const FusedParams &P) {
    Hdr *hd = reinterpret_cast<Hdr *>(P.ws);
    atomicExch(&hd->abort_flag, 1);
    flag_error(P.err, 1);
}
// Wait until *flag >= target (gpu-scope acquire), a flag another CTA sets; false on
// abort or after `limit_ns`. Polls every `sleep_ns` (0: back to back, for waits
// expected to be short).
__device__ __forceinline__ bool wait_flag_geq(const int *flag, int target, const int *abort_flag,
                                              uint64_t limit_ns, unsigned sleep_ns = 100) {
    if (ld_acquire_gpu(flag) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (sleep_ns) __nanosleep(sleep_ns);
        if (ld_acquire_gpu(flag) >= target) return true;
        if (ld_relaxed_gpu(abort_flag) || globaltimer_ns() - t0 > limit_ns) return false;
    }
}
// mbarrier wait of a scan thread on another thread of its CTA: like mbar_wait
// (bound kWaitNs), and it also gives up once the call's abort flag is set, so a
// failed call ends within microseconds. Not for a CTA's own copies and products
// in flight: those are always waited for (bounded) before the CTA exits.
__device__ __forceinline__ bool mbar_wait_call(uint64_t *bar, uint32_t parity, const int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 31) == 0 && (ld_relaxed_gpu(abort_flag) || globaltimer_ns() - t0 > kWaitNs)) return false;
    }
}

// --------------------------------------------------------------- plan ----
// One CTA: chunks per unit, each unit's first position in its stream (units
// st, st + NS, ... in order), stream lengths L, the streams ordered by
// decreasing length, and zeroed counters and ring flags.
constexpr int PLAN_T = 1024;
__global__ void __launch_bounds__(PLAN_T)
plan_kernel(const int32_t *__restrict__ cu, long long total, int N, int H, int ns, int R, char *__restrict__ ws) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long NH = (long long)N * H;
    Hdr *hd = reinterpret_cast<Hdr *>(ws);
    long long *L = reinterpret_cast<long long *>(ws + WS_L);
    int *order = reinterpret_cast<int *>(ws + WS_ORDER);
    long long *ustart = reinterpret_cast<long long *>(ws + WS_USTART);
    int *nch = reinterpret_cast<int *>(ws + ws_nch(NH));
    int *flags = reinterpret_cast<int *>(ws + ws_flags(NH));
    for (long long u = tid; u < NH; u += PLAN_T) {
        int64_t bos, eos;
        seq_bounds(cu, (int)(u / H), total, bos, eos);
        nch[u] = (int)((eos - bos + C - 1) / C);
    }
    for (size_t i = tid; i < 2 * kFlagInts; i += PLAN_T) flags[i] = 0;
    for (size_t i = tid; i < kXchWords; i += PLAN_T) reinterpret_cast<unsigned long long *>(ws + ws_xch(NH, ns, R))[i] = 0;
    __syncthreads();
    // one warp per stream: lanes own contiguous runs of the stream's units
    for (int st = warp; st < ns; st += PLAN_T / 32) {
        const long long K = (NH - st + ns - 1) / ns;
        const long long per = (K + 31) / 32, k0 = lane * per, k1 = (k0 + per < K) ? k0 + per : K;
        long long sum = 0;
        for (long long kk = k0; kk < k1; ++kk) sum += nch[st + kk * ns];
        long long incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        long long acc = incl - sum;
        for (long long kk = k0; kk < k1; ++kk) {
            ustart[st + kk * ns] = acc;
            acc += nch[st + kk * ns];
        }
        if (lane == 31) L[st] = incl;
    }
    __syncthreads();
    if (tid < ns) {
        int rank = 0;
        for (int j = 0; j < ns; ++j) rank += (L[j] > L[tid]) || (L[j] == L[tid] && j < tid);
        order[rank] = tid;
    }
    if (tid == 0) {
        long long tot = 0, mx = 0, mn = L[0];
        for (int j = 0; j < ns; ++j) {
            tot += L[j];
            mx = L[j] > mx ? L[j] : mx;
            mn = L[j] < mn ? L[j] : mn;
        }
        hd->claim = 0;
        hd->total = tot;
        hd->maxlen = mx;
        hd->uniform = (mx == mn);
        hd->abort_flag = 0;
    }
}

// ------------------------------------------------------ shared memory ----
// Prep engine (one per 256 threads, two per CTA):
constexpr int PT = 256;
constexpr uint32_t PS_LA = 0;                  // log_alpha -> G [64][128] fp32; later A/X, R2, T
constexpr uint32_t PS_GA = 32768;              // [Qg ; Kg] K-major 128 x 128 -> WQ
constexpr uint32_t PS_GB = PS_GA + 32768;      // q of the next item, then K e^-G (K-major 64 x 128)
constexpr uint32_t PS_KS = PS_GB + 16384;      // k of the next item (K-major 64 x 128)
constexpr uint32_t PS_SMALL = PS_KS + 16384;   // invq[64] invk[64] beta[2][64] eGl[128] gate[2][64]
constexpr uint32_t PS_BAR = PS_SMALL + 2048;   // la, mma, q/k barriers; 3 item records; flags
constexpr uint32_t PS_HALO = PS_BAR + 256;     // fused convolution: 3 raw rows before the item, q and k
constexpr uint32_t PS_BYTES = PS_HALO + 1536;
constexpr uint32_t PS_STRIDE = 102400;         // engine 1 starts here (1024-aligned)
constexpr int ALD = 68;                        // row stride of A / X (floats)
constexpr uint32_t PS_AF = PS_LA;              // A, then X in place: 64 x 68 fp32
constexpr uint32_t PS_T = PS_LA + 17408;       // T, 64 x 64 bf16 K-major (1024-aligned)
constexpr uint32_t PS_R2 = PS_LA + 25600;      // solve scratch: 32 x R2LD fp32
constexpr int R2LD = 36;
static_assert(PS_BYTES <= PS_STRIDE, "prep engine layout");

// Scan CTA: the tiles of a chunk from its ring slot: A (WQ, KD) double-buffered,
// B (T, P, e^{Gl}) triple-buffered; the V tile, an input independent of the
// prep, in a ring of four loaded ahead by its own thread.
constexpr uint32_t SA_WQ = 0, SA_KD = 32768, SA_BYTES = 49152;             // x2
constexpr uint32_t SB_T = 0, SB_P = 8192, SB_D = 16384, SB_BYTES = 17408;  // x3
constexpr uint32_t SV_BYTES = 8192;                                        // x4
constexpr uint32_t SS_A = 0;
constexpr uint32_t SS_B = 2 * SA_BYTES;         // T of B0 is preceded by the last A buffer
constexpr uint32_t SS_V = SS_B + 3 * SB_BYTES;
constexpr uint32_t SS_S = SS_V + 4 * SV_BYTES;  // [128 (c)][64 (j)] MN-major bf16 state
constexpr uint32_t SS_U = SS_S + 16384;         // [64 (r)][64 (j)] MN-major bf16 pseudo-values
constexpr uint32_t SS_BAR = SS_U + 8192;        // 31 mbarriers, the consumed-position counter, a flag
constexpr uint32_t SS_OGW = SS_BAR + 512;       // output-step weights of this CTA's 64 columns
constexpr uint32_t SS_VPREV = SS_OGW + 256;     // fused convolution of v: raw rows 61..63 of the last tile
constexpr uint32_t SS_BYTES = SS_VPREV + 384;
constexpr uint32_t COPY_A = 32768 + 16384, COPY_B = 8192 + 8192 + 1024;
constexpr int NY = 4;  // Y buffers in TMEM: the O epilogue may lag NY - 1 chunks
constexpr uint32_t TM_X = 0, TM_Y = 128, TM_Z = TM_Y + 64 * NY;  // scan TMEM columns: X x2, Y x NY, Z
static_assert(TM_Z + 64 <= 512, "scan TMEM columns");
// scan mbarrier indices
constexpr int MB_FULLA = 0, MB_FULLB = 2, MB_FULLV = 5, MB_EMPTYA = 9, MB_EMPTYB = 11, MB_EMPTYV = 14,
              MB_U = 18, MB_S = 19, MB_O = 20,  // MB_O and MB_OREADY: one barrier per Y buffer
              MB_UREADY = MB_O + NY, MB_SREADY = MB_UREADY + 1, MB_FIN = MB_SREADY + 1, MB_OREADY = MB_FIN + 1,
              MB_X = MB_OREADY + NY,  // one per X buffer: T V of a position complete
              MB_FIN2 = MB_X + 2,
              MB_CV = MB_FIN2 + 1,  // four, one per V buffer: the fused convolution of the tile is done
              MB_COUNT = MB_CV + 4;

// Per-CTA control block after both layouts.
struct Ctrl {
    uint32_t tbase;
    int uniform;
    int ucache, ccache;  // the unit starts / the sequence bounds are cached in shared memory
    long long total, maxlen;
    long long L[kTcMaxStreams];
    int order[kTcMaxStreams];
};
constexpr uint32_t CTRL_OFF = SS_BYTES > 2 * PS_STRIDE ? SS_BYTES : 2 * PS_STRIDE;
// Prep CTAs cache each unit's first position in its stream and the sequence bounds
// (when they fit), so that mapping a claimed item to its chunk costs no global loads.
constexpr int kUnitCache = 2048, kSeqCache = 1025;
constexpr uint32_t CACHE_OFF = CTRL_OFF + 512;
constexpr uint32_t SMEM_ALLOC = CACHE_OFF + 4 * (kUnitCache + kSeqCache) + 1024;  // + alignment slack
static_assert(2 * PS_STRIDE <= CTRL_OFF, "prep engines overlap the control block");
static_assert(MB_O + NY == MB_UREADY && MB_OREADY + NY == MB_X, "scan barrier indices");
static_assert(MB_COUNT * 8 + 16 <= SS_OGW - SS_BAR, "scan barrier area");
static_assert(sizeof(Ctrl) <= 512, "control block");

// ---------------------------------------------------------------- prep ----
struct ItemS {
    long long t0, p;  // first token; position in the stream
    int n, h, st, valid;
    int s, first;     // sequence; the item is its first chunk
    int slot, gen;    // ring slot (stream st, position p % R) and its generation p / R
};
static_assert(3 * 8 + 3 * sizeof(ItemS) + 3 * 4 <= PS_HALO - PS_BAR, "prep barrier block: mbarriers, item records, flags");


// Item g of the global claim order: position-major over the streams still
// running at that position, longest streams first.
__device__ bool map_item(unsigned long long g, const FusedParams &P, const Ctrl *ctl, ItemS &it) {
    if ((long long)g >= ctl->total) return false;
    const int ns = P.ns;
    long long p;
    int i;
    if (ctl->uniform) {  // item indices, positions and units fit in 32 bits (checked on the host)
        p = (long long)((unsigned)g / (unsigned)ns);
        i = (int)((unsigned)g % (unsigned)ns);
    } else {
        // largest p with sum_st min(L_st, p) <= g
        long long lo = 0, hi = ctl->maxlen - 1;
        while (lo < hi) {
            const long long mid = (lo + hi + 1) >> 1;
            long long s = 0;
            for (int t = 0; t < ns; ++t) s += ctl->L[t] < mid ? ctl->L[t] : mid;
            if (s <= (long long)g) lo = mid;
            else hi = mid - 1;
        }
        p = lo;
        long long s = 0;
        for (int t = 0; t < ns; ++t) s += ctl->L[t] < p ? ctl->L[t] : p;
        i = (int)((long long)g - s);
    }
    const int st = ctl->order[i];
    const long long NH = (long long)P.N * P.H;
    const long long *ustart = reinterpret_cast<const long long *>(P.ws + WS_USTART);
    const int *uc = reinterpret_cast<const int *>(reinterpret_cast<const uint8_t *>(ctl) + 512);
    long long lo = 0, hi = (long long)(((unsigned)(NH - st) + (unsigned)ns - 1u) / (unsigned)ns) - 1;  // last unit of the stream starting at or before p
    while (lo < hi) {
        const long long mid = (lo + hi + 1) >> 1;
        const long long us = ctl->ucache ? (long long)uc[st + mid * ns] : ustart[st + mid * ns];
        if (us <= p) lo = mid;
        else hi = mid - 1;
    }
    const long long u = st + lo * ns;
    const long long j = p - (ctl->ucache ? (long long)uc[u] : ustart[u]);
    int64_t bos, eos;
    const int s = (int)((unsigned)u / (unsigned)P.H);
    if (ctl->ccache) {
        bos = uc[kUnitCache + s];
        eos = uc[kUnitCache + s + 1];
    } else {
        seq_bounds(P.cu, s, P.total, bos, eos);
    }
    it.t0 = bos + j * C;
    it.n = (int)((eos - it.t0) < C ? (eos - it.t0) : C);
    it.s = s;
    it.first = j == 0;
    it.h = (int)((unsigned)u % (unsigned)P.H);
    it.st = st;
    it.p = p;
    it.slot = st * P.R + (int)((unsigned)p % (unsigned)P.R);
    it.gen = (int)((unsigned)p / (unsigned)P.R);
    return true;
}

// An fp32 value rounded to tf32 (10 stored significand bits), to nearest with ties away
// from zero, done on the bit pattern (finite inputs): the operand format of the tf32
// mma.sync below.
__device__ __forceinline__ uint32_t tf32_bits(float x) { return (__float_as_uint(x) + 0x1000u) & 0xFFFFE000u; }
// D (16x8) += A (16x8, row-major) x B (8x8) with tf32 operands, fp32 accumulation.
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// One warp: C[16 x 8] = A[16 x K] B[K x 8] for A(r, k), B(k, n) given as functors (every
// operand is read first, then the K / 8 products run back to back). The result stays in
// the accumulator layout: acc = C(g, 2t), C(g, 2t+1), C(g+8, 2t), C(g+8, 2t+1) for lane
// 4g + t.
template <int K, typename FA, typename FB>
__device__ __forceinline__ void warp_gemm_16x8(int lane, FA A, FB B, float (&acc)[4]) {
    const int g = lane >> 2, t = lane & 3;
    uint32_t a[K / 8][4], b[K / 8][2];
#pragma unroll
    for (int ks = 0; ks < K / 8; ++ks) {
        a[ks][0] = tf32_bits(A(g, 8 * ks + t));
        a[ks][1] = tf32_bits(A(g + 8, 8 * ks + t));
        a[ks][2] = tf32_bits(A(g, 8 * ks + t + 4));
        a[ks][3] = tf32_bits(A(g + 8, 8 * ks + t + 4));
        b[ks][0] = tf32_bits(B(8 * ks + t, g));
        b[ks][1] = tf32_bits(B(8 * ks + t + 4, g));
    }
    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < K / 8; ++ks) mma_tf32(acc, a[ks], b[ks]);
}

// Prep engine e (threads 256 e .. 256 e + 255) with its shared memory `sm` and
// TMEM columns [tm, tm + 256). Named barriers 1 + e (the engine) and 3 + 2e,
// 4 + 2e (warp pairs of the solve).
template <bool CV>
__device__ __forceinline__ void prep_engine(const FusedParams &P, const Ctrl *ctl, int e, uint8_t *sm,
                                            uint32_t tm) {
    const int tid = (int)threadIdx.x - PT * e, warp = tid >> 5, lane = tid & 31;
    const uint32_t bar_id = 1 + e;
    const int H = P.H;
    float *G = reinterpret_cast<float *>(sm + PS_LA);
    float *AF = reinterpret_cast<float *>(sm + PS_AF);
    float *R2 = reinterpret_cast<float *>(sm + PS_R2);
    uint8_t *TT = sm + PS_T;
    uint8_t *GA = sm + PS_GA;
    uint8_t *GB = sm + PS_GB;
    uint8_t *KS = sm + PS_KS;
    uint8_t *HALO = sm + PS_HALO;
    float *invq = reinterpret_cast<float *>(sm + PS_SMALL);
    float *invk = invq + 64, *sbeta2 = invk + 64, *eGl = sbeta2 + 128, *sgate2 = eGl + 128;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + PS_BAR);  // [0] log_alpha box, [1] MMA, [2] q, k boxes
    // Item records of iterations it (current), it + 1 (claimed during the Gram)
    // and it - 1 (published by the store thread) in entries it % 3, ...
    ItemS *sitem = reinterpret_cast<ItemS *>(bars + 3);
    int *sflag = reinterpret_cast<int *>(sitem + 3);  // [0] unsafe range, [1] a wait failed, [2] next slot known free
    Hdr *hd = reinterpret_cast<Hdr *>(P.ws);
    const long long NH = (long long)P.N * H;
    int *ready = reinterpret_cast<int *>(P.ws + ws_flags(NH));
    int *freed = ready + kFlagInts;
    char *ring = P.ws + ws_ring(NH);
    auto sync = [&]() { bar_sync(bar_id, PT); };
    uint32_t la_phase = 0, mma_phase = 0, qk_phase = 0;
    const int c8 = tid & 15, rb = tid >> 4;  // thread's 16-byte channel chunk and first row


    // Thread 128 claims items, issues the slot's bulk stores (bulk groups belong
    // to the issuing thread) and the log_alpha boxes, and publishes each item:
    // after the item's generic slot stores (ordered before it by the engine's
    // barriers) and its bulk stores completed, one gpu-scope release of the
    // slot's ready generation. The previous item is published during the Gram
    // (warps 4..7 are idle there), or at once if the current item has to wait
    // for its slot (that wait may depend on the previous item).
    constexpr int kStoreTid = 128;
    bool prev_pending = false;  // store thread: the previous item is not yet published
    bool la_pending = false;    // store thread: a log_alpha box is in flight
    bool qk_pending = false;    // store thread: q, k boxes are in flight
    auto publish_prev = [&](const ItemS &pv) {
        if (!prev_pending) return;
        bulk_wait_all();
        fence_proxy_async_global();
        st_release_gpu(&ready[pv.slot], pv.gen + 1);
        prev_pending = false;
    };
    auto slot_free = [&](const ItemS &it) {
        return ld_acquire_gpu(&freed[it.slot]) >= 2 * it.gen;
    };
    auto claim = [&](ItemS &it) {
        it.valid = 0;
        if (ld_relaxed_gpu(&hd->abort_flag)) return;
        it.valid = map_item(atomicAdd(&hd->claim, 1ull), P, ctl, it) ? 1 : 0;
    };
    auto fetch_la = [&](const ItemS &it) {  // store thread: log_alpha rows by one TMA box
        if (P.la_scalar) return;             // one gate per row: with q, k below
        mbar_arrive_expect_tx(&bars[0], 32768u);
        tma_load_3d(G, &P.tmap_la, 0, it.h, (int)it.t0, &bars[0]);
        la_pending = true;
    };
    // The item's q and k rows into GB / KS (K-major SW128 64 x 128 tiles) by four
    // TMA boxes from the store thread (K e^-G later overwrites q in place; rows
    // past the sequence are cleared after arrival); beta of row `tid` (threads
    // < 64) by cp.async into sbeta2[buf], and with a scalar gate log_alpha of row
    // `tid` into sgate2[buf] (zero past the sequence).
    auto fetch_qk = [&](const ItemS &it, int buf) {
        if (tid == kStoreTid) {
            mbar_arrive_expect_tx(&bars[2], 32768u);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tma_load_3d(GB + half * 8192, &P.tmap_q, 64 * half, it.h, (int)it.t0, &bars[2]);
                tma_load_3d(KS + half * 8192, &P.tmap_k, 64 * half, it.h, (int)it.t0, &bars[2]);
            }
            qk_pending = true;
        }
        if (tid < C) {
            const size_t row = (size_t)(it.t0 + (tid < it.n ? tid : 0)) * H + it.h;
            cp_async4(sbeta2 + buf * 64 + tid, P.beta + row, tid < it.n ? 4u : 0u);
            if (P.la_scalar) cp_async4(sgate2 + buf * 64 + tid, P.la + row, tid < it.n ? 4u : 0u);
        } else if (CV && tid < C + 96) {  // fused convolution: raw rows t0 - 3 .. t0 - 1 of q and k
            const int hid = tid - C, tsel = hid / 48, jh = (hid % 48) >> 4, cc = hid & 15;
            const int W = P.cw[tsel];
            if (W > 0) {
                const bf16 *x = tsel ? P.k : P.q;
                const bf16 *srcp = x;
                uint32_t bytes = 0;
                if (!it.first) {  // inside the sequence
                    srcp = x + ((size_t)(it.t0 - 3 + jh) * H + it.h) * DK + cc * 8;
                    bytes = 16;
                } else if (P.cst[tsel] != nullptr && jh + W - 4 >= 0) {  // before it: the initial state
                    srcp = P.cst[tsel] + ((size_t)it.s * (W - 1) + (jh + W - 4)) * ((size_t)H * DK) + (size_t)it.h * DK + cc * 8;
                    bytes = 16;
                }
                cp_async16(HALO + ((tsel * 3 + jh) * 16 + cc) * 16, srcp, bytes);
            }
        }
        cp_async_commit();
    };

    // Fused short convolution + Swish of q (threads 0..127) and k (128..255), in place on
    // the item's GB / KS tiles (before the row norms): warp (tensor, row segment seg) takes
    // rows 16 seg .. 16 seg + 15, lane c4 channels 4 c4 .. 4 c4 + 3, with the three raw
    // rows before them from the halo (seg 0) or from the tile before any row is rewritten.
    // The same arithmetic as the standalone convolution kernel: taps oldest first, one fma
    // each, then z / (1 + e^-z), rounded to bf16.
    auto conv_qk = [&](const ItemS &it) {
        const int tsel = tid >> 7, seg = (tid >> 5) & 3, c4 = tid & 31;
        const int W = P.cw[tsel];
        uint8_t *tile = tsel ? KS : GB;
        const uint32_t cofs = (uint32_t)(c4 & 1) * 8;  // within the 16-byte chunk c4 / 2
        f2_t wp[2][4], win[3][2];
        if (W > 0) {
            const float *wt = P.cwt[tsel] + ((size_t)it.h * DK + c4 * 4) * W;
#pragma unroll
            for (int pr = 0; pr < 2; ++pr)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int jj = j - (4 - W);  // taps padded in front to four
                    wp[pr][j] = jj >= 0 ? f2(__ldg(wt + (2 * pr) * W + jj), __ldg(wt + (2 * pr + 1) * W + jj)) : f2(0.f, 0.f);
                }
#pragma unroll
            for (int jh = 0; jh < 3; ++jh) {
                const uint2 u = seg == 0 ? *reinterpret_cast<const uint2 *>(HALO + ((tsel * 3 + jh) * 16 + (c4 >> 1)) * 16 + cofs)
                                         : *reinterpret_cast<const uint2 *>(tile + kmaj_chunk(16 * seg - 3 + jh, c4 >> 1, 64) + cofs);
                win[jh][0] = unpack2(u.x);
                win[jh][1] = unpack2(u.y);
            }
        }
        sync();  // every window is read before a row is rewritten
        if (W > 0) {
            uint8_t *base = tile + kmaj_chunk(16 * seg, c4 >> 1, 64) + cofs;
#pragma unroll
            for (int r8 = 0; r8 < 16; r8 += 8) {  // eight rows at a time, loads first
                uint2 u[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    u[i] = *reinterpret_cast<const uint2 *>(base + (r8 + i) * 128 + ((((c4 >> 1) ^ (r8 + i)) & 7) - ((c4 >> 1) & 7)) * 16);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const f2_t x[2] = {unpack2(u[i].x), unpack2(u[i].y)};
                    uint32_t ow[2];
#pragma unroll
                    for (int pr = 0; pr < 2; ++pr) {
                        f2_t z = f2fma(wp[pr][0], win[0][pr], f2(0.f, 0.f));
                        z = f2fma(wp[pr][1], win[1][pr], z);
                        z = f2fma(wp[pr][2], win[2][pr], z);
                        z = f2fma(wp[pr][3], x[pr], z);
                        ow[pr] = pack2(swish2(z));
                        win[0][pr] = win[1][pr];
                        win[1][pr] = win[2][pr];
                        win[2][pr] = x[pr];
                    }
                    *reinterpret_cast<uint2 *>(base + (r8 + i) * 128 + ((((c4 >> 1) ^ (r8 + i)) & 7) - ((c4 >> 1) & 7)) * 16) =
                        make_uint2(ow[0], ow[1]);
                }
            }
        }
        sync();
    };

    if (tid == kStoreTid) claim(sitem[0]);
    sync();
    if (tid == kStoreTid && sitem[0].valid) fetch_la(sitem[0]);
    if (sitem[0].valid) fetch_qk(sitem[0], 0);
    bool failed = false;
    int iter = 0;
    for (; sitem[iter % 3].valid; ++iter) {
        const ItemS &cur = sitem[iter % 3];
        ItemS &next = sitem[(iter + 1) % 3];
        const ItemS &prev = sitem[(iter + 2) % 3];
        const int n = cur.n;
        char *gslot = ring + (size_t)cur.slot * SL_BYTES;
        const float *sbeta = sbeta2 + (iter & 1) * 64;
        if (tid == kStoreTid) {
            // This item's slot is written below: both scan CTAs of the stream must
            // have released its previous generation.
            if (!sflag[2]) {
                publish_prev(prev);
                if (!wait_flag_geq(&freed[cur.slot], 2 * cur.gen, &hd->abort_flag, P.xwait_ns))
                    sflag[1] = 1;
            }
            sflag[2] = 0;
        }

        // 1. Warps 0..3: G = cumulative sum of log_alpha over the rows, in place, one
        //    thread per channel. Warps 4..7: the row norms of q (threads 128..191) and
        //    k (192..255), one row per thread, from the chunks every thread copied.
        cp_async_wait_all();  // this thread's beta (and scalar gate)
        {
            const bool qk_in = mbar_wait(&bars[2], qk_phase, kWaitNs);
            if (!qk_in) sflag[1] = 1;
            if (tid == kStoreTid && qk_in) qk_pending = false;
            qk_phase ^= 1;
        }
        sync();
        if constexpr (CV) {
            if (!sflag[1]) conv_qk(cur);
        }
        if (tid < DK) {
            const float *sgate = sgate2 + (iter & 1) * 64;
            if (!P.la_scalar && !mbar_wait(&bars[0], la_phase, kWaitNs)) sflag[1] = 1;
            const int c = tid;
            float run = 0.f;
#pragma unroll
            for (int r0 = 0; r0 < C; r0 += 16) {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    v[i] = (r0 + i < n) ? (P.la_scalar ? sgate[r0 + i] : G[(r0 + i) * DK + c]) : 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    run = fmaf(v[i], kLog2e, run);
                    G[(r0 + i) * DK + c] = run;
                }
            }
            eGl[c] = ex2f(run);
            if (-run > kTau * kLog2e) sflag[0] = 1;
        } else {
            const int r = tid & (C - 1);
            uint8_t *src = (tid < 192) ? GB : KS;
            float ss = 0.f;
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) {
                float x[8];
                unpack8(*reinterpret_cast<const uint4 *>(src + kmaj_chunk(r, cc, 64)), x);
#pragma unroll
                for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], ss);
            }
            if (r >= n) {  // the box ran into the next sequence (or the zero fill past the end)
#pragma unroll
                for (int cc = 0; cc < 16; ++cc)
                    *reinterpret_cast<uint4 *>(src + kmaj_chunk(r, cc, 64)) = make_uint4(0, 0, 0, 0);
            }
            // 1 / max(||x||, eps) = rsqrt(max(||x||^2, eps^2))
            const float inv = (r >= n) ? 0.f : (P.l2norm ? rsqrtf(fmaxf(ss, P.eps * P.eps)) : 1.f);
            ((tid < 192) ? invq : invk)[r] = inv;
        }
        if (!P.la_scalar) la_phase ^= 1;
        if (tid == kStoreTid) bulk_wait_read();  // the previous item's bulk stores no longer read GA
        sync();
        if (sflag[1]) {
            failed = true;
            break;
        }
        if (tid == kStoreTid) la_pending = false;
        const bool safe = sflag[0] == 0;

        // 2. Operands for (row, 8-channel chunk): [Qg ; Kg] to GA, K e^-G to GB (over q),
        //    Kd to the slot, one channel pair at a time (packed as soon as computed).
        //    Unsafe range: [Q ; K] without exponents (the element-wise Gram needs them).
        if (safe) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int r = rb + 16 * m;
                const float ik = invk[r], iq = invq[r];
                const uint4 qv = *reinterpret_cast<const uint4 *>(GB + kmaj_chunk(r, c8, 64));
                const uint4 kv = *reinterpret_cast<const uint4 *>(KS + kmaj_chunk(r, c8, 64));
                const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
                const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
                uint32_t pq[4], pk[4], pn[4];
                const f2_t iq2 = f2(iq, iq), ik2 = f2(ik, ik);
#pragma unroll
                for (int w = 0; w < 4; ++w) {  // channel pairs, in fp32 pairs
                    const f2_t g = *reinterpret_cast<const f2_t *>(G + r * DK + c8 * 8 + 2 * w);
                    const float gx = f2lo(g), gy = f2hi(g);
                    const f2_t ep = f2(ex2f(gx), ex2f(gy)), en = f2(ex2f(-gx), ex2f(-gy));
                    const f2_t qn = f2mul(unpack2(qw[w]), iq2), kn = f2mul(unpack2(kw[w]), ik2);
                    pq[w] = pack2(f2mul(qn, ep));
                    pk[w] = pack2(f2mul(kn, ep));
                    pn[w] = pack2(f2mul(kn, en));
                }
                *reinterpret_cast<uint4 *>(GA + kmaj_chunk(r, c8, 128)) = make_uint4(pq[0], pq[1], pq[2], pq[3]);
                *reinterpret_cast<uint4 *>(GA + kmaj_chunk(64 + r, c8, 128)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                *reinterpret_cast<uint4 *>(GB + kmaj_chunk(r, c8, 64)) = make_uint4(pn[0], pn[1], pn[2], pn[3]);
                *reinterpret_cast<uint4 *>(gslot + SL_KD + mnmaj_chunk(r, c8, 64)) = make_uint4(pn[0], pn[1], pn[2], pn[3]);  // the slot carries K e^-G
            }
        } else {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int r = rb + 16 * m;
                float kf[8], qf[8], kd[8];
                unpack8(*reinterpret_cast<const uint4 *>(KS + kmaj_chunk(r, c8, 64)), kf);
                unpack8(*reinterpret_cast<const uint4 *>(GB + kmaj_chunk(r, c8, 64)), qf);
                const float ik = invk[r], iq = invq[r];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    kf[i] *= ik;
                    qf[i] *= iq;
                    kd[i] = kf[i] * ex2f(G[(C - 1) * DK + c8 * 8 + i] - G[r * DK + c8 * 8 + i]);
                }
                *reinterpret_cast<uint4 *>(GA + kmaj_chunk(r, c8, 128)) = pack8(qf);
                *reinterpret_cast<uint4 *>(GA + kmaj_chunk(64 + r, c8, 128)) = pack8(kf);
                *reinterpret_cast<uint4 *>(gslot + SL_KD + mnmaj_chunk(r, c8, 64)) = pack8(kd);
            }
        }
        if (tid < DK) {
            reinterpret_cast<float *>(gslot + SL_D)[tid] = eGl[tid];
            reinterpret_cast<float *>(gslot + SL_D)[DK + tid] = safe ? eGl[tid] : 1.f;
        }
        fence_async_smem();
        tc_fence_before();
        sync();
        tc_fence_after();

        // 3. Gram: TMEM cols [0,64) = [Qg ; Kg] (K e^-G)^T = [P ; A] before masking.
        if (safe) {
            if (tid == 0) {
                const uint32_t a = smem_u32(GA), b = smem_u32(GB);
                const uint32_t idg = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int s8 = 0; s8 < DK / 16; ++s8)
                    mma_bf16(tm, kmaj_desc(a, s8, 128), kmaj_desc(b, s8, 64), idg, s8 > 0);
                mma_commit(&bars[1]);
            }
            if (tid == kStoreTid + 32) {  // another warp than the store thread's
                claim(next);
                if (next.valid && !P.la_scalar) tma_prefetch_3d(&P.tmap_la, 0, next.h, (int)next.t0);
            }
            if (!mbar_wait(&bars[1], mma_phase, kWaitNs)) sflag[1] = 1;
            mma_phase ^= 1;
            tc_fence_after();
        } else {
            // Element-wise: row `row` of [Q ; K] against rows i of K, exponents G_r - G_i <= 0.
            const int row = (warp & 3) * 32 + lane, r = row & (C - 1);
            const bool isq = row < C;
            for (int i0 = (warp >> 2) * 32; i0 < (warp >> 2) * 32 + 32; i0 += 16) {
                float acc[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] = 0.f;
                for (int c = 0; c < DK; ++c) {
                    const float gr = G[r * DK + c];
                    const float xr = __bfloat162float(*reinterpret_cast<const bf16 *>(GA + kmaj_off(row, c, 128)));
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int ii = i0 + i;
                        const float ki = __bfloat162float(*reinterpret_cast<const bf16 *>(GA + kmaj_off(64 + ii, c, 128)));
                        const bool keep = isq ? (ii <= r) : (ii < r);
                        acc[i] += keep ? xr * ki * ex2f(gr - G[ii * DK + c]) : 0.f;
                    }
                }
                tmem_st16(tm + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)i0, acc);
            }
            tmem_wait_st();
            tc_fence_before();
            sync();
            tc_fence_after();
            // [Q ; K] -> [Q e^G ; K e^G] in place for the W product.
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int rr = rb + 16 * m, r2 = rr & (C - 1);
                float x[8];
                unpack8(*reinterpret_cast<const uint4 *>(GA + kmaj_chunk(rr, c8, 128)), x);
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] *= ex2f(G[r2 * DK + c8 * 8 + i]);
                *reinterpret_cast<uint4 *>(GA + kmaj_chunk(rr, c8, 128)) = pack8(x);
            }
            fence_async_smem();
            if (tid == kStoreTid + 32) claim(next);
            sync();  // G is overwritten by A below
        }
        if (tid == 0) sflag[0] = 0;

        // 4. P (bf16, lower incl. diagonal; TMEM lanes 0..63) to the slot; A (fp32,
        //    strictly lower, zero elsewhere; lanes 64..127) over the consumed G.
        //    Warps w and w + 4 share TMEM lanes 32 (w % 4) .. and take 32 columns each.
        {
            const int row = (warp & 3) * 32 + lane;
            for (int c0 = (warp >> 2) * 32; c0 < (warp >> 2) * 32 + 32; c0 += 16) {
                float v[16];
                tmem_ld16(tm + ((uint32_t)((warp & 3) * 32) << 16) + c0, v);
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
        }
        tc_fence_before();
        sync();
        // The next item is known (claimed during the Gram): its q, k rows load into
        // GB (free: the Gram has consumed K e^-G) and KS while this item finishes,
        // and the store thread checks its slot.
        if (next.valid) fetch_qk(next, (iter + 1) & 1);
        if (tid == kStoreTid) {  // warp 4 is idle in the diagonal-block solve below
            publish_prev(prev);
        }
        if (tid == kStoreTid + 96 && next.valid) sflag[2] = slot_free(next);  // beside the publish

        // 5. X = (I + Diag(beta) A)^{-1}, in place over A (fp32), and T = X Diag(beta) (bf16,
        //    the A operand of W and the slot's T tile), by 16 x 16 blocks.
        //    Level 0, warps 0..3: diagonal block b = warp by a right-looking forward
        //    substitution in registers, one column per lane (lanes 16..31 repeat 0..15):
        //    after x_i is known, its term is added to every later row's sum at once, so the
        //    dependent chain is one multiply-add per row. Warps 4..7: T's zero upper blocks.
        if (warp < 4) {
            const int r0 = 16 * warp, cc = lane & 15;
            float x[16], acc[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) acc[r] = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                x[i] = (i == cc) ? 1.f : (i > cc ? -sbeta[r0 + i] * acc[i] : 0.f);
#pragma unroll
                for (int r = i + 1; r < 16; ++r) acc[r] = fmaf(AF[(r0 + r) * ALD + r0 + i], x[i], acc[r]);
            }
            __syncwarp();  // every lane has read the block
            if (lane < 16) {
#pragma unroll
                for (int r = 0; r < 16; ++r) AF[(r0 + r) * ALD + r0 + cc] = x[r];
            }
        } else {
            // upper blocks (bi, bj), bj > bi: 6 blocks x 16 rows x 2 chunks of 8 columns
            for (int i = tid - 128; i < 6 * 16 * 2; i += 128) {
                const int blk = i >> 5, rr = (i >> 1) & 15, half = i & 1;
                const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
                const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
                *reinterpret_cast<uint4 *>(TT + kmaj_chunk(16 * bi + rr, 2 * bj + half, 64)) = make_uint4(0, 0, 0, 0);
            }
        }
        sync();
        // T's element pair (r, c), (r, c + 1) from X's, scaled by beta of the columns.
        auto t_store2 = [&](int r, int c, float x0, float x1) {
            *reinterpret_cast<uint32_t *>(TT + kmaj_off(r, c, 64)) = pack_bf16(x0 * sbeta[c], x1 * sbeta[c + 1]);
        };
        const int fg = lane >> 2, ft = lane & 3;  // accumulator layout of the tf32 products
        if (warp >= 4) {
            // T's diagonal blocks: block i >> 5, row (i >> 1) & 15, 8-column half i & 1
            const int i = tid - 128, bd = i >> 5, r = 16 * bd + ((i >> 1) & 15), c0 = 16 * bd + 8 * (i & 1);
            float t8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) t8[j] = (c0 + j <= r) ? AF[r * ALD + c0 + j] * sbeta[c0 + j] : 0.f;
            *reinterpret_cast<uint4 *>(TT + kmaj_chunk(r, c0 >> 3, 64)) = pack8(t8);
        } else {
            // Level 1, warps 0..3: X21 = -X22 (Diag(beta) A21) X11 for the 32-row blocks at 0
            // (warps 0, 1) and 32 (warps 2, 3), 8 of the 16 columns per warp; R = N21 X11
            // passes through a per-warp scratch to become the second product's B operand.
            const int o = (warp >> 1) * 32, nh = (warp & 1) * 8;
            float *Rw = R2 + warp * 128;  // 16 x 8
            float acc[4];
            warp_gemm_16x8<16>(
                lane, [&](int r, int kk) { return sbeta[o + 16 + r] * AF[(o + 16 + r) * ALD + o + kk]; },
                [&](int kk, int nn) { return AF[(o + kk) * ALD + o + nh + nn]; }, acc);
            *reinterpret_cast<float2 *>(Rw + fg * 8 + 2 * ft) = make_float2(acc[0], acc[1]);
            *reinterpret_cast<float2 *>(Rw + (fg + 8) * 8 + 2 * ft) = make_float2(acc[2], acc[3]);
            bar_sync(3 + 2 * e + (warp >> 1), 64);  // both column halves have read A21; R is in
            warp_gemm_16x8<16>(
                lane, [&](int r, int kk) { return AF[(o + 16 + r) * ALD + o + 16 + kk]; },
                [&](int kk, int nn) { return Rw[kk * 8 + nn]; }, acc);
            const int r = o + 16 + fg, c = o + nh + 2 * ft;
            *reinterpret_cast<float2 *>(AF + r * ALD + c) = make_float2(-acc[0], -acc[1]);
            *reinterpret_cast<float2 *>(AF + (r + 8) * ALD + c) = make_float2(-acc[2], -acc[3]);
            t_store2(r, c, -acc[0], -acc[1]);
            t_store2(r + 8, c, -acc[2], -acc[3]);
        }
        sync();
        // Level 2, all warps: R2 = (Diag(beta) A)[32..63][0..31] X[0..31][0..31] (kept transposed,
        // row stride R2LD), then X[32..63][0..31] = -X[32..63][32..63] R2, of which only T is kept.
        {
            const int mt = warp >> 2, nt = warp & 3;  // 16-row tile, 8-column tile
            float acc[4];
            warp_gemm_16x8<32>(
                lane, [&](int r, int kk) { return sbeta[32 + 16 * mt + r] * AF[(32 + 16 * mt + r) * ALD + kk]; },
                [&](int kk, int nn) { return AF[kk * ALD + 8 * nt + nn]; }, acc);
            const int rr = 16 * mt + fg, cc = 8 * nt + 2 * ft;
            R2[cc * R2LD + rr] = acc[0];
            R2[(cc + 1) * R2LD + rr] = acc[1];
            R2[cc * R2LD + rr + 8] = acc[2];
            R2[(cc + 1) * R2LD + rr + 8] = acc[3];
            sync();
            warp_gemm_16x8<32>(
                lane, [&](int r, int kk) { return AF[(32 + 16 * mt + r) * ALD + 32 + kk]; },
                [&](int kk, int nn) { return R2[(8 * nt + nn) * R2LD + kk]; }, acc);
            t_store2(32 + rr, cc, -acc[0], -acc[1]);
            t_store2(32 + rr + 8, cc, -acc[2], -acc[3]);
        }
        fence_async_smem();
        tc_fence_before();
        sync();
        tc_fence_after();

        // 6. W = T (K e^G): M = 64 MMA, A = T (K-major), B = rows 64..127 of [Qg ; Kg] read as
        //    an MN-major tile (64-column blocks 128 rows apart); TMEM cols [64,192), M=64 layout:
        //    row r in lane (r % 16) + 32 (r / 16).
        if (tid == kStoreTid) {
            bulk_s2g(gslot + SL_T, TT, 8192);
            bulk_commit();
        }
        if (tid == 0) {
            const uint32_t a = smem_u32(TT), b = smem_u32(GA);
            const uint32_t idw = idesc_bf16(64, 128, false, true);
#pragma unroll
            for (int s4 = 0; s4 < C / 16; ++s4)
                mma_bf16(tm + 64, kmaj_desc(a, s4, 64), sdesc(b + 64 * 128 + s4 * 16 * 128, 128 * 128, 1024), idw,
                         s4 > 0);
            mma_commit(&bars[1]);
        }
        if (!mbar_wait(&bars[1], mma_phase, kWaitNs)) sflag[1] = 1;
        mma_phase ^= 1;
        tc_fence_after();
        // T has been read by the MMA and, once the bulk store has read it too, the
        // log_alpha region is free for the next item's box.
        if (tid == kStoreTid && next.valid) {
            bulk_wait_read();
            fetch_la(next);
        }

        // 7. W rows (16-byte chunks) into the lower half of WQ = [Qg ; W] (its Kg rows are consumed).
        //    Warps w and w + 4 share TMEM lanes 32 (w % 4) .. and take 64 columns each.
        {
            const int r = 16 * (warp & 3) + (lane & 15);
            for (int c0 = (warp >> 2) * 64; c0 < (warp >> 2) * 64 + 64; c0 += 32) {
                float v[32];
                tmem_ld32(tm + 64 + ((uint32_t)((warp & 3) * 32) << 16) + c0, v);
                tmem_wait_ld();
                if (lane < 16) {
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        float w8[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) w8[i] = v[q8 * 8 + i];
                        *reinterpret_cast<uint4 *>(GA + kmaj_chunk(64 + r, c0 / 8 + q8, 128)) = pack8(w8);
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        sync();

        // 8. WQ leaves in one bulk store; the slot is published once it completed:
        //    the engine's first item at once (the scan is waiting for the first
        //    positions), later ones during the next item.
        if (tid == kStoreTid) {
            bulk_s2g(gslot + SL_WQ, GA, 32768);
            bulk_commit();
            prev_pending = true;  // `cur` is the previous item of the next iteration
            if (iter == 0) publish_prev(cur);
        }
    }
    // Publish the last item (after a failed wait: settle what is in flight).
    cp_async_wait_all();
    if (tid == kStoreTid) {
        bulk_wait_all();
        if (!failed && !sflag[1]) publish_prev(sitem[(iter + 2) % 3]);  // the last item
        if (la_pending) mbar_wait(&bars[0], la_phase ^ (failed ? 1u : 0u), kWaitNs);
        if (qk_pending) mbar_wait(&bars[2], qk_phase ^ 1u, kWaitNs);  // only after a failed wait
    }
    sync();
    if (tid == 0 && (failed || sflag[1])) fail_call(P);
}
// ---------------------------------------------------------------- scan ----
// Scan CTA for stream st, state columns [64 jv, 64 jv + 64). Warps 0..7:
// TMEM-lane epilogues (warp w: lanes 32 (w % 4) .., columns 32 (w / 4) ..);
// warp 8: the state chain's MMAs (Y, Z); warp 14: the other MMAs (O, the next
// position's T V), from its own thread so that their issue (tens of cycles per
// instruction) never delays the chain; warp 9: ring-slot copies; warp 10: V copies;
// warp 11: slot release; warps 12, 13: O rows to HBM (with the fused output step: RMSNorm over
// the row's 128 columns, the two scan CTAs of a stream exchanging their halves'
// sums of squares, and the sigmoid gate). TMEM lanes 0..63 hold O = Q e^G S + P U,
// 64..127 hold W S and T V (their difference is U); Z = Kd^T U fills all 128.
// The 128-row A operands of T V and P U take the 64 rows next to T (before) and
// P (after) as filler whose output rows are never read.
template <bool OG, bool CV>
__device__ __forceinline__ void scan_role(const FusedParams &P, uint8_t *sm, uint32_t tm, int st, int jv) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ns = P.ns, R = P.R, H = P.H;
    const long long NH = (long long)P.N * H;
    const long long K = (NH - st + ns - 1) / ns;  // units of this stream
    const long long L = reinterpret_cast<const long long *>(P.ws + WS_L)[st];
    Hdr *hd = reinterpret_cast<Hdr *>(P.ws);
    const int *ready = reinterpret_cast<const int *>(P.ws + ws_flags(NH));
    int *freed = const_cast<int *>(ready) + kFlagInts;
    const char *ring = P.ws + ws_ring(NH);
    uint8_t *sS = sm + SS_S, *sU = sm + SS_U;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SS_BAR);
    uint64_t *fullA = bars + MB_FULLA, *fullB = bars + MB_FULLB, *fullV = bars + MB_FULLV, *emptyA = bars + MB_EMPTYA,
             *emptyB = bars + MB_EMPTYB, *emptyV = bars + MB_EMPTYV, *bU = bars + MB_U, *bS = bars + MB_S,
             *bO = bars + MB_O, *uready = bars + MB_UREADY, *sready = bars + MB_SREADY, *bFin = bars + MB_FIN,
             *oready = bars + MB_OREADY, *bX = bars + MB_X, *bFin2 = bars + MB_FIN2, *convV = bars + MB_CV;
    auto unit_bounds = [&](long long kk, int &s, int &h, int64_t &bos, int64_t &eos) {
        const long long u = st + kk * ns;
        s = (int)(u / H);
        h = (int)(u % H);
        seq_bounds(P.cu, s, P.total, bos, eos);
    };

    if (warp == 9) {
        // ---------------- ring-slot copies (one thread) ----------------
        if (lane != 0) return;
        long long p = 0, nA = 0, nB = 0;  // positions whose A / B groups were issued
        int rpos = 0, rgen = 0;           // p % R and p / R
        bool ok = true;
        for (long long kk = 0; kk < K && ok; ++kk) {
            int s, h;
            int64_t bos, eos;
            unit_bounds(kk, s, h, bos, eos);
            const long long nch = (eos - bos + C - 1) / C;
            for (long long j = 0; j < nch; ++j, ++p) {
                // The slot's ready flag first (usually set long before: its gpu-scope read
                // then overlaps the wait for a free buffer), then the B group (three
                // buffers: free one position before the A group's two), then A.
                const int ab = (int)(p & 1), bb = (int)(p % 3);
                const int slot = st * R + rpos;
                ok = wait_flag_geq(&ready[slot], rgen + 1, &hd->abort_flag, P.xwait_ns, 32);
                if (++rpos == R) {
                    rpos = 0;
                    ++rgen;
                }
                if (ok && p >= 3) ok = mbar_wait_call(&emptyB[bb], (uint32_t)((p / 3 - 1) & 1), &hd->abort_flag);
                if (!ok) break;
                fence_proxy_async_global();
                const char *g = ring + (size_t)slot * SL_BYTES;
                uint8_t *A = sm + SS_A + ab * SA_BYTES, *B = sm + SS_B + bb * SB_BYTES;
                mbar_arrive_expect_tx(&fullB[bb], COPY_B);
                bulk_g2s(B + SB_T, g + SL_T, 8192, &fullB[bb]);
                bulk_g2s(B + SB_P, g + SL_P, 8192, &fullB[bb]);
                bulk_g2s(B + SB_D, g + SL_D, 1024, &fullB[bb]);
                nB = p + 1;
                if (p >= 2) ok = mbar_wait_call(&emptyA[ab], (uint32_t)((p / 2 - 1) & 1), &hd->abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(&fullA[ab], COPY_A);
                bulk_g2s(A + SA_WQ, g + SL_WQ, 32768, &fullA[ab]);
                bulk_g2s(A + SA_KD, g + SL_KD, 16384, &fullA[ab]);
                nA = p + 1;
            }
        }
        // Settle the copies still in flight (consumed ones return at once).
        for (long long q = (nA > 2 ? nA - 2 : 0); q < nA; ++q) mbar_wait(&fullA[q & 1], (uint32_t)((q / 2) & 1), kWaitNs);
        for (long long q = (nB > 3 ? nB - 3 : 0); q < nB; ++q) mbar_wait(&fullB[q % 3], (uint32_t)((q / 3) & 1), kWaitNs);
        if (!ok) fail_call(P);
        return;
    }
    // Positions whose tiles are in shared memory (written by the MMA thread).
    volatile long long *consumed = reinterpret_cast<volatile long long *>(bars + MB_COUNT);
    if (warp == 11) {
        // ---------------- ring-slot release (one thread) ----------------
        // Both scan CTAs of the stream release each slot once its tiles are in
        // their shared memory; the gpu-scope release (with the proxy fence it
        // needs) stays off the MMA thread.
        if (lane != 0) return;
        bool ok = true;
        for (long long p = 0; p < L && ok;) {
            long long upto = *consumed;
            if (upto <= p) {
                const uint64_t t0 = globaltimer_ns();
                while ((upto = *consumed) <= p) {
                    __nanosleep(64);
                    if (ld_relaxed_gpu(&hd->abort_flag) || globaltimer_ns() - t0 > kWaitNs) {
                        ok = false;
                        break;
                    }
                }
                if (!ok) break;
            }
            __threadfence_block();
            fence_proxy_async_global();
            for (; p < upto; ++p) red_release_gpu_add(&freed[st * R + (int)(p % R)], 1);
        }
        if (!ok) fail_call(P);
        return;
    }
    if (warp == 10) {
        // ---------------- V tiles (one thread), ahead of the ring ----------------
        if (lane != 0) return;
        long long p = 0;
        bool ok = true;
        for (long long kk = 0; kk < K && ok; ++kk) {
            int s, h;
            int64_t bos, eos;
            unit_bounds(kk, s, h, bos, eos);
            const long long nch = (eos - bos + C - 1) / C;
            for (long long j = 0; j < nch; ++j, ++p) {
                const int vb = (int)(p & 3);
                if (p >= 4) ok = mbar_wait_call(&emptyV[vb], (uint32_t)((p / 4 - 1) & 1), &hd->abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(&fullV[vb], SV_BYTES);
                tma_load_3d(sm + SS_V + vb * SV_BYTES, &P.tmap_v, jv * DVT, h, (int)(bos + j * C), &fullV[vb]);
            }
        }
        for (long long q = (p > 4 ? p - 4 : 0); q < p; ++q) mbar_wait(&fullV[q & 3], (uint32_t)((q / 4) & 1), kWaitNs);
        if (!ok) fail_call(P);
        return;
    }
    if (warp == 8) {
        // ---------------- the state chain's MMAs (one thread) ----------------
        if (lane != 0) return;
        const uint32_t id128 = idesc_bf16(128, DVT, false, true);  // K-major A, MN-major B
        const uint32_t idKd = idesc_bf16(128, DVT, true, true);    // MN-major A (Kd^T)
        // Descriptors of buffer 0; buffer i is i strides further (16-byte units).
        const uint64_t dWQ = sdesc(smem_u32(sm + SS_A + SA_WQ), 16, 1024);
        const uint64_t dKD = sdesc(smem_u32(sm + SS_A + SA_KD), C * 128, 1024);
        const uint64_t dS = sdesc(smem_u32(sS), DK * 128, 1024), dU = sdesc(smem_u32(sU), C * 128, 1024);
        constexpr uint64_t kA = SA_BYTES >> 4;
        bool ok = true;
        for (long long p = 0; p < L && ok; ++p) {
            const int ab = (int)(p & 1);
            const uint32_t yb = (uint32_t)(p % NY) * 64;
            ok = mbar_wait_call(&fullA[ab], (uint32_t)((p >> 1) & 1), &hd->abort_flag) &&
                 mbar_wait_call(&fullB[p % 3], (uint32_t)((p / 3) & 1), &hd->abort_flag);
            if (!ok) break;
            // Both tile groups of position p are in shared memory: its ring slot can be released.
            __threadfence_block();
            *consumed = p + 1;
            // S(p) in smem, and O(p - NY) read out of Y[p % NY] (one barrier per Y buffer: it
            // completes for positions p % NY, p % NY + NY, ... and so never runs two ahead)
            ok = mbar_wait_call(sready, (uint32_t)(p & 1), &hd->abort_flag) &&
                 (p < NY || mbar_wait_call(&oready[p % NY], (uint32_t)((p / NY + 1) & 1), &hd->abort_flag));
            if (!ok) break;
            if (p >= 1) mbar_arrive(&emptyB[(p - 1) % 3]);  // e^{Gl} of p-1 has been read
            tc_fence_after();
            // Y = [Q e^G ; W] S
            const uint64_t dWQa = dWQ + ab * kA, dKDa = dKD + ab * kA;
#pragma unroll
            for (int s8 = 0; s8 < DK / 16; ++s8)
                mma_bf16(tm + TM_Y + yb, dWQa + kmaj_step(s8, 128), dS + mnmaj_step(s8), id128, s8 > 0);
            mma_commit(bU);
            ok = mbar_wait_call(uready, (uint32_t)(p & 1), &hd->abort_flag);  // U(p) in smem
            if (!ok) break;
            tc_fence_after();
            // Z = Kd^T U (the state chain)
#pragma unroll
            for (int s4 = 0; s4 < C / 16; ++s4)
                mma_bf16(tm + TM_Z, dKDa + mnmaj_step(s4), dU + mnmaj_step(s4), idKd, s4 > 0);
            mma_commit(bS);
            mma_commit(&emptyA[ab]);
        }
        mma_commit(bFin);  // every MMA of this CTA completes before TMEM is freed
        if (!mbar_wait(bFin, 0, kWaitNs)) ok = false;
        if (!ok) fail_call(P);
        return;
    }
    if (warp == 12 || warp == 13) {
        // ---------------- O rows (warps 12, 13: TMEM lanes 0..63) ----------------
        const int c = (warp & 3) * 32 + lane;  // chunk row
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        constexpr bool gated = OG;
        float *sw = reinterpret_cast<float *>(sm + SS_OGW);
        unsigned long long *xw = reinterpret_cast<unsigned long long *>(P.ws + ws_xch(NH, P.ns, P.R));
        if (gated) {
            sw[c] = 0.5f * P.og_w[jv * DVT + c];
            bar_sync(7, 64);
        }
        // Row c of position q (Y buffer q % NY) to o: as it is, or with the output step
        // y * scale * w * sigmoid(g) = a + a tanh(g / 2), a = y scale (w / 2), in fp32 pairs.
        auto store_row = [&](long long q, int64_t t, int h, long long nn, float scale, const uint4 (&graw)[8]) {
            const uint32_t ybuf = tm + TM_Y + (uint32_t)(q % NY) * 64 + lane_base;
            bf16 *dst = P.o + ((size_t)t * H + h) * DV + jv * DVT;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float y[32];
                tmem_ld32(ybuf + half * 32, y);
                tmem_wait_ld();
                if (c < nn) {
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        uint32_t ow[4];
                        if (gated) {
                            const uint4 gr = graw[half * 4 + q8];
                            const uint32_t gw[4] = {gr.x, gr.y, gr.z, gr.w};
                            const f2_t s2 = f2(scale, scale), h2 = f2(0.5f, 0.5f);
#pragma unroll
                            for (int w = 0; w < 4; ++w) {
                                const f2_t g2 = f2mul(unpack2(gw[w]), h2);
                                float tl, th;
                                asm("tanh.approx.f32 %0, %1;" : "=f"(tl) : "f"(f2lo(g2)));
                                asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(f2hi(g2)));
                                const f2_t wv = *reinterpret_cast<const f2_t *>(sw + half * 32 + q8 * 8 + 2 * w);
                                const f2_t a = f2mul(f2mul(f2(y[q8 * 8 + 2 * w], y[q8 * 8 + 2 * w + 1]), s2), wv);
                                ow[w] = pack2(f2fma(a, f2(tl, th), a));
                            }
                        } else {
#pragma unroll
                            for (int w = 0; w < 4; ++w) ow[w] = pack2(f2(y[q8 * 8 + 2 * w], y[q8 * 8 + 2 * w + 1]));
                        }
                        reinterpret_cast<uint4 *>(dst)[half * 4 + q8] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&oready[q % NY]);  // Y[q % NY] may be overwritten (by Y(q + NY))
        };
        auto wait_o = [&](long long q) {  // O(q) complete
            const bool r = __all_sync(0xffffffffu, mbar_wait_call(&bO[q % NY], (uint32_t)((q / NY) & 1), &hd->abort_flag));
            tc_fence_after();
            return r;
        };
        bool ok = true;
        long long p = 0;
        if (!gated) {
            const uint4 none[8] = {};
            // With the fused convolution of v (and no output step) these two warps also
            // convolve the V tiles, two positions ahead of the O rows they store: lane l
            // takes channels 2 l, 2 l + 1 of this CTA's 64, warp 12 rows 0..31 and warp 13
            // rows 32..63 of the tile. Every raw row either warp needs is read before
            // either rewrites one; warp 13 leaves raw rows 61..63 in VPREV for warp 12's
            // window at the next chunk (a unit's first chunk reads the initial state).
            const bool vconv = CV && P.cw[2] != 0;
            const int hv = warp & 1, ch = jv * DVT + 2 * lane;  // first channel within the head
            const int Wv = P.cw[2];
            uint32_t *vprev = reinterpret_cast<uint32_t *>(sm + SS_VPREV);  // [3][32] raw pairs
            long long vk = -1, vj = 0, vn = 0;  // the convolution's unit and chunk cursor
            f2_t vw[4] = {0ull, 0ull, 0ull, 0ull};
            f2_t vstate[3] = {0ull, 0ull, 0ull};  // warp 12: the unit's initial window
            auto conv_v = [&](long long q) {  // the V tile of position q (positions in order)
                bool unit_start = false;
                while (vj >= vn) {  // the next unit with chunks: its taps and initial state
                    int s, h;
                    int64_t bos, eos;
                    unit_bounds(++vk, s, h, bos, eos);
                    vn = (eos - bos + C - 1) / C;
                    vj = 0;
                    unit_start = true;
                    const float *wt = P.cwt[2] + ((size_t)h * DV + ch) * Wv;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        vw[j] = j - (4 - Wv) >= 0 ? f2(__ldg(wt + j - (4 - Wv)), __ldg(wt + Wv + j - (4 - Wv))) : f2(0.f, 0.f);
#pragma unroll
                    for (int jh = 0; jh < 3; ++jh) {
                        const int js = jh + Wv - 4;
                        vstate[jh] = (P.cst[2] != nullptr && js >= 0)
                                         ? unpack2(*reinterpret_cast<const uint32_t *>(
                                               P.cst[2] + ((size_t)s * (Wv - 1) + js) * ((size_t)H * DV) + (size_t)h * DV + ch))
                                         : f2(0.f, 0.f);
                    }
                }
                const int vb = (int)(q & 3);
                if (!__all_sync(0xffffffffu, mbar_wait_call(&fullV[vb], (uint32_t)((q >> 2) & 1), &hd->abort_flag)))
                    return false;
                uint8_t *tile = sm + SS_V + vb * SV_BYTES;
                auto word = [&](int r) {  // this lane's pair of row r (SW128 rows of 128 bytes)
                    return reinterpret_cast<uint32_t *>(tile + r * 128 + (((lane >> 2) ^ (r & 7)) << 4) + (lane & 3) * 4);
                };
                const int r0 = hv * 32;
                f2_t win[3];  // the three raw rows before the next one to convolve
                if (hv == 0) {
#pragma unroll
                    for (int jh = 0; jh < 3; ++jh) win[jh] = unit_start ? vstate[jh] : unpack2(vprev[jh * 32 + lane]);
                } else {
#pragma unroll
                    for (int jh = 0; jh < 3; ++jh) win[jh] = unpack2(*word(r0 - 3 + jh));
                }
                bar_sync(7, 64);  // the rows each warp needs from the other's half are in registers
                for (int r8 = 0; r8 < 32; r8 += 8) {  // eight rows at a time, loads first
                    f2_t x[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) x[i] = unpack2(*word(r0 + r8 + i));
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        f2_t z = f2fma(vw[0], win[0], f2(0.f, 0.f));
                        z = f2fma(vw[1], win[1], z);
                        z = f2fma(vw[2], win[2], z);
                        z = f2fma(vw[3], x[i], z);
                        *word(r0 + r8 + i) = pack2(swish2(z));
                        win[0] = win[1];
                        win[1] = win[2];
                        win[2] = x[i];
                    }
                }
                if (hv == 1) {
#pragma unroll
                    for (int jh = 0; jh < 3; ++jh) vprev[jh * 32 + lane] = pack2(win[jh]);
                }
                ++vj;
                fence_async_smem();  // the rewritten tile is read by the tensor cores
                bar_sync(7, 64);
                if (warp == 12 && lane == 0) mbar_arrive(&convV[vb]);
                return true;
            };
            if (vconv)
                for (long long q = 0; q < 2 && q < L && ok; ++q) ok = conv_v(q);
            for (long long kk = 0; kk < K && ok; ++kk) {
                int s, h;
                int64_t bos, eos;
                unit_bounds(kk, s, h, bos, eos);
                const long long len = eos - bos, nch = (len + C - 1) / C;
                for (long long j = 0; j < nch; ++j, ++p) {
                    if (!(ok = wait_o(p))) break;
                    const long long nn = (len - j * C) < C ? (len - j * C) : C;
                    store_row(p, bos + j * C + c, h, nn, 1.f, none);
                    if (vconv && p + 2 < L && !(ok = conv_v(p + 2))) break;
                }
            }
        } else {
            // With the output step a row's RMSNorm needs the partner CTA's 64 columns:
            // each thread publishes its row's sum of squares, tagged with the position,
            // in one 8-byte word (four per row, by position modulo 4) and reads the
            // partner's word one position later: position p - 1 is stored after the sum
            // of p is published, so the round trip is hidden behind O(p). A word is
            // rewritten four positions later; the partner has read it by then (it
            // published p - 2, which this CTA needed for p - 2, only after finishing
            // p - 4's read).
            auto publish = [&](long long q, float ss) {
                const unsigned long long tag = (unsigned long long)(q + 1) << 32;
                st_relaxed_gpu_u64(&xw[((st * 2 + jv) * 4 + (q & 3)) * 64 + c], tag | __float_as_uint(ss));
            };
            auto partner = [&](long long q, float &v) {
                const unsigned long long tag = (unsigned long long)(q + 1) << 32;
                const unsigned long long *pw = &xw[((st * 2 + (jv ^ 1)) * 4 + (q & 3)) * 64 + c];
                unsigned long long got = ld_relaxed_gpu_u64(pw);
                if ((got >> 32) != (tag >> 32)) {
                    const uint64_t t0 = globaltimer_ns();
                    while (((got = ld_relaxed_gpu_u64(pw)) >> 32) != (tag >> 32))
                        if (globaltimer_ns() - t0 > P.xwait_ns || ld_relaxed_gpu(&hd->abort_flag)) break;
                }
                v = __uint_as_float((uint32_t)got);
                return __all_sync(0xffffffffu, (got >> 32) == (tag >> 32));
            };
            auto load_gate = [&](int64_t t, int h, long long nn, uint4 (&graw)[8]) {
                const bf16 *grow = P.og_gate + ((size_t)t * H + h) * DV + jv * DVT;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    graw[i] = c < nn ? __ldg(reinterpret_cast<const uint4 *>(grow) + i) : make_uint4(0, 0, 0, 0);
            };
            bool havep = false;  // position p - 1 is still to be stored
            int64_t tp = 0;
            int hp = 0;
            long long nnp = 0;
            float ssp = 0.f;
            for (long long kk = 0; kk < K && ok; ++kk) {
                int s, h;
                int64_t bos, eos;
                unit_bounds(kk, s, h, bos, eos);
                const long long len = eos - bos, nch = (len + C - 1) / C;
                for (long long j = 0; j < nch; ++j, ++p) {
                    uint4 graw[8];
                    if (havep) load_gate(tp, hp, nnp, graw);  // in flight during the wait and the sum
                    if (!(ok = wait_o(p))) break;
                    float ss = 0.f;
                    const uint32_t ybuf = tm + TM_Y + (uint32_t)(p % NY) * 64 + lane_base;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float y[32];
                        tmem_ld32(ybuf + half * 32, y);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) ss = fmaf(y[i], y[i], ss);
                    }
                    publish(p, ss);
                    if (havep) {
                        float other;
                        if (!(ok = partner(p - 1, other))) break;
                        store_row(p - 1, tp, hp, nnp, rsqrtf((ssp + other) * (1.f / DV) + P.og_eps), graw);
                    }
                    havep = true;
                    tp = bos + j * C + c;
                    hp = h;
                    nnp = (len - j * C) < C ? (len - j * C) : C;
                    ssp = ss;
                    if (c < nnp)  // this row's gate, read in the next iteration: into L2 now
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(P.og_gate + ((size_t)tp * H + hp) * DV + jv * DVT));
                }
            }
            if (ok && havep) {
                uint4 graw[8];
                load_gate(tp, hp, nnp, graw);
                float other;
                if ((ok = partner(p - 1, other)))
                    store_row(p - 1, tp, hp, nnp, rsqrtf((ssp + other) * (1.f / DV) + P.og_eps), graw);
            }
        }
        if (!ok) fail_call(P);
        return;
    }
    if (warp == 14) {
        // ---------------- the other MMAs (one thread) ----------------
        // After U(p) is in shared memory: O(p) into Y[p % NY] (Y(p) has completed: the U
        // epilogue read it) and T V of the next position into its X buffer (read by the
        // U epilogue of position p - 1, which has finished).
        if (lane != 0) return;
        const uint32_t id128 = idesc_bf16(128, DVT, false, true);  // K-major A, MN-major B
        const uint64_t dTf = sdesc(smem_u32(sm + SS_B + SB_T) - 8192, 16, 1024);  // filler, then T
        const uint64_t dP = sdesc(smem_u32(sm + SS_B + SB_P), 16, 1024);          // P, then filler
        const uint64_t dV = sdesc(smem_u32(sm + SS_V), C * 128, 1024);
        const uint64_t dU = sdesc(smem_u32(sU), C * 128, 1024);
        constexpr uint64_t kB = SB_BYTES >> 4, kV = SV_BYTES >> 4;
        // X[q & 1] = [filler ; T] V of position q, once its T and V tiles are in.
        auto issue_x = [&](long long q) {
            const int bb = (int)(q % 3), vb = (int)(q & 3);
            if (!(mbar_wait_call(&fullB[bb], (uint32_t)((q / 3) & 1), &hd->abort_flag) &&
                  mbar_wait_call(CV && P.cw[2] ? &convV[vb] : &fullV[vb], (uint32_t)((q >> 2) & 1), &hd->abort_flag)))
                return false;
            tc_fence_after();
#pragma unroll
            for (int s4 = 0; s4 < C / 16; ++s4)
                mma_bf16(tm + TM_X + (uint32_t)(q & 1) * 64, dTf + bb * kB + kmaj_step(s4, 128), dV + vb * kV + mnmaj_step(s4),
                         id128, s4 > 0);
            mma_commit(&emptyV[vb]);
            mma_commit(&bX[q & 1]);
            return true;
        };
        bool ok = true;
        if (L > 0) ok = issue_x(0);
        for (long long p = 0; p < L && ok; ++p) {
            const int bb = (int)(p % 3);
            const uint32_t yb = (uint32_t)(p % NY) * 64;
            // Z(p) complete (so U(p) is in smem and Y(p) complete): the chain's product runs first
            ok = mbar_wait_call(bS, (uint32_t)(p & 1), &hd->abort_flag);
            if (!ok) break;
            tc_fence_after();
            // O: Y += [P ; filler] U
#pragma unroll
            for (int s4 = 0; s4 < C / 16; ++s4)
                mma_bf16(tm + TM_Y + yb, dP + bb * kB + kmaj_step(s4, 128), dU + mnmaj_step(s4), id128, 1);
            mma_commit(&bO[p % NY]);
            mma_commit(&emptyB[bb]);
            if (p + 1 < L && !(ok = issue_x(p + 1))) break;
        }
        mma_commit(bFin2);  // every MMA of this thread completes before TMEM is freed
        if (!mbar_wait(bFin2, 0, kWaitNs)) ok = false;
        if (!ok) fail_call(P);
        return;
    }
    if (warp == 15) {
        // ---------------- fused short convolution of the V tiles ----------------
        // Lane l takes channels 2 l, 2 l + 1 of this CTA's 64 (SW128 rows of 128 bytes),
        // row by row in place, keeping the last three raw rows in registers: from the
        // initial state (or zeros) at a unit's first chunk, then from the previous tile.
        // The same arithmetic as the standalone convolution kernel.
        if (!CV || !OG || P.cw[2] == 0) return;  // without the output step warps 12, 13 do it
        const int W = P.cw[2];
        const int ch = jv * DVT + 2 * lane;  // channel within the head
        bool ok = true;
        long long p = 0;
        for (long long kk = 0; kk < K && ok; ++kk) {
            int s, h;
            int64_t bos, eos;
            unit_bounds(kk, s, h, bos, eos);
            const long long nch = (eos - bos + C - 1) / C;
            if (nch == 0) continue;
            const float *wt = P.cwt[2] + ((size_t)h * DV + ch) * W;
            f2_t wp[4], win[3];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int jj = j - (4 - W);
                wp[j] = jj >= 0 ? f2(__ldg(wt + jj), __ldg(wt + W + jj)) : f2(0.f, 0.f);
            }
#pragma unroll
            for (int jh = 0; jh < 3; ++jh) {
                const int js = jh + W - 4;
                win[jh] = (P.cst[2] != nullptr && js >= 0)
                              ? unpack2(*reinterpret_cast<const uint32_t *>(
                                    P.cst[2] + ((size_t)s * (W - 1) + js) * ((size_t)H * DV) + (size_t)h * DV + ch))
                              : f2(0.f, 0.f);
            }
            for (long long j = 0; j < nch; ++j, ++p) {
                const int vb = (int)(p & 3);
                if (!(ok = __all_sync(0xffffffffu, mbar_wait_call(&fullV[vb], (uint32_t)((p >> 2) & 1), &hd->abort_flag))))
                    break;
                uint8_t *tile = sm + SS_V + vb * SV_BYTES;
                for (int r0 = 0; r0 < C; r0 += 16) {  // 16 rows at a time, all loads first
                    f2_t ext[19];                       // raw rows r0 - 3 .. r0 + 15
                    ext[0] = win[0];
                    ext[1] = win[1];
                    ext[2] = win[2];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int r = r0 + i;
                        ext[3 + i] = unpack2(*reinterpret_cast<const uint32_t *>(
                            tile + r * 128 + (((lane >> 2) ^ (r & 7)) << 4) + (lane & 3) * 4));
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int r = r0 + i;
                        f2_t z = f2fma(wp[0], ext[i], f2(0.f, 0.f));
                        z = f2fma(wp[1], ext[i + 1], z);
                        z = f2fma(wp[2], ext[i + 2], z);
                        z = f2fma(wp[3], ext[i + 3], z);
                        *reinterpret_cast<uint32_t *>(tile + r * 128 + (((lane >> 2) ^ (r & 7)) << 4) + (lane & 3) * 4) =
                            pack2(swish2(z));
                    }
                    win[0] = ext[16];
                    win[1] = ext[17];
                    win[2] = ext[18];
                }
                fence_async_smem();  // the rewritten tile is read by the tensor cores
                __syncwarp();
                if (lane == 0) mbar_arrive(&convV[vb]);
            }
        }
        if (!ok) fail_call(P);
        return;
    }
    if (warp >= 8) return;

    // ---------------- epilogues (TMEM lane = state row c) ----------------
    const int q4 = warp & 3, hf = warp >> 2;
    const int c = q4 * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16, col = (uint32_t)(hf * 32);
    float Sr[32];
    auto load_state = [&](const float *src, size_t sofs) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 x = src ? *reinterpret_cast<const float4 *>(src + sofs + 4 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
            Sr[4 * q] = x.x;
            Sr[4 * q + 1] = x.y;
            Sr[4 * q + 2] = x.z;
            Sr[4 * q + 3] = x.w;
        }
    };
    auto store_state = [&](float *dst, size_t sofs) {
        if (!dst) return;
#pragma unroll
        for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4 *>(dst + sofs + 4 * q) = make_float4(Sr[4 * q], Sr[4 * q + 1], Sr[4 * q + 2], Sr[4 * q + 3]);
    };
    auto state_to_smem = [&]() {  // bf16 copy: B operand of the next chunk's products
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
            float x[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = Sr[q8 * 8 + i];
            *reinterpret_cast<uint4 *>(sS + mnmaj_chunk(c, hf * 4 + q8, DK)) = pack8(x);
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(sready);
    };
    bool ok = true;
    long long p = 0;
    for (long long kk = 0; kk < K && ok; ++kk) {
        int s, h;
        int64_t bos, eos;
        unit_bounds(kk, s, h, bos, eos);
        const long long len = eos - bos, nch = (len + C - 1) / C;
        const size_t sofs = ((size_t)((long long)s * H + h) * DK + c) * DV + jv * DVT + hf * 32;
        load_state(P.S0, sofs);
        if (nch == 0) {
            store_state(P.S_T, sofs);
            continue;
        }
        state_to_smem();
        for (long long j = 0; j < nch; ++j, ++p) {
            const uint32_t xb = (uint32_t)(p & 1) * 64, yb = (uint32_t)(p % NY) * 64;
            const uint32_t par = (uint32_t)(p & 1);
            if (q4 >= 2) {
                // U = T V - W S for rows r = c - 64 (TMEM lanes 64..127), once Y(p) and X(p) have
                // completed and O(p - 1) has read the previous U
                ok = __all_sync(0xffffffffu, mbar_wait_call(bU, par, &hd->abort_flag) &&
                                                 mbar_wait_call(&bX[p & 1], (uint32_t)((p >> 1) & 1), &hd->abort_flag) &&
                                                 (p == 0 || mbar_wait_call(&bO[(p - 1) % NY], (uint32_t)(((p - 1) / NY) & 1),
                                                                           &hd->abort_flag)));
                if (!ok) break;
                tc_fence_after();
                float xv[32], yv[32];
                tmem_ld32(tm + TM_X + xb + lane_base + col, xv);
                tmem_ld32(tm + TM_Y + yb + lane_base + col, yv);
                tmem_wait_ld();
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    float u8[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) u8[i] = xv[q8 * 8 + i] - yv[q8 * 8 + i];
                    *reinterpret_cast<uint4 *>(sU + mnmaj_chunk(c - 64, hf * 4 + q8, C)) = pack8(u8);
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(uready);
            }
            // S' = Diag(e^{G_last}) S + Z  (row c)
            ok = __all_sync(0xffffffffu, mbar_wait_call(bS, par, &hd->abort_flag) &&
                                             mbar_wait_call(&fullB[p % 3], (uint32_t)((p / 3) & 1), &hd->abort_flag));
            if (!ok) break;
            tc_fence_after();
            const float *dd = reinterpret_cast<const float *>(sm + SS_B + (p % 3) * SB_BYTES + SB_D);
            const float dc = dd[c], dz = dd[DK + c];
            {
                float zv[32];
                tmem_ld32(tm + TM_Z + lane_base + col, zv);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) Sr[i] = fmaf(dc, Sr[i], dz * zv[i]);
            }
            if (j + 1 < nch) state_to_smem();
        }
        if (ok) store_state(P.S_T, sofs);
    }
    if (!ok) fail_call(P);
}

// ----------------------------------------------------------- the kernel ----
// OG: with the fused output step; CV: with the fused short convolution (each its own
// instantiation, so that the plain prefill carries neither's code).
template <bool OG, bool CV>
__global__ void __launch_bounds__(kThreads, 1) fused_kernel(const __grid_constant__ FusedParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctrl *ctl = reinterpret_cast<Ctrl *>(sm + CTRL_OFF);
    const int tid = threadIdx.x, warp = tid >> 5;
    const bool scan = (int)blockIdx.x < 2 * P.ns;
    if (tid == 0) {
        if (scan) {
            uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SS_BAR);
            for (int i = 0; i < MB_COUNT; ++i) {
                uint32_t count = 1;
                if (i >= MB_EMPTYB && i < MB_EMPTYB + 3) count = 2;  // MMA commit + e^{Gl} read
                if (i == MB_UREADY) count = 128;  // epilogue threads of TMEM lanes 64..127
                if (i == MB_SREADY) count = 256;  // all epilogue threads
                if (i >= MB_OREADY && i < MB_OREADY + NY) count = 64;  // O epilogue threads
                mbar_init(&bars[i], count);
            }
            *reinterpret_cast<long long *>(bars + MB_COUNT) = 0;
        } else {
            for (int e = 0; e < 2; ++e) {
                uint64_t *bars = reinterpret_cast<uint64_t *>(sm + e * PS_STRIDE + PS_BAR);
                mbar_init(&bars[0], 1);
                mbar_init(&bars[1], 1);
                mbar_init(&bars[2], 1);
                int *sflag = reinterpret_cast<int *>(reinterpret_cast<ItemS *>(bars + 3) + 3);
                sflag[0] = 0;
                sflag[1] = 0;
                sflag[2] = 0;
            }
        }
        fence_barrier_init();
    }
    if (!scan) {
        const Hdr *hd = reinterpret_cast<const Hdr *>(P.ws);
        if (tid < P.ns) {
            ctl->L[tid] = reinterpret_cast<const long long *>(P.ws + WS_L)[tid];
            ctl->order[tid] = reinterpret_cast<const int *>(P.ws + WS_ORDER)[tid];
        }
        if (tid == 64) {
            ctl->total = hd->total;
            ctl->maxlen = hd->maxlen;
            ctl->uniform = hd->uniform;
        }
        const long long NH = (long long)P.N * P.H;
        int *uc = reinterpret_cast<int *>(sm + CACHE_OFF);
        const bool ucache = NH <= kUnitCache, ccache = P.cu != nullptr && P.N + 1 <= kSeqCache;
        if (tid == 96) {
            ctl->ucache = ucache;
            ctl->ccache = ccache;
        }
        if (ucache)  // positions in a stream fit in 32 bits
            for (int u = tid; u < (int)NH; u += kThreads) uc[u] = (int)reinterpret_cast<const long long *>(P.ws + WS_USTART)[u];
        if (ccache)
            for (int s = tid; s <= P.N; s += kThreads) uc[kUnitCache + s] = P.cu[s];
    }
    if (warp == 0) {
        tmem_alloc(&ctl->tbase, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = ctl->tbase;
    if (scan) scan_role<OG, CV>(P, sm, tm, blockIdx.x >> 1, blockIdx.x & 1);
    else prep_engine<CV>(P, ctl, tid >> 8, sm + (tid >> 8) * PS_STRIDE, tm + 256u * (uint32_t)(tid >> 8));
    tc_fence_before();
    __syncthreads();
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

// q, k or v viewed as [T][H][128] bf16; a box is 64 columns x 1 head x 64 tokens, SW128.
bool make_rows_map(CUtensorMap *m, const void *v, int64_t total, int H) {
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

// log_alpha viewed as [T][H][128] fp32; a box is 128 channels x 1 head x 64 tokens.
bool make_la_map(CUtensorMap *m, const void *base, int64_t total, int H) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)DK, (cuuint64_t)H, (cuuint64_t)total};
    const cuuint64_t strides[2] = {(cuuint64_t)DK * 4, (cuuint64_t)H * DK * 4};
    const cuuint32_t box[3] = {(cuuint32_t)DK, 1, (cuuint32_t)C};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t tc_workspace_bytes(long long NH, int ns, int R) {
    return ws_xch(NH, ns, R) + kXchWords * 8;
}

int tc_ring_slots(long long NH, int ns, size_t bytes) {
    const size_t base = ws_ring(NH) + kXchWords * 8;  // the ring, then the exchange words
    if (ns < 1 || bytes < base) return 0;
    const size_t r = (bytes - base) / ((size_t)ns * SL_BYTES);
    return (int)(r < (size_t)kMaxRing ? r : (size_t)kMaxRing);
}

int tc_max_ring() { return kMaxRing; }

namespace {
std::atomic<unsigned long long> g_xwait_ns{kDefaultWaitNs};
}
uint64_t tc_set_wait_limit(uint64_t ns) { return g_xwait_ns.exchange(ns ? ns : kDefaultWaitNs); }

cudaError_t tc_prefill(const PrefillArgs &a, char *ws, size_t ws_bytes, int ns, int *err, cudaStream_t st) {
    cudaError_t e;
    const bool og = a.og_gate != nullptr, cv = (a.conv_W[0] | a.conv_W[1] | a.conv_W[2]) != 0;
    void (*kern)(FusedParams) = og ? (cv ? fused_kernel<true, true> : fused_kernel<true, false>)
                                   : (cv ? fused_kernel<false, true> : fused_kernel<false, false>);
    // Per device (context): cheap enough to set on every call.
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC)) !=
        cudaSuccess)
        return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, SMEM_ALLOC)) != cudaSuccess)
        return e;
    const int grid = per_sm * sms;
    // At least two prep CTAs beside the scan CTAs.
    if (2 * ns + 2 > grid) ns = (grid - 2) / 2;
    if (ns < 1) return cudaErrorLaunchOutOfResources;
    const long long NH = (long long)a.N * a.H;
    const int R = tc_ring_slots(NH, ns, ws_bytes);
    if (R < 1) return cudaErrorInvalidValue;

    FusedParams P;
    memset(&P, 0, sizeof(P));
    if (a.total > 0 && ((!a.la_scalar && !make_la_map(&P.tmap_la, a.log_alpha, a.total, a.H)) ||
                        !make_rows_map(&P.tmap_v, a.v, a.total, a.H) || !make_rows_map(&P.tmap_q, a.q, a.total, a.H) ||
                        !make_rows_map(&P.tmap_k, a.k, a.total, a.H)))
        return cudaErrorInvalidValue;
    P.la = a.log_alpha;
    P.la_scalar = a.la_scalar;
    P.og_gate = static_cast<const bf16 *>(a.og_gate);
    P.og_w = a.og_w;
    P.og_eps = a.og_eps;
    P.q = static_cast<const bf16 *>(a.q);
    P.k = static_cast<const bf16 *>(a.k);
    P.v = static_cast<const bf16 *>(a.v);
    for (int i = 0; i < 3; ++i) {
        P.cw[i] = a.conv_W[i];
        P.cwt[i] = a.conv_w[i];
        P.cst[i] = static_cast<const bf16 *>(a.conv_state[i]);
    }
    P.beta = a.beta;
    P.S0 = a.S0;
    P.cu = a.cu;
    P.S_T = a.S_T;
    P.o = static_cast<bf16 *>(a.o);
    P.ws = ws;
    P.err = err;
    P.total = a.total;
    P.xwait_ns = g_xwait_ns.load();
    P.N = a.N;
    P.H = a.H;
    P.ns = ns;
    P.R = R;
    P.l2norm = a.l2norm;
    P.eps = a.eps;

    plan_kernel<<<1, PLAN_T, 0, st>>>(a.cu, a.total, a.N, a.H, ns, R, ws);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_ALLOC;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, P);
}

}  // namespace kda
