// chunk_cluster.cu -- cluster engine of the chunked KDA prefill on sm_100a
// (bf16 q/k/v, d_k = d_v = 128, chunk C = 64, fp32 gates and state).
//
// Chunked form (Kimi Linear summary, es.news.hada.io/topic?id=31936, sections
// "Algoritmo paralelo por chunks" and "Menor cantidad de operaciones que DPLR
// general"). Per chunk, with g the in-chunk inclusive prefix sum of log alpha:
//   A = Diag(beta) strict_lower(K~ K^T),  P = lower(Q~ K^T)   (entries carry e^{g_i - g_j})
//   T = (I + A)^{-1} Diag(beta),  [W | U'] = T [Ks | V]       (Ks = K e^{g})
//   state chain: X = [Qs ; W] S, U = U' - W S, O = Qs S + P U,
//                S <- Diag(e^{g_C}) S + Kb^T U                 (Qs = Q e^{g}, Kb = K e^{g_C - g})
//
// The two intra-chunk products are built from 16-token sub-chunks (the
// summary's secondary chunking for fine-grained decay), so that no gate factor
// leaves the floating-point range whatever the decay:
//   * a block (I, J) below the diagonal (row sub-chunk I, column sub-chunk
//     J < I) uses e^{g_i - g_j} = e^{g_i - G_I} e^{G_I - G_{J+1}} e^{G_{J+1} - g_j},
//     G_I = g at the end of sub-chunk I-1: all three factors are <= 1. The row
//     operand (with the middle factor, per channel) stays in the registers of
//     the warp that owns sub-chunk I; the column operand K e^{G_{J+1} - g} is
//     written once to shared memory; tf32 mma.sync, like the diagonal blocks;
//   * a diagonal block (I, I) anchors both factors at the sub-chunk's 8th token
//     m: e^{g_i - g_m} e^{g_m - g_j}, each within e^{87} whenever the
//     sub-chunk's total decay is within e^{-87}; computed in tf32 with
//     warp-level mma.sync from registers. A channel whose sub-chunk decays
//     further takes its factors from log alpha clamped at -10 per token: every
//     product that changes is then below e^-10 before and after, a change
//     (< 4.6e-5) below the tf32 rounding of the same factor (2^-11).
//
// The work of one chunk splits into a key-side part that does not depend on
// the state (everything up to W, U', P, T, Qs, Kb) and the state chain, which
// is sequential over chunks. One head runs on a cluster of 4 CTAs (4 SMs):
//   * ranks 0..2 are producers: rank p computes the key-side part of chunks
//     p, p+3, p+6, ... as an 82 KB image and writes it into one of its three
//     slots of a small ring in the workspace (it stays in L2). Each part (Qs,
//     Kb, [P;T] -- also an operand of its own MMA --, W, U') is staged in
//     shared memory in its image layout and bulk-stored (cp.async.bulk shared
//     -> global) by one thread of a warp that has no share of the phase that
//     follows, so that the copies (~27 B/cycle per SM, like any store path of
//     an SM into L2) overlap the computation; e^{g_C} goes straight from
//     registers. Once the stores are complete, the same thread arrives
//     (release, cluster scope; the generic stores of all threads precede it
//     through a CTA barrier) on the consumer's "ready" barrier of that slot;
//   * rank 3 is the consumer: it keeps the 128x128 fp32 state in registers and
//     runs the chain for every chunk, on all 128 value columns. Its thread 0
//     pulls published images into two shared-memory slots (bulk global ->
//     shared loads) as soon as a slot is free, and tells the producer (its
//     "loaded" barrier) that the ring slot may be reused.
// The ring goes through L2 because a DSMEM bulk copy moves only ~20 B/cycle
// between two SMs, whereas an L2 bulk load of the same 82 KB takes ~1K cycles.
// Every wait is bounded; after a timeout a CTA records an error in the device
// error word, stops waiting and still reaches the final cluster barrier and
// frees its tensor memory.
#include <cuda.h>

#include "kda_internal.cuh"
#include "tc_sm100.cuh"
#include "ut_solve.cuh"

namespace kda {
namespace {

using tc::fence_proxy_async_smem;
using tc::mma_f16;
using tc::pack_bf16;
using tc::pack_f16;
using tc::sw128k_off;
using tc::tc_fence_after;
using tc::tc_fence_before;
using ut::kLD;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 256;
constexpr int kLoader = 32;     // producer thread that issues the TMA input loads (warp 1)
constexpr int kStorer = 224;    // producer thread that issues the bulk stores and publishes (warp 7)
constexpr int kProducers = 3;
constexpr int kCluster = kProducers + 1;
constexpr int kRingDepth = 3;   // ring slots per producer
constexpr int kRingSlots = kRingDepth * kProducers;
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr uint32_t kTestWaitLimit = 1u << 12;   // polls of a bounded wait under the test hook
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRangeLog = -87.f;   // e^-87 ~ 1.6e-38: factors of a sub-chunk stay normal above it
constexpr float kClampLog = -10.f;   // per-token clamp of log alpha for the fallback factors
constexpr float kFastTot = 40.f;     // sub-chunk decay bound of the one-anchor path (chunk total <= 160)

// ---- slot image: what a producer hands the consumer for one chunk
constexpr uint32_t SL_QW = 0;          // [Qs ; W] fp16 K-major SW128, 2 K-blocks x 16 KB
constexpr uint32_t kQWBlk = 16384;
constexpr uint32_t SL_KB = 32768;      // Kb fp16 [token][channel], 2 blocks x 8 KB
constexpr uint32_t SL_PT = 49152;      // [P ; T] fp16 K-major SW128, K = 64
constexpr uint32_t SL_UP = 65536;      // U' fp16 [token][col], 2 blocks x 8 KB
constexpr uint32_t SL_GAM = 81920;     // e^{g_C} fp32 [128]
constexpr uint32_t kSlotBytes = 82432;
constexpr uint32_t kSlotStride = 82944;
constexpr uint32_t kTokBlk = 8192;
static_assert(kRingSlots * kSlotStride == kClusterRingBytesPerHead, "ring size");
static_assert(kClusterMaxRings <= 8 * static_cast<int>(kClusterPoolHeader), "pool bitmap");

// ---- producer shared memory
// Inputs of a chunk (TMA). q, k and log alpha come as 128-byte rows in the
// 128-byte swizzle (16-byte piece p of token row r stored at piece p ^ (r % 8)),
// so that the prologue's fragment-ordered reads are free of bank conflicts.
constexpr uint32_t P_IN_Q = 0;         // q: 2 boxes (64 channels each) x [64 tokens][128 B]
constexpr uint32_t P_IN_K = 16384;     // k: same
constexpr uint32_t P_IN_LA = 32768;    // log alpha: 4 boxes (32 channels each) x [64][128 B]
constexpr uint32_t P_IN_V = 65536;     // v [64][128] bf16, plain rows
constexpr uint32_t kBoxBytes = 8192;
constexpr uint32_t kInBytes = 81920;
// ... or, for the fused layer prologue (raw q, k and the gate's pre-activation x):
constexpr uint32_t P_IN_X = 32768;     // x: 2 boxes (64 channels each, bf16) x [64][128 B]
constexpr uint32_t P_IN_VF = 49152;    // v
constexpr uint32_t kInBytesF = 65536;
// ... and once the prologue has read them, the same region holds:
constexpr uint32_t P_AF = 0;                   // A fp32 [64][kLD]
constexpr uint32_t P_XF = 64 * kLD * 4;        // X = (I + A)^{-1} fp32 [64][kLD]
constexpr uint32_t P_DX = 2 * 64 * kLD * 4;    // diagonal-block partials of channels 64..127 (8 KB)
constexpr uint32_t P_PX = P_DX + 8192;         // off-diagonal-block partials, both halves: 2 x 6 x 2 KB
// K e^{G_{J+1} - g} (fp32), the column operand of the off-diagonal blocks, in the
// swizzled layout of log alpha (phases 1b and 2); then W (2 K-blocks x 8 KB) and U'
// (16 KB) staged for the ring, until their bulk stores have read them (before the next
// image's phase 1b)
constexpr uint32_t P_KSIG = 81920;
// (one-anchor path: the tf32 operands of [A;P] over the same region, 0 .. 96 KB)
constexpr uint32_t P_KQT = 0;          // [K e^{g - g_C/2} ; Q e^{g - g_C/2}], 4 K-blocks (32 channels) x 16 KB
constexpr uint32_t kKQTBlk = 16384;
constexpr uint32_t P_KHT = 65536;      // K e^{g_C/2 - g}, 4 K-blocks x 8 KB
constexpr uint32_t kKHTBlk = 8192;
constexpr uint32_t P_WS = P_KSIG;
constexpr uint32_t P_US = P_KSIG + 16384;
constexpr uint32_t P_KBS = P_KSIG + 32768;   // Kb staged for the ring (image layout)
constexpr uint32_t P_STAGE = 131072;
constexpr uint32_t ST_PT = 0;          // [P;T] 16 KB (A operand of [W | U'], bulk-stored to the ring)
constexpr uint32_t ST_GL = 16384;      // g^L in the layout of log alpha (32 KB, phases 1a-1b), then
constexpr uint32_t ST_QS = ST_GL;      // Qs staged for the ring, 2 K-blocks x 8 KB
constexpr uint32_t P_KSV = 180224;     // [Ks | V] fp16 [token][col], 4 blocks x 8 KB
// beta of two chunks [2][64] (the next one arrives by cp.async during this one); per
// sub-chunk I and channel c ([4][128] each): tot = total log alpha of the sub-chunk,
// e^{-g_m}, e^{g_m - tot} (g_m = g^L at its 8th token) and e^{tot}; a flag
constexpr uint32_t P_VEC = 212992;
constexpr uint32_t V_TOT = 128, V_EM = V_TOT + 512, V_EC = V_EM + 512, V_P = V_EC + 512, V_FLAG = V_P + 512;
constexpr uint32_t V_SLOW = V_FLAG + 1;  // some sub-chunk decays by more than e^{-kFastTot}
constexpr uint32_t V_INV = V_FLAG + 4;   // fused prologue: 1 / ||q_t||, 1 / ||k_t|| ([2][64])
constexpr uint32_t P_BAR = P_VEC + (V_INV + 128) * 4;
// ---- consumer shared memory
constexpr uint32_t C_SLOT = 0;         // 2 slots
constexpr uint32_t C_S16 = 2 * kSlotStride;        // S fp16, MN-major SW128: 2 blocks x 16 KB
constexpr uint32_t C_U16 = C_S16 + 32768;          // U fp16, MN-major SW128: 2 blocks x 8 KB
constexpr uint32_t C_BAR = C_U16 + 16384;
// layer epilogue (RMSNorm + output gate): per-row partial sums of squares [128][2] and the
// norm weight [128], after the barriers
constexpr uint32_t C_RED = C_BAR + 256;
constexpr uint32_t C_NW = C_RED + 1024;
constexpr uint32_t kSmemBytes =
    (P_BAR > C_BAR ? P_BAR : C_BAR) + 192 + 1024;  // + barriers + alignment slack
static_assert(P_PX + 2 * 6 * 2048 <= P_KSIG, "producer layout");
static_assert(C_NW + 512 <= (P_BAR > C_BAR ? P_BAR : C_BAR) + 192, "consumer layout");
static_assert(P_KBS + 16384 <= P_STAGE, "producer layout");
static_assert(P_KHT + 4 * kKHTBlk <= P_KBS, "producer layout");

// TMEM columns.
constexpr uint32_t PCOL_AP = 0;        // producer, one-anchor path: [A;P] (64 cols)
constexpr uint32_t PCOL_WU = 128;      // producer: [P;T][Ks|V], lanes 64-127 = [W | U'] (256)
constexpr uint32_t CCOL_X = 0;         // consumer: 2 x 128 cols ([Qs;W]S (+ [P;T]U))
constexpr uint32_t CCOL_S = 256;       // consumer: Kb^T U (128 cols)
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t IDESC_AP = tc::idesc(tc::kFmtTF32, 128, 64, 0, 0);
constexpr uint32_t IDESC_WU = tc::idesc(tc::kFmtF16, 128, 256, 0, 1);
constexpr uint32_t IDESC_X = tc::idesc(tc::kFmtF16, 128, 128, 0, 1);   // A K-major, B MN-major
constexpr uint32_t IDESC_S = tc::idesc(tc::kFmtF16, 128, 128, 1, 1);   // A MN-major, B MN-major

// Give-up protocol. Every wait on a peer or on an asynchronous operation is bounded
// (`limit` polls). A thread whose wait runs out records KDA_ERR_DEVICE_TIMEOUT in the
// device error word and sets the abort flag of every CTA of the cluster; any wait that
// sees the flag stops waiting. From then on no thread issues a new TMA load, MMA, bulk
// copy or remote arrive; each CTA leaves its chunk loop at the next uniform check,
// waits (bounded again) for the asynchronous operations it has issued and not yet
// seen complete -- those complete by themselves -- and then reaches the final cluster
// barrier and frees its tensor memory. At most one operation per barrier is ever in
// flight, so "pending" is a flag and the parity to drain is the next expected one.
struct Ctl {
    int *abort;              // this CTA's abort flag (shared memory)
    int *err;                // device error word
    uint32_t peer_abort[4];  // the abort flag of every CTA of the cluster (shared::cluster)
    uint32_t limit;          // polls of a bounded wait
};

__device__ __forceinline__ bool aborted(const Ctl &k) { return *reinterpret_cast<volatile int *>(k.abort) != 0; }
__device__ __forceinline__ void fail(const Ctl &k) {
    atomicExch(k.err, 2);
#pragma unroll
    for (int r = 0; r < 4; ++r)
        asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(k.peer_abort[r]), "r"(1) : "memory");
}
// Waits for the phase `parity` of `bar`; false if the cluster gave up (now or earlier).
__device__ __forceinline__ bool wait_local(uint64_t *bar, uint32_t parity, const Ctl &k) {
    for (uint32_t i = 0; i < k.limit; ++i) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 0 && aborted(k)) return false;
    }
    fail(k);
    return false;
}
// The same with acquire at cluster scope (barriers that peers arrive on).
__device__ __forceinline__ bool wait_cluster(uint64_t *bar, uint32_t parity, const Ctl &k) {
    for (uint32_t i = 0; i < k.limit; ++i) {
        if (tc::mbar_try_wait_cluster(bar, parity)) return true;
        if ((i & 63) == 0 && aborted(k)) return false;
    }
    fail(k);
    return false;
}
// Drain: waits (bounded, regardless of the abort flag) for an operation this thread
// issued; they complete by themselves.
__device__ __forceinline__ void drain(uint64_t *bar, uint32_t parity, const Ctl &k) {
    if (!tc::mbar_wait(bar, parity, kWaitLimit)) atomicExch(k.err, 2);
}

// 4-byte asynchronous copy global -> shared (completion by cp.async.wait_group).
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(tc::smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// log alpha = -softplus(x) = -(max(x, 0) + log(1 + e^{-|x|})) for the gate's pre-activation x
// (Kimi Linear summary, section "Configuracion del modelo Kimi Linear": a data-dependent
// per-channel decay gate like GDN's and Mamba's). For e^{-|x|} < 1e-3 the logarithm is
// its series e - e^2/2, exact to e^3/3, where 1 + e would lose e's digits in fp32.
__device__ __forceinline__ float neg_softplus(float x) {
    constexpr float kLn2 = 0.6931471805599453f;
    const float e = tc::ex2(-fabsf(x) * kLog2e);
    const float l = e < 1e-3f ? e * (1.f - 0.5f * e) : tc::lg2(1.f + e) * kLn2;
    return -(fmaxf(x, 0.f) + l);
}

// tanh by the hardware approximation (relative error about 2^-11, below the bf16
// rounding of the outputs it scales).
__device__ __forceinline__ float tanh_fast(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Inclusive prefix sum over the 8 lanes 4g + t (g = 0..7) that share t.
__device__ __forceinline__ float scan8(float x, int g) {
    float y = __shfl_up_sync(0xffffffffu, x, 4);
    if (g >= 1) x += y;
    y = __shfl_up_sync(0xffffffffu, x, 8);
    if (g >= 2) x += y;
    y = __shfl_up_sync(0xffffffffu, x, 16);
    if (g >= 4) x += y;
    return x;
}

// Claims a free ring of the workspace's pool (bit r of the in-use bitmap), waiting
// (bounded) while all are taken; -1 if the wait runs out. The returned ring is this
// cluster's until release_ring: the acquire below orders the cluster's use of it after
// the previous holder's release.
__device__ int claim_ring(uint32_t *pool, int nrings, uint32_t limit) {
    const int words = (nrings + 31) >> 5;
    for (uint32_t it = 0; it < limit; ++it) {
        for (int w = 0; w < words; ++w) {
            const uint32_t valid = 32 * (w + 1) <= nrings ? 0xffffffffu : (1u << (nrings - 32 * w)) - 1u;
            uint32_t free_bits = ~*reinterpret_cast<volatile uint32_t *>(pool + w) & valid;
            while (free_bits) {
                const int b = __ffs(free_bits) - 1;
                const uint32_t old = atomicOr(pool + w, 1u << b);
                if (!(old & (1u << b))) {
                    __threadfence();
                    tc::fence_proxy_async_global();
                    return 32 * w + b;
                }
                free_bits &= ~old & ~(1u << b);
            }
        }
        __nanosleep(256);
    }
    return -1;
}
// Releases ring r after every access of the cluster to it (the final cluster barrier).
__device__ void release_ring(uint32_t *pool, int r) {
    __threadfence();
    atomicAnd(pool + (r >> 5), ~(1u << (r & 31)));
}

// Index of the off-diagonal block (I, J), J < I, among the six: (1,0) (2,0) (2,1) (3,0) (3,1) (3,2).
__device__ __forceinline__ int pair_index(int I, int J) { return I * (I - 1) / 2 + J; }

// Receives the blocks of X = (I + A)^{-1} from the UT solve and writes T = X Diag(beta)
// as fp16 into the K-major, 128-byte-swizzled T operand (rows 64..127 of [P;T]).
struct TWriter {
    uint8_t *t;
    const float *beta;
    __device__ __forceinline__ void one(int i, int j, float x) const {
        *reinterpret_cast<__half *>(t + sw128k_off(i, j, 0)) = __float2half_rn(x * beta[j]);
    }
    __device__ __forceinline__ void pair(int i, int j, float x0, float x1) const {
        *reinterpret_cast<uint32_t *>(t + sw128k_off(i, j, 0)) = pack_f16(x0 * beta[j], x1 * beta[j + 1]);
    }
};

// ============================================================ producer
// Thread mapping of the gate prologue: warp w handles sub-chunk I = w % 4 (16
// tokens) and channel half w / 4 (64 channels); lane (g, t) = (lane / 4, lane % 4)
// holds tokens 16 I + g and 16 I + g + 8 and, for s = 0..7, the channel pair
// 8 s + 2 t, 8 s + 2 t + 1 of its half -- exactly the elements of the tf32
// mma.sync fragments of the diagonal block (k-step s: channel 8 s + 2 t is
// fragment column t, channel 8 s + 2 t + 1 is column t + 4), so the diagonal
// products need no shared-memory round trip.
template <bool kFused>
__device__ void producer(uint8_t *sm, uint32_t tmem, int rank, uint8_t *ring,
                         const CUtensorMap *tm_v, const CUtensorMap *tm_qs, const CUtensorMap *tm_ks,
                         const CUtensorMap *tm_las, const float *__restrict__ beta, int T, int H,
                         int h, long ztok, int nchunks, const Ctl &ctl, int test_timeout) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = 32 * quad + lane;
    // sub-chunk of this warp: warps w and w + 4 share a scheduler, and sub-chunk I writes
    // 3 - I copies of the off-diagonal columns, so a scheduler gets sub-chunks I and 3 - I
    const int I = half == 0 ? quad : 3 - quad, g = lane >> 2, t4 = lane & 3;
    const int ta = 16 * I + g, tb = ta + 8;
    const uint32_t sbase = tc::smem_u32(sm);
    float *vec = reinterpret_cast<float *>(sm + P_VEC);   // beta buffers and per-channel tables
    // beta of chunk cc (token rows of this head) into buffer b, by threads 0..63; tokens past
    // T are identity steps (beta = 0)
    auto load_beta = [&](int cc, int b) {
        if (tid < kC && cc < nchunks) {
            const int t = cc * kC + tid;
            if (t < T) cp_async4(vec + 64 * b + tid, beta + (ztok + t) * H + h);
            else vec[64 * b + tid] = 0.f;
        }
        cp_async_commit();
    };
    float *Af = reinterpret_cast<float *>(sm + P_AF);
    float *Xf = reinterpret_cast<float *>(sm + P_XF);
    uint64_t *bar_mma = reinterpret_cast<uint64_t *>(sm + P_BAR);
    uint64_t *bar_loaded = bar_mma + 1;  // [kRingDepth]: one per ring slot of this producer
    uint64_t *bar_in = bar_mma + 1 + kRingDepth;
    uint8_t *st = sm + P_STAGE;
    uint32_t ph_mma = 0, ph_in = 0;
    bool pend_in = false, pend_mma = false;   // kLoader: a TMA input batch; thread 0: an MMA group in flight
    // bulk stores of the staged parts (thread kStorer); a CTA barrier follows each wait
    auto store_part = [&](uint8_t *dst, const uint8_t *src, uint32_t bytes) {
        if (!aborted(ctl)) tc::bulk_store_global(dst, src, bytes);
    };
    int img = 0;  // index of this producer's next image

    const uint64_t d_pt = tc::smem_desc(sbase + P_STAGE + ST_PT, 16, 1024, tc::kSwizzle128);
    const uint64_t d_ksv = tc::smem_desc(sbase + P_KSV, kTokBlk, 1024, tc::kSwizzle128);
    const uint64_t d_kqt = tc::smem_desc(sbase + P_KQT, 16, 1024, tc::kSwizzle128);
    const uint64_t d_kht = tc::smem_desc(sbase + P_KHT, 16, 1024, tc::kSwizzle128);
    // the consumer's "ready" barriers for this producer's ring slots
    const uint32_t c_ready = tc::map_to_rank(sbase + C_BAR + 40 + 8 * kRingDepth * rank, kCluster - 1);

    // the blocks of P and T above the diagonal are zero in every image; nothing else writes them
    for (int e = tid; e < 128 * 32; e += kThreads) {
        const int i = (e >> 5) & 63, j = 2 * (e & 31);
        if (j >= 16 * ((i >> 4) + 1))
            *reinterpret_cast<uint32_t *>(st + ST_PT + (e >> 11) * 8192 + sw128k_off(i, j, 0)) = 0u;
    }
    if (tid == 0) {
        *reinterpret_cast<volatile int *>(vec + V_FLAG) = 0;
        *reinterpret_cast<volatile int *>(vec + V_SLOW) = 0;
    }
    __syncthreads();

    auto load_inputs = [&](int cc) {   // TMA: the 64-token chunk cc of head h (all channels)
        if (aborted(ctl)) return;
        pend_in = true;
        const int z = static_cast<int>(ztok + static_cast<long>(cc) * kC);
        tc::mbar_arrive_expect_tx(bar_in, kFused ? kInBytesF : kInBytes);
        tc::tma_load_3d(sm + P_IN_Q, tm_qs, bar_in, 0, h, z);
        tc::tma_load_3d(sm + P_IN_Q + kBoxBytes, tm_qs, bar_in, 64, h, z);
        tc::tma_load_3d(sm + P_IN_K, tm_ks, bar_in, 0, h, z);
        tc::tma_load_3d(sm + P_IN_K + kBoxBytes, tm_ks, bar_in, 64, h, z);
        if (kFused) {   // tm_las maps the gate's pre-activation x (bf16, 64-channel boxes)
            tc::tma_load_3d(sm + P_IN_X, tm_las, bar_in, 0, h, z);
            tc::tma_load_3d(sm + P_IN_X + kBoxBytes, tm_las, bar_in, 64, h, z);
            tc::tma_load_3d(sm + P_IN_VF, tm_v, bar_in, 0, h, z);
        } else {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                tc::tma_load_3d(sm + P_IN_LA + b * kBoxBytes, tm_las, bar_in, 32 * b, h, z);
            tc::tma_load_3d(sm + P_IN_V, tm_v, bar_in, 0, h, z);
        }
    };
    // Publication of an image: thread kStorer waits until its bulk stores of the image are
    // complete, then arrives (release, cluster scope; the generic stores of all threads into
    // the slot precede it through CTA barriers) on the consumer's "ready" barrier of the
    // image's ring slot.
    // (A test hook withholds producer 0's first "ready", so that the consumer's wait runs out.)
    int pending = -1, pending_img = 0;
    auto publish = [&]() {
        if (tid == kStorer && pending >= 0) {
            tc::bulk_wait_all();
            tc::fence_proxy_async_global();
            const bool withheld = test_timeout && rank == 0 && pending_img == 0;
            if (!aborted(ctl) && !withheld) tc::mbar_arrive_remote(c_ready + 8 * pending);
        }
        pending = -1;
    };
    if (tid == kLoader && rank < nchunks) load_inputs(rank);
    load_beta(rank, 0);
    for (int c = rank; c < nchunks; c += kProducers) {
        if (__syncthreads_or(aborted(ctl))) break;   // uniform: the cluster gave up
        const float *beta_s = vec + 64 * (img & 1);
        const int t0 = c * kC;
        const int valid = min(kC, T - t0);
        if (wait_local(bar_in, ph_in, ctl)) {
            ph_in ^= 1;
            pend_in = false;
        }

        load_beta(c + kProducers, (img + 1) & 1);   // the next image's beta, one image ahead
        {   // V -> fp16 columns 128..255 of the [Ks | V] operand (read by [W | U'] only); 16-byte
            // piece e = tid + 256 m of the [64][128] bf16 tile, so a warp reads 512 contiguous bytes
            const uint4 *src = reinterpret_cast<const uint4 *>(sm + (kFused ? P_IN_VF : P_IN_V));
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int e = tid + m * kThreads, t = e >> 4;
                const uint4 vin = t < valid ? src[e] : make_uint4(0, 0, 0, 0);
                uint4 w;
                w.x = pack_f16(tc::bf16_lo(vin.x), tc::bf16_hi(vin.x));
                w.y = pack_f16(tc::bf16_lo(vin.y), tc::bf16_hi(vin.y));
                w.z = pack_f16(tc::bf16_lo(vin.z), tc::bf16_hi(vin.z));
                w.w = pack_f16(tc::bf16_lo(vin.w), tc::bf16_hi(vin.w));
                *reinterpret_cast<uint4 *>(sm + P_KSV + 2 * kTokBlk + sw128k_off(t, (e & 15) * 8, kTokBlk)) = w;
            }
        }

        // ------------------------------------------------ phase 1a: in-sub-chunk prefix sums
        // Thread (p, I) = (tid % 64, tid / 64) runs channels 2p, 2p + 1 of sub-chunk I token by
        // token: g^L into ST_GL (the swizzled layout of log alpha), and the per-channel table.
        if (kFused) {   // 1 / ||q_t|| and 1 / ||k_t|| over the 128 channels (a zero row stays zero)
            const int t = tid >> 2, which = (tid >> 1) & 1, hf = tid & 1;
            const uint8_t *rowp = sm + (which ? P_IN_K : P_IN_Q) + hf * kBoxBytes + t * 128;
            float ss = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 x = *reinterpret_cast<const uint4 *>(rowp + (((c ^ (t & 7)) & 7) << 4));
                const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float lo = tc::bf16_lo(w[m]), hi = tc::bf16_hi(w[m]);
                    ss = fmaf(lo, lo, fmaf(hi, hi, ss));
                }
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            if (hf == 0) vec[V_INV + which * 64 + t] = ss > 0.f ? rsqrtf(ss) : 0.f;
        }
        {
            const int p = tid & 63, Ib = tid >> 6, cp = 2 * p;
            const uint32_t off = (cp >> 5) * kBoxBytes + (cp & 3) * 4;
            const uint32_t ch = (cp & 31) >> 2;
            float s0 = 0.f, s1 = 0.f, m0 = 0.f, m1 = 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int t = 16 * Ib + u;
                const uint32_t o = off + t * 128u + (((ch ^ (t & 7)) & 7u) << 4);
                float2 x = make_float2(0.f, 0.f);
                if (t < valid) {
                    if (kFused) {   // log alpha = -softplus(x), x from its bf16 box
                        const uint32_t xo = (cp >> 6) * kBoxBytes + t * 128u +
                                            (((((cp & 63) >> 3) ^ (t & 7)) & 7u) << 4) + (cp & 7) * 2;
                        const uint32_t xv = *reinterpret_cast<const uint32_t *>(sm + P_IN_X + xo);
                        x = make_float2(neg_softplus(tc::bf16_lo(xv)), neg_softplus(tc::bf16_hi(xv)));
                    } else {
                        x = *reinterpret_cast<const float2 *>(sm + P_IN_LA + o);
                    }
                }
                s0 += x.x;
                s1 += x.y;
                *reinterpret_cast<float2 *>(st + ST_GL + o) = make_float2(s0, s1);
                if (u == 7) { m0 = s0; m1 = s1; }
            }
            const int e = Ib * 128 + cp;
            *reinterpret_cast<float2 *>(vec + V_TOT + e) = make_float2(s0, s1);
            *reinterpret_cast<float2 *>(vec + V_EM + e) =
                make_float2(tc::ex2(-m0 * kLog2e), tc::ex2(-m1 * kLog2e));
            *reinterpret_cast<float2 *>(vec + V_EC + e) =
                make_float2(tc::ex2((m0 - s0) * kLog2e), tc::ex2((m1 - s1) * kLog2e));
            *reinterpret_cast<float2 *>(vec + V_P + e) =
                make_float2(tc::ex2(s0 * kLog2e), tc::ex2(s1 * kLog2e));
            if (s0 < kRangeLog || s1 < kRangeLog) *reinterpret_cast<volatile int *>(vec + V_FLAG) = 1;
            if (s0 < -kFastTot || s1 < -kFastTot) *reinterpret_cast<volatile int *>(vec + V_SLOW) = 1;
        }
        if (tid == kStorer) tc::bulk_wait_read_all();   // the previous W and U' have left P_KSIG
        __syncthreads();
        const int rb = img % kRingDepth;  // ring slot of this image; image img-kRingDepth used it before
        uint8_t *gs = ring + (kRingDepth * rank + rb) * kSlotStride;
        if (*reinterpret_cast<volatile int *>(vec + V_SLOW) == 0) {   // uniform: read after a CTA barrier
            // -------------------------------------------- one-anchor path: every sub-chunk decays by
            // at most e^{-kFastTot}, so the chunk by at most e^{-160}, and the factors e^{g - g_C/2},
            // e^{g_C/2 - g} stay within e^{80}: [A;P] = [K~ ; Q~] K^T is one tf32 tcgen05 MMA over
            // all 128 channels (K~ = K e^{g - g_C/2}, Q~ likewise, K^ = K e^{g_C/2 - g}).
            // Thread (p, I) = (tid % 64, tid / 64) owns channels 2p, 2p + 1 of sub-chunk I.
            const int p = tid & 63, Ib = tid >> 6, cp = 2 * p;
            uint32_t qv[16], kv[16];
            float2 gl[16];
            {
                const uint32_t off = (cp >> 5) * kBoxBytes + (cp & 3) * 4, ch = (cp & 31) >> 2;
                const uint32_t qk = (cp >> 6) * kBoxBytes + (cp & 7) * 2, ch16 = (cp & 63) >> 3;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int t = 16 * Ib + u;
                    const bool ok = t < valid;
                    gl[u] = *reinterpret_cast<const float2 *>(st + ST_GL + off + t * 128u + (((ch ^ (t & 7)) & 7u) << 4));
                    const uint32_t o = qk + t * 128u + (((ch16 ^ (t & 7)) & 7u) << 4);
                    qv[u] = ok ? *reinterpret_cast<const uint32_t *>(sm + P_IN_Q + o) : 0u;
                    kv[u] = ok ? *reinterpret_cast<const uint32_t *>(sm + P_IN_K + o) : 0u;
                }
            }
            float G0 = 0.f, G1 = 0.f, C0 = 0.f, C1 = 0.f;   // g before sub-chunk Ib; g_C
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                const float2 tj = *reinterpret_cast<const float2 *>(vec + V_TOT + J * 128 + cp);
                if (J < Ib) { G0 += tj.x; G1 += tj.y; }
                C0 += tj.x;
                C1 += tj.y;
            }
            __syncthreads();   // all inputs are in registers: the operand tiles may overwrite them
            if (tid == 0) {   // for the next image
                *reinterpret_cast<volatile int *>(vec + V_FLAG) = 0;
                *reinterpret_cast<volatile int *>(vec + V_SLOW) = 0;
            }
            const float ga0 = 0.5f * C0, ga1 = 0.5f * C1;
            const float ea0 = tc::ex2(ga0 * kLog2e), ea1 = tc::ex2(ga1 * kLog2e);   // e^{g_C/2}
            // tf32 tiles: 32-channel K-blocks; fp16 tiles: 64-channel K-blocks; 128-byte rows, swizzled
            const uint32_t rowq = Ib * 2048u;
            const uint32_t b32 = (cp & 3u) * 4u + rowq, ch32 = (cp & 31u) >> 2, kb32 = cp >> 5;
            const uint32_t b16 = (cp & 7u) * 2u + rowq, ch16 = (cp & 63u) >> 3, kb16 = cp >> 6;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int t = 16 * Ib + u;
                const uint32_t r = (u >> 3) * 1024u + (u & 7) * 128u;
                const uint32_t o32 = b32 + r + (((ch32 ^ (u & 7)) & 7u) << 4);
                const uint32_t o16 = b16 + r + (((ch16 ^ (u & 7)) & 7u) << 4);
                const float d0 = (G0 + gl[u].x - ga0) * kLog2e, d1 = (G1 + gl[u].y - ga1) * kLog2e;
                const float nq = kFused ? vec[V_INV + t] : 1.f, nk = kFused ? vec[V_INV + 64 + t] : 1.f;
                const float q0 = tc::bf16_lo(qv[u]) * nq, q1 = tc::bf16_hi(qv[u]) * nq;
                const float k0 = tc::bf16_lo(kv[u]) * nk, k1 = tc::bf16_hi(kv[u]) * nk;
                const float E0 = tc::ex2(d0), E1 = tc::ex2(d1), F0 = tc::ex2(-d0), F1 = tc::ex2(-d1);
                const float ke0 = k0 * E0, ke1 = k1 * E1, qe0 = q0 * E0, qe1 = q1 * E1;
                const float kf0 = k0 * F0, kf1 = k1 * F1;
                *reinterpret_cast<float2 *>(sm + P_KQT + kb32 * kKQTBlk + o32) = make_float2(ke0, ke1);
                *reinterpret_cast<float2 *>(sm + P_KQT + kb32 * kKQTBlk + 8192 + o32) = make_float2(qe0, qe1);
                *reinterpret_cast<float2 *>(sm + P_KHT + kb32 * kKHTBlk + o32) = make_float2(kf0, kf1);
                // Qs = Q e^{g}, Ks = K e^{g}, Kb = K e^{g_C - g}
                *reinterpret_cast<uint32_t *>(st + ST_QS + kb16 * 8192 + o16) = pack_f16(qe0 * ea0, qe1 * ea1);
                *reinterpret_cast<uint32_t *>(sm + P_KSV + kb16 * kTokBlk + o16) = pack_f16(ke0 * ea0, ke1 * ea1);
                *reinterpret_cast<uint32_t *>(sm + P_KBS + kb16 * 8192 + o16) = pack_f16(kf0 * ea0, kf1 * ea1);
            }
            fence_proxy_async_smem();
            publish();   // the previous image (its stores have had phase 1a to land)
            if (tid == 0 && img >= kRingDepth) wait_cluster(bar_loaded + rb, ((img / kRingDepth) - 1) & 1, ctl);
            cp_async_wait_prev();   // this image's beta (all but the group just issued)
            __syncthreads();
            if (tid == 0 && !aborted(ctl)) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 16; ++kk)
                    tc::mma_tf32(tmem + PCOL_AP, d_kqt + (((kk >> 2) * kKQTBlk + (kk & 3) * 32) >> 4),
                                 d_kht + (((kk >> 2) * kKHTBlk + (kk & 3) * 32) >> 4), IDESC_AP, kk > 0);
                tc::mma_commit(bar_mma);
                pend_mma = true;
            }
            if (tid == kStorer) {
                store_part(gs + SL_QW, st + ST_QS, 8192);                 // Qs, K-block 0
                store_part(gs + SL_QW + kQWBlk, st + ST_QS + 8192, 8192); // Qs, K-block 1
                store_part(gs + SL_KB, sm + P_KBS, 16384);                // Kb
                tc::bulk_commit();
            }
            if (Ib == 0)
                *reinterpret_cast<float2 *>(gs + SL_GAM + 4 * cp) =
                    make_float2(tc::ex2(C0 * kLog2e), tc::ex2(C1 * kLog2e));   // e^{g_C}
            if (wait_local(bar_mma, ph_mma, ctl)) {
                ph_mma ^= 1;
                pend_mma = false;
            }
            tc_fence_after();
            {   // A = Diag(beta) strict_lower(K~ K^T) (fp32), P = lower(Q~ K^T) (fp16, into [P;T])
                float vv[32];
                tc::tmem_ld32(tc::tmem_addr(tmem, 32 * quad, PCOL_AP + half * 32), vv);
                tc::tmem_wait_ld();
                if (quad < 2) {
                    const int i = row;
                    const float bi = beta_s[i];
#pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        const int j = half * 32 + u;
                        Af[i * kLD + j] = j < i ? bi * vv[u] : 0.f;
                    }
                } else {
                    const int i = row - 64;
#pragma unroll
                    for (int u = 0; u < 32; u += 2) {
                        const int j = half * 32 + u;
                        const float lo = j <= i ? vv[u] : 0.f, hi = j + 1 <= i ? vv[u + 1] : 0.f;
                        *reinterpret_cast<uint32_t *>(st + ST_PT + sw128k_off(i, j, 0)) = pack_f16(lo, hi);
                    }
                }
            }
            tc_fence_before();
        } else {
            // -------------------------------------------- sub-chunk path (any decay)
            const bool far_decay = *reinterpret_cast<volatile int *>(vec + V_FLAG) != 0;

            // ------------------------------------------------ phase 1b: diagonal blocks (tf32
            // mma.sync, fragments straight from registers), rows of the off-diagonal blocks
            const bool va = ta < valid, vb = tb < valid;
            // the fused prologue's L2 normalisation, applied where q and k are unpacked
            const float nqa = kFused ? vec[V_INV + ta] : 1.f, nqb = kFused ? vec[V_INV + tb] : 1.f;
            const float nka = kFused ? vec[V_INV + 64 + ta] : 1.f, nkb = kFused ? vec[V_INV + 64 + tb] : 1.f;
            uint32_t qA[8], qB[8], kA[8], kB[8];
            float rA[8][2], rB[8][2], sA[8][2], sB[8][2];   // e^{g^L}, e^{tot - g^L} of tokens a, b
            float accA[2][4] = {}, accP[2][4] = {};
            const uint32_t rowa = static_cast<uint32_t>(ta) * 128u, rowb = static_cast<uint32_t>(tb) * 128u;
    #pragma unroll
            for (int s = 0; s < 8; ++s) {
                const int c0 = 64 * half + 8 * s + 2 * t4;
                const uint32_t qk_off = half * kBoxBytes + ((s ^ g) << 4) + 4 * t4;
                const uint32_t la_off = (c0 >> 5) * kBoxBytes + (((((c0 & 31) >> 2) ^ g) & 7) << 4) + 8 * (t4 & 1);
                qA[s] = va ? *reinterpret_cast<const uint32_t *>(sm + P_IN_Q + rowa + qk_off) : 0u;
                qB[s] = vb ? *reinterpret_cast<const uint32_t *>(sm + P_IN_Q + rowb + qk_off) : 0u;
                kA[s] = va ? *reinterpret_cast<const uint32_t *>(sm + P_IN_K + rowa + qk_off) : 0u;
                kB[s] = vb ? *reinterpret_cast<const uint32_t *>(sm + P_IN_K + rowb + qk_off) : 0u;
                const float2 xa = *reinterpret_cast<const float2 *>(st + ST_GL + rowa + la_off);
                const float2 xb = *reinterpret_cast<const float2 *>(st + ST_GL + rowb + la_off);
                const int e = I * 128 + c0;
                const float2 tot = *reinterpret_cast<const float2 *>(vec + V_TOT + e);
                const float2 em = *reinterpret_cast<const float2 *>(vec + V_EM + e);
                const float2 ec = *reinterpret_cast<const float2 *>(vec + V_EC + e);
                // factors anchored at the sub-chunk's start (rho) and end (sigma), both <= 1
                rA[s][0] = tc::ex2(xa.x * kLog2e);
                rA[s][1] = tc::ex2(xa.y * kLog2e);
                rB[s][0] = tc::ex2(xb.x * kLog2e);
                rB[s][1] = tc::ex2(xb.y * kLog2e);
                sA[s][0] = tc::ex2((tot.x - xa.x) * kLog2e);
                sA[s][1] = tc::ex2((tot.y - xa.y) * kLog2e);
                sB[s][0] = tc::ex2((tot.x - xb.x) * kLog2e);
                sB[s][1] = tc::ex2((tot.y - xb.y) * kLog2e);
                // diagonal-block factors around token 7: rows e^{g_i - g_m} = rho_i e^{-g_m},
                // columns e^{g_m - g_j} = sigma_j e^{g_m - tot}
                float ra0 = rA[s][0] * em.x, ra1 = rA[s][1] * em.y, rb0 = rB[s][0] * em.x, rb1 = rB[s][1] * em.y;
                float ca0 = sA[s][0] * ec.x, ca1 = sA[s][1] * ec.y, cb0 = sB[s][0] * ec.x, cb1 = sB[s][1] * ec.y;
                if (far_decay) {
                    // some channel of the chunk decays by more than e^-87 inside one sub-chunk: such a
                    // channel takes its diagonal factors from log alpha clamped at -10 per token
                    const bool f0 = tot.x >= kRangeLog, f1 = tot.y >= kRangeLog;
                    float2 la = make_float2(0.f, 0.f), lb = make_float2(0.f, 0.f);
                    if (kFused) {
                        const uint32_t xa2 = va ? *reinterpret_cast<const uint32_t *>(sm + P_IN_X + rowa + qk_off) : 0u;
                        const uint32_t xb2 = vb ? *reinterpret_cast<const uint32_t *>(sm + P_IN_X + rowb + qk_off) : 0u;
                        if (va) la = make_float2(neg_softplus(tc::bf16_lo(xa2)), neg_softplus(tc::bf16_hi(xa2)));
                        if (vb) lb = make_float2(neg_softplus(tc::bf16_lo(xb2)), neg_softplus(tc::bf16_hi(xb2)));
                    } else {
                        if (va) la = *reinterpret_cast<const float2 *>(sm + P_IN_LA + rowa + la_off);
                        if (vb) lb = *reinterpret_cast<const float2 *>(sm + P_IN_LA + rowb + la_off);
                    }
                    float ya0 = scan8(fmaxf(la.x, kClampLog), g), ya1 = scan8(fmaxf(la.y, kClampLog), g);
                    float yb0 = scan8(fmaxf(lb.x, kClampLog), g), yb1 = scan8(fmaxf(lb.y, kClampLog), g);
                    const float ym0 = __shfl_sync(0xffffffffu, ya0, 28 + t4);   // at token 7
                    const float ym1 = __shfl_sync(0xffffffffu, ya1, 28 + t4);
                    yb0 += ym0;
                    yb1 += ym1;
                    if (!f0) {
                        ra0 = tc::ex2((ya0 - ym0) * kLog2e);
                        rb0 = tc::ex2((yb0 - ym0) * kLog2e);
                        ca0 = tc::ex2((ym0 - ya0) * kLog2e);
                        cb0 = tc::ex2((ym0 - yb0) * kLog2e);
                    }
                    if (!f1) {
                        ra1 = tc::ex2((ya1 - ym1) * kLog2e);
                        rb1 = tc::ex2((yb1 - ym1) * kLog2e);
                        ca1 = tc::ex2((ym1 - ya1) * kLog2e);
                        cb1 = tc::ex2((ym1 - yb1) * kLog2e);
                    }
                }
                const float qa0 = tc::bf16_lo(qA[s]) * nqa, qa1 = tc::bf16_hi(qA[s]) * nqa;
                const float qb0 = tc::bf16_lo(qB[s]) * nqb, qb1 = tc::bf16_hi(qB[s]) * nqb;
                const float ka0 = tc::bf16_lo(kA[s]) * nka, ka1 = tc::bf16_hi(kA[s]) * nka;
                const float kb0 = tc::bf16_lo(kB[s]) * nkb, kb1 = tc::bf16_hi(kB[s]) * nkb;
                {   // diagonal block: A^d += K~ K^^T, P^d += Q~ K^^T over this k-step's 8 channels
                    // (fp32 operands; the tensor cores read them as tf32)
                    const uint32_t ak[4] = {__float_as_uint(ka0 * ra0), __float_as_uint(kb0 * rb0),
                                            __float_as_uint(ka1 * ra1), __float_as_uint(kb1 * rb1)};
                    const uint32_t aq[4] = {__float_as_uint(qa0 * ra0), __float_as_uint(qb0 * rb0),
                                            __float_as_uint(qa1 * ra1), __float_as_uint(qb1 * rb1)};
                    const uint32_t b00 = __float_as_uint(ka0 * ca0), b01 = __float_as_uint(ka1 * ca1);  // column token g
                    const uint32_t b10 = __float_as_uint(kb0 * cb0), b11 = __float_as_uint(kb1 * cb1);  // column token g + 8
                    tc::mma_16x8x8_tf32(accA[0], ak, b00, b01);
                    tc::mma_16x8x8_tf32(accA[1], ak, b10, b11);
                    tc::mma_16x8x8_tf32(accP[0], aq, b00, b01);
                    tc::mma_16x8x8_tf32(accP[1], aq, b10, b11);
                }
                // column operand of the off-diagonal blocks: K e^{G_{J+1} - g_j} for this sub-chunk J = I
                *reinterpret_cast<float2 *>(sm + P_KSIG + rowa + la_off) = make_float2(ka0 * sA[s][0], ka1 * sA[s][1]);
                *reinterpret_cast<float2 *>(sm + P_KSIG + rowb + la_off) = make_float2(kb0 * sB[s][0], kb1 * sB[s][1]);
            }

            publish();   // the previous image (its stores have had phases 1a and 1b to land)
            if (tid == 0 && img >= kRingDepth) wait_cluster(bar_loaded + rb, ((img / kRingDepth) - 1) & 1, ctl);
            cp_async_wait_prev();   // this image's beta (all but the group just issued)
            __syncthreads();   // the inputs and g^L are dead; every thread has read the flag
            if (tid == 0) {   // for the next image
                *reinterpret_cast<volatile int *>(vec + V_FLAG) = 0;
                *reinterpret_cast<volatile int *>(vec + V_SLOW) = 0;
            }

            // ------------------------------------------------ phase 2: chunk-level factors
            // (products of the sub-chunks' e^{tot}: e^{G_I}, e^{g_C - G_{I+1}}) and the off-diagonal blocks
            if (half == 1) {   // diagonal partials of channels 64..127 for the half-0 warp of sub-chunk I
                float4 *dx = reinterpret_cast<float4 *>(sm + P_DX) + (I * 32 + lane) * 4;
                dx[0] = make_float4(accA[0][0], accA[0][1], accA[0][2], accA[0][3]);
                dx[1] = make_float4(accA[1][0], accA[1][1], accA[1][2], accA[1][3]);
                dx[2] = make_float4(accP[0][0], accP[0][1], accP[0][2], accP[0][3]);
                dx[3] = make_float4(accP[1][0], accP[1][1], accP[1][2], accP[1][3]);
            }
            const uint32_t row_a = half * 8192u + (ta >> 3) * 1024u + g * 128u + 4u * t4;   // token a, no swizzle term
    #pragma unroll
            for (int s = 0; s < 8; ++s) {
                const int c0 = 64 * half + 8 * s + 2 * t4;
                float2 pj[4];   // e^{tot_J} of the four sub-chunks
    #pragma unroll
                for (int J = 0; J < 4; ++J) pj[J] = *reinterpret_cast<const float2 *>(vec + V_P + J * 128 + c0);
                float eG0 = 1.f, eG1 = 1.f, eK0 = 1.f, eK1 = 1.f;
    #pragma unroll
                for (int J = 0; J < 4; ++J) {
                    if (J < I) { eG0 *= pj[J].x; eG1 *= pj[J].y; }
                    if (J > I) { eK0 *= pj[J].x; eK1 *= pj[J].y; }
                }
                const float qa0 = tc::bf16_lo(qA[s]) * nqa, qa1 = tc::bf16_hi(qA[s]) * nqa;
                const float qb0 = tc::bf16_lo(qB[s]) * nqb, qb1 = tc::bf16_hi(qB[s]) * nqb;
                const float ka0 = tc::bf16_lo(kA[s]) * nka, ka1 = tc::bf16_hi(kA[s]) * nka;
                const float kb0 = tc::bf16_lo(kB[s]) * nkb, kb1 = tc::bf16_hi(kB[s]) * nkb;
                const float fa0 = rA[s][0] * eG0, fa1 = rA[s][1] * eG1, fb0 = rB[s][0] * eG0, fb1 = rB[s][1] * eG1;
                // Qs = Q e^{g} and Kb = K e^{g_C - g} (staged for the ring slot), Ks = K e^{g} into
                // [Ks | V]; all three are [token][channel] tiles of 64-channel K-blocks 8 KB apart in
                // the 128-byte swizzle
                const uint32_t oa = row_a + (((s ^ g) & 7) << 4), ob = oa + 1024;
                *reinterpret_cast<uint32_t *>(st + ST_QS + oa) = pack_f16(qa0 * fa0, qa1 * fa1);
                *reinterpret_cast<uint32_t *>(st + ST_QS + ob) = pack_f16(qb0 * fb0, qb1 * fb1);
                *reinterpret_cast<uint32_t *>(sm + P_KSV + oa) = pack_f16(ka0 * fa0, ka1 * fa1);
                *reinterpret_cast<uint32_t *>(sm + P_KSV + ob) = pack_f16(kb0 * fb0, kb1 * fb1);
                *reinterpret_cast<uint32_t *>(sm + P_KBS + oa) = pack_f16(ka0 * sA[s][0] * eK0, ka1 * sA[s][1] * eK1);
                *reinterpret_cast<uint32_t *>(sm + P_KBS + ob) = pack_f16(kb0 * sB[s][0] * eK0, kb1 * sB[s][1] * eK1);
                if (I == 0 && g == 0)
                    *reinterpret_cast<float2 *>(gs + SL_GAM + 4 * c0) =
                        make_float2(pj[0].x * pj[1].x * pj[2].x * pj[3].x, pj[0].y * pj[1].y * pj[2].y * pj[3].y);
            }
            // Off-diagonal blocks (I, J), J < I, over this warp's 64 channels:
            //   A^o += [K e^{g - G_I} Diag(e^{G_I - G_{J+1}})] (K e^{G_{J+1} - g})^T, P^o likewise with Q;
            // partials of both channel halves go to shared memory, summed by the half-1 warp below.
            for (int J = 0; J < I; ++J) {
                float oA[2][4] = {}, oP[2][4] = {};
    #pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const int c0 = 64 * half + 8 * s + 2 * t4;
                    float D0 = 1.f, D1 = 1.f;   // e^{G_I - G_{J+1}}: the sub-chunks strictly between J and I
    #pragma unroll
                    for (int Jm = 1; Jm < 3; ++Jm)
                        if (Jm > J && Jm < I) {
                            const float2 pm = *reinterpret_cast<const float2 *>(vec + V_P + Jm * 128 + c0);
                            D0 *= pm.x;
                            D1 *= pm.y;
                        }
                    const float ra0 = rA[s][0] * D0, ra1 = rA[s][1] * D1, rb0 = rB[s][0] * D0, rb1 = rB[s][1] * D1;
                    const uint32_t ak[4] = {__float_as_uint(tc::bf16_lo(kA[s]) * nka * ra0), __float_as_uint(tc::bf16_lo(kB[s]) * nkb * rb0),
                                            __float_as_uint(tc::bf16_hi(kA[s]) * nka * ra1), __float_as_uint(tc::bf16_hi(kB[s]) * nkb * rb1)};
                    const uint32_t aq[4] = {__float_as_uint(tc::bf16_lo(qA[s]) * nqa * ra0), __float_as_uint(tc::bf16_lo(qB[s]) * nqb * rb0),
                                            __float_as_uint(tc::bf16_hi(qA[s]) * nqa * ra1), __float_as_uint(tc::bf16_hi(qB[s]) * nqb * rb1)};
                    const uint32_t la_off = (c0 >> 5) * kBoxBytes + (((((c0 & 31) >> 2) ^ g) & 7) << 4) + 8 * (t4 & 1);
                    const uint32_t rj = static_cast<uint32_t>(16 * J + g) * 128u;   // column token g of sub-chunk J
                    const float2 y0 = *reinterpret_cast<const float2 *>(sm + P_KSIG + rj + la_off);
                    const float2 y1 = *reinterpret_cast<const float2 *>(sm + P_KSIG + rj + 1024 + la_off);  // token g + 8
                    tc::mma_16x8x8_tf32(oA[0], ak, __float_as_uint(y0.x), __float_as_uint(y0.y));
                    tc::mma_16x8x8_tf32(oA[1], ak, __float_as_uint(y1.x), __float_as_uint(y1.y));
                    tc::mma_16x8x8_tf32(oP[0], aq, __float_as_uint(y0.x), __float_as_uint(y0.y));
                    tc::mma_16x8x8_tf32(oP[1], aq, __float_as_uint(y1.x), __float_as_uint(y1.y));
                }
                float4 *px = reinterpret_cast<float4 *>(sm + P_PX) + ((half * 6 + pair_index(I, J)) * 32 + lane) * 4;
                px[0] = make_float4(oA[0][0], oA[0][1], oA[0][2], oA[0][3]);
                px[1] = make_float4(oA[1][0], oA[1][1], oA[1][2], oA[1][3]);
                px[2] = make_float4(oP[0][0], oP[0][1], oP[0][2], oP[0][3]);
                px[3] = make_float4(oP[1][0], oP[1][1], oP[1][2], oP[1][3]);
            }
            fence_proxy_async_smem();   // Ks, and the staged Qs and Kb, reach the async proxy
            __syncthreads();
            if (tid == kStorer) {   // warp 7 (sub-chunk 0, channel half 1) has no share of the combine
                store_part(gs + SL_QW, st + ST_QS, 8192);                 // Qs, K-block 0
                store_part(gs + SL_QW + kQWBlk, st + ST_QS + 8192, 8192); // Qs, K-block 1
                store_part(gs + SL_KB, sm + P_KBS, 16384);                // Kb
                tc::bulk_commit();
            }
            const float ba = beta_s[ta], bb = beta_s[tb];
            if (half == 0) {
                // diagonal blocks of A (times beta, strictly lower) and P (lower), both channel halves summed
                const float4 *dx = reinterpret_cast<const float4 *>(sm + P_DX) + (I * 32 + lane) * 4;
                const float4 x0 = dx[0], x1 = dx[1], x2 = dx[2], x3 = dx[3];
                accA[0][0] += x0.x; accA[0][1] += x0.y; accA[0][2] += x0.z; accA[0][3] += x0.w;
                accA[1][0] += x1.x; accA[1][1] += x1.y; accA[1][2] += x1.z; accA[1][3] += x1.w;
                accP[0][0] += x2.x; accP[0][1] += x2.y; accP[0][2] += x2.z; accP[0][3] += x2.w;
                accP[1][0] += x3.x; accP[1][1] += x3.y; accP[1][2] += x3.z; accP[1][3] += x3.w;
    #pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int jl = 8 * nt + 2 * t4, j = 16 * I + jl;
                    *reinterpret_cast<float2 *>(Af + ta * kLD + j) =
                        make_float2(jl < g ? ba * accA[nt][0] : 0.f, jl + 1 < g ? ba * accA[nt][1] : 0.f);
                    *reinterpret_cast<float2 *>(Af + tb * kLD + j) =
                        make_float2(jl < g + 8 ? bb * accA[nt][2] : 0.f, jl + 1 < g + 8 ? bb * accA[nt][3] : 0.f);
                    *reinterpret_cast<uint32_t *>(st + ST_PT + sw128k_off(ta, j, 0)) =
                        pack_f16(jl <= g ? accP[nt][0] : 0.f, jl + 1 <= g ? accP[nt][1] : 0.f);
                    *reinterpret_cast<uint32_t *>(st + ST_PT + sw128k_off(tb, j, 0)) =
                        pack_f16(jl <= g + 8 ? accP[nt][2] : 0.f, jl + 1 <= g + 8 ? accP[nt][3] : 0.f);
                }
            } else {
                // off-diagonal blocks (I, J) of A and P, both channel halves summed
                for (int J = 0; J < I; ++J) {
                    const float4 *p0 = reinterpret_cast<const float4 *>(sm + P_PX) + (pair_index(I, J) * 32 + lane) * 4;
                    const float4 *p1 = p0 + 6 * 32 * 4;
    #pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const float4 a0 = p0[nt], a1 = p1[nt], q0 = p0[2 + nt], q1 = p1[2 + nt];
                        const int j = 16 * J + 8 * nt + 2 * t4;
                        *reinterpret_cast<float2 *>(Af + ta * kLD + j) = make_float2(ba * (a0.x + a1.x), ba * (a0.y + a1.y));
                        *reinterpret_cast<float2 *>(Af + tb * kLD + j) = make_float2(bb * (a0.z + a1.z), bb * (a0.w + a1.w));
                        *reinterpret_cast<uint32_t *>(st + ST_PT + sw128k_off(ta, j, 0)) = pack_f16(q0.x + q1.x, q0.y + q1.y);
                        *reinterpret_cast<uint32_t *>(st + ST_PT + sw128k_off(tb, j, 0)) = pack_f16(q0.z + q1.z, q0.w + q1.w);
                    }
                }
            }
        }
        __syncthreads();

        // ------------------------------------------------ UT solve; T = X Diag(beta) (fp16)
        // written block by block as the solve finishes it
        ut::unit_lower_inverse(Af, Xf, tid, TWriter{st + ST_PT + 8192, beta_s});
        fence_proxy_async_smem();
        __syncthreads();

        // ------------------------------------------------ [W | U'] = T [Ks | V] (fp16, N = 256)
        if (tid == 0 && !aborted(ctl)) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + PCOL_WU, d_pt + ((kk * 32) >> 4), d_ksv + ((kk * 2048) >> 4), IDESC_WU, kk > 0);
            tc::mma_commit(bar_mma);
            pend_mma = true;
        }
        // the input region (A, X) is dead until the next chunk: stage its inputs there
        if (tid == kLoader && c + kProducers < nchunks) load_inputs(c + kProducers);
        if (tid == kStorer) {
            store_part(gs + SL_PT, st + ST_PT, 16384);   // [P;T], while the MMA runs
            tc::bulk_commit();
        }
        if (wait_local(bar_mma, ph_mma, ctl)) {
            ph_mma ^= 1;
            pend_mma = false;
        }
        tc_fence_after();
        if (quad >= 2) {   // W (rows 64..127 of [Qs ; W]) and U', staged in their image layout
            const int i = row - 64;
#pragma unroll
            for (int part = 0; part < 2; ++part) {   // part 0: W, part 1: U'
                float w[64];
                const uint32_t taddr = tc::tmem_addr(tmem, 32 * quad, PCOL_WU + part * 128 + half * 64);
                tc::tmem_ld32(taddr, *reinterpret_cast<float(*)[32]>(&w[0]));
                tc::tmem_ld32(taddr + 32, *reinterpret_cast<float(*)[32]>(&w[32]));
                tc::tmem_wait_ld();
                uint8_t *dst = sm + (part == 0 ? P_WS : P_US) + half * 8192;
#pragma unroll
                for (int u = 0; u < 64; u += 8) {
                    uint4 x;
                    x.x = pack_f16(w[u], w[u + 1]);
                    x.y = pack_f16(w[u + 2], w[u + 3]);
                    x.z = pack_f16(w[u + 4], w[u + 5]);
                    x.w = pack_f16(w[u + 6], w[u + 7]);
                    *reinterpret_cast<uint4 *>(dst + sw128k_off(i, u, 0)) = x;
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (tid == kStorer) tc::bulk_wait_read_all();   // the staged Qs has left ST_QS (= g^L)
        __syncthreads();
        if (tid == kStorer) {
            store_part(gs + SL_QW + 8192, sm + P_WS, 8192);                // W, K-block 0
            store_part(gs + SL_QW + kQWBlk + 8192, sm + P_WS + 8192, 8192);
            store_part(gs + SL_UP, sm + P_US, 16384);                      // U'
            tc::bulk_commit();
        }
        // Every thread's generic stores into the slot precede the storer's release through the
        // CTA barriers (the release is cumulative). The "ready" of this image is sent once its
        // bulk stores are complete: after the next image's phase 1b, or after the loop.
        pending = rb;
        pending_img = img;
        ++img;
    }
    publish();
    // drain: what this CTA issued and has not seen complete (all of it after a give-up)
    if (tid == kLoader && pend_in) drain(bar_in, ph_in, ctl);
    if (tid == 0 && pend_mma) drain(bar_mma, ph_mma, ctl);
    if (tid == kStorer) tc::bulk_wait_all();
    asm volatile("cp.async.wait_all;" ::: "memory");
}
// ============================================================ consumer
// S0 and S_T may be the same array (a state cache updated in place): each CTA reads its
// row of S0 before the chunk loop and writes the same row of S_T after it.
// kGated: the layer's epilogue on each output row (Kimi Linear summary, section
// "Configuracion del modelo Kimi Linear": per-head RMSNorm and a data-dependent output
// gate before the output projection), out = o / sqrt(mean(o^2) + eps) * norm_w *
// sigmoid(z), z the gate's pre-activation (bf16, the layout of out).
template <bool kGated>
__device__ void consumer(uint8_t *sm, uint32_t tmem, const uint8_t *ring, const float *S0,
                         __nv_bfloat16 *__restrict__ out, float *S_T, int T, int H,
                         int h, long srow, long ztok, int nchunks, const Ctl &ctl,
                         const __nv_bfloat16 *__restrict__ out_gate, const float *__restrict__ norm_w,
                         float eps, const CUtensorMap *tm_z) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = 32 * quad + lane;   // TMEM lane; state row (key channel)
    const uint32_t sbase = tc::smem_u32(sm);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + C_BAR);  // [2]
    uint64_t *bar_x = full + 2;
    uint64_t *bar_s = full + 3;
    uint64_t *bar_o = full + 4;
    uint64_t *ready = full + 5;  // [kRingSlots]: producer p, ring slot b at ready[kRingDepth p + b]
    uint32_t ph_full = 0;   // bit s: parity of slot s's next fill
    uint32_t ph_x = 0, ph_s = 0, ph_o = 0;
    uint32_t pend_full = 0;   // thread 0: bit s = a pull into slot s is in flight
    bool pend_x = false, pend_s = false, pend_o = false;   // thread 0: an MMA group in flight

    const uint64_t d_s16 = tc::smem_desc(sbase + C_S16, 16384, 1024, tc::kSwizzle128);
    const uint64_t d_u16 = tc::smem_desc(sbase + C_U16, kTokBlk, 1024, tc::kSwizzle128);
    // Operand descriptors of slot 0; slot 1 is kSlotStride bytes further. They are
    // selected arithmetically so that they stay in registers (an array indexed by the
    // slot would live in local memory and be reloaded before every MMA).
    const uint64_t d_qw0 = tc::smem_desc(sbase + C_SLOT + SL_QW, 16, 1024, tc::kSwizzle128);
    const uint64_t d_kb0 = tc::smem_desc(sbase + C_SLOT + SL_KB, kTokBlk, 1024, tc::kSwizzle128);
    const uint64_t d_pt0 = tc::smem_desc(sbase + C_SLOT + SL_PT, 16, 1024, tc::kSwizzle128);
    constexpr uint64_t kSlotDesc = kSlotStride >> 4;   // slot stride in descriptor units
    const uint32_t p_loaded = sbase + P_BAR + 8;  // producers' "loaded" barrier (same offset)

    // Thread 0 pulls published images: chunks next_load .. limit (their slots are free).
    int next_load = 0;
    auto pull = [&](int limit, bool block) {
        while (next_load <= limit && next_load < nchunks) {
            const int pc = next_load % kProducers, j = next_load / kProducers;
            const int rs = kRingDepth * pc + j % kRingDepth;  // ring slot (and its ready barrier)
            const uint32_t par = (j / kRingDepth) & 1;
            if (block)
                wait_cluster(ready + rs, par, ctl);
            else if (!tc::mbar_test_cluster(ready + rs, par))
                return;
            if (aborted(ctl)) return;
            tc::fence_proxy_async_global();
            const int sl = next_load & 1;
            pend_full |= 1u << sl;
            tc::mbar_arrive_expect_tx(full + sl, kSlotBytes);
            tc::bulk_load_global(sm + C_SLOT + sl * kSlotStride, ring + rs * kSlotStride, kSlotBytes,
                                 full + sl);
            ++next_load;
        }
    };

    // fp32 state: row `row`, columns half*64 .. +64
    float S[64];
#pragma unroll
    for (int j = 0; j < 64; ++j)
        S[j] = S0 ? S0[(srow * kD + row) * kD + half * 64 + j] : 0.f;
    auto write_s16 = [&]() {
#pragma unroll
        for (int u = 0; u < 64; u += 8) {
            uint4 x;
            x.x = pack_f16(S[u], S[u + 1]);
            x.y = pack_f16(S[u + 2], S[u + 3]);
            x.z = pack_f16(S[u + 4], S[u + 5]);
            x.w = pack_f16(S[u + 6], S[u + 7]);
            *reinterpret_cast<uint4 *>(sm + C_S16 + half * 16384 + sw128k_off(row, u, 0)) = x;
        }
    };
    auto issue_x = [&](int c) {   // X[c&1] = [Qs;W] S16
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            mma_f16(tmem + CCOL_X + (c & 1) * 128, d_qw0 + (c & 1) * kSlotDesc + (((kk >> 2) * kQWBlk + (kk & 3) * 32) >> 4),
                    d_s16 + ((kk * 2048) >> 4), IDESC_X, kk > 0);
        tc::mma_commit(bar_x);
    };
    float *red = reinterpret_cast<float *>(sm + C_RED);
    float *nw = reinterpret_cast<float *>(sm + C_NW);
    if (kGated && tid < kD) nw[tid] = norm_w[tid];
    write_s16();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) pull(0, true);
    if (nchunks > 0) {
        if (wait_local(full, ph_full & 1, ctl)) pend_full &= ~1u;
        if (tid == 0 && !aborted(ctl)) {
            issue_x(0);
            pend_x = true;
        }
    }

    if (kGated && tid == 32)   // the output gate's rows of the first two chunks, into L2
        for (int c2 = 0; c2 < 2 && c2 < nchunks; ++c2)
            tc::tma_prefetch_l2_3d(tm_z, 0, h, static_cast<int>(ztok + c2 * kC));
    for (int c = 0; c < nchunks; ++c) {
        if (__syncthreads_or(aborted(ctl))) break;   // uniform: the cluster gave up
        const int s = c & 1;
        const int t0 = c * kC;
        const int valid = min(kC, T - t0);
        // the epilogue reads the output gate's rows from L2, two chunks after their prefetch
        if (kGated && tid == 32 && c + 2 < nchunks)
            tc::tma_prefetch_l2_3d(tm_z, 0, h, static_cast<int>(ztok + (c + 2) * kC));
        const uint8_t *slot = sm + C_SLOT + s * kSlotStride;
        const uint32_t xcol = CCOL_X + s * 128;
        if (wait_local(full + s, (ph_full >> s) & 1, ctl)) {  // (already complete) makes the slot visible
            ph_full ^= 1u << s;
            pend_full &= ~(1u << s);
        }
        if (tid == 0 && c + kRingSlots < nchunks && !aborted(ctl)) {  // the ring slot of chunk c is reusable
            // relaxed: the slot's bulk load has completed (observed above); no writes of
            // this thread need to be ordered before the producer's reuse of the slot
            const uint32_t rb = tc::map_to_rank(p_loaded + 8 * ((c / kProducers) % kRingDepth), c % kProducers);
            asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(rb) : "memory");
        }
        if (wait_local(bar_x, ph_x, ctl)) {
            ph_x ^= 1;
            pend_x = false;
        }
        tc_fence_after();
        if (tid == 0) pull(c + 1, false);

        // U = U' - W S  (lanes 64..127 = tokens)
        if (quad >= 2) {
            const int i = row - 64;
            float x[64];
            const uint32_t ta = tc::tmem_addr(tmem, 32 * quad, xcol + half * 64);
            tc::tmem_ld32(ta, *reinterpret_cast<float(*)[32]>(&x[0]));
            tc::tmem_ld32(ta + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
            tc::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 64; u += 8) {
                const uint4 up = *reinterpret_cast<const uint4 *>(slot + SL_UP +
                                                                  sw128k_off(i, half * 64 + u, kTokBlk));
                const __half2 *h2 = reinterpret_cast<const __half2 *>(&up);
                uint4 y;
                uint32_t *yy = reinterpret_cast<uint32_t *>(&y);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float2 f = __half22float2(h2[m]);
                    yy[m] = pack_f16(f.x - x[u + 2 * m], f.y - x[u + 2 * m + 1]);
                }
                *reinterpret_cast<uint4 *>(sm + C_U16 + half * kTokBlk + sw128k_off(i, u, 0)) = y;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && !aborted(ctl)) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + CCOL_S, d_kb0 + s * kSlotDesc + ((kk * 2048) >> 4), d_u16 + ((kk * 2048) >> 4), IDESC_S, kk > 0);
            tc::mma_commit(bar_s);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + xcol, d_pt0 + s * kSlotDesc + ((kk * 32) >> 4), d_u16 + ((kk * 2048) >> 4), IDESC_X, 1);
            tc::mma_commit(bar_o);
            pend_s = pend_o = true;
            pull(c + 1, false);
        }
        // S <- Diag(e^{g_C}) S + Kb^T U
        if (wait_local(bar_s, ph_s, ctl)) {
            ph_s ^= 1;
            pend_s = false;
        }
        tc_fence_after();
        {
            const float gm = reinterpret_cast<const float *>(slot + SL_GAM)[row];
            float sv[64];
            const uint32_t ta = tc::tmem_addr(tmem, 32 * quad, CCOL_S + half * 64);
            tc::tmem_ld32(ta, *reinterpret_cast<float(*)[32]>(&sv[0]));
            tc::tmem_ld32(ta + 32, *reinterpret_cast<float(*)[32]>(&sv[32]));
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 64; ++j) S[j] = fmaf(gm, S[j], sv[j]);
        }
        write_s16();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (c + 1 < nchunks) {
            if (tid == 0) pull(c + 1, true);
            if (wait_local(full + (s ^ 1), (ph_full >> (s ^ 1)) & 1, ctl)) pend_full &= ~(1u << (s ^ 1));
            if (tid == 0 && !aborted(ctl)) {
                issue_x(c + 1);
                pend_x = true;
            }
        }
        // O = Qs S + P U  (lanes 0..63 = tokens)
        if (wait_local(bar_o, ph_o, ctl)) {
            ph_o ^= 1;
            pend_o = false;
        }
        tc_fence_after();
        if constexpr (!kGated) {
            if (quad < 2) {
                float o[64];
                const uint32_t ta = tc::tmem_addr(tmem, 32 * quad, xcol + half * 64);
                tc::tmem_ld32(ta, *reinterpret_cast<float(*)[32]>(&o[0]));
                tc::tmem_ld32(ta + 32, *reinterpret_cast<float(*)[32]>(&o[32]));
                tc::tmem_wait_ld();
                if (row < valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(out + ((ztok + t0 + row) * H + h) * kD + half * 64);
#pragma unroll
                    for (int u = 0; u < 64; u += 8) {
                        uint4 x;
                        x.x = pack_bf16(o[u], o[u + 1]);
                        x.y = pack_bf16(o[u + 2], o[u + 3]);
                        x.z = pack_bf16(o[u + 4], o[u + 5]);
                        x.w = pack_bf16(o[u + 6], o[u + 7]);
                        dst[u / 8] = x;
                    }
                }
            }
        } else {   // the layer epilogue: RMSNorm over the row's 128 channels, then the output gate
            float o[64];
            if (quad < 2) {
                const uint32_t ta = tc::tmem_addr(tmem, 32 * quad, xcol + half * 64);
                tc::tmem_ld32(ta, *reinterpret_cast<float(*)[32]>(&o[0]));
                tc::tmem_ld32(ta + 32, *reinterpret_cast<float(*)[32]>(&o[32]));
                tc::tmem_wait_ld();
                float ss0 = 0.f, ss1 = 0.f;   // this thread's half of the row's sum of squares
#pragma unroll
                for (int j = 0; j < 64; j += 2) {
                    ss0 = fmaf(o[j], o[j], ss0);
                    ss1 = fmaf(o[j + 1], o[j + 1], ss1);
                }
                red[2 * row + half] = ss0 + ss1;
            }
            __syncthreads();
            if (quad < 2 && row < valid) {
                const long orow = ((ztok + t0 + row) * H + h) * kD + half * 64;
                const float r = rsqrtf((red[2 * row] + red[2 * row + 1]) * (1.f / kD) + eps);
                const uint4 *zp = reinterpret_cast<const uint4 *>(out_gate + orow);
#pragma unroll
                for (int u = 0; u < 64; u += 8) {
                    const uint4 z4 = zp[u / 8];
                    const uint32_t zw[4] = {z4.x, z4.y, z4.z, z4.w};
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float z0 = tc::bf16_lo(zw[m]), z1 = tc::bf16_hi(zw[m]);
                        const int j = u + 2 * m;
                        // sigmoid(z) = (1 + tanh(z / 2)) / 2: one MUFU operation per element
                        o[j] *= r * nw[half * 64 + j] * fmaf(0.5f, tanh_fast(0.5f * z0), 0.5f);
                        o[j + 1] *= r * nw[half * 64 + j + 1] * fmaf(0.5f, tanh_fast(0.5f * z1), 0.5f);
                    }
                }
                uint4 *dst = reinterpret_cast<uint4 *>(out + orow);
#pragma unroll
                for (int u = 0; u < 64; u += 8) {
                    uint4 x;
                    x.x = pack_bf16(o[u], o[u + 1]);
                    x.y = pack_bf16(o[u + 2], o[u + 3]);
                    x.z = pack_bf16(o[u + 4], o[u + 5]);
                    x.w = pack_bf16(o[u + 6], o[u + 7]);
                    dst[u / 8] = x;
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0) pull(c + 2, false);  // the slot of chunk c is free
    }
    // drain: what this CTA issued and has not seen complete (all of it after a give-up)
    if (tid == 0) {
#pragma unroll
        for (int sl = 0; sl < 2; ++sl)
            if ((pend_full >> sl) & 1) drain(full + sl, (ph_full >> sl) & 1, ctl);
        if (pend_x) drain(bar_x, ph_x, ctl);
        if (pend_s) drain(bar_s, ph_s, ctl);
        if (pend_o) drain(bar_o, ph_o, ctl);
    }
    if (S_T) {
#pragma unroll
        for (int j = 0; j < 64; ++j) S_T[(srow * kD + row) * kD + half * 64 + j] = S[j];
    }
}

template <bool kFused, bool kGated>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 1)
chunk_cluster_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_qs, const __grid_constant__ CUtensorMap tm_ks,
                     const __grid_constant__ CUtensorMap tm_las, const float *__restrict__ beta,
                     const float *S0, __nv_bfloat16 *__restrict__ out,
                     float *S_T, uint8_t *__restrict__ ws, int T, int H, int *err,
                     int test_timeout, const int32_t *__restrict__ cu_seqlens,
                     const int32_t *__restrict__ slot, const __nv_bfloat16 *__restrict__ out_gate,
                     const float *__restrict__ norm_w, float norm_eps,
                     const __grid_constant__ CUtensorMap tm_z, int nrings) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int rank = static_cast<int>(tc::cluster_rank());
    const long bh = blockIdx.x / kCluster;
    const int b = static_cast<int>(bh / H), h = static_cast<int>(bh - static_cast<long>(b) * H);
    // this cluster's tokens and state row: batch b of a dense [B, T] batch, or packed sequence
    // b (T is then the packed total; offsets clamped to [0, T]) with an optional slot map
    long ztok = static_cast<long>(b) * T, srow = bh;
    int len = T;
    if (cu_seqlens) {
        const int a0 = min(max(cu_seqlens[b], 0), T), a1 = min(max(cu_seqlens[b + 1], a0), T);
        ztok = a0;
        len = a1 - a0;
        if (slot) srow = static_cast<long>(slot[b]) * H + h;
    }
    const int nchunks = (len + kC - 1) / kC;
    const bool is_consumer = rank == kCluster - 1;
    const uint32_t bar_off = is_consumer ? C_BAR : P_BAR;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + bar_off);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + bar_off + 128);
    int *abort = reinterpret_cast<int *>(sm + bar_off + 132);
    const int tid = threadIdx.x;

    int *ring_slot = reinterpret_cast<int *>(sm + bar_off + 136);
    uint32_t *pool = reinterpret_cast<uint32_t *>(ws);
    if (tid == 0) {
        for (int i = 0; i < 14; ++i) tc::mbar_init(bars + i, 1);
        *abort = 0;
        tc::fence_mbar_init();
        if (rank == 0) *ring_slot = claim_ring(pool, nrings, kWaitLimit);   // this cluster's ring
    }
    if ((tid >> 5) == 0) {
        tc::tmem_alloc(tmem_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tc::cluster_sync();  // every barrier of the cluster is initialised before any remote use
    const uint32_t tmem = *tmem_slot;
    Ctl ctl{abort, err, {0, 0, 0, 0}, test_timeout ? kTestWaitLimit : kWaitLimit};
#pragma unroll
    for (int r = 0; r < kCluster; ++r)   // every CTA's abort flag (a producer's or the consumer's offset)
        ctl.peer_abort[r] = tc::map_to_rank(tc::smem_u32(sm) + (r == kCluster - 1 ? C_BAR : P_BAR) + 132, r);

    // the ring rank 0 claimed (read from its shared memory after the cluster barrier above)
    int ring_id;
    asm volatile("ld.shared::cluster.u32 %0, [%1];"
                 : "=r"(ring_id) : "r"(tc::map_to_rank(tc::smem_u32(sm) + P_BAR + 136, 0)) : "memory");
    uint8_t *ring = ws + kClusterPoolHeader + static_cast<size_t>(ring_id < 0 ? 0 : ring_id) * kRingSlots * kSlotStride;
    if (ring_id < 0) {   // no ring became free within the wait: report it and do nothing
        if (rank == 0 && tid == 0) atomicExch(err, 2);
    } else if (is_consumer)
        consumer<kGated>(sm, tmem, ring, S0, out, S_T, len, H, h, srow, ztok, nchunks, ctl, out_gate,
                         norm_w, norm_eps, &tm_z);
    else
        producer<kFused>(sm, tmem, rank, ring, &tm_v, &tm_qs, &tm_ks, &tm_las, beta, len, H, h, ztok, nchunks,
                         ctl, test_timeout);

    tc_fence_before();
    __syncthreads();
    tc::cluster_sync();  // no CTA leaves while a peer may still touch its shared memory
    if (rank == 0 && tid == 0 && ring_id >= 0) release_ring(pool, ring_id);   // every access to it is done
    if ((tid >> 5) == 0) {
        tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
                cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 3-D map over a [B*T, H, 128] tensor with a (box_x, 1, 64) box. box_x = 128 without
// swizzle (plain 256/512-byte rows: v loads and L2 prefetches), or 128 bytes' worth of
// channels with the 128-byte swizzle (q, k, log alpha for the prologue).
bool make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int esize, int H, long tokens,
              bool swizzled) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(tokens)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * esize,
                                   static_cast<cuuint64_t>(kD) * esize * H};
    const cuuint32_t box[3] = {swizzled ? static_cast<cuuint32_t>(128 / esize) : static_cast<cuuint32_t>(kD),
                               1, kC};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE,
               swizzled ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Test hook (kda_test_inject_wait_timeout): small wait limits and one withheld "ready".
int g_test_timeout = 0;

bool chunk_cluster_supported(int dk, int dv, int chunk, int dtype) {
    return dtype == KDA_BF16 && dk == kD && dv == kD && chunk == kC;
}

size_t chunk_cluster_workspace_bytes(int B, int H) {
    const long heads = static_cast<long>(B) * H;
    return kClusterPoolHeader + static_cast<size_t>(heads < kClusterMaxRings ? heads : kClusterMaxRings) *
                                    kRingSlots * kSlotStride;
}

cudaError_t launch_chunk_cluster(const ChunkArgs &a, cudaStream_t s) {
    const long tokens = a.cu_seqlens ? static_cast<long>(a.T) : static_cast<long>(a.B) * a.T;
    const CUtensorMapDataType kB16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kF32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const bool fused = a.gate != nullptr;   // the layer prologue: gate pre-activation instead of log alpha
    CUtensorMap mv, mqs, mks, mlas;
    const bool ok =
        make_map(&mv, a.v, kB16, 2, a.H, tokens, false) &&
        make_map(&mqs, a.q, kB16, 2, a.H, tokens, true) && make_map(&mks, a.k, kB16, 2, a.H, tokens, true) &&
        (fused ? make_map(&mlas, a.gate, kB16, 2, a.H, tokens, true)
               : make_map(&mlas, a.log_alpha, kF32, 4, a.H, tokens, true));
    if (!ok) return cudaErrorInvalidValue;
    // the layer epilogue comes with the layer prologue only (kda_layer_fwd); its output gate
    // is prefetched into L2 through a map over [tokens, H, 128] bf16 (unused otherwise)
    const bool gated = fused && a.out_gate != nullptr;
    CUtensorMap mz{};
    if (gated && !make_map(&mz, a.out_gate, kB16, 2, a.H, tokens, false)) return cudaErrorInvalidValue;
    auto kern = gated ? chunk_cluster_kernel<true, true>
                      : (fused ? chunk_cluster_kernel<true, false> : chunk_cluster_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    // the ring pool: as many rings as the workspace was sized for; a caller's workspace has its
    // in-use bitmap cleared here (the library's fixed pool keeps its own clear between calls)
    const long heads = static_cast<long>(a.B) * a.H;
    const int nrings = static_cast<int>(heads < kClusterMaxRings ? heads : kClusterMaxRings);
    if (!a.fixed_pool && (e = cudaMemsetAsync(a.workspace, 0, kClusterPoolHeader, s)) != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(a.B) * a.H * kCluster);
    kern<<<grid, kThreads, kSmemBytes, s>>>(
        mv, mqs, mks, mlas, a.beta, a.S0, static_cast<__nv_bfloat16 *>(a.out), a.S_T,
        static_cast<uint8_t *>(a.workspace), a.T, a.H, a.device_error, g_test_timeout, a.cu_seqlens, a.slot,
        static_cast<const __nv_bfloat16 *>(a.out_gate), a.norm_weight, a.norm_eps, mz, nrings);
    return cudaGetLastError();
}

int set_test_timeout(int on) {
    const int old = g_test_timeout;
    g_test_timeout = on ? 1 : 0;
    return old;
}

}  // namespace kda
