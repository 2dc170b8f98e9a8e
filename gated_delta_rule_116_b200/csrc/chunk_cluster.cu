// chunk_cluster.cu -- cluster engine of the chunked KDA prefill on sm_100a
// (bf16 q/k/v, d_k = d_v = 128, chunk C = 64, fp32 gates and state).
//
// Same chunked form and operand precisions as chunk_tc.cu (Kimi Linear
// summary, es.news.hada.io/topic?id=31936, sections "Algoritmo paralelo por
// chunks" and "Menor cantidad de operaciones que DPLR general"):
//   [A;P] = [K*E ; Q*E](K*F)^T (tf32), T = (I + A)^{-1} Diag(beta),
//   [W | U'] = T [Ks | V] (fp16), then the state chain
//   X = [Qs ; W] S, U = U' - W S, S <- Diag(e^{g_C}) S + Kb^T U, O = Qs S + P U.
//
// The work of one chunk splits into a key-side part that does not depend on
// the state (everything up to W, U', P, T, Qs, Kb) and the state chain, which
// is sequential over chunks. One head runs on a cluster of 4 CTAs (4 SMs):
//   * ranks 0..2 are producers: rank p computes the key-side part of chunks
//     p, p+3, p+6, ... as an 82 KB image and writes it into one of its three
//     slots of a small ring in the workspace (it stays in L2): Qs, Kb and
//     e^{g_C} straight from registers in the gate prologue; [P;T] (an operand
//     of its own MMA), W and U' staged in shared memory and bulk-stored
//     (cp.async.bulk shared -> global), [P;T] as soon as T is formed and W
//     while U' is formed. Once the
//     stores are complete, thread 0 arrives (release, cluster scope; the
//     generic stores of all threads precede it through a CTA barrier) on the
//     consumer's "ready" barrier of that slot;
//   * rank 3 is the consumer: it keeps the 128x128 fp32 state in registers and
//     runs the chain for every chunk, on all 128 value columns. Its thread 0
//     pulls published images into two shared-memory slots (bulk global ->
//     shared loads) as soon as a slot is free, and tells the producer (its
//     "loaded" barrier) that the ring slot may be reused.
// The ring goes through L2 because a DSMEM bulk copy moves only ~20 B/cycle
// between two SMs, whereas an L2 bulk load of the same 82 KB takes ~1K cycles.
// The producers set the pace of the cluster, so their image stores are kept
// short: writing Qs and Kb from registers and storing [P;T] and W early
// leaves only U' (16 KB) to store and wait for at the end of an image.
// A producer thus has three chunk periods for the key-side latency, and the
// consumer's chunk period is the chain alone. Every wait is bounded; after a
// timeout a CTA records an error in the device error word, stops waiting and
// still reaches the final cluster barrier and frees its tensor memory.
#include <cuda.h>

#include "kda_internal.cuh"
#include "tc_sm100.cuh"
#include "ut_solve.cuh"

namespace kda {
namespace {

using tc::fence_proxy_async_smem;
using tc::mma_f16;
using tc::mma_tf32;
using tc::pack_bf16;
using tc::pack_f16;
using tc::sw128k_off;
using tc::tc_fence_after;
using tc::tc_fence_before;
using ut::kLD;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 256;
constexpr int kProducers = 3;
constexpr int kCluster = kProducers + 1;
constexpr int kRingDepth = 3;   // ring slots per producer
constexpr int kRingSlots = kRingDepth * kProducers;
constexpr uint32_t kWaitLimit = 1u << 22;

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

// ---- producer shared memory
constexpr uint32_t P_KQT = 0;          // [K*E ; Q*E] tf32, 4 K-blocks x 16 KB
constexpr uint32_t kKQTBlk = 16384;
constexpr uint32_t P_KHT = 65536;      // K*F tf32, 4 K-blocks x 8 KB
constexpr uint32_t kKHTBlk = 8192;
constexpr uint32_t P_AF = 0;           // A (fp32), reuses the tf32 region after the product
constexpr uint32_t P_XF = 64 * kLD * 4;
// ... and after the UT solve, holds the TMA-loaded inputs of the producer's next chunk:
constexpr uint32_t P_IN_Q = 0;         // q  [64 tokens][128] bf16
constexpr uint32_t P_IN_K = 16384;     // k
constexpr uint32_t P_IN_LA = 32768;    // log alpha [64][128] fp32
constexpr uint32_t P_IN_V = 65536;     // v  [64][128] bf16
constexpr uint32_t kInBytes = 81920;
constexpr uint32_t P_STAGE = 98304;    // image-sized area: [P;T], W and U' are staged here
constexpr uint32_t P_KSV = P_STAGE + kSlotStride;  // [Ks | V] fp16 [token][col], 4 blocks x 8 KB
constexpr uint32_t P_VEC = P_KSV + 32768;          // beta[64], psum[4][128]
constexpr uint32_t P_BAR = P_VEC + (64 + 512) * 4;
// ---- consumer shared memory
constexpr uint32_t C_SLOT = 0;         // 2 slots
constexpr uint32_t C_S16 = 2 * kSlotStride;        // S fp16, MN-major SW128: 2 blocks x 16 KB
constexpr uint32_t C_U16 = C_S16 + 32768;          // U fp16, MN-major SW128: 2 blocks x 8 KB
constexpr uint32_t C_BAR = C_U16 + 16384;
#ifdef KDA_PHASE_TIMING
constexpr uint32_t kDbgBytes = 256;    // per-phase cycle accumulators, after the barriers
#else
constexpr uint32_t kDbgBytes = 0;
#endif
constexpr uint32_t kSmemBytes =
    (P_BAR > C_BAR ? P_BAR : C_BAR) + 192 + kDbgBytes + 1024;  // + barriers + alignment slack

// TMEM columns.
constexpr uint32_t PCOL_AP = 0;        // producer: [A;P] (64 cols)
constexpr uint32_t PCOL_WU = 64;       // producer: [P;T][Ks|V], lanes 64-127 = [W | U'] (256)
constexpr uint32_t CCOL_X = 0;         // consumer: 2 x 128 cols ([Qs;W]S (+ [P;T]U))
constexpr uint32_t CCOL_S = 256;       // consumer: Kb^T U (128 cols)
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t IDESC_AP = tc::idesc(tc::kFmtTF32, 128, 64, 0, 0);
constexpr uint32_t IDESC_WU = tc::idesc(tc::kFmtF16, 128, 256, 0, 1);
constexpr uint32_t IDESC_X = tc::idesc(tc::kFmtF16, 128, 128, 0, 1);   // A K-major, B MN-major
constexpr uint32_t IDESC_S = tc::idesc(tc::kFmtF16, 128, 128, 1, 1);   // A MN-major, B MN-major

#ifdef KDA_PHASE_TIMING
// Debug builds only: cycles per phase summed over chunks, for cluster 0
// (slots 0..9 producer rank 0, slots 16..23 the consumer). Thread 0 of each CTA
// accumulates in shared memory (a global read-modify-write per mark would cost
// ~1K cycles and distort the phases) and adds its slots to the global array once.
__device__ unsigned long long g_cluster_cycles[32];
#define CMARK(idx)                                                        \
    do {                                                                  \
        if (threadIdx.x == 0 && (idx) < 32) {                             \
            const unsigned long long now_ = clock64();                    \
            t_acc_[idx] += now_ - t_prev_;                                \
            t_prev_ = now_;                                               \
        }                                                                 \
    } while (0)
#define CMARK_INIT(bar_off)                                                                 \
    unsigned long long *t_acc_ = reinterpret_cast<unsigned long long *>(sm + (bar_off) + 192); \
    if (threadIdx.x == 0)                                                                   \
        for (int i_ = 0; i_ < 32; ++i_) t_acc_[i_] = 0;                                     \
    unsigned long long t_prev_ = clock64()
#define CMARK_FLUSH(lo, hi)                                                               \
    do {                                                                                  \
        if (blockIdx.x < kCluster && threadIdx.x == 0)                                    \
            for (int i_ = (lo); i_ < (hi); ++i_) atomicAdd(&g_cluster_cycles[i_], t_acc_[i_]); \
    } while (0)
#else
#define CMARK(idx) \
    do {           \
    } while (0)
#define CMARK_INIT(bar_off)
#define CMARK_FLUSH(lo, hi) \
    do {                    \
    } while (0)
#endif

struct Ctl {
    int *abort;
    int *err;
};

__device__ __forceinline__ void fail(const Ctl &k) {
    *reinterpret_cast<volatile int *>(k.abort) = 1;
    atomicExch(k.err, 2);
}
__device__ __forceinline__ void wait_local(uint64_t *bar, uint32_t parity, const Ctl &k) {
    if (*reinterpret_cast<volatile int *>(k.abort)) return;
    if (!tc::mbar_wait(bar, parity, kWaitLimit)) fail(k);
}
__device__ __forceinline__ void wait_cluster(uint64_t *bar, uint32_t parity, const Ctl &k) {
    if (*reinterpret_cast<volatile int *>(k.abort)) return;
    if (!tc::mbar_wait_cluster(bar, parity, kWaitLimit)) fail(k);
}

// ============================================================ producer
__device__ void producer(uint8_t *sm, uint32_t tmem, int rank, uint8_t *ring, const CUtensorMap *tm_q,
                         const CUtensorMap *tm_k, const CUtensorMap *tm_la,
                         const CUtensorMap *tm_v, const __nv_bfloat16 *__restrict__ q,
                         const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
                         const float *__restrict__ log_alpha, const float *__restrict__ beta,
                         int T, int H, int h, long ztok, int nchunks, const Ctl &ctl) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = 32 * quad + lane;
    const uint32_t sbase = tc::smem_u32(sm);
    float *beta_s = reinterpret_cast<float *>(sm + P_VEC);
    float *psum = beta_s + 64;
    float *Af = reinterpret_cast<float *>(sm + P_AF);
    float *Xf = reinterpret_cast<float *>(sm + P_XF);
    uint64_t *bar_mma = reinterpret_cast<uint64_t *>(sm + P_BAR);
    uint64_t *bar_loaded = bar_mma + 1;  // [kRingDepth]: one per ring slot of this producer
    uint8_t *st = sm + P_STAGE;
    uint32_t ph_mma = 0;
    int img = 0;  // index of this producer's next image

    const uint64_t d_kqt = tc::smem_desc(sbase + P_KQT, 16, 1024, tc::kSwizzle128);
    const uint64_t d_kht = tc::smem_desc(sbase + P_KHT, 16, 1024, tc::kSwizzle128);
    const uint64_t d_pt = tc::smem_desc(sbase + P_STAGE + SL_PT, 16, 1024, tc::kSwizzle128);
    const uint64_t d_ksv = tc::smem_desc(sbase + P_KSV, kTokBlk, 1024, tc::kSwizzle128);
    // the consumer's "ready" barriers for this producer's ring slots
    const uint32_t c_ready = tc::map_to_rank(sbase + C_BAR + 40 + 8 * kRingDepth * rank, kCluster - 1);

    CMARK_INIT(P_BAR);
    const int mk = rank == 0 ? 0 : 64;  // only rank 0 records (slots 0..8)
    uint64_t *bar_in = bar_mma + 1 + kRingDepth;
    uint32_t ph_in = 0;
    auto load_inputs = [&](int cc) {   // TMA: the 64-token chunk cc of head h (all channels)
        const int z = static_cast<int>(ztok + static_cast<long>(cc) * kC);
        tc::mbar_arrive_expect_tx(bar_in, kInBytes);
        tc::tma_load_3d(sm + P_IN_Q, tm_q, bar_in, 0, h, z);
        tc::tma_load_3d(sm + P_IN_K, tm_k, bar_in, 0, h, z);
        tc::tma_load_3d(sm + P_IN_LA, tm_la, bar_in, 0, h, z);
        tc::tma_load_3d(sm + P_IN_V, tm_v, bar_in, 0, h, z);
    };
    if (tid == 0 && rank < nchunks) load_inputs(rank);
    for (int c = rank; c < nchunks; c += kProducers) {
        const int t0 = c * kC;
        const int valid = min(kC, T - t0);
        const long trow0 = ztok + t0;
        if (tid == 0 && c + 2 * kProducers < nchunks) {
            const int z = static_cast<int>(trow0 + 2 * kProducers * kC);
            tc::tma_prefetch_l2_3d(tm_q, 0, h, z);
            tc::tma_prefetch_l2_3d(tm_k, 0, h, z);
            tc::tma_prefetch_l2_3d(tm_la, 0, h, z);
            tc::tma_prefetch_l2_3d(tm_v, 0, h, z);
        }
        wait_local(bar_in, ph_in, ctl);
        ph_in ^= 1;
        CMARK(mk + 0);

        // ------------------------------------------------ gates and operands
        if (tid < kC) beta_s[tid] = tid < valid ? beta[(trow0 + tid) * H + h] : 0.f;
        uint4 vin[4];   // V row tid/4, columns 32 (tid%4) .. +32 (bf16); stored while [A;P] runs
        {
            const int t = tid >> 2, piece = tid & 3;
            const uint4 *src = reinterpret_cast<const uint4 *>(sm + P_IN_V + t * 256 + 64 * piece);
#pragma unroll
            for (int m = 0; m < 4; ++m) vin[m] = t < valid ? src[m] : make_uint4(0, 0, 0, 0);
        }
        const int p = tid & 63, qq = tid >> 6;  // channels 2p, 2p+1; tokens 16qq .. 16qq+15
        float2 lg[16];
        uint32_t qv[16], kv[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int t = 16 * qq + u;
            const bool ok = t < valid;
            lg[u] = ok ? *reinterpret_cast<const float2 *>(sm + P_IN_LA + t * 512 + 8 * p)
                       : make_float2(0.f, 0.f);
            qv[u] = ok ? *reinterpret_cast<const uint32_t *>(sm + P_IN_Q + t * 256 + 4 * p) : 0u;
            kv[u] = ok ? *reinterpret_cast<const uint32_t *>(sm + P_IN_K + t * 256 + 4 * p) : 0u;
        }
        {
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) { s0 += lg[u].x; s1 += lg[u].y; }
            psum[qq * 128 + 2 * p] = s0;
            psum[qq * 128 + 2 * p + 1] = s1;
        }
        const int rb = img % kRingDepth;  // ring slot of this image; image img-kRingDepth used it before
        uint8_t *gs = ring + (kRingDepth * rank + rb) * kSlotStride;
        if (tid == 0) {
            tc::bulk_wait_read_all();  // the previous [P;T] has left the staging area
            if (img >= kRingDepth) wait_cluster(bar_loaded + rb, ((img / kRingDepth) - 1) & 1, ctl);
        }
        __syncthreads();  // inputs are in registers: the tf32 tiles may now overwrite them
        {
            float pre0 = 0.f, pre1 = 0.f, tot0 = 0.f, tot1 = 0.f;
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
                const float a0 = psum[q2 * 128 + 2 * p], a1 = psum[q2 * 128 + 2 * p + 1];
                if (q2 < qq) { pre0 += a0; pre1 += a1; }
                tot0 += a0;
                tot1 += a1;
            }
            const float ga0 = 0.5f * tot0, ga1 = 0.5f * tot1;
            const float ea0 = expf(ga0), ea1 = expf(ga1);                  // e^{g_a}
            const float eca0 = expf(tot0 - ga0), eca1 = expf(tot1 - ga1);  // e^{g_C - g_a}
            if (qq == 0) {
                float *gam = reinterpret_cast<float *>(gs + SL_GAM);
                gam[2 * p] = expf(tot0);
                gam[2 * p + 1] = expf(tot1);
            }
            constexpr float kLog2e = 1.4426950408889634f;
            float d0 = (pre0 - ga0) * kLog2e, d1 = (pre1 - ga1) * kLog2e;
            const uint32_t cc = 2 * p;
            const uint32_t rowq = qq * 2048u;
            const uint32_t b32 = (cc & 3u) * 4u + rowq;
            const uint32_t ch32 = (cc & 31u) >> 2, kb32 = cc >> 5;
            const uint32_t b16 = (cc & 7u) * 2u + rowq;
            const uint32_t ch16 = (cc & 63u) >> 3, kb16 = cc >> 6;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const uint32_t r = (u >> 3) * 1024u + (u & 7) * 128u;
                const uint32_t o32 = b32 + r + (((ch32 ^ (u & 7)) & 7u) << 4);
                const uint32_t o16 = b16 + r + (((ch16 ^ (u & 7)) & 7u) << 4);
                d0 = fmaf(lg[u].x, kLog2e, d0);
                d1 = fmaf(lg[u].y, kLog2e, d1);
                const float q0 = tc::bf16_lo(qv[u]), q1 = tc::bf16_hi(qv[u]);
                const float k0 = tc::bf16_lo(kv[u]), k1 = tc::bf16_hi(kv[u]);
                const float E0 = tc::ex2(d0), E1 = tc::ex2(d1);
                const float F0 = tc::ex2(-d0), F1 = tc::ex2(-d1);
                const float ke0 = k0 * E0, ke1 = k1 * E1, qe0 = q0 * E0, qe1 = q1 * E1;
                const float kf0 = k0 * F0, kf1 = k1 * F1;
                *reinterpret_cast<float2 *>(sm + P_KQT + kb32 * kKQTBlk + o32) = make_float2(ke0, ke1);
                *reinterpret_cast<float2 *>(sm + P_KQT + kb32 * kKQTBlk + 8192 + o32) = make_float2(qe0, qe1);
                *reinterpret_cast<float2 *>(sm + P_KHT + kb32 * kKHTBlk + o32) = make_float2(kf0, kf1);
                *reinterpret_cast<uint32_t *>(gs + SL_QW + kb16 * kQWBlk + o16) = pack_f16(qe0 * ea0, qe1 * ea1);
                *reinterpret_cast<uint32_t *>(sm + P_KSV + kb16 * kTokBlk + o16) = pack_f16(ke0 * ea0, ke1 * ea1);
                *reinterpret_cast<uint32_t *>(gs + SL_KB + kb16 * kTokBlk + o16) = pack_f16(kf0 * eca0, kf1 * eca1);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        CMARK(mk + 1);

        // ------------------------------------------------ [A;P] (tf32)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 16; ++kk)
                mma_tf32(tmem + PCOL_AP, d_kqt + (((kk >> 2) * kKQTBlk + (kk & 3) * 32) >> 4),
                         d_kht + (((kk >> 2) * kKHTBlk + (kk & 3) * 32) >> 4), IDESC_AP, kk > 0);
            tc::mma_commit(bar_mma);
        }
        {   // V -> fp16 columns 128..255 of the [Ks | V] operand (read by [W | U'] only)
            const int t = tid >> 2, piece = tid & 3;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                uint4 w;
                w.x = pack_f16(tc::bf16_lo(vin[m].x), tc::bf16_hi(vin[m].x));
                w.y = pack_f16(tc::bf16_lo(vin[m].y), tc::bf16_hi(vin[m].y));
                w.z = pack_f16(tc::bf16_lo(vin[m].z), tc::bf16_hi(vin[m].z));
                w.w = pack_f16(tc::bf16_lo(vin[m].w), tc::bf16_hi(vin[m].w));
                *reinterpret_cast<uint4 *>(sm + P_KSV + 2 * kTokBlk +
                                           sw128k_off(t, 32 * piece + 8 * m, kTokBlk)) = w;
            }
        }
        wait_local(bar_mma, ph_mma, ctl);
        ph_mma ^= 1;
        tc_fence_after();
        CMARK(mk + 2);

        // ------------------------------------------------ A (fp32), P (fp16), UT solve, T (fp16)
        {
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
                    *reinterpret_cast<uint32_t *>(st + SL_PT + sw128k_off(i, j, 0)) = pack_f16(lo, hi);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        CMARK(mk + 3);
        ut::unit_lower_inverse(Af, Xf, tid);
        CMARK(mk + 4);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = tid + u * kThreads;
            const int i = e >> 5, j = (e & 31) * 2;
            const float lo = j <= i ? Xf[i * kLD + j] * beta_s[j] : 0.f;
            const float hi = j + 1 <= i ? Xf[i * kLD + j + 1] * beta_s[j + 1] : 0.f;
            *reinterpret_cast<uint32_t *>(st + SL_PT + 8192 + sw128k_off(i, j, 0)) = pack_f16(lo, hi);
        }
        fence_proxy_async_smem();
        __syncthreads();
        // the tf32 region (tiles, A, X) is dead until the next chunk: stage its inputs there
        if (tid == 0) {
            if (c + kProducers < nchunks) load_inputs(c + kProducers);
            tc::bulk_store_global(gs + SL_PT, st + SL_PT, 16384);   // [P;T] to the ring slot
            tc::bulk_commit();
        }
        CMARK(mk + 5);

        // ------------------------------------------------ [W | U'] = T [Ks | V] (fp16, N = 256)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + PCOL_WU, d_pt + ((kk * 32) >> 4), d_ksv + ((kk * 2048) >> 4), IDESC_WU, kk > 0);
            tc::mma_commit(bar_mma);
        }
        wait_local(bar_mma, ph_mma, ctl);
        ph_mma ^= 1;
        tc_fence_after();
        CMARK(mk + 6);
#pragma unroll
        for (int part = 0; part < 2; ++part) {   // part 0: W, part 1: U'
            if (quad >= 2) {
                const int i = row - 64;
                float w[64];
                const uint32_t ta = tc::tmem_addr(tmem, 32 * quad, PCOL_WU + part * 128 + half * 64);
                tc::tmem_ld32(ta, *reinterpret_cast<float(*)[32]>(&w[0]));
                tc::tmem_ld32(ta + 32, *reinterpret_cast<float(*)[32]>(&w[32]));
                tc::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 64; u += 8) {
                    uint4 x;
                    x.x = pack_f16(w[u], w[u + 1]);
                    x.y = pack_f16(w[u + 2], w[u + 3]);
                    x.z = pack_f16(w[u + 4], w[u + 5]);
                    x.w = pack_f16(w[u + 6], w[u + 7]);
                    const int col = half * 64 + u;
                    const uint32_t off = part == 0 ? SL_QW + sw128k_off(64 + i, col, kQWBlk)
                                                   : SL_UP + sw128k_off(i, col, kTokBlk);
                    *reinterpret_cast<uint4 *>(st + off) = x;
                }
            }
            fence_proxy_async_smem();
            if (part == 0) {   // W leaves while U' is formed
                __syncthreads();
                if (tid == 0) {
                    tc::bulk_store_global(gs + SL_QW + 8192, st + SL_QW + 8192, 8192);   // W, K-block 0
                    tc::bulk_store_global(gs + SL_QW + kQWBlk + 8192, st + SL_QW + kQWBlk + 8192, 8192);
                    tc::bulk_commit();
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        CMARK(mk + 7);

        // ------------------------------------------------ publish the image through L2
        // Every thread's generic stores into the slot (Qs, Kb, e^{g_C}) precede thread 0's
        // release through the CTA barrier above; the release is cumulative.
        if (tid == 0) {
            CMARK(mk + 9);
            tc::bulk_store_global(gs + SL_UP, st + SL_UP, 16384);                  // U'
            tc::bulk_commit();
            tc::bulk_wait_all();   // [P;T], W and U' have reached the slot
            tc::fence_proxy_async_global();
            if (!*reinterpret_cast<volatile int *>(ctl.abort)) tc::mbar_arrive_remote(c_ready + 8 * rb);
        }
        CMARK(mk + 8);
        ++img;
    }
    if (tid == 0) tc::bulk_wait_read_all();
    CMARK_FLUSH(0, 10);
}

// ============================================================ consumer
__device__ void consumer(uint8_t *sm, uint32_t tmem, const uint8_t *ring, const float *__restrict__ S0,
                         __nv_bfloat16 *__restrict__ out, float *__restrict__ S_T, int T, int H,
                         int h, long bh, long ztok, int nchunks, const Ctl &ctl) {
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
            if (*reinterpret_cast<volatile int *>(ctl.abort)) return;
            tc::fence_proxy_async_global();
            const int sl = next_load & 1;
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
        S[j] = S0 ? S0[(bh * kD + row) * kD + half * 64 + j] : 0.f;
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
    write_s16();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) pull(0, true);
    if (nchunks > 0) {
        wait_local(full, ph_full & 1, ctl);
        if (tid == 0) issue_x(0);
    }

    CMARK_INIT(C_BAR);
    for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1;
        const int t0 = c * kC;
        const int valid = min(kC, T - t0);
        const uint8_t *slot = sm + C_SLOT + s * kSlotStride;
        const uint32_t xcol = CCOL_X + s * 128;
        wait_local(full + s, (ph_full >> s) & 1, ctl);  // (already complete) makes the slot visible
        ph_full ^= 1u << s;
        if (tid == 0 && c + kRingSlots < nchunks) {  // the ring slot of chunk c is reusable
            // relaxed: the slot's bulk load has completed (observed above); no writes of
            // this thread need to be ordered before the producer's reuse of the slot
            const uint32_t rb = tc::map_to_rank(p_loaded + 8 * ((c / kProducers) % kRingDepth), c % kProducers);
            asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(rb) : "memory");
        }
        CMARK(16);
#ifdef KDA_PHASE_TIMING
        const unsigned long long w0_ = clock64();
#endif
        wait_local(bar_x, ph_x, ctl);
        ph_x ^= 1;
        tc_fence_after();
#ifndef KDA_NO_EARLY_PULL
        if (tid == 0) pull(c + 1, false);
#endif
        CMARK(17);

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
#ifdef KDA_PHASE_TIMING
        if (blockIdx.x == kCluster - 1 && (threadIdx.x & 31) == 0)
            atomicAdd(&g_cluster_cycles[24 + (threadIdx.x >> 5)], clock64() - w0_);
#endif
        __syncthreads();
        CMARK(18);
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + CCOL_S, d_kb0 + s * kSlotDesc + ((kk * 2048) >> 4), d_u16 + ((kk * 2048) >> 4), IDESC_S, kk > 0);
            tc::mma_commit(bar_s);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + xcol, d_pt0 + s * kSlotDesc + ((kk * 32) >> 4), d_u16 + ((kk * 2048) >> 4), IDESC_X, 1);
            tc::mma_commit(bar_o);
            pull(c + 1, false);
        }
        // S <- Diag(e^{g_C}) S + Kb^T U
        wait_local(bar_s, ph_s, ctl);
        ph_s ^= 1;
        tc_fence_after();
        CMARK(19);
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
        CMARK(20);
        if (c + 1 < nchunks) {
            if (tid == 0) pull(c + 1, true);
            wait_local(full + (s ^ 1), (ph_full >> (s ^ 1)) & 1, ctl);
            if (tid == 0) issue_x(c + 1);
        }
        CMARK(21);
        // O = Qs S + P U  (lanes 0..63 = tokens)
        wait_local(bar_o, ph_o, ctl);
        ph_o ^= 1;
        tc_fence_after();
        CMARK(22);
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
        tc_fence_before();
        __syncthreads();
        if (tid == 0) pull(c + 2, false);  // the slot of chunk c is free
        CMARK(23);
    }
    if (S_T) {
#pragma unroll
        for (int j = 0; j < 64; ++j) S_T[(bh * kD + row) * kD + half * 64 + j] = S[j];
    }
    CMARK_FLUSH(16, 24);
}

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 1)
chunk_cluster_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_v,
                     const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                     const __nv_bfloat16 *__restrict__ v, const float *__restrict__ log_alpha,
                     const float *__restrict__ beta, const float *__restrict__ S0,
                     __nv_bfloat16 *__restrict__ out, float *__restrict__ S_T, uint8_t *__restrict__ ws,
                     int T, int H, int *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int rank = static_cast<int>(tc::cluster_rank());
    const long bh = blockIdx.x / kCluster;
    const int b = static_cast<int>(bh / H), h = static_cast<int>(bh - static_cast<long>(b) * H);
    const long ztok = static_cast<long>(b) * T;
    const int nchunks = (T + kC - 1) / kC;
    const bool is_consumer = rank == kCluster - 1;
    const uint32_t bar_off = is_consumer ? C_BAR : P_BAR;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + bar_off);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + bar_off + 128);
    int *abort = reinterpret_cast<int *>(sm + bar_off + 132);
    const int tid = threadIdx.x;

    if (tid == 0) {
        for (int i = 0; i < 14; ++i) tc::mbar_init(bars + i, 1);
        *abort = 0;
        tc::fence_mbar_init();
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
    const Ctl ctl{abort, err};

    uint8_t *ring = ws + bh * kRingSlots * kSlotStride;  // this head's ring: kRingDepth slots per producer
    if (is_consumer)
        consumer(sm, tmem, ring, S0, out, S_T, T, H, h, bh, ztok, nchunks, ctl);
    else
        producer(sm, tmem, rank, ring, &tm_q, &tm_k, &tm_la, &tm_v, q, k, v, log_alpha, beta, T, H, h,
                 ztok, nchunks, ctl);

    tc_fence_before();
    __syncthreads();
    tc::cluster_sync();  // no CTA leaves while a peer may still touch its shared memory
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

// 3-D map over a [B*T, H, 128] tensor with a (128, 1, 64) box, used for L2 prefetches.
bool make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int esize, int H, long tokens) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(tokens)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * esize,
                                   static_cast<cuuint64_t>(kD) * esize * H};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kD), 1, kC};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

#ifdef KDA_PHASE_TIMING
extern "C" int kda_debug_cluster_cycles(unsigned long long *out32, int reset) {
    cudaError_t e = cudaMemcpyFromSymbol(out32, g_cluster_cycles, sizeof(unsigned long long) * 32);
    if (reset) {
        unsigned long long z[32] = {0};
        cudaMemcpyToSymbol(g_cluster_cycles, z, sizeof z);
    }
    return e == cudaSuccess ? 0 : -1;
}
#endif

bool chunk_cluster_supported(int dk, int dv, int chunk, int dtype) {
    return dtype == KDA_BF16 && dk == kD && dv == kD && chunk == kC;
}

size_t chunk_cluster_workspace_bytes(int B, int H) {
    return static_cast<size_t>(B) * H * kRingSlots * kSlotStride;
}

cudaError_t launch_chunk_cluster(const ChunkArgs &a, cudaStream_t s) {
    const long tokens = static_cast<long>(a.B) * a.T;
    CUtensorMap mq, mk, mla, mv;
    if (!make_map(&mq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, tokens) ||
        !make_map(&mk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, tokens) ||
        !make_map(&mla, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.H, tokens) ||
        !make_map(&mv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, tokens))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_cluster_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(a.B) * a.H * kCluster);
    chunk_cluster_kernel<<<grid, kThreads, kSmemBytes, s>>>(
        mq, mk, mla, mv, static_cast<const __nv_bfloat16 *>(a.q),
        static_cast<const __nv_bfloat16 *>(a.k), static_cast<const __nv_bfloat16 *>(a.v),
        a.log_alpha, a.beta, a.S0, static_cast<__nv_bfloat16 *>(a.out), a.S_T,
        static_cast<uint8_t *>(a.workspace), a.T, a.H, a.device_error);
    return cudaGetLastError();
}

}  // namespace kda
