// chunk_tc.cu -- tensor-core (tcgen05 / TMEM) engine of the chunked KDA
// prefill for bf16 q/k/v, d_k = d_v = 128, chunk C = 64, fp32 gates and state.
//
// The chunked form (Kimi Linear summary, es.news.hada.io/topic?id=31936,
// section "Algoritmo paralelo por chunks"; the two intra-chunk products tied
// to the key, section "Menor cantidad de operaciones que DPLR general"). Per
// chunk, with g the in-chunk prefix sum of log alpha (per channel), anchor
// g_a = g_C / 2, E = e^{g - g_a} and F = 1/E:
//   [A;P] = [K*E ; Q*E] (K*F)^T        tf32 tcgen05 (M=128 N=64 K=128): the two
//       A = Diag(beta) strict_lower(.)  products; factors up to e^{|g_C|/2}
//       P = lower(.)                    need a wide exponent range
//   T = (I + A)^{-1} Diag(beta)        blocked forward substitution, fp32
//   W = T Ks,  U' = T V                fp16 tcgen05 (WY / UT form),
//                                      Ks = K*e^{g}, Qs = Q*e^{g} (|.| <= |k|, |q|)
//   [Qs S ; W S] = [Qs;W] S            fp16 tcgen05 on an fp16 copy of S
//   U = U' - W S
//   O = Qs S + P U                     fp16 tcgen05
//   S <- Diag(e^{g_C}) S + Kb^T U      Kb = K*e^{g_C - g} (|.| <= |k|), fp16
//                                      tcgen05 + fp32 add in registers
// In exact arithmetic O and S equal the token-by-token recurrence. Every
// fp16 operand is bounded by the inputs (the gate factors are <= 1), which
// keeps fp16's 11-bit precision inside its range; only the two intra-chunk
// products see factors of e^{+-|g_C|/2} and run in tf32. S stays in fp32
// registers for the whole sequence.
//
// Mapping: one CTA (8 warps) per (b, h, 32 value columns). Value columns of
// the state evolve independently, so the 4 slices of a head never talk; each
// recomputes the key-side work of its chunk. Phases run one after another;
// each tcgen05.mma is issued by thread 0 and its completion is signalled
// through an mbarrier (tcgen05.commit). Inputs are read with coalesced loads
// after a TMA prefetch of the chunk into L2. Every wait is bounded: on timeout
// the kernel records an error in the device error word, stops waiting, and
// still releases its tensor memory.
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
using tc::sw128k_off32;
using tc::sw64mn_off;
using tc::tc_fence_after;
using tc::tc_fence_before;

constexpr int kC = 64;       // chunk length
constexpr int kD = 128;      // d_k = d_v
constexpr int kNV = 32;      // value columns per CTA
constexpr int kThreads = 256;
constexpr uint32_t kWaitLimit = 1u << 24;

// Shared-memory map (bytes from a 1024-aligned base).
// Key-side tf32 operands, dead after the first MMA of the chunk:
constexpr uint32_t OFF_KQT = 0;           // [K*E ; Q*E] tf32, 4 K-blocks x 16 KB (128 rows)
constexpr uint32_t kKQTBlk = 16384;
constexpr uint32_t OFF_KHT = 65536;       // K*F tf32, 4 K-blocks x 8 KB (64 rows)
constexpr uint32_t kKHTBlk = 8192;
// ... then reused for the solve and the [P;T] operand:
using ut::kLD;                            // row stride (floats) of A / X
constexpr uint32_t OFF_AF = 0;            // A (fp32)
constexpr uint32_t OFF_XF = 64 * kLD * 4;  // X = (I + A)^{-1} (fp32)
constexpr uint32_t OFF_PT = 34816;        // [P 8K | T 8K] fp16, K-major, K = 64
// fp16 operands:
constexpr uint32_t OFF_QW = 98304;        // [Qs ; W] fp16, 2 K-blocks x 16 KB (128 rows)
constexpr uint32_t kQWBlk = 16384;
constexpr uint32_t OFF_KS = 131072;       // [Ks | V] fp16 [token][col]: 3 blocks x 8 KB of 64
                                          // cols (Ks channels 0-63, 64-127, then V's 32 cols)
constexpr uint32_t kTokBlk = 8192;
constexpr uint32_t OFF_V16 = OFF_KS + 2 * kTokBlk;
constexpr uint32_t OFF_KB = 155648;       // Kb fp16 [token][channel], 2 blocks x 8 KB
constexpr uint32_t OFF_S16 = 172032;      // S fp16, 128 K-rows x 32, SW64 MN
constexpr uint32_t OFF_U16 = 180224;      // U fp16, 64 K-rows x 32, SW64 MN
constexpr uint32_t OFF_VEC = 184320;      // gam[128] beta[64] psum[4][128]
constexpr uint32_t OFF_BAR = OFF_VEC + (128 + 64 + 4 * 128) * 4;
constexpr uint32_t kSmemBytes = OFF_BAR + 64 + 1024;  // + alignment slack

// TMEM columns (512 allocated).
constexpr uint32_t COL_AP = 0;     // [KE;QE](KF)^T: lanes 0-63 A part, 64-127 P part (64 cols)
constexpr uint32_t COL_W = 64;     // [P;T][Ks|V]: lanes 64-127 = [W | U'] (128 + 32 cols)
constexpr uint32_t COL_UP = COL_W + 128;
constexpr uint32_t COL_X = 224;    // [Qs;W]S (+ [P;T]U): lanes 0-63 = O (32 cols)
constexpr uint32_t COL_S = 256;    // Kb^T U (32 cols)
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t IDESC_AP = tc::idesc(tc::kFmtTF32, 128, 64, 0, 0);
constexpr uint32_t IDESC_W = tc::idesc(tc::kFmtF16, 128, 128 + kNV, 0, 1);
constexpr uint32_t IDESC_NV_KB = tc::idesc(tc::kFmtF16, 128, kNV, 0, 1);  // A K-major, B MN-major
constexpr uint32_t IDESC_NV_MB = tc::idesc(tc::kFmtF16, 128, kNV, 1, 1);  // A MN-major, B MN-major

#ifdef KDA_PHASE_TIMING
// Debug builds only: cycles spent per phase by CTA 0, summed over chunks.
__device__ unsigned long long g_phase_cycles[16];
#define PHASE_MARK(idx)                                                    \
    do {                                                                   \
        if (blockIdx.x == 0 && threadIdx.x == 0) {                         \
            const unsigned long long now_ = clock64();                     \
            g_phase_cycles[idx] += now_ - t_prev_;                         \
            t_prev_ = now_;                                                \
        }                                                                  \
    } while (0)
#else
#define PHASE_MARK(idx) \
    do {                \
    } while (0)
#endif

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, int *abort, int *err) {
    if (*reinterpret_cast<volatile int *>(abort)) return false;
    if (tc::mbar_wait(bar, parity, kWaitLimit)) return true;
    *reinterpret_cast<volatile int *>(abort) = 1;
    atomicExch(err, 1);
    return false;
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_v,
                const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                const __nv_bfloat16 *__restrict__ v, const float *__restrict__ log_alpha,
                const float *__restrict__ beta, const float *__restrict__ S0,
                __nv_bfloat16 *__restrict__ out, float *__restrict__ S_T, int T, int H, int *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    float *gam = reinterpret_cast<float *>(sm + OFF_VEC);
    float *beta_s = gam + 128;
    float *psum = beta_s + 64;
    float *Af = reinterpret_cast<float *>(sm + OFF_AF);
    float *Xf = reinterpret_cast<float *>(sm + OFF_XF);
    uint64_t *bar_mma = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *bar_pu = bar_mma + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_mma + 2);
    int *abort = reinterpret_cast<int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int row = 32 * quad + lane;  // TMEM lane this thread reads
    constexpr int kSlices = kD / kNV;
    const int bh = blockIdx.x / kSlices, slice = blockIdx.x - bh * kSlices;
    const int b = bh / H, h = bh - b * H;
    const int n0 = slice * kNV;
    const int nchunks = (T + kC - 1) / kC;
    const long ztok = static_cast<long>(b) * T;  // row of (b, t = 0) in the [B*T] token dimension

    if (tid == 0) {
        tc::mbar_init(bar_mma, 1);
        tc::mbar_init(bar_pu, 1);
        *abort = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tm_q);
        tc::tma_prefetch_desc(&tm_k);
        tc::tma_prefetch_desc(&tm_la);
        tc::tma_prefetch_desc(&tm_v);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    // fp32 state slice in registers: row (key channel) `row`, columns half*16 .. +16
    float S[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
        S[j] = S0 ? S0[(static_cast<long>(bh) * kD + row) * kD + n0 + half * 16 + j] : 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t ph_mma = 0, ph_pu = 0;
    // Shared-memory descriptors of the fixed operand buffers; a K step adds its
    // byte offset / 16 to the start-address field.
    const uint64_t d_kqt = tc::smem_desc(sbase + OFF_KQT, 16, 1024, tc::kSwizzle128);
    const uint64_t d_kht = tc::smem_desc(sbase + OFF_KHT, 16, 1024, tc::kSwizzle128);
    const uint64_t d_pt = tc::smem_desc(sbase + OFF_PT, 16, 1024, tc::kSwizzle128);
    const uint64_t d_ksv = tc::smem_desc(sbase + OFF_KS, kTokBlk, 1024, tc::kSwizzle128);
    const uint64_t d_qw = tc::smem_desc(sbase + OFF_QW, 16, 1024, tc::kSwizzle128);
    const uint64_t d_s16 = tc::smem_desc(sbase + OFF_S16, 8192, 512, tc::kSwizzle64);
    const uint64_t d_kb = tc::smem_desc(sbase + OFF_KB, kTokBlk, 1024, tc::kSwizzle128);
    const uint64_t d_u16 = tc::smem_desc(sbase + OFF_U16, 4096, 512, tc::kSwizzle64);
#ifdef KDA_PHASE_TIMING
    unsigned long long t_prev_ = clock64();
#endif

    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * kC;
        const int valid = min(kC, T - t0);
        const long trow0 = ztok + t0;  // token row of the chunk's first token
        if (tid == 0 && c + 1 < nchunks) {
            const int z = static_cast<int>(trow0 + kC);
            tc::tma_prefetch_l2_3d(&tm_q, 0, h, z);
            tc::tma_prefetch_l2_3d(&tm_k, 0, h, z);
            tc::tma_prefetch_l2_3d(&tm_la, 0, h, z);
            tc::tma_prefetch_l2_3d(&tm_v, n0, h, z);
        }

        // ---------------------------------------------------------- P1: gates and operands
        if (tid < kC) beta_s[tid] = tid < valid ? beta[(trow0 + tid) * H + h] : 0.f;
        {   // V slice -> fp16 operand (tokens past T are zero)
            const int t = tid >> 2, piece = tid & 3;
            uint4 w = make_uint4(0, 0, 0, 0);
            if (t < valid) {
                const uint4 x = *reinterpret_cast<const uint4 *>(
                    v + ((trow0 + t) * H + h) * kD + n0 + 8 * piece);
                w.x = pack_f16(tc::bf16_lo(x.x), tc::bf16_hi(x.x));
                w.y = pack_f16(tc::bf16_lo(x.y), tc::bf16_hi(x.y));
                w.z = pack_f16(tc::bf16_lo(x.z), tc::bf16_hi(x.z));
                w.w = pack_f16(tc::bf16_lo(x.w), tc::bf16_hi(x.w));
            }
            *reinterpret_cast<uint4 *>(sm + OFF_V16 + sw128k_off(t, 8 * piece, 0)) = w;
        }
        const int p = tid & 63, qq = tid >> 6;  // channels 2p, 2p+1; tokens 16qq .. 16qq+15
        float2 lg[16];
        uint32_t qv[16], kv[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int t = 16 * qq + u;
            const long o = ((trow0 + t) * H + h) * kD + 2 * p;
            const bool ok = t < valid;
            lg[u] = ok ? *reinterpret_cast<const float2 *>(log_alpha + o) : make_float2(0.f, 0.f);
            qv[u] = ok ? *reinterpret_cast<const uint32_t *>(q + o) : 0u;
            kv[u] = ok ? *reinterpret_cast<const uint32_t *>(k + o) : 0u;
        }
        {
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) { s0 += lg[u].x; s1 += lg[u].y; }
            psum[qq * 128 + 2 * p] = s0;
            psum[qq * 128 + 2 * p + 1] = s1;
        }
        __syncthreads();
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
                gam[2 * p] = expf(tot0);
                gam[2 * p + 1] = expf(tot1);
            }
            // Running prefix in log2 units relative to the anchor: d = (g - g_a) * log2(e).
            constexpr float kLog2e = 1.4426950408889634f;
            float d0 = (pre0 - ga0) * kLog2e, d1 = (pre1 - ga1) * kLog2e;
            // Byte offsets of this thread's channel pair; rows 16qq + u have
            // (row >> 3) = 2qq + (u >> 3) and (row & 7) = u & 7.
            const uint32_t c = 2 * p;
            const uint32_t rowq = qq * 2048u;
            const uint32_t b32 = (c & 3u) * 4u + rowq;  // tf32 tiles
            const uint32_t ch32 = (c & 31u) >> 2, kb32 = c >> 5;
            const uint32_t b16 = (c & 7u) * 2u + rowq;                      // fp16 tiles
            const uint32_t ch16 = (c & 63u) >> 3, kb16 = c >> 6;
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
                *reinterpret_cast<float2 *>(sm + OFF_KQT + kb32 * kKQTBlk + o32) = make_float2(ke0, ke1);
                *reinterpret_cast<float2 *>(sm + OFF_KQT + kb32 * kKQTBlk + 8192 + o32) =
                    make_float2(qe0, qe1);
                *reinterpret_cast<float2 *>(sm + OFF_KHT + kb32 * kKHTBlk + o32) = make_float2(kf0, kf1);
                *reinterpret_cast<uint32_t *>(sm + OFF_QW + kb16 * kQWBlk + o16) =
                    pack_f16(qe0 * ea0, qe1 * ea1);
                *reinterpret_cast<uint32_t *>(sm + OFF_KS + kb16 * kTokBlk + o16) =
                    pack_f16(ke0 * ea0, ke1 * ea1);
                *reinterpret_cast<uint32_t *>(sm + OFF_KB + kb16 * kTokBlk + o16) =
                    pack_f16(kf0 * eca0, kf1 * eca1);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        PHASE_MARK(0);

        // ---------------------------------------------------------- M1: [A;P] (tf32)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 16; ++kk)
                mma_tf32(tmem + COL_AP, d_kqt + (((kk >> 2) * kKQTBlk + (kk & 3) * 32) >> 4),
                         d_kht + (((kk >> 2) * kKHTBlk + (kk & 3) * 32) >> 4), IDESC_AP, kk > 0);
            tc::mma_commit(bar_mma);
        }
        wait_bar(bar_mma, ph_mma, abort, err);
        ph_mma ^= 1;
        tc_fence_after();
        PHASE_MARK(1);

        // ---------------------------------------------------------- P2: A (fp32), P (fp16), T
        {
            float vv[32];
            const uint32_t ta = tc::tmem_addr(tmem, 32 * quad, COL_AP + half * 32);
            tc::tmem_ld16(ta, *reinterpret_cast<float(*)[16]>(vv));
            tc::tmem_ld16(ta + 16, *reinterpret_cast<float(*)[16]>(vv + 16));
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
                    *reinterpret_cast<uint32_t *>(sm + OFF_PT + sw128k_off(i, j, 0)) = pack_f16(lo, hi);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        PHASE_MARK(2);
        ut::unit_lower_inverse(Af, Xf, tid);
        PHASE_MARK(3);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = tid + u * kThreads;  // pair index 0..2047
            const int i = e >> 5, j = (e & 31) * 2;
            const float lo = j <= i ? Xf[i * kLD + j] * beta_s[j] : 0.f;
            const float hi = j + 1 <= i ? Xf[i * kLD + j + 1] * beta_s[j + 1] : 0.f;
            *reinterpret_cast<uint32_t *>(sm + OFF_PT + 8192 + sw128k_off(i, j, 0)) = pack_f16(lo, hi);
        }
        fence_proxy_async_smem();
        __syncthreads();
        PHASE_MARK(4);

        // ---------------------------------------------------------- M2: W = T Ks, U' = T V
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + COL_W, d_pt + ((kk * 32) >> 4), d_ksv + ((kk * 2048) >> 4), IDESC_W, kk > 0);
            tc::mma_commit(bar_mma);
        }
        wait_bar(bar_mma, ph_mma, abort, err);
        ph_mma ^= 1;
        tc_fence_after();
        PHASE_MARK(5);

        // ---------------------------------------------------------- P3: W -> fp16; S -> fp16
        if (quad >= 2) {
            const int i = row - 64;
            float w[4][16];
#pragma unroll
            for (int part = 0; part < 4; ++part)
                tc::tmem_ld16(tc::tmem_addr(tmem, 32 * quad, COL_W + half * 64 + part * 16), w[part]);
            tc::tmem_wait_ld();
#pragma unroll
            for (int part = 0; part < 4; ++part) {
#pragma unroll
                for (int u = 0; u < 16; u += 8) {
                    const int ch = half * 64 + part * 16 + u;
                    uint4 x;
                    x.x = pack_f16(w[part][u], w[part][u + 1]);
                    x.y = pack_f16(w[part][u + 2], w[part][u + 3]);
                    x.z = pack_f16(w[part][u + 4], w[part][u + 5]);
                    x.w = pack_f16(w[part][u + 6], w[part][u + 7]);
                    *reinterpret_cast<uint4 *>(sm + OFF_QW + sw128k_off(64 + i, ch, kQWBlk)) = x;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 16; u += 8) {
            uint4 w;
            w.x = pack_f16(S[u], S[u + 1]);
            w.y = pack_f16(S[u + 2], S[u + 3]);
            w.z = pack_f16(S[u + 4], S[u + 5]);
            w.w = pack_f16(S[u + 6], S[u + 7]);
            *reinterpret_cast<uint4 *>(sm + OFF_S16 + sw64mn_off(row, half * 16 + u)) = w;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        PHASE_MARK(6);

        // ---------------------------------------------------------- C1: [Qs;W] S
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_f16(tmem + COL_X, d_qw + (((kk >> 2) * kQWBlk + (kk & 3) * 32) >> 4),
                        d_s16 + ((kk * 1024) >> 4), IDESC_NV_KB, kk > 0);
            tc::mma_commit(bar_mma);
        }
        wait_bar(bar_mma, ph_mma, abort, err);
        ph_mma ^= 1;
        tc_fence_after();
        PHASE_MARK(7);

        // ---------------------------------------------------------- C2: U = U' - W S
        if (quad >= 2) {
            const int i = row - 64;
            float x[16], up[16];
            tc::tmem_ld16(tc::tmem_addr(tmem, 32 * quad, COL_X + half * 16), x);
            tc::tmem_ld16(tc::tmem_addr(tmem, 32 * quad, COL_UP + half * 16), up);
            tc::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; u += 8) {
                uint4 w;
                w.x = pack_f16(up[u] - x[u], up[u + 1] - x[u + 1]);
                w.y = pack_f16(up[u + 2] - x[u + 2], up[u + 3] - x[u + 3]);
                w.z = pack_f16(up[u + 4] - x[u + 4], up[u + 5] - x[u + 5]);
                w.w = pack_f16(up[u + 6] - x[u + 6], up[u + 7] - x[u + 7]);
                *reinterpret_cast<uint4 *>(sm + OFF_U16 + sw64mn_off(i, half * 16 + u)) = w;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        PHASE_MARK(8);

        // ---------------------------------------------------------- C3: Kb^T U ; O += P U
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + COL_S, d_kb + ((kk * 2048) >> 4), d_u16 + ((kk * 1024) >> 4), IDESC_NV_MB,
                        kk > 0);
            tc::mma_commit(bar_mma);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_f16(tmem + COL_X, d_pt + ((kk * 32) >> 4), d_u16 + ((kk * 1024) >> 4), IDESC_NV_KB, 1);
            tc::mma_commit(bar_pu);
        }
        wait_bar(bar_mma, ph_mma, abort, err);
        ph_mma ^= 1;
        tc_fence_after();
        PHASE_MARK(9);

        // ---------------------------------------------------------- C4: state update, output
        {
            float sv[16];
            tc::tmem_ld16(tc::tmem_addr(tmem, 32 * quad, COL_S + half * 16), sv);
            tc::tmem_wait_ld();
            const float gm = gam[row];
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = fmaf(gm, S[j], sv[j]);
            wait_bar(bar_pu, ph_pu, abort, err);
            ph_pu ^= 1;
            tc_fence_after();
            float o[16];
            if (quad < 2) {
                tc::tmem_ld16(tc::tmem_addr(tmem, 32 * quad, COL_X + half * 16), o);
                tc::tmem_wait_ld();
            }
            if (quad < 2 && row < valid) {
                uint4 w0, w1;
                w0.x = pack_bf16(o[0], o[1]);   w0.y = pack_bf16(o[2], o[3]);
                w0.z = pack_bf16(o[4], o[5]);   w0.w = pack_bf16(o[6], o[7]);
                w1.x = pack_bf16(o[8], o[9]);   w1.y = pack_bf16(o[10], o[11]);
                w1.z = pack_bf16(o[12], o[13]); w1.w = pack_bf16(o[14], o[15]);
                uint4 *dst = reinterpret_cast<uint4 *>(out + ((trow0 + row) * H + h) * kD + n0 + half * 16);
                dst[0] = w0;
                dst[1] = w1;
            }
        }
        tc_fence_before();
        __syncthreads();
        PHASE_MARK(10);
    }

    if (S_T) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            S_T[(static_cast<long>(bh) * kD + row) * kD + n0 + half * 16 + j] = S[j];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 3-D map over a [B*T, H, inner] tensor: box (box_inner, 1, 64 tokens).
bool make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int esize, int inner,
              int H, long tokens, int box_inner, CUtensorMapSwizzle sw) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(tokens)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner) * esize,
                                   static_cast<cuuint64_t>(inner) * esize * H};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), 1, kC};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

#ifdef KDA_PHASE_TIMING
extern "C" int kda_debug_phase_cycles(unsigned long long *out16, int reset) {
    cudaError_t e = cudaMemcpyFromSymbol(out16, g_phase_cycles, sizeof(unsigned long long) * 16);
    if (reset) {
        unsigned long long z[16] = {0};
        cudaMemcpyToSymbol(g_phase_cycles, z, sizeof z);
    }
    return e == cudaSuccess ? 0 : -1;
}
#endif

bool chunk_tc_supported(int dk, int dv, int chunk, int dtype) {
    return dtype == KDA_BF16 && dk == kD && dv == kD && chunk == kC;
}

size_t chunk_tc_workspace_bytes(int, int, int) { return 0; }

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t s) {
    const long tokens = static_cast<long>(a.B) * a.T;
    CUtensorMap mq, mk, mla, mv;
    if (!make_map(&mq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, a.H, tokens, kD,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, a.H, tokens, kD,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mla, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kD, a.H, tokens, kD,
                  CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, a.H, tokens, kNV,
                  CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(a.B) * a.H * (kD / kNV));
    chunk_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(
        mq, mk, mla, mv, static_cast<const __nv_bfloat16 *>(a.q),
        static_cast<const __nv_bfloat16 *>(a.k), static_cast<const __nv_bfloat16 *>(a.v),
        a.log_alpha, a.beta, a.S0, static_cast<__nv_bfloat16 *>(a.out), a.S_T, a.T, a.H,
        a.device_error);
    return cudaGetLastError();
}

}  // namespace kda
