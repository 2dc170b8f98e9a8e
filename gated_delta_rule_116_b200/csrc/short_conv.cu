// short_conv.cu -- the KDA layer's q/k/v prologue ahead of the prefill: ShortConv
// followed by Swish (Kimi Linear summary, es.news.hada.io/topic?id=31936, section
// "Configuracion del modelo Kimi Linear": each head's queries, keys and values pass
// through ShortConv and Swish). ShortConv is read as a causal depthwise convolution
// along the tokens of each sequence, one filter of W <= 4 taps per (head, channel):
//   y_t = swish(sum_{j<W} w[h][c][j] x_{t-j}),  swish(u) = u / (1 + e^{-u}),
// with x before a sequence's first token taken as zero. Computed in fp32, rounded once
// to the output type.
//
// Bandwidth-bound: each thread owns 8 channels of one head-row and walks kRun
// consecutive tokens, keeping the W-1 previous inputs in registers, so every input
// is read once (plus a W-1 token halo per run) and every output written once; its
// loads run kAhead tokens ahead of the arithmetic, so a thread keeps that many
// 16-byte loads in flight, and the grid is about one wave. The
// 32 lanes of a warp cover 256 consecutive channels of one token: 512 contiguous
// bytes per access for bf16.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kRun = 128;     // consecutive tokens per thread
// tokens loaded ahead of the arithmetic, a ring of packed registers (4 per token for bf16, 8 for fp32)
template <typename Tin> constexpr int ahead_of() { return sizeof(Tin) == 2 ? 8 : 4; }
constexpr int kThreadsSC = 256;
constexpr float kLog2eSC = 1.4426950408889634f;

__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&x)[8]) {
    const uint4 v = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        x[2 * m] = __uint_as_float(w[m] << 16);
        x[2 * m + 1] = __uint_as_float(w[m] & 0xffff0000u);
    }
}
__device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
    const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&x)[8]) {
    uint4 v;
    uint32_t *w = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * m], x[2 * m + 1]);
        w[m] = *reinterpret_cast<const uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(p) = v;
}
__device__ __forceinline__ void store8(float *p, const float (&x)[8]) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// A token's 8 channels as loaded (bf16: one 16-byte piece; fp32: two), widened when used.
template <typename Tin> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 v;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { v = *reinterpret_cast<const uint4 *>(p); }
    __device__ __forceinline__ float at(int m) const {
        const uint32_t word = (m >> 1) == 0 ? v.x : ((m >> 1) == 1 ? v.y : ((m >> 1) == 2 ? v.z : v.w));
        return (m & 1) ? __uint_as_float(word & 0xffff0000u) : __uint_as_float(word << 16);
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float *p) {
        a = reinterpret_cast<const float4 *>(p)[0];
        b = reinterpret_cast<const float4 *>(p)[1];
    }
    __device__ __forceinline__ float at(int m) const {
        const float4 &h = m < 4 ? a : b;
        const int r = m & 3;
        return r == 0 ? h.x : (r == 1 ? h.y : (r == 2 ? h.z : h.w));
    }
};

// Token range [s, e) of packed sequence n, offsets clamped to [0, total].
__device__ __forceinline__ void seq_range(const int32_t *cu, int n, long total, long &s, long &e) {
    s = min(max(static_cast<long>(cu[n]), 0L), total);
    e = min(max(static_cast<long>(cu[n + 1]), s), total);
}

// One thread: 8 channels (group g) of a run of kRun consecutive tokens starting at t0,
// loads kept kAhead tokens ahead of the arithmetic in a register ring.
template <typename Tin, int W>
__global__ void __launch_bounds__(kThreadsSC, 2)
short_conv_swish_kernel(const Tin *__restrict__ x, const float *__restrict__ w, Tin *__restrict__ y,
                        const int32_t *__restrict__ cu, int nseq, long total, int T, int H, int d) {
    constexpr int kAhead = ahead_of<Tin>();
    const int groups = H * d / 8;   // 8-channel groups of one token's [H][d] row
    const long gid = static_cast<long>(blockIdx.x) * kThreadsSC + threadIdx.x;
    const int g = static_cast<int>(gid % groups);
    const long t0 = (gid / groups) * kRun;
    if (t0 >= total) return;
    const long t1 = min(t0 + kRun, total);
    const int h = (8 * g) / d, c0 = (8 * g) % d;
    const long row = static_cast<long>(H) * d;   // elements per token
    float tap[W][8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
        for (int j = 0; j < W; ++j) tap[j][e] = w[(static_cast<long>(h) * d + c0 + e) * W + j];
    // the sequence holding t0: a dense batch row of T tokens, or the last packed sequence
    // starting at or before t0 (tokens outside every sequence are left untouched)
    long s, e;
    int n = 0;
    if (cu) {
        int lo = 0, hi = nseq - 1;   // largest n in [0, nseq) with start(n) <= t0 (nseq >= 1)
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (min(max(static_cast<long>(cu[mid]), 0L), total) <= t0) lo = mid;
            else hi = mid - 1;
        }
        n = lo;
        seq_range(cu, n, total, s, e);
    } else {
        s = (t0 / T) * T;
        e = s + T;
    }
    float prev[W > 1 ? W - 1 : 1][8];   // prev[j - 1] = x_{t - j}
#pragma unroll
    for (int j = 1; j < W; ++j) {
        if (t0 - j >= s && t0 < e) load8(x + (t0 - j) * row + 8 * g, prev[j - 1]);
        else
#pragma unroll
            for (int m = 0; m < 8; ++m) prev[j - 1][m] = 0.f;
    }
    Raw8<Tin> ring[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u)
        if (t0 + u < t1) ring[u].load(x + (t0 + u) * row + 8 * g);
    for (long tb = t0; tb < t1; tb += kAhead) {
#pragma unroll
        for (int u = 0; u < kAhead; ++u) {
            const long t = tb + u;
            if (t >= t1) continue;
            float cur[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) cur[m] = ring[u].at(m);
            if (t + kAhead < t1) ring[u].load(x + (t + kAhead) * row + 8 * g);   // refill the slot
            if (t >= e || t < s) {   // into the next sequence: its first tokens see zeros before them
                if (cu) {
                    while (n + 1 < nseq && t >= e) {
                        ++n;
                        seq_range(cu, n, total, s, e);
                    }
                } else {
                    s = (t / T) * T;
                    e = s + T;
                }
#pragma unroll
                for (int j = 1; j < W; ++j)
#pragma unroll
                    for (int m = 0; m < 8; ++m) prev[j - 1][m] = 0.f;
            }
            if (t < s || t >= e) continue;   // outside every sequence
            float out[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                float a = tap[0][m] * cur[m];
#pragma unroll
                for (int j = 1; j < W; ++j) a = fmaf(tap[j][m], prev[j - 1][m], a);
                // swish(a) = a / (1 + e^{-a}): hardware exp2 and a fast divide (relative error
                // about 2^-21, far below the output's rounding; e^{-a} = inf for a << 0 gives 0)
                out[m] = __fdividef(a, 1.f + ex2_approx(-a * kLog2eSC));
            }
            store8(y + t * row + 8 * g, out);
#pragma unroll
            for (int j = W - 1; j >= 1; --j)
#pragma unroll
                for (int m = 0; m < 8; ++m) prev[j - 1][m] = j == 1 ? cur[m] : prev[j - 2][m];
        }
    }
}

template <typename Tin>
cudaError_t launch_typed(const void *x, const float *w, void *y, const int32_t *cu, int nseq, long total,
                         int T, int H, int d, int W, cudaStream_t s) {
    const long threads = static_cast<long>(H) * d / 8 * ((total + kRun - 1) / kRun);
    const unsigned blocks = static_cast<unsigned>((threads + kThreadsSC - 1) / kThreadsSC);
    const Tin *xi = static_cast<const Tin *>(x);
    Tin *yo = static_cast<Tin *>(y);
    switch (W) {
        case 1: short_conv_swish_kernel<Tin, 1><<<blocks, kThreadsSC, 0, s>>>(xi, w, yo, cu, nseq, total, T, H, d); break;
        case 2: short_conv_swish_kernel<Tin, 2><<<blocks, kThreadsSC, 0, s>>>(xi, w, yo, cu, nseq, total, T, H, d); break;
        case 3: short_conv_swish_kernel<Tin, 3><<<blocks, kThreadsSC, 0, s>>>(xi, w, yo, cu, nseq, total, T, H, d); break;
        default: short_conv_swish_kernel<Tin, 4><<<blocks, kThreadsSC, 0, s>>>(xi, w, yo, cu, nseq, total, T, H, d); break;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_short_conv_swish(const void *x, const float *w, void *y, const int32_t *cu_seqlens,
                                    int B, int T, int H, int d, int W, int dtype, cudaStream_t s) {
    // dense: B rows of T tokens; packed (cu_seqlens): B sequences over T tokens in all
    const long total = cu_seqlens ? static_cast<long>(T) : static_cast<long>(B) * T;
    if (total == 0) return cudaSuccess;
    return dtype == KDA_BF16 ? launch_typed<__nv_bfloat16>(x, w, y, cu_seqlens, B, total, T, H, d, W, s)
                             : launch_typed<float>(x, w, y, cu_seqlens, B, total, T, H, d, W, s);
}

}  // namespace kda
