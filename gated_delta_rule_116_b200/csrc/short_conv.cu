// short_conv.cu -- the KDA layer's q/k/v prologue ahead of the prefill: ShortConv
// followed by Swish (Kimi Linear summary, es.news.hada.io/topic?id=31936, section
// "Configuracion del modelo Kimi Linear": each head's queries, keys and values pass
// through ShortConv and Swish). ShortConv is read as a causal depthwise convolution
// along the tokens of each sequence, one filter of W <= 4 taps per (head, channel):
//   y_t = swish(sum_{j<W} w[h][c][j] x_{t-j}),  swish(u) = u / (1 + e^{-u}),
// with x before a sequence's first token taken as zero.
//
// Bandwidth-bound: each thread owns 8 channels of one head-row and walks kTile
// consecutive tokens, keeping the W-1 previous inputs in registers, so every input
// is read once (plus a W-1 token halo per tile) and every output written once. The
// 32 lanes of a warp cover 256 consecutive channels of one token: 512 contiguous
// bytes per access for bf16.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kTile = 16;
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

// Token range [s, e) of packed sequence n, offsets clamped to [0, total].
__device__ __forceinline__ void seq_range(const int32_t *cu, int n, long total, long &s, long &e) {
    s = min(max(static_cast<long>(cu[n]), 0L), total);
    e = min(max(static_cast<long>(cu[n + 1]), s), total);
}

template <typename Tin, int W>
__global__ void __launch_bounds__(kThreadsSC)
short_conv_swish_kernel(const Tin *__restrict__ x, const float *__restrict__ w, Tin *__restrict__ y,
                        const int32_t *__restrict__ cu, int nseq, long total, int T, int H, int d) {
    const int groups = H * d / 8;   // 8-channel groups of one token's [H][d] row
    const long gid = static_cast<long>(blockIdx.x) * kThreadsSC + threadIdx.x;
    const int g = static_cast<int>(gid % groups);
    const long t0 = (gid / groups) * kTile;
    if (t0 >= total) return;
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
    for (int u = 0; u < kTile; ++u) {
        const long t = t0 + u;
        if (t >= total) break;
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
            if (t < s || t >= e) continue;   // outside every sequence
        }
        float cur[8], out[8];
        load8(x + t * row + 8 * g, cur);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            float a = tap[0][m] * cur[m];
#pragma unroll
            for (int j = 1; j < W; ++j) a = fmaf(tap[j][m], prev[j - 1][m], a);
            out[m] = a / (1.f + exp2f(-a * kLog2eSC));
        }
        store8(y + t * row + 8 * g, out);
#pragma unroll
        for (int j = W - 1; j >= 1; --j)
#pragma unroll
            for (int m = 0; m < 8; ++m) prev[j - 1][m] = j == 1 ? cur[m] : prev[j - 2][m];
    }
}

template <typename Tin>
cudaError_t launch_typed(const void *x, const float *w, void *y, const int32_t *cu, int nseq, long total,
                         int T, int H, int d, int W, cudaStream_t s) {
    const long threads = static_cast<long>(H) * d / 8 * ((total + kTile - 1) / kTile);
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
