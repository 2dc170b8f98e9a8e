// decode.cu -- single-token KDA decode against an fp32 state cache (in place).
//
// Per (sequence n, head h) one step of the recurrence (Kimi Linear summary,
// es.news.hada.io/topic?id=31936, sections "De la atencion lineal a Gated
// DeltaNet" and "Control fino de memoria en Kimi Delta Attention"):
//     S' = Diag(alpha) S,  r = S'^T k,  p = S'^T q,  u = beta (v - r),
//     S  = S' + k u^T,     o = S^T q = p + (k.q) u.
// The step is bound by HBM bandwidth: each 128 x 128 fp32 state (64 KiB) is
// read once and written once, everything else is < 2 KiB per head.
//
// Mapping, d_k = d_v = 128 (decode_half_kernel): one CTA of 256 threads per
// (n, h, half of the value columns); the columns of S evolve independently, so
// the halves need no exchange. Thread (warp w, lane l) owns float4 column
// l % 16 of its half in rows g, g+16, ..., g+112 with g = 2w + l/16: 8 float4
// registers, so the CTA holds its 32 KiB of state in registers between the read
// and the write, and three CTAs share an SM (their read, reduce and write phases
// overlap). Each warp instruction touches two 256-byte row halves: fully
// coalesced 16-byte accesses. Other sizes (decode_kernel): one CTA per (n, h),
// thread (w, l) owns columns 4l..4l+3 of rows w, w+8, ..., w+120. Both
// dk-reductions are done in one pass: per-thread partial sums, then a
// cross-thread sum through shared memory.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerThread = 128 / kWarps;  // dk <= 128

__device__ __forceinline__ float4 ld_state(const float *p) {
    return __ldcs(reinterpret_cast<const float4 *>(p));
}
__device__ __forceinline__ void st_state(float *p, float4 x) {
    __stcs(reinterpret_cast<float4 *>(p), x);
}

template <typename Tin, bool kFull>
__global__ void __launch_bounds__(kThreads, 2)
decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              const float *__restrict__ log_alpha, const float *__restrict__ beta,
              float *__restrict__ state, const int32_t *__restrict__ slot, Tin *__restrict__ out,
              int H, int dk, int dv) {
    __shared__ float s_k[128], s_q[128], s_a[128];
    __shared__ float4 red_r[kWarps][32], red_p[kWarps][32];

    const int nh = blockIdx.x;
    const int n = nh / H;
    const int h = nh - n * H;
    const long srow = slot ? static_cast<long>(slot[n]) : static_cast<long>(n);
    float *S = state + (srow * H + h) * static_cast<long>(dk) * dv;

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int col = lane * 4;
    const bool col_ok = kFull || col < dv;

    // Issue all state loads first; the small per-head vectors overlap with them.
    float4 x[kRowsPerThread];
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) {
        const int row = warp + kWarps * r;
        if (col_ok && (kFull || row < dk))
            x[r] = ld_state(S + static_cast<long>(row) * dv + col);
        else
            x[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (tid < dk) {
        const long o = static_cast<long>(nh) * dk + tid;
        s_k[tid] = to_f32(k[o]);
        s_q[tid] = to_f32(q[o]);
        s_a[tid] = expf(log_alpha[o]);
    }
    __syncthreads();

    float4 pr = make_float4(0.f, 0.f, 0.f, 0.f), pp = pr;
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) {
        const int row = warp + kWarps * r;
        if (kFull || row < dk) {
            const float a = s_a[row], kr = s_k[row], qr = s_q[row];
            x[r].x *= a; x[r].y *= a; x[r].z *= a; x[r].w *= a;
            pr.x = fmaf(kr, x[r].x, pr.x); pr.y = fmaf(kr, x[r].y, pr.y);
            pr.z = fmaf(kr, x[r].z, pr.z); pr.w = fmaf(kr, x[r].w, pr.w);
            pp.x = fmaf(qr, x[r].x, pp.x); pp.y = fmaf(qr, x[r].y, pp.y);
            pp.z = fmaf(qr, x[r].z, pp.z); pp.w = fmaf(qr, x[r].w, pp.w);
        }
    }
    red_r[warp][lane] = pr;
    red_p[warp][lane] = pp;
    __syncthreads();

    float4 R = red_r[0][lane], P = red_p[0][lane];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
        const float4 a = red_r[w][lane], b = red_p[w][lane];
        R.x += a.x; R.y += a.y; R.z += a.z; R.w += a.w;
        P.x += b.x; P.y += b.y; P.z += b.z; P.w += b.w;
    }
    const float bt = beta[nh];
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
    if (col_ok) {
        const Tin *vp = v + static_cast<long>(nh) * dv + col;
        u.x = bt * (to_f32(vp[0]) - R.x);
        u.y = bt * (to_f32(vp[1]) - R.y);
        u.z = bt * (to_f32(vp[2]) - R.z);
        u.w = bt * (to_f32(vp[3]) - R.w);
    }
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) {
        const int row = warp + kWarps * r;
        if (col_ok && (kFull || row < dk)) {
            const float kr = s_k[row];
            x[r].x = fmaf(kr, u.x, x[r].x); x[r].y = fmaf(kr, u.y, x[r].y);
            x[r].z = fmaf(kr, u.z, x[r].z); x[r].w = fmaf(kr, u.w, x[r].w);
            st_state(S + static_cast<long>(row) * dv + col, x[r]);
        }
    }
    if (warp == 0) {
        float kq = 0.f;
        for (int i = lane; i < dk; i += 32) kq = fmaf(s_k[i], s_q[i], kq);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        if (col_ok) {
            Tin *op = out + static_cast<long>(nh) * dv + col;
            op[0] = from_f32<Tin>(fmaf(kq, u.x, P.x));
            op[1] = from_f32<Tin>(fmaf(kq, u.y, P.y));
            op[2] = from_f32<Tin>(fmaf(kq, u.z, P.z));
            op[3] = from_f32<Tin>(fmaf(kq, u.w, P.w));
        }
    }
}


// d_k = d_v = 128: one CTA per (n, h, half of the value columns); see the top.
template <typename Tin>
__global__ void __launch_bounds__(kThreads, 3)
decode_half_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                   const float *__restrict__ log_alpha, const float *__restrict__ beta,
                   float *__restrict__ state, const int32_t *__restrict__ slot, Tin *__restrict__ out,
                   int H) {
    __shared__ float s_k[128], s_q[128], s_a[128];
    __shared__ float4 red_r[16][16], red_p[16][16];
    const int nh = blockIdx.x >> 1, cb = blockIdx.x & 1;
    const int n = nh / H;
    const int h = nh - n * H;
    const long srow = slot ? static_cast<long>(slot[n]) : static_cast<long>(n);
    float *S = state + (srow * H + h) * 16384L + cb * 64;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c4 = lane & 15, g = 2 * warp + (lane >> 4);
    float4 x[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) x[r] = ld_state(S + (g + 16 * r) * 128 + 4 * c4);
    if (tid < 128) {
        const long o = static_cast<long>(nh) * 128 + tid;
        s_k[tid] = to_f32(k[o]);
        s_q[tid] = to_f32(q[o]);
        s_a[tid] = expf(log_alpha[o]);
    }
    __syncthreads();
    float4 pr = make_float4(0.f, 0.f, 0.f, 0.f), pp = pr;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int row = g + 16 * r;
        const float a = s_a[row], kr = s_k[row], qr = s_q[row];
        x[r].x *= a; x[r].y *= a; x[r].z *= a; x[r].w *= a;
        pr.x = fmaf(kr, x[r].x, pr.x); pr.y = fmaf(kr, x[r].y, pr.y);
        pr.z = fmaf(kr, x[r].z, pr.z); pr.w = fmaf(kr, x[r].w, pr.w);
        pp.x = fmaf(qr, x[r].x, pp.x); pp.y = fmaf(qr, x[r].y, pp.y);
        pp.z = fmaf(qr, x[r].z, pp.z); pp.w = fmaf(qr, x[r].w, pp.w);
    }
    red_r[g][c4] = pr;
    red_p[g][c4] = pp;
    __syncthreads();
    float4 R = red_r[0][c4], P = red_p[0][c4];
#pragma unroll
    for (int j = 1; j < 16; ++j) {
        const float4 a = red_r[j][c4], b = red_p[j][c4];
        R.x += a.x; R.y += a.y; R.z += a.z; R.w += a.w;
        P.x += b.x; P.y += b.y; P.z += b.z; P.w += b.w;
    }
    const float bt = beta[nh];
    const Tin *vp = v + static_cast<long>(nh) * 128 + cb * 64 + 4 * c4;
    float4 u;
    u.x = bt * (to_f32(vp[0]) - R.x);
    u.y = bt * (to_f32(vp[1]) - R.y);
    u.z = bt * (to_f32(vp[2]) - R.z);
    u.w = bt * (to_f32(vp[3]) - R.w);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int row = g + 16 * r;
        const float kr = s_k[row];
        x[r].x = fmaf(kr, u.x, x[r].x); x[r].y = fmaf(kr, u.y, x[r].y);
        x[r].z = fmaf(kr, u.z, x[r].z); x[r].w = fmaf(kr, u.w, x[r].w);
        st_state(S + row * 128 + 4 * c4, x[r]);
    }
    if (warp == 0) {
        float kq = fmaf(s_k[lane], s_q[lane], 0.f);
#pragma unroll
        for (int i = 1; i < 4; ++i) kq = fmaf(s_k[lane + 32 * i], s_q[lane + 32 * i], kq);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        if (lane < 16) {
            Tin *op = out + static_cast<long>(nh) * 128 + cb * 64 + 4 * c4;
            op[0] = from_f32<Tin>(fmaf(kq, u.x, P.x));
            op[1] = from_f32<Tin>(fmaf(kq, u.y, P.y));
            op[2] = from_f32<Tin>(fmaf(kq, u.z, P.z));
            op[3] = from_f32<Tin>(fmaf(kq, u.w, P.w));
        }
    }
}

template <typename Tin>
cudaError_t launch_typed(const DecodeArgs &a, cudaStream_t s) {
    const dim3 grid(static_cast<unsigned>(a.N) * static_cast<unsigned>(a.H));
    const bool full = a.dk == 128 && a.dv == 128;
    if (full) {
        decode_half_kernel<Tin><<<2 * grid.x, kThreads, 0, s>>>(
            static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k), static_cast<const Tin *>(a.v),
            a.log_alpha, a.beta, a.state, a.slot, static_cast<Tin *>(a.out), a.H);
        return cudaGetLastError();
    }
    auto kern = full ? decode_kernel<Tin, true> : decode_kernel<Tin, false>;
    kern<<<grid, kThreads, 0, s>>>(static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k),
                                   static_cast<const Tin *>(a.v), a.log_alpha, a.beta, a.state,
                                   a.slot, static_cast<Tin *>(a.out), a.H, a.dk, a.dv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
    if (a.N == 0 || a.H == 0) return cudaSuccess;
    return a.dtype == KDA_BF16 ? launch_typed<__nv_bfloat16>(a, s) : launch_typed<float>(a, s);
}

}  // namespace kda
