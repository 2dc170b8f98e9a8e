// chunk_generic.cu -- fp32 CUDA-core engine of the chunked KDA prefill.
//
// Serves every shape the tensor-core engine does not (fp32 inputs, any
// d_k, d_v <= 128, chunk 16/32/64) and computes entirely in fp32.
//
// Chunked form (Kimi Linear summary, es.news.hada.io/topic?id=31936, section
// "Algoritmo paralelo por chunks"). For one chunk of C tokens starting from
// state S (d_k x d_v), with g_t the in-chunk inclusive prefix sum of log alpha
// (per channel):
//   A  = Diag(beta) * strict_lower(a_ij),  a_ij = sum_c k_ic k_jc e^{g_ic - g_jc}
//   P  = lower(p_ij),                      p_ij = sum_c q_ic k_jc e^{g_ic - g_jc}
//   T  = (I + A)^{-1} Diag(beta)                      (forward substitution)
//   W  = T Ks,  U' = T V                              (WY / UT form, Ks = K e^{g})
//   U  = U' - W S
//   O  = Qs S + P U                                   (Qs = Q e^{g})
//   S <- Diag(e^{g_C}) S + Kb^T U                     (Kb = K e^{g_C - g})
// In exact arithmetic this equals the token-by-token recurrence. The entries
// of A and P take e^{g_i - g_j} <= 1 per term, evaluated directly for every
// pair j <= i: no factor is split, so no decay, however fine-grained (section
// "Menor cantidad de operaciones que DPLR general"), leaves the fp32 range.
// Every other factor (e^{g}, e^{g_C - g}, e^{g_C}) is <= 1 as well.
//
// Mapping: one CTA of 256 threads per (b, h, slice of NV <= 32 value
// columns). State columns evolve independently, so slices never communicate;
// each recomputes the d_k-side work (A, P, T, W) of its chunk.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxNV = 32;

struct Smem {
    int C, dk, NV, LD, LC;
    __host__ __device__ Smem(int C_, int dk_, int NV_)
        : C(C_), dk(dk_), NV(NV_), LD(dk_ + 1), LC(C_ + 1) {}
    __host__ __device__ size_t floats() const {
        return 4ull * C * LD + 3ull * C * LC + 2ull * C * NV + 1ull * dk * NV + 2ull * dk + C;
    }
};

template <typename Tin>
__global__ void __launch_bounds__(kThreads, 1)
chunk_generic_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                     const Tin *__restrict__ v, const float *__restrict__ log_alpha,
                     const float *__restrict__ beta, const float *__restrict__ S0,
                     Tin *__restrict__ out, float *__restrict__ S_T, int T, int H, int dk, int dv,
                     int C, int NV) {
    extern __shared__ float sm[];
    const Smem L(C, dk, NV);
    const int LD = L.LD, LC = L.LC;
    float *Qt = sm;                 // [C][LD]  q, then Qs = q e^{g}
    float *Kt = Qt + C * LD;        // [C][LD]  k, then Ks = k e^{g}
    float *Kh = Kt + C * LD;        // [C][LD]  Kb = k e^{g_C - g}
    float *G = Kh + C * LD;         // [C][LD]  prefix sums g, then W
    float *A = G + C * LD;          // [C][LC]
    float *Tm = A + C * LC;         // [C][LC]
    float *P = Tm + C * LC;         // [C][LC]
    float *V = P + C * LC;          // [C][NV]
    float *U = V + C * NV;          // [C][NV]
    float *S = U + C * NV;          // [dk][NV]
    float *e_c = S + dk * NV;       // [dk] e^{g_C}
    float *gsum = e_c + dk;         // [dk] g_C
    float *bt = gsum + dk;          // [C]  beta of the chunk
    const int tid = threadIdx.x;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh - (bh / H) * H;
    const int n0 = blockIdx.y * NV;
    const int nv = min(NV, dv - n0);

    for (int e = tid; e < dk * NV; e += kThreads) {
        const int c = e / NV, n = e - c * NV;
        float s = 0.f;
        if (S0 && n < nv) s = S0[(static_cast<long>(bh) * dk + c) * dv + n0 + n];
        S[e] = s;
    }

    const int nchunks = (T + C - 1) / C;
    for (int ch = 0; ch < nchunks; ++ch) {
        const int t0 = ch * C;
        const int valid = min(C, T - t0);
        __syncthreads();
        // 1. load the chunk; tokens past T are identity steps (k = v = q = 0, beta = 0, log a = 0)
        for (int e = tid; e < C * dk; e += kThreads) {
            const int t = e / dk, c = e - t * dk;
            float qv = 0.f, kv = 0.f, gv = 0.f;
            if (t < valid) {
                const long o = ((static_cast<long>(b) * T + t0 + t) * H + h) * dk + c;
                qv = to_f32(q[o]);
                kv = to_f32(k[o]);
                gv = log_alpha[o];
            }
            Qt[t * LD + c] = qv;
            Kt[t * LD + c] = kv;
            G[t * LD + c] = gv;
        }
        for (int e = tid; e < C * NV; e += kThreads) {
            const int t = e / NV, n = e - t * NV;
            float vv = 0.f;
            if (t < valid && n < nv)
                vv = to_f32(v[((static_cast<long>(b) * T + t0 + t) * H + h) * dv + n0 + n]);
            V[e] = vv;
        }
        for (int t = tid; t < C; t += kThreads)
            bt[t] = t < valid ? beta[(static_cast<long>(b) * T + t0 + t) * H + h] : 0.f;
        __syncthreads();
        // 2. in-chunk prefix sum of log alpha per channel
        for (int c = tid; c < dk; c += kThreads) {
            float acc = 0.f;
            for (int t = 0; t < C; ++t) {
                acc += G[t * LD + c];
                G[t * LD + c] = acc;
            }
            gsum[c] = acc;
            e_c[c] = expf(acc);
        }
        __syncthreads();
        // 3. A = Diag(beta) strict_lower(a), P = lower(p), every term with its own e^{g_i - g_j}
        for (int e = tid; e < C * C; e += kThreads) {
            const int i = e / C, j = e - i * C;
            float a = 0.f, p = 0.f;
            if (j <= i) {
                const float *qi = Qt + i * LD, *ki = Kt + i * LD, *kj = Kt + j * LD;
                const float *gi = G + i * LD, *gj = G + j * LD;
                for (int c = 0; c < dk; ++c) {
                    const float kd = kj[c] * expf(gi[c] - gj[c]);
                    p = fmaf(qi[c], kd, p);
                    a = fmaf(ki[c], kd, a);
                }
                a = j < i ? a * bt[i] : 0.f;
            }
            A[i * LC + j] = a;
            P[i * LC + j] = p;
        }
        __syncthreads();
        // 4. Qs = q e^{g}, Ks = k e^{g}, Kb = k e^{g_C - g}
        for (int e = tid; e < C * dk; e += kThreads) {
            const int t = e / dk, c = e - t * dk;
            const float gv = G[t * LD + c];
            const float up = expf(gv), down = expf(gsum[c] - gv);
            const float kv = Kt[t * LD + c];
            Qt[t * LD + c] *= up;
            Kt[t * LD + c] = kv * up;
            Kh[t * LD + c] = kv * down;
        }
        __syncthreads();
        // 5. T = (I + A)^{-1} Diag(beta), one column per thread, forward substitution
        for (int j = tid; j < C; j += kThreads) {
            for (int i = 0; i < j; ++i) Tm[i * LC + j] = 0.f;
            Tm[j * LC + j] = bt[j];
            for (int i = j + 1; i < C; ++i) {
                float s = 0.f;
                for (int m = j; m < i; ++m) s = fmaf(A[i * LC + m], Tm[m * LC + j], s);
                Tm[i * LC + j] = -s;
            }
        }
        __syncthreads();
        // 6. W = T Ks (into G), U' = T V
        for (int e = tid; e < C * dk; e += kThreads) {
            const int i = e / dk, c = e - i * dk;
            float w = 0.f;
            for (int j = 0; j <= i; ++j) w = fmaf(Tm[i * LC + j], Kt[j * LD + c], w);
            G[i * LD + c] = w;
        }
        for (int e = tid; e < C * NV; e += kThreads) {
            const int i = e / NV, n = e - i * NV;
            float u = 0.f;
            for (int j = 0; j <= i; ++j) u = fmaf(Tm[i * LC + j], V[j * NV + n], u);
            U[e] = u;
        }
        __syncthreads();
        // 7. U = U' - W S
        for (int e = tid; e < C * NV; e += kThreads) {
            const int i = e / NV, n = e - i * NV;
            float u = U[e];
            for (int c = 0; c < dk; ++c) u = fmaf(-G[i * LD + c], S[c * NV + n], u);
            U[e] = u;
        }
        __syncthreads();
        // 8. O = Qs S + P U
        for (int e = tid; e < C * NV; e += kThreads) {
            const int i = e / NV, n = e - i * NV;
            if (i < valid && n < nv) {
                float o = 0.f;
                for (int c = 0; c < dk; ++c) o = fmaf(Qt[i * LD + c], S[c * NV + n], o);
                for (int j = 0; j <= i; ++j) o = fmaf(P[i * LC + j], U[j * NV + n], o);
                out[((static_cast<long>(b) * T + t0 + i) * H + h) * dv + n0 + n] = from_f32<Tin>(o);
            }
        }
        __syncthreads();
        // 9. S = Diag(e^{g_C}) S + Kb^T U
        for (int e = tid; e < dk * NV; e += kThreads) {
            const int c = e / NV, n = e - c * NV;
            float s = S[e] * e_c[c];
            for (int t = 0; t < C; ++t) s = fmaf(Kh[t * LD + c], U[t * NV + n], s);
            S[e] = s;
        }
    }
    __syncthreads();
    if (S_T) {
        for (int e = tid; e < dk * NV; e += kThreads) {
            const int c = e / NV, n = e - c * NV;
            if (n < nv) S_T[(static_cast<long>(bh) * dk + c) * dv + n0 + n] = S[e];
        }
    }
}

template <typename Tin>
cudaError_t launch_typed(const ChunkArgs &a, cudaStream_t s) {
    const int NV = a.dv < kMaxNV ? a.dv : kMaxNV;
    const Smem L(a.chunk, a.dk, NV);
    const size_t bytes = L.floats() * sizeof(float);
    auto kern = chunk_generic_kernel<Tin>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(bytes));
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(a.B) * static_cast<unsigned>(a.H),
                    static_cast<unsigned>((a.dv + NV - 1) / NV));
    kern<<<grid, kThreads, bytes, s>>>(static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k),
                                       static_cast<const Tin *>(a.v), a.log_alpha, a.beta, a.S0,
                                       static_cast<Tin *>(a.out), a.S_T, a.T, a.H, a.dk, a.dv,
                                       a.chunk, NV);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_generic(const ChunkArgs &a, cudaStream_t s) {
    return a.dtype == KDA_BF16 ? launch_typed<__nv_bfloat16>(a, s) : launch_typed<float>(a, s);
}

}  // namespace kda
