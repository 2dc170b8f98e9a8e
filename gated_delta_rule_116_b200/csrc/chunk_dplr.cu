// chunk_dplr.cu -- fp32 CUDA-core chunked engine of the general DPLR delta recurrence,
// the comparator of KDA's operator efficiency (Kimi Linear summary,
// es.news.hada.io/topic?id=31936, section "Menor cantidad de operaciones que DPLR
// general": KDA ties both low-rank vectors of the DPLR transition to the key, which
// takes the secondary-chunk products from 4 to 2 and removes 3 matrix products; its
// operator efficiency is about twice the general form's).
//
// Recurrence (per head, d_k x d_v state): S_t = (Diag(alpha_t) + a_t b_t^T) S_{t-1}
// + k_t v_t^T, o_t = S_t^T q_t. It is written like the fp32 KDA engine
// (chunk_generic.cu: same CTA mapping, same loops, same evaluation of every gate
// factor per term), so that timing the two measures the algorithms, not the code.
//
// Chunked form, for one chunk of C tokens from state S, with g the in-chunk inclusive
// prefix sum of log alpha and g^- = g - log alpha (exclusive): the probe u_t =
// b_t^T S_{t-1} of every token solves
//   (I - M_ba) U = Bs S + M_bk V,   Bs = b e^{g^-},
//   (M_ba)_ij = sum_c b_ic e^{g^-_ic - g_jc} a_jc,  (M_bk)_ij likewise with k  (j < i),
// and then
//   O = Qs S + M_qa U + M_qk V,     Qs = q e^{g}, (M_qa)_ij = sum_c q_ic e^{g_ic - g_jc} a_jc,
//                                    (M_qk)_ij likewise with k (j <= i),
//   S <- Diag(e^{g_C}) S + Ad^T U + Kd^T V,   Ad = a e^{g_C - g}, Kd = k e^{g_C - g}.
// Four secondary-chunk products (KDA: two) and, per chunk, the extra products M_bk V,
// M_qk V and Kd^T V (KDA folds them into one T [Ks | V] and one Kb^T U).
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
        return 5ull * C * LD + 5ull * C * LC + 3ull * C * NV + 1ull * dk * NV + 2ull * dk;
    }
};

template <typename Tin>
__global__ void __launch_bounds__(kThreads, 1)
chunk_dplr_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                  const Tin *__restrict__ av, const Tin *__restrict__ bv,
                  const float *__restrict__ log_alpha, const float *__restrict__ S0,
                  Tin *__restrict__ out, float *__restrict__ S_T, int T, int H, int dk, int dv,
                  int C, int NV) {
    extern __shared__ float sm[];
    const Smem L(C, dk, NV);
    const int LD = L.LD, LC = L.LC;
    float *Qt = sm;                 // [C][LD] q, then Qs = q e^{g}
    float *Kt = Qt + C * LD;        // [C][LD] k, then Kd = k e^{g_C - g}
    float *At = Kt + C * LD;        // [C][LD] a, then Ad = a e^{g_C - g}
    float *Bt = At + C * LD;        // [C][LD] b, then Bs = b e^{g^-}
    float *G = Bt + C * LD;         // [C][LD] prefix sums g
    float *Mba = G + C * LD;        // [C][LC]
    float *Mbk = Mba + C * LC;      // [C][LC]
    float *Mqa = Mbk + C * LC;      // [C][LC]
    float *Mqk = Mqa + C * LC;      // [C][LC]
    float *Tm = Mqk + C * LC;       // [C][LC] (I - M_ba)^{-1}
    float *V = Tm + C * LC;         // [C][NV]
    float *R = V + C * NV;          // [C][NV] Bs S + M_bk V
    float *U = R + C * NV;          // [C][NV] probes
    float *S = U + C * NV;          // [dk][NV]
    float *e_c = S + dk * NV;       // [dk] e^{g_C}
    float *gsum = e_c + dk;         // [dk] g_C
    const int tid = threadIdx.x;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh - (bh / H) * H;
    const int n0 = blockIdx.y * NV;
    const int nv = min(NV, dv - n0);

    for (int e = tid; e < dk * NV; e += kThreads) {
        const int c = e / NV, n = e - c * NV;
        S[e] = (S0 && n < nv) ? S0[(static_cast<long>(bh) * dk + c) * dv + n0 + n] : 0.f;
    }
    const int nchunks = (T + C - 1) / C;
    for (int ch = 0; ch < nchunks; ++ch) {
        const int t0 = ch * C;
        const int valid = min(C, T - t0);
        __syncthreads();
        // 1. load; tokens past T are identity steps
        for (int e = tid; e < C * dk; e += kThreads) {
            const int t = e / dk, c = e - t * dk;
            float qv = 0.f, kv = 0.f, a_ = 0.f, b_ = 0.f, gv = 0.f;
            if (t < valid) {
                const long o = ((static_cast<long>(b) * T + t0 + t) * H + h) * dk + c;
                qv = to_f32(q[o]);
                kv = to_f32(k[o]);
                a_ = to_f32(av[o]);
                b_ = to_f32(bv[o]);
                gv = log_alpha[o];
            }
            Qt[t * LD + c] = qv;
            Kt[t * LD + c] = kv;
            At[t * LD + c] = a_;
            Bt[t * LD + c] = b_;
            G[t * LD + c] = gv;
        }
        for (int e = tid; e < C * NV; e += kThreads) {
            const int t = e / NV, n = e - t * NV;
            V[e] = (t < valid && n < nv)
                       ? to_f32(v[((static_cast<long>(b) * T + t0 + t) * H + h) * dv + n0 + n])
                       : 0.f;
        }
        __syncthreads();
        // 2. in-chunk prefix sums
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
        // 3. the four secondary-chunk products, every term with its own gate factor
        for (int e = tid; e < C * C; e += kThreads) {
            const int i = e / C, j = e - i * C;
            float ba = 0.f, bk = 0.f, qa = 0.f, qk = 0.f;
            if (j <= i) {
                const float *qi = Qt + i * LD, *bi = Bt + i * LD, *aj = At + j * LD, *kj = Kt + j * LD;
                const float *gi = G + i * LD, *gj = G + j * LD, *gm = G + (i > 0 ? i - 1 : 0) * LD;
                for (int c = 0; c < dk; ++c) {
                    const float f = expf(gi[c] - gj[c]);
                    qa = fmaf(qi[c] * f, aj[c], qa);
                    qk = fmaf(qi[c] * f, kj[c], qk);
                    if (j < i) {   // i >= 1: g^-_i = g_{i-1}
                        const float fm = expf(gm[c] - gj[c]);
                        ba = fmaf(bi[c] * fm, aj[c], ba);
                        bk = fmaf(bi[c] * fm, kj[c], bk);
                    }
                }
            }
            Mba[i * LC + j] = ba;
            Mbk[i * LC + j] = bk;
            Mqa[i * LC + j] = qa;
            Mqk[i * LC + j] = qk;
        }
        __syncthreads();
        // 4. Tm = (I - M_ba)^{-1}, one column per thread, forward substitution
        for (int j = tid; j < C; j += kThreads) {
            for (int i = 0; i < j; ++i) Tm[i * LC + j] = 0.f;
            Tm[j * LC + j] = 1.f;
            for (int i = j + 1; i < C; ++i) {
                float s = 0.f;
                for (int m = j; m < i; ++m) s = fmaf(Mba[i * LC + m], Tm[m * LC + j], s);
                Tm[i * LC + j] = s;
            }
        }
        // 5. Qs = q e^{g}, Bs = b e^{g^-}, Ad = a e^{g_C - g}, Kd = k e^{g_C - g}
        for (int e = tid; e < C * dk; e += kThreads) {
            const int t = e / dk, c = e - t * dk;
            const float gv = G[t * LD + c], gp = t > 0 ? G[(t - 1) * LD + c] : 0.f;
            const float down = expf(gsum[c] - gv);
            Qt[t * LD + c] *= expf(gv);
            Bt[t * LD + c] *= expf(gp);
            At[t * LD + c] *= down;
            Kt[t * LD + c] *= down;
        }
        __syncthreads();
        // 6. R = Bs S + M_bk V
        for (int e = tid; e < C * NV; e += kThreads) {
            const int i = e / NV, n = e - i * NV;
            float r = 0.f;
            for (int c = 0; c < dk; ++c) r = fmaf(Bt[i * LD + c], S[c * NV + n], r);
            for (int j = 0; j < i; ++j) r = fmaf(Mbk[i * LC + j], V[j * NV + n], r);
            R[e] = r;
        }
        __syncthreads();
        // 7. U = Tm R
        for (int e = tid; e < C * NV; e += kThreads) {
            const int i = e / NV, n = e - i * NV;
            float u = 0.f;
            for (int j = 0; j <= i; ++j) u = fmaf(Tm[i * LC + j], R[j * NV + n], u);
            U[e] = u;
        }
        __syncthreads();
        // 8. O = Qs S + M_qa U + M_qk V
        for (int e = tid; e < C * NV; e += kThreads) {
            const int i = e / NV, n = e - i * NV;
            if (i < valid && n < nv) {
                float o = 0.f;
                for (int c = 0; c < dk; ++c) o = fmaf(Qt[i * LD + c], S[c * NV + n], o);
                for (int j = 0; j <= i; ++j) {
                    o = fmaf(Mqa[i * LC + j], U[j * NV + n], o);
                    o = fmaf(Mqk[i * LC + j], V[j * NV + n], o);
                }
                out[((static_cast<long>(b) * T + t0 + i) * H + h) * dv + n0 + n] = from_f32<Tin>(o);
            }
        }
        __syncthreads();
        // 9. S = Diag(e^{g_C}) S + Ad^T U + Kd^T V
        for (int e = tid; e < dk * NV; e += kThreads) {
            const int c = e / NV, n = e - c * NV;
            float s = S[e] * e_c[c];
            for (int t = 0; t < C; ++t) {
                s = fmaf(At[t * LD + c], U[t * NV + n], s);
                s = fmaf(Kt[t * LD + c], V[t * NV + n], s);
            }
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
cudaError_t launch_typed(const void *q, const void *k, const void *v, const void *a, const void *b,
                         const float *la, const float *S0, void *out, float *S_T, int B, int T, int H,
                         int dk, int dv, int chunk, cudaStream_t s) {
    const int NV = dv < kMaxNV ? dv : kMaxNV;
    const Smem L(chunk, dk, NV);
    const size_t bytes = L.floats() * sizeof(float);
    auto kern = chunk_dplr_kernel<Tin>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(bytes));
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(B) * static_cast<unsigned>(H), static_cast<unsigned>((dv + NV - 1) / NV));
    kern<<<grid, kThreads, bytes, s>>>(static_cast<const Tin *>(q), static_cast<const Tin *>(k),
                                       static_cast<const Tin *>(v), static_cast<const Tin *>(a),
                                       static_cast<const Tin *>(b), la, S0, static_cast<Tin *>(out), S_T, T,
                                       H, dk, dv, chunk, NV);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_dplr_smem_bytes(int chunk, int dk, int dv) {
    return Smem(chunk, dk, dv < kMaxNV ? dv : kMaxNV).floats() * sizeof(float);
}

cudaError_t launch_chunk_dplr(const void *q, const void *k, const void *v, const void *a, const void *b,
                              const float *la, const float *S0, void *out, float *S_T, int B, int T, int H,
                              int dk, int dv, int chunk, int dtype, cudaStream_t s) {
    return dtype == KDA_BF16
               ? launch_typed<__nv_bfloat16>(q, k, v, a, b, la, S0, out, S_T, B, T, H, dk, dv, chunk, s)
               : launch_typed<float>(q, k, v, a, b, la, S0, out, S_T, B, T, H, dk, dv, chunk, s);
}

}  // namespace kda
