// chunk_bwd.cuh -- backward pass of the chunked KDA prefill, fp32 on CUDA cores.
//
// The pages print no backward pass (Kimi Linear summary,
// es.news.hada.io/topic?id=31936, section "Algoritmo paralelo por chunks",
// builds the chunked form for training throughput); this is the derivative of
// the chunked forward (the same WY/UT form as the prefill engines), whose
// equations tests/test_chunked_form.py checks against the fp64 reverse
// recurrence of oracle/grad.py. Chunks are visited last to first; dS is the
// gradient of the state leaving the chunk and S the state entering it:
//   chain:  dU = P^T dO + Kb dS,   dS <- Qs^T dO + Diag(gamma) dS - W^T dU
//   local:  dQs = dO S^T, dP = lower(dO U^T), dKb = U dS^T, dW = -dU S^T,
//           dT = dW Ks^T + dU V^T, dKs = T^T dW, dV = T^T dU,
//           dX = dT Diag(beta), dA = -strict_lower(X^T dX X^T),
//           dbeta = colsum(dT o X) + rowsum(dA o At), dAt = Diag(beta) dA,
//           dKt = dAt Kh, dKh = dAt^T Kt + dP^T Qt, dQt = dP Kh,
//           dk, dq and dg from the factors; dlog_alpha = in-chunk suffix sum of dg.
// Value columns are independent in the chain, so a CTA owns (b, h, a slice of
// NV value columns). The key-side gradients (dq, dk, dbeta, dlog_alpha) are
// linear in a slice's partial terms and are summed over slices with atomics.
// Two kernels: a forward pass that stores every chunk's entry state, then the
// reverse pass. Chunk length 16 (the chunk length is free in exact
// arithmetic; 16 keeps a CTA's tiles within shared memory at d = 128).
// The bodies use only plain CUDA-core code; the kernels, their launch and the
// fp32 -> dtype casts are in chunk_bwd.cu.
#pragma once

namespace kbwd {

constexpr int kThreads = 256;
constexpr int kC = 16;
constexpr int kNV = 32;

// Row strides are one float longer than the rows (LD = dk + 1, LC = C + 1, NP = NV + 1), so
// that a warp reading a column (one row per lane) hits 32 different banks.
struct Layout {
    int dk, NV, NP, LD, LC;
    __host__ __device__ Layout(int dk_, int NV_) : dk(dk_), NV(NV_), NP(NV_ + 1), LD(dk_ + 1), LC(kC + 1) {}
    // 12 [C][LD] tiles, 7 [C][LC], 5 [C][NP], 3 [dk][NP], vectors
    __host__ __device__ size_t floats() const {
        return 12ull * kC * LD + 7ull * kC * LC + 5ull * kC * NP + 3ull * dk * NP + 3ull * dk + 3ull * kC;
    }
};

struct Tiles {
    // Qt, Kt: q and k; Qs = q e^{g}, Ks = k e^{g}, Kh = Kb = k e^{g_C - g}; G: prefix sums g
    float *Qt, *Kt, *Kh, *G, *W, *dQs, *dKb, *dW, *dKs, *dQt, *Qs, *Ks;   // [C][LD]
    float *At, *P, *X, *Tm, *dT, *dA, *dP;                      // [C][LC]
    float *V, *Up, *U, *dO, *dU;                                 // [C][NP]
    float *S, *dS, *dSn;                                         // [dk][NP]
    float *gam, *dgam, *gsum;                                    // [dk]
    float *bt, *dbt, *pad;                                       // [C]
    __device__ Tiles(float *sm, const Layout &L) {
        const int CD = kC * L.LD, CC = kC * L.LC, CN = kC * L.NP, DN = L.dk * L.NP;
        float *p = sm;
        Qt = p; p += CD; Kt = p; p += CD; Kh = p; p += CD; G = p; p += CD; W = p; p += CD;
        dQs = p; p += CD; dKb = p; p += CD; dW = p; p += CD; dKs = p; p += CD; dQt = p; p += CD;
        Qs = p; p += CD; Ks = p; p += CD;
        At = p; p += CC; P = p; p += CC; X = p; p += CC; Tm = p; p += CC; dT = p; p += CC;
        dA = p; p += CC; dP = p; p += CC;
        V = p; p += CN; Up = p; p += CN; U = p; p += CN; dO = p; p += CN; dU = p; p += CN;
        S = p; p += DN; dS = p; p += DN; dSn = p; p += DN;
        gam = p; p += L.dk;
        dgam = p; p += L.dk; gsum = p; p += L.dk;
        bt = p; p += kC; dbt = p; p += kC; pad = p;
    }
};

// The state-independent terms of one chunk: g, Qs, Ks, Kb, At, P,
// X = (I + A)^{-1}, T, W = T Ks, U' = T V. Loads q, k, log alpha, v (slice), beta.
template <typename Tin>
__device__ void chunk_terms(Tiles &s, const Layout &L, const Tin *q, const Tin *k, const Tin *v,
                            const float *log_alpha, const float *beta, int b, int h, int T, int H,
                            int dv, int t0, int valid, int n0, int nv, bool need_p) {
    const int tid = threadIdx.x, dk = L.dk, LD = L.LD, LC = L.LC, NV = L.NV, NP = L.NP;
    for (int e = tid; e < kC * dk; e += kThreads) {
        const int t = e / dk, c = e - t * dk;
        float qv = 0.f, kv = 0.f, gv = 0.f;
        if (t < valid) {
            const long o = ((static_cast<long>(b) * T + t0 + t) * H + h) * dk + c;
            qv = to_f32(q[o]);
            kv = to_f32(k[o]);
            gv = log_alpha[o];
        }
        s.Qt[t * LD + c] = qv;
        s.Kt[t * LD + c] = kv;
        s.G[t * LD + c] = gv;
    }
    for (int e = tid; e < kC * NV; e += kThreads) {
        const int t = e / NV, n = e - t * NV;
        float vv = 0.f;
        if (t < valid && n < nv) vv = to_f32(v[((static_cast<long>(b) * T + t0 + t) * H + h) * dv + n0 + n]);
        s.V[t * NP + n] = vv;
    }
    for (int t = tid; t < kC; t += kThreads)
        s.bt[t] = t < valid ? beta[(static_cast<long>(b) * T + t0 + t) * H + h] : 0.f;
    __syncthreads();
    for (int c = tid; c < dk; c += kThreads) {   // prefix sums
        float acc = 0.f;
        for (int t = 0; t < kC; ++t) {
            acc += s.G[t * LD + c];
            s.G[t * LD + c] = acc;
        }
        s.gsum[c] = acc;
        s.gam[c] = expf(acc);
    }
    __syncthreads();
    for (int e = tid; e < kC * dk; e += kThreads) {   // Qs = q e^{g}, Ks = k e^{g}, Kb = k e^{g_C - g}
        const int t = e / dk, c = e - t * dk;
        const float gv = s.G[t * LD + c];
        const float up = expf(gv), down = expf(s.gsum[c] - gv);
        const float kv = s.Kt[t * LD + c];
        s.Qs[t * LD + c] = s.Qt[t * LD + c] * up;
        s.Ks[t * LD + c] = kv * up;
        s.Kh[t * LD + c] = kv * down;
    }
    for (int e = tid; e < 2 * kC * kC; e += kThreads) {   // At (strict lower), P (lower)
        const int which = e / (kC * kC), r = e - which * kC * kC;
        const int i = r / kC, j = r - i * kC;
        float acc = 0.f;
        if (which == 0 ? j < i : (need_p && j <= i)) {
            const float *x = (which == 0 ? s.Kt : s.Qt) + i * LD;
            const float *y = s.Kt + j * LD;
            const float *gi = s.G + i * LD, *gj = s.G + j * LD;
            for (int c = 0; c < dk; ++c) acc = fmaf(x[c], y[c] * expf(gi[c] - gj[c]), acc);
        }
        (which == 0 ? s.At : s.P)[i * LC + j] = acc;
    }
    __syncthreads();
    if (tid < kC) {   // X = (I + A)^{-1}, A = Diag(beta) At: column j by forward substitution
        const int j = tid;
        for (int i = 0; i < kC; ++i) {
            float x = i == j ? 1.f : 0.f;
            if (i > j) {
                float acc = 0.f;
                for (int m = j; m < i; ++m) acc = fmaf(s.At[i * LC + m], s.X[m * LC + j], acc);
                x = -s.bt[i] * acc;
            }
            s.X[i * LC + j] = x;
            s.Tm[i * LC + j] = x * s.bt[j];
        }
    }
    __syncthreads();
    for (int e = tid; e < kC * dk + kC * NV; e += kThreads) {   // W = T Ks, U' = T V
        if (e < kC * dk) {
            const int i = e / dk, c = e - i * dk;
            float acc = 0.f;
            for (int j = 0; j <= i; ++j) acc = fmaf(s.Tm[i * LC + j], s.Ks[j * LD + c], acc);
            s.W[i * LD + c] = acc;
        } else {
            const int r = e - kC * dk, i = r / NV, n = r - i * NV;
            float acc = 0.f;
            for (int j = 0; j <= i; ++j) acc = fmaf(s.Tm[i * LC + j], s.V[j * NP + n], acc);
            s.Up[i * NP + n] = acc;
        }
    }
    __syncthreads();
}

// Forward chain storing the entry state of every chunk: states[bh][chunk][dk][dv].
template <typename Tin>
__device__ void states_body(float *sm, const Tin *q, const Tin *k, const Tin *v, const float *log_alpha,
                            const float *beta, const float *S0, float *states, int T, int H, int dk,
                            int dv) {
    const Layout L(dk, kNV);
    Tiles s(sm, L);
    const int tid = threadIdx.x, LD = L.LD, NV = L.NV, NP = L.NP;
    const int bh = blockIdx.x, b = bh / H, h = bh - b * H;
    const int n0 = blockIdx.y * NV, nv = min(NV, dv - n0);
    const int nchunks = (T + kC - 1) / kC;
    for (int e = tid; e < dk * NV; e += kThreads) {
        const int c = e / NV, n = e - c * NV;
        s.S[c * NP + n] = (S0 && n < nv) ? S0[(static_cast<long>(bh) * dk + c) * dv + n0 + n] : 0.f;
    }
    for (int ch = 0; ch < nchunks; ++ch) {
        const int t0 = ch * kC, valid = min(kC, T - t0);
        __syncthreads();
        float *dst = states + (static_cast<long>(bh) * nchunks + ch) * dk * dv;
        for (int e = tid; e < dk * NV; e += kThreads) {
            const int c = e / NV, n = e - c * NV;
            if (n < nv) dst[static_cast<long>(c) * dv + n0 + n] = s.S[c * NP + n];
        }
        chunk_terms(s, L, q, k, v, log_alpha, beta, b, h, T, H, dv, t0, valid, n0, nv, false);
        for (int e = tid; e < kC * NV; e += kThreads) {   // U = U' - W S
            const int i = e / NV, n = e - i * NV;
            float acc = s.Up[i * NP + n];
            for (int c = 0; c < dk; ++c) acc = fmaf(-s.W[i * LD + c], s.S[c * NP + n], acc);
            s.U[i * NP + n] = acc;
        }
        __syncthreads();
        for (int e = tid; e < dk * NV; e += kThreads) {   // S <- Diag(gamma) S + Kb^T U
            const int c = e / NV, n = e - c * NV;
            float acc = s.gam[c] * s.S[c * NP + n];
            for (int t = 0; t < kC; ++t) acc = fmaf(s.Kh[t * LD + c], s.U[t * NP + n], acc);
            s.S[c * NP + n] = acc;
        }
    }
}

// Reverse pass. dq_acc, dk_acc [B,T,H,dk], dbeta [B,T,H] and dlog_alpha [B,T,H,dk]
// are fp32 and must be zero on entry (atomically accumulated over value slices);
// dv [B,T,H,dv] and dS0 [B,H,dk,dv] are written.
template <typename Tin>
__device__ void bwd_body(float *sm, const Tin *q, const Tin *k, const Tin *v, const float *log_alpha,
                         const float *beta, const Tin *dout, const float *dS_T, const float *states,
                         float *dq_acc, float *dk_acc, Tin *dv_out, float *dlog_alpha, float *dbeta,
                         float *dS0, int T, int H, int dk, int dv) {
    const Layout L(dk, kNV);
    Tiles s(sm, L);
    const int tid = threadIdx.x, LD = L.LD, LC = L.LC, NV = L.NV, NP = L.NP;
    const int bh = blockIdx.x, b = bh / H, h = bh - b * H;
    const int n0 = blockIdx.y * NV, nv = min(NV, dv - n0);
    const int nchunks = (T + kC - 1) / kC;
    for (int e = tid; e < dk * NV; e += kThreads) {
        const int c = e / NV, n = e - c * NV;
        s.dS[c * NP + n] = (dS_T && n < nv) ? dS_T[(static_cast<long>(bh) * dk + c) * dv + n0 + n] : 0.f;
    }
    for (int ch = nchunks - 1; ch >= 0; --ch) {
        const int t0 = ch * kC, valid = min(kC, T - t0);
        __syncthreads();
        const float *src = states + (static_cast<long>(bh) * nchunks + ch) * dk * dv;
        for (int e = tid; e < dk * NV; e += kThreads) {
            const int c = e / NV, n = e - c * NV;
            s.S[c * NP + n] = n < nv ? src[static_cast<long>(c) * dv + n0 + n] : 0.f;
        }
        for (int e = tid; e < kC * NV; e += kThreads) {
            const int t = e / NV, n = e - t * NV;
            s.dO[t * NP + n] = (t < valid && n < nv)
                          ? to_f32(dout[((static_cast<long>(b) * T + t0 + t) * H + h) * dv + n0 + n])
                          : 0.f;
        }
        chunk_terms(s, L, q, k, v, log_alpha, beta, b, h, T, H, dv, t0, valid, n0, nv, true);
        // U = U' - W S
        for (int e = tid; e < kC * NV; e += kThreads) {
            const int i = e / NV, n = e - i * NV;
            float acc = s.Up[i * NP + n];
            for (int c = 0; c < dk; ++c) acc = fmaf(-s.W[i * LD + c], s.S[c * NP + n], acc);
            s.U[i * NP + n] = acc;
        }
        __syncthreads();
        // dU = P^T dO + Kb dS
        for (int e = tid; e < kC * NV; e += kThreads) {
            const int j = e / NV, n = e - j * NV;
            float acc = 0.f;
            for (int i = j; i < kC; ++i) acc = fmaf(s.P[i * LC + j], s.dO[i * NP + n], acc);
            for (int c = 0; c < dk; ++c) acc = fmaf(s.Kh[j * LD + c], s.dS[c * NP + n], acc);
            s.dU[j * NP + n] = acc;
        }
        __syncthreads();
        // the new state gradient, and the slice's partial key-side terms
        for (int e = tid; e < dk * NV; e += kThreads) {   // dSn = Qs^T dO + Diag(gamma) dS - W^T dU
            const int c = e / NV, n = e - c * NV;
            float acc = s.gam[c] * s.dS[c * NP + n];
            for (int i = 0; i < kC; ++i) {
                acc = fmaf(s.Qs[i * LD + c], s.dO[i * NP + n], acc);
                acc = fmaf(-s.W[i * LD + c], s.dU[i * NP + n], acc);
            }
            s.dSn[c * NP + n] = acc;
        }
        for (int c = tid; c < dk; c += kThreads) {   // gamma's gradient (through the state decay)
            float acc = 0.f;
            for (int n = 0; n < NV; ++n) acc = fmaf(s.dS[c * NP + n], s.S[c * NP + n], acc);
            s.dgam[c] = acc * s.gam[c];
        }
        for (int e = tid; e < 3 * kC * dk; e += kThreads) {   // dQs = dO S^T, dKb = U dS^T, dW = -dU S^T
            const int which = e / (kC * dk), r = e - which * kC * dk;
            const int i = r / dk, c = r - i * dk;
            const float *a = which == 0 ? s.dO : (which == 1 ? s.U : s.dU);
            const float *m = which == 1 ? s.dS : s.S;
            float acc = 0.f;
            for (int n = 0; n < NV; ++n) acc = fmaf(a[i * NP + n], m[c * NP + n], acc);
            (which == 0 ? s.dQs : (which == 1 ? s.dKb : s.dW))[i * LD + c] = which == 2 ? -acc : acc;
        }
        for (int e = tid; e < kC * kC + kC * NV; e += kThreads) {   // dP = lower(dO U^T), dV = T^T dU
            if (e < kC * kC) {
                const int i = e / kC, j = e - i * kC;
                float acc = 0.f;
                if (j <= i)
                    for (int n = 0; n < NV; ++n) acc = fmaf(s.dO[i * NP + n], s.U[j * NP + n], acc);
                s.dP[i * LC + j] = acc;
            } else {
                const int r = e - kC * kC, j = r / NV, n = r - j * NV;
                float acc = 0.f;
                for (int i = j; i < kC; ++i) acc = fmaf(s.Tm[i * LC + j], s.dU[i * NP + n], acc);
                if (j < valid && n < nv)
                    dv_out[((static_cast<long>(b) * T + t0 + j) * H + h) * dv + n0 + n] = from_f32<Tin>(acc);
            }
        }
        __syncthreads();
        {   // the state gradient moves one chunk back
            float *t = s.dS;
            s.dS = s.dSn;
            s.dSn = t;
        }
        // dT = dW Ks^T + dU V^T (lower incl. diagonal), dKs = T^T dW
        for (int e = tid; e < kC * kC + kC * dk; e += kThreads) {
            if (e < kC * kC) {
                const int i = e / kC, j = e - i * kC;
                float acc = 0.f;
                if (j <= i) {
                    for (int c = 0; c < dk; ++c) acc = fmaf(s.dW[i * LD + c], s.Ks[j * LD + c], acc);
                    for (int n = 0; n < NV; ++n) acc = fmaf(s.dU[i * NP + n], s.V[j * NP + n], acc);
                }
                s.dT[i * LC + j] = acc;
            } else {
                const int r = e - kC * kC, j = r / dk, c = r - j * dk;
                float acc = 0.f;
                for (int i = j; i < kC; ++i) acc = fmaf(s.Tm[i * LC + j], s.dW[i * LD + c], acc);
                s.dKs[j * LD + c] = acc;
            }
        }
        __syncthreads();
        // Z = X^T dX with dX = dT Diag(beta) (kept in dA), and dbeta's T part
        for (int e = tid; e < kC * kC + kC; e += kThreads) {
            if (e < kC * kC) {
                const int i = e / kC, bcol = e - i * kC;
                float acc = 0.f;
                for (int a = i; a < kC; ++a) acc = fmaf(s.X[a * LC + i], s.dT[a * LC + bcol] * s.bt[bcol], acc);
                s.dA[i * LC + bcol] = acc;
            } else {
                const int j = e - kC * kC;
                float acc = 0.f;
                for (int i = j; i < kC; ++i) acc = fmaf(s.dT[i * LC + j], s.X[i * LC + j], acc);
                s.dbt[j] = acc;
            }
        }
        __syncthreads();
        // dA = -strict_lower(Z X^T) (into dT, whose values are no longer needed)
        for (int e = tid; e < kC * kC; e += kThreads) {
            const int i = e / kC, j = e - i * kC;
            float acc = 0.f;
            if (j < i)
                for (int bcol = 0; bcol <= j; ++bcol) acc = fmaf(s.dA[i * LC + bcol], s.X[j * LC + bcol], acc);
            s.dT[i * LC + j] = -acc;
        }
        __syncthreads();
        // dbeta's A part; dAt = Diag(beta) dA (in dT)
        for (int i = tid; i < kC; i += kThreads) {
            float acc = 0.f;
            for (int j = 0; j < i; ++j) acc = fmaf(s.dT[i * LC + j], s.At[i * LC + j], acc);
            s.dbt[i] += acc;
        }
        __syncthreads();
        for (int e = tid; e < kC * kC; e += kThreads) {
            const int i = e / kC;
            s.dT[(i)*LC + (e - i * kC)] *= s.bt[i];
        }
        __syncthreads();
        // The intra-chunk products, term by term (E_ij = e^{g_i - g_j} per channel):
        //   R_i  = sum_{j<i}  dAt_ij k_j E_ij             (row side of A,   into dW)
        //   Cc_j = sum_{i>j}  dAt_ij k_i E_ij
        //        + sum_{i>=j} dP_ij  q_i E_ij             (column side,     into W)
        //   Rq_i = sum_{j<=i} dP_ij  k_j E_ij             (row side of P,   into dQt)
        for (int e = tid; e < 3 * kC * dk; e += kThreads) {
            const int which = e / (kC * dk), r = e - which * kC * dk;
            const int i = r / dk, c = r - i * dk;
            const float gi = s.G[i * LD + c];
            float acc = 0.f;
            if (which == 0) {
                for (int j = 0; j < i; ++j)
                    acc = fmaf(s.dT[i * LC + j], s.Kt[j * LD + c] * expf(gi - s.G[j * LD + c]), acc);
            } else if (which == 1) {
                for (int a = i + 1; a < kC; ++a)
                    acc = fmaf(s.dT[a * LC + i], s.Kt[a * LD + c] * expf(s.G[a * LD + c] - gi), acc);
                for (int a = i; a < kC; ++a)
                    acc = fmaf(s.dP[a * LC + i], s.Qt[a * LD + c] * expf(s.G[a * LD + c] - gi), acc);
            } else {
                for (int j = 0; j <= i; ++j)
                    acc = fmaf(s.dP[i * LC + j], s.Kt[j * LD + c] * expf(gi - s.G[j * LD + c]), acc);
            }
            (which == 0 ? s.dW : (which == 1 ? s.W : s.dQt))[i * LD + c] = acc;
        }
        __syncthreads();
        // dk, dq; dg per token and channel (into dKs, after its use)
        for (int e = tid; e < kC * dk; e += kThreads) {
            const int t = e / dk, c = e - t * dk;
            const float gv = s.G[t * LD + c];
            const float up = expf(gv), down = expf(s.gsum[c] - gv);
            const float kv = s.Kt[t * LD + c], qv = s.Qt[t * LD + c];
            const float rk = s.dW[t * LD + c], cc = s.W[t * LD + c], rq = s.dQt[t * LD + c];
            const float dks = s.dKs[t * LD + c], dkb = s.dKb[t * LD + c], dqs = s.dQs[t * LD + c];
            const float dk_v = rk + cc + dks * up + dkb * down;
            const float dq_v = rq + dqs * up;
            const float dg = kv * (rk - cc) + qv * rq + dks * s.Ks[t * LD + c] + dqs * s.Qs[t * LD + c] -
                             dkb * s.Kh[t * LD + c];
            s.dKs[t * LD + c] = dg;
            if (t < valid) {
                const long o = ((static_cast<long>(b) * T + t0 + t) * H + h) * dk + c;
                atomicAdd(dk_acc + o, dk_v);
                atomicAdd(dq_acc + o, dq_v);
            }
        }
        __syncthreads();
        for (int c = tid; c < dk; c += kThreads) {   // g_C's own terms, then the in-chunk suffix sums
            float gc = s.dgam[c];
            for (int t = 0; t < kC; ++t) gc = fmaf(s.dKb[t * LD + c], s.Kh[t * LD + c], gc);
            float acc = gc;
            for (int t = kC - 1; t >= 0; --t) {
                acc += s.dKs[t * LD + c];
                if (t < valid)
                    atomicAdd(dlog_alpha + ((static_cast<long>(b) * T + t0 + t) * H + h) * dk + c, acc);
            }
        }
        for (int t = tid; t < valid; t += kThreads)
            atomicAdd(dbeta + (static_cast<long>(b) * T + t0 + t) * H + h, s.dbt[t]);
    }
    __syncthreads();
    if (dS0)
        for (int e = tid; e < dk * NV; e += kThreads) {
            const int c = e / NV, n = e - c * NV;
            if (n < nv) dS0[(static_cast<long>(bh) * dk + c) * dv + n0 + n] = s.dS[c * NP + n];
        }
}

}  // namespace kbwd
